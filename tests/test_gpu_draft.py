"""Draft step on the GPU against the oracle (parity), through the C ABI.

Acceptance rule (the same as the verification's): drafted tokens bit-exact
except where the oracle's fp64 margin of the draw is below 1e-6 (counted,
share below 1e-4); ln q(token) within 1e-5 absolute (q within 1e-5
relative); the entropy within 1e-5 absolute plus 1e-5 relative (the fp32
first-moment sums carry about 2^-24 of the logit range)."""
import math

import numpy as np
import pytest
import torch

from oracle.draft import draft_step
from speculative_decoding_verification_89_b200 import workloads as W
from tests.gpu_run import to_np
from tests.parity import Tally

pytestmark = pytest.mark.gpu

MARGIN = 1e-6
LOGQ_ATOL = 1e-5
H_TOL = 1e-5


def _padded2(t):
    """[B, V] copy whose rows start on 16-byte boundaries."""
    B, V = t.shape
    mult = 16 // t.element_size()
    ld = (V + mult - 1) // mult * mult
    if ld == V:
        return t
    big = torch.zeros((B, ld), dtype=t.dtype, device=t.device)
    big[:, :V] = t
    return big[:, :V]


def run_gpu(prob, want_extra=True):
    from speculative_decoding_verification_89_b200 import capi
    dev = torch.device("cuda")
    lg = _padded2(prob.logits.to(dev))
    B, V = lg.shape
    ws = capi.draft_workspace(B, V, lg.dtype, device=dev)
    tok = torch.full((B,), -7, dtype=torch.int32, device=dev)
    logq = torch.full((B,), 7.0, dtype=torch.float64, device=dev) if want_extra else None
    ent = torch.full((B,), 7.0, dtype=torch.float64, device=dev) if want_extra else None
    st = torch.zeros(1, dtype=torch.int32, device=dev)
    capi.spec_draft_sample(lg, prob.temperature.to(dev), prob.seed, prob.seq_id.to(dev),
                           prob.rnd, prob.pos.to(dev), tok, st, ws, logq=logq, entropy=ent)
    torch.cuda.synchronize()
    return (tok.cpu().numpy(), None if logq is None else logq.cpu().numpy(),
            None if ent is None else ent.cpu().numpy(), int(st.item()))


def compare(prob, tag, counts, rows=None):
    tok, logq, ent, st = run_gpu(prob)
    assert st == 0, f"{tag}: device status {st}"
    lg = to_np(prob.logits)
    B = lg.shape[0]
    rows = range(B) if rows is None else rows
    sub = [int(b) for b in rows]
    ref = draft_step(lg[sub], prob.temperature.numpy()[sub], prob.seed,
                     prob.seq_id.numpy()[sub], prob.rnd, prob.pos.numpy()[sub])
    for b, r in zip(sub, ref):
        counts[0] += 1
        if int(tok[b]) != r.token:
            assert r.margin < MARGIN, (f"{tag}/row{b}: token {int(tok[b])} vs oracle {r.token} "
                                       f"(margin {r.margin:.3g})")
            counts[1] += 1
            continue
        assert abs(logq[b] - r.logq) <= LOGQ_ATOL, f"{tag}/row{b}: ln q {logq[b]} vs {r.logq}"
        assert abs(ent[b] - r.entropy) <= H_TOL * (1.0 + abs(r.entropy)), \
            f"{tag}/row{b}: entropy {ent[b]} vs {r.entropy}"


def _check_share(counts):
    """The acceptance rule's share: excused near-margin draws (oracle margin
    below 1e-6) must be fewer than 1e-4 of all draws compared -- none at all
    for a test with fewer than 10 000 draws."""
    t = Tally()
    t.decisions, t.excused = counts
    t.check_share()
    print(f"draws compared: {counts[0]}, excused: {counts[1]}")


CASES = [
    # B, V, dtype, temperature, extra generator arguments
    (4, 1000, torch.float32, 1.0, {}),
    (3, 1, torch.float32, 1.0, {}),                        # single-token vocabulary
    (5, 7, torch.bfloat16, 0.9, {}),                       # shorter than one vector
    (6, 4097, torch.bfloat16, 0.8, {}),                    # ragged tiles
    (4, 8191, torch.float32, 1.3, {}),                     # odd fp32 tail
    (8, 32000, torch.bfloat16, 0.7, {"mask_frac": 0.3}),   # masked entries
    (4, 50000, torch.float32, 1e-3, {}),                   # near-greedy
    (4, 50000, torch.bfloat16, 50.0, {}),                  # flat laws
    (6, 151936, torch.float32, 1.0, {"zipf_s": 1.1}),      # Qwen-size fp32 rows (8-CTA slices)
    (2, 262144, torch.float32, 0.9, {}),                   # too large to stage: two launches
]


@pytest.mark.parametrize("case", range(len(CASES)))
def test_draft_parity_shapes(case):
    B, V, dt, T, kw = CASES[case]
    counts = [0, 0]
    for rnd in range(3):
        prob = W.draft_problem(B, V, dt, seed=case, rnd=rnd, temperature=T, **kw)
        compare(prob, f"case{case}/r{rnd}", counts)
    _check_share(counts)


def test_draft_mixed_greedy():
    g = torch.Generator().manual_seed(3)
    T = torch.rand(16, generator=g) * 1.2 + 0.05
    T[::3] = 0.0
    prob = W.draft_problem(16, 12345, torch.bfloat16, seed=9, temperature=T)
    counts = [0, 0]
    compare(prob, "mixed", counts)
    tok, logq, ent, _ = run_gpu(prob)
    lg = to_np(prob.logits)
    for b in range(0, 16, 3):
        assert int(tok[b]) == int(np.argmax(lg[b])) and logq[b] == 0.0 and ent[b] == 0.0


def test_draft_full_size_batch():
    """The benchmark's shape: B=64, V=128256 bf16, every row against the oracle,
    over four rounds."""
    counts = [0, 0]
    for rnd in range(4):
        compare(W.draft_batch(rnd=rnd), f"full/r{rnd}", counts)
    _check_share(counts)


def test_draft_without_optional_outputs():
    prob = W.draft_problem(4, 3000, torch.bfloat16, seed=2)
    tok, _, _, st = run_gpu(prob, want_extra=False)
    assert st == 0
    ref = draft_step(to_np(prob.logits), prob.temperature.numpy(), prob.seed,
                     prob.seq_id.numpy(), prob.rnd, prob.pos.numpy())
    assert [int(x) for x in tok] == [r.token for r in ref]


def test_draft_invalid_rows_flag_the_status():
    prob = W.draft_problem(4, 2000, torch.float32, seed=4)
    prob.temperature[1] = -1.0                  # invalid temperature
    prob.logits[2] = float("-inf")              # no finite maximum
    tok, logq, ent, st = run_gpu(prob)
    assert st == -6
    assert int(tok[1]) == -1 and int(tok[2]) == -1
    assert math.isnan(logq[1]) and math.isnan(ent[2])
    ref = draft_step(to_np(prob.logits)[[0, 3]], prob.temperature.numpy()[[0, 3]], prob.seed,
                     prob.seq_id.numpy()[[0, 3]], prob.rnd, prob.pos.numpy()[[0, 3]])
    assert [int(tok[0]), int(tok[3])] == [r.token for r in ref]


def test_draft_stream_follows_counter_fields():
    """Two rounds, two slots: the drafted tokens change with the Philox
    counter exactly as the oracle's do (seq_id, round and pos wiring)."""
    counts = [0, 0]
    base = W.draft_problem(32, 64, torch.bfloat16, seed=8, std=0.5)
    for rnd in (0, 1):
        for shift in (0, 5):
            prob = W.DraftProblem(base.logits, base.temperature, base.seq_id + 100 * shift,
                                  base.pos + shift, base.seed, rnd)
            compare(prob, f"stream/r{rnd}/s{shift}", counts)
    assert counts[1] == 0
