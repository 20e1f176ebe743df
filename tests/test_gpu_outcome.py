"""Outcome law of a chain check (drafts fixed) on the GPU against the oracle,
through the C ABI.

Acceptance rule: the length law P(a = k), the accept probabilities beta and
the residual masses within 1e-5 relative (plus 1e-12 absolute for values near
0). The top outcomes: each joint probability P(a = k) w_v / Z_k within 1e-5
relative (the kept weights w_v = max(0, p_v - q_v) are formed in fp64 from the
two logits, so no cancellation loosens this); the list is sorted, and no
outcome the GPU left out is more likely than the least likely it kept beyond
that tolerance (only near-ties may be chosen differently)."""
import numpy as np
import pytest
import torch

from oracle.outcome import outcome_law, top_outcomes
from speculative_decoding_verification_89_b200 import workloads as W
from tests.gpu_run import padded, to_np

pytestmark = pytest.mark.gpu

RTOL = 1e-5
ATOL = 1e-12


def run_gpu(prob, n_top):
    from speculative_decoding_verification_89_b200 import capi
    dev = torch.device("cuda")
    tgt = padded(prob.tgt.to(dev))
    drf = padded(prob.drf.to(dev))
    B, Kp1, V = tgt.shape
    K = Kp1 - 1
    ws = capi.outcome_workspace(B, K, V, tgt.dtype, n_top, device=dev)
    f64 = dict(dtype=torch.float64, device=dev)
    p_len = torch.full((B, K + 1), 7.0, **f64)
    beta = torch.full((B, max(K, 1)), 7.0, **f64)
    mass = torch.full((B, K + 1), 7.0, **f64)
    tl = torch.full((B, max(n_top, 1)), -7, dtype=torch.int32, device=dev)
    tt = torch.full((B, max(n_top, 1)), -7, dtype=torch.int32, device=dev)
    tp = torch.full((B, max(n_top, 1)), 7.0, **f64)
    st = torch.zeros(1, dtype=torch.int32, device=dev)
    capi.spec_outcome_law(tgt, drf, prob.draft_tok.to(dev).contiguous(), prob.temperature.to(dev),
                          n_top, p_len, st, ws, beta=beta, mass=mass, top_len=tl, top_tok=tt,
                          top_prob=tp)
    torch.cuda.synchronize()
    return (p_len.cpu().numpy(), beta.cpu().numpy(), mass.cpu().numpy(), tl.cpu().numpy(),
            tt.cpu().numpy(), tp.cpu().numpy(), int(st.item()))


def _close(a, b):
    return abs(a - b) <= RTOL * max(abs(a), abs(b)) + ATOL


def compare(prob, n_top, tag, rows=None):
    p_len, beta, mass, tl, tt, tp, st = run_gpu(prob, n_top)
    assert st == 0, f"{tag}: device status {st}"
    tgt, drf = to_np(prob.tgt), to_np(prob.drf)
    B, Kp1, _ = tgt.shape
    K = Kp1 - 1
    for b in (range(B) if rows is None else rows):
        T = float(prob.temperature[b])
        law = outcome_law(tgt[b], drf[b], prob.draft_tok[b].numpy(), T)
        for k in range(K + 1):
            assert _close(p_len[b, k], law.p_len[k]), (tag, b, k, p_len[b, k], law.p_len[k])
            assert _close(mass[b, k], law.mass[k]), (tag, b, k, mass[b, k], law.mass[k])
        for j in range(K):
            assert _close(beta[b, j], law.beta[j]), (tag, b, j, beta[b, j], law.beta[j])
        if n_top == 0:
            continue
        joint = law.p_len[:, None] * law.resid

        def tol(k, v, p):
            return RTOL * max(p, joint[k, v]) + ATOL

        got = [(int(tl[b, i]), int(tt[b, i]), float(tp[b, i])) for i in range(n_top)
               if int(tl[b, i]) >= 0]
        ref = top_outcomes(law, n_top)
        assert len(got) == len(ref), (tag, b, len(got), len(ref))
        probs = [p for _, _, p in got]
        assert all(x >= y for x, y in zip(probs, probs[1:])), (tag, b, "not sorted")
        for k, v, p in got:
            assert abs(p - joint[k, v]) <= tol(k, v, p), (tag, b, k, v, p, joint[k, v])
        if got:
            kept = {(k, v) for k, v, _ in got}
            kl, vl, floor = got[-1]
            for k, v, p in ref:
                if (k, v) not in kept:
                    assert p <= floor + tol(kl, vl, floor) + tol(k, v, p), \
                        (tag, b, "missed", k, v, p, floor)


CASES = [
    # B, K, V, dtype, temperature
    (4, 4, 1000, torch.float32, 1.0),
    (3, 1, 7, torch.bfloat16, 0.9),
    (4, 3, 4097, torch.bfloat16, 0.8),
    (5, 2, 12345, torch.bfloat16, "mixed"),
    (2, 40, 3000, torch.bfloat16, 1.0),       # K > 32
    (3, 0, 2000, torch.float32, 1.0),         # bonus only
    (4, 5, 32000, torch.float32, 0.3),
]


@pytest.mark.parametrize("case", range(len(CASES)))
@pytest.mark.parametrize("n_top", [0, 1, 8, 32])
def test_outcome_parity(case, n_top):
    B, K, V, dt, T = CASES[case]
    if T == "mixed":
        T = torch.tensor([1.0, 0.0, 0.7, 0.0, 1.4])
    prob = W.chain_problem(B, K, V, dt, seed=40 + case, temperature=T, target_std=1.5)
    compare(prob, n_top, f"case{case}/n{n_top}")


def test_outcome_full_size():
    """The benchmark's shape (B=64, K=8, V=128256 bf16), n_top = 32, every
    sequence against the oracle."""
    compare(W.chain_batch(), 32, "full")


def test_outcome_invalid_rows():
    T = torch.tensor([1.0, -2.0, 0.8])
    prob = W.chain_problem(3, 2, 500, torch.float32, seed=7, temperature=T)
    prob.draft_tok[2, 1] = 500                 # draft id outside [0, V)
    p_len, _, _, tl, _, _, st = run_gpu(prob, 4)
    assert st == -6
    assert np.isnan(p_len[1]).all() and np.isnan(p_len[2]).all()
    assert (tl[1] == -1).all() and (tl[2] == -1).all()
    law = outcome_law(to_np(prob.tgt)[0], to_np(prob.drf)[0], prob.draft_tok[0].numpy(), 1.0)
    assert all(_close(p_len[0, k], law.p_len[k]) for k in range(3))
