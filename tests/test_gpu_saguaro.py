"""Saguaro sampling on the GPU against the oracle (parity), through the C ABI.

Speculative Speculative Decoding (gist.science summary of arXiv 2603.03251),
Technische Zusammenfassung 3.B: the draft probabilities of the tokens held in
the speculation cache are lowered, q'(v) proportional to q(v) (1 - eps) for a
cached v; on logits at temperature T that is T ln(1 - eps) added to the
cached tokens. spec_saguaro_adjust does that in place; the draft step and the
chain check then run unchanged on the lowered rows.

* the lowered rows: bit-exact against the oracle's stored form (the float32
  shift added in float32, rounded to the rows' type), untouched elsewhere;
* the draft step and the check on them: the same acceptance rule as without
  the lowering (decisions bit-exact except within the 1e-6 margin, counted,
  share below 1e-4; probabilities within 1e-5 relative)."""
import numpy as np
import pytest
import torch

from oracle.draft import draft_step, saguaro_logits
from oracle.verify import verify_chain
from speculative_decoding_verification_89_b200 import workloads as W
from tests.gpu_run import to_np
from tests.parity import MARGIN, Tally, compare_check, compare_probs

pytestmark = pytest.mark.gpu


def _padded_rows(t, extra=0):
    """Device copy of [B, n, V] rows in a buffer of row stride ld >= V (16-byte
    multiple, plus ``extra`` elements); returns (view, buffer)."""
    B, n, V = t.shape
    mult = 16 // t.element_size()
    ld = (V + extra + mult - 1) // mult * mult
    buf = torch.full((B, n, ld), 3.0, dtype=t.dtype, device="cuda")
    buf[:, :, :V] = t.to("cuda")
    return buf[:, :, :V], buf


def _oracle_rows(lg, T, cached, eps, kind):
    """The oracle's lowered rows, [B, n, V] fp64; ``cached`` [B, c] (one list
    per sequence) or [B, n, c] (one per row)."""
    x = to_np(lg)
    B, n, _ = x.shape
    c = cached.cpu().numpy()
    out = np.empty_like(x)
    for b in range(B):
        Tb = float(T[b])
        for r in range(n):
            ids = c[b, r] if c.ndim == 3 else c[b]
            out[b, r] = saguaro_logits(x[b, r], Tb if Tb > 0 else 0.0, ids, eps, kind)
    return out


ADJUST = [
    # B, rows per sequence, V, dtype, one list per row, eps, ids per list
    (64, 1, 128256, torch.bfloat16, False, 0.3, 32),
    (16, 8, 4097, torch.bfloat16, True, 0.9, 16),
    (5, 3, 1000, torch.float32, False, 0.5, 9),
    (4, 2, 7, torch.float32, True, 0.999, 5),
    (3, 4, 50000, torch.float32, True, 1e-4, 40),
]


@pytest.mark.parametrize("case", range(len(ADJUST)))
def test_adjusted_rows_bit_exact(case):
    from speculative_decoding_verification_89_b200 import capi
    B, n, V, dt, per_row, eps, c = ADJUST[case]
    gen = W.generator(100 + case, "cpu")
    lg = (W.gaussian((B, n, V), 2.0, gen, "cpu") + W.zipf_prior(V, 1.1, "cpu")).to(dt)
    T = torch.linspace(0.0, 2.5, B)
    T[B // 2] = -1.0                       # invalid temperature: row left as it is
    src = lg if per_row else lg[:, 0]
    cached = W.cached_tokens(src, c, seed=200 + case)
    view, buf = _padded_rows(lg, extra=3)
    capi.spec_saguaro_adjust(view, cached.to("cuda"), eps, T.to("cuda"))
    torch.cuda.synchronize()
    want = _oracle_rows(lg, T, cached, eps, "bf16" if dt == torch.bfloat16 else "f32")
    got = to_np(view)
    assert np.array_equal(got, want)
    assert torch.all(buf[:, :, V:] == 3.0)            # row padding untouched
    changed = (got != to_np(lg)).sum()
    assert changed > 0


def test_adjust_argument_checks_and_no_ops():
    from speculative_decoding_verification_89_b200 import capi
    lg = W.gaussian((2, 3, 100), 1.0, W.generator(5, "cpu"), "cpu").to(torch.bfloat16).cuda()
    before = lg.clone()
    T = torch.ones(2, device="cuda")
    ids = torch.tensor([[1, 2], [3, 4]], dtype=torch.int32, device="cuda")
    for eps in (1.0, -0.1, float("nan")):
        with pytest.raises(capi.SpecError) as err:
            capi.spec_saguaro_adjust(lg, ids, eps, T)
        assert err.value.code == capi.SPEC_EINVAL
    capi.spec_saguaro_adjust(lg, ids, 0.0, T)          # eps = 0: nothing to do
    capi.spec_saguaro_adjust(lg, ids[:, :0].contiguous(), 0.5, T)   # empty lists
    capi.spec_saguaro_adjust(lg, ids, 0.5, torch.zeros(2, device="cuda"))   # greedy
    torch.cuda.synchronize()
    assert torch.equal(lg, before)


def _draft_gpu(lg, prob, ws, st):
    from speculative_decoding_verification_89_b200 import capi
    B = lg.shape[0]
    tok = torch.full((B,), -7, dtype=torch.int32, device="cuda")
    logq = torch.full((B,), 7.0, dtype=torch.float64, device="cuda")
    ent = torch.full((B,), 7.0, dtype=torch.float64, device="cuda")
    capi.spec_draft_sample(lg, prob.temperature.cuda(), prob.seed, prob.seq_id.cuda(), prob.rnd,
                           prob.pos.cuda(), tok, st, ws, logq=logq, entropy=ent)
    torch.cuda.synchronize()
    return tok.cpu().numpy(), logq.cpu().numpy(), ent.cpu().numpy()


def test_saguaro_draft_step_full_size():
    """B=64, V=128256 bf16 drafting rows, 32 cached ids per sequence (the 29
    likeliest draft tokens, a repeat, two pads), eps = 0.5, four rounds: the
    lowered rows and the draft step on them against the oracle."""
    from speculative_decoding_verification_89_b200 import capi
    eps = 0.5
    tally = Tally()
    hits = [0, 0]
    for rnd in range(4):
        prob = W.draft_batch(rnd=rnd)
        B, V = prob.logits.shape
        cached = W.cached_tokens(prob.logits, 32, seed=300 + rnd)
        ws = capi.draft_workspace(B, V, torch.bfloat16, device="cuda")
        st = torch.zeros(1, dtype=torch.int32, device="cuda")
        plain = prob.logits.cuda().contiguous()
        tok0, _, _ = _draft_gpu(plain, prob, ws, st)
        lg = prob.logits.cuda().contiguous()
        capi.spec_saguaro_adjust(lg, cached.cuda(), eps, prob.temperature.cuda())
        tok, logq, ent = _draft_gpu(lg, prob, ws, st)
        assert int(st.item()) == 0
        adj = _oracle_rows(prob.logits[:, None], prob.temperature, cached, eps, "bf16")[:, 0]
        assert np.array_equal(to_np(lg), adj)
        ref = draft_step(adj, prob.temperature.numpy(), prob.seed, prob.seq_id.numpy(), prob.rnd,
                         prob.pos.numpy())
        c = cached.numpy()
        for b, r in enumerate(ref):
            tally.decisions += 1
            hits[0] += int(tok0[b] in c[b])
            hits[1] += int(tok[b] in c[b])
            if int(tok[b]) != r.token:
                assert r.margin < MARGIN, (rnd, b, int(tok[b]), r.token, r.margin)
                tally.excused += 1
                tally.details.append((rnd, b, "draft", r.margin))
                continue
            assert abs(logq[b] - r.logq) <= 1e-5, (rnd, b, logq[b], r.logq)
            assert abs(ent[b] - r.entropy) <= 1e-5 * (1.0 + abs(r.entropy)), (rnd, b)
    tally.check_share()
    assert hits[1] < hits[0], hits    # the lowered tokens are drafted less often


def test_saguaro_chain_check_full_size():
    """B=64, K=8, V=128256 bf16 chain batch; one cache list per position (the
    29 likeliest target tokens there, the drafted token for even sequences,
    two pads); eps = 0.3; the lowered draft rows checked on the GPU against
    the oracle's check of its own lowered rows, two rounds."""
    from speculative_decoding_verification_89_b200 import capi
    eps = 0.3
    tally = Tally()
    for rnd in range(2):
        prob = W.chain_batch(rnd=rnd)
        B, Kp1, V = prob.tgt.shape
        K = Kp1 - 1
        extra = prob.draft_tok.clone()
        extra[1::2] = -1
        cached = W.cached_tokens(prob.tgt[:, :K], 32, seed=400 + rnd, extra=extra)
        tgt = prob.tgt.cuda().contiguous()
        drf = prob.drf.cuda().contiguous()
        T = prob.temperature.cuda()
        capi.spec_saguaro_adjust(drf, cached.cuda(), eps, T)
        ws = capi.workspace(B, K, V, torch.bfloat16, device="cuda")
        acc = torch.full((B,), -7, dtype=torch.int32, device="cuda")
        out = torch.full((B, K + 1), -7, dtype=torch.int32, device="cuda")
        dg = torch.full((B, 4 * K + 2), -7.0, dtype=torch.float64, device="cuda")
        st = torch.zeros(1, dtype=torch.int32, device="cuda")
        capi.spec_verify_chain(tgt, drf, prob.draft_tok.cuda(), T, prob.seed, prob.seq_id.cuda(),
                               prob.rnd, acc, out, st, ws, diag=dg)
        torch.cuda.synchronize()
        assert int(st.item()) == 0
        adj = _oracle_rows(prob.drf, prob.temperature, cached, eps, "bf16")
        assert np.array_equal(to_np(drf), adj)
        ref = verify_chain(to_np(prob.tgt), adj, prob.draft_tok.numpy(),
                           prob.temperature.numpy(), prob.seed, prob.seq_id.numpy(), prob.rnd)
        a_all, o_all, d_all = acc.cpu().numpy(), out.cpu().numpy(), dg.cpu().numpy()
        for b, r in enumerate(ref):
            a = int(a_all[b])
            if compare_check(f"r{rnd}/seq{b}", r, a, [int(x) for x in o_all[b, :a + 1]], tally):
                compare_probs(f"r{rnd}/seq{b}", r, d_all[b], K, float(prob.temperature[b]))
    tally.check_share()
