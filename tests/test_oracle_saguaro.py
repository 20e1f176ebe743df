"""Pins of the oracle's Saguaro lowering (Speculative Speculative Decoding,
gist.science summary of arXiv 2603.03251, Technische Zusammenfassung 3.B:
the cached tokens' probabilities are lowered a little in the draft so the
residual -- proportional to the target-minus-draft difference -- lands on
them more often).

* The shifted draft law equals q(v) (1 - eps [v cached]) renormalised, written
  out from that definition here.
* Drafting from the lowered law and checking with it as the draft law is
  still lossless: the exact output law (interval enumeration) equals
  softmax(l_target / T), for every eps tried.
* The residual-hit probability (a rejection whose drawn token is cached) is
  sum_{v cached} max(0, p_v - q'_v), the closed form, and it grows with eps
  on the example.
* The bfloat16 rounding of the stored rows is round-to-nearest-even.
"""
import numpy as np
import pytest

from oracle.draft import round_bf16, saguaro_logits
from oracle.verify import softmax, speculative_check
from tests.law_enum import ScriptedSource, draw_draft, enumerate_law, max_law_error

TOL = 1e-12


def _lowered_law(l, T, cached, eps):
    """q'(v) = q(v) (1 - eps [v cached]) / sum, from the definition."""
    z = np.asarray(l, np.float64) / T
    q = np.exp(z - z.max())
    q /= q.sum()
    f = np.ones_like(q)
    for v in set(int(c) for c in cached if 0 <= c < len(q)):
        f[v] = 1.0 - eps
    w = q * f
    return w / w.sum()


@pytest.mark.parametrize("eps", [0.0, 0.2, 0.9])
@pytest.mark.parametrize("T", [0.3, 1.0, 2.5])
def test_lowered_softmax_is_the_renormalised_product(eps, T):
    rng = np.random.default_rng(int(eps * 10) + int(T * 7))
    V = 50
    l = rng.normal(0, 2, V)
    l[[3, 17]] = -np.inf                          # masked entries stay masked
    cached = [5, 9, 9, 44, -1, 50, 17]            # duplicate, pads, a masked id
    got = softmax(saguaro_logits(l, T, cached, eps), T)
    ref = _lowered_law(np.where(np.isinf(l), -1e300, l), T, cached, eps)
    ref[[3, 17]] = 0.0
    ref /= ref.sum()
    assert np.allclose(got, ref, rtol=1e-12, atol=1e-300)
    assert got[3] == 0.0 and got[17] == 0.0


def test_greedy_and_zero_eps_leave_the_row():
    l = np.random.default_rng(3).normal(0, 1, 20)
    assert np.array_equal(saguaro_logits(l, 0.0, [1, 2, 3], 0.5), l)
    assert np.array_equal(saguaro_logits(l, 1.3, [1, 2, 3], 0.0), l)
    assert np.array_equal(saguaro_logits(l, 1.3, [], 0.5), l)


def _run(tgt, drf_lowered, K, T):
    def run(script):
        trace, drafts = [], []
        for j in range(K):
            x, dec = draw_draft(script, drf_lowered[j], T)
            drafts.append(x)
            if dec is not None:
                trace.append(dec)
        res = speculative_check(tgt[:K + 1], drf_lowered[:K], drafts, T, ScriptedSource(script))
        trace += res.decisions
        return tuple(res.tokens), trace
    return run


@pytest.mark.parametrize("K", [1, 2])
@pytest.mark.parametrize("eps", [0.3, 0.9])
def test_drafting_from_the_lowered_law_stays_lossless(K, eps):
    rng = np.random.default_rng(40 + K)
    V, T = 8, 0.8
    tgt = rng.normal(0, 2, (K + 1, V))
    drf = tgt[:K] + rng.normal(0, 1, (K, V))
    cached = [1, 4, 6]
    low = np.stack([saguaro_logits(drf[j], T, cached, eps) for j in range(K)])
    law = enumerate_law(_run(tgt, low, K, T))
    assert abs(sum(law.values()) - 1.0) < TOL
    assert max_law_error(law, tgt, T) < TOL


def _residual_hit(tgt, drf, T, cached, eps):
    """P(the first position is rejected and the drawn token is cached), from
    the enumerated output law of one draft."""
    low = saguaro_logits(drf[0], T, cached, eps)[None]
    hit = 0.0

    def run(script):
        x, dec = draw_draft(script, low[0], T)
        res = speculative_check(tgt[:2], low, [x], T, ScriptedSource(script))
        return (res.accepted, tuple(res.tokens)), [dec] + res.decisions

    for (a, toks), pr in enumerate_law(run).items():
        if a == 0 and toks[0] in cached:
            hit += pr
    return hit


def test_residual_hit_probability_closed_form_and_growth():
    rng = np.random.default_rng(9)
    V, T = 8, 1.0
    tgt = rng.normal(0, 2, (2, V))
    drf = tgt[:1] + rng.normal(0, 1.5, (1, V))
    cached = [2, 5]
    hits = []
    for eps in (0.0, 0.3, 0.6, 0.9):
        p = softmax(tgt[0], T)
        q = _lowered_law(drf[0], T, cached, eps)
        closed = sum(max(0.0, p[v] - q[v]) for v in cached)
        got = _residual_hit(tgt, drf, T, cached, eps)
        assert abs(got - closed) < TOL, (eps, got, closed)
        hits.append(got)
    assert all(b >= a for a, b in zip(hits, hits[1:])) and hits[-1] > hits[0]


def test_bf16_rounding_is_nearest_even():
    # 1 + 2^-8 lies halfway between 1 and 1 + 2^-7: ties go to the even one (1).
    half = np.float32(1.0 + 2.0 ** -8)
    assert round_bf16(half) == np.float32(1.0)
    # 1 + 3 * 2^-8 is halfway between 1 + 2^-7 and 1 + 2^-6: even is 1 + 2^-6.
    assert round_bf16(np.float32(1.0 + 3 * 2.0 ** -8)) == np.float32(1.0 + 2.0 ** -6)
    # just above a half rounds up, just below rounds down
    assert round_bf16(np.nextafter(half, np.float32(2))) == np.float32(1.0 + 2.0 ** -7)
    assert round_bf16(np.nextafter(half, np.float32(0))) == np.float32(1.0)
    # representable values are fixed points; infinities stay
    for v in (0.0, -2.5, 3.0 * 2.0 ** 100, -np.inf, np.inf):
        assert round_bf16(np.float32(v)) == np.float32(v)
    assert np.isnan(round_bf16(np.float32(np.nan)))
    # rounding up carries into the exponent: the float just below 2 becomes 2
    assert round_bf16(np.nextafter(np.float32(2.0), np.float32(0))) == np.float32(2.0)
    assert round_bf16(np.float32(-(2.0 - 2.0 ** -23))) == np.float32(-2.0)
    # the sign of zero is kept
    assert np.signbit(round_bf16(np.float32(-0.0)))


def test_stored_shift_follows_the_kernel_arithmetic():
    """The f32 / bf16 forms differ from the exact shift by the storage
    rounding only."""
    rng = np.random.default_rng(5)
    l = rng.normal(0, 3, 64).astype(np.float32).astype(np.float64)
    cached = list(range(0, 64, 3))
    exact = saguaro_logits(l, 0.7, cached, 0.25)
    for dt, ulp in (("f32", 2.0 ** -23), ("bf16", 2.0 ** -7)):
        got = saguaro_logits(l, 0.7, cached, 0.25, dtype=dt)
        err = np.abs(got - exact)[cached] / np.maximum(np.abs(exact[cached]), 1e-30)
        assert np.all(err <= ulp), dt
        other = [v for v in range(64) if v not in cached]
        assert np.array_equal(got[other], l[other])
