"""Closed forms and special cases the oracle must reproduce.

* P(accept a draft x ~ q) = sum_v min(p_v, q_v) = 1 - TV(p, q), and the
  residual mass of a rejection is TV(p, q): the standard facts behind the
  lossless speculative-sampling argument that HiSpec (gist.science summary of
  arXiv 2510.01336, section 2, "Verlustfreie Garantie") appeals to, and the
  "residual distribution proportional to the target-minus-draft difference"
  of Speculative Speculative Decoding (gist.science summary of arXiv
  2603.03251, Technische Zusammenfassung 3.B).
* Greedy decoding (temperature 0) equals autoregressive argmax.
* No drafts: the draw is plain inverse-CDF sampling from the target row.
* One-hot and single-token vocabularies are deterministic.
"""
import numpy as np
import pytest

from oracle.philox import PhiloxUniforms
from oracle.verify import speculative_check, verify_chain
from tests.law_enum import ScriptedSource, draw_draft, enumerate_law


def _tv(p, q):
    return 0.5 * float(np.sum(np.abs(p - q)))


def _sm(l, T):
    z = np.asarray(l, np.float64) / T
    e = np.exp(z - z.max())
    return e / e.sum()


@pytest.mark.parametrize("seed", [0, 1, 2])
def test_accept_probability_is_one_minus_tv(seed):
    rng = np.random.default_rng(seed)
    V, T = 9, 0.8
    tgt = rng.normal(0, 2, size=(2, V))
    drf = tgt[:1] + rng.normal(0, 1.2, size=(1, V))

    def run(script):
        x, dec = draw_draft(script, drf[0], T)
        res = speculative_check(tgt, drf, [x], T, ScriptedSource(script))
        return (res.accepted,), [dec] + res.decisions[:1]

    law = enumerate_law(run)
    p, q = _sm(tgt[0], T), _sm(drf[0], T)
    assert abs(law[(1,)] - (1.0 - _tv(p, q))) < 1e-12
    assert abs(law[(1,)] - float(np.sum(np.minimum(p, q)))) < 1e-12


def test_residual_mass_is_tv():
    rng = np.random.default_rng(4)
    V, T = 50, 1.3
    for _ in range(20):
        tgt = rng.normal(0, 2, size=(2, V))
        drf = tgt[:1] + rng.normal(0, 1.0, size=(1, V))
        x = int(np.argmin(_sm(tgt[0], T) / _sm(drf[0], T)))  # likely reject
        res = speculative_check(tgt, drf, [x], T,
                                _FixedUniform(0.999999))
        if res.accepted == 0:
            assert abs(res.residual_mass - _tv(_sm(tgt[0], T), _sm(drf[0], T))) < 1e-13


class _FixedUniform:
    """Uniform source returning one value for every draw."""

    def __init__(self, u):
        self.u = u

    def accept(self, pos):
        return self.u

    def sample(self, pos):
        return self.u


def test_greedy_equals_autoregressive_argmax():
    rng = np.random.default_rng(8)
    B, K, V = 16, 6, 40
    tgt = rng.normal(0, 2, size=(B, K + 1, V))
    drf = tgt[:, :K] + rng.normal(0, 1.0, size=(B, K, V))
    drafts = np.argmax(drf, axis=-1)
    res = verify_chain(tgt, drf, drafts, np.zeros(B), 0, np.arange(B), 0)
    for b in range(B):
        want = []
        for j in range(K + 1):       # autoregressive argmax, stop at mismatch
            top = int(np.argmax(tgt[b, j]))
            want.append(top)
            if j == K or drafts[b, j] != top:
                break
        assert res[b].tokens == want
        assert res[b].accepted == len(want) - 1


def test_greedy_ties_take_smallest_id():
    tgt = np.array([[1.0, 3.0, 3.0, 0.0], [2.0, 2.0, 2.0, 2.0]])
    res = speculative_check(tgt, None, [1], 0.0, None)
    assert res.tokens == [1, 0]
    res = speculative_check(tgt, None, [2], 0.0, None)
    assert res.tokens == [1]


def test_no_drafts_is_inverse_cdf_sampling():
    """K = 0: the token is the inverse-CDF draw from p with the lane-1
    uniform of position 0, checked against a brute-force running sum."""
    rng = np.random.default_rng(12)
    V, T = 30, 0.9
    for r in range(50):
        tgt = rng.normal(0, 2, size=(1, V))
        uni = PhiloxUniforms(3, 1, r, 1)
        res = speculative_check(tgt, np.zeros((0, V)), [], T, uni)
        p = _sm(tgt[0], T)
        u = uni.sample(0)
        acc, want = 0.0, None
        for v in range(V):          # brute force: first v with sum > u
            acc += p[v]
            if acc > u * 1.0 and want is None:
                want = v
        assert res.accepted == 0 and res.tokens == [want]


def test_one_hot_target_is_deterministic():
    V, K, T = 12, 3, 1.0
    tgt = np.full((K + 1, V), -1e4)
    tgt[np.arange(K + 1), [3, 5, 7, 9]] = 0.0
    rng = np.random.default_rng(1)
    drf = rng.normal(0, 1, size=(K, V))
    for r in range(20):
        drafts = [3, 5, int(rng.integers(V))]
        res = speculative_check(tgt, drf, drafts, T, PhiloxUniforms(0, 0, r, 1))
        want = [3, 5, 7] if drafts[2] != 7 else [3, 5, 7, 9]
        assert res.tokens == want


def test_single_token_vocabulary():
    tgt = np.zeros((4, 1))
    res = speculative_check(tgt, np.zeros((3, 1)), [0, 0, 0], 0.7,
                            PhiloxUniforms(0, 0, 0, 1))
    assert res.tokens == [0, 0, 0, 0] and res.accepted == 3


def test_empirical_acceptance_with_philox():
    """Acceptance frequency over Philox rounds lies within 5 sigma of the
    closed form 1 - TV(p, q)."""
    rng = np.random.default_rng(21)
    V, T, n = 16, 1.0, 4000
    tgt = rng.normal(0, 2, size=(2, V))
    drf = tgt[:1] + rng.normal(0, 1.0, size=(1, V))
    p, q = _sm(tgt[0], T), _sm(drf[0], T)
    acc = 0
    for r in range(n):
        x = int(np.searchsorted(np.cumsum(q), rng.random() * q.sum(), "right"))
        res = speculative_check(tgt, drf, [min(x, V - 1)], T,
                                PhiloxUniforms(77, 5, r, 1))
        acc += res.accepted
    mean = 1.0 - _tv(p, q)
    sd = np.sqrt(mean * (1 - mean) / n)
    assert abs(acc / n - mean) < 5 * sd


def test_log_partition_is_logsumexp():
    """The oracle's row log-partition equals scipy's logsumexp(l / T),
    including rows with masked (-inf) entries and extreme temperatures."""
    import scipy.special
    from oracle.verify import log_partition
    rng = np.random.default_rng(33)
    for T in (1e-3, 0.7, 1.0, 50.0):
        for _ in range(10):
            l = rng.normal(0, 3, size=257)
            l[rng.integers(0, 257, size=5)] = -np.inf
            want = scipy.special.logsumexp(l / T)
            assert abs(log_partition(l, T) - want) <= 1e-13 * max(1.0, abs(want))


def test_inverse_cdf_boundary_and_rounding_fallback():
    """The draw's boundary rule (smallest v with C(v) > u * Z) at the
    interval ends, and the fallback for a target that reaches Z itself:
    u * Z == Z happens for u = 1 (valid Philox uniforms stop at 1 - 2^-24,
    so only rounding could get there); the draw then takes the last token
    with mass, never a zero-mass token past it."""
    from oracle.verify import inverse_cdf
    w = np.array([0.0, 0.25, 0.0, 0.5, 0.25, 0.0, 0.0])
    z = w.sum()
    # Interval ends: C = [0, .25, .25, .75, 1, 1, 1].
    assert inverse_cdf(w, 0.0)[0] == 1              # C(1) = .25 > 0
    assert inverse_cdf(w, 0.25)[0] == 3             # C(1) = .25 is not > .25
    assert inverse_cdf(w, np.nextafter(0.25, 0))[0] == 1
    assert inverse_cdf(w, 0.75)[0] == 4
    # u * Z == Z: the last token with positive mass (index 4), margin 0.
    assert 1.0 * z == z
    tok, margin = inverse_cdf(w, 1.0)
    assert tok == 4 and margin == 0.0
    # The largest valid uniform lands on the same token without the fallback.
    assert inverse_cdf(w, 1.0 - 2.0 ** -24)[0] == 4
    # A single token with mass is drawn for every u, the fallback included.
    one = np.array([0.0, 0.0, 3.0, 0.0])
    for u in (2.0 ** -24, 0.5, 1.0 - 2.0 ** -24, 1.0):
        assert inverse_cdf(one, u)[0] == 2
