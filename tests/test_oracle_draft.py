"""Pins of the oracle's draft step (draft token and draft entropy).

* The draft token is a draw from the drafting exit's distribution
  softmax(l_d / T) (HiSpec, gist.science summary of arXiv 2510.01336,
  section 2 "Kernmechanismus"): its law, found by probing the oracle with
  uniforms at the ends of every outcome interval, is that softmax exactly.
* The entropy of the draft distribution is the uncertainty signal of SVIP
  (Optimierung der Inferenzgeschwindigkeit von Sprachmodellen durch
  spekulative Dekodierung, mind-verse.de, SVIP paragraphs): checked against
  closed forms (uniform rows, two-point rows), scipy's entropy, and the
  temperature scaling identity H(l, T) = H(l / T, 1).
"""
import math

import numpy as np
import pytest
import scipy.special
import scipy.stats

from oracle.draft import draft_sample, draft_step, entropy
from oracle.philox import STAGE_DRAFT, uniforms


def _sm(l, T):
    z = np.asarray(l, np.float64) / T
    return np.exp(z - scipy.special.logsumexp(z))


# ---------------------------------------------------------------------------
# Entropy
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("V", [1, 2, 7, 1000])
def test_uniform_row_entropy_is_log_v(V):
    for T in (0.3, 1.0, 4.0):
        assert abs(entropy(np.full(V, 1.25), T) - math.log(V)) < 1e-12


def test_two_point_entropy_closed_form():
    for d in (-8.0, -1.0, 0.0, 0.5, 3.0, 20.0):
        for T in (0.5, 1.0, 2.0):
            p = 1.0 / (1.0 + math.exp(-d / T))   # p of the second entry
            want = -sum(x * math.log(x) for x in (p, 1.0 - p) if x > 0.0)
            assert abs(entropy(np.array([0.0, d]), T) - want) < 1e-12


def test_entropy_matches_scipy_with_masked_entries():
    rng = np.random.default_rng(5)
    for T in (1e-2, 0.7, 1.0, 30.0):
        for _ in range(10):
            l = rng.normal(0, 3, size=300)
            l[rng.integers(0, 300, size=7)] = -np.inf
            want = scipy.stats.entropy(_sm(l, T))
            assert abs(entropy(l, T) - want) <= 1e-12 * max(1.0, want)


def test_entropy_temperature_scaling():
    rng = np.random.default_rng(6)
    l = rng.normal(0, 2, size=64)
    for T in (0.25, 1.7):
        assert abs(entropy(l, T) - entropy(l / T, 1.0)) < 1e-12


def test_greedy_and_point_mass_have_zero_entropy():
    l = np.array([1.0, 5.0, 2.0])
    assert entropy(l, 0.0) == 0.0
    m = np.full(10, -np.inf)
    m[3] = 0.0
    assert entropy(m, 1.0) == 0.0


# ---------------------------------------------------------------------------
# Draft token
# ---------------------------------------------------------------------------

def _probe_law(l, T):
    """Law of draft_sample's token over u in (0, 1): every interval of u that
    maps to one token, found from the probability the oracle reports for the
    token it returns (checked at both ends of the interval)."""
    law = {}
    u = 0.0
    while u < 1.0:
        mid = min(u + 1e-13, 1.0 - 1e-16)
        r = draft_sample(l, T, mid)
        width = math.exp(r.logq)
        hi = min(1.0, u + width)
        # the whole interval maps to the same token
        for probe in (u + 0.25 * width, hi - max(1e-12, 1e-9 * width)):
            if u < probe < 1.0:
                assert draft_sample(l, T, probe).token == r.token
        law[r.token] = law.get(r.token, 0.0) + (hi - u)
        u = hi
    return law


@pytest.mark.parametrize("seed", [0, 1])
def test_draft_law_is_softmax(seed):
    rng = np.random.default_rng(seed)
    for T in (0.6, 1.0, 2.5):
        l = rng.normal(0, 2, size=9)
        l[rng.integers(0, 9)] = -np.inf
        law = _probe_law(l, T)
        p = _sm(l, T)
        for v in range(9):
            assert abs(law.get(v, 0.0) - p[v]) < 1e-12, (v, law.get(v), p[v])


def test_logq_is_log_softmax_of_the_token():
    rng = np.random.default_rng(9)
    l = rng.normal(0, 2, size=50)
    for u in (0.01, 0.3, 0.77, 0.999):
        r = draft_sample(l, 0.9, u)
        want = l[r.token] / 0.9 - scipy.special.logsumexp(l / 0.9)
        assert abs(r.logq - want) < 1e-12


def test_greedy_draft_is_first_argmax():
    l = np.array([0.5, 3.0, -1.0, 3.0])
    r = draft_sample(l, 0.0, 0.42)
    assert r.token == 1 and r.logq == 0.0 and r.entropy == 0.0


def test_draft_step_uses_the_draft_stage_stream():
    """Row b's token is the draw with the lane-1 uniform of counter
    (seq_id[b], round, pos[b], stage 0)."""
    rng = np.random.default_rng(12)
    B, V = 5, 40
    l = rng.normal(0, 2, size=(B, V))
    T = np.array([1.0, 0.5, 0.0, 2.0, 1.0])
    seq = np.array([3, 9, 11, 0, 7])
    pos = np.array([0, 4, 2, 7, 1])
    res = draft_step(l, T, 77, seq, 5, pos)
    for b in range(B):
        u = uniforms(77, int(seq[b]), 5, int(pos[b]), STAGE_DRAFT)[1]
        assert res[b].token == draft_sample(l[b], float(T[b]), u).token


def test_draft_step_empirical_frequencies():
    """With the real Philox stream the drafted tokens follow softmax(l/T):
    chi-square over 4000 rounds."""
    rng = np.random.default_rng(13)
    V, T, n = 6, 0.8, 4000
    l = rng.normal(0, 1.5, size=V)
    counts = np.zeros(V)
    for r in range(n):
        counts[draft_step(l[None, :], [T], 21, [4], r, [3])[0].token] += 1
    p = _sm(l, T)
    stat = float(np.sum((counts - n * p) ** 2 / (n * p)))
    assert stat < scipy.stats.chi2.ppf(0.9999, V - 1)
