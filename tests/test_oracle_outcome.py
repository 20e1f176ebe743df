"""Pins of the oracle's outcome law (outcome prediction for a speculation
cache: Speculative Speculative Decoding, gist.science summary of arXiv
2603.03251, Technische Zusammenfassung 2 and 3.A-B).

The law is checked against the law the oracle's own verification actually
implements, found by enumerating every outcome interval of every uniform it
draws (the drafts held fixed): the two are written independently (a product
formula here, a branching check there), so a dropped term, a wrong index or an
exchanged row breaks the match."""
import numpy as np
import pytest

from oracle.outcome import fan_out, outcome_law, top_outcomes
from oracle.verify import speculative_check
from tests.law_enum import ScriptedSource, enumerate_law


def _enumerated(tgt, drf, drafts, T):
    def run(script):
        res = speculative_check(tgt, drf, drafts, T, ScriptedSource(script))
        return (res.accepted, res.tokens[-1]), res.decisions
    return enumerate_law(run)


@pytest.mark.parametrize("K,T,seed", [(1, 1.0, 0), (2, 0.7, 1), (3, 1.3, 2), (3, 0.0, 3),
                                      (2, 1.0, 4)])
def test_outcome_law_equals_the_enumerated_check(K, T, seed):
    rng = np.random.default_rng(seed)
    V = 7
    tgt = rng.normal(0, 1.5, size=(K + 1, V))
    drf = tgt[:K] + rng.normal(0, 1.0, size=(K, V))
    drafts = [int(rng.integers(0, V)) for _ in range(K)]
    if T == 0.0:   # make some greedy drafts match
        drafts[0] = int(np.argmax(tgt[0]))
    law = outcome_law(tgt, drf, drafts, T)
    enum = _enumerated(tgt, drf, drafts, T)
    assert abs(sum(enum.values()) - 1.0) < 1e-12
    joint = law.p_len[:, None] * law.resid
    for k in range(K + 1):
        for v in range(V):
            assert abs(enum.get((k, v), 0.0) - joint[k, v]) < 1e-12, (k, v)


def test_equal_rows_accept_everything():
    rng = np.random.default_rng(7)
    l = rng.normal(0, 1, size=(3, 11))
    law = outcome_law(l, l[:2], [3, 5], 1.0)
    assert np.allclose(law.beta, 1.0) and law.p_len[2] == 1.0 and law.p_len[:2].sum() == 0.0


def test_geometric_lengths_for_equal_accept_probabilities():
    """With the same beta at every position, P(a = k) is geometric:
    beta^k (1 - beta), and beta^K at k = K."""
    V, K = 4, 5
    tgt = np.log(np.array([[0.4, 0.3, 0.2, 0.1]] * (K + 1)))
    drf = np.log(np.array([[0.1, 0.3, 0.2, 0.4]] * K))
    law = outcome_law(tgt, drf, [0] * K, 1.0)       # beta = min(1, 0.4/0.1) = 1
    assert np.allclose(law.beta, 1.0)
    law = outcome_law(tgt, drf, [3] * K, 1.0)       # beta = 0.1 / 0.4
    b = 0.25
    want = [b ** k * (1 - b) for k in range(K)] + [b ** K]
    assert np.allclose(law.p_len, want, atol=1e-15)


def test_top_outcomes_cover_the_most_mass_and_fan_out():
    rng = np.random.default_rng(8)
    K, V = 4, 30
    tgt = rng.normal(0, 2, size=(K + 1, V))
    drf = tgt[:K] + rng.normal(0, 1.5, size=(K, V))
    drafts = [int(np.argmax(drf[j])) for j in range(K)]
    law = outcome_law(tgt, drf, drafts, 1.0)
    joint = law.p_len[:, None] * law.resid
    for n in (1, 5, 17, 60):
        top = top_outcomes(law, n)
        assert len(top) == n
        probs = [p for _, _, p in top]
        assert probs == sorted(probs, reverse=True)
        # no excluded outcome is more likely than the least likely included one
        chosen = {(k, v) for k, v, _ in top}
        rest = [joint[k, v] for k in range(K + 1) for v in range(V) if (k, v) not in chosen]
        assert max(rest) <= min(probs)
        assert fan_out(top, K).sum() == n


def test_greedy_outcome_is_a_point_mass():
    tgt = np.array([[0.0, 2.0, 1.0], [3.0, 0.0, 1.0], [0.0, 0.0, 5.0]])
    drf = np.zeros((2, 3))
    law = outcome_law(tgt, drf, [1, 2], 0.0)         # x_0 = argmax, x_1 != argmax (0)
    assert list(law.p_len) == [0.0, 1.0, 0.0]
    assert top_outcomes(law, 3) == [(1, 0, 1.0)]
