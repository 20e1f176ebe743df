"""Exact output-law pins of the oracle (lossless property).

HiSpec (gist.science summary of arXiv 2510.01336), section 2, bullet
"Verlustfreie Garantie", and section 4 ("100 % accuracy"): the tokens the
scheme commits follow the final layer's autoregressive law, stage by stage and
composed, whatever the intermediate exit says. Here that is checked exactly
(to 1e-12) on tiny vocabularies by enumerating every outcome interval of every
uniform the oracle draws (see ``law_enum``).
"""
import numpy as np
import pytest

from oracle.verify import speculative_check, verify_hier_seq
from tests.law_enum import (ScriptedSource, draw_draft, enumerate_law,
                            max_law_error)

TOL = 1e-12


def _rows(rng, n, V, scale=2.0):
    return rng.normal(0.0, scale, size=(n, V))


def _chain_run(tgt, drf, K, T):
    """Draw K drafts from the draft rows, then verify them (stage one)."""
    def run(script):
        trace, drafts = [], []
        for j in range(K):
            x, dec = draw_draft(script, drf[j], T)
            drafts.append(x)
            if dec is not None:
                trace.append(dec)
        res = speculative_check(tgt[:K + 1], drf[:K], drafts, T,
                                ScriptedSource(script))
        trace += res.decisions
        return tuple(res.tokens), trace
    return run


@pytest.mark.parametrize("K", [0, 1, 2, 3])
@pytest.mark.parametrize("T", [1.0, 0.6])
def test_single_stage_law_equals_target(K, T):
    rng = np.random.default_rng(100 + K)
    V = 8 if K < 3 else 6
    tgt = _rows(rng, K + 1, V)
    drf = tgt[:K] + rng.normal(0, 1.0, size=(K, V))
    law = enumerate_law(_chain_run(tgt, drf, K, T))
    assert abs(sum(law.values()) - 1.0) < TOL
    assert max_law_error(law, tgt, T) < TOL


def test_single_stage_adversarial_rows():
    """Draft far from target, near one-hot rows, zero-mass tokens, p == q."""
    rng = np.random.default_rng(7)
    V, K, T = 8, 2, 1.0
    tgt = _rows(rng, K + 1, V)
    cases = {
        "reversed": -tgt[:K],
        "one_hot_draft": np.where(np.arange(V) == 3, 25.0, 0.0)[None].repeat(K, 0),
        "equal": tgt[:K].copy(),
    }
    for name, drf in cases.items():
        law = enumerate_law(_chain_run(tgt, drf, K, T))
        assert max_law_error(law, tgt, T) < TOL, name
    # zero-mass tokens in the target: never emitted
    tgt2 = tgt.copy()
    tgt2[:, 5] = -np.inf
    drf2 = tgt2[:K] + rng.normal(0, 1.0, size=(K, V))
    drf2[:, 5] = 0.0
    law = enumerate_law(_chain_run(tgt2, drf2, K, T))
    assert max_law_error(law, tgt2, T) < TOL
    assert all(5 not in toks for toks in law)


def test_equal_laws_accept_everything():
    """p == q: every draft is accepted and the bonus comes from row K."""
    rng = np.random.default_rng(3)
    V, K, T = 8, 3, 0.8
    tgt = _rows(rng, K + 1, V)
    run = _chain_run(tgt, tgt[:K].copy(), K, T)
    law = enumerate_law(run, probe_edges=False)
    assert all(len(t) == K + 1 for t in law)


def _stage_two_run(lg_i, lg_f, W, T):
    """Window tokens drawn from the L_i law per slot, then stage two."""
    def run(script):
        trace, window = [], []
        for s in range(W):
            x, dec = draw_draft(script, lg_i[s], T)
            window.append(x)
            if dec is not None:
                trace.append(dec)
        res = speculative_check(lg_f[:W + 1], lg_i[:W], window, T,
                                ScriptedSource(script))
        trace += res.decisions
        return tuple(res.tokens), trace
    return run


@pytest.mark.parametrize("W", [1, 2, 3])
def test_stage_two_law_equals_final(W):
    rng = np.random.default_rng(200 + W)
    V, T = 6, 0.9
    lg_f = _rows(rng, W + 1, V)
    lg_i = lg_f[:W] + rng.normal(0, 0.7, size=(W, V))
    law = enumerate_law(_stage_two_run(lg_i, lg_f, W, T), probe_edges=False)
    assert max_law_error(law, lg_f, T) < TOL


def _cycle_run(lg_d, lg_i, lg_f, K, n_i, T, max_rounds=8):
    """Full window cycle: stage-one rounds until stage two commits."""
    def run(script):
        trace, window = [], []
        for _ in range(max_rounds):
            w = len(window)
            drafts = []
            for j in range(K):
                x, dec = draw_draft(script, lg_d[w + j], T)
                drafts.append(x)
                if dec is not None:
                    trace.append(dec)
            src = ScriptedSource(script)
            res = verify_hier_seq(lg_d, lg_i, lg_f, drafts, T, window, n_i,
                                  src, src)
            trace += res.stage1.decisions
            if res.stage2 is not None:
                trace += res.stage2.decisions
                return tuple(res.committed), trace
            window = res.window
        raise AssertionError("window never filled")
    return run


@pytest.mark.parametrize("K,n_i,V", [(1, 1, 6), (1, 2, 5), (2, 2, 4), (1, 3, 4)])
def test_composed_cycle_law_equals_final(K, n_i, V):
    """L_d -> L_i -> L_f over a whole window cycle commits the L_f law."""
    rng = np.random.default_rng(300 + 10 * K + n_i)
    T = 1.0
    S = n_i + K + 1
    lg_f = _rows(rng, S, V)
    lg_i = lg_f + rng.normal(0, 0.7, size=(S, V))
    lg_d = lg_f + rng.normal(0, 1.5, size=(S, V))
    law = enumerate_law(_cycle_run(lg_d, lg_i, lg_f, K, n_i, T),
                        probe_edges=False)
    assert abs(sum(law.values()) - 1.0) < TOL
    assert max_law_error(law, lg_f, T) < TOL


def test_composed_cycle_adversarial_intermediate():
    """An intermediate exit unrelated to the final layer cannot bias it."""
    rng = np.random.default_rng(41)
    K, n_i, V, T = 1, 2, 5, 0.7
    S = n_i + K + 1
    lg_f = _rows(rng, S, V)
    lg_i = -lg_f                       # maximally wrong intermediate exit
    lg_d = rng.normal(0, 3.0, size=(S, V))
    law = enumerate_law(_cycle_run(lg_d, lg_i, lg_f, K, n_i, T),
                        probe_edges=False)
    assert max_law_error(law, lg_f, T) < TOL


def test_stage_one_window_follows_intermediate_law():
    """Stage one alone: each window token follows the L_i law of its slot."""
    rng = np.random.default_rng(5)
    K, V, T = 2, 6, 1.0
    lg_i = _rows(rng, K + 1, V)
    lg_d = lg_i[:K] + rng.normal(0, 1.5, size=(K, V))
    law = enumerate_law(_chain_run(lg_i, lg_d, K, T), probe_edges=False)
    assert max_law_error(law, lg_i, T) < TOL


def test_greedy_cycle_is_autoregressive_argmax():
    """T = 0 through the whole hierarchy commits argmax of L_f per slot."""
    rng = np.random.default_rng(9)
    K, n_i, V = 2, 2, 7
    S = n_i + K + 1
    lg_f = _rows(rng, S, V)
    lg_i = lg_f + rng.normal(0, 1.0, size=(S, V))
    lg_d = lg_f + rng.normal(0, 2.0, size=(S, V))
    law = enumerate_law(_cycle_run(lg_d, lg_i, lg_f, K, n_i, 0.0))
    assert len(law) == 1
    (toks, p), = law.items()
    assert p == 1.0
    assert list(toks) == [int(np.argmax(lg_f[s])) for s in range(len(toks))]


def test_swapped_roles_are_caught():
    """The pin has teeth: verifying with target and draft rows exchanged (a
    plausible operand mistake, planted on the CPU by calling the oracle with
    the rows swapped) gives a law far from the target."""
    rng = np.random.default_rng(11)
    V, K, T = 6, 1, 1.0
    tgt = _rows(rng, K + 1, V)
    drf = tgt[:K] + rng.normal(0, 1.5, size=(K, V))

    def run(script):
        x, dec = draw_draft(script, drf[0], T)
        res = speculative_check(np.vstack([drf[0], tgt[1]]), tgt[:1], [x], T,
                                ScriptedSource(script))
        return tuple(res.tokens), [dec] + res.decisions

    law = enumerate_law(run, probe_edges=False)
    assert max_law_error(law, tgt, T) > 1e-3
