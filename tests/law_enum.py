"""Exact output-law enumeration of the oracle with injected uniforms.

The oracle is driven as a black box through its uniform sources. A run is
replayed with a fixed prefix of uniforms; the oracle's decision trace tells
which decision comes next and the outcome intervals it claims (accept
probability, or the CDF of a draw). Each interval is then *checked* by running
the oracle with a uniform inside it (and just inside both of its ends) and
observing the outcome, so the law recorded is the law the oracle actually
implements; the search recurses with the interval's length as the branch
weight. Leaves carry the exact probability of each output.
"""
from __future__ import annotations

from collections import defaultdict

import numpy as np
import scipy.special

from oracle.verify import inverse_cdf, softmax


class Script:
    """Uniforms handed out in request order: fixed prefix, then 0.5."""

    def __init__(self, values):
        self.values = list(values)
        self.n = 0

    def next(self):
        v = self.values[self.n] if self.n < len(self.values) else 0.5
        self.n += 1
        return v


class ScriptedSource:
    """Adapter with the oracle's uniform-source interface."""

    def __init__(self, script: Script):
        self.script = script

    def accept(self, pos):
        return self.script.next()

    def sample(self, pos):
        return self.script.next()


class DraftDecision:
    """Trace entry of a draft drawn by the harness from the draft law."""

    def __init__(self, u, token, cdf):
        self.kind, self.u, self.outcome, self.law = "sample", u, token, cdf


def draw_draft(script: Script, logits, T):
    """Harness draft sampler: inverse CDF of softmax(l / T) (argmax at T=0)."""
    if T == 0.0:
        return int(np.argmax(logits)), None
    q = softmax(logits, T)
    u = script.next()
    tok, _ = inverse_cdf(q, u)
    c = np.cumsum(q)
    return tok, DraftDecision(u, tok, c / c[-1])


def _intervals(dec):
    """Outcome intervals (outcome, lo, hi) a decision claims."""
    if dec.kind == "accept":
        P = float(dec.law)
        out = []
        if P > 0:
            out.append((1, 0.0, P))
        if P < 1:
            out.append((0, P, 1.0))
        return out
    cdf = np.asarray(dec.law, dtype=np.float64)
    out, lo = [], 0.0
    for v, hi in enumerate(cdf):
        hi = min(float(hi), 1.0)
        if hi > lo:
            out.append((v, lo, hi))
        lo = max(lo, hi)
    return out


def enumerate_law(run, probe_edges=True, max_nodes=2_000_000):
    """Enumerate every output of ``run`` with its exact probability.

    ``run(script) -> (output, trace)``; ``trace`` lists decision objects with
    ``kind``, ``outcome`` and ``law`` in the order the uniforms were drawn.
    Returns {output: probability}.
    """
    law = defaultdict(float)
    nodes = [0]

    def outcome_at(prefix, d):
        _, tr = run(Script(prefix))
        return tr[d].outcome

    def dfs(prefix, weight):
        nodes[0] += 1
        if nodes[0] > max_nodes:
            raise RuntimeError("enumeration too large")
        out, trace = run(Script(prefix))
        d = len(prefix)
        if len(trace) <= d:
            law[out] += weight
            return
        for outcome, lo, hi in _intervals(trace[d]):
            rep = 0.5 * (lo + hi)
            got = outcome_at(prefix + [rep], d)
            assert got == outcome, f"decision {d}: claimed {outcome}, oracle did {got}"
            eps = max(1e-9 * (hi - lo), 1e-13)
            if probe_edges and hi - lo > 4 * eps:
                assert outcome_at(prefix + [lo + eps], d) == outcome
                assert outcome_at(prefix + [hi - eps], d) == outcome
            dfs(prefix + [rep], weight * (hi - lo))

    dfs([], 1.0)
    return dict(law)


def conditional_laws(law):
    """From {token tuple: prob} build {prefix: {token: P(c_m=token, m emitted
    | c_<m = prefix)}} normalised over the tokens emitted at m."""
    joint = defaultdict(lambda: defaultdict(float))
    for toks, p in law.items():
        for m in range(len(toks)):
            joint[tuple(toks[:m])][toks[m]] += p
    cond = {}
    for prefix, row in joint.items():
        tot = sum(row.values())
        cond[prefix] = {v: x / tot for v, x in row.items()}
    return cond


def target_law(logits, T):
    """Reference law of a slot: scipy's softmax of l / T (argmax at T=0)."""
    logits = np.asarray(logits, dtype=np.float64)
    if T == 0.0:
        e = np.zeros_like(logits)
        e[int(np.argmax(logits))] = 1.0
        return e
    return scipy.special.softmax(logits / T)


def max_law_error(law, slot_logits, T, slot_of=lambda prefix: len(prefix)):
    """Largest |P(c_m = v | prefix) - target_m(v)| over all prefixes and v."""
    worst = 0.0
    for prefix, row in conditional_laws(law).items():
        ref = target_law(slot_logits[slot_of(prefix)], T)
        for v in range(len(ref)):
            worst = max(worst, abs(row.get(v, 0.0) - ref[v]))
    return worst
