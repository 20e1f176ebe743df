"""Comparison of CUDA-path outputs with the oracle, with the acceptance rule:

* accepted counts and emitted tokens bit-exact, except at decisions whose
  fp64 oracle margin is below 1e-6 (counted; their share of all decisions
  must stay below 1e-4);
* probabilities (row log-partitions, p_j(x_j), q_j(x_j), residual mass Z)
  within 1e-5 relative.
"""
from __future__ import annotations

import math

import numpy as np

MARGIN = 1e-6
PROB_RTOL = 1e-5


class Tally:
    def __init__(self):
        self.decisions = 0
        self.excused = 0
        self.details = []

    def check_share(self):
        print(f"decisions compared: {self.decisions}, excused near-margin: {self.excused}")
        assert self.excused <= 1e-4 * max(self.decisions, 1) or self.excused == 0, \
            f"{self.excused} near-margin decisions of {self.decisions}: {self.details[:5]}"


def compare_check(tag, res, a_gpu, toks_gpu, tally: Tally):
    """Compare one speculative check (oracle ``CheckResult``) with the GPU's
    accepted count and emitted tokens. Returns True if they agree exactly,
    False if they diverge at an excused near-margin decision; raises
    otherwise."""
    tally.decisions += len(res.decisions)
    if a_gpu == res.accepted and list(toks_gpu) == list(res.tokens):
        return True
    # Locate the first decision where the outcomes differ.
    for d in res.decisions:
        if d.kind == "accept":
            j = d.pos - (res.decisions[0].pos if res.decisions else 0)
            gpu_acc = int(a_gpu > j)
            if gpu_acc != d.outcome:
                break
        else:
            if toks_gpu[-1] != d.outcome:
                break
    else:
        raise AssertionError(f"{tag}: outputs differ without a differing decision: "
                             f"gpu a={a_gpu} {list(toks_gpu)} oracle a={res.accepted} {res.tokens}")
    if d.margin < MARGIN:
        tally.excused += 1
        tally.details.append((tag, d.kind, d.pos, d.margin))
        return False
    raise AssertionError(
        f"{tag}: {d.kind} decision at pos {d.pos} differs with margin {d.margin:.3g} "
        f"(u={d.u!r}); gpu a={a_gpu} {list(toks_gpu)} oracle a={res.accepted} {res.tokens}")


def close(a, b, rtol=PROB_RTOL, floor=0.0):
    if math.isnan(a) or math.isnan(b):
        return math.isnan(a) and math.isnan(b)
    return abs(a - b) <= rtol * max(abs(b), floor)


def compare_probs(tag, res, diag_row, K, T):
    """Chain diagnostic layout: lse target [K+1], lse draft [K], p [K], q [K], Z."""
    if T == 0.0:
        assert np.all(np.isnan(diag_row)), f"{tag}: greedy diag must be NaN"
        return
    lt = diag_row[0:K + 1]
    ld = diag_row[K + 1:2 * K + 1]
    p = diag_row[2 * K + 1:3 * K + 1]
    q = diag_row[3 * K + 1:4 * K + 1]
    Z = diag_row[4 * K + 1]
    for j in range(K + 1):
        assert close(lt[j], res.lse_target[j], floor=1.0), (tag, "lse_t", j, lt[j], res.lse_target[j])
    for j in range(K):
        assert close(ld[j], res.lse_draft[j], floor=1.0), (tag, "lse_d", j, ld[j], res.lse_draft[j])
        if res.p_draft_tok[j] > 1e-290:
            assert close(p[j], res.p_draft_tok[j]), (tag, "p", j, p[j], res.p_draft_tok[j])
        if res.q_draft_tok[j] > 1e-290:
            assert close(q[j], res.q_draft_tok[j]), (tag, "q", j, q[j], res.q_draft_tok[j])
    assert close(Z, res.residual_mass), (tag, "Z", Z, res.residual_mass)
