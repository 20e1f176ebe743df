"""Plain fp64 law of a verification's outcome (the oracle), for outcome
prediction.

TEST INFRASTRUCTURE ONLY. Only ``tests/``, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` may import this
module. It shares no code with the CUDA path.

What it follows
---------------
* Speculative Speculative Decoding (gist.science summary of arXiv
  2603.03251), "Technische Zusammenfassung" section 2 items 1-2: while the
  target verifies, the outcomes of that verification -- how many tokens are
  accepted and which bonus token is drawn -- are predicted, and continuations
  are prepared for the likely ones in a speculation cache; section 3.A: under
  a budget, more predictions go to short acceptance lengths, whose
  probability decays geometrically; section 3.B: the token drawn after a
  rejection follows the residual distribution, proportional to the
  target-minus-draft difference.

Readings taken where the pages are silent
-----------------------------------------
* The outcome of one chain check with the drafts x_0..x_{K-1} already drawn is
  (a, v): a accepted drafts, then token v. With beta_j = min(1, p_j(x_j) /
  q_j(x_j)) its law is P(a = k) = beta_0 ... beta_{k-1} (1 - beta_k) for
  k < K and beta_0 ... beta_{K-1} for k = K; given a = k the token follows
  r_k = normalize(max(0, p_k - q_k)) (p_k where that mass is zero) for k < K
  and r_K = p_K. At T == 0, beta_j = [x_j == argmax p_j] and r_k is the point
  mass on argmax p_k.
* A budget of n cached outcomes covers the n most likely pairs (k, v) by
  P(a = k) r_k(v) (ties in (k, v) order): the allocation that maximises the
  probability of a hit. How many of them fall on each k is the fan-out; it
  decays with k as P(a = k) does.
"""
from __future__ import annotations

from dataclasses import dataclass
from typing import List, Tuple

import numpy as np

from .verify import argmax_first, softmax


@dataclass
class OutcomeLaw:
    p_len: np.ndarray    # [K+1] P(a = k)
    beta: np.ndarray     # [K] accept probability of each fixed draft
    resid: np.ndarray    # [K+1, V] r_k
    mass: np.ndarray     # [K+1] residual mass sum max(0, p_k - q_k) (k < K); 1 for k = K


def outcome_law(tgt_rows, drf_rows, drafts, T: float) -> OutcomeLaw:
    """Law of (a, token) of one chain check of the drafts against target rows
    tgt_rows [K+1, V] with draft rows drf_rows [K, V] at temperature T."""
    tgt_rows = np.asarray(tgt_rows)
    drf_rows = np.asarray(drf_rows)
    K = len(drafts)
    V = tgt_rows.shape[1]
    beta = np.zeros(K)
    resid = np.zeros((K + 1, V))
    mass = np.ones(K + 1)
    for j in range(K + 1):
        if T == 0.0:
            top = argmax_first(tgt_rows[j])
            resid[j, top] = 1.0
            if j < K:
                beta[j] = 1.0 if int(drafts[j]) == top else 0.0
            continue
        p = softmax(tgt_rows[j], T)
        if j == K:
            resid[j] = p
            continue
        q = softmax(drf_rows[j], T)
        x = int(drafts[j])
        beta[j] = min(1.0, p[x] / q[x]) if q[x] > 0 else 1.0
        w = np.maximum(p - q, 0.0)
        mass[j] = float(np.sum(w))
        resid[j] = w / mass[j] if mass[j] > 0 else p
    p_len = np.zeros(K + 1)
    run = 1.0
    for k in range(K):
        p_len[k] = run * (1.0 - beta[k])
        run *= beta[k]
    p_len[K] = run
    return OutcomeLaw(p_len, beta, resid, mass)


def top_outcomes(law: OutcomeLaw, n: int) -> List[Tuple[int, int, float]]:
    """The n most likely outcomes (k, v, P(a = k) r_k(v)), most likely first,
    ties in (k, v) order; outcomes of probability 0 are left out."""
    joint = law.p_len[:, None] * law.resid
    K1, V = joint.shape
    flat = joint.ravel()
    order = np.lexsort((np.arange(K1 * V), -flat))  # by -prob, then by index
    out = []
    for i in order[:n]:
        if flat[i] <= 0.0:
            break
        out.append((int(i // V), int(i % V), float(flat[i])))
    return out


def fan_out(top: List[Tuple[int, int, float]], K: int) -> np.ndarray:
    """How many of the cached outcomes fall on each acceptance length."""
    f = np.zeros(K + 1, dtype=np.int64)
    for k, _, _ in top:
        f[k] += 1
    return f
