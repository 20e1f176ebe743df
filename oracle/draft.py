"""Plain fp64 draft step (the oracle): the token the drafting exit proposes at
one position, and the entropy of its distribution.

TEST INFRASTRUCTURE ONLY. Only ``tests/``, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` may import this
module. It shares no code with the CUDA path.

What it follows
---------------
* HiSpec: Hierarchical Speculative Decoding for LLMs (gist.science summary of
  arXiv 2510.01336), section 2 "Kernmechanismus": the shallow exit L_d drafts
  the tokens that the intermediate and final exits then check; each draft is a
  draw from the exit's token distribution softmax(l_d / T).
* Optimierung der Inferenzgeschwindigkeit von Sprachmodellen durch
  spekulative Dekodierung (mind-verse.de), paragraphs on SVIP: the entropy of
  the draft-token distribution is the uncertainty signal from which the draft
  length is chosen. The entropy computed here is the Shannon entropy, in nats,
  of that distribution.

Readings taken where the pages are silent
-----------------------------------------
* The draft draw is inverse-CDF sampling from softmax(l_d / T) with the lane-1
  uniform of the Philox counter (seq_id, round, pos, stage 0 = draft), pos
  being the slot the drafted token will occupy; T == 0 drafts the argmax
  (smallest id on ties).
* For T == 0 the draft distribution is the point mass on the argmax: its
  entropy is 0 and ln q(token) is 0.
* Masked entries (logit -inf) have probability 0 and contribute 0 to the
  entropy (0 * ln 0 = 0).
"""
from __future__ import annotations

from dataclasses import dataclass

import numpy as np

from .philox import STAGE_DRAFT, uniforms
from .verify import argmax_first, inverse_cdf, softmax


def entropy(logits, T: float) -> float:
    """Shannon entropy -sum_v p_v ln p_v of p = softmax(l / T), in nats; 0 for
    T == 0. Terms with p_v == 0 contribute 0."""
    if T == 0.0:
        return 0.0
    p = softmax(logits, T)
    nz = p > 0.0
    return float(-np.sum(p[nz] * np.log(p[nz])))


@dataclass
class DraftResult:
    token: int
    logq: float      # ln q(token)
    entropy: float   # nats
    margin: float    # fp64 distance of u to the chosen token's CDF boundary (inf for greedy)


def draft_sample(logits, T: float, u: float) -> DraftResult:
    """One draft token from the row ``logits`` at temperature T with uniform u
    (inverse CDF over softmax(l / T)); T == 0 takes the argmax."""
    if T == 0.0:
        return DraftResult(argmax_first(logits), 0.0, 0.0, float("inf"))
    p = softmax(logits, T)
    tok, margin = inverse_cdf(p, u)
    return DraftResult(tok, float(np.log(p[tok])), entropy(logits, T), margin)


def draft_step(logits, temperature, seed: int, seq_id, rnd: int, pos):
    """Draft tokens of a batch of rows.

    logits [B, V], temperature [B], seq_id [B], pos [B]: row b drafts the token
    of slot pos[b] of sequence seq_id[b] in round ``rnd``. Returns a list of
    DraftResult.
    """
    logits = np.asarray(logits)
    out = []
    for b in range(logits.shape[0]):
        _, u = uniforms(seed, int(seq_id[b]), rnd, int(pos[b]), STAGE_DRAFT)
        out.append(draft_sample(logits[b], float(temperature[b]), u))
    return out
