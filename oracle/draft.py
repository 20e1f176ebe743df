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

* Speculative Speculative Decoding (gist.science summary of arXiv
  2603.03251), Technische Zusammenfassung 3.B (Saguaro sampling): the
  probabilities of the tokens held in the speculation cache are lowered a
  little in the draft, which raises the chance that the residual -- which is
  proportional to the target-minus-draft difference -- lands on them.

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
* Saguaro's lowering is the factor (1 - eps), eps in [0, 1), on the draft
  probability of every cached token, renormalised: q'(v) is proportional to
  q(v) (1 - eps [v cached]). On logits at temperature T > 0 this is the shift
  l(v) + T ln(1 - eps) of the cached tokens (a duplicate id counts once); a
  greedy row (T == 0) is unchanged. The draft draw and the check both use q'
  as the draft law, so the check stays lossless. Where the rows are stored in
  a narrower type the shifted logit is rounded to it, as the kernel stores
  it: the shift is formed as float32(T * ln(1 - eps)) and added in float32,
  then rounded (to nearest, ties to even) to bfloat16 for bfloat16 rows.
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


def round_bf16(x):
    """float32 values rounded to the nearest bfloat16 (ties to even), returned
    as float32: the upper 16 bits of the IEEE single after adding half of the
    dropped unit plus the parity of the kept one. NaN is kept as NaN."""
    x = np.asarray(x, dtype=np.float32)
    bits = x.view(np.uint32).astype(np.uint64)
    keep_odd = (bits >> 16) & 1
    r = ((bits + 0x7FFF + keep_odd) >> 16) << 16
    out = r.astype(np.uint32).view(np.float32)
    return np.where(np.isnan(x), x, out)


def saguaro_logits(logits, T: float, cached, eps: float, dtype: str = "f64"):
    """Draft logits with Saguaro's lowering of the cached tokens (see the
    readings above): every id in ``cached`` within [0, V) (duplicates once)
    gets T ln(1 - eps) added; T == 0 leaves the row as it is. ``dtype``
    "f64" keeps the exact shift; "f32" / "bf16" store it as the kernel does."""
    x = np.array(logits, dtype=np.float64, copy=True)
    V = x.shape[-1]
    ids = sorted({int(v) for v in np.asarray(cached).ravel() if 0 <= int(v) < V})
    if T == 0.0 or not ids:
        return x
    if dtype == "f64":
        x[..., ids] += T * np.log1p(-eps)
        return x
    d = np.float32(np.float64(T) * np.log1p(-np.float64(eps)))
    y = (x[..., ids].astype(np.float32) + d).astype(np.float32)
    if dtype == "bf16":
        y = round_bf16(y)
    x[..., ids] = y.astype(np.float64)
    return x

