"""Plain fp64 single-threaded speculative-sampling verification (the oracle).

TEST INFRASTRUCTURE ONLY. Only ``tests/``, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` may import this
module. It shares no code with the CUDA path.

What it follows
---------------
* HiSpec: Hierarchical Speculative Decoding for LLMs (gist.science summary of
  arXiv 2510.01336), section 2 "Methodik", bullet "Verlustfreie Garantie": the
  lossless speculative-decoding argument is applied once per stage, first with
  the intermediate exit L_i as target for drafts from the shallow exit L_d,
  then with the final layer L_f as target over the window of tentatively
  accepted tokens; the intermediate stage only rejects early.
* Same page, section 2, bullet "Dynamische Verifizierungsrichtlinie": a window
  of N_i (default 4) tentatively accepted tokens is gathered before the full
  check.
* Speculative Speculative Decoding (gist.science summary of arXiv 2603.03251),
  "Technische Zusammenfassung" section 2 item 1 (a verification outcome is the
  number of accepted tokens plus one bonus token) and section 3.B (the
  residual distribution is proportional to the target-minus-draft difference).

The pages print no formula. The rules written out below are the standard
speculative-sampling rules those passages appeal to: accept draft x with
probability min(1, p(x)/q(x)); at the first rejection draw from
normalize(max(0, p - q)); if every draft is accepted draw a bonus token from
the target row after the last draft; at temperature 0 accept iff the draft is
the target argmax and emit the target argmax.

Readings taken where the pages are silent
-----------------------------------------
* p = softmax(l / T) of a row of logits l, T > 0; the same T for every exit of
  a sequence. T == 0 is the greedy path; argmax ties go to the smallest id.
* The accept test is ``u * q(x) < p(x)`` with u the lane-0 uniform of the
  position's counter (strict, so a ratio >= 1 always accepts).
* Inverse CDF: the token drawn from weights w with uniform u is the smallest v
  with sum_{t<=v} w_t > u * sum_t w_t.
* If the residual mass is zero (p == q as computed) the draw falls back to p.
* Stage two uses, as its draft law at window slot s, softmax(l_i(s) / T) --
  the law every stage-one output at that slot follows -- so the second stage
  is again plain speculative sampling.
* Window: every stage-one output (accepted drafts and the resampled or bonus
  token) enters the window; the second stage fires after a round that leaves
  at least N_i tokens in it; its bonus row is the final-layer row at slot |W|;
  a2 + 1 tokens are committed and the window is emptied. Logit rows are
  indexed by slot since the last commit.
"""
from __future__ import annotations

from dataclasses import dataclass, field
from typing import List, Optional

import numpy as np

from .philox import PhiloxUniforms, STAGE_ONE, STAGE_TWO


# ----------------------------------------------------------------------------
# Row laws
# ----------------------------------------------------------------------------

def softmax(logits, T: float) -> np.ndarray:
    """softmax(l / T) in fp64: subtract the max of l / T, exponentiate, divide
    by the sum. ``T`` must be > 0."""
    z = np.asarray(logits, dtype=np.float64) / np.float64(T)
    e = np.exp(z - np.max(z))
    return e / np.sum(e)


def log_partition(logits, T: float) -> float:
    """ln sum_v exp(l_v / T), the row's log-sum-exp at temperature T."""
    z = np.asarray(logits, dtype=np.float64) / np.float64(T)
    m = np.max(z)
    return float(m + np.log(np.sum(np.exp(z - m))))


def argmax_first(logits) -> int:
    """Index of the largest logit; the smallest index among ties."""
    return int(np.argmax(np.asarray(logits)))  # numpy returns the first maximum


def inverse_cdf(w: np.ndarray, u: float):
    """Draw from weights ``w`` (not necessarily normalised) with uniform u.

    Returns (token, margin): token = smallest v with C(v) > u * Z, where
    C = cumulative sum and Z = C[-1]; margin = distance of u to the nearest
    boundary C(token-1)/Z, C(token)/Z of the chosen token's interval.
    """
    c = np.cumsum(np.asarray(w, dtype=np.float64))
    z = c[-1]
    target = u * z
    v = int(np.searchsorted(c, target, side="right"))
    if v >= len(c):  # only reachable through rounding when u*Z == Z
        v = int(np.nonzero(w > 0)[0][-1])
    lo = c[v - 1] / z if v > 0 else 0.0
    hi = c[v] / z
    return v, float(min(u - lo, hi - u))


# ----------------------------------------------------------------------------
# One speculative-sampling check (one stage)
# ----------------------------------------------------------------------------

@dataclass
class Decision:
    kind: str            # "accept" or "sample"
    pos: int             # counter position of the uniform
    u: float
    margin: float        # fp64 distance of u to the decision boundary
    outcome: int         # 1/0 for accept, token id for sample
    law: object = None   # accept: min(1, p/q); sample: normalised CDF array


@dataclass
class CheckResult:
    accepted: int                    # a: leading drafts accepted, 0..n
    tokens: List[int]                # drafts[:a] + [resampled / bonus token]
    decisions: List[Decision] = field(default_factory=list)
    lse_target: List[float] = field(default_factory=list)  # per target row
    lse_draft: List[float] = field(default_factory=list)   # per draft row
    p_draft_tok: List[float] = field(default_factory=list) # p_j(x_j), all j
    q_draft_tok: List[float] = field(default_factory=list) # q_j(x_j), all j
    residual_mass: float = float("nan")  # Z of the final draw (1 for bonus)
    fell_back_to_p: bool = False


def speculative_check(target_rows, draft_laws, drafts, T: float, uni,
                      pos0: int = 0) -> CheckResult:
    """Verify ``n = len(drafts)`` drafts against ``n + 1`` target rows.

    target_rows : array [n+1, V] of target logits (row j is the law of slot j).
    draft_laws  : array [n, V] of draft logits (row j is the law x_j was drawn
                  from); unused when T == 0.
    drafts      : n token ids.
    uni         : uniform source with ``accept(pos)`` and ``sample(pos)``.
    pos0        : counter position of draft 0 (slot index for the hierarchy).

    Every position's p_j(x_j), q_j(x_j) and row log-partition are recorded (the
    CUDA path evaluates all positions in parallel); the decisions stop at the
    first rejection.
    """
    target_rows = np.asarray(target_rows)
    drafts = [int(x) for x in drafts]
    n = len(drafts)
    res = CheckResult(accepted=n, tokens=[])

    if T == 0.0:
        # Greedy: accept while the draft equals the target argmax; emit the
        # target argmax at the first mismatch (or after the last draft).
        a = n
        for j in range(n):
            if drafts[j] != argmax_first(target_rows[j]):
                a = j
                break
        res.accepted = a
        res.tokens = drafts[:a] + [argmax_first(target_rows[a])]
        return res

    draft_laws = np.asarray(draft_laws)
    p_rows = [softmax(target_rows[j], T) for j in range(n + 1)]
    q_rows = [softmax(draft_laws[j], T) for j in range(n)]
    res.lse_target = [log_partition(target_rows[j], T) for j in range(n + 1)]
    res.lse_draft = [log_partition(draft_laws[j], T) for j in range(n)]
    res.p_draft_tok = [float(p_rows[j][drafts[j]]) for j in range(n)]
    res.q_draft_tok = [float(q_rows[j][drafts[j]]) for j in range(n)]

    a = n
    for j in range(n):
        p, q = res.p_draft_tok[j], res.q_draft_tok[j]
        u = uni.accept(pos0 + j)
        ok = (u * q < p)
        ratio = (p / q) if q > 0 else float("inf")
        res.decisions.append(Decision("accept", pos0 + j, u, abs(u - ratio),
                                      int(ok), min(1.0, ratio)))
        if not ok:
            a = j
            break

    if a < n:
        w = np.maximum(0.0, p_rows[a] - q_rows[a])
        if not np.sum(w) > 0.0:       # p == q as computed: fall back to p
            w = p_rows[a]
            res.fell_back_to_p = True
    else:
        w = p_rows[n]                 # bonus token from the row after the drafts
    res.residual_mass = float(np.sum(w))
    u2 = uni.sample(pos0 + a)
    y, margin = inverse_cdf(w, u2)
    c = np.cumsum(w)
    res.decisions.append(Decision("sample", pos0 + a, u2, margin, y, c / c[-1]))
    res.accepted = a
    res.tokens = drafts[:a] + [y]
    return res


# ----------------------------------------------------------------------------
# Chain verification of a batch
# ----------------------------------------------------------------------------

def verify_chain(tgt, drf, drafts, temperature, seed, seq_id, rnd):
    """Chain verification of a batch, one sequence after another.

    tgt [B, K+1, V], drf [B, K, V] logits (any float dtype; read as fp64);
    drafts [B, K] ints; temperature [B]; seq_id [B]. Uniforms are Philox
    lanes of counter (seq_id[b], rnd, j, stage 1).
    Returns a list of ``CheckResult``, one per sequence.
    """
    out = []
    for b in range(len(drafts)):
        uni = PhiloxUniforms(seed, int(seq_id[b]), rnd, STAGE_ONE)
        out.append(speculative_check(tgt[b], drf[b], drafts[b],
                                     float(temperature[b]), uni))
    return out


# ----------------------------------------------------------------------------
# Two-stage (hierarchical) verification of one sequence
# ----------------------------------------------------------------------------

@dataclass
class HierResult:
    stage1: CheckResult
    stage2: Optional[CheckResult]   # None when the window did not fill
    window: List[int]               # window after this call (empty on commit)
    committed: List[int]            # tokens committed by this call


def verify_hier_seq(lg_d, lg_i, lg_f, drafts, T: float, window, n_i: int,
                    uni1, uni2) -> HierResult:
    """One round of the two-stage check for one sequence.

    lg_d, lg_i, lg_f : [S, V] slot-indexed logits of the three exits since the
                       last commit (S >= N_i + K + 1).
    drafts           : K drafts for slots w .. w+K-1, w = len(window).
    window           : tokens tentatively accepted so far in this cycle.
    uni1, uni2       : uniform sources of stage one and stage two.
    """
    w = len(window)
    k = len(drafts)
    lg_d, lg_i, lg_f = np.asarray(lg_d), np.asarray(lg_i), np.asarray(lg_f)
    # Stage one: L_i is the target of drafts from L_d, at slots w .. w+K.
    s1 = speculative_check(lg_i[w:w + k + 1], lg_d[w:w + k], drafts, T, uni1,
                           pos0=w)
    new_window = list(window) + s1.tokens
    if len(new_window) < n_i:
        return HierResult(s1, None, new_window, [])
    # Stage two: L_f is the target, the window tokens are the drafts and the
    # L_i law of each slot is their draft law.
    W = len(new_window)
    s2 = speculative_check(lg_f[0:W + 1], lg_i[0:W], new_window, T, uni2,
                           pos0=0)
    return HierResult(s1, s2, [], s2.tokens)


def verify_hier(lg_d, lg_i, lg_f, drafts, temperature, seed, seq_id, rnd,
                windows, n_i):
    """Batched two-stage round: ``windows`` is a list of per-sequence token
    lists (updated copies are returned inside the results)."""
    out = []
    for b in range(len(drafts)):
        u1 = PhiloxUniforms(seed, int(seq_id[b]), rnd, STAGE_ONE)
        u2 = PhiloxUniforms(seed, int(seq_id[b]), rnd, STAGE_TWO)
        out.append(verify_hier_seq(lg_d[b], lg_i[b], lg_f[b], drafts[b],
                                   float(temperature[b]), windows[b], n_i,
                                   u1, u2))
    return out
