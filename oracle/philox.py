"""Philox4x32-10 counter-based generator and the uniform map, for the oracle.

TEST INFRASTRUCTURE ONLY. Nothing under ``oracle/`` is part of the product: only
``tests/``, ``__graft_entry__.smoke()`` and the ``cpu_baseline`` / ``--impl
reference`` legs of ``bench.py`` may import it. It shares no code with the CUDA
path; the device generator is a separate implementation of the same published
definition.

Definition followed: J. K. Salmon, M. A. Moraes, R. O. Dror, D. E. Shaw,
"Parallel Random Numbers: As Easy as 1, 2, 3", SC'11, section 3.2 (the Philox
S-P network) with the 4x32 multipliers and Weyl key increments of its table 2,
ten rounds. Pinned by the Random123 known-answer vectors in
``tests/golden/philox4x32_10_kat.txt``.

How the method uses it (the pages name no generator; this is the reading the
whole build uses): key = (seed & 0xffffffff, seed >> 32); counter =
(sequence id, round, position, stage); lane 0 of the output block is the
uniform of the accept test, lane 1 the uniform of the residual / bonus draw.
Stage tags: 0 = draft sampling, 1 = chain verification or the first
(intermediate-exit) stage, 2 = the second (final-layer) stage.

The uniform map is u = (2 * (x >> 9) + 1) * 2**-24: an odd multiple of 2**-24
in the open interval (0, 1), exact in both fp32 and fp64.
"""
from __future__ import annotations

import numpy as np

MASK32 = 0xFFFFFFFF
# Round multipliers and key increments for Philox4x32 (SC'11, table 2).
PHILOX_M0 = 0xD2511F53
PHILOX_M1 = 0xCD9E8D57
PHILOX_W0 = 0x9E3779B9  # golden ratio
PHILOX_W1 = 0xBB67AE85  # sqrt(3) - 1

STAGE_DRAFT = 0
STAGE_ONE = 1   # chain verification and the first stage of the hierarchy
STAGE_TWO = 2   # second stage (final layer over the window)


def _round(c0, c1, c2, c3, k0, k1):
    """One Philox S-P round on uint64 numpy arrays holding 32-bit values."""
    p0 = PHILOX_M0 * c0          # full 64-bit product (fits: 32 x 32 bits)
    p1 = PHILOX_M1 * c2
    hi0, lo0 = p0 >> 32, p0 & MASK32
    hi1, lo1 = p1 >> 32, p1 & MASK32
    return (hi1 ^ c1 ^ k0, lo1, hi0 ^ c3 ^ k1, lo0)


def philox4x32_10(ctr, key):
    """Philox4x32 with ten rounds.

    ``ctr`` is a sequence of four counter words and ``key`` of two key words;
    each word may be a Python int or a numpy integer array (broadcast
    together). Returns a tuple of four uint64 arrays holding 32-bit results.
    """
    c = [np.asarray(x, dtype=np.uint64) & np.uint64(MASK32) for x in ctr]
    k0 = np.asarray(key[0], dtype=np.uint64) & np.uint64(MASK32)
    k1 = np.asarray(key[1], dtype=np.uint64) & np.uint64(MASK32)
    c0, c1, c2, c3 = np.broadcast_arrays(*c)
    for r in range(10):
        if r > 0:  # the key is bumped between rounds
            k0 = (k0 + np.uint64(PHILOX_W0)) & np.uint64(MASK32)
            k1 = (k1 + np.uint64(PHILOX_W1)) & np.uint64(MASK32)
        c0, c1, c2, c3 = _round(c0, c1, c2, c3, k0, k1)
    return c0, c1, c2, c3


def to_uniform(x):
    """Map a 32-bit word to an odd multiple of 2**-24 in (0, 1), as float64."""
    x = np.asarray(x, dtype=np.uint64)
    return (2.0 * (x >> np.uint64(9)).astype(np.float64) + 1.0) * 2.0 ** -24


def seed_key(seed: int):
    seed = int(seed) & 0xFFFFFFFFFFFFFFFF
    return (seed & MASK32, seed >> 32)


def uniforms(seed: int, seq_id, rnd, pos, stage):
    """The two uniforms (accept, sample) of counter (seq_id, rnd, pos, stage).

    Arguments other than ``seed`` may be ints or integer arrays. Returns
    ``(u_accept, u_sample)`` as float64 scalars or arrays.
    """
    out = philox4x32_10((seq_id, rnd, pos, stage), seed_key(seed))
    u0 = to_uniform(out[0])
    u1 = to_uniform(out[1])
    if u0.ndim == 0:
        return float(u0), float(u1)
    return u0, u1


class PhiloxUniforms:
    """Uniform source used by the oracle's verification routines.

    ``accept(pos)`` and ``sample(pos)`` return lane 0 / lane 1 of the counter
    (seq_id, rnd, pos, stage). Tests substitute other sources with the same
    two methods to inject chosen uniforms.
    """

    def __init__(self, seed: int, seq_id: int, rnd: int, stage: int):
        self.seed, self.seq_id, self.rnd, self.stage = seed, seq_id, rnd, stage

    def accept(self, pos: int) -> float:
        return uniforms(self.seed, self.seq_id, self.rnd, pos, self.stage)[0]

    def sample(self, pos: int) -> float:
        return uniforms(self.seed, self.seq_id, self.rnd, pos, self.stage)[1]
