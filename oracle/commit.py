"""Plain paged-KV commit / rollback and hidden-state pruning (the oracle).

TEST INFRASTRUCTURE ONLY. Only ``tests/``, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` may import this
module. It shares no code with the CUDA path.

What it follows
---------------
* HiSpec: Hierarchical Speculative Decoding for LLMs (gist.science summary of
  arXiv 2510.01336), section 2 bullet "Wiederverwendung von KV-Cache und
  versteckten Zustaenden": KV entries and hidden states are buffered during
  drafting and the entries of rejected tokens are removed before the next
  phase.
* Same page, section 2 bullet "Unterstuetzung fuer Batch-Inferenz": paged
  attention with block tables gives per-sequence acceptance without padding.

The pages give no data layout or allocation order. Readings used throughout:
* A sequence's block table covers ceil(len / block_size) blocks. A commit sets
  len' = base_len + keep (for chain verification keep = accepted + 1, so
  len' = previous + accepted + 1).
* Table entries at index >= ceil(len'/bs) that were covered before are freed;
  missing entries up to ceil(len'/bs) are allocated. All frees happen first,
  sequences in ascending order, each table's tail in ascending index, pushed
  on the free stack; then all allocations, sequences in ascending order,
  popped from the top of the stack.
* Staged KV rows 0..keep-1 of a sequence go to positions base_len.. of its
  paged cache; staged hidden rows 0..keep-1 are packed, sequence after
  sequence, into one [sum keep, hidden] array with offsets = exclusive scan
  of keep.
* Every check happens before any change: a call that fails leaves all state
  untouched.
"""
from __future__ import annotations

from dataclasses import dataclass
from typing import List, Tuple

import numpy as np

STATUS_OK = 0
STATUS_EINVAL = -1
STATUS_ENOBLOCKS = -4


def blocks_for(length: int, block_size: int) -> int:
    return (length + block_size - 1) // block_size


@dataclass
class CommitResult:
    status: int
    tables: np.ndarray          # [B, max_blocks] int64
    seq_lens: np.ndarray        # [B]
    free_stack: np.ndarray      # [num_blocks]
    free_top: int
    destinations: List[Tuple[int, int, int, int]]  # (b, i, block, slot)
    hid_off: np.ndarray         # [B + 1] exclusive scan of keep


def commit_paged(tables, seq_lens, base_len, keep, free_stack, free_top,
                 block_size, num_blocks, kp1):
    """Commit ``keep[b]`` staged tokens of every sequence at ``base_len[b]``.

    Inputs are not modified; the new state is returned. ``tables`` is
    [B, max_blocks]; entries past a table's covered length are ignored.
    """
    tables = np.array(tables, dtype=np.int64, copy=True)
    seq_lens = np.array(seq_lens, dtype=np.int64, copy=True)
    free_stack = np.array(free_stack, dtype=np.int64, copy=True)
    base_len = np.asarray(base_len, dtype=np.int64)
    keep = np.asarray(keep, dtype=np.int64)
    B, max_blocks = tables.shape
    unchanged = CommitResult(STATUS_OK, tables, seq_lens, free_stack,
                             int(free_top), [], np.zeros(B + 1, np.int64))

    # ---- checks (nothing changes if one fails) --------------------------
    new_len = base_len + keep
    old_nb = [blocks_for(int(n), block_size) for n in seq_lens]
    new_nb = [blocks_for(int(n), block_size) for n in new_len]
    bad = False
    for b in range(B):
        if not (0 <= keep[b] <= kp1):
            bad = True
        if not (0 <= base_len[b] <= seq_lens[b]):
            bad = True
        if old_nb[b] > max_blocks or new_nb[b] > max_blocks:
            bad = True
        elif any(not (0 <= tables[b, i] < num_blocks) for i in range(old_nb[b])):
            bad = True
    if not (0 <= free_top <= num_blocks):
        bad = True
    if bad:
        unchanged.status = STATUS_EINVAL
        return unchanged
    n_free = sum(max(0, old_nb[b] - new_nb[b]) for b in range(B))
    n_alloc = sum(max(0, new_nb[b] - old_nb[b]) for b in range(B))
    if free_top + n_free > num_blocks:
        unchanged.status = STATUS_EINVAL   # stack overflow: state is corrupt
        return unchanged
    if free_top + n_free < n_alloc:
        unchanged.status = STATUS_ENOBLOCKS
        return unchanged
    # Blocks handed out by the pops must be valid ids (pops read the freshly
    # pushed blocks first, then the stack below free_top).
    stack_after_push = list(free_stack[:free_top])
    for b in range(B):
        stack_after_push += [int(tables[b, i]) for i in range(new_nb[b], old_nb[b])]
    popped = stack_after_push[len(stack_after_push) - n_alloc:]
    if any(not (0 <= x < num_blocks) for x in popped):
        unchanged.status = STATUS_EINVAL
        return unchanged

    # ---- frees: sequences ascending, each tail ascending, pushed -------
    stack = list(free_stack[:free_top])
    for b in range(B):
        for i in range(new_nb[b], old_nb[b]):
            stack.append(int(tables[b, i]))
            tables[b, i] = -1
    # ---- allocations: sequences ascending, popped from the top ---------
    for b in range(B):
        for i in range(old_nb[b], new_nb[b]):
            tables[b, i] = stack.pop()
    top = len(stack)
    free_stack[:top] = stack
    seq_lens[:] = new_len

    # ---- destinations of the kept rows and hidden-row offsets ----------
    dest = []
    for b in range(B):
        for i in range(int(keep[b])):
            pos = int(base_len[b]) + i
            dest.append((b, i, int(tables[b, pos // block_size]), pos % block_size))
    hid_off = np.zeros(B + 1, np.int64)
    hid_off[1:] = np.cumsum(keep)
    return CommitResult(STATUS_OK, tables, seq_lens, free_stack, top, dest,
                        hid_off)


def scatter_kv(pool, kv_stage, destinations):
    """Copy staged token rows into the paged pool (in place).

    pool     : [num_blocks, layers, 2, block_size, heads, dim]
    kv_stage : [B, K+1, layers, 2, heads, dim]
    """
    for (b, i, blk, slot) in destinations:
        pool[blk, :, :, slot, :, :] = kv_stage[b, i]


def gather_hidden(hid_stage, keep):
    """Pack rows 0..keep[b]-1 of [B, K+1, hidden] into [sum keep, hidden]."""
    rows = [hid_stage[b, :int(keep[b])] for b in range(len(keep))]
    if not rows:
        return np.zeros((0, hid_stage.shape[-1]), hid_stage.dtype)
    return np.concatenate(rows, axis=0)


def check_invariants(tables, seq_lens, free_stack, free_top, block_size,
                     num_blocks):
    """Block-table invariants; returns a list of violations (empty if ok).

    Every block id is either in exactly one table (within its covered part) or
    in the free stack below ``free_top``; no id is missing or repeated.
    """
    errs = []
    seen = {}
    B = len(seq_lens)
    for b in range(B):
        nb = blocks_for(int(seq_lens[b]), block_size)
        if nb > tables.shape[1]:
            errs.append(f"seq {b}: table too short for length {seq_lens[b]}")
            continue
        for i in range(nb):
            x = int(tables[b, i])
            if not (0 <= x < num_blocks):
                errs.append(f"seq {b} entry {i}: id {x} out of range")
            elif x in seen:
                errs.append(f"block {x} duplicated ({seen[x]} and seq {b})")
            else:
                seen[x] = f"seq {b}"
    for k in range(int(free_top)):
        x = int(free_stack[k])
        if not (0 <= x < num_blocks):
            errs.append(f"free stack slot {k}: id {x} out of range")
        elif x in seen:
            errs.append(f"block {x} duplicated ({seen[x]} and free stack)")
        else:
            seen[x] = "free"
    if len(seen) != num_blocks:
        errs.append(f"{num_blocks - len(seen)} blocks leaked")
    return errs
