"""Pins of the oracle's paged commit / rollback and hidden-row packing.

HiSpec (gist.science summary of arXiv 2510.01336), section 2, bullets on KV
and hidden-state reuse (buffer while drafting, drop the entries of rejected
tokens before the next phase) and on batch inference with paged attention and
block tables. Pinned by a hand-worked example, by the block-table invariants
(no block leaked or duplicated, len' = base + keep, table covers
ceil(len'/bs) blocks) on random tiny pools, and by brute force against a
list-of-blocks model that tracks which block holds which token position.
"""
import json
import os

import numpy as np
import pytest

from oracle.commit import (STATUS_EINVAL, STATUS_ENOBLOCKS, STATUS_OK,
                           blocks_for, check_invariants, commit_paged,
                           gather_hidden, scatter_kv)

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "commit_small.json")


def test_hand_worked_example():
    g = json.load(open(GOLDEN))
    r = commit_paged(g["tables"], g["seq_lens"], g["base_len"], g["keep"],
                     g["free_stack"], g["free_top"], g["block_size"],
                     g["num_blocks"], g["kp1"])
    assert r.status == STATUS_OK
    bs = g["block_size"]
    for b, want in enumerate(g["expect_tables"]):
        nb = blocks_for(g["expect_seq_lens"][b], bs)
        assert list(r.tables[b, :nb]) == want[:nb]
    assert list(r.seq_lens) == g["expect_seq_lens"]
    assert list(r.free_stack[:r.free_top]) == g["expect_free_stack_top"]
    assert [list(d) for d in r.destinations] == g["expect_destinations"]
    assert list(r.hid_off) == g["expect_hid_off"]


def _random_state(rng, B, bs, num_blocks, max_blocks, kp1):
    """Random valid state: blocks dealt to tables, the rest on the stack."""
    perm = list(rng.permutation(num_blocks))
    tables = -np.ones((B, max_blocks), np.int64)
    lens = np.zeros(B, np.int64)
    for b in range(B):
        n = int(rng.integers(0, min(max_blocks - 1, 3) * bs + 1))
        nb = blocks_for(n, bs)
        if nb > len(perm):
            n, nb = 0, 0
        for i in range(nb):
            tables[b, i] = perm.pop()
        lens[b] = n
    stack = -np.ones(num_blocks, np.int64)
    stack[:len(perm)] = perm
    return tables, lens, stack, len(perm)


class ListModel:
    """Brute-force model: per sequence an explicit list of (block, slot) for
    every token position, and a Python list as the free stack."""

    def __init__(self, tables, lens, stack, top, bs):
        self.bs = bs
        self.blocks = [[int(tables[b, i]) for i in range(blocks_for(int(n), bs))]
                       for b, n in enumerate(lens)]
        self.lens = [int(n) for n in lens]
        self.stack = [int(x) for x in stack[:top]]

    def commit(self, base, keep):
        new = [int(base[b]) + int(keep[b]) for b in range(len(base))]
        for b in range(len(base)):           # shrink first, in order
            while len(self.blocks[b]) > blocks_for(new[b], self.bs):
                tail = len(self.blocks[b]) - blocks_for(new[b], self.bs)
                # the tail is pushed in ascending index order
                self.stack.append(self.blocks[b][-tail])
                del self.blocks[b][-tail]
        for b in range(len(base)):           # then grow, in order
            while len(self.blocks[b]) < blocks_for(new[b], self.bs):
                self.blocks[b].append(self.stack.pop())
        self.lens = new
        return [(b, i, self.blocks[b][(int(base[b]) + i) // self.bs],
                 (int(base[b]) + i) % self.bs)
                for b in range(len(base)) for i in range(int(keep[b]))]


@pytest.mark.parametrize("trial", range(60))
def test_random_tiny_pools_against_list_model(trial):
    rng = np.random.default_rng(1000 + trial)
    B, bs, kp1 = int(rng.integers(1, 6)), int(rng.choice([1, 2, 4, 16])), 5
    num_blocks = int(rng.integers(8, 33))
    max_blocks = 6
    tables, lens, stack, top = _random_state(rng, B, bs, num_blocks,
                                             max_blocks, kp1)
    model = ListModel(tables, lens, stack, top, bs)
    for _ in range(6):
        base = np.array([int(rng.integers(0, n + 1)) for n in model.lens])
        keep = rng.integers(0, kp1 + 1, size=B)
        need = sum(max(0, blocks_for(int(base[b] + keep[b]), bs) -
                       len(model.blocks[b])) for b in range(B))
        r = commit_paged(tables, lens, base, keep, stack, top, bs,
                         num_blocks, kp1)
        over = any(blocks_for(int(base[b] + keep[b]), bs) > max_blocks
                   for b in range(B))
        frees = sum(max(0, len(model.blocks[b]) -
                        blocks_for(int(base[b] + keep[b]), bs)) for b in range(B))
        if over:
            assert r.status == STATUS_EINVAL
            continue
        if len(model.stack) + frees < need:
            assert r.status == STATUS_ENOBLOCKS
            assert np.array_equal(r.tables, tables) and r.free_top == top
            continue
        assert r.status == STATUS_OK
        dest = model.commit(base, keep)
        assert r.destinations == dest
        assert list(r.seq_lens) == model.lens
        assert list(r.seq_lens) == [int(base[b] + keep[b]) for b in range(B)]
        for b in range(B):
            nb = blocks_for(model.lens[b], bs)
            assert list(r.tables[b, :nb]) == model.blocks[b]
        assert list(r.free_stack[:r.free_top]) == model.stack
        assert check_invariants(r.tables, r.seq_lens, r.free_stack,
                                r.free_top, bs, num_blocks) == []
        tables, lens, stack, top = r.tables, r.seq_lens, r.free_stack, r.free_top


def test_failures_change_nothing():
    g = json.load(open(GOLDEN))
    args = dict(tables=g["tables"], seq_lens=g["seq_lens"],
                free_stack=g["free_stack"], free_top=g["free_top"],
                block_size=g["block_size"], num_blocks=g["num_blocks"],
                kp1=g["kp1"])
    bad = [
        ([5, 6, 3], [6, 1, 5], STATUS_EINVAL),      # keep > K+1
        ([6, 6, 3], [4, 1, 5], STATUS_EINVAL),      # base beyond length
        ([5, 6, 3], [-1, 1, 5], STATUS_EINVAL),     # negative keep
    ]
    for base, keep, want in bad:
        r = commit_paged(base_len=base, keep=keep, **args)
        assert r.status == want
        assert np.array_equal(r.tables, np.array(g["tables"]))
        assert list(r.seq_lens) == g["seq_lens"] and r.free_top == g["free_top"]
    # two allocations needed, one free block and nothing freed: exhausted
    tight = dict(args, free_top=1)
    r = commit_paged(base_len=[5, 12, 3], keep=[4, 0, 5], **tight)
    assert r.status == STATUS_ENOBLOCKS
    assert np.array_equal(r.tables, np.array(g["tables"])) and r.free_top == 1
    bad_table = dict(args, tables=[[0, 11, -1, -1], [2, 3, 4, -1], [5, -1, -1, -1]])
    r = commit_paged(base_len=[5, 6, 3], keep=[1, 1, 1], **bad_table)
    assert r.status == STATUS_EINVAL


def test_kv_scatter_and_hidden_gather_roundtrip():
    g = json.load(open(GOLDEN))
    r = commit_paged(g["tables"], g["seq_lens"], g["base_len"], g["keep"],
                     g["free_stack"], g["free_top"], g["block_size"],
                     g["num_blocks"], g["kp1"])
    L, H, D, bs = 2, 3, 4, g["block_size"]
    B, kp1 = 3, g["kp1"]
    rng = np.random.default_rng(0)
    stage = rng.integers(0, 2**16, size=(B, kp1, L, 2, H, D)).astype(np.uint16)
    pool = np.zeros((g["num_blocks"], L, 2, bs, H, D), np.uint16)
    scatter_kv(pool, stage, r.destinations)
    for b in range(B):
        for i in range(g["keep"][b]):
            pos = g["base_len"][b] + i
            blk = r.tables[b, pos // bs]
            assert np.array_equal(pool[blk, :, :, pos % bs], stage[b, i])
    hid = rng.normal(size=(B, kp1, 8))
    packed = gather_hidden(hid, g["keep"])
    assert packed.shape == (sum(g["keep"]), 8)
    for b in range(B):
        o = r.hid_off[b]
        assert np.array_equal(packed[o:o + g["keep"][b]], hid[b, :g["keep"][b]])


def test_invariant_checker_detects_leaks_and_duplicates():
    tables = np.array([[0, 1], [1, -1]])
    errs = check_invariants(tables, [8, 4], np.array([2, 3]), 1, 4, 4)
    assert any("duplicated" in e for e in errs)
    assert any("leaked" in e for e in errs)
