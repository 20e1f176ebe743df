"""Vocabulary-parallel chain verification, one process per GPU.

Rank r of R holds the columns [v0, v0 + Vs) of every target and draft row (the
output of a vocabulary-parallel LM head) and runs the library's three
vocabulary-parallel launches (include/spec_verify.h, spec_vp_*). Between them
go two all-gathers in rank order and one max-reduction, through
torch.distributed: NCCL over NVLink between GPUs, or gloo, which stages the
few bytes through host memory. This module only moves arguments and calls the
collectives; every step of the check runs in the library's kernels.

What crosses between ranks per sequence: 32 (2K+1) bytes of row records,
16 bytes of draw masses and 4 (K+1) bytes of tokens -- against the 2 (2K+1) Vs
bytes of logits each rank reads.
"""
from __future__ import annotations

import torch
import torch.distributed as dist

from . import capi

RESIDUAL_TILE = 256   # elements per residual tile of the draw


def vocab_shards(V, R, align=RESIDUAL_TILE):
    """R contiguous shards (v0, Vs) covering [0, V) in rank order. Every start
    is a multiple of ``align`` elements (whole residual tiles; 16-byte aligned
    row starts for both dtypes); the ceil(V / align) tiles are dealt out so
    that shard sizes differ by at most one tile (the last tile may be short).
    Raises ValueError if a shard would be empty."""
    if R < 1 or R > capi.VP_MAX_RANKS:
        raise ValueError(f"1 <= R <= {capi.VP_MAX_RANKS} shards")
    if align < 8 or align % 8:
        raise ValueError("shard starts must be multiples of 8 elements")
    tiles = -(-V // align)
    if tiles < R:
        raise ValueError(f"V={V} has {tiles} tiles of {align}: too few for {R} shards")
    out = []
    for r in range(R):
        v0 = min(V, r * tiles // R * align)
        v1 = min(V, (r + 1) * tiles // R * align)
        out.append((v0, v1 - v0))
    return out


class ChainShard:
    """One rank's workspace and exchange buffers for the vocabulary-parallel
    check of B sequences with K drafts over shard [v0, v0 + Vs) of [0, V)."""

    def __init__(self, B, K, V, v0, Vs, R, rank, dtype, device="cuda"):
        self.B, self.K, self.V, self.v0, self.Vs, self.R, self.rank = B, K, V, v0, Vs, R, rank
        n = capi.spec_vp_workspace_bytes(B, K, Vs, dtype)
        if n == 0:
            raise ValueError("invalid sizes")
        self.ws = torch.zeros(n, dtype=torch.uint8, device=device)
        per = 2 * K + 1
        u8 = dict(dtype=torch.uint8, device=device)
        self.rows = torch.zeros((B, per, capi.VP_ROW_BYTES), **u8)
        self.rows_all = torch.zeros((R, B, per, capi.VP_ROW_BYTES), **u8)
        self.mass = torch.zeros((B, capi.VP_MASS_BYTES), **u8)
        self.mass_all = torch.zeros((R, B, capi.VP_MASS_BYTES), **u8)

    def _check(self, tgt):
        B, Kp1, Vs = tgt.shape
        if (B, Kp1 - 1, Vs) != (self.B, self.K, self.Vs):
            raise ValueError(f"shard rows {tuple(tgt.shape)} do not match "
                             f"B={self.B}, K={self.K}, Vs={self.Vs}")

    def stats(self, tgt, drf, draft_tok, temperature, status, stream=None):
        self._check(tgt)
        capi.spec_vp_shard_stats(tgt, drf, self.v0, self.V, draft_tok, temperature, self.rows,
                                 status, self.ws, stream=stream)

    def decide(self, tgt, drf, draft_tok, temperature, seed, seq_id, rnd, status, diag=None,
               stream=None):
        self._check(tgt)
        capi.spec_vp_decide(tgt, drf, self.v0, self.V, self.R, self.rank, self.rows_all,
                            draft_tok, temperature, seed, seq_id, rnd, self.mass, status, self.ws,
                            diag=diag, stream=stream)

    def pick(self, tgt, drf, draft_tok, temperature, accept_len, out_tok, status, diag=None,
             stream=None):
        self._check(tgt)
        capi.spec_vp_pick(tgt, drf, self.v0, self.V, self.R, self.rank, self.mass_all,
                          draft_tok, temperature, accept_len, out_tok, status, self.ws,
                          diag=diag, stream=stream)


def _device_collectives(t, group):
    return t.is_cuda and dist.get_backend(group) == "nccl"


def all_gather_rank_order(out_all, local, group=None):
    """out_all[r] = rank r's ``local``, on every rank."""
    if _device_collectives(local, group):
        dist.all_gather_into_tensor(out_all, local.contiguous(), group=group)
        return
    src = local.cpu() if local.is_cuda else local.contiguous()
    parts = [torch.empty_like(src) for _ in range(dist.get_world_size(group))]
    dist.all_gather(parts, src, group=group)
    out_all.copy_(torch.stack(parts))


def all_reduce_max(t, group=None):
    if _device_collectives(t, group):
        dist.all_reduce(t, op=dist.ReduceOp.MAX, group=group)
        return
    c = t.cpu() if t.is_cuda else t
    dist.all_reduce(c, op=dist.ReduceOp.MAX, group=group)
    if c is not t:
        t.copy_(c)


def verify_chain_vocab_parallel(shard, tgt, drf, draft_tok, temperature, seed, seq_id, rnd,
                                accept_len, out_tok, status, diag=None, group=None, stream=None):
    """This rank's part of one vocabulary-parallel chain check. ``tgt`` /
    ``drf``: its columns [B, K+1, Vs] / [B, K, Vs]; the rest as
    spec_verify_chain. Every rank of ``group`` calls this with its own shard
    and identical draft_tok, temperature, seed, seq_id and rnd; afterwards
    accept_len, out_tok and diag are the same on every rank. With a
    ``stream``, the launches and the collectives both run in its order."""
    if stream is not None:
        with torch.cuda.stream(stream):
            return verify_chain_vocab_parallel(shard, tgt, drf, draft_tok, temperature, seed,
                                               seq_id, rnd, accept_len, out_tok, status,
                                               diag=diag, group=group)
    shard.stats(tgt, drf, draft_tok, temperature, status, stream=stream)
    all_gather_rank_order(shard.rows_all, shard.rows, group)
    shard.decide(tgt, drf, draft_tok, temperature, seed, seq_id, rnd, status, diag=diag,
                 stream=stream)
    all_gather_rank_order(shard.mass_all, shard.mass, group)
    shard.pick(tgt, drf, draft_tok, temperature, accept_len, out_tok, status, diag=diag,
               stream=stream)
    all_reduce_max(out_tok, group)
