"""Helpers that run the CUDA path (through the C ABI binding) and the oracle
on the same seeded inputs."""
from __future__ import annotations

import numpy as np
import torch

from oracle.verify import verify_chain


def padded(t):
    """Copy of a [B, n, V] logits tensor whose rows start on 16-byte
    boundaries (row stride rounded up), returned as the [B, n, V] view."""
    B, n, V = t.shape
    mult = 16 // t.element_size()
    ld = (V + mult - 1) // mult * mult
    if ld == V:
        return t
    big = torch.zeros((B, n, ld), dtype=t.dtype, device=t.device)
    big[:, :, :V] = t
    return big[:, :, :V]


def to_np(t):
    return t.detach().float().cpu().numpy().astype(np.float64)


def run_chain_gpu(prob, diag=True, split=False, persistent=False):
    from speculative_decoding_verification_89_b200 import capi
    dev = torch.device("cuda")
    tgt = padded(prob.tgt.to(dev))
    drf = padded(prob.drf.to(dev))
    B, Kp1, V = tgt.shape
    K = Kp1 - 1
    dt = prob.draft_tok.to(dev).contiguous()
    T = prob.temperature.to(dev)
    sid = prob.seq_id.to(dev)
    ws = capi.workspace(B, K, V, tgt.dtype, device=dev)
    acc = torch.full((B,), -7, dtype=torch.int32, device=dev)
    out = torch.full((B, K + 1), -7, dtype=torch.int32, device=dev)
    dg = torch.full((B, 4 * K + 2), -7.0, dtype=torch.float64, device=dev) if diag else None
    st = torch.zeros(1, dtype=torch.int32, device=dev)
    if split:
        capi.spec_chain_row_stats(tgt, drf, T, st, ws)
        capi.spec_chain_decide(tgt, drf, dt, T, prob.seed, sid, prob.rnd, acc, out, st, ws,
                               diag=dg)
    else:
        fn = capi.spec_verify_chain_persistent if persistent else capi.spec_verify_chain
        fn(tgt, drf, dt, T, prob.seed, sid, prob.rnd, acc, out, st, ws, diag=dg)
    torch.cuda.synchronize()
    return (acc.cpu().numpy(), out.cpu().numpy(),
            dg.cpu().numpy() if diag else None, int(st.item()))


def run_chain_oracle(prob, seqs=None):
    seqs = range(prob.tgt.shape[0]) if seqs is None else seqs
    res = {}
    for b in seqs:
        r = verify_chain(to_np(prob.tgt[b:b + 1]), to_np(prob.drf[b:b + 1]),
                         prob.draft_tok[b:b + 1].cpu().numpy(),
                         prob.temperature[b:b + 1].cpu().numpy(), prob.seed,
                         prob.seq_id[b:b + 1].cpu().numpy(), prob.rnd)
        res[b] = r[0]
    return res
