"""A small, repeatable launch sequence for profilers (ncu) and timing.

Runs the chain verification of the benchmark's logit model (K=8, V=128256
bf16, Zipf prior, T=1) on B sequences, and optionally the paged commit that
follows it, `--iters` times. B=32 keeps the logits (140 MB) above the L2 size
while the whole case stays well under a few GB of device memory.

    python -m speculative_decoding_verification_89_b200.profile_case --B 32
    python -m speculative_decoding_verification_89_b200.profile_case --B 64 --commit
"""
from __future__ import annotations

import argparse

import torch

from . import capi
from . import workloads as W


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--B", type=int, default=32)
    ap.add_argument("--iters", type=int, default=6)
    ap.add_argument("--commit", action="store_true", help="also run the paged commit")
    ap.add_argument("--no-verify", action="store_true", help="commit only (random accept lengths)")
    args = ap.parse_args()
    B, K, V = args.B, 8, W.LLAMA3_V
    dev = torch.device("cuda")
    acc = torch.zeros(B, dtype=torch.int32, device=dev)
    st = torch.zeros(1, dtype=torch.int32, device=dev)
    if not args.no_verify:
        prob = W.chain_batch(device=dev, B=B)
        ws = capi.workspace(B, K, V, torch.bfloat16, device=dev)
        out = torch.empty((B, K + 1), dtype=torch.int32, device=dev)
    if args.commit:
        state, bufs = W.commit_setup(B, K, device=dev)
        base = state.seq_lens.clone()
        gen = torch.Generator(device=dev)
        gen.manual_seed(0)
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(2)]
    times = []
    for i in range(args.iters):
        ev[0].record()
        if not args.no_verify:
            capi.spec_verify_chain(prob.tgt, prob.drf, prob.draft_tok, prob.temperature, prob.seed,
                                   prob.seq_id, i, acc, out, st, ws)
        elif args.commit:
            acc = torch.randint(0, K + 1, (B,), generator=gen, device=dev, dtype=torch.int32)
        if args.commit:
            capi.spec_commit_paged(state.tables, state.seq_lens, base, acc, 1, state.free_stack,
                                   state.free_top, K + 1, st, block_size=16,
                                   kv_stage=bufs.kv_stage, kv_pool=bufs.kv_pool,
                                   hid_stage=bufs.hid_stage, hid_out=bufs.hid_out,
                                   hid_off=bufs.hid_off)
        ev[1].record()
        torch.cuda.synchronize()
        times.append(ev[0].elapsed_time(ev[1]) * 1e3)
    print(f"B={B} status={int(st.item())} us/iter median={sorted(times)[len(times) // 2]:.1f}")
    if int(st.item()) != 0:
        raise SystemExit(1)


if __name__ == "__main__":
    main()
