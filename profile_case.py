"""A small, repeatable launch sequence for profilers (ncu) and timing.

Runs the chain verification of the benchmark's logit model (K=8, V=128256
bf16, Zipf prior, T=1) on B sequences, and optionally the paged commit that
follows it, `--iters` times. B=32 keeps the logits (140 MB) above the L2 size
while the whole case stays well under a few GB of device memory.

    python profile_case.py --B 32
    python profile_case.py --B 64 --commit
    python profile_case.py --B 64 --vp 8
    python profile_case.py --small        (B=1, K=4, V=1024 fp32: the one-launch check)
    python profile_case.py --engine --iters 8   (rounds of the benchmark's engine loop)
"""
from __future__ import annotations

import argparse
import os
import sys

import torch

sys.path.insert(0, os.path.dirname(os.path.abspath(__file__)))
from speculative_decoding_verification_89_b200 import capi  # noqa: E402
from speculative_decoding_verification_89_b200 import workloads as W  # noqa: E402


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--B", type=int, default=32)
    ap.add_argument("--iters", type=int, default=6)
    ap.add_argument("--commit", action="store_true", help="also run the paged commit")
    ap.add_argument("--fused", action="store_true",
                    help="spec_verify_chain_commit on a small pool (4 layers, contexts 256-1024)")
    ap.add_argument("--no-verify", action="store_true", help="commit only (random accept lengths)")
    ap.add_argument("--outcome", type=int, default=-1,
                    help="run the outcome law with this many outcomes instead of verifying")
    ap.add_argument("--draft", action="store_true", help="run the draft step instead of verifying")
    ap.add_argument("--engine", action="store_true",
                    help="--iters rounds of the engine loop (64 sequences, V=32000 bf16)")
    ap.add_argument("--small", action="store_true",
                    help="chain verification of B=1, K=4, V=1024 fp32 (fresh rows each call)")
    ap.add_argument("--vp", type=int, default=0,
                    help="run the vocabulary-parallel check over this many shards, the ranks "
                         "in turn on this GPU, instead of verifying")
    args = ap.parse_args()
    B, K, V = args.B, 8, W.LLAMA3_V
    dev = torch.device("cuda")
    if args.small:
        return small(args, dev)
    if args.engine:
        import bench
        r = bench.run_cfg_engine(dev, rounds=args.iters)
        print(f"engine: {args.iters} rounds, {r['ms_per_round_device'] * 1e3:.1f} us per round")
        return None
    acc = torch.zeros(B, dtype=torch.int32, device=dev)
    st = torch.zeros(1, dtype=torch.int32, device=dev)
    if not args.no_verify:
        prob = W.chain_batch(device=dev, B=B)
        ws = capi.workspace(B, K, V, torch.bfloat16, device=dev)
        out = torch.empty((B, K + 1), dtype=torch.int32, device=dev)
    if args.fused:
        state, bufs = W.commit_setup(B, K, ctx_lo=256, ctx_hi=1024, layers=4, device=dev)
        base = state.seq_lens.clone()
    if args.commit:
        state, bufs = W.commit_setup(B, K, device=dev)
        base = state.seq_lens.clone()
        gen = torch.Generator(device=dev)
        gen.manual_seed(0)
    if args.outcome >= 0 or args.draft or args.vp > 0:
        return other(args, B, K, V, dev)
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(2)]
    times = []
    for i in range(args.iters):
        ev[0].record()
        if args.fused:
            capi.spec_verify_chain_commit(prob.tgt, prob.drf, prob.draft_tok, prob.temperature,
                                          prob.seed, prob.seq_id, i, acc, out, state.tables,
                                          state.seq_lens, base, state.free_stack,
                                          state.free_top, st, ws, block_size=16,
                                          kv_stage=bufs.kv_stage, kv_pool=bufs.kv_pool,
                                          hid_stage=bufs.hid_stage, hid_out=bufs.hid_out,
                                          hid_off=bufs.hid_off)
        elif not args.no_verify:
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


def small(args, dev):
    """B=1, K=4, V=1024 fp32 chain checks on fresh rows each call."""
    probs = [W.chain_small(rnd=r, device=dev) for r in range(args.iters)]
    ws = capi.workspace(1, 4, 1024, torch.float32, device=dev)
    acc = torch.empty(1, dtype=torch.int32, device=dev)
    out = torch.empty((1, 5), dtype=torch.int32, device=dev)
    st = torch.zeros(1, dtype=torch.int32, device=dev)
    for i, p in enumerate(probs):
        capi.spec_verify_chain(p.tgt, p.drf, p.draft_tok, p.temperature, p.seed, p.seq_id, i, acc,
                               out, st, ws)
    torch.cuda.synchronize()
    print(f"small: {len(probs)} calls, status={int(st.item())}")
    if int(st.item()) != 0:
        raise SystemExit(1)


def other(args, B, K, V, dev):
    """The outcome law (on the verification inputs), the draft step, or the
    vocabulary-parallel check with its ranks in turn (exchanges as copies)."""
    st = torch.zeros(1, dtype=torch.int32, device=dev)
    if args.vp > 0:
        from speculative_decoding_verification_89_b200.vocab_parallel import (ChainShard,
                                                                              vocab_shards)
        prob = W.chain_batch(device=dev, B=B)
        R = args.vp
        ranks = []
        for r, (v0, Vs) in enumerate(vocab_shards(V, R)):
            ranks.append((ChainShard(B, K, V, v0, Vs, R, r, torch.bfloat16, device=dev),
                          prob.tgt[:, :, v0:v0 + Vs].contiguous(),
                          prob.drf[:, :, v0:v0 + Vs].contiguous(),
                          torch.empty(B, dtype=torch.int32, device=dev),
                          torch.empty((B, K + 1), dtype=torch.int32, device=dev)))

        def call(i):
            for sh, tgt, drf, _, _ in ranks:
                sh.stats(tgt, drf, prob.draft_tok, prob.temperature, st)
            for r, (sh, _, _, _, _) in enumerate(ranks):
                ranks[0][0].rows_all[r].copy_(sh.rows)
            for sh, tgt, drf, _, _ in ranks:
                sh.rows_all = ranks[0][0].rows_all
                sh.decide(tgt, drf, prob.draft_tok, prob.temperature, prob.seed, prob.seq_id, i,
                          st)
            for r, (sh, _, _, _, _) in enumerate(ranks):
                ranks[0][0].mass_all[r].copy_(sh.mass)
            for sh, tgt, drf, a, o in ranks:
                sh.mass_all = ranks[0][0].mass_all
                sh.pick(tgt, drf, prob.draft_tok, prob.temperature, a, o, st)
    elif args.draft:
        prob = W.draft_batch(device=dev, B=B)
        ws = capi.draft_workspace(B, V, torch.bfloat16, device=dev)
        tok = torch.empty(B, dtype=torch.int32, device=dev)
        ent = torch.empty(B, dtype=torch.float64, device=dev)

        def call(i):
            capi.spec_draft_sample(prob.logits, prob.temperature, prob.seed, prob.seq_id, i,
                                   prob.pos, tok, st, ws, entropy=ent)
    else:
        prob = W.chain_batch(device=dev, B=B)
        n = args.outcome
        ws = capi.outcome_workspace(B, K, V, torch.bfloat16, n, device=dev)
        p_len = torch.empty((B, K + 1), dtype=torch.float64, device=dev)
        tl = torch.empty((B, max(n, 1)), dtype=torch.int32, device=dev)
        tt = torch.empty((B, max(n, 1)), dtype=torch.int32, device=dev)
        tp = torch.empty((B, max(n, 1)), dtype=torch.float64, device=dev)

        def call(i):
            capi.spec_outcome_law(prob.tgt, prob.drf, prob.draft_tok, prob.temperature, n, p_len,
                                  st, ws, top_len=tl, top_tok=tt, top_prob=tp)
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(2)]
    times = []
    for i in range(args.iters):
        ev[0].record()
        call(i)
        ev[1].record()
        torch.cuda.synchronize()
        times.append(ev[0].elapsed_time(ev[1]) * 1e3)
    print(f"B={B} status={int(st.item())} us/iter median={sorted(times)[len(times) // 2]:.1f}")
    if int(st.item()) != 0:
        raise SystemExit(1)


if __name__ == "__main__":
    main()
