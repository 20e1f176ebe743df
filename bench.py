#!/usr/bin/env python
"""Benchmark of the verification hot path on B200.

Workload (per GPU): batched chain verification of B=64 sequences with K=8
drafts over a V=128256 bf16 vocabulary (targets N(0, 2^2) plus a Zipf(1.1)
log-prior over ids, drafts = target + N(0, 1), T = 1), followed by the
paged-KV commit of a+1 rows per sequence (block 16, contexts U[512, 4096],
128 KiB of K/V per token, hidden rows of 4096 bf16). One step = the fused
verify-and-commit path through the C ABI (spec_verify_chain_commit's
launches: row statistics; the check and draw per sequence, whose last
sequence to pass its accept test plans the commit; the copy of the kept
rows). Each step verifies a fresh Philox round and commits against the same
committed prefix, so it rolls the previous round back and grows again: the
pool stays bounded and every step does the same kind of work.

Prints one JSON line (rank 0). ``--impl reference`` times the fp64 oracle on
the host cores instead: a plain single-threaded program as the reference arm.
"""
from __future__ import annotations

import argparse
import datetime
import hashlib
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402
import torch  # noqa: E402

METRIC = "verified tokens/s and achieved HBM GB/s vs peak (B=64,K=8,V=128256 bf16)"
B, K, V = 64, 8, 128256
KV_BYTES_PER_TOKEN = 32 * 2 * 8 * 128 * 2       # layers x {K,V} x heads x dim x bf16
HID_BYTES_PER_TOKEN = 4096 * 2
LOGIT_BYTES = B * (2 * K + 1) * V * 2           # every target and draft row once
RS_SAMPLE = 8                                   # steps per row-statistics timing sample
WORKLOAD = ("batched chain verification + paged commit: B=64, K=8, V=128256 bf16 logits "
            "(N(0,4) + Zipf(1.1) log-prior targets, drafts +N(0,1), T=1), block 16, "
            "contexts U[512,4096], 128 KiB K/V + 8 KiB hidden per token")
NCU_TRAFFIC = os.path.join(ROOT, "profiles", "ncu_traffic.json")
ROW_STATS_SOURCES = ["row_stats.cu", "rowmath.cuh", "common.cuh", "kernels.cuh"]


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--plan-only", action="store_true",
                    help="print each rank's device and sequence assignment (gloo, no GPU work)")
    return ap.parse_args()


def free_port():
    import socket
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def relaunch(args):
    """`--gpus N` with N > 1 outside a launcher: run this script again as N
    ranks (one process per GPU) under torch.distributed.run on this node,
    bounded by a timeout, and return its exit status."""
    cmd = ["timeout", "-k", "60", "3600", sys.executable, "-m", "torch.distributed.run",
           "--nnodes=1", f"--nproc-per-node={args.gpus}", "--master-addr", "127.0.0.1",
           "--master-port", str(free_port()), os.path.abspath(__file__), *sys.argv[1:]]
    return subprocess.call(cmd)


def rank_plan(dist):
    """What rank `dist.rank` works on: its own GPU (LOCAL_RANK), its own B
    sequences (ids B*rank ..), its own logits and block pool (seeds)."""
    return {"rank": dist.rank, "world": dist.world, "device": dist.local,
            "seq_id_base": B * dist.rank, "logit_seed": 2 + 1000 * dist.rank,
            "pool_seed": 2 + dist.rank}


# ----------------------------------------------------------------------------
# Distributed plumbing (one process per GPU, no collective on the data path)
# ----------------------------------------------------------------------------
class Dist:
    def __init__(self):
        self.world = int(os.environ.get("WORLD_SIZE", "1"))
        self.rank = int(os.environ.get("RANK", "0"))
        self.local = int(os.environ.get("LOCAL_RANK", "0"))
        self.pg = None

    def init(self, backend="nccl"):
        if self.world > 1:
            import torch.distributed as dist
            dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
            self.pg = dist

    def barrier(self):
        if self.pg:
            self.pg.barrier()

    def reduce(self, x: float, op: str) -> float:
        if not self.pg:
            return x
        dev = "cuda" if torch.cuda.is_available() and self.pg.get_backend() == "nccl" else "cpu"
        t = torch.tensor([x], dtype=torch.float64, device=dev)
        self.pg.all_reduce(t, op=self.pg.ReduceOp.MAX if op == "max" else self.pg.ReduceOp.SUM)
        return float(t.item())

    def close(self):
        if self.pg:
            self.pg.destroy_process_group()


# ----------------------------------------------------------------------------
# Clock sampling during the timed region
# ----------------------------------------------------------------------------
class Clocks:
    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap")

    def __init__(self, index):
        self.index = index
        self.proc = None
        self.file = None

    def start(self):
        try:
            self.file = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.index), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=self.file, stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None
            return
        # The sampler takes a moment to start: wait (up to 5 s) for its first
        # line so the timed region is covered.
        t0 = time.time()
        while time.time() - t0 < 5.0 and self.proc.poll() is None:
            if os.path.getsize(self.file.name) > 0:
                break
            time.sleep(0.05)

    def stop(self):
        if not self.proc:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.file.flush()
        rows = []
        with open(self.file.name) as fh:
            for line in fh:
                parts = [p.strip() for p in line.split(",")]
                if len(parts) == 7:
                    rows.append(parts)
        os.unlink(self.file.name)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        sm = [float(r[0]) for r in rows if r[0].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[3 + i] == "Active"})
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": float(rows[0][1]) if rows[0][1].replace(".", "").isdigit() else None,
                "reasons": reasons, "samples": len(rows)}


def measured_peak():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as fh:
            return float(json.load(fh)["hbm_gbs"]), "measured"
    except (OSError, KeyError, ValueError):
        return 6650.0, "fallback"


def row_stats_source_hash():
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "speculative_decoding_verification_89_b200", "csrc")
    for f in ROW_STATS_SOURCES:
        with open(os.path.join(csrc, f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()


def ncu_traffic():
    """DRAM bytes per launch of the row-statistics kernel from the committed
    ncu summary, or None if absent or taken on different kernel source."""
    try:
        with open(NCU_TRAFFIC) as fh:
            rec = json.load(fh)
    except (OSError, ValueError):
        return None
    if rec.get("source_sha256") != row_stats_source_hash():
        return None
    return rec.get("dram_bytes_per_launch")


# ----------------------------------------------------------------------------
# The oracle on the host (cpu_baseline and the reference arm)
# ----------------------------------------------------------------------------
def run_oracle_steps(prob_host, tables, seq_lens, free_stack, free_top, seqs, n_steps,
                     rnd0=0):
    """n_steps oracle steps; step s verifies sequence seqs[s % len] at round
    rnd0 + s // len and commits its rows. Returns (tokens, seconds)."""
    from oracle.commit import commit_paged
    from oracle.verify import verify_chain
    tok = 0
    t0 = time.perf_counter()
    for s in range(n_steps):
        b = seqs[s % len(seqs)]
        r = verify_chain(prob_host["tgt"][b:b + 1], prob_host["drf"][b:b + 1],
                         prob_host["draft"][b:b + 1], prob_host["T"][b:b + 1], 2,
                         prob_host["sid"][b:b + 1], rnd0 + s // len(seqs))[0]
        keep = np.array([r.accepted + 1])
        c = commit_paged(tables[b:b + 1], seq_lens[b:b + 1], seq_lens[b:b + 1], keep,
                         free_stack, free_top, 16, len(free_stack), K + 1)
        assert c.status == 0
        tok += r.accepted + 1
    return tok, time.perf_counter() - t0


def host_problem(prob, state):
    to64 = lambda t: t.detach().float().cpu().numpy().astype(np.float64)  # noqa: E731
    return ({"tgt": to64(prob.tgt), "drf": to64(prob.drf),
             "draft": prob.draft_tok.cpu().numpy(), "T": prob.temperature.cpu().numpy(),
             "sid": prob.seq_id.cpu().numpy()},
            state.tables.cpu().numpy(), state.seq_lens.cpu().numpy(),
            state.free_stack.cpu().numpy(), int(state.free_top.cpu()[0]))


def cpu_baseline(prob, state, budget_s=12.0):
    hp, tables, lens, stack, top = host_problem(prob, state)
    tok1, t1 = run_oracle_steps(hp, tables, lens, stack, top, [0], 1)
    n = max(2, min(4 * B, int(budget_s / max(t1, 1e-3))))
    tok, sec = run_oracle_steps(hp, tables, lens, stack, top, list(range(B)), n)
    return {"value": tok / sec, "unit": "tokens/s", "cores": 1, "kind": "oracle",
            "sample": f"{n} sequence-rounds of the same workload (chain verify + commit, "
                      f"fp64 numpy, single thread), {sec:.1f} s"}


def spot_check(prob, acc, out, rnd):
    """Oracle vs GPU on every sequence of one step run after the timed region
    (accepted count and emitted tokens), with the verification rule: a
    difference is allowed only at a decision whose fp64 oracle margin is
    below 1e-6, and such decisions must stay under 1e-4 of all."""
    from oracle.verify import verify_chain
    to64 = lambda t: t.detach().float().cpu().numpy().astype(np.float64)  # noqa: E731
    ref = verify_chain(to64(prob.tgt), to64(prob.drf), prob.draft_tok.cpu().numpy(),
                       prob.temperature.cpu().numpy(), prob.seed, prob.seq_id.cpu().numpy(), rnd)
    decisions = excused = 0
    for b, r in enumerate(ref):
        decisions += len(r.decisions)
        a = int(acc[b])
        if a == r.accepted and [int(x) for x in out[b, :a + 1]] == list(r.tokens):
            continue
        if min(d.margin for d in r.decisions) < 1e-6:
            excused += 1
        else:
            return {"result": "MISMATCH", "sequence": b}
    ok = excused == 0 or excused <= 1e-4 * decisions
    return {"result": "ok" if ok else "too many near-margin differences",
            "sequences": len(ref), "decisions": decisions, "excused": excused}


# ----------------------------------------------------------------------------
# Our arm
# ----------------------------------------------------------------------------
def run_ours(args, dist):
    from speculative_decoding_verification_89_b200 import capi
    from speculative_decoding_verification_89_b200 import workloads as W

    plan = rank_plan(dist)
    dev = torch.device("cuda", plan["device"])
    torch.cuda.set_device(dev)
    stream = torch.cuda.current_stream()
    prob = W.chain_batch(device=dev, seed=plan["logit_seed"], seq_id_base=plan["seq_id_base"])
    state, bufs = W.commit_setup(B, K, device=dev, seed=plan["pool_seed"])
    base = state.seq_lens.clone()
    total = args.warmup + args.steps
    hist = torch.zeros((total, B), dtype=torch.int32, device=dev)
    out_tok = torch.empty((B, K + 1), dtype=torch.int32, device=dev)
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    ws = capi.workspace(B, K, V, torch.bfloat16, device=dev)
    tgt, drf, T, sid, dt = prob.tgt, prob.drf, prob.temperature, prob.seq_id, prob.draft_tok

    def row_stats():
        capi.spec_chain_row_stats(tgt, drf, T, status, ws, stream=stream)

    def decide_commit(i):
        capi.spec_chain_decide_commit(tgt, drf, dt, T, prob.seed, sid, i, hist[i], out_tok,
                                      state.tables, state.seq_lens, base, state.free_stack,
                                      state.free_top, status, ws, block_size=16,
                                      kv_stage=bufs.kv_stage, kv_pool=bufs.kv_pool,
                                      hid_stage=bufs.hid_stage, hid_out=bufs.hid_out,
                                      hid_off=bufs.hid_off, stream=stream)

    clocks = Clocks(plan["device"])
    clocks.start()
    for i in range(args.warmup):
        row_stats()
        decide_commit(i)
    torch.cuda.synchronize()
    dist.barrier()
    # The row-statistics launches of every RS_SAMPLE-th step are bracketed by
    # events for the roofline; an event between two launches ends their
    # programmatic overlap, so the other steps run without them.
    sampled = [s for s in range(args.steps) if s % RS_SAMPLE == RS_SAMPLE - 1] or [0]
    ev = {s: (torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for s in sampled}
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    e0.record(stream)
    for s in range(args.steps):
        i = args.warmup + s
        if s in ev:
            ev[s][0].record(stream)
            row_stats()
            ev[s][1].record(stream)
        else:
            row_stats()
        decide_commit(i)
    e1.record(stream)
    torch.cuda.synchronize()
    dist.barrier()
    clk = clocks.stop()
    st = int(status.item())
    if st != 0:
        raise RuntimeError(f"device status {st}: {capi.spec_status_string(st)}")
    ms = e0.elapsed_time(e1)
    ms_max = dist.reduce(ms, "max")
    acc = hist[args.warmup:].cpu().numpy()
    tokens = float((acc + 1).sum())
    tokens_all = dist.reduce(tokens, "sum")
    rs_ms = statistics.mean(a.elapsed_time(b) for a, b in ev.values())
    commit_bytes = tokens * 2 * (KV_BYTES_PER_TOKEN + HID_BYTES_PER_TOKEN)
    step_bytes = LOGIT_BYTES * args.steps + commit_bytes
    bytes_all = dist.reduce(step_bytes, "sum")

    peak, peak_kind = measured_peak()
    achieved = LOGIT_BYTES / (rs_ms * 1e-3) / 1e9
    result = {
        "metric": METRIC,
        "value": tokens_all / (ms_max * 1e-3),
        "unit": "tokens/s",
        "n_gpus": dist.world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": ms_max / args.steps,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "f32",
        "data": "synthetic",
        "config": {"workload": WORKLOAD, "logits_dtype": "bf16", "batch_per_gpu": B,
                   "drafts": K, "vocab": V, "l2": "inputs 279 MB per step > 126 MB L2; no flush",
                   "parallelism": f"replicas x{dist.world} (independent sequences per GPU)"},
        "hbm_gbs": bytes_all / (ms_max * 1e-3) / 1e9,
        "hbm_frac_of_8tbs": bytes_all / (ms_max * 1e-3) / 8e12,
        "hbm_frac_of_measured": bytes_all / (ms_max * 1e-3) / 1e9 / peak,
        "mean_accepted": float(acc.mean()),
        "roofline": {"bound": "hbm", "kernel": "row_stats_kernel (bf16, chain rows)",
                     "achieved": achieved, "peak": peak, "unit": "GB/s",
                     "frac": achieved / peak, "peak_kind": peak_kind,
                     "traffic": ncu_traffic(), "algorithmic_bytes_per_launch": LOGIT_BYTES,
                     "launch_ms": rs_ms},
        "gpu_launches": 3 * args.steps,
        "clocks": clk,
    }
    result["persistent_step"] = run_persistent_step(args, prob, state, bufs, base, dev, dist)
    result["two_call_step"] = run_two_call_step(args, prob, state, bufs, base, dev, dist)
    if not args.no_e2e:
        result["e2e"] = run_e2e(args, prob, state, bufs, base, dev, dist)
    result["draft_step"] = run_draft_step(args, dev, dist, peak)
    result["saguaro_draft"] = run_saguaro_draft(args, dev, dist)
    result["outcome_law"] = run_outcome_law(args, prob, dev, dist, peak)
    result["vocab_parallel_emulated"] = run_vocab_parallel(args, prob, dev, dist)
    result["configs"] = run_configs(args, dev, dist, peak, result)
    if dist.world == 1 and dist.rank == 0 and not args.no_cpu_baseline:
        for key, kind in (("draft_step", "draft"), ("saguaro_draft", "saguaro"),
                          ("outcome_law", "outcome"), ("vocab_parallel_emulated", "chain")):
            result[key]["oracle"] = oracle_rates(kind)
    if dist.world == 1 and dist.rank == 0:
        rnd = args.warmup + args.steps
        acc1 = torch.empty(B, dtype=torch.int32, device=dev)
        capi.spec_verify_chain_commit(tgt, drf, dt, T, prob.seed, sid, rnd, acc1, out_tok,
                                      state.tables, state.seq_lens, base, state.free_stack,
                                      state.free_top, status, ws, block_size=16,
                                      kv_stage=bufs.kv_stage, kv_pool=bufs.kv_pool,
                                      hid_stage=bufs.hid_stage, hid_out=bufs.hid_out,
                                      hid_off=bufs.hid_off, stream=stream)
        torch.cuda.synchronize()
        result["parity_spot_check"] = spot_check(prob, acc1.cpu().numpy(),
                                                 out_tok.cpu().numpy(), rnd)
        if not args.no_cpu_baseline:
            cb = cpu_baseline(prob, state)
            r = oracle_rates("chain_commit")
            if "all_cores" in r:
                cb["single_thread_value"] = cb["value"]
                cb["value"] = r["all_cores"]
                cb["cores"] = r["cores"]
                cb["sample"] += (f"; all cores: {r['tasks']} tasks of {r['task']}, one process "
                                 f"per core, tokens over the busiest process's oracle time")
            result["cpu_baseline"] = cb
    return result


def run_persistent_step(args, prob, state, bufs, base, dev, dist):
    """The same step through spec_verify_chain_commit_persistent: a prologue
    launch, then one persistent kernel for the row statistics, the checks,
    the draws, the plan and the copy -- two launches."""
    from speculative_decoding_verification_89_b200 import capi
    n = max(10, min(args.steps, 2000))
    acc = torch.empty((n, B), dtype=torch.int32, device=dev)
    out = torch.empty((B, K + 1), dtype=torch.int32, device=dev)
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    ws = capi.workspace(B, K, V, torch.bfloat16, device=dev)

    def step(i):
        capi.spec_verify_chain_commit_persistent(
            prob.tgt, prob.drf, prob.draft_tok, prob.temperature, prob.seed, prob.seq_id, i,
            acc[i], out, state.tables, state.seq_lens, base, state.free_stack, state.free_top,
            status, ws, block_size=16, kv_stage=bufs.kv_stage, kv_pool=bufs.kv_pool,
            hid_stage=bufs.hid_stage, hid_out=bufs.hid_out, hid_off=bufs.hid_off)

    for i in range(max(3, args.warmup)):
        step(i)
    torch.cuda.synchronize()
    dist.barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for i in range(n):
        step(i)
    e1.record()
    torch.cuda.synchronize()
    ms = dist.reduce(e0.elapsed_time(e1), "max")
    if int(status.item()) != 0:
        raise RuntimeError("device status during the persistent run")
    tokens = float((acc.cpu().numpy() + 1).sum())
    return {"steps": n, "ms_per_step": ms / n, "tokens_per_s": tokens / (ms * 1e-3),
            "gpu_launches_per_step": 2}


def run_two_call_step(args, prob, state, bufs, base, dev, dist):
    """The same step as separate calls -- spec_verify_chain (row statistics,
    decide) then spec_commit_paged (plan, copy): four launches, each waiting
    for the one before."""
    from speculative_decoding_verification_89_b200 import capi
    n = max(10, min(args.steps, 2000))
    acc = torch.empty((n, B), dtype=torch.int32, device=dev)
    out = torch.empty((B, K + 1), dtype=torch.int32, device=dev)
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    ws = capi.workspace(B, K, V, torch.bfloat16, device=dev)

    def step(i):
        capi.spec_verify_chain(prob.tgt, prob.drf, prob.draft_tok, prob.temperature, prob.seed,
                               prob.seq_id, i, acc[i], out, status, ws)
        capi.spec_commit_paged(state.tables, state.seq_lens, base, acc[i], 1, state.free_stack,
                               state.free_top, K + 1, status, block_size=16,
                               kv_stage=bufs.kv_stage, kv_pool=bufs.kv_pool,
                               hid_stage=bufs.hid_stage, hid_out=bufs.hid_out,
                               hid_off=bufs.hid_off)

    for i in range(max(3, args.warmup)):
        step(i)
    torch.cuda.synchronize()
    dist.barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for i in range(n):
        step(i)
    e1.record()
    torch.cuda.synchronize()
    ms = dist.reduce(e0.elapsed_time(e1), "max")
    if int(status.item()) != 0:
        raise RuntimeError("device status during the two-call run")
    tokens = float((acc.cpu().numpy() + 1).sum())
    return {"steps": n, "ms_per_step": ms / n, "tokens_per_s": tokens / (ms * 1e-3),
            "gpu_launches_per_step": 4}


def graph_us_per_call(calls, reps, dist):
    """Device time per call of a short launch sequence: the calls (each a
    closure that launches on the current stream) captured once in a CUDA
    graph and the graph replayed `reps` times between events, so that the
    Python-side cost of each call does not set the pace."""
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        for fn in calls:  # warm-up outside the capture (attributes, lookups)
            fn()
    torch.cuda.current_stream().wait_stream(s)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        for fn in calls:
            fn()
    for _ in range(3):
        g.replay()
    torch.cuda.synchronize()
    dist.barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(reps):
        g.replay()
    e1.record()
    torch.cuda.synchronize()
    ms = dist.reduce(e0.elapsed_time(e1), "max") / (reps * len(calls))
    del g
    return ms * 1e3


def run_draft_step(args, dev, dist, peak):
    """The draft step (next token of each sequence from the drafting exit,
    with its entropy) on B=64 rows of V=128256 bf16: calls per second and the
    algorithmic HBM rate (each logit read once). The calls cycle through 10
    such batches (164 MB, more than the 126 MB L2), so the rows come from HBM.
    Same timing rules: warm-up, device events around a run of calls, max over
    ranks."""
    from speculative_decoding_verification_89_b200 import capi
    from speculative_decoding_verification_89_b200 import workloads as W
    probs = [W.draft_batch(device=dev, rnd=r) for r in range(10)]
    prob = probs[0]
    T, sid, pos = prob.temperature, prob.seq_id, prob.pos
    ws = capi.draft_workspace(B, V, prob.logits.dtype, device=dev)
    tok = torch.empty(B, dtype=torch.int32, device=dev)
    logq = torch.empty(B, dtype=torch.float64, device=dev)
    ent = torch.empty(B, dtype=torch.float64, device=dev)
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    n = max(10, min(args.steps, 2000))
    for i in range(max(3, args.warmup)):
        capi.spec_draft_sample(probs[i % 10].logits, T, prob.seed, sid, i, pos, tok, status, ws,
                               logq=logq, entropy=ent)
    torch.cuda.synchronize()
    dist.barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for i in range(n):
        capi.spec_draft_sample(probs[i % 10].logits, T, prob.seed, sid, i, pos, tok, status, ws,
                               logq=logq, entropy=ent)
    e1.record()
    torch.cuda.synchronize()
    ms_host = dist.reduce(e0.elapsed_time(e1), "max") / n
    calls = [lambda i=i: capi.spec_draft_sample(probs[i].logits, T, prob.seed, sid, i, pos, tok,
                                                status, ws, logq=logq, entropy=ent)
             for i in range(10)]
    ms = graph_us_per_call(calls, max(10, n // 10), dist) * 1e-3
    if int(status.item()) != 0:
        raise RuntimeError(f"draft step: device status {int(status.item())}")
    nbytes = B * V * 2
    return {"workload": "draft step: B=64 rows, V=128256 bf16 (N(0,4) + Zipf(1.1)), T=1, "
                        "token + ln q + entropy per row; 10 batches in turn (164 MB > L2)",
            "us_per_call": ms * 1e3, "timing": "CUDA graph of 10 calls, replayed",
            "us_per_call_from_python": ms_host * 1e3, "calls": n,
            "tokens_per_s": B * dist.world / (ms * 1e-3),
            "algorithmic_bytes_per_call": nbytes,
            "achieved_gbs": nbytes / (ms * 1e-3) / 1e9,
            "frac_of_measured_hbm": nbytes / (ms * 1e-3) / 1e9 / peak,
            "gpu_launches_per_call": 1}


def run_saguaro_draft(args, dev, dist):
    """Saguaro sampling before the draft step: the 32 cached tokens of each of
    B=64 sequences lowered in place (eps = 0.5) in rows of V=128256 bf16, then
    the draft step on the lowered rows; 10 batches in turn. The lowering
    accumulates over the calls on the same batch; timing is not affected."""
    from speculative_decoding_verification_89_b200 import capi
    from speculative_decoding_verification_89_b200 import workloads as W
    probs = [W.draft_batch(device=dev, rnd=r) for r in range(10)]
    cached = [W.cached_tokens(p.logits, 32, seed=700 + r).to(dev) for r, p in enumerate(probs)]
    prob = probs[0]
    T, sid, pos = prob.temperature, prob.seq_id, prob.pos
    ws = capi.draft_workspace(B, V, prob.logits.dtype, device=dev)
    tok = torch.empty(B, dtype=torch.int32, device=dev)
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    n = max(10, min(args.steps, 2000))

    def adjust(i):
        capi.spec_saguaro_adjust(probs[i % 10].logits, cached[i % 10], 0.5, T)

    def both(i):
        adjust(i)
        capi.spec_draft_sample(probs[i % 10].logits, T, prob.seed, sid, i, pos, tok, status, ws)

    out = {}
    for name, fn in (("us_per_call_adjust", adjust), ("us_per_call_adjust_and_draft", both)):
        out[name] = graph_us_per_call([lambda i=i: fn(i) for i in range(10)],
                                      max(10, n // 10), dist)
    if int(status.item()) != 0:
        raise RuntimeError(f"saguaro draft: device status {int(status.item())}")
    return {"workload": "Saguaro lowering (eps 0.5, 32 cached ids per sequence) of B=64 rows, "
                        "V=128256 bf16, then the draft step; 10 batches in turn",
            **out, "timing": "CUDA graph of 10 calls, replayed", "calls": n,
            "bound": "latency (2048 logits updated per call)",
            "gpu_launches_per_call": 2}


def run_vocab_parallel(args, prob, dev, dist):
    """The vocabulary-parallel check at the benchmark's verification shape
    with its R=8 ranks emulated on this one GPU: each rank's three launches
    (after the row statistics of its shard) run in turn and the exchanges are
    device copies in rank order. The NVLink exchange of a multi-GPU run is
    not measured here; the figure is the kernels' total over the ranks."""
    from speculative_decoding_verification_89_b200.vocab_parallel import ChainShard, vocab_shards
    R = 8
    Bp, Kp1, Vv = prob.tgt.shape
    K1 = Kp1 - 1
    dt, T, sid = prob.draft_tok, prob.temperature, prob.seq_id
    ranks = []
    for r, (v0, Vs) in enumerate(vocab_shards(Vv, R)):
        ranks.append(dict(
            sh=ChainShard(Bp, K1, Vv, v0, Vs, R, r, prob.tgt.dtype, device=dev),
            tgt=prob.tgt[:, :, v0:v0 + Vs].contiguous(),
            drf=prob.drf[:, :, v0:v0 + Vs].contiguous(),
            acc=torch.empty(Bp, dtype=torch.int32, device=dev),
            out=torch.empty((Bp, Kp1), dtype=torch.int32, device=dev)))
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    rows_all = ranks[0]["sh"].rows_all
    mass_all = ranks[0]["sh"].mass_all
    out_all = torch.empty((R, Bp, Kp1), dtype=torch.int32, device=dev)

    def check(i):
        for x in ranks:
            x["sh"].stats(x["tgt"], x["drf"], dt, T, status)
        for r, x in enumerate(ranks):
            rows_all[r].copy_(x["sh"].rows)
        for x in ranks:
            x["sh"].rows_all = rows_all
            x["sh"].decide(x["tgt"], x["drf"], dt, T, prob.seed, sid, i, status)
        for r, x in enumerate(ranks):
            mass_all[r].copy_(x["sh"].mass)
        for r, x in enumerate(ranks):
            x["sh"].mass_all = mass_all
            x["sh"].pick(x["tgt"], x["drf"], dt, T, x["acc"], out_all[r], status)
        return out_all.amax(0)

    n = max(10, min(args.steps // 20, 200))
    ms = graph_us_per_call([lambda: check(0)], n, dist) * 1e-3
    if int(status.item()) != 0:
        raise RuntimeError(f"vocabulary-parallel check: device status {int(status.item())}")
    per_seq = 32 * (2 * K1 + 1) + 16 + 4 * (K1 + 1)
    return {"workload": f"vocabulary-parallel chain check, B={Bp}, K={K1}, V={Vv} bf16 over "
                        f"R={R} shards, ranks emulated in turn on one GPU",
            "us_per_check_all_ranks": ms * 1e3, "checks": n,
            "timing": "CUDA graph of one check (all ranks), replayed",
            "exchange_bytes_per_rank_per_check": Bp * per_seq,
            "note": "unmeasured on hardware with R GPUs: exchanges here are device copies",
            "gpu_launches_per_check": 4 * R}


def run_outcome_law(args, prob, dev, dist, peak):
    """Outcome prediction on the benchmark's verification inputs (B=64, K=8,
    V=128256 bf16, drafts fixed): the acceptance-length law and the 32 most
    likely (length, token) outcomes per sequence. Algorithmic bytes: each
    logit once (the per-position pass re-reads the row pairs)."""
    from speculative_decoding_verification_89_b200 import capi
    n_top = 32
    ws = capi.outcome_workspace(B, K, V, torch.bfloat16, n_top, device=dev)
    f64 = dict(dtype=torch.float64, device=dev)
    p_len = torch.empty((B, K + 1), **f64)
    tl = torch.empty((B, n_top), dtype=torch.int32, device=dev)
    tt = torch.empty((B, n_top), dtype=torch.int32, device=dev)
    tp = torch.empty((B, n_top), **f64)
    status = torch.zeros(1, dtype=torch.int32, device=dev)

    def call():
        capi.spec_outcome_law(prob.tgt, prob.drf, prob.draft_tok, prob.temperature, n_top, p_len,
                              status, ws, top_len=tl, top_tok=tt, top_prob=tp)

    n = max(10, min(args.steps // 10, 500))
    for _ in range(max(3, args.warmup)):
        call()
    torch.cuda.synchronize()
    dist.barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(n):
        call()
    e1.record()
    torch.cuda.synchronize()
    ms = dist.reduce(e0.elapsed_time(e1), "max") / n
    if int(status.item()) != 0:
        raise RuntimeError(f"outcome law: device status {int(status.item())}")
    return {"workload": "outcome law: B=64, K=8, V=128256 bf16 (the verification inputs), "
                        "32 outcomes per sequence",
            "us_per_call": ms * 1e3, "calls": n,
            "sequences_per_s": B * dist.world / (ms * 1e-3),
            "algorithmic_bytes_per_call": LOGIT_BYTES,
            "achieved_gbs": LOGIT_BYTES / (ms * 1e-3) / 1e9,
            "frac_of_measured_hbm": LOGIT_BYTES / (ms * 1e-3) / 1e9 / peak,
            "gpu_launches_per_call": 3}


# ----------------------------------------------------------------------------
# The other configurations (chain small, two-stage peaked, two-stage mixed,
# engine loop): per-config throughput at one GPU, each against the oracle's on
# the host cores (one core, and one process per core)
# ----------------------------------------------------------------------------
class HierLoop:
    """Rolling two-stage verification of B sequences on the device: before
    every round the rows of slots >= win_len are redrawn (earlier slots keep
    the rows the window was checked against), drafts come from L_d at the
    window's next slots, and spec_verify_hier runs on the stream."""

    def __init__(self, B, K, Ni, V, dtype, dev):
        from speculative_decoding_verification_89_b200 import capi
        self.capi, self.B, self.K, self.Ni, self.S, self.dev = capi, B, K, Ni, Ni + K + 1, dev
        i32 = dict(dtype=torch.int32, device=dev)
        WC = Ni + K
        self.win_len = torch.zeros(B, **i32)
        self.win_tok = torch.full((B, WC), -1, **i32)
        self.win_stat = torch.zeros((B, WC, 2), dtype=torch.float64, device=dev)
        self.acc1, self.acc2 = torch.empty(B, **i32), torch.empty(B, **i32)
        self.ctok, self.cn = torch.empty((B, WC + 1), **i32), torch.empty(B, **i32)
        self.status = torch.zeros(1, **i32)
        self.ws = capi.workspace(B, K, V, dtype, Ni=Ni, device=dev)
        self.lg = None

    def logits(self, fresh):
        """This round's rows: fresh ones for slots >= win_len."""
        if self.lg is None:
            self.lg = [x.clone() for x in fresh]
        else:
            keep = torch.arange(self.S, device=self.dev).view(1, -1, 1) < \
                self.win_len.view(-1, 1, 1)
            self.lg = [torch.where(keep, o, n) for o, n in zip(self.lg, fresh)]
        return self.lg

    def call(self, drafts, T, seed, seq_id, rnd):
        lg_d, lg_i, lg_f = self.lg
        self.capi.spec_verify_hier(lg_d, lg_i, lg_f, self.Ni, drafts, T, seed, seq_id, rnd,
                                   self.win_len, self.win_tok, self.win_stat, self.acc1,
                                   self.acc2, self.ctok, self.cn, self.status, self.ws)

    def rows_read(self, w_before, greedy):
        """Logit rows the call had to read once: stage one K+1 L_i rows and K
        L_d rows (sampled sequences); stage two W+1 L_f rows where it ran."""
        a1, a2 = self.acc1.cpu().numpy(), self.acc2.cpu().numpy()
        st1 = (self.K + 1) + np.where(greedy, 0, self.K)
        W = w_before + a1 + 1
        st2 = np.where(a2 >= 0, W + 1, 0)
        return int(st1.sum() + st2.sum())


def _timed(fn):
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    fn()
    e1.record()
    return e0, e1


def run_cfg_chain_small(dev, dist):
    """Chain verification, B=1, K=4, V=1024 fp32, T=1, fresh logits every
    round for 100 rounds: latency of one spec_verify_chain call, as called
    from Python (events around each call) and on the device alone (the 100
    calls captured in a CUDA graph and replayed)."""
    from speculative_decoding_verification_89_b200 import capi
    from speculative_decoding_verification_89_b200 import workloads as W
    probs = [W.chain_small(rnd=r, device=dev) for r in range(100)]
    ws = capi.workspace(1, 4, 1024, torch.float32, device=dev)
    acc = torch.empty((100, 1), dtype=torch.int32, device=dev)
    out = torch.empty((1, 5), dtype=torch.int32, device=dev)
    st = torch.zeros(1, dtype=torch.int32, device=dev)

    def call(p, i):
        capi.spec_verify_chain(p.tgt, p.drf, p.draft_tok, p.temperature, p.seed, p.seq_id, p.rnd,
                               acc[i], out, st, ws)

    for i in range(5):
        call(probs[i], i)
    torch.cuda.synchronize()
    ev = [_timed(lambda i=i: call(probs[i], i)) for i in range(100)]
    torch.cuda.synchronize()
    us = [a.elapsed_time(b) * 1e3 for a, b in ev]
    tokens = float((acc.cpu().numpy() + 1).sum())
    us_graph = graph_us_per_call([lambda i=i: call(probs[i], i) for i in range(100)], 20, dist)
    if int(st.item()) != 0:
        raise RuntimeError("chain small: device status")
    return {"workload": "chain verification B=1, K=4, V=1024 fp32 (N(0,4) targets, drafts "
                        "+N(0,1), T=1), fresh logits each of 100 rounds",
            "us_per_round_median": statistics.median(us), "us_per_round_mean": statistics.mean(us),
            "us_per_round_graph": us_graph,
            "tokens_per_s": tokens / (sum(us) * 1e-6), "rounds": 100,
            "bound": "latency (9 rows of 4 KB; one launch)", "gpu_launches_per_round": 1}


def run_cfg_hier(dev, peak, kind, rounds):
    """Two-stage verification as a rolling loop (the window carries from call
    to call): kind 'peaked' = B=8, V=32000 bf16, T=0.7 with one greedy
    sequence; kind 'mixed' = B=256, V=151936 fp32, T ~ U(0, 1.2] with 51
    greedy sequences. Each call is timed alone with events around it, the
    row redraw and the drafts outside: us_per_call as called from Python
    (a small call's pace is then set by its launches), us_per_call_device
    the same rounds again with the call's launches queued behind a short
    device sleep, so that the events see the device time alone."""
    from speculative_decoding_verification_89_b200 import workloads as W
    if kind == "peaked":
        base = W.hier_peaked(device=dev)
        kw = dict(final_std=2.5, inter_noise=0.7, draft_noise=1.5, boost_p=0.05, boost=6.0)
        dtype, desc = torch.bfloat16, ("two-stage verification B=8, K=N_i=4, V=32000 bf16, peaked "
                                       "rows (+6 on 5%), T=0.7 with one greedy sequence")
    else:
        base = W.hier_mixed(device=dev)
        kw = dict(final_std=2.0, inter_noise=0.5, draft_noise=2.0)
        dtype, desc = torch.float32, ("two-stage verification B=256, K=N_i=4, V=151936 fp32, "
                                      "T ~ U(0,1.2] with 51 greedy sequences")
    B, K, Ni, V = base.lg_f.shape[0], base.K, base.Ni, base.lg_f.shape[2]
    T = base.temperature.to(dev)
    greedy = (base.temperature == 0).cpu().numpy()
    esz = torch.tensor([], dtype=dtype).element_size()

    def rolling(ahead):
        """The rounds from fresh windows; returns (ms, rows, committed, calls,
        hashable outputs)."""
        loop = HierLoop(B, K, Ni, V, dtype, dev)
        ms = 0.0
        rows = committed = calls = 0
        outs = []
        for r in range(rounds + 3):
            fresh = [base.lg_d, base.lg_i, base.lg_f] if r == 0 else list(
                W.hier_logits(B, loop.S, V, dtype, W.generator(9000 + r, dev), dev, **kw))
            loop.logits(fresh)
            w_before = loop.win_len.cpu().numpy()
            drafts = W.window_drafts(loop.lg[0], loop.win_len, K, T, W.generator(40 + r, dev))
            torch.cuda.synchronize()
            if ahead:
                torch.cuda._sleep(200_000)  # ~100 us: the host queues the call meanwhile
            e0, e1 = _timed(lambda: loop.call(drafts, T, base.seed, base.seq_id, r))
            torch.cuda.synchronize()
            outs.append((loop.ctok.cpu().numpy().tobytes(), loop.cn.cpu().numpy().tobytes()))
            if r >= 3:  # the first rounds fill the windows
                ms += e0.elapsed_time(e1)
                rows += loop.rows_read(w_before, greedy)
                committed += int(loop.cn.sum().item())
                calls += 1
        if int(loop.status.item()) != 0:
            raise RuntimeError(f"two-stage {kind}: device status")
        return ms, rows, committed, calls, outs

    ms, rows, committed, calls, outs = rolling(False)
    ms_dev, _, _, _, outs_dev = rolling(True)
    if outs_dev != outs:
        raise RuntimeError(f"two-stage {kind}: the device-timed rounds differ")
    nbytes = rows * V * esz
    return {"workload": desc + ", rolling windows", "calls": calls,
            "us_per_call": ms * 1e3 / calls, "us_per_call_device": ms_dev * 1e3 / calls,
            "committed_tokens_per_s": committed / (ms * 1e-3),
            "achieved_gbs": nbytes / (ms * 1e-3) / 1e9,
            "frac_of_peak_hbm": nbytes / (ms * 1e-3) / 1e9 / peak,
            "achieved_gbs_device": nbytes / (ms_dev * 1e-3) / 1e9,
            "frac_of_peak_hbm_device": nbytes / (ms_dev * 1e-3) / 1e9 / peak,
            "algorithmic_bytes_per_call": nbytes / calls,
            "gpu_launches_per_call": 4}


def run_cfg_engine(dev, rounds=256):
    """The engine loop from a fresh state, timed as called from Python and
    again with each round's work queued behind a short device sleep (the
    device time alone); the two passes must commit the same tokens."""
    paced = _engine_loop(dev, rounds, ahead=False)
    ahead = _engine_loop(dev, rounds, ahead=True)
    if ahead["outputs"] != paced["outputs"]:
        raise RuntimeError("engine loop: the device-timed pass differs")
    out = {k: v for k, v in paced.items() if k != "outputs"}
    out["ms_per_round_device"] = ahead["ms_per_round"]
    out["committed_tokens_per_s_device"] = ahead["committed_tokens_per_s"]
    return out


def _engine_loop(dev, rounds, ahead):
    """Engine loop: 64 sequences x 256 rounds, K = N_i = 4, V=32000 bf16,
    logits regenerated each round from a generator seeded by (4, round); each
    round reserves the cycle's slots in the block tables, drafts its K tokens
    per sequence from the L_d rows with the library's draft step (the K rows
    of each window gathered, one draw per row with the Philox counter
    (sequence, round, slot)), verifies, commits the committed tokens and
    rolls the reservation back (block 16, pool of 65536 blocks, starts
    U[128, 2048]). Committed tokens per second of the device work, with and
    without the round's logit generation (ahead: the work queued behind a
    device sleep, without the generation)."""
    from speculative_decoding_verification_89_b200 import capi
    from speculative_decoding_verification_89_b200 import workloads as W
    B, K, Ni, V = 64, 4, 4, 32000
    S = Ni + K + 1
    ctx = W.context_lengths(B, 128, 2048, seed=4)
    max_blocks = (max(ctx) + rounds * S + S) // 16 + 2
    state = W.paged_state(ctx, 16, max_blocks, 65536, device=dev)
    committed = state.seq_lens.clone()
    T = torch.ones(B, device=dev)
    seq_id = torch.arange(B, dtype=torch.int32, device=dev)
    full = torch.full((B,), S, dtype=torch.int32, device=dev)
    loop = HierLoop(B, K, Ni, V, torch.bfloat16, dev)
    st = torch.zeros(1, dtype=torch.int32, device=dev)
    draft_rows = torch.empty((B * K, V), dtype=torch.bfloat16, device=dev)
    draft_ws = capi.draft_workspace(B * K, V, torch.bfloat16, device=dev)
    draft_sid = seq_id.repeat_interleave(K)
    draft_T = torch.ones(B * K, device=dev)
    draft_tok = torch.empty(B * K, dtype=torch.int32, device=dev)
    kk = torch.arange(K, dtype=torch.int32, device=dev).view(1, K)
    base_row = torch.arange(B, device=dev).view(B, 1) * S  # int64: the flat row index
    ms_work = ms_all = 0.0
    total = 0
    h = hashlib.sha256()
    for r in range(rounds):
        a0 = torch.cuda.Event(enable_timing=True)
        a0.record()
        fresh, _ = W.engine_round_logits(B, S, V, r, dev)
        loop.logits(fresh)
        if ahead:
            torch.cuda.synchronize()
            torch.cuda._sleep(400_000)  # ~200 us: the host queues the round meanwhile
        w0 = torch.cuda.Event(enable_timing=True)
        w0.record()
        capi.spec_commit_paged(state.tables, state.seq_lens, committed, full, 0,
                               state.free_stack, state.free_top, S, st, block_size=16)
        slots = loop.win_len.view(B, 1) + kk  # the window's next K slots (int32)
        torch.index_select(loop.lg[0].view(B * S, V), 0, (base_row + slots).view(-1),
                           out=draft_rows)  # whole rows: (b, slot) -> b * S + slot
        capi.spec_draft_sample(draft_rows, draft_T, 40, draft_sid, r, slots.view(-1), draft_tok,
                               st, draft_ws)
        loop.call(draft_tok.view(B, K), T, 4, seq_id, r)
        capi.spec_commit_paged(state.tables, state.seq_lens, committed, loop.cn, 0,
                               state.free_stack, state.free_top, S, st, block_size=16)
        committed.copy_(state.seq_lens)
        w1 = torch.cuda.Event(enable_timing=True)
        w1.record()
        torch.cuda.synchronize()
        ms_work += w0.elapsed_time(w1)
        ms_all += a0.elapsed_time(w1)
        total += int(loop.cn.sum().item())
        h.update(loop.ctok.cpu().numpy().tobytes())
    h.update(state.tables.cpu().numpy().tobytes())
    if int(st.item()) != 0 or int(loop.status.item()) != 0:
        raise RuntimeError("engine loop: device status")
    return {"workload": "engine loop 64 sequences x 256 rounds, K=N_i=4, V=32000 bf16, drafts "
                        "by the draft step, paged commit/rollback every round (block 16, pool "
                        "65536)",
            "rounds": rounds, "committed_tokens": total,
            "committed_tokens_per_s": total / (ms_work * 1e-3),
            "committed_tokens_per_s_with_logit_generation": total / (ms_all * 1e-3),
            "ms_per_round": ms_work / rounds, "ms_per_round_with_logit_generation": ms_all / rounds,
            "outputs": h.hexdigest()}


# ----------------------------------------------------------------------------
# Oracle throughput per configuration on the host cores
# ----------------------------------------------------------------------------
ORACLE_CFG = {
    # kind: (description of one task, tasks per process)
    "chain_small": ("20 rounds of B=1, K=4, V=1024 chain verification", 2),
    "hier_peaked": ("one sequence, 6 rolling two-stage rounds, K=N_i=4, V=32000, peaked rows", 2),
    "chain_commit": ("one sequence-round of B=64-shape chain verification (K=8, V=128256) "
                     "plus its paged commit", 2),
    "hier_mixed": ("one sequence, 8 rolling two-stage rounds, K=N_i=4, V=151936", 1),
    "engine": ("one sequence, 8 rolling two-stage rounds with paged commit, K=N_i=4, V=32000", 2),
    "draft": ("16 draft rows of V=128256 (N(0,4) + Zipf(1.1)), token + ln q + entropy", 2),
    "saguaro": ("16 draft rows of V=128256: 32 cached ids lowered (eps 0.5, bf16 form), then "
                "the draft step", 2),
    "outcome": ("one sequence's outcome law, K=8, V=128256, 32 outcomes", 2),
    "chain": ("one sequence-round of B=64-shape chain verification (K=8, V=128256)", 2),
}
ORACLE_UNIT = {"outcome": "sequences/s"}


def _softmax_draw(rows, T, rng):
    """Drafts by the Gumbel-max construction from rows [n, V] at temperature T."""
    if T == 0.0:
        return rows.argmax(axis=1)
    g = -np.log(-np.log(rng.random(rows.shape)))
    return (rows / T + g).argmax(axis=1)


def _oracle_task(job):
    """One task of oracle work on inputs drawn (numpy) with the recipe of the
    configuration; returns (pid, tokens, seconds spent in the oracle)."""
    kind, i = job
    from oracle.commit import commit_paged
    from oracle.philox import STAGE_ONE, STAGE_TWO, PhiloxUniforms
    from oracle.verify import verify_chain, verify_hier_seq
    rng = np.random.default_rng(7000 + 13 * i + len(kind))
    tok, sec = 0, 0.0

    def hier_rounds(V, rounds, fstd, inoise, dnoise, T, boost=0.0, commit=False):
        nonlocal tok, sec
        K, Ni = 4, 4
        S = Ni + K + 1
        lf = rng.normal(0, fstd, (S, V))
        if boost:
            lf += boost * (rng.random((S, V)) < 0.05)
        rows = [lf + rng.normal(0, dnoise, (S, V)), lf + rng.normal(0, inoise, (S, V)), lf]
        window = []
        length = int(rng.integers(128, 2048))
        table = np.arange((length + S * rounds) // 16 + 4, dtype=np.int64)
        for r in range(rounds):
            w = len(window)
            fresh_f = rng.normal(0, fstd, (S, V))
            fresh = [fresh_f + rng.normal(0, dnoise, (S, V)), fresh_f + rng.normal(0, inoise, (S, V)),
                     fresh_f]
            for e in range(3):
                rows[e][w:] = fresh[e][w:]
            drafts = _softmax_draw(rows[0][w:w + K], T, rng)
            t0 = time.perf_counter()
            res = verify_hier_seq(rows[0], rows[1], rows[2], drafts, T, window, Ni,
                                  PhiloxUniforms(5, i, r, STAGE_ONE),
                                  PhiloxUniforms(5, i, r, STAGE_TWO))
            n = len(res.committed)
            if commit:
                stack = np.zeros(1064, dtype=np.int64)
                stack[:64] = np.arange(1000, 1064)
                commit_paged(table[None, :], np.array([length + S]), np.array([length]),
                             np.array([n]), stack, 64, 16, 1064, S)
            sec += time.perf_counter() - t0
            tok += n
            length += n
            window = list(res.window) if res.stage2 is None else []

    if kind == "chain_small":
        for r in range(20):
            tgt = rng.normal(0, 2, (1, 5, 1024))
            drf = tgt[:, :4] + rng.normal(0, 1, (1, 4, 1024))
            drafts = _softmax_draw(drf[0], 1.0, rng)[None, :]
            t0 = time.perf_counter()
            res = verify_chain(tgt, drf, drafts, np.array([1.0]), 0, np.array([i]), r)
            sec += time.perf_counter() - t0
            tok += res[0].accepted + 1
    elif kind == "chain_commit":
        V = 128256
        prior = -1.1 * np.log(np.arange(V) + 1.0)
        tgt = (rng.normal(0, 2, (1, 9, V)) + prior).astype(np.float32).astype(np.float64)
        drf = (tgt[:, :8] + rng.normal(0, 1, (1, 8, V))).astype(np.float32).astype(np.float64)
        drafts = _softmax_draw(drf[0], 1.0, rng)[None, :]
        length = int(rng.integers(512, 4096))
        tabs = np.arange((length + 9) // 16 + 2, dtype=np.int64)[None, :]
        t0 = time.perf_counter()
        res = verify_chain(tgt, drf, drafts, np.array([1.0]), 2, np.array([i]), 0)[0]
        stack = np.zeros(1032, dtype=np.int64)
        stack[:32] = np.arange(1000, 1032)
        commit_paged(tabs, np.array([length]), np.array([length]), np.array([res.accepted + 1]),
                     stack, 32, 16, 1032, 9)
        sec += time.perf_counter() - t0
        tok += res.accepted + 1
    elif kind in ("draft", "saguaro"):
        from oracle.draft import draft_step, saguaro_logits
        V = 128256
        prior = -1.1 * np.log(np.arange(V) + 1.0)
        lg = (rng.normal(0, 2, (16, V)) + prior).astype(np.float32).astype(np.float64)
        T = np.ones(16)
        cached = np.argsort(-lg, axis=1)[:, :32] if kind == "saguaro" else None
        t0 = time.perf_counter()
        if kind == "saguaro":
            lg = np.stack([saguaro_logits(lg[r], 1.0, cached[r], 0.5, "bf16") for r in range(16)])
        draft_step(lg, T, 5, np.arange(16) + 100 * i, 0, np.zeros(16, dtype=np.int64))
        sec += time.perf_counter() - t0
        tok += 16
    elif kind == "outcome":
        from oracle.outcome import outcome_law, top_outcomes
        V = 128256
        prior = -1.1 * np.log(np.arange(V) + 1.0)
        tgt = (rng.normal(0, 2, (9, V)) + prior).astype(np.float32).astype(np.float64)
        drf = (tgt[:8] + rng.normal(0, 1, (8, V))).astype(np.float32).astype(np.float64)
        drafts = _softmax_draw(drf, 1.0, rng)
        t0 = time.perf_counter()
        top_outcomes(outcome_law(tgt, drf, drafts, 1.0), 32)
        sec += time.perf_counter() - t0
        tok += 1
    elif kind == "chain":
        V = 128256
        prior = -1.1 * np.log(np.arange(V) + 1.0)
        tgt = (rng.normal(0, 2, (1, 9, V)) + prior).astype(np.float32).astype(np.float64)
        drf = (tgt[:, :8] + rng.normal(0, 1, (1, 8, V))).astype(np.float32).astype(np.float64)
        drafts = _softmax_draw(drf[0], 1.0, rng)[None, :]
        t0 = time.perf_counter()
        res = verify_chain(tgt, drf, drafts, np.array([1.0]), 2, np.array([i]), 0)[0]
        sec += time.perf_counter() - t0
        tok += res.accepted + 1
    elif kind == "hier_peaked":
        hier_rounds(32000, 6, 2.5, 0.7, 1.5, 0.7, boost=6.0)
    elif kind == "hier_mixed":
        hier_rounds(151936, 8, 2.0, 0.5, 2.0, float(rng.uniform(0.05, 1.2)))
    elif kind == "engine":
        hier_rounds(32000, 8, 2.0, 0.5, 1.0, 1.0, commit=True)
    return os.getpid(), tok, sec


_POOL = None


def start_oracle_pool():
    """A process pool for the oracle, forked before any GPU call (a process
    forked after CUDA starts would hang); one process per host core, at most
    64."""
    global _POOL
    import multiprocessing as mp
    n = max(1, min(os.cpu_count() or 1, 64))
    os.environ.setdefault("OMP_NUM_THREADS", "1")
    _POOL = mp.get_context("fork").Pool(n)
    return n


def oracle_rates(kind):
    """Oracle tokens per second for one configuration: single-threaded (tasks
    run in turn in this process), and with one process per core (tokens over
    the busiest process's oracle time)."""
    desc, per = ORACLE_CFG[kind]
    one = [_oracle_task((kind, 10_000 + k)) for k in range(per)]
    r1 = sum(t for _, t, _ in one) / max(sum(s for _, _, s in one), 1e-9)
    out = {"unit": ORACLE_UNIT.get(kind, "tokens/s"), "kind": "oracle", "task": desc,
           "single_thread": r1}
    if _POOL is not None:
        procs = _POOL._processes
        res = _POOL.map(_oracle_task, [(kind, k) for k in range(procs * per)])
        busy = {}
        for pid, _, sec in res:
            busy[pid] = busy.get(pid, 0.0) + sec
        out["all_cores"] = sum(t for _, t, _ in res) / max(max(busy.values()), 1e-9)
        out["cores"] = procs
        out["tasks"] = len(res)
    return out


def run_configs(args, dev, dist, peak, head):
    """Every configuration at one GPU: config 1 (latency), 2 and 4 (rolling
    two-stage loops), 3 (the headline step above), 5 (engine loop), each with
    the oracle's throughput on one host core and on all of them."""
    with_oracle = dist.world == 1 and dist.rank == 0 and not args.no_cpu_baseline
    out = {
        "cfg1_chain_small": run_cfg_chain_small(dev, dist),
        "cfg2_hier_peaked": run_cfg_hier(dev, peak, "peaked", rounds=24),
        "cfg3_chain_commit": {"workload": "the headline step", "tokens_per_s": head["value"],
                              "ms_per_step": head["ms_per_step"], "hbm_gbs": head["hbm_gbs"],
                              "frac_of_peak_hbm": head["hbm_frac_of_measured"]},
        "cfg4_hier_mixed": run_cfg_hier(dev, peak, "mixed", rounds=10),
        "cfg5_engine_loop": run_cfg_engine(dev),
    }
    if with_oracle:
        for key, kind in (("cfg1_chain_small", "chain_small"), ("cfg2_hier_peaked", "hier_peaked"),
                          ("cfg3_chain_commit", "chain_commit"), ("cfg4_hier_mixed", "hier_mixed"),
                          ("cfg5_engine_loop", "engine")):
            out[key]["oracle"] = oracle_rates(kind)
    return out


def run_e2e(args, prob, state, bufs, base, dev, dist):
    """Same step through the public API with pinned host inputs: each step
    copies its logits, drafts, temperatures, ids and staged K/V + hidden rows
    host->device and reads accept lengths and tokens back."""
    from speculative_decoding_verification_89_b200 import capi
    steps = max(3, min(args.steps, 100))
    host = {k: v.cpu().pin_memory() for k, v in
            dict(tgt=prob.tgt, drf=prob.drf, dt=prob.draft_tok, T=prob.temperature,
                 sid=prob.seq_id, kv=bufs.kv_stage, hid=bufs.hid_stage).items()}
    d = {k: torch.empty_like(v, device=dev) for k, v in host.items()}
    acc = torch.empty(B, dtype=torch.int32, device=dev)
    out = torch.empty((B, K + 1), dtype=torch.int32, device=dev)
    acc_h = torch.empty((steps, B), dtype=torch.int32).pin_memory()
    out_h = torch.empty((steps, B, K + 1), dtype=torch.int32).pin_memory()
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    ws = capi.workspace(B, K, V, torch.bfloat16, device=dev)
    stream = torch.cuda.current_stream()
    h2d = sum(v.numel() * v.element_size() for v in host.values())
    d2h = acc.numel() * 4 + out.numel() * 4

    def step(i):
        for k in host:
            d[k].copy_(host[k], non_blocking=True)
        capi.spec_verify_chain_commit(d["tgt"], d["drf"], d["dt"], d["T"], prob.seed, d["sid"],
                                      i, acc, out, state.tables, state.seq_lens, base,
                                      state.free_stack, state.free_top, status, ws,
                                      block_size=16, kv_stage=d["kv"], kv_pool=bufs.kv_pool,
                                      hid_stage=d["hid"], hid_out=bufs.hid_out,
                                      hid_off=bufs.hid_off, stream=stream)
        acc_h[i].copy_(acc, non_blocking=True)
        out_h[i].copy_(out, non_blocking=True)

    for i in range(3):
        step(i)
    torch.cuda.synchronize()
    dist.barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for i in range(steps):
        step(i)
    e1.record(stream)
    torch.cuda.synchronize()
    ms = dist.reduce(e0.elapsed_time(e1), "max")
    tokens = dist.reduce(float((acc_h.numpy() + 1).sum()), "sum")
    if int(status.item()) != 0:
        raise RuntimeError("device status during e2e run")
    return {"value": tokens / (ms * 1e-3), "unit": "tokens/s", "h2d_bytes_per_step": h2d,
            "d2h_bytes_per_step": d2h, "steps": steps}


# ----------------------------------------------------------------------------
# Reference arm: the oracle on the host cores
# ----------------------------------------------------------------------------
def run_reference(args, dist):
    from speculative_decoding_verification_89_b200 import workloads as W
    prob = W.chain_batch(device="cpu")
    state, _ = W.commit_setup(B, K, device="cpu", with_kv=False)
    hp, tables, lens, stack, top = host_problem(prob, state)
    # One step = one sequence-round; bounded so the whole run takes minutes.
    _, t1 = run_oracle_steps(hp, tables, lens, stack, top, [0], 1)
    steps = max(3, min(args.steps, int(120.0 / max(t1, 1e-3))))
    warm = max(1, min(args.warmup, 3))
    run_oracle_steps(hp, tables, lens, stack, top, list(range(B)), warm)
    tok, sec = run_oracle_steps(hp, tables, lens, stack, top, list(range(B)), steps, rnd0=warm)
    value = tok / sec
    sample = (f"{steps} sequence-rounds (one sequence's chain verify + commit per step) of the "
              f"B=64 K=8 V=128256 workload, fp64 numpy oracle, single thread")
    return {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s",
        "n_gpus": dist.world, "steps": steps, "warmup": warm, "ms_per_step": sec * 1e3 / steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic", "config": {"workload": WORKLOAD, "logits_dtype": "bf16"},
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": 1, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }


def main():
    args = parse()
    if args.gpus > 1 and "WORLD_SIZE" not in os.environ:
        return relaunch(args)
    dist = Dist()
    if dist.world != args.gpus:
        print(f"bench.py: --gpus {args.gpus} but WORLD_SIZE={dist.world}; running "
              f"{dist.world} rank(s)", file=sys.stderr)
    if args.plan_only:
        dist.init("gloo")
        plans = [rank_plan(dist)]
        if dist.pg:
            plans = [None] * dist.world
            dist.pg.all_gather_object(plans, rank_plan(dist))
        if dist.rank == 0:
            print(json.dumps({"plans": plans}), flush=True)
        dist.close()
        return 0
    if args.impl == "reference":
        if dist.rank == 0:
            print(json.dumps(run_reference(args, dist)), flush=True)
        return 0
    if dist.world == 1 and dist.rank == 0 and not args.no_cpu_baseline:
        start_oracle_pool()  # before the first GPU call
    dist.init("nccl")
    try:
        res = run_ours(args, dist)
        if dist.rank == 0:
            print(json.dumps(res), flush=True)
    finally:
        if _POOL is not None:
            _POOL.terminate()
            _POOL.join()
        dist.close()
    return 0


if __name__ == "__main__":
    sys.exit(main())
