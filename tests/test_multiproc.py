"""Multi-process host logic of bench.py on CPU with gloo (world size 2):
barrier, max-over-ranks timing and whole-job sums, disjoint per-rank
sequences, and the reference arm's rank-0-only behaviour."""
import json
import os
import socket
import subprocess
import sys

import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), WORLD_SIZE=str(world),
                      RANK=str(rank), LOCAL_RANK=str(rank))
    sys.path.insert(0, ROOT)
    import bench
    from speculative_decoding_verification_89_b200 import workloads as W
    d = bench.Dist()
    d.init("gloo")
    d.barrier()
    mx = d.reduce(10.0 + rank, "max")
    sm = d.reduce(1.0 + rank, "sum")
    p = W.chain_problem(4, 2, 64, torch.float32, seed=2 + 1000 * rank, seq_id_base=4 * rank)
    d.close()
    q.put((rank, mx, sm, p.seq_id.tolist(), float(p.tgt[0, 0, 0])))


def test_two_ranks_reduce_and_shard():
    port = _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    out = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert out[0][1] == out[1][1] == 11.0          # max over ranks
    assert out[0][2] == out[1][2] == 3.0           # whole-job sum
    assert set(out[0][3]).isdisjoint(out[1][3])    # each rank its own sequences
    assert out[0][4] != out[1][4]                  # and its own logits


def test_reference_arm_only_rank0_prints():
    env = dict(os.environ, WORLD_SIZE="2", RANK="1", LOCAL_RANK="1")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--steps", "3", "--warmup", "1"], env=env, capture_output=True,
                       text=True, timeout=300)
    assert r.returncode == 0 and r.stdout.strip() == ""


def test_reference_arm_json_line():
    env = dict(os.environ, WORLD_SIZE="1", RANK="0", LOCAL_RANK="0")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--steps", "3", "--warmup", "1"], env=env, capture_output=True,
                       text=True, timeout=600)
    assert r.returncode == 0, r.stderr[-2000:]
    line = json.loads(r.stdout.strip().splitlines()[-1])
    assert line["impl"] == "reference" and line["unit"] == "tokens/s" and line["value"] > 0
    assert line["cpu_baseline"]["kind"] == "oracle" and line["cpu_baseline"]["cores"] == 1
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["e2e"]["value"] == line["value"]


def test_gpus_flag_launches_one_rank_per_gpu():
    """`bench.py --gpus 2` outside a launcher starts two ranks itself (gloo
    here, --plan-only: no GPU work); each rank takes its own device index,
    its own sequences and its own seeds."""
    env = {k: v for k, v in os.environ.items()
           if k not in ("WORLD_SIZE", "RANK", "LOCAL_RANK", "MASTER_ADDR", "MASTER_PORT")}
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--gpus", "2",
                        "--plan-only"], env=env, capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [l for l in r.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1, r.stdout          # rank 0 alone prints
    plans = json.loads(lines[0])["plans"]
    assert [p["rank"] for p in plans] == [0, 1] and all(p["world"] == 2 for p in plans)
    assert [p["device"] for p in plans] == [0, 1]
    assert plans[0]["seq_id_base"] != plans[1]["seq_id_base"]
    assert plans[1]["seq_id_base"] - plans[0]["seq_id_base"] >= 64   # disjoint B=64 ranges
    assert plans[0]["logit_seed"] != plans[1]["logit_seed"]
    assert plans[0]["pool_seed"] != plans[1]["pool_seed"]
