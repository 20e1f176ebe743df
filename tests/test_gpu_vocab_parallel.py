"""Vocabulary-parallel chain verification on the GPU against the oracle.

The oracle checks whole rows; the vocabulary-parallel path never holds one.
Every rank gets only its columns [v0, v0 + Vs) of the rows, and the ranks
exchange only their records and masses. The acceptance rule is the chain
check's (accepted counts and tokens bit-exact except at decisions within the
1e-6 fp64 margin, counted, share below 1e-4; probabilities within 1e-5
relative). Every rank must also end with identical outputs.

Most tests run the R ranks in one process: each launch for every shard, and
the exchanges as plain stacking of their outputs in rank order. Two tests go
through torch.distributed: two gloo processes sharing the GPU (their kernels
never wait on one another; only the host collectives do), and a world of one
NCCL rank, which takes the device-tensor collectives."""
import os
import socket
import sys

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

from speculative_decoding_verification_89_b200 import workloads as W
from tests.gpu_run import padded, run_chain_gpu, run_chain_oracle
from tests.parity import Tally, compare_check, compare_probs

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _cols(t, v0, Vs):
    """Device copy of columns [v0, v0 + Vs) of [B, n, V] rows, rows 16-byte
    aligned (what a vocabulary-parallel LM head leaves on one rank)."""
    return padded(t[:, :, v0:v0 + Vs].contiguous().to("cuda"))


def run_vp(prob, R, diag=True):
    """The R ranks in one process. Returns (acc, out, diag, status) of rank 0
    after checking that every rank holds the same."""
    from speculative_decoding_verification_89_b200.vocab_parallel import ChainShard, vocab_shards
    B, Kp1, V = prob.tgt.shape
    K = Kp1 - 1
    dev = torch.device("cuda")
    dt = prob.draft_tok.to(dev).contiguous()
    T = prob.temperature.to(dev)
    sid = prob.seq_id.to(dev)
    ranks = []
    for r, (v0, Vs) in enumerate(vocab_shards(V, R)):
        sh = ChainShard(B, K, V, v0, Vs, R, r, prob.tgt.dtype, device=dev)
        tgt = _cols(prob.tgt, v0, Vs)
        drf = _cols(prob.drf, v0, Vs) if K > 0 else None
        ranks.append(dict(sh=sh, tgt=tgt, drf=drf,
                          st=torch.zeros(1, dtype=torch.int32, device=dev),
                          acc=torch.full((B,), -7, dtype=torch.int32, device=dev),
                          out=torch.full((B, K + 1), -7, dtype=torch.int32, device=dev),
                          dg=torch.full((B, 4 * K + 2), -7.0, dtype=torch.float64, device=dev)
                          if diag else None))
    for x in ranks:
        x["sh"].stats(x["tgt"], x["drf"], dt, T, x["st"])
    rows_all = torch.stack([x["sh"].rows for x in ranks])
    for x in ranks:
        x["sh"].rows_all.copy_(rows_all)
        x["sh"].decide(x["tgt"], x["drf"], dt, T, prob.seed, sid, prob.rnd, x["st"], diag=x["dg"])
    mass_all = torch.stack([x["sh"].mass for x in ranks])
    for x in ranks:
        x["sh"].mass_all.copy_(mass_all)
        x["sh"].pick(x["tgt"], x["drf"], dt, T, x["acc"], x["out"], x["st"], diag=x["dg"])
    out = torch.stack([x["out"] for x in ranks]).amax(0)
    torch.cuda.synchronize()
    for x in ranks[1:]:
        assert torch.equal(x["acc"], ranks[0]["acc"])
        assert int(x["st"].item()) == int(ranks[0]["st"].item())
        if diag:
            assert np.array_equal(x["dg"].cpu().numpy(), ranks[0]["dg"].cpu().numpy(),
                                  equal_nan=True)
    return (ranks[0]["acc"].cpu().numpy(), out.cpu().numpy(),
            ranks[0]["dg"].cpu().numpy() if diag else None, int(ranks[0]["st"].item()))


def _compare(prob, R, tag, tally, seqs=None):
    acc, out, diag, st = run_vp(prob, R)
    assert st == 0, f"{tag}: device status {st}"
    ref = run_chain_oracle(prob, seqs)
    K = prob.draft_tok.shape[1]
    for b, r in ref.items():
        a = int(acc[b])
        toks = [int(x) for x in out[b, :a + 1]]
        assert all(int(x) == -1 for x in out[b, a + 1:]), f"{tag}: padding"
        if compare_check(f"{tag}/seq{b}", r, a, toks, tally):
            compare_probs(f"{tag}/seq{b}", r, diag[b], K, float(prob.temperature[b]))
    return acc, out


@pytest.mark.parametrize("R", [2, 3, 8])
def test_vp_full_size_batch(R):
    """B=64, K=8, V=128256 bf16 chain batch, vocabulary over R ranks; also
    against the one-GPU check on the same inputs."""
    tally = Tally()
    same = 0
    for rnd in range(2 if R == 2 else 1):
        prob = W.chain_batch(rnd=rnd)
        acc, out = _compare(prob, R, f"R{R}/r{rnd}", tally)
        a1, o1, _, _ = run_chain_gpu(prob, diag=False)
        same += int(np.array_equal(acc, a1) and np.array_equal(out, o1))
    tally.check_share()
    assert same == (2 if R == 2 else 1) or tally.excused > 0


EDGE = [
    # B, K, V, dtype, temperature spec, ranks
    (3, 0, 1000, torch.float32, 1.0, 2),          # no drafts: plain draw from p
    (2, 1, 1, torch.float32, 1.0, 1),             # single-token vocabulary, one shard
    (4, 3, 4097, torch.bfloat16, 0.8, 3),         # ragged last shard
    (5, 2, 12345, torch.bfloat16, "mixed", 2),    # greedy and sampled in a batch
    (2, 40, 3000, torch.bfloat16, 1.0, 2),        # K > 32
    (3, 5, 777, torch.bfloat16, 0.0, 2),          # all greedy
    (6, 4, 50000, torch.bfloat16, 1e-3, 4),       # near-greedy
    (6, 4, 50000, torch.float32, 50.0, 4),        # flat laws
    (3, 6, 70000, torch.float32, 0.7, 5),         # fp32, five shards
]


@pytest.mark.parametrize("B,K,V,dtype,tspec,R", EDGE)
def test_vp_edge_cases(B, K, V, dtype, tspec, R):
    if tspec == "mixed":
        T = torch.tensor([0.0, 0.5, 1.0, 0.0, 2.0])[:B]
    else:
        T = float(tspec)
    tally = Tally()
    for rnd in range(3):
        prob = W.chain_problem(B, K, V, dtype, seed=40 + K, rnd=rnd, temperature=T)
        _compare(prob, R, f"edge/r{rnd}", tally)
    tally.check_share()


def test_vp_masked_shard_and_equal_laws():
    """A shard whose columns are all -inf in some rows (drafts there have
    p = 0), and sequences whose draft law equals the target law (every draft
    accepted, bonus token from p_K across the shards)."""
    prob = W.chain_problem(6, 4, 9000, torch.bfloat16, seed=51, temperature=0.9)
    tgt, drf = prob.tgt.clone(), prob.drf.clone()
    tgt[0, :, 3072:6144] = float("-inf")           # shard 1 of 3 masked in sequence 0
    drf[1] = tgt[1, :4]                            # equal laws
    drf[2] = tgt[2, :4]
    prob.tgt, prob.drf = tgt, drf
    tally = Tally()
    acc, _ = _compare(prob, 3, "masked", tally)
    assert acc[1] == 4 and acc[2] == 4


def test_vp_invalid_values_match_the_one_gpu_check():
    """A drafted id outside [0, V), an invalid temperature and a NaN logit in
    one shard: the sequences are flagged as the one-GPU check flags them, on
    every rank; the others match the oracle."""
    prob = W.chain_problem(5, 3, 2000, torch.float32, seed=6, temperature=1.0)
    prob.draft_tok[1, 2] = 2000
    prob.temperature[2] = -1.0
    prob.tgt[3, 1, 1500] = float("nan")
    acc, out, _, st = run_vp(prob, 2)
    a1, o1, _, st1 = run_chain_gpu(prob, diag=False)
    assert st == st1 == -6
    assert np.array_equal(acc, a1) and np.array_equal(out, o1)
    assert acc[1] == -1 and acc[2] == -1
    ref = run_chain_oracle(prob, [0, 4])
    tally = Tally()
    for b in (0, 4):
        compare_check(f"seq{b}", ref[b], int(acc[b]), list(out[b, :acc[b] + 1]), tally)


def test_vp_host_checks():
    from speculative_decoding_verification_89_b200 import capi
    from speculative_decoding_verification_89_b200.vocab_parallel import ChainShard
    prob = W.chain_problem(2, 2, 1000, torch.float32, seed=3)
    sh = ChainShard(2, 2, 1000, 512, 488, 2, 1, torch.float32)
    tgt = _cols(prob.tgt, 512, 488)
    drf = _cols(prob.drf, 512, 488)
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    dt, T = prob.draft_tok.cuda(), prob.temperature.cuda()
    with pytest.raises(capi.SpecError) as e:      # shard past the vocabulary
        capi.spec_vp_shard_stats(tgt, drf, 600, 1000, dt, T, sh.rows, st, sh.ws)
    assert e.value.code == capi.SPEC_EINVAL
    with pytest.raises(capi.SpecError) as e:      # rank outside [0, R)
        capi.spec_vp_decide(tgt, drf, 512, 1000, 2, 2, sh.rows_all, dt, T, 0,
                            prob.seq_id.cuda(), 0, sh.mass, st, sh.ws)
    assert e.value.code == capi.SPEC_EINVAL
    with pytest.raises(capi.SpecError) as e:      # workspace too small
        capi.spec_vp_pick(tgt, drf, 512, 1000, 2, 1, sh.mass_all, dt, T,
                          torch.zeros(2, dtype=torch.int32, device="cuda"),
                          torch.zeros((2, 3), dtype=torch.int32, device="cuda"), st, sh.ws[:64])
    assert e.value.code == capi.SPEC_EWORKSPACE


# ---------------------------------------------------------------------------
# Two processes, gloo
# ---------------------------------------------------------------------------
def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    sys.path.insert(0, ROOT)
    import datetime

    import torch.distributed as dist
    from speculative_decoding_verification_89_b200.vocab_parallel import (
        ChainShard, verify_chain_vocab_parallel, vocab_shards)
    from speculative_decoding_verification_89_b200 import workloads as W2
    try:
        torch.cuda.set_device(0)
        dist.init_process_group("gloo", rank=rank, world_size=world,
                                timeout=datetime.timedelta(seconds=120))
        prob = W2.chain_batch(rnd=1)
        B, Kp1, V = prob.tgt.shape
        K = Kp1 - 1
        v0, Vs = vocab_shards(V, world)[rank]
        tgt = prob.tgt[:, :, v0:v0 + Vs].contiguous().cuda()
        drf = prob.drf[:, :, v0:v0 + Vs].contiguous().cuda()
        sh = ChainShard(B, K, V, v0, Vs, world, rank, prob.tgt.dtype)
        acc = torch.full((B,), -7, dtype=torch.int32, device="cuda")
        out = torch.full((B, K + 1), -7, dtype=torch.int32, device="cuda")
        dg = torch.zeros((B, 4 * K + 2), dtype=torch.float64, device="cuda")
        st = torch.zeros(1, dtype=torch.int32, device="cuda")
        verify_chain_vocab_parallel(sh, tgt, drf, prob.draft_tok.cuda(), prob.temperature.cuda(),
                                    prob.seed, prob.seq_id.cuda(), prob.rnd, acc, out, st,
                                    diag=dg)
        torch.cuda.synchronize()
        dist.barrier()
        dist.destroy_process_group()
        q.put((rank, acc.cpu().numpy(), out.cpu().numpy(), dg.cpu().numpy(), int(st.item())))
    except Exception as exc:  # report instead of leaving the parent waiting
        q.put((rank, repr(exc), None, None, None))
        raise


def test_vp_two_gloo_processes_on_one_gpu():
    port = _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted((q.get(timeout=300) for _ in procs), key=lambda x: x[0])
    for p in procs:
        p.join(timeout=120)
    assert all(r[2] is not None for r in res), res
    assert all(p.exitcode == 0 for p in procs)
    (_, a0, o0, d0, s0), (_, a1, o1, d1, s1) = res
    assert s0 == s1 == 0
    assert np.array_equal(a0, a1) and np.array_equal(o0, o1)
    assert np.array_equal(d0, d1, equal_nan=True)
    prob = W.chain_batch(rnd=1)
    ref = run_chain_oracle(prob)
    tally = Tally()
    K = prob.draft_tok.shape[1]
    for b, r in ref.items():
        a = int(a0[b])
        if compare_check(f"gloo/seq{b}", r, a, [int(x) for x in o0[b, :a + 1]], tally):
            compare_probs(f"gloo/seq{b}", r, d0[b], K, float(prob.temperature[b]))
    tally.check_share()


# ---------------------------------------------------------------------------
# One rank over NCCL: the device-tensor exchange calls
# ---------------------------------------------------------------------------
def _nccl_worker(port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    sys.path.insert(0, ROOT)
    import datetime

    import torch.distributed as dist
    from speculative_decoding_verification_89_b200.vocab_parallel import (
        ChainShard, verify_chain_vocab_parallel)
    from speculative_decoding_verification_89_b200 import workloads as W2
    try:
        torch.cuda.set_device(0)
        dist.init_process_group("nccl", rank=0, world_size=1,
                                timeout=datetime.timedelta(seconds=120))
        prob = W2.chain_problem(16, 4, 5000, torch.bfloat16, seed=77, temperature=0.9)
        B, Kp1, V = prob.tgt.shape
        K = Kp1 - 1
        sh = ChainShard(B, K, V, 0, V, 1, 0, prob.tgt.dtype)
        acc = torch.full((B,), -7, dtype=torch.int32, device="cuda")
        out = torch.full((B, K + 1), -7, dtype=torch.int32, device="cuda")
        st = torch.zeros(1, dtype=torch.int32, device="cuda")
        verify_chain_vocab_parallel(sh, prob.tgt.cuda(), prob.drf.cuda(), prob.draft_tok.cuda(),
                                    prob.temperature.cuda(), prob.seed, prob.seq_id.cuda(),
                                    prob.rnd, acc, out, st)
        torch.cuda.synchronize()
        dist.destroy_process_group()
        q.put((acc.cpu().numpy(), out.cpu().numpy(), int(st.item())))
    except Exception as exc:  # report instead of leaving the parent waiting
        q.put((repr(exc), None, None))
        raise


def test_vp_one_rank_over_nccl():
    """A world of one NCCL rank holding the whole vocabulary: the exchanges
    take the device-tensor collectives (all_gather_into_tensor, all_reduce
    MAX) and the result is the oracle's check."""
    port = _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    p = ctx.Process(target=_nccl_worker, args=(port, q))
    p.start()
    acc, out, st = q.get(timeout=300)
    p.join(timeout=120)
    assert out is not None, acc
    assert p.exitcode == 0 and st == 0
    prob = W.chain_problem(16, 4, 5000, torch.bfloat16, seed=77, temperature=0.9)
    ref = run_chain_oracle(prob)
    tally = Tally()
    for b, r in ref.items():
        a = int(acc[b])
        compare_check(f"nccl/seq{b}", r, a, [int(x) for x in out[b, :a + 1]], tally)
    tally.check_share()
