"""The persistent-kernel entry points (spec_verify_chain_persistent,
spec_verify_chain_commit_persistent) against the oracle, through the C ABI,
with the chain and commit acceptance rules: the same contract as
spec_verify_chain and spec_verify_chain_commit, computed by one persistent
launch (after its prologue) instead of the staged launches."""
import numpy as np
import pytest
import torch

from speculative_decoding_verification_89_b200 import workloads as W
from tests.gpu_run import run_chain_gpu, run_chain_oracle
from tests.parity import Tally, compare_check, compare_probs
from tests.test_gpu_fused import _check_oracle, _run, _small_case

pytestmark = pytest.mark.gpu


def _verify(prob, tag, tally):
    acc, out, diag, st = run_chain_gpu(prob, persistent=True)
    assert st == 0, f"{tag}: device status {st}"
    K = prob.draft_tok.shape[1]
    for b, r in run_chain_oracle(prob).items():
        a = int(acc[b])
        toks = [int(x) for x in out[b, :a + 1]]
        assert all(int(x) == -1 for x in out[b, a + 1:]), f"{tag}: padding"
        if compare_check(f"{tag}/seq{b}", r, a, toks, tally):
            compare_probs(f"{tag}/seq{b}", r, diag[b], K, float(prob.temperature[b]))


@pytest.mark.parametrize("B,K,V,dtype,T", [
    (1, 4, 1024, torch.float32, 1.0),
    (7, 3, 4097, torch.bfloat16, torch.tensor([1.0, 0.0, 0.6, 2.0, 0.0, 0.9, 1.3])),
    (4, 6, 50000, torch.float32, torch.tensor([1e-3, 50.0, 0.0, 1.0])),
    (3, 0, 777, torch.bfloat16, 0.8),
    (2, 40, 3000, torch.bfloat16, 1.0),
])
def test_persistent_verify_shapes(B, K, V, dtype, T):
    tally = Tally()
    for rnd in range(3):
        prob = W.chain_problem(B, K, V, dtype, seed=5 * B + K, rnd=rnd,
                               temperature=T if isinstance(T, torch.Tensor) else float(T))
        _verify(prob, f"B{B}K{K}V{V}/r{rnd}", tally)
    tally.check_share()


def test_persistent_full_size_commit():
    """B=64, K=8, V=128256 bf16 with the commit of a + 1 rows per sequence."""
    tally = Tally()
    for rnd in range(2):
        prob = W.chain_batch(device="cuda", rnd=rnd)
        state, bufs = W.commit_setup(64, 8, device="cuda")
        state = W.PagedState(state.tables.cpu(), state.seq_lens.cpu(), state.free_stack.cpu(),
                             state.free_top.cpu(), 16)
        r = _run(prob, state, bufs, True, persistent=True)
        assert r["status"] == 0
        _check_oracle(prob, state, bufs, r, f"full/r{rnd}", tally)
    tally.check_share()


def test_persistent_commit_small_and_failures():
    tally = Tally()
    prob, state, bufs = _small_case(6, 4, 3000, torch.bfloat16,
                                    torch.tensor([1.0, 0.0, 0.7, 1.2, 0.9, 0.0]), seed=71)
    for rnd in range(3):
        prob.rnd = rnd
        r = _run(prob, state, bufs, True, persistent=True)
        _check_oracle(prob, state, bufs, r, f"small/r{rnd}", tally)
        state = r["state"]
        bufs = W.CommitBuffers(bufs.kv_stage, r["kv_pool"].cpu(), bufs.hid_stage,
                               r["hid_out"].cpu(), r["hid_off"].cpu())
    # an invalid temperature and draft id fail their sequences and block the commit
    prob, state, bufs = _small_case(4, 3, 1000, torch.float32, 1.0, seed=41)
    prob.temperature[2] = -1.0
    prob.draft_tok[1, 2] = 1000
    r = _run(prob, state, bufs, True, persistent=True)
    assert r["status"] == -6 and int(r["acc"][1]) == -1 and int(r["acc"][2]) == -1
    _check_oracle(prob, state, bufs, r, "invalid", tally)
    assert torch.equal(r["kv_pool"].cpu(), bufs.kv_pool)
    # a pool that cannot cover the kept rows fails the commit, nothing moves
    prob, state, bufs = _small_case(8, 6, 1000, torch.float32, 1.0, seed=43, spare=0,
                                    ctx=[4 * i for i in range(8)])
    r = _run(prob, state, bufs, True, persistent=True)
    assert r["status"] == -4
    _check_oracle(prob, state, bufs, r, "pool", tally)
    assert torch.equal(r["kv_pool"].cpu(), bufs.kv_pool)
    tally.check_share()
