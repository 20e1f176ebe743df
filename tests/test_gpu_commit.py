"""Paged commit / rollback on the GPU against the oracle, through the C ABI:
tables, lengths, free stack and gathered rows bit-exact; failures leave all
state untouched; block-table invariants after every call."""
import numpy as np
import pytest
import torch

from oracle.commit import check_invariants, commit_paged, gather_hidden
from speculative_decoding_verification_89_b200 import workloads as W
from tests.gpu_run import run_chain_gpu

pytestmark = pytest.mark.gpu


def _gpu_commit(state, base_len, keep, keep_add, Kp1, bufs=None, status=0):
    from speculative_decoding_verification_89_b200 import capi
    dev = "cuda"
    st = state.clone()
    t, l, f, top = (st.tables.to(dev), st.seq_lens.to(dev), st.free_stack.to(dev),
                    st.free_top.to(dev))
    s = torch.tensor([status], dtype=torch.int32, device=dev)
    kw = {}
    if bufs is not None:
        kw = dict(kv_stage=bufs.kv_stage.to(dev), kv_pool=bufs.kv_pool.to(dev),
                  hid_stage=bufs.hid_stage.to(dev), hid_out=bufs.hid_out.to(dev),
                  hid_off=bufs.hid_off.to(dev))
    capi.spec_commit_paged(t, l, None if base_len is None else base_len.to(dev),
                           keep.to(dev), keep_add, f, top, Kp1, s,
                           block_size=state.block_size, **kw)
    torch.cuda.synchronize()
    out = W.PagedState(t.cpu(), l.cpu(), f.cpu(), top.cpu(), state.block_size)
    return out, int(s.item()), {k: v.cpu() for k, v in kw.items()}


def _oracle(state, base_len, keep, keep_add, Kp1):
    base = state.seq_lens if base_len is None else base_len
    return commit_paged(state.tables.numpy(), state.seq_lens.numpy(), base.numpy(),
                        keep.numpy() + keep_add, state.free_stack.numpy(),
                        int(state.free_top[0]), state.block_size,
                        state.free_stack.numel(), Kp1)


def _assert_state(gpu, ref, bs):
    assert list(gpu.seq_lens.numpy()) == list(ref.seq_lens)
    assert int(gpu.free_top[0]) == ref.free_top
    assert np.array_equal(gpu.free_stack.numpy()[:ref.free_top], ref.free_stack[:ref.free_top])
    for b in range(len(ref.seq_lens)):
        nb = (int(ref.seq_lens[b]) + bs - 1) // bs
        assert np.array_equal(gpu.tables.numpy()[b, :nb], ref.tables[b, :nb])


@pytest.mark.parametrize("trial", range(40))
def test_random_tiny_pools(trial):
    rng = np.random.default_rng(500 + trial)
    B = int(rng.integers(1, 9))
    bs = int(rng.choice([1, 4, 16]))
    Kp1 = 5
    ctx = [int(x) for x in rng.integers(0, 3 * bs + 1, size=B)]
    need = sum((n + bs - 1) // bs for n in ctx)
    num_blocks = need + int(rng.integers(0, 6))
    max_blocks = max(1, (max(ctx) + Kp1 + bs - 1) // bs + 1)
    state = W.paged_state(ctx, bs, max_blocks, num_blocks)
    # Shuffle the pool so ids are not monotone.
    perm = torch.from_numpy(rng.permutation(num_blocks).astype(np.int32))
    nb = [(n + bs - 1) // bs for n in ctx]
    for b in range(B):
        state.tables[b, :nb[b]] = perm[state.tables[b, :nb[b]].long()]
    top = int(state.free_top[0])
    state.free_stack[:top] = perm[state.free_stack[:top].long()]
    L, H, D, hidden = 2, 1, 8, 8
    gen = W.generator(trial, "cpu")
    bufs = W.CommitBuffers(W.random_bf16((B, Kp1, L, 2, H, D), gen, "cpu"),
                           torch.zeros((num_blocks, L, 2, bs, H, D), dtype=torch.bfloat16),
                           W.random_bf16((B, Kp1, hidden), gen, "cpu"),
                           torch.zeros((B * Kp1, hidden), dtype=torch.bfloat16),
                           torch.zeros((B + 1,), dtype=torch.int32))
    for step in range(4):
        base = torch.tensor([int(rng.integers(0, n + 1)) for n in state.seq_lens],
                            dtype=torch.int32)
        keep = torch.from_numpy(rng.integers(-1, Kp1, size=B).astype(np.int32))
        ref = _oracle(state, base, keep, 1, Kp1)
        gpu, status, got = _gpu_commit(state, base, keep, 1, Kp1, bufs)
        assert status == ref.status, (status, ref.status)
        if ref.status != 0:
            for a, b in ((gpu.tables, state.tables), (gpu.seq_lens, state.seq_lens),
                         (gpu.free_stack, state.free_stack), (gpu.free_top, state.free_top)):
                assert torch.equal(a, b)
            continue
        _assert_state(gpu, ref, bs)
        assert check_invariants(gpu.tables.numpy(), gpu.seq_lens.numpy(),
                                gpu.free_stack.numpy(), int(gpu.free_top[0]), bs,
                                num_blocks) == []
        pool = got["kv_pool"].view(torch.int16).numpy()
        stage = bufs.kv_stage.view(torch.int16).numpy()
        for (b, i, blk, slot) in ref.destinations:
            assert np.array_equal(pool[blk, :, :, slot], stage[b, i])
        kept = (keep + 1).numpy()
        assert list(got["hid_off"].numpy()) == list(ref.hid_off)
        packed = gather_hidden(bufs.hid_stage.view(torch.int16).numpy(), kept)
        assert np.array_equal(got["hid_out"].view(torch.int16).numpy()[:len(packed)], packed)
        state = gpu
        bufs.kv_pool = got["kv_pool"]


def test_failures_leave_state_untouched():
    state = W.paged_state([5, 12, 3], 4, 4, 10)
    Kp1 = 5
    cases = [
        (torch.tensor([5, 6, 3]), torch.tensor([6, 0, 4]), -1),    # keep > K+1
        (torch.tensor([6, 6, 3]), torch.tensor([3, 0, 4]), -1),    # base beyond length
    ]
    for base, keep, code in cases:
        gpu, status, _ = _gpu_commit(state, base.int(), keep.int(), 0, Kp1)
        assert status == code
        assert torch.equal(gpu.tables, state.tables) and torch.equal(gpu.seq_lens, state.seq_lens)
        assert torch.equal(gpu.free_stack, state.free_stack)
        assert torch.equal(gpu.free_top, state.free_top)
    # pool exhausted: two blocks needed, one free, nothing freed
    tight = W.paged_state([5, 12, 3], 4, 4, 7)
    gpu, status, _ = _gpu_commit(tight, torch.tensor([5, 12, 3]).int(),
                                 torch.tensor([4, 0, 5]).int(), 0, Kp1)
    assert status == -4
    for a, b in ((gpu.tables, tight.tables), (gpu.seq_lens, tight.seq_lens),
                 (gpu.free_stack, tight.free_stack), (gpu.free_top, tight.free_top)):
        assert torch.equal(a, b)
    # a pending error blocks the commit entirely
    gpu, status, _ = _gpu_commit(state, None, torch.tensor([1, 1, 1], dtype=torch.int32), 0,
                                 Kp1, status=-6)
    assert status == -6 and torch.equal(gpu.tables, state.tables)


def test_chain_verify_then_commit_full_size():
    """B=64, K=8, V=128256 bf16 chain verification, then the commit of
    a + 1 rows per sequence into a paged pool (block 16, contexts U[512,
    4096], 128 KiB of K/V per token, hidden 4096): tables and every moved row
    against the oracle."""
    prob = W.chain_batch(device="cuda")
    acc, out, _, st = run_chain_gpu(prob, diag=False)
    assert st == 0
    state, bufs = W.commit_setup(64, 8, device="cuda")
    state_cpu = W.PagedState(state.tables.cpu(), state.seq_lens.cpu(), state.free_stack.cpu(),
                             state.free_top.cpu(), 16)
    keep = torch.from_numpy(acc.astype(np.int32))
    ref = _oracle(state_cpu, None, keep, 1, 9)
    assert ref.status == 0
    from speculative_decoding_verification_89_b200 import capi
    s = torch.zeros(1, dtype=torch.int32, device="cuda")
    capi.spec_commit_paged(state.tables, state.seq_lens, None, keep.cuda(), 1,
                           state.free_stack, state.free_top, 9, s, block_size=16,
                           kv_stage=bufs.kv_stage, kv_pool=bufs.kv_pool,
                           hid_stage=bufs.hid_stage, hid_out=bufs.hid_out, hid_off=bufs.hid_off)
    torch.cuda.synchronize()
    assert int(s.item()) == 0
    gpu = W.PagedState(state.tables.cpu(), state.seq_lens.cpu(), state.free_stack.cpu(),
                       state.free_top.cpu(), 16)
    _assert_state(gpu, ref, 16)
    assert check_invariants(gpu.tables.numpy(), gpu.seq_lens.numpy(), gpu.free_stack.numpy(),
                            int(gpu.free_top[0]), 16, gpu.free_stack.numel()) == []
    for (b, i, blk, slot) in ref.destinations:
        assert torch.equal(bufs.kv_pool[blk, :, :, slot], bufs.kv_stage[b, i])
    kept = acc + 1
    assert list(bufs.hid_off.cpu().numpy()) == list(ref.hid_off)
    packed = torch.cat([bufs.hid_stage[b, :kept[b]] for b in range(64)])
    assert torch.equal(bufs.hid_out[:packed.shape[0]], packed)
