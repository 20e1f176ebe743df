"""Chain verification fused with the paged commit (spec_verify_chain_commit)
against the oracle and against the separate calls of the same kernels
(spec_chain_row_stats and spec_chain_decide, then spec_commit_paged with
keep = accept_len + 1) on the same inputs: accepted
counts, tokens, probabilities, tables, lengths, free stack, moved K/V rows and
the packed hidden rows. The two GPU paths must agree bit for bit; the oracle
comparison follows the chain and commit acceptance rules."""
import numpy as np
import pytest
import torch

from oracle.commit import check_invariants, commit_paged, gather_hidden
from speculative_decoding_verification_89_b200 import workloads as W
from tests.gpu_run import padded, run_chain_oracle
from tests.parity import Tally, compare_check, compare_probs

pytestmark = pytest.mark.gpu

FIELDS = ("acc", "out", "diag", "status", "tables", "seq_lens", "free_stack", "free_top",
          "kv_pool", "hid_out", "hid_off")


def _run(prob, state, bufs, fused, base=None, status0=0, persistent=False):
    from speculative_decoding_verification_89_b200 import capi
    dev = "cuda"
    tgt = padded(prob.tgt.to(dev))
    B, Kp1, V = tgt.shape
    K = Kp1 - 1
    drf = padded(prob.drf.to(dev)) if K > 0 else prob.drf.to(dev)
    dt = prob.draft_tok.to(dev).contiguous()
    T, sid = prob.temperature.to(dev), prob.seq_id.to(dev)
    st = state.clone()
    t, l, f, top = (st.tables.to(dev), st.seq_lens.to(dev), st.free_stack.to(dev),
                    st.free_top.to(dev))
    kw = {}
    if bufs is not None:
        kw = dict(kv_stage=bufs.kv_stage.to(dev), kv_pool=bufs.kv_pool.clone().to(dev),
                  hid_stage=bufs.hid_stage.to(dev), hid_out=bufs.hid_out.clone().to(dev),
                  hid_off=bufs.hid_off.clone().to(dev))
    b_len = None if base is None else base.to(dev)
    ws = capi.workspace(B, K, V, tgt.dtype, device=dev)
    acc = torch.full((B,), -7, dtype=torch.int32, device=dev)
    out = torch.full((B, K + 1), -7, dtype=torch.int32, device=dev)
    dg = torch.full((B, 4 * K + 2), -7.0, dtype=torch.float64, device=dev)
    s = torch.full((1,), status0, dtype=torch.int32, device=dev)
    if fused:
        fn = capi.spec_verify_chain_commit_persistent if persistent else \
            capi.spec_verify_chain_commit
        fn(tgt, drf, dt, T, prob.seed, sid, prob.rnd, acc, out, t, l, b_len, f, top, s, ws,
           block_size=state.block_size, diag=dg, **kw)
    else:
        capi.spec_chain_row_stats(tgt, drf, T, s, ws)
        capi.spec_chain_decide(tgt, drf, dt, T, prob.seed, sid, prob.rnd, acc, out, s, ws,
                               diag=dg)
        capi.spec_commit_paged(t, l, b_len, acc, 1, f, top, K + 1, s,
                               block_size=state.block_size, **kw)
    torch.cuda.synchronize()
    r = dict(acc=acc.cpu(), out=out.cpu(), diag=dg.cpu(), status=int(s.item()), tables=t.cpu(),
             seq_lens=l.cpu(), free_stack=f.cpu(), free_top=top.cpu())
    for k in ("kv_pool", "hid_out", "hid_off"):  # left on the device (the pool is large)
        r[k] = kw[k] if k in kw else None
    r["state"] = W.PagedState(r["tables"], r["seq_lens"], r["free_stack"], r["free_top"],
                              state.block_size)
    return r


def _same(a, b, tag, skip=()):
    for k in FIELDS:
        if k in skip:
            continue
        x, y = a[k], b[k]
        if x is None or isinstance(x, int):
            assert x == y, f"{tag}: {k}"
        elif x.dtype == torch.float64:
            assert torch.equal(torch.nan_to_num(x, nan=-99.0), torch.nan_to_num(y, nan=-99.0)), \
                f"{tag}: {k}"
        else:
            assert torch.equal(x.view(torch.int16) if x.dtype == torch.bfloat16 else x,
                               (y.view(torch.int16) if y.dtype == torch.bfloat16 else y)
                               .to(x.device)), f"{tag}: {k}"


def _check_oracle(prob, state, bufs, r, tag, tally, base=None):
    """The fused result against the oracle: the check per sequence, then the
    commit of the GPU's kept counts."""
    K = prob.draft_tok.shape[1]
    ok = [b for b in range(prob.tgt.shape[0]) if int(r["acc"][b]) >= 0]
    ref = run_chain_oracle(prob, ok)
    for b, res in ref.items():
        a = int(r["acc"][b])
        toks = [int(x) for x in r["out"][b, :a + 1]]
        assert all(int(x) == -1 for x in r["out"][b, a + 1:]), f"{tag}: padding"
        if compare_check(f"{tag}/seq{b}", res, a, toks, tally):
            compare_probs(f"{tag}/seq{b}", res, r["diag"][b].numpy(), K,
                          float(prob.temperature[b]))
    if r["status"] == -6:  # a sequence failed: nothing is committed
        assert torch.equal(r["tables"], state.tables)
        assert torch.equal(r["seq_lens"], state.seq_lens)
        assert torch.equal(r["free_top"], state.free_top)
        return
    keep = r["acc"].numpy().astype(np.int64) + 1
    b_arr = state.seq_lens.numpy() if base is None else base.numpy()
    oc = commit_paged(state.tables.numpy(), state.seq_lens.numpy(), b_arr, keep,
                      state.free_stack.numpy(), int(state.free_top[0]), state.block_size,
                      state.free_stack.numel(), K + 1)
    assert r["status"] == oc.status, (tag, r["status"], oc.status)
    if oc.status != 0:
        assert torch.equal(r["tables"], state.tables)
        assert torch.equal(r["free_stack"], state.free_stack)
        assert torch.equal(r["free_top"], state.free_top)
        return
    bs = state.block_size
    assert list(r["seq_lens"].numpy()) == list(oc.seq_lens)
    assert int(r["free_top"][0]) == oc.free_top
    assert np.array_equal(r["free_stack"].numpy()[:oc.free_top], oc.free_stack[:oc.free_top])
    for b in range(len(oc.seq_lens)):
        nb = (int(oc.seq_lens[b]) + bs - 1) // bs
        assert np.array_equal(r["tables"].numpy()[b, :nb], oc.tables[b, :nb])
    assert check_invariants(r["tables"].numpy(), r["seq_lens"].numpy(),
                            r["free_stack"].numpy(), int(r["free_top"][0]), bs,
                            state.free_stack.numel()) == []
    if bufs is not None:
        pool, stage = r["kv_pool"], bufs.kv_stage.to(r["kv_pool"].device)
        for (b, i, blk, slot) in oc.destinations:
            assert torch.equal(pool[blk, :, :, slot].view(torch.int16),
                               stage[b, i].view(torch.int16))
        assert list(r["hid_off"].cpu().numpy()) == list(oc.hid_off)
        packed = gather_hidden(bufs.hid_stage.cpu().view(torch.int16).numpy(), keep)
        got = r["hid_out"].cpu().view(torch.int16).numpy()[:len(packed)]
        assert np.array_equal(got, packed)


def test_fused_full_size():
    """B=64, K=8, V=128256 bf16 chain check plus the commit of a + 1 rows per
    sequence (block 16, contexts U[512, 4096], 128 KiB of K/V per token,
    hidden 4096)."""
    tally = Tally()
    for rnd in range(2):
        prob = W.chain_batch(device="cuda", rnd=rnd)
        state, bufs = W.commit_setup(64, 8, device="cuda")
        state = W.PagedState(state.tables.cpu(), state.seq_lens.cpu(), state.free_stack.cpu(),
                             state.free_top.cpu(), 16)
        fused = _run(prob, state, bufs, True)
        two = _run(prob, state, bufs, False)
        assert fused["status"] == 0
        _same(fused, two, f"full{rnd}")
        _check_oracle(prob, state, bufs, fused, f"full{rnd}", tally)
    tally.check_share()


def _small_case(B, K, V, dtype, T, seed, bs=4, spare=None, ctx_hi=40, ctx=None):
    prob = W.chain_problem(B, K, V, dtype, seed=seed, temperature=1.0)
    prob.temperature = T if isinstance(T, torch.Tensor) else torch.full((B,), float(T))
    rng = np.random.default_rng(seed)
    if ctx is None:
        ctx = [int(x) for x in rng.integers(0, ctx_hi, size=B)]
    need = sum((n + bs - 1) // bs for n in ctx)
    if spare is None:  # room for about two rounds of kept rows
        spare = B * ((K + bs) // bs + 1)
    max_blocks = (max(ctx) + 3 * (K + 1) + bs - 1) // bs + 1
    state = W.paged_state(ctx, bs, max_blocks, need + spare)
    nb = state.free_stack.numel()
    gen = W.generator(seed + 100, "cpu")
    L, H, D, hidden = 2, 2, 8, 24
    bufs = W.CommitBuffers(W.random_bf16((B, K + 1, L, 2, H, D), gen, "cpu"),
                           torch.zeros((nb, L, 2, bs, H, D), dtype=torch.bfloat16),
                           W.random_bf16((B, K + 1, hidden), gen, "cpu"),
                           torch.zeros((B * (K + 1), hidden), dtype=torch.bfloat16),
                           torch.zeros((B + 1,), dtype=torch.int32))
    return prob, state, bufs


SMALL = [
    # B, K, V, dtype, temperature
    (3, 0, 1000, torch.float32, 1.0),            # no drafts: one row kept per sequence
    (5, 2, 12345, torch.bfloat16, torch.tensor([0.0, 0.5, 1.0, 0.0, 2.0])),
    (4, 3, 8191, torch.float32, 1.3),            # ragged tiles
    (2, 40, 3000, torch.bfloat16, 1.0),          # K > 32
    (3, 5, 777, torch.bfloat16, 0.0),            # all greedy
    (37, 4, 5000, torch.bfloat16, 0.9),          # more sequences than draw clusters of 4 fit
    (300, 3, 2000, torch.float32, 1.0),          # clusters in several waves: late tickets
    (4096, 1, 64, torch.float32, 0.8),           # the largest batch of the fused call
]


@pytest.mark.parametrize("B,K,V,dtype,T", SMALL)
def test_fused_small(B, K, V, dtype, T):
    tally = Tally()
    prob, state, bufs = _small_case(B, K, V, dtype, T, seed=B * 7 + K)
    for rnd in range(3):  # the state carries over: lengths grow each round
        prob.rnd = rnd
        fused = _run(prob, state, bufs, True)
        two = _run(prob, state, bufs, False)
        _same(fused, two, f"rnd{rnd}")
        _check_oracle(prob, state, bufs, fused, f"rnd{rnd}", tally)
        state = fused["state"]
        bufs = W.CommitBuffers(bufs.kv_stage, fused["kv_pool"].cpu(), bufs.hid_stage,
                               fused["hid_out"].cpu(), fused["hid_off"].cpu())
    tally.check_share()


def test_fused_tables_only_and_rollback():
    """No K/V or hidden buffers (tables only), with a base length below the
    current one (rollback of blocks held for the previous speculation)."""
    tally = Tally()
    prob, state, _ = _small_case(6, 4, 2048, torch.float32, 0.8, seed=31)
    base = torch.clamp(state.seq_lens - 5, min=0).int()
    fused = _run(prob, state, None, True, base=base)
    two = _run(prob, state, None, False, base=base)
    _same(fused, two, "rollback")
    _check_oracle(prob, state, None, fused, "rollback", tally, base=base)


def test_fused_failures():
    """An invalid temperature or draft id fails its sequence and blocks the
    commit; an exhausted pool fails the commit. Either way no table, length,
    stack entry, pool slot or hidden row changes, and the check's outputs
    equal the two-call path's."""
    tally = Tally()
    prob, state, bufs = _small_case(4, 3, 1000, torch.float32, 1.0, seed=41)
    prob.temperature[2] = -1.0
    prob.draft_tok[1, 2] = 1000
    fused = _run(prob, state, bufs, True)
    two = _run(prob, state, bufs, False)
    assert fused["status"] == -6
    assert int(fused["acc"][1]) == -1 and int(fused["acc"][2]) == -1
    _same(fused, two, "invalid")
    _check_oracle(prob, state, bufs, fused, "invalid", tally)
    assert torch.equal(fused["kv_pool"].cpu(), bufs.kv_pool)
    # every context ends on a block boundary, so every kept row needs a new block
    prob, state, bufs = _small_case(8, 6, 1000, torch.float32, 1.0, seed=43, spare=0,
                                    ctx=[4 * i for i in range(8)])
    fused = _run(prob, state, bufs, True)
    two = _run(prob, state, bufs, False)
    assert fused["status"] == -4
    _same(fused, two, "pool")
    _check_oracle(prob, state, bufs, fused, "pool", tally)
    assert torch.equal(fused["kv_pool"].cpu(), bufs.kv_pool)
    # contexts that end inside a block: the first rows fit held blocks, the
    # rest need new ones the pool cannot give
    prob, state, bufs = _small_case(8, 6, 1000, torch.float32, 1.0, seed=45, spare=0,
                                    ctx=[4 * i + 2 for i in range(8)])
    fused = _run(prob, state, bufs, True)
    two = _run(prob, state, bufs, False)
    _same(fused, two, "pool2")
    _check_oracle(prob, state, bufs, fused, "pool2", tally)
    tally.check_share()


def test_fused_pending_status_commits_nothing():
    """A status word that already holds an error on entry: the check still
    runs and writes its outputs, the commit changes nothing -- as for the two
    calls."""
    prob, state, bufs = _small_case(5, 4, 3000, torch.bfloat16, 0.9, seed=51)
    fused = _run(prob, state, bufs, True, status0=-6)
    two = _run(prob, state, bufs, False, status0=-6)
    assert fused["status"] == -6
    _same(fused, two, "pending")
    assert torch.equal(fused["tables"], state.tables)
    assert torch.equal(fused["seq_lens"], state.seq_lens)
    assert torch.equal(fused["free_stack"], state.free_stack)
    assert torch.equal(fused["kv_pool"].cpu(), bufs.kv_pool)
    assert torch.equal(fused["hid_out"].cpu(), bufs.hid_out)


def test_split_entry_points_repeat_after_one_row_pass():
    """spec_chain_row_stats once, then spec_chain_decide_commit for two rounds
    on the same rows: each round equals spec_chain_decide + spec_commit_paged
    (the accept launch's tickets keep counting past B)."""
    from speculative_decoding_verification_89_b200 import capi
    dev = "cuda"
    prob, state, bufs = _small_case(6, 3, 4000, torch.bfloat16, 1.1, seed=61, spare=24)
    tgt, drf = padded(prob.tgt.to(dev)), padded(prob.drf.to(dev))
    dt, T, sid = prob.draft_tok.to(dev), prob.temperature.to(dev), prob.seq_id.to(dev)
    B, K, V = 6, 3, 4000
    res = []
    for fused in (True, False):
        st = state.clone()
        t, l, f, top = (st.tables.to(dev), st.seq_lens.to(dev), st.free_stack.to(dev),
                        st.free_top.to(dev))
        pool, hout, hoff = bufs.kv_pool.clone().to(dev), bufs.hid_out.clone().to(dev), \
            bufs.hid_off.clone().to(dev)
        kw = dict(kv_stage=bufs.kv_stage.to(dev), kv_pool=pool, hid_stage=bufs.hid_stage.to(dev),
                  hid_out=hout, hid_off=hoff)
        ws = capi.workspace(B, K, V, tgt.dtype, device=dev)
        s = torch.zeros(1, dtype=torch.int32, device=dev)
        capi.spec_chain_row_stats(tgt, drf, T, s, ws)
        outs = []
        for rnd in (7, 8):
            acc = torch.empty(B, dtype=torch.int32, device=dev)
            out = torch.empty((B, K + 1), dtype=torch.int32, device=dev)
            if fused:
                capi.spec_chain_decide_commit(tgt, drf, dt, T, prob.seed, sid, rnd, acc, out, t, l,
                                              None, f, top, s, ws, block_size=state.block_size,
                                              **kw)
            else:
                capi.spec_chain_decide(tgt, drf, dt, T, prob.seed, sid, rnd, acc, out, s, ws)
                capi.spec_commit_paged(t, l, None, acc, 1, f, top, K + 1, s,
                                       block_size=state.block_size, **kw)
            torch.cuda.synchronize()
            outs.append((acc.cpu(), out.cpu(), t.cpu().clone(), l.cpu().clone(),
                         top.cpu().clone(), hoff.cpu().clone()))
        res.append((outs, pool.cpu(), hout.cpu(), int(s.item())))
    assert res[0][3] == res[1][3]
    for (a, b) in zip(res[0][0], res[1][0]):
        for x, y in zip(a, b):
            assert torch.equal(x, y)
    assert torch.equal(res[0][1].view(torch.int16), res[1][1].view(torch.int16))
    assert torch.equal(res[0][2].view(torch.int16), res[1][2].view(torch.int16))


def test_fused_deep_rollback_and_invalid_entries():
    """The per-sequence commit records of the fused path: rollbacks that free
    more table entries than a record carries (the rest read from the table),
    batches where a planner thread owns several sequences, and a held table
    entry or a base length that is invalid (nothing changes). Each against the
    two-call path and the oracle."""
    tally = Tally()
    for B, seed in ((7, 71), (1100, 73)):
        prob, state, bufs = _small_case(B, 3, 300, torch.float32, 0.9, seed=seed, ctx_hi=60)
        rng = np.random.default_rng(seed)
        drop = torch.from_numpy(rng.integers(0, 41, size=B)).int()
        base = torch.clamp(state.seq_lens - drop, min=0).int()
        fused = _run(prob, state, bufs, True, base=base)
        two = _run(prob, state, bufs, False, base=base)
        assert fused["status"] == 0
        _same(fused, two, f"rollback{B}")
        _check_oracle(prob, state, bufs, fused, f"rollback{B}", tally, base=base)
    prob, state, bufs = _small_case(6, 3, 500, torch.float32, 1.0, seed=75, ctx_hi=60)
    held = (state.seq_lens + state.block_size - 1) // state.block_size
    b = int(torch.argmax(held))
    bad_tab = state.clone()
    bad_tab.tables[b, int(held[b]) - 1] = state.free_stack.numel() + 5
    bad_base = state.seq_lens.clone()
    bad_base[4] += 1
    for tag, st, base in (("entry", bad_tab, None), ("base", state, bad_base)):
        fused = _run(prob, st, bufs, True, base=base)
        two = _run(prob, st, bufs, False, base=base)
        assert fused["status"] == -1, tag
        _same(fused, two, tag)
        _check_oracle(prob, st, bufs, fused, tag, tally, base=base)
        assert torch.equal(fused["kv_pool"].cpu(), bufs.kv_pool)
    tally.check_share()
