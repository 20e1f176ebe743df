"""The bounded-wait timeout path, exercised without any hang: with the
row-statistics kernel's wait limit set to 0 (one non-blocking test per wait)
its first wait finds its tile copy still in flight and runs out. The call
must then report SPEC_ETIMEOUT, drain its copies, commit nothing (tables,
lengths, free stack, pool and hidden rows unchanged), and the next normal
call on the same stream must succeed and match the oracle."""
import pytest
import torch

from speculative_decoding_verification_89_b200 import workloads as W
from tests.parity import Tally
from tests.test_gpu_fused import _check_oracle, _run, _small_case

pytestmark = pytest.mark.gpu


def test_wait_timeout_records_status_and_commits_nothing():
    from speculative_decoding_verification_89_b200 import capi
    prob, state, bufs = _small_case(6, 4, 128256, torch.bfloat16, 1.0, seed=81)
    assert capi._lib.spec_test_set_wait_limit_ns(0) == capi.SPEC_OK
    try:
        r = _run(prob, state, bufs, True)
    finally:
        assert capi._lib.spec_test_set_wait_limit_ns(2_000_000_000) == capi.SPEC_OK
    assert r["status"] == capi.SPEC_ETIMEOUT
    assert torch.equal(r["tables"], state.tables)
    assert torch.equal(r["seq_lens"], state.seq_lens)
    assert torch.equal(r["free_stack"], state.free_stack)
    assert torch.equal(r["free_top"], state.free_top)
    assert torch.equal(r["kv_pool"].cpu(), bufs.kv_pool)
    assert torch.equal(r["hid_out"].cpu(), bufs.hid_out)
    # The next normal call on the same stream works and matches the oracle.
    tally = Tally()
    r2 = _run(prob, state, bufs, True)
    assert r2["status"] == 0
    _check_oracle(prob, state, bufs, r2, "after-timeout", tally)
    tally.check_share()


def test_copy_wait_timeout_records_status():
    """The verify-and-commit copy launch's bounded wait for the plan word,
    run out on purpose (limit 0: one poll, while the decide launch has not yet
    planned): SPEC_ETIMEOUT, the verification outputs as in a normal call, the
    plan made in full or not at all (a timeout recorded before the planner
    reads the status word stops it, as any earlier error does), and the next
    normal call on the same stream matches the oracle."""
    from speculative_decoding_verification_89_b200 import capi
    prob = W.chain_batch(device="cuda")
    state, bufs = W.commit_setup(64, 8, device="cuda")
    state = W.PagedState(state.tables.cpu(), state.seq_lens.cpu(), state.free_stack.cpu(),
                         state.free_top.cpu(), 16)
    ref = _run(prob, state, bufs, True)
    assert ref["status"] == 0
    assert capi._lib.spec_test_set_copy_wait_limit_ns(0) == capi.SPEC_OK
    try:
        r = _run(prob, state, bufs, True)
    finally:
        assert capi._lib.spec_test_set_copy_wait_limit_ns(2_000_000_000) == capi.SPEC_OK
    assert r["status"] == capi.SPEC_ETIMEOUT
    for k in ("acc", "out"):
        assert torch.equal(r[k], ref[k]), k
    assert torch.equal(torch.nan_to_num(r["diag"], nan=-99.0),
                       torch.nan_to_num(ref["diag"], nan=-99.0))
    planned = torch.equal(r["tables"], ref["tables"])
    before = dict(tables=state.tables, seq_lens=state.seq_lens, free_stack=state.free_stack,
                  free_top=state.free_top)
    for k in ("tables", "seq_lens", "free_stack", "free_top"):
        assert torch.equal(r[k], ref[k] if planned else before[k]), (k, planned)
    tally = Tally()
    r2 = _run(prob, state, bufs, True)
    assert r2["status"] == 0
    _check_oracle(prob, state, bufs, r2, "after-copy-timeout", tally)
    tally.check_share()
