"""spec_verify_chain_noalloc: chain verification for callers that cannot
allocate device memory (a fixed memory budget, an allocator owned by the host
program, a loop that must not call an allocator). It uses the scratch array
compiled into the library instead of a caller workspace; its outputs must
match spec_verify_chain's on the same inputs, call after call, whatever the
previous call left in the shared array, and sizes beyond the array must be
refused.

This file is collected last so that a run that stops at the first failure has
already run every other test; it passes alone and after the others."""
import ctypes

import numpy as np
import pytest
import torch

from speculative_decoding_verification_89_b200 import workloads as W

pytestmark = pytest.mark.gpu


def _outputs(fn, prob, **kw):
    dev = "cuda"
    B, Kp1, V = prob.tgt.shape
    acc = torch.full((B,), -7, dtype=torch.int32, device=dev)
    out = torch.full((B, Kp1), -7, dtype=torch.int32, device=dev)
    diag = torch.full((B, 4 * (Kp1 - 1) + 2), -7.0, dtype=torch.float64, device=dev)
    st = torch.zeros(1, dtype=torch.int32, device=dev)
    fn(prob.tgt, prob.drf, prob.draft_tok, prob.temperature, prob.seed, prob.seq_id, prob.rnd,
       acc, out, st, diag=diag, **kw)
    torch.cuda.synchronize()
    return acc.cpu().numpy(), out.cpu().numpy(), diag.cpu().numpy(), int(st.item())


def _same(prob):
    """The no-alloc call against spec_verify_chain on a freshly zeroed
    workspace: both run the same kernels, so every output, diagnostics
    included, must agree exactly (NaN where greedy)."""
    from speculative_decoding_verification_89_b200 import capi
    B, Kp1, V = prob.tgt.shape
    ws = capi.workspace(B, Kp1 - 1, V, prob.tgt.dtype)
    ws.zero_()
    a1, o1, d1, s1 = _outputs(capi.spec_verify_chain, prob, ws=ws)
    a2, o2, d2, s2 = _outputs(capi.spec_verify_chain_noalloc, prob)
    assert s1 == 0 and s2 == 0
    assert np.array_equal(a1, a2) and np.array_equal(o1, o2)
    assert np.array_equal(d1, d2, equal_nan=True)


def test_noalloc_matches_workspace_entry_on_two_calls_in_a_row():
    T = torch.tensor([1.0, 0.0, 0.7, 1.3, 0.0, 0.9, 2.0, 1.0, 0.5, 1.0, 0.8, 0.0, 1.1, 1.0, 0.6, 1.2])
    for rnd in (0, 1):
        _same(W.chain_problem(16, 6, 20000, torch.bfloat16, seed=21, rnd=rnd, temperature=T,
                              device="cuda"))


def test_noalloc_after_larger_and_other_dtype_calls():
    """A larger call leaves its row statistics, partials and counters in the
    shared array; a smaller call, then one of the other dtype and another
    draft count, must not read any of it."""
    for (B, K, V, dt, seed) in [(24, 10, 40000, torch.bfloat16, 31),
                                (3, 2, 5000, torch.bfloat16, 32),
                                (7, 5, 9000, torch.float32, 33),
                                (2, 1, 700, torch.float32, 34)]:
        T = torch.linspace(0.0, 1.4, B)
        _same(W.chain_problem(B, K, V, dt, seed=seed, temperature=T, device="cuda"))


def test_noalloc_failed_lookup_is_not_kept():
    """A lookup of the array's address that fails (as one inside a stream
    capture does) returns SPEC_ECUDA with the CUDA error's text, launches
    nothing, and is not remembered: the next call looks again and works."""
    from speculative_decoding_verification_89_b200 import capi
    prob = W.chain_problem(4, 3, 3000, torch.bfloat16, seed=35, device="cuda")
    assert capi._lib.spec_noalloc_test_fail_lookups(1) == capi.SPEC_OK
    try:
        with pytest.raises(capi.SpecError) as err:
            _outputs(capi.spec_verify_chain_noalloc, prob)
        assert err.value.code == capi.SPEC_ECUDA
        assert "no error" not in str(err.value)
    finally:
        capi._lib.spec_noalloc_test_fail_lookups(0)
    _same(prob)


def test_noalloc_refuses_sizes_beyond_its_array():
    from speculative_decoding_verification_89_b200 import capi
    f = capi._lib.spec_verify_chain_noalloc
    B, K, V = 4096, 16, 128256
    need = capi.spec_workspace_bytes(B, K, V, torch.bfloat16)
    assert need > 16 << 20
    fake = ctypes.c_void_p(0x10000)   # never dereferenced: the size check comes first
    rc = f(fake, V, fake, V, capi.SPEC_BF16, B, K, V, fake, fake, 0, fake, 0, fake, fake, None,
           None, None)
    assert rc == capi.SPEC_EWORKSPACE
