"""spec_verify_chain_noalloc: chain verification for callers that cannot
allocate device memory (a fixed memory budget, an allocator owned by the host
program, a loop that must not call an allocator). It uses the scratch array
compiled into the library instead of a caller workspace; its outputs must
match spec_verify_chain's on the same inputs, call after call, and sizes
beyond the array must be refused.

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


def test_noalloc_matches_workspace_entry_on_two_calls_in_a_row():
    from speculative_decoding_verification_89_b200 import capi
    T = torch.tensor([1.0, 0.0, 0.7, 1.3, 0.0, 0.9, 2.0, 1.0, 0.5, 1.0, 0.8, 0.0, 1.1, 1.0, 0.6, 1.2])
    for rnd in (0, 1):
        prob = W.chain_problem(16, 6, 20000, torch.bfloat16, seed=21, rnd=rnd, temperature=T,
                               device="cuda")
        ws = capi.workspace(16, 6, 20000, torch.bfloat16)
        a1, o1, d1, s1 = _outputs(capi.spec_verify_chain, prob, ws=ws)
        a2, o2, d2, s2 = _outputs(capi.spec_verify_chain_noalloc, prob)
        assert s1 == 0 and s2 == 0
        assert np.array_equal(a1, a2) and np.array_equal(o1, o2)
        both = ~np.isnan(d1)
        assert np.array_equal(both, ~np.isnan(d2))
        assert np.all(np.abs(d1[both] - d2[both]) <= 1e-5 * np.maximum(1.0, np.abs(d1[both])))


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
