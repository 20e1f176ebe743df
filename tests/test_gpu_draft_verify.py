"""Draft then verify, both on the GPU, against the oracle doing the same.

The single-sequence chain workload (B=1, K=4, V=1024 fp32, T=1, 100 rounds of
fresh logits) with its drafts drawn the way the workload describes them: from
the draft softmax with the Philox draft stream (counter (seq, round, pos, 0)),
here by the draft-step entry point, then checked by spec_verify_chain. The
oracle drafts with its own draft step and verifies with its own check; the
drafted tokens, the accepted counts and the emitted tokens must agree (up to
decisions within the 1e-6 margin, counted)."""
import numpy as np
import pytest
import torch

from oracle.draft import draft_step
from oracle.verify import verify_chain
from speculative_decoding_verification_89_b200 import workloads as W
from tests.gpu_run import to_np
from tests.parity import MARGIN, Tally, compare_check

pytestmark = pytest.mark.gpu


def test_draft_then_verify_hundred_rounds():
    from speculative_decoding_verification_89_b200 import capi
    dev = torch.device("cuda")
    K, V = 4, 1024
    tally = Tally()
    wsd = capi.draft_workspace(K, V, torch.float32, device=dev)
    wsv = capi.workspace(1, K, V, torch.float32, device=dev)
    st = torch.zeros(1, dtype=torch.int32, device=dev)
    for rnd in range(100):
        prob = W.chain_small(rnd=rnd)
        drf = prob.drf[0].to(dev).contiguous()                      # [K, V]
        T_rows = prob.temperature.repeat(K)
        sid_rows = prob.seq_id.repeat(K)
        pos = torch.arange(K, dtype=torch.int32)
        tok = torch.empty(K, dtype=torch.int32, device=dev)
        capi.spec_draft_sample(drf, T_rows.to(dev), prob.seed, sid_rows.to(dev), rnd,
                               pos.to(dev), tok, st, wsd)
        ref_d = draft_step(to_np(prob.drf[0]), T_rows.numpy(), prob.seed, sid_rows.numpy(), rnd,
                           pos.numpy())
        drafts = tok.cpu()
        for j in range(K):
            if int(drafts[j]) != ref_d[j].token:
                assert ref_d[j].margin < MARGIN, (rnd, j, int(drafts[j]), ref_d[j].token)
                tally.excused += 1
        tally.decisions += K
        acc = torch.empty(1, dtype=torch.int32, device=dev)
        out = torch.empty((1, K + 1), dtype=torch.int32, device=dev)
        capi.spec_verify_chain(prob.tgt.to(dev), prob.drf.to(dev), drafts[None, :].to(dev),
                               prob.temperature.to(dev), prob.seed, prob.seq_id.to(dev), rnd,
                               acc, out, st, wsv)
        torch.cuda.synchronize()
        assert int(st.item()) == 0
        ref = verify_chain(to_np(prob.tgt), to_np(prob.drf), drafts[None, :].numpy(),
                           prob.temperature.numpy(), prob.seed, prob.seq_id.numpy(), rnd)[0]
        a = int(acc[0])
        compare_check(f"round{rnd}", ref, a, [int(x) for x in out[0, :a + 1]], tally)
    tally.check_share()
