"""The seeded input generators: shapes, determinism, value models."""
import numpy as np
import torch

from oracle.commit import check_invariants
from speculative_decoding_verification_89_b200 import workloads as W


def test_chain_small_shapes_and_determinism():
    a = W.chain_small(rnd=3)
    b = W.chain_small(rnd=3)
    c = W.chain_small(rnd=4)
    assert a.tgt.shape == (1, 5, 1024) and a.drf.shape == (1, 4, 1024)
    assert a.tgt.dtype == torch.float32 and a.draft_tok.dtype == torch.int32
    assert torch.equal(a.tgt, b.tgt) and torch.equal(a.draft_tok, b.draft_tok)
    assert not torch.equal(a.tgt, c.tgt)
    assert abs(float(a.tgt.std()) - 2.0) < 0.15


def test_gumbel_drafts_follow_the_draft_law():
    g = W.generator(0, "cpu")
    logits = torch.tensor([[[0.0, 1.0, 2.0, -1.0]]]).repeat(1, 20000, 1)
    d = W.gumbel_drafts(logits, torch.tensor([1.0]), g)
    freq = np.bincount(d.numpy().ravel(), minlength=4) / d.numel()
    p = np.exp([0.0, 1.0, 2.0, -1.0]); p /= p.sum()
    assert np.max(np.abs(freq - p)) < 0.015
    d0 = W.gumbel_drafts(logits[:, :5], torch.tensor([0.0]), g)
    assert torch.all(d0 == 2)


def test_mixed_temperatures_exact_greedy_count():
    T = W.mixed_temperatures(256, 51, 1.2, W.generator(3, "cpu"), "cpu")
    assert int((T == 0).sum()) == 51
    assert float(T.max()) <= 1.2 and float(T[T > 0].min()) > 0


def test_paged_state_is_a_partition():
    ctx = W.context_lengths(8, 5, 70, seed=1)
    st = W.paged_state(ctx, 16, 8, 64)
    errs = check_invariants(st.tables.numpy(), st.seq_lens.numpy(), st.free_stack.numpy(),
                            int(st.free_top[0]), 16, 64)
    assert errs == []
    # the lowest free id is on top of the stack
    top = int(st.free_top[0])
    assert int(st.free_stack[top - 1]) == int(st.free_stack[:top].min())


def test_hier_peaked_model():
    p = W.hier_peaked()
    assert p.lg_f.shape == (8, 9, 32000) and p.lg_f.dtype == torch.bfloat16
    assert float(p.temperature[0]) == 0.0 and abs(float(p.temperature[1]) - 0.7) < 1e-6
    frac_boost = float((p.lg_f.float() > 6.0).float().mean())
    assert 0.03 < frac_boost < 0.07
