"""Seeded synthetic inputs for the verification path.

This module only draws inputs: logits of the three exits, drafted tokens,
temperatures, sequence ids and the paged-KV state. It holds none of the
verification arithmetic; both the CUDA path and the oracle consume what it
produces (the oracle from host copies of the same tensors).

Logit models (all per entry, independent):
* final layer l_f ~ N(0, sigma_f^2), optionally plus a Zipf log-prior
  -s * ln(id + 1) over token ids and a "+boost on a Bernoulli(p) mask" for
  peaked rows;
* intermediate exit l_i = l_f + N(0, sigma_i^2); draft exit l_d = l_f +
  N(0, sigma_d^2) (for a single-stage chain the target is l_f and the draft
  l_d);
* bf16 workloads round the fp32 draws to bfloat16 once; every consumer sees
  the same rounded values.
Drafts are drawn from softmax(l_d / T) with the Gumbel-max construction
argmax(l_d / T + G) (argmax of l_d when T = 0), using torch's seeded
generator; the verification's own uniforms come from Philox inside the
library.
"""
from __future__ import annotations

from dataclasses import dataclass

import torch

# ----------------------------------------------------------------------------
# Primitive draws
# ----------------------------------------------------------------------------


def generator(seed: int, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(int(seed) & 0x7FFFFFFFFFFFFFFF)
    return g


def gaussian(shape, std, gen, device) -> torch.Tensor:
    return torch.randn(shape, generator=gen, device=device, dtype=torch.float32) * std


def zipf_prior(V, s, device) -> torch.Tensor:
    ids = torch.arange(V, device=device, dtype=torch.float64)
    return (-s * torch.log(ids + 1.0)).to(torch.float32)


def gumbel_drafts(draft_logits: torch.Tensor, temperature: torch.Tensor, gen) -> torch.Tensor:
    """Tokens drawn from softmax(l / T) row by row (argmax at T == 0).

    draft_logits [B, n, V]; temperature [B]. Returns int32 [B, n]."""
    x = draft_logits.float()
    u = torch.rand(x.shape, generator=gen, device=x.device, dtype=torch.float32)
    u = u.clamp_(min=1e-12, max=1.0 - 1e-7)
    g = -torch.log(-torch.log(u))
    T = temperature.to(x.device).float().view(-1, 1, 1)
    scaled = torch.where(T > 0, x / torch.where(T > 0, T, torch.ones_like(T)) + g, x)
    return scaled.argmax(dim=-1).to(torch.int32)


# ----------------------------------------------------------------------------
# Chain verification problems
# ----------------------------------------------------------------------------


@dataclass
class ChainProblem:
    tgt: torch.Tensor          # [B, K+1, V]
    drf: torch.Tensor          # [B, K, V]
    draft_tok: torch.Tensor    # int32 [B, K]
    temperature: torch.Tensor  # float32 [B]
    seq_id: torch.Tensor       # int32 [B]
    seed: int                  # Philox key of the verification
    rnd: int                   # Philox round field


def chain_problem(B, K, V, dtype=torch.bfloat16, *, seed=0, rnd=0, device="cpu",
                  target_std=2.0, zipf_s=0.0, draft_noise=1.0, temperature=1.0,
                  philox_seed=None, seq_id_base=0) -> ChainProblem:
    gen = generator(seed * 1_000_003 + rnd, device)
    tgt = gaussian((B, K + 1, V), target_std, gen, device)
    if zipf_s:
        tgt += zipf_prior(V, zipf_s, device)
    drf = tgt[:, :K] + gaussian((B, K, V), draft_noise, gen, device)
    tgt, drf = tgt.to(dtype), drf.to(dtype)
    if isinstance(temperature, torch.Tensor):
        T = temperature.to(device=device, dtype=torch.float32)
    else:
        T = torch.full((B,), float(temperature), dtype=torch.float32, device=device)
    drafts = gumbel_drafts(drf, T, gen) if K > 0 else torch.zeros((B, 0), dtype=torch.int32,
                                                                  device=device)
    seq_id = torch.arange(seq_id_base, seq_id_base + B, dtype=torch.int32, device=device)
    return ChainProblem(tgt, drf, drafts, T, seq_id,
                        seed if philox_seed is None else philox_seed, rnd)


# ----------------------------------------------------------------------------
# Two-stage problems
# ----------------------------------------------------------------------------


@dataclass
class HierProblem:
    lg_d: torch.Tensor         # [B, S, V], S = Ni + K + 1
    lg_i: torch.Tensor
    lg_f: torch.Tensor
    temperature: torch.Tensor
    seq_id: torch.Tensor
    K: int
    Ni: int
    seed: int


def hier_logits(B, S, V, dtype, gen, device, *, final_std, inter_noise, draft_noise,
                boost_p=0.0, boost=0.0, zipf_s=0.0):
    lf = gaussian((B, S, V), final_std, gen, device)
    if boost_p:
        mask = torch.rand((B, S, V), generator=gen, device=device) < boost_p
        lf = lf + boost * mask.float()
    if zipf_s:
        lf = lf + zipf_prior(V, zipf_s, device)
    li = lf + gaussian((B, S, V), inter_noise, gen, device)
    ld = lf + gaussian((B, S, V), draft_noise, gen, device)
    return ld.to(dtype), li.to(dtype), lf.to(dtype)


def hier_problem(B, K, Ni, V, dtype=torch.bfloat16, *, seed=0, device="cpu", final_std=2.0,
                 inter_noise=0.5, draft_noise=1.0, boost_p=0.0, boost=0.0,
                 temperature=1.0, philox_seed=None) -> HierProblem:
    S = Ni + K + 1
    gen = generator(seed * 7919 + 17, device)
    ld, li, lf = hier_logits(B, S, V, dtype, gen, device, final_std=final_std,
                             inter_noise=inter_noise, draft_noise=draft_noise,
                             boost_p=boost_p, boost=boost)
    if isinstance(temperature, torch.Tensor):
        T = temperature.to(device=device, dtype=torch.float32)
    else:
        T = torch.full((B,), float(temperature), dtype=torch.float32, device=device)
    seq_id = torch.arange(B, dtype=torch.int32, device=device)
    return HierProblem(ld, li, lf, T, seq_id, K, Ni, seed if philox_seed is None else philox_seed)


def window_drafts(lg_d, win_len, K, temperature, gen):
    """Drafts for slots win_len[b] .. win_len[b]+K-1 from the L_d rows there."""
    B, S, V = lg_d.shape
    idx = win_len.long().view(B, 1) + torch.arange(K, device=lg_d.device).view(1, K)
    rows = torch.gather(lg_d, 1, idx.view(B, K, 1).expand(B, K, V))
    return gumbel_drafts(rows, temperature, gen)


def mixed_temperatures(B, n_greedy, t_max, gen, device):
    """U(0, t_max] per sequence with exactly n_greedy sequences at 0."""
    u = torch.rand((B,), generator=gen, device=device)
    T = (t_max * (1.0 - u)).float()
    pick = torch.randperm(B, generator=gen, device=device)[:n_greedy]
    T[pick] = 0.0
    return T


# ----------------------------------------------------------------------------
# Draft-step problems
# ----------------------------------------------------------------------------


@dataclass
class DraftProblem:
    logits: torch.Tensor       # [B, V] drafting-exit rows
    temperature: torch.Tensor  # float32 [B]
    seq_id: torch.Tensor       # int32 [B]
    pos: torch.Tensor          # int32 [B] slot of the drafted token
    seed: int                  # Philox key
    rnd: int                   # Philox round field


def draft_problem(B, V, dtype=torch.bfloat16, *, seed=0, rnd=0, device="cpu", std=2.0,
                  zipf_s=0.0, mask_frac=0.0, temperature=1.0, philox_seed=None,
                  seq_id_base=0) -> DraftProblem:
    """l_d ~ N(0, std^2) (+ Zipf log-prior), a random mask_frac of the entries
    set to -inf; slots pos ~ U{0..15}."""
    gen = generator(seed * 1_000_003 + rnd + 17, device)
    lg = gaussian((B, V), std, gen, device)
    if zipf_s:
        lg += zipf_prior(V, zipf_s, device)
    if mask_frac:
        m = torch.rand((B, V), generator=gen, device=device) < mask_frac
        lg = lg.masked_fill(m, float("-inf"))
    lg = lg.to(dtype)
    if isinstance(temperature, torch.Tensor):
        T = temperature.to(device=device, dtype=torch.float32)
    else:
        T = torch.full((B,), float(temperature), dtype=torch.float32, device=device)
    seq_id = torch.arange(seq_id_base, seq_id_base + B, dtype=torch.int32, device=device)
    pos = torch.randint(0, 16, (B,), generator=gen, device=device, dtype=torch.int32)
    return DraftProblem(lg, T, seq_id, pos, seed if philox_seed is None else philox_seed, rnd)


def draft_batch(device="cpu", rnd=0, B=64, V=128256, seed=5):
    """B=64, V=128256 bf16 drafting rows l_d ~ N(0, 2^2) - 1.1 ln(id + 1);
    T = 1; Philox seed 5."""
    return draft_problem(B, V, torch.bfloat16, seed=seed, rnd=rnd, device=device, zipf_s=1.1,
                         temperature=1.0, philox_seed=5)


def cached_tokens(lg, n_cached, *, seed, extra=None):
    """Synthetic speculation-cache lists (Saguaro sampling), one per row of
    lg [..., V]: the ids of the row's n_cached - 3 largest logits (the likely
    bonus tokens a cache prepares), then ``extra[...]`` (e.g. the drafted
    token) or a repeat of the top id, then the padding ids -1 and V; each list
    shuffled. Returns int32 [..., n_cached] on lg's device."""
    V = lg.shape[-1]
    top = torch.topk(lg.float(), max(n_cached - 3, 1), dim=-1).indices.to(torch.int32)
    top = top[..., :n_cached - 3]
    third = top[..., :1] if extra is None else extra.to(torch.int32)[..., None]
    pad = torch.tensor([-1, V], dtype=torch.int32, device=lg.device).expand(*lg.shape[:-1], 2)
    ids = torch.cat([top, third, pad], dim=-1)
    gen = generator(seed, "cpu")
    flat = ids.reshape(-1, n_cached)
    perm = torch.stack([torch.randperm(n_cached, generator=gen) for _ in range(flat.shape[0])])
    return torch.gather(flat, 1, perm.to(flat.device)).reshape(ids.shape).contiguous()


# ----------------------------------------------------------------------------
# Paged KV state
# ----------------------------------------------------------------------------


@dataclass
class PagedState:
    tables: torch.Tensor       # int32 [B, max_blocks]
    seq_lens: torch.Tensor     # int32 [B]
    free_stack: torch.Tensor   # int32 [num_blocks]
    free_top: torch.Tensor     # int32 [1]
    block_size: int

    def clone(self):
        return PagedState(self.tables.clone(), self.seq_lens.clone(),
                          self.free_stack.clone(), self.free_top.clone(), self.block_size)


def paged_state(ctx_lens, block_size, max_blocks, num_blocks, device="cpu") -> PagedState:
    """Tables dealt from block 0 upward in sequence order; the rest of the
    pool on the free stack with the lowest free id on top."""
    B = len(ctx_lens)
    tables = torch.full((B, max_blocks), -1, dtype=torch.int32)
    nxt = 0
    for b, n in enumerate(ctx_lens):
        nb = (int(n) + block_size - 1) // block_size
        if nb > max_blocks or nxt + nb > num_blocks:
            raise ValueError("pool or table too small for the context lengths")
        tables[b, :nb] = torch.arange(nxt, nxt + nb, dtype=torch.int32)
        nxt += nb
    free = torch.full((num_blocks,), -1, dtype=torch.int32)
    rest = torch.arange(num_blocks - 1, nxt - 1, -1, dtype=torch.int32)
    free[:len(rest)] = rest
    return PagedState(tables.to(device), torch.tensor([int(n) for n in ctx_lens],
                                                      dtype=torch.int32).to(device),
                      free.to(device), torch.tensor([len(rest)], dtype=torch.int32).to(device),
                      block_size)


def context_lengths(B, lo, hi, seed):
    g = generator(seed, "cpu")
    return torch.randint(lo, hi + 1, (B,), generator=g).tolist()


def random_bf16(shape, gen, device):
    """Random finite bf16 payload (KV rows, hidden rows)."""
    return torch.randn(shape, generator=gen, device=device, dtype=torch.float32).to(torch.bfloat16)


# ----------------------------------------------------------------------------
# The workloads used by the tests and the benchmark
# ----------------------------------------------------------------------------

def chain_small(rnd=0, device="cpu"):
    """B=1, K=4, V=1024 fp32, l_f ~ N(0, 2^2), l_d = l_f + N(0, 1), T = 1,
    Philox seed 0; one round of a 100-round run (fresh logits per round)."""
    return chain_problem(1, 4, 1024, torch.float32, seed=0, rnd=rnd, device=device,
                         target_std=2.0, draft_noise=1.0, temperature=1.0, philox_seed=0)


def hier_peaked(device="cpu"):
    """B=8, K=4, N_i=4, V=32000 bf16; l_f ~ N(0, 2.5^2) with +6 on a
    Bernoulli(0.05) mask; l_i = l_f + N(0, 0.7^2); l_d = l_f + N(0, 1.5^2);
    T = 0.7 except sequence 0 at T = 0; Philox seed 1."""
    T = torch.full((8,), 0.7)
    T[0] = 0.0
    return hier_problem(8, 4, 4, 32000, torch.bfloat16, seed=1, device=device, final_std=2.5,
                        inter_noise=0.7, draft_noise=1.5, boost_p=0.05, boost=6.0,
                        temperature=T, philox_seed=1)


LLAMA3_V = 128256


def chain_batch(device="cpu", rnd=0, B=64, K=8, V=LLAMA3_V, seed=2, seq_id_base=0):
    """B=64, K=8, V=128256 bf16; l_t ~ N(0, 2^2) - 1.1 ln(id + 1);
    l_d = l_t + N(0, 1); T = 1; Philox seed 2."""
    return chain_problem(B, K, V, torch.bfloat16, seed=seed, rnd=rnd, device=device,
                         target_std=2.0, zipf_s=1.1, draft_noise=1.0, temperature=1.0,
                         philox_seed=2, seq_id_base=seq_id_base)


@dataclass
class CommitBuffers:
    kv_stage: torch.Tensor     # [B, K+1, layers, 2, heads, dim] bf16
    kv_pool: torch.Tensor      # [num_blocks, layers, 2, bs, heads, dim] bf16
    hid_stage: torch.Tensor    # [B, K+1, hidden] bf16
    hid_out: torch.Tensor      # [B*(K+1), hidden] bf16
    hid_off: torch.Tensor      # int32 [B+1]


def commit_setup(B, K, ctx_lo=512, ctx_hi=4096, block_size=16, layers=32, heads=8, dim=128,
                 hidden=4096, spare_blocks=None, extra_len=0, seed=2, device="cpu",
                 with_kv=True):
    """Paged state for contexts U[ctx_lo, ctx_hi] plus staged KV / hidden rows."""
    ctx = context_lengths(B, ctx_lo, ctx_hi, seed)
    need = sum((n + block_size - 1) // block_size for n in ctx)
    max_len = max(ctx) + K + 1 + extra_len
    max_blocks = (max_len + block_size - 1) // block_size + 1
    spare = spare_blocks if spare_blocks is not None else B * ((K + block_size) // block_size + 1)
    state = paged_state(ctx, block_size, max_blocks, need + spare, device)
    bufs = None
    if with_kv:
        gen = generator(seed * 31 + 5, device)
        nb = need + spare
        bufs = CommitBuffers(
            random_bf16((B, K + 1, layers, 2, heads, dim), gen, device),
            torch.zeros((nb, layers, 2, block_size, heads, dim), dtype=torch.bfloat16,
                        device=device),
            random_bf16((B, K + 1, hidden), gen, device),
            torch.zeros((B * (K + 1), hidden), dtype=torch.bfloat16, device=device),
            torch.zeros((B + 1,), dtype=torch.int32, device=device))
    return state, bufs


def hier_mixed(device="cpu"):
    """B=256, K=4, N_i=4, V=151936 fp32; T ~ U(0, 1.2] with exactly 51
    sequences at 0; l_f ~ N(0, 2^2), l_i = l_f + N(0, 0.5^2),
    l_d = l_f + N(0, 2^2); Philox seed 3."""
    gen = generator(3, "cpu")
    T = mixed_temperatures(256, round(0.2 * 256), 1.2, gen, "cpu")
    return hier_problem(256, 4, 4, 151936, torch.float32, seed=3, device=device,
                        final_std=2.0, inter_noise=0.5, draft_noise=2.0, temperature=T,
                        philox_seed=3)


def engine_round_logits(B, S, V, rnd, device, seed=4):
    """Per-round logits of the engine loop: l_f ~ N(0, 2^2),
    l_i = l_f + N(0, 0.5^2), l_d = l_f + N(0, 1), bf16, drawn from a
    generator seeded by (seed, round)."""
    gen = generator(seed * 1_000_003 + rnd + 1, device)
    return hier_logits(B, S, V, torch.bfloat16, gen, device, final_std=2.0,
                       inter_noise=0.5, draft_noise=1.0), gen
