// Chain verification step: row statistics, accept tests, draws and the paged
// commit of the kept rows in one persistent launch (after a prologue launch
// that clears the call's counters).
//
// What it computes is the chain check of HiSpec (gist.science summary of
// arXiv 2510.01336, section 2, "Verlustfreie Garantie": the lossless check of
// speculative sampling) and the buffered-entry pruning with paged block tables
// of the same section ("Wiederverwendung von KV-Cache und versteckten
// Zustaenden", "Unterstuetzung fuer Batch-Inferenz"); accepted count plus
// drawn token per sequence as in Speculative Speculative Decoding (summary,
// Technische Zusammenfassung 2.1), the residual proportional to the target-
// minus-draft difference (same page, 3.B).
//
// Design (B200). One CTA of 16 warps per SM; every warp is an independent
// worker and every hand-out comes from a counter in global memory, so no
// warp waits for a CTA or for the grid:
//   1. Stream: the (row, chunk) items of all rows the check needs -- chunks of
//      about kChunkTiles 6 KiB tiles, staged by 1-D bulk copies into a
//      per-warp ring of two tiles -- handed out one at a time in a fixed
//      order (rows of late positions last, so the rows the draws re-read are
//      still in L2). A chunk ends in one ChunkStat (max, shift, sum of
//      2^(l*c - M) or first argmax); the warp that completes the last chunk
//      of a sequence combines its rows and runs its accept test at once.
//   2. Draws: each sampled sequence's residual (or bonus) row pair is cut
//      into D parts of 256-element tiles; whichever warp finishes the last
//      part prefixes the tile sums, finds the tile holding u * Z, rescans it
//      and writes the token.
//   3. Commit (optional): the warp that checks the last sequence plans the
//      commit (frees and allocations in sequence order, lengths, offsets);
//      then every warp copies 8 KiB units of the kept K/V and hidden rows.
// A warp waits only for work that a running warp has already taken (a
// sequence's last chunk, a plan), with a bounded wait that records
// SPEC_ETIMEOUT and stops every other wait; no co-residency is assumed.
#include <algorithm>
#include <climits>

#include "commit.cuh"
#include "draw.cuh"
#include "rowmath.cuh"

namespace specv {

constexpr int kFifo = 4;  // items a warp's producer may run ahead (ring of 2 tiles)

// A stream item as the warp's producer resolved it (shared memory).
struct StepItem {
  const unsigned char* rowp;
  int b, r, c, t0, t1;
  int greedy, early;
  float chi, clo;  // the temperature scale c = chi + clo (sampled rows)
  int nc;          // chunks of this row
  int pad;
};
// A finished chunk whose row count is checked one chunk later.
struct PendRow {
  int row, b, nc, greedy;
  float chi;
  int on;
};
constexpr int kTempCache = 2048;  // temperatures kept in shared memory (B up to this)
constexpr int kStepSmem = kRsSmem + kRsWarps * kFifo * (int)sizeof(StepItem) +
                          kTempCache * (int)sizeof(float);
static_assert(kStepSmem <= 227 * 1024, "step kernel shared memory");

// ---------------------------------------------------------------------------
// Flags in global memory
// ---------------------------------------------------------------------------
__device__ __forceinline__ int atom_add_acq_rel(int* p, int v) {
  int old;
  asm volatile("atom.add.acq_rel.gpu.global.s32 %0, [%1], %2;" : "=r"(old) : "l"(p), "r"(v) : "memory");
  return old;
}
__device__ __forceinline__ int atom_add_release(int* p, int v) {
  int old;
  asm volatile("atom.add.release.gpu.global.s32 %0, [%1], %2;" : "=r"(old) : "l"(p), "r"(v) : "memory");
  return old;
}

// Give up every wait of the call: record the timeout once and raise `abort`.
__device__ __forceinline__ void step_abort(const StepArgs& A) {
  set_status(A.status, SPEC_ETIMEOUT);
  atomicExch(&A.ctr->abort, 1);
}

// Wait (one lane) until *flag != 0; returns the value, or 0 when the wait ran
// out or the call was aborted. The polls back off exponentially (to about
// 2 us) and look at the abort word every 8th time, so a crowd of waiting
// warps does not keep one L2 slice busy.
__device__ int wait_flag(const StepArgs& A, const int* flag) {
  // Polls are relaxed (an acquire per poll would drop the SM's L1 each time);
  // one acquire fence follows the poll that sees the flag.
  int v = ld_relaxed(flag);
  if (v) {
    fence_acq_rel();
    return v;
  }
  const uint64_t t0 = globaltimer_ns();
  unsigned ns = 128;
  for (unsigned k = 1;; ++k) {
    __nanosleep(ns);
    if (ns < 2048) ns <<= 1;
    v = ld_relaxed(flag);
    if (v) {
      fence_acq_rel();
      return v;
    }
    if ((k & 7) == 0) {
      if (ld_relaxed(&A.ctr->abort)) return 0;
      if (globaltimer_ns() - t0 > kWaitLimitNs) {
        step_abort(A);
        return 0;
      }
    }
  }
}
__device__ __forceinline__ int warp_wait_flag(const StepArgs& A, const int* flag) {
  int v = 0;
  if ((threadIdx.x & 31) == 0) v = wait_flag(A, flag);
  return __shfl_sync(0xffffffffu, v, 0);
}

__device__ __forceinline__ unsigned warp_grab(unsigned* ctr) {
  unsigned i = 0;
  if ((threadIdx.x & 31) == 0) i = atomicAdd(ctr, 1u);
  return __shfl_sync(0xffffffffu, i, 0);
}

// ---------------------------------------------------------------------------
// Item map: item i -> (sequence, row, chunk). Early items come first in
// sequence order (per sequence: target rows lp..K, then draft rows lp..K-1),
// then the late items (target rows 0..lp-1, then draft rows 0..lp-1).
// Row index r within a sequence: target row j is r = j, draft row j is
// r = K + 1 + j. Returns false for rows the check does not need.
// ---------------------------------------------------------------------------
__device__ __forceinline__ bool map_item(const StepArgs& A, unsigned i, const float* s_temp,
                                         StepItem* it) {
  const int K = A.K, lp = A.lp;
  int b, rr, c, r, NC;
  bool early;
  if (i < A.n_early) {
    NC = A.NCe;
    const unsigned per = (unsigned)A.re * NC;
    b = (int)(i / per);
    const int rem = (int)(i - (unsigned)b * per);
    rr = rem / NC;
    c = rem - rr * NC;
    const int nt_rows = K + 1 - lp;
    r = rr < nt_rows ? lp + rr : K + 1 + lp + (rr - nt_rows);
    early = true;
  } else {
    NC = A.NCl;
    const unsigned j = i - A.n_early, per = (unsigned)A.rl * NC;
    b = (int)(j / per);
    const int rem = (int)(j - (unsigned)b * per);
    rr = rem / NC;
    c = rem - rr * NC;
    r = rr < lp ? rr : K + 1 + (rr - lp);
    early = false;
  }
  const float T = A.B <= kTempCache ? s_temp[b] : __ldg(A.temperature + b);
  if (!temp_valid(T) || (r > K && T == 0.0f)) return false;
  it->rowp = r <= K ? A.tgt + ((long long)b * (K + 1) + r) * A.ld_tgt
                    : A.drf + ((long long)b * K + (r - K - 1)) * A.ld_drf;
  it->b = b;
  it->r = r;
  it->c = c;
  it->t0 = (int)((long long)c * A.nt / NC);
  it->t1 = (int)((long long)(c + 1) * A.nt / NC);
  it->greedy = T == 0.0f;
  it->early = early;
  if (T != 0.0f) {
    const Scale sc = make_scale(T);
    it->chi = sc.hi;
    it->clo = sc.lo;
  } else {
    it->chi = it->clo = 0.0f;
  }
  it->nc = NC;
  return true;
}

// ---------------------------------------------------------------------------
// Combine a row's chunks (one lane per row)
// ---------------------------------------------------------------------------
__device__ __forceinline__ ChunkStat ld_chunk(const ChunkStat* p) {
  const double2 v = __ldcg(reinterpret_cast<const double2*>(p));
  ChunkStat c;
  const unsigned long long w = (unsigned long long)__double_as_longlong(v.x);
  c.m = __uint_as_float((unsigned)(w & 0xffffffffull));
  c.aux = (int)(w >> 32);
  c.s = v.y;
  return c;
}

// Row statistics from its NC chunks (one warp, every lane's chunks loaded
// together): max m (first index for greedy rows), shift M = fl(m * c_hi) and
// L = log2 sum 2^(l*c - M), so the row's log2-partition is M + L. Valid in
// every lane.
__device__ RowFinal warp_combine_row(const ChunkStat* p, int NC, bool greedy, float chi) {
  const int lane = threadIdx.x & 31;
  float m = -INFINITY;
  int idx = INT_MAX;
  for (int c = lane; c < NC; c += 32) {
    const ChunkStat q = ld_chunk(p + c);
    // chunks in index order: among equal maxima the earlier chunk's index wins
    if (q.m > m || (greedy && q.m == m && q.aux < idx)) {
      m = q.m;
      idx = q.aux;
    }
  }
  if (greedy) {
    warp_argmax(m, idx);
  } else {
#pragma unroll
    for (int o = 16; o; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
  }
  RowFinal f;
  f.m = m;
  f.amax = greedy ? idx : -1;
  f.M = 0.0;
  f.L = 0.0;
  f.pad = 0;
  bool ok = (m > -INFINITY && m < INFINITY);
  if (ok && !greedy) {
    f.M = (double)__fmul_rn(m, chi);
    double sl = 0.0;
    for (int c = lane; c < NC; c += 32) {
      const ChunkStat q = ld_chunk(p + c);
      if (q.s != 0.0) sl += q.s * exp2((double)__int_as_float(q.aux) - f.M);
    }
    const double sum = warp_sum_d(sl);
    ok = (sum > 0.0 && sum < INFINITY);
    f.L = log2(sum);
  }
  f.ok = ok;
  return f;
}

__device__ __forceinline__ RowFinal ld_final(const RowFinal* p) {
  RowFinal f;
  f.M = __ldcg(&p->M);
  f.L = __ldcg(&p->L);
  f.m = __ldcg(&p->m);
  f.amax = __ldcg(&p->amax);
  f.ok = __ldcg(&p->ok);
  f.pad = 0;
  return f;
}

// ---------------------------------------------------------------------------
// Commit: the plan (one warp) once every sequence is checked
// ---------------------------------------------------------------------------
// Frees (table tails past the new length, sequences ascending, pushed), then
// allocations (missing blocks, sequences ascending, popped), lengths, hidden
// offsets, the kept-token map for the copy units. Every check comes before
// any write; a failed check records its status and plans nothing.
__device__ __noinline__ void plan_warp(const StepArgs& A) {
  const CommitArgs& a = A.cm;
  const int lane = threadIdx.x & 31;
  const int B = a.B, bs = a.block_size;
  __threadfence();  // every sequence's snapshot was released before its ticket
  int st0 = 0;
  if (lane == 0) st0 = a.status ? *(volatile int32_t*)a.status : SPEC_OK;
  st0 = __shfl_sync(0xffffffffu, st0, 0);
  auto finish = [&](int v) {
    __threadfence();
    if (lane == 0) st_release(&A.ctr->plan, v);
  };
  if (st0 != SPEC_OK) {
    finish(2);
    return;
  }
  const int per = (B + 31) / 32;
  const int b0 = min(B, lane * per), b1 = min(B, b0 + per);
  int nf = 0, na = 0, nk = 0, bad = 0;
  for (int b = b0; b < b1; ++b) {
    const SeqState* s = A.seq + b;
    const int old_len = __ldcg(&s->old_len), base = __ldcg(&s->base), kept = __ldcg(&s->kept);
    bad |= __ldcg(&s->bad);
    const int nbo = ceil_div(max(old_len, 0), bs), nbn = ceil_div(base + kept, bs);
    nf += max(0, nbo - nbn);
    na += max(0, nbn - nbo);
    nk += kept;
  }
  // Exclusive prefixes over the lanes' runs (sequence order).
  int pf = nf, pa = na, pk = nk;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int yf = __shfl_up_sync(0xffffffffu, pf, o);
    const int ya = __shfl_up_sync(0xffffffffu, pa, o);
    const int yk = __shfl_up_sync(0xffffffffu, pk, o);
    if (lane >= o) { pf += yf; pa += ya; pk += yk; }
  }
  const int F = __shfl_sync(0xffffffffu, pf, 31), NA = __shfl_sync(0xffffffffu, pa, 31);
  const int KT = __shfl_sync(0xffffffffu, pk, 31);
  pf -= nf;
  pa -= na;
  pk -= nk;
  const bool anybad = __any_sync(0xffffffffu, bad);
  int ft = 0;
  if (lane == 0) ft = *(volatile int32_t*)a.free_top;
  ft = __shfl_sync(0xffffffffu, ft, 0);
  int code = 0;
  if (anybad || ft < 0 || ft > a.num_blocks || ft + F > a.num_blocks) {
    code = SPEC_EINVAL;
  } else if (ft + F < NA) {
    code = SPEC_ENOBLOCKS;
  } else {
    // Stack entries popped from below the old top must be valid block ids.
    const int lo = max(0, ft + F - NA);
    int sbad = 0;
    for (int p = lo + lane; p < ft; p += 32) {
      const int x = __ldcg(a.free_stack + p);
      if (x < 0 || x >= a.num_blocks) sbad = 1;
    }
    if (__any_sync(0xffffffffu, sbad)) code = SPEC_EINVAL;
  }
  if (code) {
    if (lane == 0) set_status(a.status, code);
    finish(2);
    return;
  }
  // Frees: push table tails in sequence order.
  int fpos = pf;
  for (int b = b0; b < b1; ++b) {
    const SeqState* s = A.seq + b;
    const int old_len = __ldcg(&s->old_len), base = __ldcg(&s->base), kept = __ldcg(&s->kept);
    const int held = ceil_div(max(old_len, 0), bs);
    int32_t* tab = a.tables + (size_t)b * a.max_blocks;
    for (int i = ceil_div(base + kept, bs); i < held; ++i) {
      a.free_stack[ft + fpos++] = __ldcg(tab + i);
      tab[i] = -1;
    }
  }
  __threadfence();
  __syncwarp();
  // Allocations: pop from the new top in sequence order; lengths, offsets and
  // the sequence of every kept token.
  const int top = ft + F;
  int k = pa, off = pk;
  for (int b = b0; b < b1; ++b) {
    const SeqState* s = A.seq + b;
    const int old_len = __ldcg(&s->old_len), base = __ldcg(&s->base), kept = __ldcg(&s->kept);
    const int held = ceil_div(max(old_len, 0), bs), nbn = ceil_div(base + kept, bs);
    int32_t* tab = a.tables + (size_t)b * a.max_blocks;
    for (int i = held; i < nbn; ++i) tab[i] = __ldcg(a.free_stack + (top - 1 - (k++)));
    if (a.hid_off) a.hid_off[b] = off;
    A.tok_off[b] = off;
    for (int t = 0; t < kept; ++t) A.tok_seq[off + t] = b;
    off += kept;
    a.seq_lens[b] = base + kept;
  }
  if (lane == 0) {
    *a.free_top = top - NA;
    if (a.hid_off) a.hid_off[B] = KT;
    A.ctr->kt = KT;
  }
  finish(1);
}

// ---------------------------------------------------------------------------
// Accept test of one sequence (one warp), once all its chunks are in
// ---------------------------------------------------------------------------
template <typename T, bool kCommit>
__device__ __noinline__ void accept_seq(const StepArgs& A, int b) {
  const int lane = threadIdx.x & 31;
  const int K = A.K, V = A.V, R = 2 * K + 1;
  const float Tb = __ldg(A.temperature + b);  // valid: invalid ones never reach here
  const bool greedy = (Tb == 0.0f);
  const Scale sc = greedy ? Scale{0.f, 0.f, 0.0} : make_scale(Tb);
  const int32_t* drafts = A.draft_tok + (size_t)b * K;
  double* diag = A.diag ? A.diag + (size_t)b * (4 * K + 2) : nullptr;
  const RowFinal* fr = A.fin + (size_t)b * R;
  const uint32_t sid = (uint32_t)__ldg(A.seq_id + b);
  int a = K, bad = 0;
  bool captured = false;
  double lt_a = 0.0, lq_a = 0.0;
  float mt_a = 0.0f, mq_a = 0.0f;
  int amax_a = -1;
  float u_a = 0.0f;
  for (int j0 = 0; j0 <= K; j0 += 32) {
    const int j = j0 + lane;
    // This lane's draft id, its two logits and the rows' statistics: every
    // load of the group issued before any is used.
    const int x = j < K ? __ldg(drafts + j) : -1;
    const bool xok = (x >= 0 && x < V);
    float lt = 0.0f, ld = 0.0f;
    if (j < K && xok && !greedy) {
      lt = load_elem(reinterpret_cast<const T*>(A.tgt + ((long long)b * (K + 1) + j) * A.ld_tgt) + x);
      ld = load_elem(reinterpret_cast<const T*>(A.drf + ((long long)b * K + j) * A.ld_drf) + x);
    }
    RowFinal ft{0.0, 0.0, 0.f, -1, 1, 0}, fd{0.0, 0.0, 0.f, -1, 1, 0};
    if (j <= K) ft = ld_final(fr + j);
    if (j < K && !greedy) fd = ld_final(fr + K + 1 + j);
    bool acc = true, badj = (j <= K && !ft.ok) || (j < K && !greedy && !fd.ok);
    float ud = 0.0f;
    if (j < K) {
      if (!xok) {
        badj = true;
      } else if (greedy) {
        acc = (x == ft.amax);
      } else {
        const double lp = (double)lt * sc.d - (ft.M + ft.L);
        const double lq = (double)ld * sc.d - (fd.M + fd.L);
        const float2 u = spec_uniforms(A.seed, sid, A.round, (uint32_t)j, 1u);
        acc = (double)u.x < exp2(lp - lq);
        ud = u.y;
        if (diag) {
          diag[2 * K + 1 + j] = exp2(lp);
          diag[3 * K + 1 + j] = exp2(lq);
        }
      }
    } else if (j == K && !greedy) {
      ud = spec_uniforms(A.seed, sid, A.round, (uint32_t)K, 1u).y;
    }
    if (diag && !greedy) {
      if (j <= K) diag[j] = (ft.M + ft.L) * kLn2;
      if (j < K) diag[K + 1 + j] = (fd.M + fd.L) * kLn2;
    }
    if (__any_sync(0xffffffffu, badj)) bad = 1;
    const unsigned rej = __ballot_sync(0xffffffffu, j < K && !acc);
    if (a == K && rej) a = j0 + __ffs(rej) - 1;
    if (!captured && a >= j0 && a < j0 + 32) {
      const int src = a - j0;
      lt_a = __shfl_sync(0xffffffffu, ft.M + ft.L, src);
      lq_a = __shfl_sync(0xffffffffu, fd.M + fd.L, src);
      mt_a = __shfl_sync(0xffffffffu, ft.m, src);
      mq_a = __shfl_sync(0xffffffffu, fd.m, src);
      amax_a = __shfl_sync(0xffffffffu, ft.amax, src);
      u_a = __shfl_sync(0xffffffffu, ud, src);
      captured = true;
    }
  }
  int32_t* out = A.out_tok + (size_t)b * (K + 1);
  SeqState* st = A.seq + b;
  __syncwarp();  // the loop's diagnostics come before any overwrite below
  if (bad) {
    if (lane == 0) {
      set_status(A.status, SPEC_EDEVICE);
      A.accept_len[b] = -1;
    }
    for (int j = lane; j <= K; j += 32) out[j] = -1;
    if (diag)
      for (int j = lane; j < 4 * K + 2; j += 32) diag[j] = dnan();
    a = -1;
  } else {
    // A sampled sequence's token at a is written by its draw.
    for (int j = lane; j <= K; j += 32)
      if (j != a || greedy) out[j] = j < a ? __ldg(drafts + j) : (j == a ? amax_a : -1);
    if (lane == 0) A.accept_len[b] = a;
    if (diag && greedy)
      for (int j = lane; j < 4 * K + 2; j += 32) diag[j] = dnan();
  }
  if (lane == 0) {
    st->lt = lt_a;
    st->lq = lq_a;
    st->mt = mt_a;
    st->mq = mq_a;
    st->u = u_a;
    st->a = a;
    st->flags = (!bad && !greedy ? kSeqDraw : 0) | (a >= 0 && a < K ? kSeqHasQ : 0);
  }
  if constexpr (kCommit) {
    // Snapshot of the lengths before the plan changes them, and the checks
    // of this sequence's part of the commit (the plan makes the global ones).
    const CommitArgs& c = A.cm;
    const int old_len = *(volatile int32_t*)(c.seq_lens + b);
    const int base = c.base_len ? __ldg(c.base_len + b) : old_len;
    const int kept = a + 1;
    const int nbo = ceil_div(max(old_len, 0), c.block_size);
    const int nbn = ceil_div(base + kept, c.block_size);
    int cbad = (kept < 0 || kept > c.Kp1 || base < 0 || base > old_len || old_len < 0 ||
                nbo > c.max_blocks || nbn > c.max_blocks);
    if (!cbad) {
      const int32_t* tab = c.tables + (size_t)b * c.max_blocks;
      int e = 0;
      for (int i = lane; i < nbo; i += 32) {
        const int v = __ldcg(tab + i);
        if (v < 0 || v >= c.num_blocks) e = 1;
      }
      cbad = __any_sync(0xffffffffu, e);
    }
    if (lane == 0) {
      st->old_len = old_len;
      st->base = base;
      st->kept = kept;
      st->bad = cbad;
    }
  }
  __threadfence();
  __syncwarp();
  if (lane == 0) st_release(A.seq_done + b, 1);
  if constexpr (kCommit) {
    int last = 0;
    if (lane == 0) last = (atomicAdd(&A.ctr->ticket, 1) + 1 == A.B);
    if (__shfl_sync(0xffffffffu, last, 0)) plan_warp(A);
  }
}

// ---------------------------------------------------------------------------
// Draws
// ---------------------------------------------------------------------------
// The warp's copy ring (idle once its stream items are done) holds a draw
// part's slice of each row: a part is kPartBytes of the p row and of the q
// row, fetched by two bulk copies that land on the ring's two mbarriers.
struct WarpRing {
  unsigned char* buf;  // two stages of kTileBytes
  uint64_t* bars;      // their mbarriers
  uint32_t* phase;     // the stages' parity bits (shared memory, lane-uniform)
};

// Tile sums of the weights over residual tiles [t0, t1) of one row pair (one
// warp) to out[t]; returns their sum in tile order (every lane). The slice
// [t0*256, min(V, t1*256)) of each row is staged in the ring first; a sub-
// 16-byte ragged end is read from global memory.
template <typename T>
__device__ double warp_tile_sums(const T* prow, const T* qrow, int V, const ProbCoef& kp,
                                 const ProbCoef& kq, int t0, int t1, double* out,
                                 const WarpRing& ring) {
  const int lane = threadIdx.x & 31;
  const bool hq = qrow != nullptr;
  const int e0 = t0 * kResTile, e1 = min(V, t1 * kResTile);
  const uint32_t bytes = ((uint32_t)(e1 - e0) * sizeof(T)) & ~15u;
  const int nfull = (int)(bytes / sizeof(T));  // elements staged
  if (lane == 0) {
    fence_proxy_async_smem();
    mbar_arrive_expect_tx(&ring.bars[0], bytes);
    if (bytes) bulk_g2s(ring.buf, prow + e0, bytes, &ring.bars[0]);
    const uint32_t qb = hq ? bytes : 0u;
    mbar_arrive_expect_tx(&ring.bars[1], qb);
    if (qb) bulk_g2s(ring.buf + kTileBytes, qrow + e0, qb, &ring.bars[1]);
  }
  uint32_t ph = *ring.phase;
  const bool ok0 = mbar_wait_bounded(&ring.bars[0], ph & 1u, kWaitLimitNs);
  const bool ok1 = mbar_wait_bounded(&ring.bars[1], (ph >> 1) & 1u, kWaitLimitNs);
  __syncwarp();
  if (lane == 0) *ring.phase = ph ^ 3u;
  double total = 0.0;
  if (!__all_sync(0xffffffffu, ok0 && ok1)) return -1.0;  // timed out: the caller aborts
  const T* sp = reinterpret_cast<const T*>(ring.buf);
  const T* sq = reinterpret_cast<const T*>(ring.buf + kTileBytes);
  for (int t = t0; t < t1; ++t) {
    const int le = (t - t0) * kResTile + lane * 8, e = e0 + le;
    float w[8];
    if (le + 8 <= nfull) {
      float xp[8], xq[8];
      unpack8(*reinterpret_cast<const Raw8<T>*>(sp + le), xp);
      if (hq) unpack8(*reinterpret_cast<const Raw8<T>*>(sq + le), xq);
      weights_of(xp, xq, hq, kp, kq, w);
    } else if (e < V) {
      weights8<T>(prow, qrow, e, V, kp, kq, w);  // the row's ragged end
    } else {
#pragma unroll
      for (int k = 0; k < 8; ++k) w[k] = 0.0f;
    }
    const double v = warp_sum_d(lane_sum8(w));
    if (lane == 0) out[t] = v;
    total += v;
  }
  __syncwarp();  // every lane's reads of the ring come before its next refill
  return total;
}

// Among n values v[0..n) spread over the lanes (lane l holds the contiguous
// run [l*per, l*per + per)), prefix them in that order starting from `base`
// and find the last index with v > 0 whose prefix does not exceed `target`.
// Returns the index (-1 if none) and its prefix in *pre; *total = base +
// sum of all. Loads come from global memory through L2.
__device__ int warp_find(const double* v, int n, double base, double target, double* pre,
                         double* total) {
  const int lane = threadIdx.x & 31;
  const int per = (n + 31) / 32;
  const int a0 = min(n, lane * per), a1 = min(n, a0 + per);
  constexpr int kReg = 4;
  double r[kReg];
  double run = 0.0;
#pragma unroll
  for (int k = 0; k < kReg; ++k) r[k] = (a0 + k < a1) ? __ldcg(v + a0 + k) : 0.0;
#pragma unroll
  for (int k = 0; k < kReg; ++k) run += r[k];
  for (int t = a0 + kReg; t < a1; ++t) run += __ldcg(v + t);
  double incl = run;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const double y = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += y;
  }
  *total = base + __shfl_sync(0xffffffffu, incl, 31);
  double c = base + incl - run, cpre = 0.0;
  int cand = -1;
#pragma unroll
  for (int k = 0; k < kReg; ++k)
    if (a0 + k < a1) {
      if (c <= target && r[k] > 0.0) { cand = a0 + k; cpre = c; }
      c += r[k];
    }
  for (int t = a0 + kReg; t < a1; ++t) {
    const double x = __ldcg(v + t);
    if (c <= target && x > 0.0) { cand = t; cpre = c; }
    c += x;
  }
  int best = cand;
#pragma unroll
  for (int o = 16; o; o >>= 1) best = max(best, __shfl_xor_sync(0xffffffffu, best, o));
  const unsigned who = __ballot_sync(0xffffffffu, cand == best && best >= 0);
  *pre = who ? __shfl_sync(0xffffffffu, cpre, __ffs(who) - 1) : 0.0;
  return best;
}

// The draw from the part totals and tile sums of a row pair (one warp):
// find the draw part, then the tile in it, whose prefix holds u * Z, then
// rescan that tile. Returns the token (-1 if there is no mass); *Z_out gets
// Z.
template <typename T>
__device__ int warp_pick(const StepArgs& A, int b, const T* prow, const T* qrow,
                         const ProbCoef& kp, const ProbCoef& kq, float u, double* Z_out) {
  const int lane = threadIdx.x & 31;
  const int V = A.V, nrt = A.nrt, D = A.D;
  const double* ts = A.tsum + (size_t)b * nrt;
  const double* pt = A.ptot + (size_t)b * D;
  // Z, in the order of the parts.
  double Z, pre_p;
  int part = warp_find(pt, D, 0.0, -1.0, &pre_p, &Z);
  *Z_out = Z;
  if (!(Z > 0.0)) return -1;
  const double target = (double)u * Z;
  part = warp_find(pt, D, 0.0, target, &pre_p, &Z);
  if (part < 0) part = 0;
  constexpr int PT = part_tiles((int)sizeof(T));
  const int t0 = part * PT, t1 = min(nrt, t0 + PT);
  double pre_t, zt;
  int tile = warp_find(ts + t0, t1 - t0, pre_p, target, &pre_t, &zt);
  if (tile < 0) {
    tile = 0;
    pre_t = pre_p;
  }
  tile += t0;
  float w[8];
  weights8<T>(prow, qrow, tile * kResTile + lane * 8, V, kp, kq, w);
  const double ls = lane_sum8(w);
  double li = ls;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const double y = __shfl_up_sync(0xffffffffu, li, o);
    if (lane >= o) li += y;
  }
  const double start = pre_t + (li - ls);
  int found = INT_MAX;
  if (start <= target) {
    double acc = start;
    for (int e = 0; e < 8; ++e) {
      acc += (double)w[e];
      if (acc > target && w[e] > 0.0f) {
        found = tile * kResTile + lane * 8 + e;
        break;
      }
    }
  }
#pragma unroll
  for (int o = 16; o; o >>= 1) found = min(found, __shfl_xor_sync(0xffffffffu, found, o));
  if (found == INT_MAX) {
    // The target sits at this tile's end by rounding: last element with mass.
    int last = -1;
    for (int e = 7; e >= 0; --e)
      if (w[e] > 0.0f) {
        last = tile * kResTile + lane * 8 + e;
        break;
      }
#pragma unroll
    for (int o = 16; o; o >>= 1) last = max(last, __shfl_xor_sync(0xffffffffu, last, o));
    found = last;
  }
  return found;
}

// Tile sums and total of draw part d of sequence b's row pair; false if a
// wait for the staged slice ran out.
template <typename T>
__device__ __forceinline__ bool part_sums(const StepArgs& A, int b, int d, const T* prow,
                                          const T* qrow, const ProbCoef& kp, const ProbCoef& kq,
                                          const WarpRing& ring) {
  constexpr int PT = part_tiles((int)sizeof(T));
  const int t0 = d * PT, t1 = min(A.nrt, t0 + PT);
  const double tot = warp_tile_sums<T>(prow, qrow, A.V, kp, kq, t0, t1,
                                       A.tsum + (size_t)b * A.nrt, ring);
  if (tot < 0.0) return false;
  if ((threadIdx.x & 31) == 0) A.ptot[(size_t)b * A.D + d] = tot;
  return true;
}

template <typename T>
__device__ __noinline__ void draw_part(const StepArgs& A, int b, int d, const WarpRing& ring) {
  const int lane = threadIdx.x & 31;
  if (!warp_wait_flag(A, A.seq_done + b)) return;
  const SeqState* st = A.seq + b;
  const int flags = __ldcg(&st->flags);
  if (!(flags & kSeqDraw)) return;
  const int a = __ldcg(&st->a), K = A.K;
  const Scale sc = make_scale(__ldg(A.temperature + b));
  const ProbCoef kp = make_coef(__ldcg(&st->lt), __ldcg(&st->mt), sc);
  const bool hq = (flags & kSeqHasQ) != 0;
  const ProbCoef kq = hq ? make_coef(__ldcg(&st->lq), __ldcg(&st->mq), sc) : make_coef(0.0, 0.0f, sc);
  const T* prow = reinterpret_cast<const T*>(A.tgt + ((long long)b * (K + 1) + a) * A.ld_tgt);
  const T* qrow =
      hq ? reinterpret_cast<const T*>(A.drf + ((long long)b * K + a) * A.ld_drf) : nullptr;
  if (!part_sums<T>(A, b, d, prow, qrow, kp, kq, ring)) {
    if (lane == 0) step_abort(A);
    return;
  }
  int last = 0;
  if (lane == 0) last = (atom_add_acq_rel(A.draw_cnt + b, 1) + 1 == A.D);
  if (!__shfl_sync(0xffffffffu, last, 0)) return;
  fence_acq_rel();
  const float u = __ldcg(&st->u);
  double Z;
  int tok = warp_pick<T>(A, b, prow, qrow, kp, kq, u, &Z);
  if (tok < 0 && qrow) {
    // No residual mass as computed (p == q): draw from p (this warp alone).
    for (int dd = 0; dd < A.D; ++dd)
      if (!part_sums<T>(A, b, dd, prow, nullptr, kp, kq, ring)) {
        if (lane == 0) step_abort(A);
        return;
      }
    __threadfence();
    __syncwarp();
    tok = warp_pick<T>(A, b, prow, nullptr, kp, kq, u, &Z);
  }
  if (lane == 0) {
    A.out_tok[(size_t)b * (K + 1) + a] = tok;
    if (A.diag) A.diag[(size_t)b * (4 * K + 2) + 4 * K + 1] = Z;
  }
}

// ---------------------------------------------------------------------------
// Copies of kept rows (after the plan)
// ---------------------------------------------------------------------------
// Unit u: kept token k = u / units_tok; part h = u % units_tok -- K/V
// segments [h*unit_segs, ...) of that token, or (h == units_kv) its hidden
// row. The source of a token's K/V row is contiguous; each segment goes to
// its own pool slot.
__device__ __noinline__ void copy_unit(const StepArgs& A, unsigned u) {
  const CommitArgs& a = A.cm;
  const int lane = threadIdx.x & 31;
  const int k = (int)(u / (unsigned)A.units_tok), h = (int)(u % (unsigned)A.units_tok);
  const int b = __ldcg(A.tok_seq + k);
  const int i = k - __ldcg(A.tok_off + b);
  const int pos = __ldcg(&A.seq[b].base) + i;
  if (h < A.units_kv) {
    const int nseg = a.layers * 2;
    const int s0 = h * A.unit_segs, s1 = min(nseg, s0 + A.unit_segs);
    const int blk = __ldcg(a.tables + (size_t)b * a.max_blocks + pos / a.block_size);
    const int slot = pos % a.block_size;
    const int vps = a.seg_bytes / 16;
    const uint4* src = reinterpret_cast<const uint4*>(
        a.kv_stage + (((size_t)b * a.Kp1 + i) * nseg + s0) * a.seg_bytes);
    const int nvec = (s1 - s0) * vps;
    for (int v0 = lane; v0 < nvec; v0 += 32 * 8) {
      uint4 r[8];
#pragma unroll
      for (int q = 0; q < 8; ++q)
        if (v0 + 32 * q < nvec) r[q] = __ldcg(src + v0 + 32 * q);
#pragma unroll
      for (int q = 0; q < 8; ++q) {
        const int v = v0 + 32 * q;
        if (v < nvec) {
          const int s = s0 + v / vps, o = v - (v / vps) * vps;
          uint4* dst = reinterpret_cast<uint4*>(
              a.kv_pool + (((size_t)blk * nseg + s) * a.block_size + slot) * (size_t)a.seg_bytes);
          __stcs(dst + o, r[q]);
        }
      }
    }
  } else {
    const uint4* src =
        reinterpret_cast<const uint4*>(a.hid_stage + ((size_t)b * a.Kp1 + i) * a.hid_bytes);
    uint4* dst = reinterpret_cast<uint4*>(a.hid_out +
                                          (size_t)(__ldcg(A.tok_off + b) + i) * a.hid_bytes);
    const int nvec = a.hid_bytes / 16;
    for (int v0 = lane; v0 < nvec; v0 += 32 * 8) {
      uint4 r[8];
#pragma unroll
      for (int q = 0; q < 8; ++q)
        if (v0 + 32 * q < nvec) r[q] = __ldcg(src + v0 + 32 * q);
#pragma unroll
      for (int q = 0; q < 8; ++q)
        if (v0 + 32 * q < nvec) __stcs(dst + v0 + 32 * q, r[q]);
    }
  }
}

// ---------------------------------------------------------------------------
// Prologue: clear the counters; fail the sequences with invalid temperatures
// (none of their rows is streamed).
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(1024) step_prologue_kernel(const __grid_constant__ StepArgs A) {
  pdl_begin();
  const size_t rows = (size_t)A.B * (2 * A.K + 1);
  for (size_t r = (size_t)blockIdx.x * blockDim.x + threadIdx.x; r < rows;
       r += (size_t)gridDim.x * blockDim.x)
    A.row_cnt[r] = 0;
  if (blockIdx.x != 0) return;
  __shared__ int s_bad;
  if (threadIdx.x == 0) s_bad = 0;
  __syncthreads();
  const int K = A.K;
  int nbad = 0;
  for (int b = threadIdx.x; b < A.B; b += blockDim.x) {
    A.seq_cnt[b] = 0;
    A.draw_cnt[b] = 0;
    const float T = __ldg(A.temperature + b);
    if (temp_valid(T)) {
      A.seq_done[b] = 0;
      continue;
    }
    ++nbad;
    A.accept_len[b] = -1;
    for (int j = 0; j <= K; ++j) A.out_tok[(size_t)b * (K + 1) + j] = -1;
    if (A.diag)
      for (int j = 0; j < 4 * K + 2; ++j) A.diag[(size_t)b * (4 * K + 2) + j] = dnan();
    SeqState s{};
    s.a = -1;
    if (A.commit) {
      s.old_len = A.cm.seq_lens[b];
      s.base = A.cm.base_len ? A.cm.base_len[b] : s.old_len;
      s.kept = 0;
      s.bad = 0;
    }
    A.seq[b] = s;
    A.seq_done[b] = 1;
  }
  if (nbad) atomicAdd(&s_bad, nbad);
  __syncthreads();
  if (threadIdx.x == 0) {
    StepCounters c{};
    c.ticket = s_bad;
    c.plan = (A.commit && s_bad == A.B) ? 2 : 0;
    *A.ctr = c;
    if (s_bad) set_status(A.status, SPEC_EDEVICE);
  }
}

// The warp whose chunk completed row `row` (of sequence b) combines the row;
// the one that completes the sequence's last needed row runs its check.
template <typename T, bool kCommit>
__device__ __noinline__ void complete_row(const StepArgs& A, int row, int b, int nc, int greedy,
                                          float chi) {
  const int lane = threadIdx.x & 31, K = A.K;
  fence_acq_rel();
  const RowFinal f = warp_combine_row(A.part + (size_t)row * A.NC, nc, greedy, chi);
  int sd = 0;
  if (lane == 0) {
    A.fin[row] = f;
    __threadfence();
    sd = atomicAdd(A.seq_cnt + b, 1) + 1;
  }
  sd = __shfl_sync(0xffffffffu, sd, 0);
  if (sd == K + 1 + (greedy ? 0 : K)) {
    __threadfence();
    accept_seq<T, kCommit>(A, b);
  }
}

// ---------------------------------------------------------------------------
// The step kernel
// ---------------------------------------------------------------------------
template <typename T, bool kCommit>
__global__ void __launch_bounds__(kRsWarps * 32, 1)
    chain_step_kernel(const __grid_constant__ StepArgs A) {
  extern __shared__ __align__(128) unsigned char smem[];
  constexpr int kVec = VecOf<T>::n;
  constexpr int kEpt = kTileBytes / (int)sizeof(T);  // elements per tile
  constexpr int kVpl = kTileBytes / 16 / 32;          // vectors per lane
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  unsigned char* wbuf = smem + (size_t)warp * kRsStages * kTileBytes;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + (size_t)kRsWarps * kRsStages * kTileBytes) +
                   warp * kRsStages;
  StepItem* fifo = reinterpret_cast<StepItem*>(smem + kRsSmem) + warp * kFifo;
  float* s_temp = reinterpret_cast<float*>(smem + kRsSmem + kRsWarps * kFifo * sizeof(StepItem));
  __shared__ PendRow s_pend[kRsWarps];
  __shared__ uint32_t s_phase[kRsWarps];
  if (lane == 0) {
    for (int s = 0; s < kRsStages; ++s) mbar_init(&bars[s], 1);
    fence_barrier_init();
  }
  pdl_begin();
  if (A.B <= kTempCache)
    for (int b = threadIdx.x; b < A.B; b += blockDim.x) s_temp[b] = __ldg(A.temperature + b);
  __syncthreads();
  StepCounters* ctr = A.ctr;
  const int K = A.K, V = A.V;

  // ---- Producer: resolves items into the fifo and issues tile copies ----
  unsigned ahead = 0;  // lane 0: the next grabbed item index
  if (lane == 0) ahead = atomicAdd(&ctr->stream, 1u);
  int nprod = 0;                 // items resolved so far
  int pt = 0, pt1 = 0;           // producer's next tile / end in its item
  const unsigned char* prow = nullptr;
  bool pearly = false, pdone = false;
  auto next_item = [&]() -> bool {
    for (;;) {
      const unsigned i = __shfl_sync(0xffffffffu, ahead, 0);
      if (i >= A.n_total) return false;
      if (lane == 0) ahead = atomicAdd(&ctr->stream, 1u);
      StepItem it;
      if (map_item(A, i, s_temp, &it)) {
        if (lane == 0) fifo[nprod % kFifo] = it;
        __syncwarp();
        ++nprod;
        prow = it.rowp;
        pt = it.t0;
        pt1 = it.t1;
        pearly = it.early;
        return true;
      }
    }
  };
  auto issue = [&](int st) -> bool {
    if (pt == pt1) {
      if (pdone || !next_item()) {
        pdone = true;
        return false;
      }
    }
    if (lane == 0) {
      const int nel = min(kEpt, V - pt * kEpt);
      const uint32_t bytes = ((uint32_t)nel * sizeof(T)) & ~15u;
      fence_proxy_async_smem();  // the warp's reads of this stage come first
      mbar_arrive_expect_tx(&bars[st], bytes);
      const unsigned char* src = prow + (size_t)pt * kTileBytes;
      if (bytes) {
        if (pearly && A.lp > 0)
          bulk_g2s_hint(wbuf + st * kTileBytes, src, bytes, &bars[st], l2_evict_first());
        else
          bulk_g2s(wbuf + st * kTileBytes, src, bytes, &bars[st]);
      }
    }
    ++pt;
    return true;
  };
  int inflight = 0;
  for (int st = 0; st < kRsStages; ++st) {
    if (!issue(st)) break;
    ++inflight;
  }

  // ---- Row completion, one chunk late: the warp checks a chunk's count
  // (an acq_rel atomic) only when its next chunk is done, so it never waits
  // for the atomic. The warp that completes a row combines it; the one that
  // completes a sequence's last row runs its check.
  PendRow* pend = s_pend + warp;  // written by lane 0, read by all after a __syncwarp
  if (lane == 0) pend->on = 0;
  __syncwarp();
  int pend_old = 0;  // lane 0
  auto settle = [&]() {
    if (!pend->on) return;
    const PendRow pr = *pend;
    __syncwarp();
    if (lane == 0) pend->on = 0;
    const int done = __shfl_sync(0xffffffffu, pend_old, 0) + 1;
    if (done == pr.nc) complete_row<T, kCommit>(A, pr.row, pr.b, pr.nc, pr.greedy, pr.chi);
  };

  // ---- Consumer ----
  int ncons = 0;
  int ct = 0, ct1 = 0;  // consumer's next tile / end in its item
  const StepItem* cip = fifo;  // the consumer's item (its fifo slot)
  uint32_t phase = 0;
  int s = 0;
  bool timed_out = false;
  float chi = 0.0f, clo = 0.0f;
  float mrun = -INFINITY, anchor = -INFINITY, Msh = 0.0f;
  double acc = 0.0;
  int gidx = 0x7fffffff;
  while (inflight > 0) {
    const bool first = (ct == ct1);
    if (first) {  // the next item's first tile
      cip = fifo + ncons % kFifo;
      ++ncons;
      ct = cip->t0;
      ct1 = cip->t1;
      chi = cip->chi;
      clo = cip->clo;
      mrun = anchor = -INFINITY;
      Msh = 0.0f;
      acc = 0.0;
      gidx = 0x7fffffff;
    }
    const bool ok = mbar_wait_bounded(&bars[s], (phase >> s) & 1u, kWaitLimitNs);
    if (__any_sync(0xffffffffu, !ok)) {
      timed_out = true;
      break;
    }
    phase ^= 1u << s;
    --inflight;
    const T* rptr = reinterpret_cast<const T*>(cip->rowp);
    const int nel = min(kEpt, V - ct * kEpt);
    const uint4* buf = reinterpret_cast<const uint4*>(wbuf + s * kTileBytes);
    uint4 x[kVpl];
    int nvec = kEpt / kVec, ntail = 0;
    float tailx = -INFINITY;
    if (nel == kEpt) {
#pragma unroll
      for (int i = 0; i < kVpl; ++i) x[i] = buf[lane + 32 * i];
    } else {
      nvec = (int)(((uint32_t)nel * sizeof(T)) >> 4);
      ntail = nel - nvec * kVec;
#pragma unroll
      for (int i = 0; i < kVpl; ++i) {
        const int v = lane + 32 * i;
        x[i] = v < nvec ? buf[v] : neg_inf_vec<T>();
      }
      if (lane < ntail) tailx = load_elem(rptr + (size_t)ct * kEpt + nvec * kVec + lane);
    }
    __syncwarp();
    if (issue(s)) ++inflight;

    const bool greedy_row = cip->greedy;
    if (greedy_row) {
      float tb = -INFINITY;
      int bv = -1;
#pragma unroll
      for (int i = 0; i < kVpl; ++i) {
        const float vm = vec_max(x[i], (T*)nullptr);
        if (vm > tb) { tb = vm; bv = i; }
      }
      if (tb > mrun) {
        uint4 w = x[0];
#pragma unroll
        for (int i = 1; i < kVpl; ++i)
          if (i == bv) w = x[i];
        int ef = 0;
#pragma unroll
        for (int e = kVec - 1; e >= 0; --e)
          if (vec_elem(w, e, (T*)nullptr) == tb) ef = e;
        mrun = tb;
        gidx = ct * kEpt + (lane + 32 * bv) * kVec + ef;
      }
      if (tailx > mrun) {
        mrun = tailx;
        gidx = ct * kEpt + nvec * kVec + lane;
      }
    } else {
      const float tm = fmaxf(regs_max<kVpl>(x, (T*)nullptr), tailx);
      if (tm > mrun) mrun = tm;
      // The lane's shift is an integer at or just above its largest scaled
      // element, moved (by an exact power of two) as soon as an element
      // passes it: the largest terms have exponents in (-1, 0], where fp32
      // rounds them least.
      const float Mn = ceilf(tm * chi);
      if (tm > -INFINITY && (!(anchor > -INFINITY) || Mn > Msh)) {
        if (acc != 0.0) acc *= pow2i(Msh - Mn);
        anchor = tm;
        Msh = Mn;
      }
      const bool has = anchor > -INFINITY;
      float a = 0.0f;
      if (__all_sync(0xffffffffu, !has || fabsf(Msh) < kFarShift)) {
        if (has) {
          const float2 chi2 = make_float2(chi, chi), clo2 = make_float2(clo, clo);
          const float2 nM2 = make_float2(-Msh, -Msh);
          float2 a0 = make_float2(0.0f, 0.0f), a1 = make_float2(0.0f, 0.0f);
#pragma unroll
          for (int i = 0; i < kVpl; i += 2) {
            a0 = __fadd2_rn(a0, vec_expsum(x[i], chi2, clo2, nM2, (T*)nullptr));
            if (i + 1 < kVpl)
              a1 = __fadd2_rn(a1, vec_expsum(x[i + 1], chi2, clo2, nM2, (T*)nullptr));
          }
          const float2 a2 = __fadd2_rn(a0, a1);
          a = a2.x + a2.y;
          if (lane < ntail) a += term(tailx, chi, clo, -Msh);
        }
      } else if (has) {
        const float rr = fmaf(anchor, chi, -Msh) + anchor * clo;
#pragma unroll
        for (int i = 0; i < kVpl; ++i) a += vec_expsum_far<T>(x[i], anchor, chi, clo, rr);
        if (lane < ntail) a += term_far(tailx, anchor, chi, clo, rr);
      }
      acc += (double)a;
    }
    ++ct;
    s = (s + 1 == kRsStages) ? 0 : s + 1;

    if (ct == ct1) {  // the chunk is done: one ChunkStat, then the row's count
      ChunkStat cs;
      if (greedy_row) {
        float v = mrun;
        int i = gidx;
        warp_argmax(v, i);
        cs.m = v;
        cs.aux = i;
        cs.s = 0.0;
      } else {
        float m = mrun;
        float Mu = (anchor > -INFINITY) ? Msh : -INFINITY;
#pragma unroll
        for (int o = 16; o; o >>= 1) {
          m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
          Mu = fmaxf(Mu, __shfl_xor_sync(0xffffffffu, Mu, o));
        }
        double sl = 0.0;
        if (acc != 0.0) sl = (Msh == Mu) ? acc : acc * pow2i(Msh - Mu);
        cs.m = m;
        cs.aux = __float_as_int(Mu > -INFINITY ? Mu : 0.0f);
        cs.s = warp_sum_d(sl);
      }
      // The previous chunk's count has had this whole chunk to come back.
      settle();
      const int cb = cip->b;
      const size_t row = (size_t)cb * (2 * K + 1) + cip->r;
      if (lane == 0) {
        A.part[row * A.NC + cip->c] = cs;
        pend_old = atom_add_release(A.row_cnt + row, 1);
        *pend = PendRow{(int)row, cb, cip->nc, (int)greedy_row, chi, 1};
      }
      __syncwarp();
    }
  }
  settle();
  if (timed_out) {
    step_abort(A);
    for (int j = 0; j < inflight; ++j) {
      const int q = (s + j) % kRsStages;
      mbar_wait_bounded(&bars[q], (phase >> q) & 1u, kWaitLimitNs);
    }
    return;
  }

  // ---- Draw parts (the warp's ring is idle now: no copy in flight) ----
  if (lane == 0) s_phase[warp] = phase;
  __syncwarp();
  const WarpRing ring{wbuf, bars, &s_phase[warp]};
  const unsigned n_draw = (unsigned)A.B * A.D;
  for (;;) {
    const unsigned i = warp_grab(&ctr->draw);
    if (i >= n_draw) break;
    draw_part<T>(A, (int)(i / A.D), (int)(i % A.D), ring);
  }

  // ---- Copies of the kept rows ----
  if constexpr (kCommit) {
    if (A.units_tok > 0 && warp_wait_flag(A, &ctr->plan) == 1) {
      const unsigned n_units = (unsigned)__ldcg(&ctr->kt) * A.units_tok;
      for (;;) {
        const unsigned u = warp_grab(&ctr->copy);
        if (u >= n_units) break;
        copy_unit(A, u);
      }
    }
  }
}

// ---------------------------------------------------------------------------
// Launcher
// ---------------------------------------------------------------------------
template <typename T, bool kCommit>
static cudaError_t launch_step_t(const StepArgs& a, cudaStream_t st) {
  const long long rows = (long long)a.B * (2 * a.K + 1);
  const unsigned pgrid = (unsigned)std::max(1LL, std::min((long long)sm_count(), (rows + 1023) / 1024));
  cudaError_t e = launch_pdl(step_prologue_kernel, dim3(pgrid), dim3(1024), 0, st, a);
  if (e != cudaSuccess) return e;
  auto kern = chain_step_kernel<T, kCommit>;
  e = reserve_dyn_smem(kern, (size_t)kStepSmem);
  if (e != cudaSuccess) return e;
  long long grid = sm_count();
  const long long need = ((long long)a.n_total + kRsWarps - 1) / kRsWarps;
  if (grid > need) grid = need;
  if (grid < 1) grid = 1;
  return launch_pdl(kern, dim3((unsigned)grid), dim3(kRsWarps * 32), (size_t)kStepSmem, st, a);
}

cudaError_t launch_chain_step(const StepArgs& a, cudaStream_t st) {
  if (a.dtype == SPEC_BF16)
    return a.commit ? launch_step_t<__nv_bfloat16, true>(a, st)
                    : launch_step_t<__nv_bfloat16, false>(a, st);
  return a.commit ? launch_step_t<float, true>(a, st) : launch_step_t<float, false>(a, st);
}

}  // namespace specv
