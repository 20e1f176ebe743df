// Decide kernels: per sequence, combine the row statistics, run the accept
// test on every draft position in parallel, find the first rejection, and
// draw the resampled / bonus token by inverse CDF over the residual
// max(0, p - q) (or p), re-reading only the two rows at the rejection.
//
// Rules: speculative sampling as appealed to by HiSpec (gist.science summary
// of arXiv 2510.01336, section 2, "Verlustfreie Garantie": accepted count plus
// bonus token per verification, Speculative Speculative Decoding summary,
// Technische Zusammenfassung 2.1; residual proportional to the target-minus-
// draft difference, same page 3.B). The window update follows HiSpec's
// "Dynamische Verifizierungsrichtlinie" (N_i tentatively accepted tokens
// before the final-layer check).
//
// Two launches per check. (1) finish: one CTA per sequence combines the tile
// partials of its rows (a warp per row), runs the accept test on all
// positions (a lane per position, ballot for the first rejection) and, for
// greedy sequences, writes the outputs. (2) draw: grid (nsplit, B); the
// residual row pair of each sampled sequence is split over nsplit CTAs, each
// writing tile sums of the weights; the last CTA to arrive (atomic counter,
// no waiting) prefixes the tile sums, finds the tile holding u' * Z, rescans
// that one tile and writes the outputs.
#include <climits>

#include "common.cuh"
#include "kernels.cuh"

namespace specv {

constexpr int kMaxRows = 2 * SPEC_MAX_K + 1;
constexpr int kWarps = kDecideThreads / 32;
constexpr int kUnroll = 8;  // residual tiles in flight per warp

int decide_split(int B, int V) {
  const int nrt = residual_tiles(V);
  int s = (4 * 148) / (B > 0 ? B : 1);  // one wave of about four CTAs per SM
  if (s > kMaxSplit) s = kMaxSplit;
  if (s > nrt) s = nrt;
  return s < 1 ? 1 : s;
}

// ---------------------------------------------------------------------------
// Residual weights of 8 consecutive elements
// ---------------------------------------------------------------------------
template <typename T>
__device__ __forceinline__ void load8(const T* row, int e0, int V, float x[8]);
template <>
__device__ __forceinline__ void load8<__nv_bfloat16>(const __nv_bfloat16* row, int e0, int V,
                                                     float x[8]) {
  if (e0 + 8 <= V) {
    const uint4 w = __ldg(reinterpret_cast<const uint4*>(row + e0));
    x[0] = bf_lo(w.x); x[1] = bf_hi(w.x); x[2] = bf_lo(w.y); x[3] = bf_hi(w.y);
    x[4] = bf_lo(w.z); x[5] = bf_hi(w.z); x[6] = bf_lo(w.w); x[7] = bf_hi(w.w);
  } else {
#pragma unroll
    for (int e = 0; e < 8; ++e) x[e] = (e0 + e < V) ? load_elem(row + e0 + e) : -INFINITY;
  }
}
template <>
__device__ __forceinline__ void load8<float>(const float* row, int e0, int V, float x[8]) {
  if (e0 + 8 <= V) {
    const float4 a = __ldg(reinterpret_cast<const float4*>(row + e0));
    const float4 b = __ldg(reinterpret_cast<const float4*>(row + e0 + 4));
    x[0] = a.x; x[1] = a.y; x[2] = a.z; x[3] = a.w;
    x[4] = b.x; x[5] = b.y; x[6] = b.z; x[7] = b.w;
  } else {
#pragma unroll
    for (int e = 0; e < 8; ++e) x[e] = (e0 + e < V) ? load_elem(row + e0 + e) : -INFINITY;
  }
}

// Probability of a logit x of a row with log2-partition Lt = M + L:
// 2^(x*c - Lt), c = chi + clo, Lt = Lhi + Llo; the product x*chi - Lhi is
// rounded once relative to the (small) result.
struct ProbCoef {
  float chi, clo, nLhi, nLlo;
};
__device__ __forceinline__ ProbCoef make_coef(double Lt, const Scale& s) {
  ProbCoef k;
  k.chi = s.hi;
  k.clo = s.lo;
  const float hi = (float)Lt;
  k.nLhi = -hi;
  k.nLlo = -(float)(Lt - (double)hi);
  return k;
}
__device__ __forceinline__ float2 prob2(float2 x, const ProbCoef& k) {
  float2 t = __ffma2_rn(x, make_float2(k.chi, k.chi), make_float2(k.nLhi, k.nLhi));
  t = __ffma2_rn(x, make_float2(k.clo, k.clo), t);
  t = __fadd2_rn(t, make_float2(k.nLlo, k.nLlo));
  return make_float2(ex2(t.x), ex2(t.y));
}

// Weights w = max(0, p - q) (or p when there is no draft row) of 8 elements.
template <typename T>
__device__ __forceinline__ void weights8(const T* prow, const T* qrow, int e0, int V,
                                         const ProbCoef& kp, const ProbCoef& kq, float w[8]) {
  float xp[8];
  load8<T>(prow, e0, V, xp);
  if (qrow) {
    float xq[8];
    load8<T>(qrow, e0, V, xq);
#pragma unroll
    for (int e = 0; e < 8; e += 2) {
      const float2 p = prob2(make_float2(xp[e], xp[e + 1]), kp);
      const float2 q = prob2(make_float2(xq[e], xq[e + 1]), kq);
      w[e] = fmaxf(p.x - q.x, 0.0f);
      w[e + 1] = fmaxf(p.y - q.y, 0.0f);
    }
  } else {
#pragma unroll
    for (int e = 0; e < 8; e += 2) {
      const float2 p = prob2(make_float2(xp[e], xp[e + 1]), kp);
      w[e] = p.x;
      w[e + 1] = p.y;
    }
  }
}
// A lane's 8 weights summed pairwise in fp32 (error ~ 3 ulp of the small
// sum), then widened; tiles and lanes combine in fp64.
__device__ __forceinline__ double lane_sum8(const float w[8]) {
  const float2 a = __fadd2_rn(make_float2(w[0], w[1]), make_float2(w[2], w[3]));
  const float2 b = __fadd2_rn(make_float2(w[4], w[5]), make_float2(w[6], w[7]));
  const float2 c = __fadd2_rn(a, b);
  return (double)(c.x + c.y);
}

// Tile sums of the weights over residual tiles [t0, t1) (one CTA's share).
template <typename T>
__device__ void residual_tile_sums(const T* prow, const T* qrow, int V, const ProbCoef& kp,
                                   const ProbCoef& kq, int t0, int t1, double* out) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  for (int tb = t0 + warp * kUnroll; tb < t1; tb += kWarps * kUnroll) {
    double s[kUnroll];
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
      const int t = tb + u;
      float w[8];
      if (t < t1) {
        weights8<T>(prow, qrow, t * kResTile + lane * 8, V, kp, kq, w);
        s[u] = lane_sum8(w);
      } else {
        s[u] = 0.0;
      }
    }
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
      const double v = warp_sum_d(s[u]);
      if (lane == 0 && tb + u < t1) out[tb + u] = v;
    }
  }
  if (lane == 0) __threadfence();  // the writers publish their tile sums
}

// Last CTA: prefix the tile sums, locate u' * Z, rescan that tile.
// Returns, in every thread, the drawn token (-1 if the weights have no mass);
// *Z_out gets Z.
template <typename T>
__device__ int residual_pick(const T* prow, const T* qrow, int V, const ProbCoef& kp,
                             const ProbCoef& kq, const double* tsum_g, int nrt, float u,
                             double* sh_pre, double* Z_out) {
  __shared__ double s_Z;
  __shared__ int s_tile, s_tok;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  double* sh_sum = sh_pre + nrt;  // second half of the dynamic buffer
  for (int t = threadIdx.x; t < nrt; t += blockDim.x) sh_sum[t] = __ldcg(tsum_g + t);
  __syncthreads();
  // Exclusive prefix over tiles in a fixed order (warp 0: each lane owns a
  // contiguous run of tiles).
  if (warp == 0) {
    const int per = (nrt + 31) / 32;
    const int a = min(nrt, lane * per), b = min(nrt, a + per);
    double run = 0.0;
    for (int t = a; t < b; ++t) run += sh_sum[t];
    double incl = run;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const double y = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += y;
    }
    double c = __shfl_up_sync(0xffffffffu, incl, 1);
    if (lane == 0) c = 0.0;
    for (int t = a; t < b; ++t) {
      sh_pre[t] = c;
      c += sh_sum[t];
    }
    if (lane == 31) s_Z = incl;
    if (lane == 0) s_tile = -1;
  }
  __syncthreads();
  const double Z = s_Z;
  *Z_out = Z;
  if (!(Z > 0.0)) return -1;
  const double target = (double)u * Z;
  // The last tile with mass whose prefix does not exceed the target.
  for (int t = threadIdx.x; t < nrt; t += blockDim.x)
    if (sh_pre[t] <= target && sh_sum[t] > 0.0) atomicMax(&s_tile, t);
  __syncthreads();
  const int tile = s_tile < 0 ? 0 : s_tile;  // s_tile >= 0 whenever Z > 0
  if (warp == 0) {
    float w[8];
    weights8<T>(prow, qrow, tile * kResTile + lane * 8, V, kp, kq, w);
    const double ls = lane_sum8(w);
    double incl = ls;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const double y = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += y;
    }
    double excl = __shfl_up_sync(0xffffffffu, incl, 1);
    if (lane == 0) excl = 0.0;
    const double start = sh_pre[tile] + excl;
    int found = INT_MAX;
    if (start <= target) {
      double acc = start;
      for (int e = 0; e < 8; ++e) {
        acc += (double)w[e];
        if (acc > target && w[e] > 0.0f) { found = tile * kResTile + lane * 8 + e; break; }
      }
    }
#pragma unroll
    for (int o = 16; o; o >>= 1) found = min(found, __shfl_xor_sync(0xffffffffu, found, o));
    if (found == INT_MAX) {
      // The target sits at this tile's end by rounding: last element with mass.
      int last = -1;
      for (int e = 7; e >= 0; --e)
        if (w[e] > 0.0f) { last = tile * kResTile + lane * 8 + e; break; }
#pragma unroll
      for (int o = 16; o; o >>= 1) last = max(last, __shfl_xor_sync(0xffffffffu, last, o));
      found = last;
    }
    if (lane == 0) s_tok = found;
  }
  __syncthreads();
  return s_tok;
}

// Residual / bonus draw of one sequence, split over the sequence's CTAs.
// Every CTA writes the tile sums of its share; the last to arrive picks the
// token. Returns false in the CTAs that are not last (they are done).
template <typename T>
__device__ bool draw_token(const DecideCommon& c, int b, int sp, const T* prow, const T* qrow,
                           const ProbCoef& kp, const ProbCoef& kq, float u, double* sh_pre,
                           int* tok_out, double* Z_out) {
  __shared__ int s_last;
  const int nrt = residual_tiles(c.V);
  const int chunk = (nrt + c.nsplit - 1) / c.nsplit;
  double* tsum = c.rsum + (size_t)b * nrt;
  residual_tile_sums<T>(prow, qrow, c.V, kp, kq, min(nrt, sp * chunk), min(nrt, (sp + 1) * chunk),
                        tsum);
  __syncthreads();
  if (threadIdx.x == 0) s_last = (atomicAdd(&c.counters[b], 1) == c.nsplit - 1);
  __syncthreads();
  if (!s_last) return false;
  __threadfence();
  int tok = residual_pick<T>(prow, qrow, c.V, kp, kq, tsum, nrt, u, sh_pre, Z_out);
  if (tok < 0 && qrow) {
    // Residual mass zero as computed (p == q): draw from p instead.
    __syncthreads();
    residual_tile_sums<T>(prow, nullptr, c.V, kp, kq, 0, nrt, tsum);
    __syncthreads();
    tok = residual_pick<T>(prow, nullptr, c.V, kp, kq, tsum, nrt, u, sh_pre, Z_out);
  }
  __syncthreads();
  if (threadIdx.x == 0) c.counters[b] = 0;
  *tok_out = tok;
  return true;
}

// ---------------------------------------------------------------------------
// Per-sequence state of the finish kernels
// ---------------------------------------------------------------------------
constexpr int kFinThreads = 1024;
constexpr int kFinWarps = kFinThreads / 32;
constexpr long long kNaNBits = 0x7ff8000000000000ll;
__device__ __forceinline__ double dnan() { return __longlong_as_double(kNaNBits); }

struct SeqShared {
  double M[kMaxRows], L[kMaxRows];
  float m[kMaxRows];
  int amax[kMaxRows];
  int ok[kMaxRows];
  int a, bad;
};

// Combine the tile partials of the rows of one sequence (a warp per row) into
// shared memory and into the RowFinal array (read later by the draw kernel).
template <typename Want>
__device__ void finish_rows(SeqShared& sh, const Partial* part, int ntiles, int row0, int nrows,
                            Want want, bool greedy, float chi, RowFinal* fin) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (warp == kFinWarps - 1) return;  // the accept warp
  for (int r = warp; r < nrows; r += kFinWarps - 1) {
    if (!want(r)) {
      if (lane == 0) { sh.ok[r] = 1; sh.m[r] = 0.f; sh.M[r] = 0; sh.L[r] = 0; sh.amax[r] = -1; }
      continue;
    }
    const RowFinal f = combine_row(part + (size_t)(row0 + r) * ntiles, ntiles, greedy, chi, lane);
    if (lane == 0) {
      fin[row0 + r] = f;
      sh.m[r] = f.m;
      sh.M[r] = f.M;
      sh.L[r] = f.L;
      sh.amax[r] = f.amax;
      sh.ok[r] = f.ok;
    }
  }
}

template <typename T>
__device__ __forceinline__ const T* row_ptr(const unsigned char* base, long long ld_bytes,
                                            long long row) {
  return reinterpret_cast<const T*>(base + row * ld_bytes);
}

// Logits of the drafted tokens for the first 32 positions, fetched by the
// accept warp while the other warps combine the rows.
struct AcceptPre {
  int x;        // draft id of position lane (or -1 past n)
  float lt, ld; // target / draft logit at x
};
template <typename T, typename TP, typename DP>
__device__ __forceinline__ AcceptPre accept_prefetch(int n, int V, bool greedy,
                                                     const int32_t* drafts, TP tp, DP dp) {
  const int lane = threadIdx.x & 31;
  AcceptPre a{-1, 0.f, 0.f};
  if (lane < n) {
    a.x = drafts[lane];
    if (!greedy && a.x >= 0 && a.x < V) {
      a.lt = load_elem(tp(lane) + a.x);
      a.ld = load_elem(dp(lane) + a.x);
    }
  }
  return a;
}

// One speculative check on n positions (one warp). Target row j: tp(j) with
// log2 partition sh.M + sh.L at index j; draft law of position j: row dp(j)
// with log2 partition dlt(j). Sets sh.a (first rejection, n if none) and
// sh.bad (a draft id outside [0, V)). Writes p_j(x_j), q_j(x_j) to diag_p /
// diag_q. Positions below 32 use the prefetched logits.
template <typename T, typename TP, typename DP, typename DS>
__device__ void accept_scan(SeqShared& sh, int n, int pos0, int stage, const DecideCommon& c,
                            int b, bool greedy, double cd, const int32_t* drafts, TP tp, DP dp,
                            DS dlt, double* diag_p, double* diag_q, const AcceptPre& pre) {
  const int lane = threadIdx.x & 31;
  int a = n, bad = 0;
  for (int j0 = 0; j0 < n; j0 += 32) {
    const int j = j0 + lane;
    bool acc = true, badj = false;
    if (j < n) {
      const int x = j0 == 0 ? pre.x : drafts[j];
      if (x < 0 || x >= c.V) {
        badj = true;
      } else if (greedy) {
        acc = (x == sh.amax[j]);
      } else {
        const float lt = j0 == 0 ? pre.lt : load_elem(tp(j) + x);
        const float ld = j0 == 0 ? pre.ld : load_elem(dp(j) + x);
        const double lp = (double)lt * cd - (sh.M[j] + sh.L[j]);
        const double lq = (double)ld * cd - dlt(j);
        const float u = spec_uniforms(c.seed, (uint32_t)c.seq_id[b], c.round, (uint32_t)(pos0 + j),
                                      (uint32_t)stage).x;
        acc = (double)u < exp2(lp - lq);
        if (diag_p) { diag_p[j] = exp2(lp); diag_q[j] = exp2(lq); }
      }
    }
    if (__any_sync(0xffffffffu, badj)) bad = 1;
    const unsigned rej = __ballot_sync(0xffffffffu, j < n && !acc);
    if (rej && a == n) a = j0 + __ffs(rej) - 1;
  }
  if (lane == 0) { sh.a = a; sh.bad = bad; }
}

__device__ __forceinline__ bool rows_ok(const SeqShared& sh, int nrows) {
  int bad = 0;
  for (int r = 0; r < nrows; ++r) bad |= !sh.ok[r];
  return !bad;
}

// ---------------------------------------------------------------------------
// Chain verification
// ---------------------------------------------------------------------------
template <typename T>
__global__ void __launch_bounds__(kFinThreads) chain_finish_kernel(ChainDecideArgs A) {
  grid_dependency_wait();
  __shared__ SeqShared sh;
  const DecideCommon& c = A.c;
  const int b = blockIdx.x, K = c.K, per = 2 * K + 1;
  const float Tb = c.temperature[b];
  const bool tvalid = temp_valid(Tb), greedy = (Tb == 0.0f);
  double* diag = c.diag ? c.diag + (size_t)b * (4 * K + 2) : nullptr;
  auto fail = [&]() {
    if (threadIdx.x == 0) {
      set_status(c.status, SPEC_EDEVICE);
      A.accept_len[b] = -1;
      c.dec[b] = SeqDecision{-1, 2};
    }
    for (int j = threadIdx.x; j <= K; j += blockDim.x) A.out_tok[(size_t)b * (K + 1) + j] = -1;
    if (diag)
      for (int j = threadIdx.x; j < 4 * K + 2; j += blockDim.x) diag[j] = dnan();
  };
  if (!tvalid) { fail(); grid_dependents_launch(); return; }
  const Scale sc = greedy ? Scale{0.f, 0.f, 0.0} : make_scale(Tb);
  const int32_t* drafts = c.draft_tok + (size_t)b * K;
  auto tp = [&](int j) { return row_ptr<T>(A.tgt, A.ld_tgt, (long long)b * (K + 1) + j); };
  auto dp = [&](int j) { return row_ptr<T>(A.drf, A.ld_drf, (long long)b * K + j); };
  auto dl = [&](int j) { return sh.M[K + 1 + j] + sh.L[K + 1 + j]; };
  const bool accept_warp = (threadIdx.x >> 5) == kFinWarps - 1;
  AcceptPre pre{-1, 0.f, 0.f};
  if (accept_warp) pre = accept_prefetch<T>(K, c.V, greedy, drafts, tp, dp);
  finish_rows(sh, c.part, c.ntiles, b * per, per, [&](int r) { return r <= K || !greedy; }, greedy,
              sc.hi, c.fin);
  __syncthreads();
  if (accept_warp)
    accept_scan<T>(sh, K, 0, 1, c, b, greedy, sc.d, drafts, tp, dp, dl,
                   diag && !greedy ? diag + 2 * K + 1 : nullptr,
                   diag && !greedy ? diag + 3 * K + 1 : nullptr, pre);
  __syncthreads();
  if (sh.bad || !rows_ok(sh, per)) { fail(); grid_dependents_launch(); return; }
  const int a = sh.a;
  if (greedy) {
    for (int j = threadIdx.x; j <= K; j += blockDim.x)
      A.out_tok[(size_t)b * (K + 1) + j] = j < a ? drafts[j] : (j == a ? sh.amax[a] : -1);
    if (threadIdx.x == 0) { A.accept_len[b] = a; c.dec[b] = SeqDecision{a, 1}; }
    if (diag)
      for (int j = threadIdx.x; j < 4 * K + 2; j += blockDim.x) diag[j] = dnan();
  } else {
    if (threadIdx.x == 0) c.dec[b] = SeqDecision{a, 0};
    if (diag)
      for (int j = threadIdx.x; j < per; j += blockDim.x) diag[j] = (sh.M[j] + sh.L[j]) * kLn2;
  }
  grid_dependents_launch();
}

template <typename T>
__global__ void __launch_bounds__(kDecideThreads, 4) chain_draw_kernel(ChainDecideArgs A) {
  grid_dependency_wait();
  extern __shared__ double dyn_pre[];
  const DecideCommon& c = A.c;
  const int b = blockIdx.y, sp = blockIdx.x, K = c.K, per = 2 * K + 1;
  const SeqDecision d = c.dec[b];
  if (d.state != 0) return;
  const int a = d.a;
  const Scale sc = make_scale(c.temperature[b]);
  const RowFinal fp = c.fin[b * per + a];
  const T* prow = row_ptr<T>(A.tgt, A.ld_tgt, (long long)b * (K + 1) + a);
  const T* qrow = a < K ? row_ptr<T>(A.drf, A.ld_drf, (long long)b * K + a) : nullptr;
  double lq = 0.0;
  if (a < K) {
    const RowFinal fq = c.fin[b * per + K + 1 + a];
    lq = fq.M + fq.L;
  }
  const ProbCoef kp = make_coef(fp.M + fp.L, sc), kq = make_coef(lq, sc);
  const float u = spec_uniforms(c.seed, (uint32_t)c.seq_id[b], c.round, (uint32_t)a, 1u).y;
  int tok;
  double Z;
  if (!draw_token<T>(c, b, sp, prow, qrow, kp, kq, u, dyn_pre, &tok, &Z)) return;
  const int32_t* drafts = c.draft_tok + (size_t)b * K;
  for (int j = threadIdx.x; j <= K; j += blockDim.x)
    A.out_tok[(size_t)b * (K + 1) + j] = j < a ? drafts[j] : (j == a ? tok : -1);
  if (threadIdx.x == 0) {
    A.accept_len[b] = a;
    if (c.diag) c.diag[(size_t)b * (4 * K + 2) + 4 * K + 1] = Z;
  }
}

// ---------------------------------------------------------------------------
// Two-stage verification
// ---------------------------------------------------------------------------
// Stage one: drafts (slots w..w+K-1) against L_i (slots w..w+K), draft law
// L_d; the a1 accepted drafts and the drawn token join the window with the
// L_i statistics of their slots.
__device__ __forceinline__ void window_append(const HierDecideArgs& A, int b, int w, int a,
                                              const int32_t* drafts, int tok, const RowFinal* rf,
                                              bool greedy, double cd) {
  const int WC = A.Ni + A.c.K;
  for (int j = threadIdx.x; j <= a; j += blockDim.x) {
    const size_t slot = (size_t)b * WC + w + j;
    A.win_tok[slot] = j < a ? drafts[j] : tok;
    if (greedy) {
      A.win_stat[2 * slot] = dnan();
      A.win_stat[2 * slot + 1] = dnan();
    } else {
      const RowFinal f = rf[j];
      A.win_stat[2 * slot] = f.m;
      A.win_stat[2 * slot + 1] = (f.M + f.L - (double)f.m * cd) * kLn2;
    }
  }
}

template <typename T>
__global__ void __launch_bounds__(kFinThreads) hier1_finish_kernel(HierDecideArgs A) {
  grid_dependency_wait();
  __shared__ SeqShared sh;
  const DecideCommon& c = A.c;
  const int b = blockIdx.x, K = c.K, S = A.S, Ni = A.Ni, WC = Ni + K, per = 2 * K + 1;
  const int D = 4 * K + 3 * S + 1;
  double* diag = c.diag ? c.diag + (size_t)b * D : nullptr;
  // Stage-two outputs default to "did not run"; stage two overwrites them.
  for (int j = threadIdx.x; j < WC + 1; j += blockDim.x) A.commit_tok[(size_t)b * (WC + 1) + j] = -1;
  if (threadIdx.x == 0) { A.commit_n[b] = 0; A.acc2[b] = -1; }
  if (diag)
    for (int j = threadIdx.x; j < D; j += blockDim.x) diag[j] = dnan();
  const float Tb = c.temperature[b];
  const bool tvalid = temp_valid(Tb), greedy = (Tb == 0.0f);
  const int w = A.win_len[b];
  auto fail = [&]() {
    if (threadIdx.x == 0) {
      set_status(c.status, SPEC_EDEVICE);
      A.acc1[b] = -1;
      c.dec[b] = SeqDecision{-1, 2};
    }
  };
  if (!tvalid || w < 0 || w >= Ni) { fail(); grid_dependents_launch(); return; }
  const Scale sc = greedy ? Scale{0.f, 0.f, 0.0} : make_scale(Tb);
  const int32_t* drafts = c.draft_tok + (size_t)b * K;
  const long long row0 = (long long)b * S + w;
  auto tp = [&](int j) { return row_ptr<T>(A.lg_i, A.ld, row0 + j); };
  auto dp = [&](int j) { return row_ptr<T>(A.lg_d, A.ld, row0 + j); };
  auto dl = [&](int j) { return sh.M[K + 1 + j] + sh.L[K + 1 + j]; };
  const bool accept_warp = (threadIdx.x >> 5) == kFinWarps - 1;
  AcceptPre pre{-1, 0.f, 0.f};
  if (accept_warp) pre = accept_prefetch<T>(K, c.V, greedy, drafts, tp, dp);
  finish_rows(sh, c.part, c.ntiles, b * per, per, [&](int r) { return r <= K || !greedy; }, greedy,
              sc.hi, c.fin);
  __syncthreads();
  if (accept_warp)
    accept_scan<T>(sh, K, w, 1, c, b, greedy, sc.d, drafts, tp, dp, dl,
                   diag && !greedy ? diag + 2 * K + 1 : nullptr,
                   diag && !greedy ? diag + 3 * K + 1 : nullptr, pre);
  __syncthreads();
  if (sh.bad || !rows_ok(sh, per)) { fail(); grid_dependents_launch(); return; }
  const int a = sh.a;
  if (greedy) {
    window_append(A, b, w, a, drafts, sh.amax[a], nullptr, true, 0.0);
    __syncthreads();
    if (threadIdx.x == 0) {
      A.win_len[b] = w + a + 1;
      A.acc1[b] = a;
      c.dec[b] = SeqDecision{a, 1};
    }
  } else {
    if (threadIdx.x == 0) c.dec[b] = SeqDecision{a, 0};
    if (diag)
      for (int j = threadIdx.x; j < per; j += blockDim.x) diag[j] = (sh.M[j] + sh.L[j]) * kLn2;
  }
  grid_dependents_launch();
}

template <typename T>
__global__ void __launch_bounds__(kDecideThreads, 4) hier1_draw_kernel(HierDecideArgs A) {
  grid_dependency_wait();
  extern __shared__ double dyn_pre[];
  const DecideCommon& c = A.c;
  const int b = blockIdx.y, sp = blockIdx.x, K = c.K, S = A.S, per = 2 * K + 1;
  const SeqDecision d = c.dec[b];
  if (d.state != 0) return;
  const int a = d.a;
  const int w = A.win_len[b];
  const Scale sc = make_scale(c.temperature[b]);
  const long long row0 = (long long)b * S + w;
  const RowFinal fp = c.fin[b * per + a];
  const T* prow = row_ptr<T>(A.lg_i, A.ld, row0 + a);
  const T* qrow = a < K ? row_ptr<T>(A.lg_d, A.ld, row0 + a) : nullptr;
  double lq = 0.0;
  if (a < K) {
    const RowFinal fq = c.fin[b * per + K + 1 + a];
    lq = fq.M + fq.L;
  }
  const ProbCoef kp = make_coef(fp.M + fp.L, sc), kq = make_coef(lq, sc);
  const float u = spec_uniforms(c.seed, (uint32_t)c.seq_id[b], c.round, (uint32_t)(w + a), 1u).y;
  int tok;
  double Z;
  if (!draw_token<T>(c, b, sp, prow, qrow, kp, kq, u, dyn_pre, &tok, &Z)) return;
  window_append(A, b, w, a, c.draft_tok + (size_t)b * K, tok, c.fin + (size_t)b * per, false, sc.d);
  __syncthreads();
  if (threadIdx.x == 0) {
    A.win_len[b] = w + a + 1;
    A.acc1[b] = a;
    if (c.diag) c.diag[(size_t)b * (4 * K + 3 * S + 1) + 4 * K + 1] = Z;
  }
}

// Stage two: for sequences whose window holds W >= Ni tokens, the window
// tokens (slots 0..W-1) against L_f (slots 0..W), draft law L_i from the
// buffered statistics; commits a2 + 1 tokens and empties the window.
template <typename T>
__global__ void __launch_bounds__(kFinThreads) hier2_finish_kernel(HierDecideArgs A) {
  grid_dependency_wait();
  __shared__ SeqShared sh;
  const DecideCommon& c = A.c;
  const int b = blockIdx.x, K = c.K, S = A.S, Ni = A.Ni, WC = Ni + K;
  const int W = A.win_len[b];
  if (A.acc1[b] < 0 || !(W >= Ni && W < S)) {
    if (threadIdx.x == 0) c.dec[b] = SeqDecision{-1, 1};  // no second stage
    grid_dependents_launch();
    return;
  }
  const float Tb = c.temperature[b];  // validated by stage one
  const bool greedy = (Tb == 0.0f);
  const Scale sc = greedy ? Scale{0.f, 0.f, 0.0} : make_scale(Tb);
  double* diag = c.diag ? c.diag + (size_t)b * (4 * K + 3 * S + 1) + (4 * K + 2) : nullptr;
  const int32_t* wtok = A.win_tok + (size_t)b * WC;
  const double* wst = A.win_stat + (size_t)b * WC * 2;
  auto tp = [&](int j) { return row_ptr<T>(A.lg_f, A.ld, (long long)b * S + j); };
  auto dp = [&](int j) { return row_ptr<T>(A.lg_i, A.ld, (long long)b * S + j); };
  auto dl = [&](int j) { return wst[2 * j] * sc.d + wst[2 * j + 1] * kLog2e; };
  const bool accept_warp = (threadIdx.x >> 5) == kFinWarps - 1;
  AcceptPre pre{-1, 0.f, 0.f};
  if (accept_warp) pre = accept_prefetch<T>(W, c.V, greedy, wtok, tp, dp);
  finish_rows(sh, c.part, c.ntiles, b * S, W + 1, [&](int) { return true; }, greedy, sc.hi, c.fin);
  __syncthreads();
  if (accept_warp)
    accept_scan<T>(sh, W, 0, 2, c, b, greedy, sc.d, wtok, tp, dp, dl,
                   diag && !greedy ? diag + S : nullptr, diag && !greedy ? diag + 2 * S - 1 : nullptr,
                   pre);
  __syncthreads();
  if (sh.bad || !rows_ok(sh, W + 1)) {
    if (threadIdx.x == 0) {
      set_status(c.status, SPEC_EDEVICE);
      A.acc2[b] = -1;
      c.dec[b] = SeqDecision{-1, 2};
    }
    grid_dependents_launch();
    return;
  }
  const int a = sh.a;
  if (greedy) {
    for (int j = threadIdx.x; j < WC + 1; j += blockDim.x)
      A.commit_tok[(size_t)b * (WC + 1) + j] = j < a ? wtok[j] : (j == a ? sh.amax[a] : -1);
    __syncthreads();
    if (threadIdx.x == 0) {
      A.commit_n[b] = a + 1;
      A.acc2[b] = a;
      A.win_len[b] = 0;
      c.dec[b] = SeqDecision{a, 1};
    }
  } else {
    if (threadIdx.x == 0) c.dec[b] = SeqDecision{a, 0};
    if (diag)
      for (int j = threadIdx.x; j <= W; j += blockDim.x) diag[j] = (sh.M[j] + sh.L[j]) * kLn2;
  }
  grid_dependents_launch();
}

template <typename T>
__global__ void __launch_bounds__(kDecideThreads, 4) hier2_draw_kernel(HierDecideArgs A) {
  grid_dependency_wait();
  extern __shared__ double dyn_pre[];
  const DecideCommon& c = A.c;
  const int b = blockIdx.y, sp = blockIdx.x, K = c.K, S = A.S, Ni = A.Ni, WC = Ni + K;
  const SeqDecision d = c.dec[b];
  if (d.state != 0) return;
  const int a = d.a;
  const int W = A.win_len[b];
  const Scale sc = make_scale(c.temperature[b]);
  const RowFinal fp = c.fin[b * S + a];
  const double* wst = A.win_stat + (size_t)b * WC * 2;
  const T* prow = row_ptr<T>(A.lg_f, A.ld, (long long)b * S + a);
  const T* qrow = a < W ? row_ptr<T>(A.lg_i, A.ld, (long long)b * S + a) : nullptr;
  const double lq = a < W ? wst[2 * a] * sc.d + wst[2 * a + 1] * kLog2e : 0.0;
  const ProbCoef kp = make_coef(fp.M + fp.L, sc), kq = make_coef(lq, sc);
  const float u = spec_uniforms(c.seed, (uint32_t)c.seq_id[b], c.round, (uint32_t)a, 2u).y;
  int tok;
  double Z;
  if (!draw_token<T>(c, b, sp, prow, qrow, kp, kq, u, dyn_pre, &tok, &Z)) return;
  const int32_t* wtok = A.win_tok + (size_t)b * WC;
  for (int j = threadIdx.x; j < WC + 1; j += blockDim.x)
    A.commit_tok[(size_t)b * (WC + 1) + j] = j < a ? wtok[j] : (j == a ? tok : -1);
  __syncthreads();
  if (threadIdx.x == 0) {
    A.commit_n[b] = a + 1;
    A.acc2[b] = a;
    A.win_len[b] = 0;
    if (c.diag) c.diag[(size_t)b * (4 * K + 3 * S + 1) + (4 * K + 2) + 3 * S - 2] = Z;
  }
}

// ---------------------------------------------------------------------------
// Launchers
// ---------------------------------------------------------------------------
template <typename Kern, typename Args>
static cudaError_t launch_draw(Kern k, const Args& a, cudaStream_t st) {
  const size_t smem = 2 * (size_t)residual_tiles(a.c.V) * sizeof(double);
  if (smem > 48 * 1024 &&
      cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) !=
          cudaSuccess)
    return cudaGetLastError();
  return launch_pdl(k, dim3(a.c.nsplit, a.c.B), dim3(kDecideThreads), smem, st, a);
}
template <typename Fin, typename Draw, typename Args>
static cudaError_t launch_pair(Fin f, Draw d, const Args& a, cudaStream_t st) {
  cudaError_t e = launch_pdl(f, dim3(a.c.B), dim3(kFinThreads), 0, st, a);
  if (e != cudaSuccess) return e;
  return launch_draw(d, a, st);
}

cudaError_t launch_chain_decide(const ChainDecideArgs& a, cudaStream_t st) {
  return a.c.dtype == SPEC_BF16
             ? launch_pair(chain_finish_kernel<__nv_bfloat16>, chain_draw_kernel<__nv_bfloat16>, a, st)
             : launch_pair(chain_finish_kernel<float>, chain_draw_kernel<float>, a, st);
}
cudaError_t launch_hier1_decide(const HierDecideArgs& a, cudaStream_t st) {
  return a.c.dtype == SPEC_BF16
             ? launch_pair(hier1_finish_kernel<__nv_bfloat16>, hier1_draw_kernel<__nv_bfloat16>, a, st)
             : launch_pair(hier1_finish_kernel<float>, hier1_draw_kernel<float>, a, st);
}
cudaError_t launch_hier2_decide(const HierDecideArgs& a, cudaStream_t st) {
  return a.c.dtype == SPEC_BF16
             ? launch_pair(hier2_finish_kernel<__nv_bfloat16>, hier2_draw_kernel<__nv_bfloat16>, a, st)
             : launch_pair(hier2_finish_kernel<float>, hier2_draw_kernel<float>, a, st);
}

}  // namespace specv
