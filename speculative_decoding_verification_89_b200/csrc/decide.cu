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
// Launch: grid (nsplit, B), 256 threads. Every CTA of a sequence repeats the
// cheap combine + accept step; the residual row pair is split over the
// nsplit CTAs, each writing tile sums of the weights; the last CTA to arrive
// (atomic counter, no waiting) prefixes the tile sums, finds the tile holding
// u' * Z, rescans that one tile and writes the outputs.
#include <climits>

#include "common.cuh"
#include "kernels.cuh"

namespace specv {

constexpr int kMaxRows = 2 * SPEC_MAX_K + 1;
constexpr int kWarps = kDecideThreads / 32;
constexpr int kUnroll = 4;  // residual tiles in flight per warp

int decide_split(int B, int V) {
  const int nrt = residual_tiles(V);
  int s = (4 * 148 + B - 1) / B;  // about four CTAs per SM over the whole grid
  if (s > kMaxSplit) s = kMaxSplit;
  if (s > nrt) s = nrt;
  return s < 1 ? 1 : s;
}

// Statistics of one row: raw max m, the exact shift M = fl(m * c_hi) and
// L = log2 sum_v 2^(l_v*c - M), so log2 p(v) = l_v*c - (M + L); first argmax.
struct RowStat {
  double m, M, L;
  int amax;
  bool ok;
};

// Warp-cooperative combine of a row's tile partials.
__device__ RowStat combine_row(const Partial* p, int ntiles, bool greedy, const Scale& sc,
                               int lane) {
  float mv = -INFINITY;
  int mi = INT_MAX;
  for (int t = lane; t < ntiles; t += 32) {
    const Partial q = p[t];
    if (q.m > mv || (q.m == mv && q.idx < mi)) { mv = q.m; mi = q.idx; }
  }
  warp_argmax(mv, mi);
  RowStat r;
  r.m = mv;
  r.amax = mi;
  r.M = 0.0;
  r.L = 0.0;
  r.ok = (mv > -INFINITY && mv < INFINITY);
  if (r.ok && !greedy) {
    r.M = (double)__fmul_rn(mv, sc.hi);
    double s = 0.0;
    for (int t = lane; t < ntiles; t += 32) {
      const Partial q = p[t];
      if (q.s != 0.0) s += q.s * exp2((double)__fmul_rn(q.m, sc.hi) - r.M);
    }
    s = warp_sum_d(s);
    r.ok = (s > 0.0 && s < INFINITY);
    r.L = log2(s);
  }
  return r;
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
  __threadfence();
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
    __threadfence();
    __syncthreads();
    tok = residual_pick<T>(prow, nullptr, c.V, kp, kq, tsum, nrt, u, sh_pre, Z_out);
  }
  __syncthreads();
  if (threadIdx.x == 0) c.counters[b] = 0;
  *tok_out = tok;
  return true;
}

// ---------------------------------------------------------------------------
// Shared per-sequence state
// ---------------------------------------------------------------------------
struct SeqShared {
  double m[kMaxRows], M[kMaxRows], L[kMaxRows];
  int amax[kMaxRows];
  int ok[kMaxRows];
  int a, bad, last, tok;
  double Z;
};

// Combine all rows of a sequence into shared memory (warp per row).
__device__ void combine_rows(SeqShared& sh, const Partial* part, int row0, int nrows_seq,
                             int ntiles, const bool* want, bool greedy, const Scale& sc) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  for (int r = warp; r < nrows_seq; r += kWarps) {
    if (!want[r]) {
      if (lane == 0) { sh.ok[r] = 1; sh.m[r] = 0; sh.M[r] = 0; sh.L[r] = 0; sh.amax[r] = -1; }
      continue;
    }
    const RowStat s = combine_row(part + (size_t)(row0 + r) * ntiles, ntiles, greedy, sc, lane);
    if (lane == 0) {
      sh.m[r] = s.m;
      sh.M[r] = s.M;
      sh.L[r] = s.L;
      sh.amax[r] = s.amax;
      sh.ok[r] = s.ok;
    }
  }
}

template <typename T>
__device__ __forceinline__ const T* row_ptr(const unsigned char* base, long long ld_bytes,
                                            long long row) {
  return reinterpret_cast<const T*>(base + row * ld_bytes);
}

// One speculative check on n positions. Target row j: tp(j) with log2
// partition sh.M + sh.L at index tr0 + j; draft law of position j: row dp(j)
// with log2 partition dlt(j). Returns a via sh.a (warp 0); sh.bad is set if a
// draft id is out of range.
template <typename T, typename TP, typename DP, typename DS>
__device__ void accept_scan(SeqShared& sh, int n, int pos0, int stage, const DecideCommon& c,
                            int b, bool greedy, double cd, const int32_t* drafts, TP tp, DP dp,
                            DS dstat, int tr0, double* diag_p, double* diag_q) {
  const int lane = threadIdx.x & 31;
  int a = n, bad = 0;
  for (int j0 = 0; j0 < n; j0 += 32) {
    const int j = j0 + lane;
    bool acc = true, badj = false;
    if (j < n) {
      const int x = drafts[j];
      if (x < 0 || x >= c.V) {
        badj = true;
      } else if (greedy) {
        acc = (x == sh.amax[tr0 + j]);
      } else {
        const double lp = (double)load_elem(tp(j) + x) * cd - (sh.M[tr0 + j] + sh.L[tr0 + j]);
        const double lq = (double)load_elem(dp(j) + x) * cd - dstat(j);
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

// ---------------------------------------------------------------------------
// Chain verification
// ---------------------------------------------------------------------------
template <typename T>
__global__ void __launch_bounds__(kDecideThreads)
    chain_decide_kernel(ChainDecideArgs A) {
  extern __shared__ double dyn_pre[];
  __shared__ SeqShared sh;
  __shared__ bool want[kMaxRows];
  const DecideCommon& c = A.c;
  const int b = blockIdx.y, sp = blockIdx.x, K = c.K, V = c.V;
  const int nrt = residual_tiles(V);
  const float Tb = c.temperature[b];
  const bool tvalid = temp_valid(Tb);
  const bool greedy = (Tb == 0.0f);
  if (sp > 0 && (greedy || !tvalid)) return;
  const Scale sc = tvalid && !greedy ? make_scale(Tb) : Scale{0.f, 0.f, 0.0};
  const double cd = sc.d;
  const int per = 2 * K + 1;
  for (int r = threadIdx.x; r < per; r += blockDim.x) want[r] = (r <= K) || !greedy;
  __syncthreads();
  double* diag = c.diag ? c.diag + (size_t)b * (4 * K + 2) : nullptr;

  auto fail = [&]() {
    if (threadIdx.x == 0) set_status(c.status, SPEC_EDEVICE);
    for (int j = threadIdx.x; j <= K; j += blockDim.x) A.out_tok[(size_t)b * (K + 1) + j] = -1;
    if (threadIdx.x == 0) A.accept_len[b] = -1;
    if (diag)
      for (int j = threadIdx.x; j < 4 * K + 2; j += blockDim.x) diag[j] = __longlong_as_double(0x7ff8000000000000ll);
  };
  if (!tvalid) { if (sp == 0) fail(); return; }

  combine_rows(sh, c.part, b * per, per, c.ntiles, want, greedy, sc);
  __syncthreads();
  const int32_t* drafts = c.draft_tok + (size_t)b * K;
  const unsigned char* tgt = A.tgt;
  const unsigned char* drf = A.drf;
  auto tp = [&](int j) { return row_ptr<T>(tgt, A.ld_tgt, (long long)b * (K + 1) + j); };
  auto dp = [&](int j) { return row_ptr<T>(drf, A.ld_drf, (long long)b * K + j); };
  auto ds = [&](int j) { return sh.M[K + 1 + j] + sh.L[K + 1 + j]; };
  if (threadIdx.x < 32) {
    const bool dg = diag && sp == 0 && !greedy;
    accept_scan<T>(sh, K, 0, 1, c, b, greedy, cd, drafts, tp, dp, ds, 0,
                   dg ? diag + 2 * K + 1 : nullptr, dg ? diag + 3 * K + 1 : nullptr);
  }
  __syncthreads();
  int rowbad = 0;
  for (int r = 0; r < per; ++r) rowbad |= (want[r] && !sh.ok[r]);
  if (sh.bad || rowbad) { if (sp == 0) fail(); return; }
  const int a = sh.a;

  int tok;
  double Z = __longlong_as_double(0x7ff8000000000000ll);
  if (greedy) {
    tok = sh.amax[a];
  } else {
    const T* prow = tp(a);
    const T* qrow = a < K ? dp(a) : nullptr;
    const ProbCoef kp = make_coef(sh.M[a] + sh.L[a], sc);
    const ProbCoef kq = make_coef(a < K ? ds(a) : 0.0, sc);
    const float u = spec_uniforms(c.seed, (uint32_t)c.seq_id[b], c.round, (uint32_t)a, 1u).y;
    if (!draw_token<T>(c, b, sp, prow, qrow, kp, kq, u, dyn_pre, &tok, &Z)) return;
  }
  // Emit.
  for (int j = threadIdx.x; j <= K; j += blockDim.x)
    A.out_tok[(size_t)b * (K + 1) + j] = j < a ? drafts[j] : (j == a ? tok : -1);
  if (threadIdx.x == 0) A.accept_len[b] = a;
  if (diag) {
    for (int j = threadIdx.x; j < per; j += blockDim.x)
      diag[j] = greedy ? __longlong_as_double(0x7ff8000000000000ll)
                       : (sh.M[j] + sh.L[j]) * kLn2;
    if (greedy)
      for (int j = threadIdx.x; j < 2 * K; j += blockDim.x)
        diag[per + j] = __longlong_as_double(0x7ff8000000000000ll);
    if (threadIdx.x == 0) diag[4 * K + 1] = Z;
  }
}

cudaError_t launch_chain_decide(const ChainDecideArgs& a, cudaStream_t st) {
  const int nrt = residual_tiles(a.c.V);
  const size_t smem = 2 * (size_t)nrt * sizeof(double);
  dim3 grid(a.c.nsplit, a.c.B);
  if (a.c.dtype == SPEC_BF16) {
    if (smem > 48 * 1024 &&
        cudaFuncSetAttribute(chain_decide_kernel<__nv_bfloat16>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) != cudaSuccess)
      return cudaGetLastError();
    chain_decide_kernel<__nv_bfloat16><<<grid, kDecideThreads, smem, st>>>(a);
  } else {
    if (smem > 48 * 1024 &&
        cudaFuncSetAttribute(chain_decide_kernel<float>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)smem) != cudaSuccess)
      return cudaGetLastError();
    chain_decide_kernel<float><<<grid, kDecideThreads, smem, st>>>(a);
  }
  return cudaGetLastError();
}


// ---------------------------------------------------------------------------
// Two-stage verification
// ---------------------------------------------------------------------------
constexpr long long kNaNBits = 0x7ff8000000000000ll;

// Stage one: drafts (slots w..w+K-1) against L_i (slots w..w+K), draft law
// L_d. The a1 accepted drafts and the drawn token join the window together
// with the L_i statistics of their slots.
template <typename T>
__global__ void __launch_bounds__(kDecideThreads)
    hier1_decide_kernel(HierDecideArgs A) {
  extern __shared__ double dyn_pre[];
  __shared__ SeqShared sh;
  __shared__ bool want[kMaxRows];
  const DecideCommon& c = A.c;
  const int b = blockIdx.y, sp = blockIdx.x, K = c.K, S = A.S, Ni = A.Ni;
  const int WC = Ni + K;  // window capacity
  const float Tb = c.temperature[b];
  const bool tvalid = temp_valid(Tb);
  const bool greedy = (Tb == 0.0f);
  if (sp > 0 && (greedy || !tvalid)) return;
  const int w = A.win_len[b];
  const bool wvalid = (w >= 0 && w < Ni);
  if (sp > 0 && !wvalid) return;
  const Scale sc = tvalid && !greedy ? make_scale(Tb) : Scale{0.f, 0.f, 0.0};
  const double cd = sc.d;
  const int per = 2 * K + 1;
  const int D = 4 * K + 3 * S + 1;
  double* diag = c.diag ? c.diag + (size_t)b * D : nullptr;

  // Stage-two outputs default to "did not run"; stage two overwrites them.
  if (sp == 0) {
    for (int j = threadIdx.x; j < WC + 1; j += blockDim.x) A.commit_tok[(size_t)b * (WC + 1) + j] = -1;
    if (threadIdx.x == 0) { A.commit_n[b] = 0; A.acc2[b] = -1; }
    if (diag)
      for (int j = threadIdx.x; j < D; j += blockDim.x) diag[j] = __longlong_as_double(kNaNBits);
  }
  if (!tvalid || !wvalid) {
    if (sp == 0 && threadIdx.x == 0) { set_status(c.status, SPEC_EDEVICE); A.acc1[b] = -1; }
    return;
  }
  for (int r = threadIdx.x; r < per; r += blockDim.x) want[r] = (r <= K) || !greedy;
  __syncthreads();

  combine_rows(sh, c.part, b * per, per, c.ntiles, want, greedy, sc);
  __syncthreads();
  const int32_t* drafts = c.draft_tok + (size_t)b * K;
  const long long row0 = (long long)b * S + w;
  auto tp = [&](int j) { return row_ptr<T>(A.lg_i, A.ld, row0 + j); };
  auto dp = [&](int j) { return row_ptr<T>(A.lg_d, A.ld, row0 + j); };
  auto ds = [&](int j) { return sh.M[K + 1 + j] + sh.L[K + 1 + j]; };
  if (threadIdx.x < 32) {
    const bool dg = diag && sp == 0 && !greedy;
    accept_scan<T>(sh, K, w, 1, c, b, greedy, cd, drafts, tp, dp, ds, 0,
                   dg ? diag + 2 * K + 1 : nullptr, dg ? diag + 3 * K + 1 : nullptr);
  }
  __syncthreads();
  int rowbad = 0;
  for (int r = 0; r < per; ++r) rowbad |= (want[r] && !sh.ok[r]);
  if (sh.bad || rowbad) {
    if (sp == 0 && threadIdx.x == 0) { set_status(c.status, SPEC_EDEVICE); A.acc1[b] = -1; }
    return;
  }
  const int a = sh.a;
  int tok;
  double Z = __longlong_as_double(kNaNBits);
  if (greedy) {
    tok = sh.amax[a];
  } else {
    const T* prow = tp(a);
    const T* qrow = a < K ? dp(a) : nullptr;
    const ProbCoef kp = make_coef(sh.M[a] + sh.L[a], sc);
    const ProbCoef kq = make_coef(a < K ? ds(a) : 0.0, sc);
    const float u =
        spec_uniforms(c.seed, (uint32_t)c.seq_id[b], c.round, (uint32_t)(w + a), 1u).y;
    if (!draw_token<T>(c, b, sp, prow, qrow, kp, kq, u, dyn_pre, &tok, &Z)) return;
  }
  // Append a + 1 tokens and their L_i statistics to the window.
  for (int j = threadIdx.x; j <= a; j += blockDim.x) {
    const size_t slot = (size_t)b * WC + w + j;
    A.win_tok[slot] = j < a ? drafts[j] : tok;
    A.win_stat[2 * slot] = greedy ? __longlong_as_double(kNaNBits) : sh.m[j];
    A.win_stat[2 * slot + 1] =
        greedy ? __longlong_as_double(kNaNBits) : (sh.M[j] + sh.L[j] - sh.m[j] * cd) * kLn2;
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    A.win_len[b] = w + a + 1;
    A.acc1[b] = a;
  }
  if (diag && !greedy) {
    for (int j = threadIdx.x; j < per; j += blockDim.x) diag[j] = (sh.M[j] + sh.L[j]) * kLn2;
    if (threadIdx.x == 0) diag[4 * K + 1] = Z;
  }
}

// Stage two: for sequences whose window holds W >= Ni tokens, the window
// tokens (slots 0..W-1) against L_f (slots 0..W), draft law L_i from the
// buffered statistics; commits a2 + 1 tokens and empties the window.
template <typename T>
__global__ void __launch_bounds__(kDecideThreads)
    hier2_decide_kernel(HierDecideArgs A) {
  extern __shared__ double dyn_pre[];
  __shared__ SeqShared sh;
  __shared__ bool want[kMaxRows];
  const DecideCommon& c = A.c;
  const int b = blockIdx.y, sp = blockIdx.x, K = c.K, S = A.S, Ni = A.Ni;
  const int WC = Ni + K;
  if (A.acc1[b] < 0) return;
  const int W = A.win_len[b];
  if (!(W >= Ni && W < S)) return;
  const float Tb = c.temperature[b];
  const bool greedy = (Tb == 0.0f);  // temperature validated by stage one
  if (sp > 0 && greedy) return;
  const Scale sc = !greedy ? make_scale(Tb) : Scale{0.f, 0.f, 0.0};
  const double cd = sc.d;
  const int D = 4 * K + 3 * S + 1;
  double* diag = c.diag ? c.diag + (size_t)b * D + (4 * K + 2) : nullptr;
  for (int r = threadIdx.x; r < S; r += blockDim.x) want[r] = (r <= W);
  __syncthreads();

  combine_rows(sh, c.part, b * S, W + 1, c.ntiles, want, greedy, sc);
  __syncthreads();
  const int32_t* wtok = A.win_tok + (size_t)b * WC;
  const double* wst = A.win_stat + (size_t)b * WC * 2;
  auto tp = [&](int j) { return row_ptr<T>(A.lg_f, A.ld, (long long)b * S + j); };
  auto dp = [&](int j) { return row_ptr<T>(A.lg_i, A.ld, (long long)b * S + j); };
  auto ds = [&](int j) { return wst[2 * j] * cd + wst[2 * j + 1] * kLog2e; };
  if (threadIdx.x < 32) {
    const bool dg = diag && sp == 0 && !greedy;
    accept_scan<T>(sh, W, 0, 2, c, b, greedy, cd, wtok, tp, dp, ds, 0,
                   dg ? diag + S : nullptr, dg ? diag + 2 * S - 1 : nullptr);
  }
  __syncthreads();
  int rowbad = 0;
  for (int r = 0; r <= W; ++r) rowbad |= !sh.ok[r];
  if (sh.bad || rowbad) {
    if (sp == 0 && threadIdx.x == 0) { set_status(c.status, SPEC_EDEVICE); A.acc2[b] = -1; }
    return;
  }
  const int a = sh.a;
  int tok;
  double Z = __longlong_as_double(kNaNBits);
  if (greedy) {
    tok = sh.amax[a];
  } else {
    const T* prow = tp(a);
    const T* qrow = a < W ? dp(a) : nullptr;
    const ProbCoef kp = make_coef(sh.M[a] + sh.L[a], sc);
    const ProbCoef kq = make_coef(a < W ? ds(a) : 0.0, sc);
    const float u = spec_uniforms(c.seed, (uint32_t)c.seq_id[b], c.round, (uint32_t)a, 2u).y;
    if (!draw_token<T>(c, b, sp, prow, qrow, kp, kq, u, dyn_pre, &tok, &Z)) return;
  }
  for (int j = threadIdx.x; j < WC + 1; j += blockDim.x)
    A.commit_tok[(size_t)b * (WC + 1) + j] = j < a ? wtok[j] : (j == a ? tok : -1);
  __syncthreads();
  if (threadIdx.x == 0) {
    A.commit_n[b] = a + 1;
    A.acc2[b] = a;
    A.win_len[b] = 0;
  }
  if (diag && !greedy) {
    for (int j = threadIdx.x; j <= W; j += blockDim.x) diag[j] = (sh.M[j] + sh.L[j]) * kLn2;
    if (threadIdx.x == 0) diag[3 * S - 2] = Z;
  }
}

template <typename K1, typename K2>
static cudaError_t launch_decide(K1 kb, K2 kf, int dtype, dim3 grid, size_t smem,
                                 const HierDecideArgs& a, cudaStream_t st) {
  if (dtype == SPEC_BF16) {
    if (smem > 48 * 1024 &&
        cudaFuncSetAttribute(kb, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) !=
            cudaSuccess)
      return cudaGetLastError();
    kb<<<grid, kDecideThreads, smem, st>>>(a);
  } else {
    if (smem > 48 * 1024 &&
        cudaFuncSetAttribute(kf, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) !=
            cudaSuccess)
      return cudaGetLastError();
    kf<<<grid, kDecideThreads, smem, st>>>(a);
  }
  return cudaGetLastError();
}

cudaError_t launch_hier1_decide(const HierDecideArgs& a, cudaStream_t st) {
  const size_t smem = 2 * (size_t)residual_tiles(a.c.V) * sizeof(double);
  return launch_decide(hier1_decide_kernel<__nv_bfloat16>, hier1_decide_kernel<float>, a.c.dtype,
                       dim3(a.c.nsplit, a.c.B), smem, a, st);
}
cudaError_t launch_hier2_decide(const HierDecideArgs& a, cudaStream_t st) {
  const size_t smem = 2 * (size_t)residual_tiles(a.c.V) * sizeof(double);
  return launch_decide(hier2_decide_kernel<__nv_bfloat16>, hier2_decide_kernel<float>, a.c.dtype,
                       dim3(a.c.nsplit, a.c.B), smem, a, st);
}

}  // namespace specv
