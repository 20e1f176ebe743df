// Inverse-CDF draw of one token from the weights max(0, p - q) (or p) of a
// row pair, shared by the decide kernels (resampled and bonus tokens) and the
// draft-step kernel (draft tokens). Probabilities are 2^(x*c - Lt) with the
// row's log2-partition Lt; a thread-block cluster of kCluster CTAs per
// sequence splits the 256-element residual tiles, writes the tile sums into
// the leader CTA's shared memory, and the leader prefixes them, finds the
// tile holding u * Z and rescans it.
//
// Rules: speculative sampling as appealed to by HiSpec (gist.science summary
// of arXiv 2510.01336, section 2, "Verlustfreie Garantie"); the residual
// proportional to the target-minus-draft difference (Speculative Speculative
// Decoding summary, Technische Zusammenfassung 3.B).
#pragma once

#include <climits>

#include <cooperative_groups.h>

#include "common.cuh"
#include "kernels.cuh"

namespace specv {

namespace cg = cooperative_groups;

constexpr int kCluster = 4;                  // CTAs per sequence
constexpr int kDecThreads = 512;
constexpr int kDecWarps = kDecThreads / 32;
// Residual tiles whose loads a warp keeps in flight together (64 bytes per
// lane and row).
template <typename T>
constexpr int kResGroup = sizeof(T) == 2 ? 4 : 2;
// Groups claimed from a counter are smaller: the finer hand-out balances the
// CTAs of a cluster better (B=64, K=8, V=128256 bf16 verify-and-commit step:
// 80.4 us with 2 tiles per group, 81.3 with 1 or 3, 82.4 with 4).
template <typename T>
constexpr int kResClaimGroup = 2;

// ---------------------------------------------------------------------------
// Residual weights of 8 consecutive elements
// ---------------------------------------------------------------------------
// 8 consecutive logits as raw 16-byte vectors (one for bf16, two for fp32);
// zeros when `on` is false (nothing is read then). The loads go to L2 and
// allocate nothing in L1: a warp keeps several tiles of them in flight, more
// than the L1 left beside a large shared-memory carve-out can hold.
template <typename T>
struct Raw8 {
  uint4 v[sizeof(T) / 2];
};
template <typename T>
__device__ __forceinline__ Raw8<T> raw8(const T* row, int e0, bool on) {
  Raw8<T> r;
  const uint4* p = reinterpret_cast<const uint4*>(row + e0);
#pragma unroll
  for (int i = 0; i < (int)(sizeof(T) / 2); ++i)
    r.v[i] = on ? __ldcg(p + i) : make_uint4(0u, 0u, 0u, 0u);
  return r;
}
__device__ __forceinline__ void unpack8(const Raw8<__nv_bfloat16>& r, float x[8]) {
  const uint4 w = r.v[0];
  x[0] = bf_lo(w.x); x[1] = bf_hi(w.x); x[2] = bf_lo(w.y); x[3] = bf_hi(w.y);
  x[4] = bf_lo(w.z); x[5] = bf_hi(w.z); x[6] = bf_lo(w.w); x[7] = bf_hi(w.w);
}
__device__ __forceinline__ void unpack8(const Raw8<float>& r, float x[8]) {
  x[0] = __uint_as_float(r.v[0].x); x[1] = __uint_as_float(r.v[0].y);
  x[2] = __uint_as_float(r.v[0].z); x[3] = __uint_as_float(r.v[0].w);
  x[4] = __uint_as_float(r.v[1].x); x[5] = __uint_as_float(r.v[1].y);
  x[6] = __uint_as_float(r.v[1].z); x[7] = __uint_as_float(r.v[1].w);
}
// Elements e0 .. e0+7 of a row of V elements; -inf past the end.
template <typename T>
__device__ __forceinline__ void load8(const T* row, int e0, int V, float x[8]) {
  if (e0 + 8 <= V) {
    unpack8(raw8(row, e0, true), x);
  } else {
#pragma unroll
    for (int e = 0; e < 8; ++e) x[e] = (e0 + e < V) ? load_elem(row + e0 + e) : -INFINITY;
  }
}

// Probability of a logit x of a row with log2-partition Lt and largest logit
// m: p = 2^(x*c - Lt) (c = chi + clo), formed as 2^(x*c - M) * k with the
// integral shift M = ceil(m * chi) and k = 2^(M - Lt) carried as two floats.
// The most likely tokens get exponents in (-1, 0], where the fp32 rounding of
// x*chi - M (once, by the FMA) is smallest; k is exact to about 2^-48.
struct ProbCoef {
  float chi, clo, nM, khi, klo;
};
__device__ __forceinline__ ProbCoef make_coef(double Lt, float m, const Scale& s) {
  ProbCoef k;
  k.chi = s.hi;
  k.clo = s.lo;
  float M = ceilf(m * s.hi);
  if (!(M > -INFINITY && M < INFINITY)) M = 0.0f;  // no finite maximum: any shift
  k.nM = -M;
  const double f = exp2((double)M - Lt);
  k.khi = (float)f;
  k.klo = (float)(f - (double)k.khi);
  return k;
}
__device__ __forceinline__ float2 prob2(float2 x, const ProbCoef& k) {
  float2 t = __ffma2_rn(x, make_float2(k.chi, k.chi), make_float2(k.nM, k.nM));
  t = __ffma2_rn(x, make_float2(k.clo, k.clo), t);
  const float2 e = make_float2(ex2(t.x), ex2(t.y));
  return __ffma2_rn(e, make_float2(k.khi, k.khi), __fmul2_rn(e, make_float2(k.klo, k.klo)));
}

// Weights w = max(0, p - q) (or p when there is no draft row) of 8 elements
// given their logits.
__device__ __forceinline__ void weights_of(const float xp[8], const float xq[8], bool has_q,
                                           const ProbCoef& kp, const ProbCoef& kq, float w[8]) {
#pragma unroll
  for (int e = 0; e < 8; e += 2) {
    const float2 p = prob2(make_float2(xp[e], xp[e + 1]), kp);
    if (has_q) {
      const float2 q = prob2(make_float2(xq[e], xq[e + 1]), kq);
      w[e] = fmaxf(p.x - q.x, 0.0f);
      w[e + 1] = fmaxf(p.y - q.y, 0.0f);
    } else {
      w[e] = p.x;
      w[e + 1] = p.y;
    }
  }
}
// Same, reading the 8 elements at e0 (any e0 < V).
template <typename T>
__device__ __forceinline__ void weights8(const T* prow, const T* qrow, int e0, int V,
                                         const ProbCoef& kp, const ProbCoef& kq, float w[8]) {
  float xp[8], xq[8];
  if (e0 + 8 <= V) {  // both loads in flight together
    const Raw8<T> rp = raw8(prow, e0, true);
    const Raw8<T> rq = raw8(qrow ? qrow : prow, e0, qrow != nullptr);
    unpack8(rp, xp);
    unpack8(rq, xq);
  } else {
    load8<T>(prow, e0, V, xp);
    if (qrow) load8<T>(qrow, e0, V, xq);
  }
  weights_of(xp, xq, qrow != nullptr, kp, kq, w);
}
// A lane's 8 weights summed pairwise in fp32 (error ~ 3 ulp of the small
// sum), then widened; tiles and lanes combine in fp64.
__device__ __forceinline__ double lane_sum8(const float w[8]) {
  const float2 a = __fadd2_rn(make_float2(w[0], w[1]), make_float2(w[2], w[3]));
  const float2 b = __fadd2_rn(make_float2(w[4], w[5]), make_float2(w[6], w[7]));
  const float2 c = __fadd2_rn(a, b);
  return (double)(c.x + c.y);
}


// ---------------------------------------------------------------------------
// Residual tile sums and the draw
// ---------------------------------------------------------------------------
// Tile sums of the weights over residual tiles [t0, t1), written to out
// (the leader CTA's shared memory, possibly remote). A warp takes groups of
// kResGroup tiles and issues all their loads before using any.
template <typename T>
__device__ void residual_tile_sums(const T* prow, const T* qrow, int V, const ProbCoef& kp,
                                   const ProbCoef& kq, int t0, int t1, double* out) {
  constexpr int G = kResGroup<T>;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const bool hq = qrow != nullptr;
  for (int tb = t0 + warp * G; tb < t1; tb += kDecWarps * G) {
    Raw8<T> rp[G], rq[G];
    bool full[G];
#pragma unroll
    for (int u = 0; u < G; ++u) {
      const int e0 = (tb + u) * kResTile + lane * 8;
      full[u] = tb + u < t1 && e0 + 8 <= V;
      rp[u] = raw8(prow, e0, full[u]);
      rq[u] = raw8(hq ? qrow : prow, e0, full[u] && hq);
    }
    double s[G];
#pragma unroll
    for (int u = 0; u < G; ++u) {
      const int t = tb + u, e0 = t * kResTile + lane * 8;
      float w[8];
      if (full[u]) {
        float xp[8], xq[8];
        unpack8(rp[u], xp);
        unpack8(rq[u], xq);
        weights_of(xp, xq, hq, kp, kq, w);
      } else if (t < t1 && e0 < V) {
        weights8<T>(prow, qrow, e0, V, kp, kq, w);  // the row's ragged end
      } else {
#pragma unroll
        for (int e = 0; e < 8; ++e) w[e] = 0.0f;
      }
      s[u] = lane_sum8(w);
    }
#pragma unroll
    for (int u = 0; u < G; ++u) {
      const double v = warp_sum_d(s[u]);
      if (lane == 0 && tb + u < t1) out[tb + u] = v;
    }
  }
}

// Same, with groups of kResClaimGroup tiles claimed one at a time from a
// counter (any shared memory of the cluster) by every warp that calls it.
template <typename T>
__device__ void residual_tile_sums_claimed(const T* prow, const T* qrow, int V,
                                           const ProbCoef& kp, const ProbCoef& kq, int nrt,
                                           double* out, int* claim) {
  constexpr int G = kResClaimGroup<T>;
  const int lane = threadIdx.x & 31;
  const bool hq = qrow != nullptr;
  const int ngroups = (nrt + G - 1) / G;
  for (;;) {
    int g = 0;
    if (lane == 0) g = atomicAdd(claim, 1);
    g = __shfl_sync(0xffffffffu, g, 0);
    if (g >= ngroups) break;
    const int tb = g * G;
    Raw8<T> rp[G], rq[G];
    bool full[G];
#pragma unroll
    for (int u = 0; u < G; ++u) {
      const int e0 = (tb + u) * kResTile + lane * 8;
      full[u] = tb + u < nrt && e0 + 8 <= V;
      rp[u] = raw8(prow, e0, full[u]);
      rq[u] = raw8(hq ? qrow : prow, e0, full[u] && hq);
    }
    double s[G];
#pragma unroll
    for (int u = 0; u < G; ++u) {
      const int t = tb + u, e0 = t * kResTile + lane * 8;
      float w[8];
      if (full[u]) {
        float xp[8], xq[8];
        unpack8(rp[u], xp);
        unpack8(rq[u], xq);
        weights_of(xp, xq, hq, kp, kq, w);
      } else if (t < nrt && e0 < V) {
        weights8<T>(prow, qrow, e0, V, kp, kq, w);
      } else {
#pragma unroll
        for (int e = 0; e < 8; ++e) w[e] = 0.0f;
      }
      s[u] = lane_sum8(w);
    }
#pragma unroll
    for (int u = 0; u < G; ++u) {
      const double v = warp_sum_d(s[u]);
      if (lane == 0 && tb + u < nrt) out[tb + u] = v;
    }
  }
}

// Leader: given all tile sums in shared memory (tsum), prefix them in a fixed
// order, locate u * Z, rescan that tile and return the drawn token in every
// thread (-1 if the weights have no mass). *Z_out gets Z. A caller that owns
// one piece of a longer row passes its own target (>= 0) instead of u * Z.
template <typename T>
__device__ int residual_pick(const T* prow, const T* qrow, int V, const ProbCoef& kp,
                             const ProbCoef& kq, const double* tsum, double* pre, int nrt,
                             float u, double* Z_out, double target_in = -1.0) {
  __shared__ double s_wtot[kDecWarps];
  __shared__ int s_tile, s_tok;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  // Each thread owns a contiguous run of tiles; the run sums are scanned over
  // the block (warp shuffles, then the warp totals in order).
  const int per = (nrt + kDecThreads - 1) / kDecThreads;
  const int a = min(nrt, (int)threadIdx.x * per), b = min(nrt, a + per);
  double run = 0.0;
  for (int t = a; t < b; ++t) run += tsum[t];
  double incl = run;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const double y = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += y;
  }
  double excl = __shfl_up_sync(0xffffffffu, incl, 1);
  if (lane == 0) excl = 0.0;
  if (lane == 31) s_wtot[warp] = incl;
  if (threadIdx.x == 0) s_tile = -1;
  __syncthreads();
  double Z = 0.0, c = 0.0;
#pragma unroll
  for (int w = 0; w < kDecWarps; ++w) {
    if (w == warp) c = Z;
    Z += s_wtot[w];
  }
  *Z_out = Z;
  if (!(Z > 0.0)) return -1;
  const double target = target_in >= 0.0 ? target_in : (double)u * Z;
  // The last tile with mass whose prefix does not exceed the target.
  c += excl;
  int cand = -1;
  for (int t = a; t < b; ++t) {
    pre[t] = c;
    if (c <= target && tsum[t] > 0.0) cand = t;
    c += tsum[t];
  }
  if (cand >= 0) atomicMax(&s_tile, cand);
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
    const double start = pre[tile] + excl;
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

// Leader, after the cluster's tile sums are in: the draw, with the fall-back
// to p when the residual mass is zero as computed (p == q).
template <typename T>
__device__ int leader_draw(const T* prow, const T* qrow, int V, const ProbCoef& kp,
                           const ProbCoef& kq, double* tsum, double* pre, float u, double* Z) {
  const int nrt = residual_tiles(V);
  int tok = residual_pick<T>(prow, qrow, V, kp, kq, tsum, pre, nrt, u, Z);
  if (tok < 0 && qrow) {
    __syncthreads();
    residual_tile_sums<T>(prow, nullptr, V, kp, kq, 0, nrt, tsum);
    __syncthreads();
    tok = residual_pick<T>(prow, nullptr, V, kp, kq, tsum, pre, nrt, u, Z);
  }
  return tok;
}

constexpr long long kNaNBits = 0x7ff8000000000000ll;
__device__ __forceinline__ double dnan() { return __longlong_as_double(kNaNBits); }

template <typename T>
__device__ __forceinline__ const T* row_ptr(const unsigned char* base, long long ld_bytes,
                                            long long row) {
  return reinterpret_cast<const T*>(base + row * ld_bytes);
}

}  // namespace specv
