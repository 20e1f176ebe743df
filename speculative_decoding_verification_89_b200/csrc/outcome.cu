// Outcome law of a chain check with the drafts fixed: the probability of each
// acceptance length and the most likely (length, token) outcomes, for a
// speculation cache that prepares continuations of the likely outcomes while
// the check runs.
//
// Speculative Speculative Decoding (gist.science summary of arXiv
// 2603.03251), Technische Zusammenfassung 2 (predict how many tokens the
// running verification accepts and which bonus token it draws, and prepare
// continuations for them), 3.A (a budget spent mostly on short acceptance
// lengths, whose probability decays geometrically) and 3.B (the token after a
// rejection follows the residual distribution, proportional to the
// target-minus-draft difference). With beta_j = min(1, p_j(x_j) / q_j(x_j)):
// P(a = k) = beta_0..beta_{k-1} (1 - beta_k), P(a = K) = beta_0..beta_{K-1};
// given a = k the token follows max(0, p_k - q_k) normalised (p_K for k = K).
// A budget of n outcomes covers the n most likely pairs (k, v).
//
// Three launches: the row statistics of the chain rows (the row pairs of the
// first positions streamed last, to be read again from L2); one CTA per
// (sequence, position k) that streams the row pair once for the residual mass
// Z_k and the exact n largest weights max(0, p_k - q_k) (sorted lists held one
// entry per lane, a shared threshold, candidates sorted and merged 32 at a
// time, their weights formed again in fp64); one CTA per sequence for beta,
// the length law and the merge of the K+1 lists by P(a = k) w / Z_k in fp64.
#include "draw.cuh"

namespace specv {

constexpr int kMaxTop = SPEC_MAX_TOP;
static_assert(kMaxTop <= 32, "a top list is held one entry per lane");

// ---------------------------------------------------------------------------
// Sorted lists of the 32 best candidates, entry i in lane i (empty: w = -1).
// Order: larger weight first, then the smaller index.
// ---------------------------------------------------------------------------
template <typename W>
struct Top {
  W w;
  int i;
};
template <typename W>
__device__ __forceinline__ Top<W> top_empty() {
  return Top<W>{W(-1), 0x7fffffff};
}
template <typename W>
__device__ __forceinline__ bool beats(W wa, int ia, W wb, int ib) {
  return wa > wb || (wa == wb && ia < ib);
}
// One compare-exchange with the lane at distance j: the lane keeps the
// better of the pair if keep_better, else the worse.
template <typename W>
__device__ __forceinline__ void top_cx(Top<W>& e, int j, bool keep_better) {
  const W ow = __shfl_xor_sync(0xffffffffu, e.w, j);
  const int oi = __shfl_xor_sync(0xffffffffu, e.i, j);
  const bool take = keep_better ? beats(ow, oi, e.w, e.i) : beats(e.w, e.i, ow, oi);
  if (take) { e.w = ow; e.i = oi; }
}
// Bitonic sort of one entry per lane, best in lane 0.
template <typename W>
__device__ __forceinline__ void top_sort(Top<W>& e, int lane) {
#pragma unroll
  for (int k = 2; k <= 32; k <<= 1)
#pragma unroll
    for (int j = k >> 1; j > 0; j >>= 1) top_cx(e, j, ((lane & k) == 0) == ((lane & j) == 0));
}
// The 32 best of a and b, both sorted: the better of a[l] and b[31 - l] form
// a bitonic sequence holding them, sorted by a bitonic merge.
template <typename W>
__device__ __noinline__ Top<W> top_merged(Top<W> a, Top<W> b, int lane) {
  const W bw = __shfl_sync(0xffffffffu, b.w, 31 - lane);
  const int bi = __shfl_sync(0xffffffffu, b.i, 31 - lane);
  if (beats(bw, bi, a.w, a.i)) { a.w = bw; a.i = bi; }
#pragma unroll
  for (int j = 16; j > 0; j >>= 1) top_cx(a, j, (lane & j) == 0);
  return a;
}

// 16 bytes of a row: plain L2 loads for the row pairs the statistics pass
// streamed last (still in L2), evict-first ones for the rest so that they do
// not push those out.
template <typename T>
__device__ __forceinline__ Raw8<T> raw8_pol(const T* row, int e0, bool on, bool hint,
                                            uint64_t pol) {
  if (!hint) return raw8(row, e0, on);
  Raw8<T> r;
  const uint4* p = reinterpret_cast<const uint4*>(row + e0);
#pragma unroll
  for (int i = 0; i < (int)(sizeof(T) / 2); ++i) {
    uint4 v = make_uint4(0u, 0u, 0u, 0u);
    if (on)
      asm("ld.global.nc.L1::no_allocate.L2::cache_hint.v4.u32 {%0, %1, %2, %3}, [%4], %5;"
          : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
          : "l"(p + i), "l"(pol));
    r.v[i] = v;
  }
  return r;
}

// ---------------------------------------------------------------------------
// One CTA of kPairWarps warps per (sequence b, position k): the residual mass
// Z_k and the n largest weights. The row pair streams through each warp's
// ring of shared-memory stages (1-D bulk copies). Each warp keeps its own
// sorted list; the CTA shares a threshold, the best n-th entry of any warp's
// list (no weight below it can be among the n largest), seeded from the
// warps' first step. A lane compares the largest of its 8 weights, each
// loosened by more than its fp32 error, with the threshold; the rare lanes
// that pass append their candidates to the warp's buffer. Once per step a
// buffer holding more than kFlushAt entries is flushed 32 entries at a time:
// each entry's weight formed again in fp64 from its two logits, filtered,
// the 32 sorted and merged into the list. The warps' lists meet in a merge
// tree at the end.
// ---------------------------------------------------------------------------
constexpr int kPairWarps = 8;
// Tiles whose loads a warp keeps in flight: 64 bytes per lane either way.
template <typename T>
constexpr int kPairGroup = sizeof(T) == 2 ? 2 : 1;
// A warp's buffer is flushed once it holds more than kFlushAt entries, so
// the threshold rises early in the stream. The count is checked once per
// step, which adds at most 2 tiles x 256 entries.
constexpr int kFlushAt = 32;
constexpr int kBufCap = kFlushAt + 2 * 32 * 8;
// The fp32 weight of a token is within 2^-18.8 (p + q) of the exact one
// when p, q >= 2^-24 k (the exponent x c - M, at most 24 in magnitude, is
// rounded twice: ln 2 * 2^-23 * 24; the ex2 approximation and the one-float
// k add about 2^-21), and far closer in absolute terms below that:
// w + kSlack (p + q) bounds the exact weight from above, w - kSlack (p + q)
// from below.
constexpr float kSlack = 1.0f / 16384.0f;

struct PairRow {
  double Lp, Lq, cd;
  bool hq;
};
// max(0, p - q) of token v in fp64 from its logits.
template <typename T>
__device__ __forceinline__ double exact_weight(const T* prow, const T* qrow, int v,
                                               const PairRow& r) {
  double w = exp2((double)load_elem(prow + v) * r.cd - r.Lp);
  if (r.hq) w -= exp2((double)load_elem(qrow + v) * r.cd - r.Lq);
  return w > 0.0 ? w : 0.0;
}

// Element pair j (elements 2j, 2j+1) of 8 consecutive logits held raw.
__device__ __forceinline__ float2 pair_of(const Raw8<__nv_bfloat16>& r, int j) {
  const uint32_t w = j == 0 ? r.v[0].x : j == 1 ? r.v[0].y : j == 2 ? r.v[0].z : r.v[0].w;
  return make_float2(bf_lo(w), bf_hi(w));
}
__device__ __forceinline__ float2 pair_of(const Raw8<float>& r, int j) {
  const uint4 h = r.v[j >> 1];
  return (j & 1) ? make_float2(__uint_as_float(h.z), __uint_as_float(h.w))
                 : make_float2(__uint_as_float(h.x), __uint_as_float(h.y));
}
// Raw logits e0 .. e0+7 of a row of V elements, -inf past the end (the
// row's ragged end, read element by element).
template <typename T>
__device__ __forceinline__ Raw8<T> raw8_ragged(const T* row, int e0, int V) {
  float x[8];
  load8<T>(row, e0, V, x);
  Raw8<T> r;
  if constexpr (sizeof(T) == 2) {
    uint32_t w[4];
#pragma unroll
    for (int j = 0; j < 4; ++j)
      w[j] = (__float_as_uint(x[2 * j]) >> 16) | (__float_as_uint(x[2 * j + 1]) & 0xffff0000u);
    r.v[0] = make_uint4(w[0], w[1], w[2], w[3]);
  } else {
    r.v[0] = make_uint4(__float_as_uint(x[0]), __float_as_uint(x[1]), __float_as_uint(x[2]),
                        __float_as_uint(x[3]));
    r.v[1] = make_uint4(__float_as_uint(x[4]), __float_as_uint(x[5]), __float_as_uint(x[6]),
                        __float_as_uint(x[7]));
  }
  return r;
}
// The streaming pass's form of a probability: 2^(x c - M) k with the row's
// integral shift M and k = 2^(M - Lt) as one float (k < 0 for the draft
// row, so that p - q is one add). Relative error about 1e-7, ample for the
// residual mass; the kept weights are formed again in fp64.
struct PairCoef {
  float chi, clo, nM, k;
};
__device__ __forceinline__ PairCoef pair_coef(double Lt, float m, const Scale& s, bool negate) {
  const ProbCoef c = make_coef(Lt, m, s);
  return PairCoef{c.chi, c.clo, c.nM, negate ? -c.khi : c.khi};
}
__device__ __forceinline__ float2 prob2s(float2 x, const PairCoef& k) {
  float2 t = __ffma2_rn(x, make_float2(k.chi, k.chi), make_float2(k.nM, k.nM));
  t = __ffma2_rn(x, make_float2(k.clo, k.clo), t);
  return __fmul2_rn(make_float2(ex2(t.x), ex2(t.y)), make_float2(k.k, k.k));
}
// The weights w = max(0, p - q) of an element pair (p alone when there is no
// draft row), and *pq = p + q. The fp32 w is within kSlack (p + q) of the
// exact weight: w + kSlack (p + q) bounds it from above, w - kSlack (p + q)
// from below.
__device__ __forceinline__ float2 pair_weights(float2 xp, float2 xq, bool hq, const PairCoef& kp,
                                               const PairCoef& kqn, float2* pq) {
  const float2 p = prob2s(xp, kp);
  const float2 qn = hq ? prob2s(xq, kqn) : make_float2(0.f, 0.f);  // -q
  const float2 d = __fadd2_rn(p, qn);
  *pq = __ffma2_rn(qn, make_float2(-1.0f, -1.0f), p);
  return make_float2(fmaxf(d.x, 0.0f), fmaxf(d.y, 0.0f));
}
__device__ __forceinline__ float2 loosened(float2 w, float2 pq, float slack) {
  return __ffma2_rn(make_float2(slack, slack), pq, w);
}

// The rare paths of the streaming loop are out of line, so that the loop
// keeps its registers: appending a lane's candidates, and flushing a warp's
// buffer into its list.
//
// Candidates among the lane's 8 elements at e0 .. e0+7 (w > 0 and
// w + kSlack (p + q) >= thr), their weights formed again from the raw logits
// as the streaming loop forms them, appended to the warp's buffer through
// its shared counter. Called by single lanes.
template <typename T>
__device__ __noinline__ void append_candidates(int* buf, int* cnt, Raw8<T> rp, Raw8<T> rq,
                                               bool hq, PairCoef kp, PairCoef kqn, float thr,
                                               int e0) {
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    float2 pq;
    const float2 w = pair_weights(pair_of(rp, j), pair_of(rq, j), hq, kp, kqn, &pq);
    const float2 hi = loosened(w, pq, kSlack);
    if (w.x > 0.0f && hi.x >= thr) buf[atomicAdd(cnt, 1)] = e0 + 2 * j;
    if (w.y > 0.0f && hi.y >= thr) buf[atomicAdd(cnt, 1)] = e0 + 2 * j + 1;
  }
}

// The buffer's count entries, 32 at a time: each entry's weight formed again
// in fp64 from its two logits, those at or above thr sorted and merged into
// the list; then the list's n-th entry raises the CTA's threshold. Returns
// the new list. Called by the whole warp.
template <typename T>
__device__ __noinline__ Top<float> flush_buffer(Top<float> list, const int* buf, int count,
                                                float thr, const T* prow, const T* qrow,
                                                const double* Lt_sh, float Tb, int n,
                                                unsigned* thr_sh, int lane) {
  const PairRow pr{Lt_sh[0], qrow ? Lt_sh[1] : 0.0, make_scale(Tb).d, qrow != nullptr};
  for (int c = 0; c < count; c += 32) {
    Top<float> x = top_empty<float>();
    if (c + lane < count) {
      const int v = buf[c + lane];
      const float key = (float)exact_weight<T>(prow, qrow, v, pr);
      if (key > 0.0f && key >= thr) x = Top<float>{key, v};
    }
    if (__any_sync(0xffffffffu, x.w > 0.0f)) {
      top_sort(x, lane);
      list = top_merged(list, x, lane);
    }
  }
  const float nth = __shfl_sync(0xffffffffu, list.w, n - 1);
  if (lane == 0 && nth > 0.0f) atomicMax(thr_sh, __float_as_uint(nth));
  __syncwarp();
  return list;
}

// The lists of the CTA's kPairWarps warps (each sorted, in lw/li) merged by
// a tree of pairwise merges; warp 0 ends with the merged list in e. Called
// by every thread of the CTA after the lists are in shared memory.
template <typename W>
__device__ __forceinline__ void merge_tree(Top<W>& e, W (*lw)[32], int (*li)[32], int warp,
                                           int lane) {
#pragma unroll
  for (int d = 1; d < kPairWarps; d <<= 1) {
    if ((warp & (2 * d - 1)) == 0) {
      e = top_merged(e, Top<W>{lw[warp + d][lane], li[warp + d][lane]}, lane);
      lw[warp][lane] = e.w;
      li[warp][lane] = e.i;
    }
    __syncthreads();
  }
}

// A warp's ring: kPairStages stages, each holding kPairGroup tiles of both
// rows, filled by 1-D bulk copies that complete on the stage's mbarrier.
constexpr int kPairStages = 2;
constexpr int kStageRowBytes = 1024;  // kPairGroup tiles of one row, either dtype
static_assert(kPairGroup<__nv_bfloat16> * kResTile * 2 == kStageRowBytes, "bf16 stage");
static_assert(kPairGroup<float> * kResTile * 4 == kStageRowBytes, "fp32 stage");
constexpr int kRingBytes = kPairWarps * kPairStages * 2 * kStageRowBytes;

template <typename T>
__global__ void __launch_bounds__(kPairWarps * 32, 4) outcome_pair_kernel(OutcomeArgs A) {
  pdl_begin();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int b = blockIdx.y, k = blockIdx.x, K = A.K, V = A.V, n = A.n_top;
  // the warps' rings (dynamic shared memory, kRingBytes)
  extern __shared__ __align__(128) unsigned char s_dyn_ring[];
  auto s_ring = reinterpret_cast<unsigned char(*)[kPairStages][2][kStageRowBytes]>(s_dyn_ring);
  __shared__ __align__(8) uint64_t s_bar[kPairWarps][kPairStages];
  __shared__ double s_Lt[2];
  __shared__ float s_m[2];
  __shared__ int s_ok[2];
  __shared__ double s_z[kPairWarps];
  __shared__ unsigned s_thr;  // bits of the shared threshold (a weight >= 0)
  __shared__ int s_late;      // a bounded wait ran out
  __shared__ int s_buf[kPairWarps][kBufCap];
  __shared__ int s_cnt[kPairWarps];  // entries in each warp's buffer
  __shared__ float s_lw[kPairWarps][32];
  __shared__ int s_li[kPairWarps][32];
  const float Tb = A.temperature[b];
  if (!temp_valid(Tb) || Tb == 0.0f) return;  // handled by the final kernel
  const Scale sc = make_scale(Tb);
  const long long row0 = (long long)b * (2 * K + 1);
  if (warp < 2 && (warp == 0 || k < K)) {
    const long long r = warp == 0 ? row0 + k : row0 + K + 1 + k;
    const RowFinal f = combine_row(A.part + (size_t)r * A.ntiles, A.ntiles, false, sc.hi, lane);
    if (lane == 0) {
      s_Lt[warp] = f.M + f.L;
      s_m[warp] = f.m;
      s_ok[warp] = f.ok;
      A.lt[r] = f.ok ? f.M + f.L : dnan();  // for the final kernel
    }
  }
  if (threadIdx.x == 0) {
    s_thr = 0u;
    s_late = 0;
  }
  __syncthreads();
  if (!s_ok[0] || (k < K && !s_ok[1])) return;  // reported by the final kernel
  const T* prow = row_ptr<T>(A.tgt, A.ld_tgt, (long long)b * (K + 1) + k);
  const T* qrow = k < K ? row_ptr<T>(A.drf, A.ld_drf, (long long)b * K + k) : nullptr;
  const bool hq = qrow != nullptr;
  const PairCoef kp = pair_coef(s_Lt[0], s_m[0], sc, false);
  const PairCoef kqn = hq ? pair_coef(s_Lt[1], s_m[1], sc, true) : PairCoef{0.f, 0.f, 0.f, 0.f};
  constexpr int G = kPairGroup<T>;
  const int nrt = residual_tiles(V);
  // This warp's steps: tiles [tb, tb + G) with tb = (i * kPairWarps + warp) * G.
  const int nsteps = max(0, (nrt - warp * G + kPairWarps * G - 1) / (kPairWarps * G));
  uint64_t* bars = s_bar[warp];
  if (lane == 0) {
    for (int st = 0; st < kPairStages; ++st) mbar_init(&bars[st], 1);
    fence_barrier_init();
    s_cnt[warp] = 0;
  }
  __syncwarp();
  // Row pairs streamed last by the statistics pass are still in L2; the
  // others' lines go first when L2 needs room.
  const bool hint = k >= A.late_pos;
  const uint64_t pol = l2_evict_first();
  auto issue = [&](int i, int st) {
    if (lane == 0) {
      const int e_start = (i * kPairWarps + warp) * G * kResTile;
      const int nel = min(G * kResTile, V - e_start);
      const uint32_t bytes = ((uint32_t)nel * sizeof(T)) & ~15u;
      fence_proxy_async_smem();  // the warp's reads of this stage come first
      mbar_arrive_expect_tx(&bars[st], hq ? 2 * bytes : bytes);
      if (bytes) {
        const T* src[2] = {prow + e_start, qrow + e_start};
        for (int r = 0; r < (hq ? 2 : 1); ++r) {
          if (hint)
            bulk_g2s_hint(s_ring[warp][st][r], src[r], bytes, &bars[st], pol);
          else
            bulk_g2s(s_ring[warp][st][r], src[r], bytes, &bars[st]);
        }
      }
    }
  };
  for (int i = 0; i < kPairStages && i < nsteps; ++i) issue(i, i);

  const volatile unsigned* thr_sh = &s_thr;
  int* buf = s_buf[warp];
  double z = 0.0;
  Top<float> list = top_empty<float>();
  float thr = 0.0f;
  // The lane's 8 raw logits of each row in tile u of step i (stage st).
  auto tile_raw = [&](int i, int u, int st, Raw8<T>& rp, Raw8<T>& rq) {
    const int t = (i * kPairWarps + warp) * G + u, e0 = t * kResTile + lane * 8;
    if (t < nrt && e0 + 8 <= V) {  // staged: 16 bytes per row (bf16), 32 (fp32)
      rp = *(reinterpret_cast<const Raw8<T>*>(s_ring[warp][st][0]) + u * 32 + lane);
      rq = hq ? *(reinterpret_cast<const Raw8<T>*>(s_ring[warp][st][1]) + u * 32 + lane) : rp;
    } else {  // the row's ragged end, or past it: plain loads
      rp = raw8_ragged<T>(prow, t < nrt ? e0 : V, V);
      rq = hq ? raw8_ragged<T>(qrow, t < nrt ? e0 : V, V) : rp;
    }
  };
  // Sum of the lane's 8 weights and the largest of them loosened by
  // slack (p + q) (upward: kSlack; downward: -kSlack).
  auto tile_weights = [&](const Raw8<T>& rp, const Raw8<T>& rq, float slack, float& sum,
                          float& top) {
    float2 zs = make_float2(0.f, 0.f), hm = make_float2(-INFINITY, -INFINITY);
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      float2 pq;
      const float2 w = pair_weights(pair_of(rp, j), pair_of(rq, j), hq, kp, kqn, &pq);
      zs = __fadd2_rn(zs, w);
      const float2 h = loosened(w, pq, slack);
      hm = make_float2(fmaxf(hm.x, h.x), fmaxf(hm.y, h.y));
    }
    sum = zs.x + zs.y;
    top = fmaxf(hm.x, hm.y);
  };
  // Starting threshold: the n-th largest of the lanes' largest lower bounds
  // w - kSlack (p + q) in every warp's first step: the lanes' tokens are
  // distinct, so it is at most the n-th largest weight of the row pair.
  if (n > 0) {
    float best = 0.0f;
    if (nsteps > 0 && __all_sync(0xffffffffu, mbar_wait_bounded(&bars[0], 0u, kWaitLimitNs))) {
#pragma unroll
      for (int u = 0; u < G; ++u) {
        Raw8<T> rp, rq;
        tile_raw(0, u, 0, rp, rq);
        float sum, low;
        tile_weights(rp, rq, -kSlack, sum, low);
        best = fmaxf(best, low);
      }
    }
    Top<float> e{best, lane};
    top_sort(e, lane);
    s_lw[warp][lane] = e.w;
    s_li[warp][lane] = lane;
    __syncthreads();
    merge_tree(e, s_lw, s_li, warp, lane);
    if (warp == 0) {
      const float nth = __shfl_sync(0xffffffffu, e.w, n - 1);
      if (lane == 0 && nth > 0.0f) s_thr = __float_as_uint(nth);
    }
    __syncthreads();
  }
  uint32_t phase = 0;  // bit st: parity of stage st's next completion
  int* cnt = &s_cnt[warp];
  int i = 0;
  for (; i < nsteps; ++i) {
    const int st = i % kPairStages;
    if (__any_sync(0xffffffffu, !mbar_wait_bounded(&bars[st], (phase >> st) & 1u, kWaitLimitNs)))
      break;
    phase ^= 1u << st;
    if (n > 0) thr = fmaxf(thr, __uint_as_float(*thr_sh));
    float step_top = -INFINITY, step_sum = 0.0f;
#pragma unroll
    for (int u = 0; u < G; ++u) {
      Raw8<T> rp, rq;
      tile_raw(i, u, st, rp, rq);
      float lsum, top;
      tile_weights(rp, rq, kSlack, lsum, top);
      z += (double)lsum;
      step_top = fmaxf(step_top, top);
      step_sum += lsum;
    }
    // candidates: w > 0 and w + kSlack (p + q) >= thr; rare once the
    // threshold has risen, so a lane that has some appends them alone
    // (reading the step's staged logits again)
    if (n > 0 && step_top >= thr && step_sum > 0.0f) {
      for (int u = 0; u < G; ++u) {
        const int e0 = ((i * kPairWarps + warp) * G + u) * kResTile + lane * 8;
        Raw8<T> rp, rq;
        tile_raw(i, u, st, rp, rq);
        append_candidates<T>(buf, cnt, rp, rq, hq, kp, kqn, thr, e0);
      }
    }
    __syncwarp();  // every lane is done with stage st and with its appends
    if (n > 0) {
      const int c = *reinterpret_cast<volatile int*>(cnt);
      if (c > kFlushAt) {
        list = flush_buffer<T>(list, buf, c, thr, prow, qrow, s_Lt, Tb, n, &s_thr, lane);
        if (lane == 0) *cnt = 0;
        __syncwarp();
      }
    }
    if (i + kPairStages < nsteps) issue(i + kPairStages, st);
  }
  if (i < nsteps) {  // a wait ran out: record it, let the copies in flight land
    if (lane == 0) {
      set_status(A.status, SPEC_ETIMEOUT);
      s_late = 1;
    }
    for (int j = i; j < nsteps && j < i + kPairStages; ++j) {
      const int st = j % kPairStages;
      mbar_wait_bounded(&bars[st], (phase >> st) & 1u, kWaitLimitNs);
      phase ^= 1u << st;
    }
  } else if (n > 0) {
    const int c = *reinterpret_cast<volatile int*>(cnt);
    if (c > 0) list = flush_buffer<T>(list, buf, c, thr, prow, qrow, s_Lt, Tb, n, &s_thr, lane);
  }
  z = warp_sum_d(z);
  if (lane == 0) s_z[warp] = z;
  s_lw[warp][lane] = list.w;
  s_li[warp][lane] = list.i;
  __syncthreads();
  if (n > 0) merge_tree(list, s_lw, s_li, warp, lane);
  if (warp != 0 || s_late) return;
  const size_t slot = (size_t)b * (K + 1) + k;
  if (lane < n) {
    const bool has = list.w > 0.0f;
    const PairRow pr{s_Lt[0], k < K ? s_Lt[1] : 0.0, sc.d, k < K};
    A.cw[slot * n + lane] = has ? exact_weight<T>(prow, qrow, list.i, pr) : -1.0;
    A.cv[slot * n + lane] = has ? list.i : 0;
  }
  if (lane == 0) {
    double zt = 0.0;
    for (int w2 = 0; w2 < kPairWarps; ++w2) zt += s_z[w2];
    A.zk[slot] = zt;
  }
}

// ---------------------------------------------------------------------------
// One CTA per sequence: beta, the length law and the joint top list, ranked
// by the fp64 joint probabilities P(a = k) w / Z_k.
// ---------------------------------------------------------------------------
constexpr int kFinThreads = 256;

template <typename T>
__global__ void __launch_bounds__(kFinThreads) outcome_final_kernel(OutcomeArgs A) {
  pdl_begin();
  const int b = blockIdx.x, K = A.K, n = A.n_top, V = A.V;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  constexpr int kFinWarps = kFinThreads / 32;
  static_assert(kFinWarps == kPairWarps, "the merge tree spans kPairWarps lists");
  extern __shared__ double s_dyn[];  // [2K+1] log2-partitions, then [K+1] p_len
  double* s_Lt = s_dyn;
  double* s_pl = s_dyn + 2 * K + 1;
  int* s_amax = reinterpret_cast<int*>(s_pl + K + 1);  // [K+1]
  __shared__ double s_jw[kFinWarps][32];
  __shared__ int s_ji[kFinWarps][32];
  __shared__ int s_bad;
  const float Tb = A.temperature[b];
  const bool greedy = (Tb == 0.0f);
  if (threadIdx.x == 0) s_bad = temp_valid(Tb) ? 0 : 1;
  __syncthreads();
  const Scale sc = greedy || s_bad ? Scale{0.f, 0.f, 0.0} : make_scale(Tb);
  const long long row0 = (long long)b * (2 * K + 1);
  if (!s_bad) {
    if (greedy) {  // the argmax of each target row
      for (int r = warp; r <= K; r += kFinWarps) {
        const RowFinal f =
            combine_row(A.part + (size_t)(row0 + r) * A.ntiles, A.ntiles, true, 0.0f, lane);
        if (lane == 0) {
          if (!f.ok) atomicOr(&s_bad, 1);
          s_amax[r] = f.amax;
        }
      }
    } else {  // the pair kernel's log2-partitions (NaN: no finite statistics)
      for (int r = threadIdx.x; r < 2 * K + 1; r += kFinThreads) {
        const double lt = A.lt[row0 + r];
        if (isnan(lt)) atomicOr(&s_bad, 1);
        s_Lt[r] = lt;
      }
    }
  }
  auto fail = [&]() {  // every thread of the CTA
    if (threadIdx.x == 0) set_status(A.status, SPEC_EDEVICE);
    for (int j = threadIdx.x; j <= K; j += kFinThreads) {
      A.p_len[(size_t)b * (K + 1) + j] = dnan();
      if (A.mass) A.mass[(size_t)b * (K + 1) + j] = dnan();
      if (A.beta && j < K) A.beta[(size_t)b * K + j] = dnan();
    }
    for (int i = threadIdx.x; i < n; i += kFinThreads) {
      A.top_len[(size_t)b * n + i] = -1;
      A.top_tok[(size_t)b * n + i] = -1;
      A.top_prob[(size_t)b * n + i] = 0.0;
    }
  };
  __syncthreads();
  if (s_bad) {
    fail();
    return;
  }
  // beta_j, then the length law (one thread: a running product).
  double* s_beta = s_pl;  // beta first, then overwritten by p_len in place
  const int32_t* drafts = A.draft_tok + (size_t)b * K;
  for (int j = threadIdx.x; j < K; j += kFinThreads) {
    const int x = drafts[j];
    double bj;
    if (x < 0 || x >= V) {
      bj = dnan();
      atomicOr(&s_bad, 1);
    } else if (greedy) {
      bj = (x == s_amax[j]) ? 1.0 : 0.0;
    } else {
      const double lt = (double)load_elem(row_ptr<T>(A.tgt, A.ld_tgt, (long long)b * (K + 1) + j) + x);
      const double ld = (double)load_elem(row_ptr<T>(A.drf, A.ld_drf, (long long)b * K + j) + x);
      const double lp = lt * sc.d - s_Lt[j], lq = ld * sc.d - s_Lt[K + 1 + j];
      bj = fmin(1.0, exp2(lp - lq));
    }
    s_beta[j] = bj;
    if (A.beta) A.beta[(size_t)b * K + j] = bj;
  }
  __syncthreads();
  if (s_bad) {  // a draft id outside [0, V)
    fail();
    return;
  }
  if (threadIdx.x == 0) {
    double run = 1.0;
    for (int j = 0; j < K; ++j) {
      const double bj = s_beta[j];
      s_beta[j] = run * (1.0 - bj);  // p_len[j]
      run *= bj;
    }
    s_pl[K] = run;
  }
  __syncthreads();
  for (int j = threadIdx.x; j <= K; j += kFinThreads) {
    A.p_len[(size_t)b * (K + 1) + j] = s_pl[j];
    if (A.mass)
      A.mass[(size_t)b * (K + 1) + j] = (greedy || j == K) ? 1.0 : A.zk[(size_t)b * (K + 1) + j];
  }
  if (n == 0) return;
  // Joint candidates: each warp sorts lists of 32 (one acceptance length k,
  // or for a greedy check 32 lengths with their argmax tokens) and merges
  // them into its own list; the warps' lists then meet in a merge tree. The
  // index k * V + v orders equal probabilities.
  Top<double> e = top_empty<double>();
  if (greedy) {
    for (int k0 = warp * 32; k0 <= K; k0 += kFinWarps * 32) {
      const int k = k0 + lane;
      Top<double> c = top_empty<double>();
      if (k <= K && s_pl[k] > 0.0) c = Top<double>{s_pl[k], k * V + s_amax[k]};
      if (__any_sync(0xffffffffu, c.w > 0.0)) {
        top_sort(c, lane);
        e = top_merged(e, c, lane);
      }
    }
  } else {
    for (int k = warp; k <= K; k += kFinWarps) {
      const size_t slot = (size_t)b * (K + 1) + k;
      const double zt = A.zk[slot], pl = s_pl[k];
      const double w = lane < n ? A.cw[slot * n + lane] : -1.0;
      const int v = lane < n ? A.cv[slot * n + lane] : 0;
      Top<double> c = top_empty<double>();
      if (w > 0.0 && zt > 0.0 && pl > 0.0) c = Top<double>{pl * w / zt, k * V + v};
      if (__any_sync(0xffffffffu, c.w > 0.0)) {
        top_sort(c, lane);
        e = top_merged(e, c, lane);
      }
    }
  }
  s_jw[warp][lane] = e.w;
  s_ji[warp][lane] = e.i;
  __syncthreads();
  merge_tree(e, s_jw, s_ji, warp, lane);
  if (warp == 0 && lane < n) {
    const bool has = e.w > 0.0;
    A.top_len[(size_t)b * n + lane] = has ? e.i / V : -1;
    A.top_tok[(size_t)b * n + lane] = has ? e.i % V : -1;
    A.top_prob[(size_t)b * n + lane] = has ? e.w : 0.0;
  }
}

template <typename T>
static cudaError_t launch_outcome_t(const OutcomeArgs& a, cudaStream_t st) {
  cudaError_t e = reserve_dyn_smem(outcome_pair_kernel<T>, (size_t)kRingBytes);
  if (e != cudaSuccess) return e;
  e = launch_pdl(outcome_pair_kernel<T>, dim3(a.K + 1, a.B), dim3(kPairWarps * 32), kRingBytes,
                 st, a);
  if (e != cudaSuccess) return e;
  const size_t smem = (size_t)(2 * a.K + 1 + a.K + 1) * sizeof(double) + (a.K + 1) * sizeof(int);
  return launch_pdl(outcome_final_kernel<T>, dim3(a.B), dim3(kFinThreads), smem, st, a);
}

cudaError_t launch_outcome(int dtype, const OutcomeArgs& a, cudaStream_t st) {
  return dtype == SPEC_BF16 ? launch_outcome_t<__nv_bfloat16>(a, st)
                            : launch_outcome_t<float>(a, st);
}

}  // namespace specv
