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
// Three launches: the row statistics of the chain rows; one CTA per
// (sequence, position k) that streams the row pair once for the residual mass
// Z_k and the exact n largest weights max(0, p_k - q_k) (sorted lists held one
// entry per lane, single candidates inserted, whole lists combined by bitonic
// merges); one CTA per sequence for beta, the length law and the merge of the
// K+1 lists by P(a = k) w / Z_k.
#include "draw.cuh"

namespace specv {

constexpr int kMaxTop = SPEC_MAX_TOP;
static_assert(kMaxTop <= 32, "a top list is held one entry per lane");

// Candidate order: larger weight first, then the smaller index.
__device__ __forceinline__ bool beats(float wa, int ia, float wb, int ib) {
  return wa > wb || (wa == wb && ia < ib);
}

// Sorted list of the 32 best candidates, entry i in lane i (empty: w = -1).
struct TopList {
  float w;
  int i;
};
__device__ __forceinline__ TopList top_empty() { return TopList{-1.0f, 0x7fffffff}; }

// One compare-exchange step with the lane at distance j: the lane keeps the
// better of the pair if keep_better, else the worse.
__device__ __forceinline__ void top_cx(TopList& e, int j, bool keep_better) {
  const float ow = __shfl_xor_sync(0xffffffffu, e.w, j);
  const int oi = __shfl_xor_sync(0xffffffffu, e.i, j);
  const bool take = keep_better ? beats(ow, oi, e.w, e.i) : beats(e.w, e.i, ow, oi);
  if (take) { e.w = ow; e.i = oi; }
}

// a <- the 32 best of a and b, both sorted descending: the better of a[l] and
// b[31 - l] form a bitonic sequence holding them, sorted by a bitonic merge.
__device__ __noinline__ TopList top_merged(TopList a, TopList b, int lane) {
  const float bw = __shfl_sync(0xffffffffu, b.w, 31 - lane);
  const int bi = __shfl_sync(0xffffffffu, b.i, 31 - lane);
  if (beats(bw, bi, a.w, a.i)) { a.w = bw; a.i = bi; }
#pragma unroll
  for (int j = 16; j > 0; j >>= 1) top_cx(a, j, (lane & j) == 0);
  return a;
}

// Insert (w, i), the same in every lane, into the sorted list (kept: n).
__device__ __forceinline__ void top_insert(TopList& e, float w, int i, int n, int lane) {
  const unsigned ahead = __ballot_sync(0xffffffffu, lane < n && beats(e.w, e.i, w, i));
  const int pos = __popc(ahead);
  if (pos >= n) return;
  const float uw = __shfl_up_sync(0xffffffffu, e.w, 1);
  const int ui = __shfl_up_sync(0xffffffffu, e.i, 1);
  if (lane > pos && lane < n) { e.w = uw; e.i = ui; }
  if (lane == pos) { e.w = w; e.i = i; }
}

// Offer one candidate per lane (w <= 0 is never an outcome): the ones that
// beat entry n-1, the last kept (cached in (tw, ti) in every lane), go in one
// at a time -- rare once the list has filled: about n ln(N / n) of N.
__device__ __forceinline__ void top_offer(TopList& e, float& tw, int& ti, float w, int i, int n,
                                          int lane) {
  bool want = w > 0.0f && beats(w, i, tw, ti);
  unsigned m = __ballot_sync(0xffffffffu, want);
  while (m) {
    const int src = __ffs(m) - 1;
    const float cw = __shfl_sync(0xffffffffu, w, src);
    const int ci = __shfl_sync(0xffffffffu, i, src);
    top_insert(e, cw, ci, n, lane);
    tw = __shfl_sync(0xffffffffu, e.w, n - 1);
    ti = __shfl_sync(0xffffffffu, e.i, n - 1);
    want = want && lane != src && beats(w, i, tw, ti);
    m = __ballot_sync(0xffffffffu, want);
  }
}

// ---------------------------------------------------------------------------
// One CTA of kPairWarps warps per (sequence b, position k): residual mass and
// best weights. Each warp keeps its own list, so few warps per row pair keep
// the number of insertions (about n ln(N / n) per list) low.
// ---------------------------------------------------------------------------
constexpr int kPairWarps = 4;

template <typename T>
__global__ void __launch_bounds__(kPairWarps * 32, 6) outcome_pair_kernel(OutcomeArgs A) {
  pdl_begin();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int b = blockIdx.y, k = blockIdx.x, K = A.K, V = A.V, n = A.n_top;
  __shared__ double s_Lt[2];
  __shared__ float s_m[2];
  __shared__ int s_ok[2];
  __shared__ double s_z[kPairWarps];
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
    }
  }
  __syncthreads();
  if (!s_ok[0] || (k < K && !s_ok[1])) return;  // reported by the final kernel
  const T* prow = row_ptr<T>(A.tgt, A.ld_tgt, (long long)b * (K + 1) + k);
  const T* qrow = k < K ? row_ptr<T>(A.drf, A.ld_drf, (long long)b * K + k) : nullptr;
  const ProbCoef kp = make_coef(s_Lt[0], s_m[0], sc);
  const ProbCoef kq = k < K ? make_coef(s_Lt[1], s_m[1], sc) : make_coef(0.0, 0.0f, sc);
  const int nrt = residual_tiles(V);
  double z = 0.0;
  TopList e = top_empty();
  float tw = -1.0f;  // entry n-1 of the list
  int ti = 0x7fffffff;
  constexpr int G = kResGroup<T>;
  const bool hq = qrow != nullptr;
  for (int tb = warp * G; tb < nrt; tb += kPairWarps * G) {
    Raw8<T> rp[G], rq[G];
    bool full[G];
#pragma unroll
    for (int u = 0; u < G; ++u) {  // every load of the group before any use
      const int e0 = (tb + u) * kResTile + lane * 8;
      full[u] = tb + u < nrt && e0 + 8 <= V;
      rp[u] = raw8(prow, e0, full[u]);
      rq[u] = raw8(hq ? qrow : prow, e0, full[u] && hq);
    }
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
        for (int q = 0; q < 8; ++q) w[q] = 0.0f;
      }
      z += lane_sum8(w);
      if (n > 0) {
#pragma unroll
        for (int q = 0; q < 8; ++q) top_offer(e, tw, ti, w[q], e0 + q, n, lane);
      }
    }
  }
  z = warp_sum_d(z);
  if (lane == 0) s_z[warp] = z;
  s_lw[warp][lane] = e.w;
  s_li[warp][lane] = e.i;
  __syncthreads();
  if (warp != 0) return;
  if (n > 0)
    for (int w2 = 1; w2 < kPairWarps; ++w2)
      e = top_merged(e, TopList{s_lw[w2][lane], s_li[w2][lane]}, lane);
  const size_t slot = (size_t)b * (K + 1) + k;
  if (lane < n) {
    A.cw[slot * n + lane] = e.w;
    A.cv[slot * n + lane] = e.i;
  }
  if (lane == 0) {
    double zt = 0.0;
    for (int w2 = 0; w2 < kPairWarps; ++w2) zt += s_z[w2];
    A.zk[slot] = zt;
  }
}

// ---------------------------------------------------------------------------
// One CTA per sequence: beta, the length law and the joint top list.
// ---------------------------------------------------------------------------
constexpr int kFinThreads = 256;

template <typename T>
__global__ void __launch_bounds__(kFinThreads) outcome_final_kernel(OutcomeArgs A) {
  pdl_begin();
  const int b = blockIdx.x, K = A.K, n = A.n_top, V = A.V;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  extern __shared__ double s_dyn[];  // [2K+1] log2-partitions, then [K+1] p_len
  double* s_Lt = s_dyn;
  double* s_pl = s_dyn + 2 * K + 1;
  int* s_amax = reinterpret_cast<int*>(s_pl + K + 1);  // [K+1]
  __shared__ int s_bad;
  const float Tb = A.temperature[b];
  const bool greedy = (Tb == 0.0f);
  if (threadIdx.x == 0) s_bad = temp_valid(Tb) ? 0 : 1;
  __syncthreads();
  const Scale sc = greedy || s_bad ? Scale{0.f, 0.f, 0.0} : make_scale(Tb);
  const long long row0 = (long long)b * (2 * K + 1);
  if (!s_bad) {
    for (int r = warp; r < 2 * K + 1; r += kFinThreads / 32) {
      if (greedy && r > K) continue;
      const RowFinal f =
          combine_row(A.part + (size_t)(row0 + r) * A.ntiles, A.ntiles, greedy, sc.hi, lane);
      if (lane == 0) {
        if (!f.ok) atomicOr(&s_bad, 1);
        s_Lt[r] = f.M + f.L;
        if (r <= K) s_amax[r] = f.amax;
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
  if (warp != 0 || n == 0) return;
  // Joint candidates P(a = k) w / Z_k, offered 32 at a time; index k * V + v
  // orders equal probabilities.
  TopList e = top_empty();
  float tw = -1.0f;
  int ti = 0x7fffffff;
  if (greedy) {
    for (int k0 = 0; k0 <= K; k0 += 32) {
      const int k = k0 + lane;
      const float pj = k <= K ? (float)s_pl[k] : 0.0f;
      top_offer(e, tw, ti, pj, k <= K ? k * V + s_amax[k] : 0x7fffffff, n, lane);
    }
  } else {
    for (int k = 0; k <= K; ++k) {  // each list is sorted; scaling keeps it so
      const size_t slot = (size_t)b * (K + 1) + k;
      const double zt = A.zk[slot], pl = s_pl[k];
      const float w = lane < n ? A.cw[slot * n + lane] : -1.0f;
      const int v = lane < n ? A.cv[slot * n + lane] : 0;
      const bool has = w > 0.0f && zt > 0.0 && pl > 0.0;
      const TopList c = has ? TopList{(float)(pl * (double)w / zt), k * V + v} : top_empty();
      if (__ballot_sync(0xffffffffu, has)) e = top_merged(e, c, lane);
    }
  }
  if (lane < n) {
    const bool has = e.w > 0.0f;
    A.top_len[(size_t)b * n + lane] = has ? e.i / V : -1;
    A.top_tok[(size_t)b * n + lane] = has ? e.i % V : -1;
    A.top_prob[(size_t)b * n + lane] = has ? (double)e.w : 0.0;
  }
}

template <typename T>
static cudaError_t launch_outcome_t(const OutcomeArgs& a, cudaStream_t st) {
  cudaError_t e = launch_pdl(outcome_pair_kernel<T>, dim3(a.K + 1, a.B), dim3(kPairWarps * 32), 0,
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
