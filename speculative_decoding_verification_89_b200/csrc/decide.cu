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
// One launch per check: a thread-block cluster of kCluster CTAs per sequence.
// The CTAs combine the tile partials of the sequence's rows (a warp per row)
// into the leader CTA's shared memory (distributed shared memory), meet at a
// cluster barrier, each run the accept test on all positions (a lane per
// position, ballot for the first rejection), take groups of residual tiles of
// the row pair from a counter in the leader (so the CTAs that share an SM with
// another take fewer) and write their tile sums into the leader, meet again, and the
// leader prefixes the tile sums, finds the tile holding u' * Z, rescans that
// one tile and writes the outputs. No spinning and no second launch; the
// variant that also plans a paged commit (chain_decide_commit_kernel, at the
// end of this file) adds one atomic ticket per sequence.
#include "draw.cuh"
#include "rowmath.cuh"
#include "commit.cuh"

namespace specv {

constexpr int kMaxRows = 2 * SPEC_MAX_K + 1;
constexpr int kRowWarps = kDecWarps - 1;     // the last warp of a CTA serves the accept test

// ---------------------------------------------------------------------------
// Row statistics and the accept test
// ---------------------------------------------------------------------------

// Statistics of a sequence's rows, gathered in the leader CTA.
struct SeqShared {
  double M[kMaxRows], L[kMaxRows];
  float m[kMaxRows];
  int amax[kMaxRows];
  int ok[kMaxRows];
};

// Split cluster barrier: every CTA arrives once it runs; a thread waits (once)
// before its first access to another CTA's shared memory.
__device__ __forceinline__ void cluster_arrive_relaxed() {
  asm volatile("barrier.cluster.arrive.relaxed;" ::: "memory");
}
__device__ __forceinline__ void cluster_wait() {
  asm volatile("barrier.cluster.wait;" ::: "memory");
}

// Combine the tile partials of a sequence's rows (a warp per row, over the
// row warps of all CTAs of the cluster) into the leader's SeqShared (lsh,
// distributed shared memory) and the RowFinal array. Completes the start
// barrier of the cluster in every thread: the first row's partials are read
// before the wait.
template <typename Want>
__device__ void cluster_rows(SeqShared* lsh, unsigned rank, const Partial* part, int ntiles,
                             int row0, int nrows, Want want, bool greedy, float chi,
                             RowFinal* fin) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  bool waited = false;
  if (warp < kRowWarps) {
    for (int r = (int)rank * kRowWarps + warp; r < nrows; r += kCluster * kRowWarps) {
      RowFinal f{0.0, 0.0, 0.f, -1, 1, 0};
      if (want(r)) f = combine_row(part + (size_t)(row0 + r) * ntiles, ntiles, greedy, chi, lane);
      if (!waited) {
        cluster_wait();
        waited = true;
      }
      if (lane == 0) {
        if (want(r)) fin[row0 + r] = f;
        lsh->m[r] = f.m;
        lsh->M[r] = f.M;
        lsh->L[r] = f.L;
        lsh->amax[r] = f.amax;
        lsh->ok[r] = f.ok;
      }
    }
  }
  if (!waited) cluster_wait();
}


// Logits of the drafted tokens and the Philox uniforms of the first 32
// positions, fetched by the accept warp while the other warps combine the
// rows.
struct AcceptPre {
  int x;         // draft id of position lane (or -1 past n)
  float lt, ld;  // target / draft logit at x
  float ua, ud;  // accept and draw uniforms of position pos0 + lane
};
template <typename T, typename TP, typename DP>
__device__ __forceinline__ AcceptPre accept_prefetch(int n, int V, bool greedy,
                                                     const int32_t* drafts, TP tp, DP dp,
                                                     const DecideCommon& c, int b, int pos0,
                                                     int stage) {
  const int lane = threadIdx.x & 31;
  AcceptPre a{-1, 0.f, 0.f, 0.f, 0.f};
  if (lane < n) {
    a.x = drafts[lane];
    if (!greedy && a.x >= 0 && a.x < V) {
      a.lt = load_elem(tp(lane) + a.x);
      a.ld = load_elem(dp(lane) + a.x);
    }
  }
  if (lane <= n && !greedy) {
    const float2 u = spec_uniforms(c.seed, (uint32_t)c.seq_id[b], c.round,
                                   (uint32_t)(pos0 + lane), (uint32_t)stage);
    a.ua = u.x;
    a.ud = u.y;
  }
  return a;
}

// One speculative check on n positions (one warp). Target row j: tp(j) with
// log2 partition sh.M + sh.L at index j; draft law of position j: row dp(j)
// with log2 partition dlt(j). Returns a (first rejection, n if none) in every
// lane; *bad is set if a draft id lies outside [0, V); *u_draw gets the draw
// uniform of position a (sampled rows only). Writes p_j(x_j) and q_j(x_j) to
// diag_p / diag_q when given. Positions below 32 use the prefetched logits
// and uniforms.
template <typename T, typename TP, typename DP, typename DS>
__device__ int accept_scan(const SeqShared* sh, int n, int pos0, int stage,
                           const DecideCommon& c, int b, bool greedy, double cd,
                           const int32_t* drafts, TP tp, DP dp, DS dlt, double* diag_p,
                           double* diag_q, const AcceptPre& pre, int* bad_out,
                           float* u_draw) {
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
        acc = (x == sh->amax[j]);
      } else {
        const float lt = j0 == 0 ? pre.lt : load_elem(tp(j) + x);
        const float ld = j0 == 0 ? pre.ld : load_elem(dp(j) + x);
        const double lp = (double)lt * cd - (sh->M[j] + sh->L[j]);
        const double lq = (double)ld * cd - dlt(j);
        const float u = j0 == 0 ? pre.ua
                                : spec_uniforms(c.seed, (uint32_t)c.seq_id[b], c.round,
                                                (uint32_t)(pos0 + j), (uint32_t)stage).x;
        acc = (double)u < exp2(lp - lq);
        if (diag_p) { diag_p[j] = exp2(lp); diag_q[j] = exp2(lq); }
      }
    }
    if (__any_sync(0xffffffffu, badj)) bad = 1;
    const unsigned rej = __ballot_sync(0xffffffffu, j < n && !acc);
    if (rej && a == n) a = j0 + __ffs(rej) - 1;
  }
  *bad_out = bad;
  const float ud = __shfl_sync(0xffffffffu, pre.ud, a & 31);
  *u_draw = (a < 32 || greedy) ? ud
                               : spec_uniforms(c.seed, (uint32_t)c.seq_id[b], c.round,
                                               (uint32_t)(pos0 + a), (uint32_t)stage).y;
  return a;
}

__device__ __forceinline__ bool rows_ok(const SeqShared* sh, int nrows) {
  int bad = 0;
  for (int r = 0; r < nrows; ++r) bad |= !sh->ok[r];
  return !bad;
}

// Per-CTA outcome of the accept test (every CTA of the cluster computes it).
struct Outcome {
  int a, bad;
  float u_draw;
};

// ---------------------------------------------------------------------------
// Chain verification
// ---------------------------------------------------------------------------
template <typename T>
__global__ void __launch_bounds__(kDecThreads, 2) chain_decide_kernel(ChainDecideArgs A) {
  pdl_begin();
  __shared__ int s_claim;
  if (threadIdx.x == 0) s_claim = 0;  // the leader's: residual groups claimed so far
  cluster_arrive_relaxed();  // paired with the wait in cluster_rows
  cg::cluster_group cl = cg::this_cluster();
  const unsigned rank = cl.block_rank();
  __shared__ SeqShared sh;
  __shared__ Outcome s_out;
  extern __shared__ double dyn[];  // leader: [nrt] tile sums, [nrt] prefixes
  SeqShared* lsh = cl.map_shared_rank(&sh, 0);
  double* ltsum = cl.map_shared_rank(dyn, 0);
  const DecideCommon& c = A.c;
  const int b = blockIdx.y, K = c.K, V = c.V, per = 2 * K + 1;
  const float Tb = c.temperature[b];
  const bool tvalid = temp_valid(Tb), greedy = (Tb == 0.0f);
  double* diag = (rank == 0 && c.diag) ? c.diag + (size_t)b * (4 * K + 2) : nullptr;
  auto fail = [&]() {  // leader only
    if (threadIdx.x == 0) {
      set_status(c.status, SPEC_EDEVICE);
      A.accept_len[b] = -1;
    }
    for (int j = threadIdx.x; j <= K; j += blockDim.x) A.out_tok[(size_t)b * (K + 1) + j] = -1;
    if (diag)
      for (int j = threadIdx.x; j < 4 * K + 2; j += blockDim.x) diag[j] = dnan();
  };
  if (!tvalid) {  // the same decision in every CTA of the cluster: all leave here
    if (rank == 0) fail();
    return;
  }
  const Scale sc = greedy ? Scale{0.f, 0.f, 0.0} : make_scale(Tb);
  const int32_t* drafts = c.draft_tok + (size_t)b * K;
  auto tp = [&](int j) { return row_ptr<T>(A.tgt, A.ld_tgt, (long long)b * (K + 1) + j); };
  auto dp = [&](int j) { return row_ptr<T>(A.drf, A.ld_drf, (long long)b * K + j); };
  auto dl = [&](int j) { return lsh->M[K + 1 + j] + lsh->L[K + 1 + j]; };
  const bool accept_warp = (threadIdx.x >> 5) == kDecWarps - 1;
  AcceptPre pre{-1, 0.f, 0.f};
  if (accept_warp) pre = accept_prefetch<T>(K, V, greedy, drafts, tp, dp, c, b, 0, 1);
  cluster_rows(lsh, rank, c.part, c.ntiles, b * per, per,
               [&](int r) { return r <= K || !greedy; }, greedy, sc.hi, c.fin);
  cl.sync();  // the leader holds every row's statistics
  if (accept_warp) {
    int bad;
    float ud;
    const int a = accept_scan<T>(lsh, K, 0, 1, c, b, greedy, sc.d, drafts, tp, dp, dl,
                                 diag && !greedy ? diag + 2 * K + 1 : nullptr,
                                 diag && !greedy ? diag + 3 * K + 1 : nullptr, pre, &bad, &ud);
    if ((threadIdx.x & 31) == 0) s_out = Outcome{a, bad || !rows_ok(lsh, per), ud};
  }
  __syncthreads();
  const Outcome o = s_out;
  const int nrt = residual_tiles(V);
  const T* prow = nullptr;
  const T* qrow = nullptr;
  ProbCoef kp{}, kq{};
  if (!o.bad && !greedy) {
    prow = tp(o.a);
    qrow = o.a < K ? dp(o.a) : nullptr;
    kp = make_coef(lsh->M[o.a] + lsh->L[o.a], lsh->m[o.a], sc);
    kq = o.a < K ? make_coef(dl(o.a), lsh->m[K + 1 + o.a], sc) : make_coef(0.0, 0.0f, sc);
    residual_tile_sums_claimed<T>(prow, qrow, V, kp, kq, nrt, ltsum,
                                  cl.map_shared_rank(&s_claim, 0));
  }
  cl.sync();  // every tile sum is in the leader
  if (rank != 0) return;
  if (o.bad) {
    fail();
    return;
  }
  const int a = o.a;
  int tok;
  double Z = dnan();
  if (greedy) {
    tok = sh.amax[a];
  } else {
    const float u = o.u_draw;
    tok = leader_draw<T>(prow, qrow, V, kp, kq, dyn, dyn + nrt, u, &Z);
  }
  for (int j = threadIdx.x; j <= K; j += blockDim.x)
    A.out_tok[(size_t)b * (K + 1) + j] = j < a ? drafts[j] : (j == a ? tok : -1);
  if (threadIdx.x == 0) A.accept_len[b] = a;
  if (diag) {
    if (greedy) {
      for (int j = threadIdx.x; j < 4 * K + 2; j += blockDim.x) diag[j] = dnan();
    } else {
      for (int j = threadIdx.x; j < per; j += blockDim.x) diag[j] = (sh.M[j] + sh.L[j]) * kLn2;
      if (threadIdx.x == 0) diag[4 * K + 1] = Z;
    }
  }
}

// ---------------------------------------------------------------------------
// Small chain checks (V <= SPEC_SMALL_V): one CTA per sequence computes its
// rows' statistics itself, then runs the accept test and the draw, in one
// launch.
// ---------------------------------------------------------------------------
// The elements of a 16-byte vector of a row as floats.
__device__ __forceinline__ void vec_elems(uint4 w, float x[8], __nv_bfloat16*) {
  x[0] = bf_lo(w.x); x[1] = bf_hi(w.x); x[2] = bf_lo(w.y); x[3] = bf_hi(w.y);
  x[4] = bf_lo(w.z); x[5] = bf_hi(w.z); x[6] = bf_lo(w.w); x[7] = bf_hi(w.w);
}
__device__ __forceinline__ void vec_elems(uint4 w, float x[4], float*) {
  x[0] = __uint_as_float(w.x); x[1] = __uint_as_float(w.y);
  x[2] = __uint_as_float(w.z); x[3] = __uint_as_float(w.w);
}

// Statistics of one row by one warp (valid in every lane): the largest logit
// and its first index; for a sampled row (chi != 0) also the log2 partition
// M + L of 2^(l c), M = fl(m chi), from the terms 2^(l c - M) formed in fp32
// as the streaming statistics form them and summed per lane in fp64. The row
// is read as 16-byte vectors (rows start on 16-byte boundaries), kSmallU
// vectors per lane in flight, the last V mod EPV elements one by one; a lane
// visits its elements in rising index order.
constexpr int kSmallU = 4;
template <typename T>
__device__ RowFinal small_row(const T* row, int V, bool greedy, float chi, float clo, int lane) {
  constexpr int EPV = 16 / (int)sizeof(T);
  const int nv = V / EPV;
  const uint4* rv = reinterpret_cast<const uint4*>(row);
  float mv = -INFINITY;
  int mi = 0x7fffffff;
  for (int i0 = lane; i0 < nv; i0 += 32 * kSmallU) {
    uint4 w[kSmallU];
#pragma unroll
    for (int u = 0; u < kSmallU; ++u) w[u] = i0 + 32 * u < nv ? __ldg(rv + i0 + 32 * u) : uint4{};
#pragma unroll
    for (int u = 0; u < kSmallU; ++u) {
      if (i0 + 32 * u >= nv) break;
      float x[EPV];
      vec_elems(w[u], x, (T*)nullptr);
#pragma unroll
      for (int e = 0; e < EPV; ++e)
        if (x[e] > mv) {  // indices rise along the lane: ties keep the first
          mv = x[e];
          mi = (i0 + 32 * u) * EPV + e;
        }
    }
  }
  for (int e = nv * EPV + lane; e < V; e += 32) {
    const float x = load_elem(row + e);
    if (x > mv) {
      mv = x;
      mi = e;
    }
  }
  warp_argmax(mv, mi);
  RowFinal f{0.0, 0.0, mv, mi, 0, 0};
  bool ok = (mv > -INFINITY && mv < INFINITY);
  if (ok && !greedy) {
    const float Mf = __fmul_rn(mv, chi);
    const bool far = !(fabsf(Mf) < kFarShift);
    const float rr = fmaf(mv, chi, -Mf) + mv * clo;
    auto t = [&](float x) { return far ? term_far(x, mv, chi, clo, rr) : term(x, chi, clo, -Mf); };
    double s = 0.0;
    for (int i0 = lane; i0 < nv; i0 += 32 * kSmallU) {
      uint4 w[kSmallU];
#pragma unroll
      for (int u = 0; u < kSmallU; ++u)
        w[u] = i0 + 32 * u < nv ? __ldg(rv + i0 + 32 * u) : uint4{};
#pragma unroll
      for (int u = 0; u < kSmallU; ++u) {
        if (i0 + 32 * u >= nv) break;
        float x[EPV];
        vec_elems(w[u], x, (T*)nullptr);
        float v = 0.0f;
#pragma unroll
        for (int e = 0; e < EPV; ++e) v += t(x[e]);
        s += (double)v;
      }
    }
    for (int e = nv * EPV + lane; e < V; e += 32) s += (double)t(load_elem(row + e));
    s = warp_sum_d(s);
    ok = (s > 0.0 && s < INFINITY);
    f.M = (double)Mf;
    f.L = log2(s);
  }
  f.ok = ok;
  return f;
}

constexpr int kSmallV = SPEC_SMALL_V;
constexpr int kSmallTiles = (kSmallV + kResTile - 1) / kResTile;

template <typename T>
__global__ void __launch_bounds__(kDecThreads) chain_small_kernel(ChainDecideArgs A) {
  pdl_begin();
  __shared__ SeqShared sh;
  __shared__ Outcome s_out;
  __shared__ double s_tsum[kSmallTiles], s_pre[kSmallTiles];
  const DecideCommon& c = A.c;
  const int b = blockIdx.x, K = c.K, V = c.V, per = 2 * K + 1;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const float Tb = c.temperature[b];
  const bool tvalid = temp_valid(Tb), greedy = (Tb == 0.0f);
  double* diag = c.diag ? c.diag + (size_t)b * (4 * K + 2) : nullptr;
  auto fail = [&]() {
    if (threadIdx.x == 0) {
      set_status(c.status, SPEC_EDEVICE);
      A.accept_len[b] = -1;
    }
    for (int j = threadIdx.x; j <= K; j += blockDim.x) A.out_tok[(size_t)b * (K + 1) + j] = -1;
    if (diag)
      for (int j = threadIdx.x; j < 4 * K + 2; j += blockDim.x) diag[j] = dnan();
  };
  if (!tvalid) {
    fail();
    return;
  }
  const Scale sc = greedy ? Scale{0.f, 0.f, 0.0} : make_scale(Tb);
  const int32_t* drafts = c.draft_tok + (size_t)b * K;
  auto tp = [&](int j) { return row_ptr<T>(A.tgt, A.ld_tgt, (long long)b * (K + 1) + j); };
  auto dp = [&](int j) { return row_ptr<T>(A.drf, A.ld_drf, (long long)b * K + j); };
  auto dl = [&](int j) { return sh.M[K + 1 + j] + sh.L[K + 1 + j]; };
  const bool accept_warp = warp == kDecWarps - 1;
  AcceptPre pre{-1, 0.f, 0.f};
  if (accept_warp) pre = accept_prefetch<T>(K, V, greedy, drafts, tp, dp, c, b, 0, 1);
  // Rows 0..K: target positions; K+1..2K: draft positions (sampled sequences only).
  for (int r = warp; r < per && warp < kRowWarps; r += kRowWarps) {
    RowFinal f{0.0, 0.0, 0.f, -1, 1, 0};
    if (r <= K || !greedy)
      f = small_row<T>(r <= K ? tp(r) : dp(r - K - 1), V, greedy, sc.hi, sc.lo, lane);
    if (lane == 0) {
      sh.m[r] = f.m;
      sh.M[r] = f.M;
      sh.L[r] = f.L;
      sh.amax[r] = f.amax;
      sh.ok[r] = f.ok;
    }
  }
  __syncthreads();
  if (accept_warp) {
    int bad;
    float ud;
    const int a = accept_scan<T>(&sh, K, 0, 1, c, b, greedy, sc.d, drafts, tp, dp, dl,
                                 diag && !greedy ? diag + 2 * K + 1 : nullptr,
                                 diag && !greedy ? diag + 3 * K + 1 : nullptr, pre, &bad, &ud);
    if (lane == 0) s_out = Outcome{a, bad || !rows_ok(&sh, per), ud};
  }
  __syncthreads();
  const Outcome o = s_out;
  if (o.bad) {
    fail();
    return;
  }
  const int a = o.a;
  int tok;
  double Z = dnan();
  if (greedy) {
    tok = sh.amax[a];
  } else {
    const T* prow = tp(a);
    const T* qrow = a < K ? dp(a) : nullptr;
    const ProbCoef kp = make_coef(sh.M[a] + sh.L[a], sh.m[a], sc);
    const ProbCoef kq = a < K ? make_coef(dl(a), sh.m[K + 1 + a], sc) : make_coef(0.0, 0.0f, sc);
    residual_tile_sums<T>(prow, qrow, V, kp, kq, 0, residual_tiles(V), s_tsum);
    __syncthreads();
    tok = leader_draw<T>(prow, qrow, V, kp, kq, s_tsum, s_pre, o.u_draw, &Z);
  }
  for (int j = threadIdx.x; j <= K; j += blockDim.x)
    A.out_tok[(size_t)b * (K + 1) + j] = j < a ? drafts[j] : (j == a ? tok : -1);
  if (threadIdx.x == 0) A.accept_len[b] = a;
  if (diag) {
    if (greedy) {
      for (int j = threadIdx.x; j < 4 * K + 2; j += blockDim.x) diag[j] = dnan();
    } else {
      for (int j = threadIdx.x; j < per; j += blockDim.x) diag[j] = (sh.M[j] + sh.L[j]) * kLn2;
      if (threadIdx.x == 0) diag[4 * K + 1] = Z;
    }
  }
}

// ---------------------------------------------------------------------------
// Two-stage verification
// ---------------------------------------------------------------------------
// Window append (leader): a + 1 tokens at slots w.. with the L_i statistics of
// their slots (raw max m and ln sum exp((l - m)/T)).
__device__ __forceinline__ void window_append(const HierDecideArgs& A, int b, int w, int a,
                                              const int32_t* drafts, int tok, const SeqShared& sh,
                                              bool greedy, double cd) {
  const int WC = A.Ni + A.c.K;
  for (int j = threadIdx.x; j <= a; j += blockDim.x) {
    const size_t slot = (size_t)b * WC + w + j;
    A.win_tok[slot] = j < a ? drafts[j] : tok;
    if (greedy) {
      A.win_stat[2 * slot] = dnan();
      A.win_stat[2 * slot + 1] = dnan();
    } else {
      A.win_stat[2 * slot] = sh.m[j];
      A.win_stat[2 * slot + 1] = (sh.M[j] + sh.L[j] - (double)sh.m[j] * cd) * kLn2;
    }
  }
}

// Stage one: drafts (slots w..w+K-1) against L_i (slots w..w+K), draft law
// L_d; the a1 accepted drafts and the drawn token join the window.
template <typename T>
__global__ void __launch_bounds__(kDecThreads, 2) hier1_decide_kernel(HierDecideArgs A) {
  pdl_begin();
  cluster_arrive_relaxed();  // paired with the wait in cluster_rows
  cg::cluster_group cl = cg::this_cluster();
  const unsigned rank = cl.block_rank();
  __shared__ SeqShared sh;
  __shared__ Outcome s_out;
  extern __shared__ double dyn[];
  SeqShared* lsh = cl.map_shared_rank(&sh, 0);
  double* ltsum = cl.map_shared_rank(dyn, 0);
  const DecideCommon& c = A.c;
  const int b = blockIdx.y, K = c.K, V = c.V, S = A.S, Ni = A.Ni, WC = Ni + K, per = 2 * K + 1;
  const int D = 4 * K + 3 * S + 1;
  double* diag = (rank == 0 && c.diag) ? c.diag + (size_t)b * D : nullptr;
  if (rank == 0) {  // stage-two outputs default to "did not run"
    for (int j = threadIdx.x; j < WC + 1; j += blockDim.x)
      A.commit_tok[(size_t)b * (WC + 1) + j] = -1;
    if (threadIdx.x == 0) { A.commit_n[b] = 0; A.acc2[b] = -1; }
    if (diag)
      for (int j = threadIdx.x; j < D; j += blockDim.x) diag[j] = dnan();
  }
  const float Tb = c.temperature[b];
  const bool tvalid = temp_valid(Tb), greedy = (Tb == 0.0f);
  const int w = A.win_len[b];
  auto fail = [&]() {  // leader only
    if (threadIdx.x == 0) {
      set_status(c.status, SPEC_EDEVICE);
      A.acc1[b] = -1;
    }
  };
  if (!tvalid || w < 0 || w >= Ni) {
    if (rank == 0) fail();
    return;
  }
  const Scale sc = greedy ? Scale{0.f, 0.f, 0.0} : make_scale(Tb);
  const int32_t* drafts = c.draft_tok + (size_t)b * K;
  const long long row0 = (long long)b * S + w;
  auto tp = [&](int j) { return row_ptr<T>(A.lg_i, A.ld, row0 + j); };
  auto dp = [&](int j) { return row_ptr<T>(A.lg_d, A.ld, row0 + j); };
  auto dl = [&](int j) { return lsh->M[K + 1 + j] + lsh->L[K + 1 + j]; };
  const bool accept_warp = (threadIdx.x >> 5) == kDecWarps - 1;
  AcceptPre pre{-1, 0.f, 0.f};
  if (accept_warp) pre = accept_prefetch<T>(K, V, greedy, drafts, tp, dp, c, b, w, 1);
  cluster_rows(lsh, rank, c.part, c.ntiles, b * per, per,
               [&](int r) { return r <= K || !greedy; }, greedy, sc.hi, c.fin);
  cl.sync();
  if (accept_warp) {
    int bad;
    float ud;
    const int a = accept_scan<T>(lsh, K, w, 1, c, b, greedy, sc.d, drafts, tp, dp, dl,
                                 diag && !greedy ? diag + 2 * K + 1 : nullptr,
                                 diag && !greedy ? diag + 3 * K + 1 : nullptr, pre, &bad, &ud);
    if ((threadIdx.x & 31) == 0) s_out = Outcome{a, bad || !rows_ok(lsh, per), ud};
  }
  __syncthreads();
  const Outcome o = s_out;
  const int nrt = residual_tiles(V);
  const T* prow = nullptr;
  const T* qrow = nullptr;
  ProbCoef kp{}, kq{};
  if (!o.bad && !greedy) {
    prow = tp(o.a);
    qrow = o.a < K ? dp(o.a) : nullptr;
    kp = make_coef(lsh->M[o.a] + lsh->L[o.a], lsh->m[o.a], sc);
    kq = o.a < K ? make_coef(dl(o.a), lsh->m[K + 1 + o.a], sc) : make_coef(0.0, 0.0f, sc);
    const int chunk = (nrt + kCluster - 1) / kCluster;
    residual_tile_sums<T>(prow, qrow, V, kp, kq, min(nrt, (int)rank * chunk),
                          min(nrt, ((int)rank + 1) * chunk), ltsum);
  }
  cl.sync();
  if (rank != 0) return;
  if (o.bad) {
    fail();
    return;
  }
  const int a = o.a;
  int tok;
  double Z = dnan();
  if (greedy) {
    tok = sh.amax[a];
  } else {
    const float u = o.u_draw;
    tok = leader_draw<T>(prow, qrow, V, kp, kq, dyn, dyn + nrt, u, &Z);
  }
  window_append(A, b, w, a, drafts, tok, sh, greedy, sc.d);
  if (diag && !greedy) {
    for (int j = threadIdx.x; j < per; j += blockDim.x) diag[j] = (sh.M[j] + sh.L[j]) * kLn2;
    if (threadIdx.x == 0) diag[4 * K + 1] = Z;
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    A.win_len[b] = w + a + 1;
    A.acc1[b] = a;
  }
}

// Stage two: for sequences whose window holds W >= Ni tokens, the window
// tokens (slots 0..W-1) against L_f (slots 0..W), draft law L_i from the
// buffered statistics; commits a2 + 1 tokens and empties the window.
template <typename T>
__global__ void __launch_bounds__(kDecThreads, 2) hier2_decide_kernel(HierDecideArgs A) {
  pdl_begin();
  cluster_arrive_relaxed();  // paired with the wait in cluster_rows
  cg::cluster_group cl = cg::this_cluster();
  const unsigned rank = cl.block_rank();
  __shared__ SeqShared sh;
  __shared__ Outcome s_out;
  extern __shared__ double dyn[];
  SeqShared* lsh = cl.map_shared_rank(&sh, 0);
  double* ltsum = cl.map_shared_rank(dyn, 0);
  const DecideCommon& c = A.c;
  const int b = blockIdx.y, K = c.K, V = c.V, S = A.S, Ni = A.Ni, WC = Ni + K;
  const int W = A.win_len[b];
  if (A.acc1[b] < 0 || !(W >= Ni && W < S)) return;  // no second stage (every CTA)
  const float Tb = c.temperature[b];  // validated by stage one
  const bool greedy = (Tb == 0.0f);
  const Scale sc = greedy ? Scale{0.f, 0.f, 0.0} : make_scale(Tb);
  double* diag =
      (rank == 0 && c.diag) ? c.diag + (size_t)b * (4 * K + 3 * S + 1) + (4 * K + 2) : nullptr;
  const int32_t* wtok = A.win_tok + (size_t)b * WC;
  const double* wst = A.win_stat + (size_t)b * WC * 2;
  auto tp = [&](int j) { return row_ptr<T>(A.lg_f, A.ld, (long long)b * S + j); };
  auto dp = [&](int j) { return row_ptr<T>(A.lg_i, A.ld, (long long)b * S + j); };
  auto dl = [&](int j) { return wst[2 * j] * sc.d + wst[2 * j + 1] * kLog2e; };
  const bool accept_warp = (threadIdx.x >> 5) == kDecWarps - 1;
  AcceptPre pre{-1, 0.f, 0.f};
  if (accept_warp) pre = accept_prefetch<T>(W, V, greedy, wtok, tp, dp, c, b, 0, 2);
  cluster_rows(lsh, rank, c.part, c.ntiles, b * S, W + 1, [&](int) { return true; }, greedy,
               sc.hi, c.fin);
  cl.sync();
  if (accept_warp) {
    int bad;
    float ud;
    const int a = accept_scan<T>(lsh, W, 0, 2, c, b, greedy, sc.d, wtok, tp, dp, dl,
                                 diag && !greedy ? diag + S : nullptr,
                                 diag && !greedy ? diag + 2 * S - 1 : nullptr, pre, &bad, &ud);
    if ((threadIdx.x & 31) == 0) s_out = Outcome{a, bad || !rows_ok(lsh, W + 1), ud};
  }
  __syncthreads();
  const Outcome o = s_out;
  const int nrt = residual_tiles(V);
  const T* prow = nullptr;
  const T* qrow = nullptr;
  ProbCoef kp{}, kq{};
  if (!o.bad && !greedy) {
    prow = tp(o.a);
    qrow = o.a < W ? dp(o.a) : nullptr;
    kp = make_coef(lsh->M[o.a] + lsh->L[o.a], lsh->m[o.a], sc);
    kq = o.a < W ? make_coef(dl(o.a), (float)wst[2 * o.a], sc) : make_coef(0.0, 0.0f, sc);
    const int chunk = (nrt + kCluster - 1) / kCluster;
    residual_tile_sums<T>(prow, qrow, V, kp, kq, min(nrt, (int)rank * chunk),
                          min(nrt, ((int)rank + 1) * chunk), ltsum);
  }
  cl.sync();
  if (rank != 0) return;
  if (o.bad) {
    if (threadIdx.x == 0) {
      set_status(c.status, SPEC_EDEVICE);
      A.acc2[b] = -1;
    }
    return;
  }
  const int a = o.a;
  int tok;
  double Z = dnan();
  if (greedy) {
    tok = sh.amax[a];
  } else {
    const float u = o.u_draw;
    tok = leader_draw<T>(prow, qrow, V, kp, kq, dyn, dyn + nrt, u, &Z);
  }
  for (int j = threadIdx.x; j < WC + 1; j += blockDim.x)
    A.commit_tok[(size_t)b * (WC + 1) + j] = j < a ? wtok[j] : (j == a ? tok : -1);
  if (diag && !greedy) {
    for (int j = threadIdx.x; j <= W; j += blockDim.x) diag[j] = (sh.M[j] + sh.L[j]) * kLn2;
    if (threadIdx.x == 0) diag[3 * S - 2] = Z;
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    A.commit_n[b] = a + 1;
    A.acc2[b] = a;
    A.win_len[b] = 0;
  }
}

// ---------------------------------------------------------------------------
// Chain verification fused with the paged commit
// ---------------------------------------------------------------------------
// chain_decide_kernel's cluster per sequence, which also plans the commit.
// Once its accept test is done the leader writes the kept count (a + 1) and
// takes a ticket (one atomic, never awaited): the CTA that takes the B-th
// ticket has seen every kept count and runs the commit planner (tables, free
// stack, lengths, hidden offsets). The leader joins the residual tiles only
// after its ticket (and the planner after the plan), taking groups from the
// same counter as the other CTAs, so the planner, which overlaps the other
// sequences' draws, delays nothing but its own sequence's draw. The
// copy launch after this one moves the kept K/V and hidden rows: it starts
// while this launch runs and waits for plan_flag, which the first CTA clears
// before it lets that launch start and the planner sets when it is done.
template <typename T>
__global__ void __launch_bounds__(kDecThreads, 2) chain_decide_commit_kernel(FusedArgs F) {
  grid_dependency_wait();
  if (F.plan_flag && blockIdx.x == 0 && blockIdx.y == 0) {
    if (threadIdx.x == 0) {
      *F.plan_flag = 0;
      __threadfence();
    }
    __syncthreads();  // cleared before any thread of this CTA lets the copy launch start
  }
  grid_dependents_launch();
  __shared__ int s_last, s_claim;
  if (threadIdx.x == 0) s_claim = 0;  // the leader's: residual groups claimed so far
  cluster_arrive_relaxed();  // paired with the wait in cluster_rows
  cg::cluster_group cl = cg::this_cluster();
  const unsigned rank = cl.block_rank();
  __shared__ SeqShared sh;
  __shared__ Outcome s_out;
  extern __shared__ double dyn[];  // leader: [nrt] tile sums, [nrt] prefixes; planner: 3B ints
  SeqShared* lsh = cl.map_shared_rank(&sh, 0);
  double* ltsum = cl.map_shared_rank(dyn, 0);
  const ChainDecideArgs& A = F.d;
  const DecideCommon& c = A.c;
  const CommitArgs& cm = F.cm;
  const int b = blockIdx.y, K = c.K, V = c.V, per = 2 * K + 1;
  const int nrt = residual_tiles(V);
  int old_len = 0;
  if (rank == 0) {  // the record reads every held table entry: bring this row's into L2
    old_len = cm.seq_lens[b];
    const int held =
        min((max(old_len, 0) + cm.block_size - 1) / cm.block_size, cm.max_blocks);
    const int32_t* row = cm.tables + (size_t)b * cm.max_blocks;
    for (int i = threadIdx.x * 32; i < held; i += blockDim.x * 32)
      asm volatile("prefetch.global.L2 [%0];" ::"l"(row + i));
  }
  const float Tb = c.temperature[b];
  const bool tvalid = temp_valid(Tb), greedy = (Tb == 0.0f);
  double* diag = (rank == 0 && c.diag) ? c.diag + (size_t)b * (4 * K + 2) : nullptr;
  const int32_t* drafts = c.draft_tok + (size_t)b * K;
  int32_t* out = A.out_tok + (size_t)b * (K + 1);
  auto tp = [&](int j) { return row_ptr<T>(A.tgt, A.ld_tgt, (long long)b * (K + 1) + j); };
  auto dp = [&](int j) { return row_ptr<T>(A.drf, A.ld_drf, (long long)b * K + j); };
  auto dl = [&](int j) { return lsh->M[K + 1 + j] + lsh->L[K + 1 + j]; };
  const Scale sc = (greedy || !tvalid) ? Scale{0.f, 0.f, 0.0} : make_scale(Tb);
  if (tvalid) {
    const bool accept_warp = (threadIdx.x >> 5) == kDecWarps - 1;
    AcceptPre pre{-1, 0.f, 0.f};
    if (accept_warp) pre = accept_prefetch<T>(K, V, greedy, drafts, tp, dp, c, b, 0, 1);
    cluster_rows(lsh, rank, c.part, c.ntiles, b * per, per,
                 [&](int r) { return r <= K || !greedy; }, greedy, sc.hi, c.fin);
    cl.sync();  // the leader holds every row's statistics
    if (accept_warp) {
      int bad;
      float ud;
      const int a = accept_scan<T>(lsh, K, 0, 1, c, b, greedy, sc.d, drafts, tp, dp, dl,
                                   diag && !greedy ? diag + 2 * K + 1 : nullptr,
                                   diag && !greedy ? diag + 3 * K + 1 : nullptr, pre, &bad, &ud);
      if ((threadIdx.x & 31) == 0) s_out = Outcome{a, bad || !rows_ok(lsh, per), ud};
    }
  } else {
    cluster_wait();  // completes the entry barrier: no rows to combine
    if (threadIdx.x == 0) s_out = Outcome{0, 1, 0.f};
  }
  __syncthreads();
  const Outcome o = s_out;
  const int a = o.a;
  // Leader: every output but a sampled sequence's drawn token, the sequence's
  // commit record, then the ticket.
  if (rank == 0) {
    commit_record(cm, b, old_len, (o.bad ? -1 : a) + cm.keep_add, F.rec + b);
    if (o.bad) {
      if (threadIdx.x == 0) {
        set_status(c.status, SPEC_EDEVICE);
        A.accept_len[b] = -1;
      }
      for (int j = threadIdx.x; j <= K; j += blockDim.x) out[j] = -1;
      if (diag)
        for (int j = threadIdx.x; j < 4 * K + 2; j += blockDim.x) diag[j] = dnan();
    } else {
      for (int j = threadIdx.x; j <= K; j += blockDim.x)
        if (j != a || greedy) out[j] = j < a ? drafts[j] : (j == a ? sh.amax[a] : -1);
      if (threadIdx.x == 0) A.accept_len[b] = a;
      if (diag) {
        if (greedy)
          for (int j = threadIdx.x; j < 4 * K + 2; j += blockDim.x) diag[j] = dnan();
        else
          for (int j = threadIdx.x; j < per; j += blockDim.x) diag[j] = (sh.M[j] + sh.L[j]) * kLn2;
      }
    }
    __threadfence();
    __syncthreads();
    if (threadIdx.x == 0) {
      __threadfence();
      // The B-th ticket of this call (modulo B: a repeated call after one
      // row-statistics launch counts on from B).
      s_last = (atomicAdd(F.ticket, 1) + 1) % c.B == 0;
    }
    __syncthreads();
    if (s_last) {
      __threadfence();  // every other sequence's kept count and status are visible
      plan_body(cm, reinterpret_cast<int*>(dyn + 2 * nrt), F.rec);
      if (F.plan_flag) {
        __syncthreads();  // every write of the plan is made
        if (threadIdx.x == 0) {
          __threadfence();
          st_release(F.plan_flag, 1);
        }
      }
    }
  }
  // Residual tile sums of a sampled sequence: groups claimed by every CTA of the cluster.
  const bool draw = !o.bad && !greedy;
  const T* prow = nullptr;
  const T* qrow = nullptr;
  ProbCoef kp{}, kq{};
  if (draw) {
    prow = tp(a);
    qrow = a < K ? dp(a) : nullptr;
    kp = make_coef(lsh->M[a] + lsh->L[a], lsh->m[a], sc);
    kq = a < K ? make_coef(dl(a), lsh->m[K + 1 + a], sc) : make_coef(0.0, 0.0f, sc);
    residual_tile_sums_claimed<T>(prow, qrow, V, kp, kq, nrt, ltsum,
                                  cl.map_shared_rank(&s_claim, 0));
  }
  // The tile sums are in the leader once every CTA has arrived; only the
  // leader waits.
  asm volatile("barrier.cluster.arrive;" ::: "memory");
  if (rank != 0) return;
  asm volatile("barrier.cluster.wait;" ::: "memory");
  if (draw) {
    double Z;
    const int tok = leader_draw<T>(prow, qrow, V, kp, kq, dyn, dyn + nrt, o.u_draw, &Z);
    if (threadIdx.x == 0) {
      out[a] = tok;
      if (diag) diag[4 * K + 1] = Z;
    }
  }
}

// ---------------------------------------------------------------------------
// Launchers: grid (kCluster, B), clusters of kCluster CTAs along x.
// ---------------------------------------------------------------------------
template <typename Kern, typename Args>
static cudaError_t launch_decide(Kern k, const Args& a, cudaStream_t st) {
  const size_t smem = 2 * (size_t)residual_tiles(a.c.V) * sizeof(double);
  const cudaError_t e = reserve_dyn_smem(k, smem);
  if (e != cudaSuccess) return e;
  return launch_pdl_cluster(k, dim3(kCluster, a.c.B), dim3(kDecThreads), smem, st, kCluster, a);
}

cudaError_t launch_chain_small(const ChainDecideArgs& a, cudaStream_t st) {
  if (a.c.V > kSmallV || a.c.V < 1) return cudaErrorInvalidValue;
  return a.c.dtype == SPEC_BF16
             ? launch_pdl(chain_small_kernel<__nv_bfloat16>, dim3(a.c.B), dim3(kDecThreads), 0,
                          st, a)
             : launch_pdl(chain_small_kernel<float>, dim3(a.c.B), dim3(kDecThreads), 0, st, a);
}

cudaError_t launch_chain_decide(const ChainDecideArgs& a, cudaStream_t st) {
  return a.c.dtype == SPEC_BF16 ? launch_decide(chain_decide_kernel<__nv_bfloat16>, a, st)
                                : launch_decide(chain_decide_kernel<float>, a, st);
}
template <typename T>
static cudaError_t launch_fused(const FusedArgs& a, cudaStream_t st) {
  auto k = chain_decide_commit_kernel<T>;
  const size_t smem = 2 * (size_t)residual_tiles(a.d.c.V) * sizeof(double) +
                      3 * (size_t)a.d.c.B * sizeof(int);
  cudaError_t e = reserve_dyn_smem(k, smem);
  if (e != cudaSuccess) return e;
  const bool copy = a.cm.B > 0 && a.cm.Kp1 > 0 && (a.cm.kv_stage || a.cm.hid_stage);
  FusedArgs f = a;
  if (!copy) f.plan_flag = nullptr;
  e = launch_pdl_cluster(k, dim3(kCluster, a.d.c.B), dim3(kDecThreads), smem, st, kCluster, f);
  if (e != cudaSuccess || !copy) return e;
  return f.plan_flag ? launch_commit_copy_planned(f.cm, f.plan_flag, st)
                     : launch_commit_copy(f.cm, st);
}

cudaError_t launch_chain_fused(const FusedArgs& a, cudaStream_t st) {
  return a.d.c.dtype == SPEC_BF16 ? launch_fused<__nv_bfloat16>(a, st)
                                  : launch_fused<float>(a, st);
}
cudaError_t launch_hier1_decide(const HierDecideArgs& a, cudaStream_t st) {
  return a.c.dtype == SPEC_BF16 ? launch_decide(hier1_decide_kernel<__nv_bfloat16>, a, st)
                                : launch_decide(hier1_decide_kernel<float>, a, st);
}
cudaError_t launch_hier2_decide(const HierDecideArgs& a, cudaStream_t st) {
  return a.c.dtype == SPEC_BF16 ? launch_decide(hier2_decide_kernel<__nv_bfloat16>, a, st)
                                : launch_decide(hier2_decide_kernel<float>, a, st);
}

}  // namespace specv
