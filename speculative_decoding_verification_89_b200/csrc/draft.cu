// Draft step: the token the drafting exit proposes at one slot of each
// sequence, ln q of that token and the entropy of the drafting distribution.
//
// HiSpec (gist.science summary of arXiv 2510.01336), section 2
// "Kernmechanismus": the shallow exit L_d drafts the tokens that the deeper
// exits check; a draft is a draw from softmax(l_d / T). The entropy of that
// distribution is the uncertainty signal of SVIP (Optimierung der
// Inferenzgeschwindigkeit von Sprachmodellen durch spekulative Dekodierung,
// mind-verse.de, SVIP paragraphs), from which a draft-length policy decides
// whether to keep drafting.
//
// One launch when a cluster of 4 (or 8) CTAs can hold a row in shared memory
// (draft_fused_kernel: every logit read from HBM once, statistics and draw
// from shared memory). Larger rows take two launches: the row-statistics
// kernel over the B rows (DraftRows, which also gathers the first moment sum
// 2^(l*c - M) * (l - m)), then one thread-block cluster per sequence that
// combines its row, and -- unless the sequence is greedy -- splits the row's
// 256-element tiles of p over the cluster, prefixes their sums in the leader
// and draws. Either way the draw is by inverse CDF with the lane-1 uniform of
// the Philox counter (seq_id, round, pos, 0).
#include <cfloat>
#include <climits>

#include "draw.cuh"

namespace specv {

// Row combine with the entropy: log2-partition Lt = M + L, raw max m, first
// argmax, ok, and H = -sum p ln p in nats. Warp-cooperative; every lane gets
// the result.
struct DraftStat {
  double Lt, H;
  float m;
  int amax, ok;
};
__device__ DraftStat combine_draft_row(const Partial* p, const double* mom, int ntiles,
                                       bool greedy, const Scale& sc, int lane) {
  const RowFinal f = combine_row(p, ntiles, greedy, sc.hi, lane);
  DraftStat d;
  d.m = __shfl_sync(0xffffffffu, f.m, 0);
  d.amax = __shfl_sync(0xffffffffu, f.amax, 0);
  d.ok = __shfl_sync(0xffffffffu, f.ok, 0);
  d.Lt = __shfl_sync(0xffffffffu, f.M + f.L, 0);
  d.H = 0.0;
  if (greedy || !d.ok) return d;
  // Moments of the runs about the row maximum m, rescaled to the shift
  // M = fl(m * c_hi): s = sum s_k 2^(M_k - M), t = sum (t_k + (m_k - m) s_k) 2^(M_k - M).
  const double M = (double)__fmul_rn(d.m, sc.hi);
  double s = 0.0, t = 0.0;
  for (int k = lane; k < ntiles; k += 32) {
    const Partial q = p[k];
    if (q.s != 0.0) {
      const double fk = exp2((double)__fmul_rn(q.m, sc.hi) - M);
      s += q.s * fk;
      t += (mom[k] + ((double)q.m - (double)d.m) * q.s) * fk;
    }
  }
  s = warp_sum_d(s);
  t = warp_sum_d(t);
  // H = ln2 * (Lt - c E[l]) with E[l] = m + t / s and Lt = M + log2 s:
  // (M - c m) + log2 s - c t / s, no cancellation (t <= 0).
  const double Mcm = (M - (double)d.m * (double)sc.hi) - (double)d.m * (double)sc.lo;
  d.H = kLn2 * (Mcm + log2(s) - sc.d * (t / s));
  return d;
}

struct DraftArgs {
  int B, V, ntiles;
  const unsigned char* lg;
  long long ld;  // bytes
  const float* temperature;
  uint64_t seed;
  const int32_t* seq_id;
  uint32_t round;
  const int32_t* pos;
  const Partial* part;
  const double* mom;
  int32_t* out_tok;
  double* out_logq;
  double* out_entropy;
  int32_t* status;
};

template <typename T>
__global__ void __launch_bounds__(kDecThreads, 2) draft_draw_kernel(DraftArgs A) {
  pdl_begin();
  asm volatile("barrier.cluster.arrive.relaxed;" ::: "memory");  // waited before remote writes
  cg::cluster_group cl = cg::this_cluster();
  const unsigned rank = cl.block_rank();
  __shared__ DraftStat s_st;
  extern __shared__ double dyn[];  // leader: [nrt] tile sums, [nrt] prefixes
  double* ltsum = cl.map_shared_rank(dyn, 0);
  const int b = blockIdx.y, V = A.V;
  const float Tb = A.temperature[b];
  const bool greedy = (Tb == 0.0f);
  auto finish = [&](int tok, double logq, double H, bool bad) {  // leader, thread 0
    if (bad) set_status(A.status, SPEC_EDEVICE);
    A.out_tok[b] = bad ? -1 : tok;
    if (A.out_logq) A.out_logq[b] = bad ? dnan() : logq;
    if (A.out_entropy) A.out_entropy[b] = bad ? dnan() : H;
  };
  if (!temp_valid(Tb)) {  // the same decision in every CTA of the cluster
    if (rank == 0 && threadIdx.x == 0) finish(-1, 0.0, 0.0, true);
    return;
  }
  const Scale sc = greedy ? Scale{0.f, 0.f, 0.0} : make_scale(Tb);
  const T* prow = row_ptr<T>(A.lg, A.ld, b);
  if (threadIdx.x < 32) {
    const DraftStat d = combine_draft_row(A.part + (size_t)b * A.ntiles,
                                          A.mom + (size_t)b * A.ntiles, A.ntiles, greedy, sc,
                                          threadIdx.x);
    if (threadIdx.x == 0) s_st = d;
  }
  __syncthreads();
  const DraftStat st = s_st;
  if (!st.ok || greedy) {  // uniform over the cluster
    if (rank == 0 && threadIdx.x == 0) finish(st.amax, 0.0, 0.0, !st.ok);
    return;
  }
  const ProbCoef kp = make_coef(st.Lt, st.m, sc);
  const int nrt = residual_tiles(V);
  const int chunk = (nrt + kCluster - 1) / kCluster;
  asm volatile("barrier.cluster.wait;" ::: "memory");  // every CTA runs: remote writes allowed
  residual_tile_sums<T>(prow, nullptr, V, kp, kp, min(nrt, (int)rank * chunk),
                        min(nrt, ((int)rank + 1) * chunk), ltsum);
  cl.sync();  // every tile sum is in the leader
  if (rank != 0) return;
  const float u = spec_uniforms(A.seed, (uint32_t)A.seq_id[b], A.round, (uint32_t)A.pos[b], 0u).y;
  double Z;
  const int tok = leader_draw<T>(prow, nullptr, V, kp, kp, dyn, dyn + nrt, u, &Z);
  if (threadIdx.x == 0) {
    const bool bad = tok < 0 || tok >= V;
    const double logq = bad ? 0.0 : kLn2 * ((double)load_elem(prow + tok) * sc.d - st.Lt);
    finish(tok, logq, st.H, bad);
  }
}

// ---------------------------------------------------------------------------
// One launch for rows that fit the cluster's shared memory
// ---------------------------------------------------------------------------
// A cluster of cs CTAs per row. CTA r stages its slice of the row -- whole
// 256-element tiles [r*tc, (r+1)*tc) -- in shared memory with bulk copies, so
// the row is read from HBM once, and finds its largest logit m_r with its
// first index, then per tile the sum of 2^(x*c - M_r) with its own exact
// shift M_r = fl(m_r * c_hi), and the first moment sum 2^(x*c - M_r) (x - m_r).
// Every CTA sends (m_r, argmax, S_r, T_r) to every other CTA of the cluster
// (distributed shared memory); after a cluster barrier each combines them in
// the same order -- the row's max and shift M, partition, entropy and the draw
// target u * S -- and the CTA whose slice holds the target prefixes its tile
// sums and rescans one tile in shared memory for the token. Results equal the
// two-launch path's up to the summation order of the partition.
constexpr int kDfMaxCluster = 8;
constexpr int kDfSliceBytes = 100 * 1024;  // staged slice per CTA, at most
constexpr uint32_t kDfChunk = 32768;        // bytes per bulk copy

struct DfPart {
  float m;
  int amax;
  double S, T;
};

// One staged element (shared memory: plain loads, not the read-only path).
__device__ __forceinline__ float smem_elem(const float* p) { return *p; }
__device__ __forceinline__ float smem_elem(const __nv_bfloat16* p) {
  return __uint_as_float(((unsigned)*reinterpret_cast<const unsigned short*>(p)) << 16);
}
template <typename T>
__device__ __forceinline__ void smem8(const T* xs, int i0, int n, float x[8]) {
  if (i0 + 8 <= n) {
    Raw8<T> r;
    const uint4* p = reinterpret_cast<const uint4*>(xs + i0);
#pragma unroll
    for (int k = 0; k < (int)(sizeof(T) / 2); ++k) r.v[k] = p[k];
    unpack8(r, x);
  } else {
#pragma unroll
    for (int e = 0; e < 8; ++e) x[e] = i0 + e < n ? smem_elem(xs + i0 + e) : -INFINITY;
  }
}

template <typename T>
__global__ void __launch_bounds__(kDecThreads, 2) draft_fused_kernel(DraftArgs A, int tc) {
  pdl_begin();
  asm volatile("barrier.cluster.arrive.relaxed;" ::: "memory");  // waited before remote writes
  cg::cluster_group cl = cg::this_cluster();
  const int rank = (int)cl.block_rank(), cs = (int)cl.num_blocks();
  extern __shared__ __align__(128) unsigned char dsm[];
  T* xs = reinterpret_cast<T*>(dsm);
  double* tsum = reinterpret_cast<double*>(dsm + (size_t)tc * kResTile * sizeof(T));
  __shared__ __align__(8) uint64_t s_bar;
  __shared__ DfPart s_part[kDfMaxCluster];
  __shared__ float s_wm[kDecWarps];
  __shared__ int s_wi[kDecWarps];
  __shared__ double s_ws[kDecWarps], s_wt[kDecWarps];
  const int b = blockIdx.y, V = A.V, lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int nrt = residual_tiles(V);
  const int t0 = min(nrt, rank * tc), t1 = min(nrt, t0 + tc), nt = t1 - t0;
  const int e0 = t0 * kResTile, n = max(0, min(V, t1 * kResTile) - e0);
  const float Tb = A.temperature[b];
  const bool greedy = (Tb == 0.0f);
  const T* row = row_ptr<T>(A.lg, A.ld, b);
  auto finish = [&](int tok, double logq, double H, bool bad) {
    if (bad) set_status(A.status, SPEC_EDEVICE);
    A.out_tok[b] = bad ? -1 : tok;
    if (A.out_logq) A.out_logq[b] = bad ? dnan() : logq;
    if (A.out_entropy) A.out_entropy[b] = bad ? dnan() : H;
  };
  if (!temp_valid(Tb)) {  // the same decision in every CTA of the cluster
    if (rank == 0 && threadIdx.x == 0) finish(-1, 0.0, 0.0, true);
    return;
  }
  const Scale sc = greedy ? Scale{0.f, 0.f, 0.0} : make_scale(Tb);

  // Stage the slice: bulk copies of its 16-byte part, plain loads of the rest.
  const uint32_t bytes = ((uint32_t)n * (uint32_t)sizeof(T)) & ~15u;
  const int nbulk = (int)(bytes / sizeof(T));
  if (threadIdx.x == 0) {
    mbar_init(&s_bar, 1);
    fence_barrier_init();
  }
  __syncthreads();
  if (threadIdx.x == 0 && bytes) {
    mbar_arrive_expect_tx(&s_bar, bytes);
    const unsigned char* src = reinterpret_cast<const unsigned char*>(row + e0);
    for (uint32_t o = 0; o < bytes; o += kDfChunk)
      bulk_g2s(dsm + o, src + o, min(kDfChunk, bytes - o), &s_bar);
  }
  for (int i = nbulk + (int)threadIdx.x; i < n; i += blockDim.x) xs[i] = row[e0 + i];
  if (bytes && !mbar_wait_bounded(&s_bar, 0, kWaitLimitNs)) {
    set_status(A.status, SPEC_ETIMEOUT);
    mbar_wait_bounded(&s_bar, 0, kWaitLimitNs);  // let the copies land before going on
  }
  __syncthreads();

  // Largest logit of the slice, and for a greedy row its first index.
  float mv = -INFINITY;
  int mi = 0x7fffffff;
  if (greedy) {
    for (int i0 = (int)threadIdx.x * 8; i0 < n; i0 += blockDim.x * 8) {
      float x[8];
      smem8(xs, i0, n, x);
#pragma unroll
      for (int e = 0; e < 8; ++e)
        if (x[e] > mv) { mv = x[e]; mi = e0 + i0 + e; }
    }
  } else {
    for (int i0 = (int)threadIdx.x * 8; i0 < n; i0 += blockDim.x * 8) {
      float x[8];
      smem8(xs, i0, n, x);
#pragma unroll
      for (int e = 0; e < 8; ++e) mv = fmaxf(mv, x[e]);
    }
  }
  warp_argmax(mv, mi);
  if (lane == 0) { s_wm[warp] = mv; s_wi[warp] = mi; }
  __syncthreads();
  float m_r = -INFINITY;
  int a_r = 0x7fffffff;
  for (int w = 0; w < kDecWarps; ++w)
    if (s_wm[w] > m_r || (s_wm[w] == m_r && s_wi[w] < a_r)) { m_r = s_wm[w]; a_r = s_wi[w]; }

  // Tile sums of 2^(x*c - M_r) and the first moment about m_r.
  double S_r = 0.0, T_r = 0.0;
  const bool fin = m_r > -INFINITY && m_r < INFINITY;
  if (!greedy && fin) {
    const float Mr = __fmul_rn(m_r, sc.hi);
    const ProbCoef kr = make_coef((double)Mr, m_r, sc);
    double ws = 0.0, wt = 0.0;
    for (int t = warp; t < nt; t += kDecWarps) {
      float x[8], w[8];
      smem8(xs, t * kResTile + lane * 8, n, x);
#pragma unroll
      for (int e = 0; e < 8; e += 2) {
        const float2 pr = prob2(make_float2(x[e], x[e + 1]), kr);
        w[e] = pr.x;
        w[e + 1] = pr.y;
      }
      float mom = 0.0f;
#pragma unroll
      for (int e = 0; e < 8; ++e) mom += w[e] * fmaxf(x[e] - m_r, -FLT_MAX);
      float ls = (float)lane_sum8(w);  // fp32 over the tile: values <= 1, 256 terms
#pragma unroll
      for (int o = 16; o; o >>= 1) ls += __shfl_xor_sync(0xffffffffu, ls, o);
      if (lane == 0) tsum[t] = (double)ls;
      ws += (double)ls;
      wt += (double)mom;
    }
    wt = warp_sum_d(wt);  // ws is the same in every lane
    if (lane == 0) { s_ws[warp] = ws; s_wt[warp] = wt; }
    __syncthreads();
    for (int w = 0; w < kDecWarps; ++w) { S_r += s_ws[w]; T_r += s_wt[w]; }
  }

  // Every CTA's summary to every CTA, then the same combine everywhere.
  asm volatile("barrier.cluster.wait;" ::: "memory");
  if (threadIdx.x < cs) {
    DfPart* dst = cl.map_shared_rank(s_part, (unsigned)threadIdx.x);
    dst[rank] = DfPart{m_r, a_r, S_r, T_r};
  }
  cl.sync();
  // The combine, by one thread (the same arithmetic in every CTA).
  __shared__ float s_m;
  __shared__ int s_amax, s_owner;
  __shared__ double s_Lt, s_H, s_local;
  if (threadIdx.x == 0) {
    float m = -INFINITY;
    int amax = 0x7fffffff;
    for (int r = 0; r < cs; ++r)
      if (s_part[r].m > m || (s_part[r].m == m && s_part[r].amax < amax)) {
        m = s_part[r].m;
        amax = s_part[r].amax;
      }
    s_m = m;
    s_amax = amax;
    s_owner = -1;
    const bool ok = m > -INFINITY && m < INFINITY;
    if (ok && !greedy) {
      const double M = (double)__fmul_rn(m, sc.hi);
      double f[kDfMaxCluster];
      double S = 0.0, Tm = 0.0;
      for (int r = 0; r < cs; ++r) {
        f[r] = 0.0;
        if (s_part[r].S > 0.0) {
          const float mr = s_part[r].m;
          f[r] = exp2((double)__fmul_rn(mr, sc.hi) - M);
          S += s_part[r].S * f[r];
          Tm += (s_part[r].T + ((double)mr - (double)m) * s_part[r].S) * f[r];
        }
      }
      const double Mcm = (M - (double)m * (double)sc.hi) - (double)m * (double)sc.lo;
      s_Lt = M + log2(S);
      s_H = kLn2 * (Mcm + log2(S) - sc.d * (Tm / S));
      const float u =
          spec_uniforms(A.seed, (uint32_t)A.seq_id[b], A.round, (uint32_t)A.pos[b], 0u).y;
      const double target = (double)u * S;
      // The CTA whose slice holds the target: the first whose running total passes it.
      double cum = 0.0;
      for (int r = 0; r < cs; ++r) {
        if (s_part[r].S > 0.0) {
          const double c_r = s_part[r].S * f[r];
          s_owner = r;  // the last with mass, if rounding leaves the target past the end
          s_local = (target - cum) / f[r];
          if (cum + c_r > target) break;
          cum += c_r;
        }
      }
    }
  }
  __syncthreads();
  const float m = s_m;
  const int amax = s_amax, owner = s_owner;
  const bool ok = m > -INFINITY && m < INFINITY;
  if (!ok || greedy) {
    if (rank == 0 && threadIdx.x == 0) finish(amax, 0.0, 0.0, !ok);
    return;
  }
  const double Lt = s_Lt, H = s_H, local = s_local;
  if (owner < 0) {  // no mass anywhere: cannot happen for a row with a finite maximum
    if (rank == 0 && threadIdx.x == 0) finish(-1, 0.0, 0.0, true);
    return;
  }
  if (rank != owner) return;

  // Owner: the tile (warp 0 prefixes the tile sums: a contiguous run per
  // lane, then a scan over the lanes), then the element.
  if (warp == 0) {
    const int per = (nt + 31) / 32;
    const int a0 = min(nt, lane * per), a1 = min(nt, a0 + per);
    double run = 0.0;
    for (int t = a0; t < a1; ++t) run += tsum[t];
    double incl = run;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const double y = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += y;
    }
    // The last tile with mass whose prefix does not pass the target.
    double c = incl - run, c_cand = 0.0;
    int cand = -1;
    for (int t = a0; t < a1; ++t) {
      if (c <= local && tsum[t] > 0.0) { cand = t; c_cand = c; }
      c += tsum[t];
    }
    int best = cand;
#pragma unroll
    for (int o = 16; o; o >>= 1) best = max(best, __shfl_xor_sync(0xffffffffu, best, o));
    const int tile = best < 0 ? 0 : best;
    const unsigned holder = __ballot_sync(0xffffffffu, cand == best && best >= 0);
    const double pre = holder ? __shfl_sync(0xffffffffu, c_cand, __ffs(holder) - 1) : 0.0;
    const float Mr = __fmul_rn(s_part[owner].m, sc.hi);
    const ProbCoef kr = make_coef((double)Mr, s_part[owner].m, sc);
    float x[8], w[8];
    smem8(xs, tile * kResTile + lane * 8, n, x);
#pragma unroll
    for (int e = 0; e < 8; e += 2) {
      const float2 pr = prob2(make_float2(x[e], x[e + 1]), kr);
      w[e] = pr.x;
      w[e + 1] = pr.y;
    }
    const double ls = lane_sum8(w);
    double li = ls;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const double y = __shfl_up_sync(0xffffffffu, li, o);
      if (lane >= o) li += y;
    }
    const double start = pre + (li - ls);
    int found = INT_MAX;
    if (start <= local) {
      double acc = start;
      for (int e = 0; e < 8; ++e) {
        acc += (double)w[e];
        if (acc > local && w[e] > 0.0f) { found = tile * kResTile + lane * 8 + e; break; }
      }
    }
#pragma unroll
    for (int o = 16; o; o >>= 1) found = min(found, __shfl_xor_sync(0xffffffffu, found, o));
    if (found == INT_MAX) {  // the target sits at the tile's end by rounding
      int last = -1;
      for (int e = 7; e >= 0; --e)
        if (w[e] > 0.0f) { last = tile * kResTile + lane * 8 + e; break; }
#pragma unroll
      for (int o = 16; o; o >>= 1) last = max(last, __shfl_xor_sync(0xffffffffu, last, o));
      found = last;
    }
    if (lane == 0) {
      const bool bad = found < 0 || found >= n;
      const int tok = bad ? -1 : e0 + found;
      const double logq = bad ? 0.0 : kLn2 * ((double)smem_elem(xs + found) * sc.d - Lt);
      finish(tok, logq, H, bad);
    }
  }
}

template <typename T>
static cudaError_t launch_draw(const DraftArgs& a, cudaStream_t st) {
  auto k = draft_draw_kernel<T>;
  const size_t smem = 2 * (size_t)residual_tiles(a.V) * sizeof(double);
  const cudaError_t e = reserve_dyn_smem(k, smem);
  if (e != cudaSuccess) return e;
  return launch_pdl_cluster(k, dim3(kCluster, a.B), dim3(kDecThreads), smem, st, kCluster, a);
}

template <typename T>
static cudaError_t launch_fused_draw(const DraftArgs& a, int cs, int tc, cudaStream_t st) {
  auto k = draft_fused_kernel<T>;
  const size_t smem = (size_t)tc * kResTile * sizeof(T) + (size_t)tc * sizeof(double);
  const cudaError_t e = reserve_dyn_smem(k, smem);
  if (e != cudaSuccess) return e;
  return launch_pdl_cluster(k, dim3(cs, a.B), dim3(kDecThreads), smem, st, (unsigned)cs, a, tc);
}

cudaError_t launch_draft_step(int dtype, const unsigned char* lg, long long ld_bytes, int B, int V,
                              const float* temperature, uint64_t seed, const int32_t* seq_id,
                              uint32_t round, const int32_t* pos, Partial* part, double* mom,
                              int32_t* out_tok, double* out_logq, double* out_entropy,
                              int32_t* status, cudaStream_t st) {
  // One launch when a cluster of 4 (or 8) CTAs holds the row in shared memory.
  const int esz = dtype == SPEC_BF16 ? 2 : 4, nrt = residual_tiles(V);
  for (int cs = 4; cs <= kDfMaxCluster; cs *= 2) {
    const int tc = (nrt + cs - 1) / cs;
    if ((size_t)tc * kResTile * esz + (size_t)tc * sizeof(double) > (size_t)kDfSliceBytes) continue;
    DraftArgs a{};
    a.B = B;
    a.V = V;
    a.lg = lg;
    a.ld = ld_bytes;
    a.temperature = temperature;
    a.seed = seed;
    a.seq_id = seq_id;
    a.round = round;
    a.pos = pos;
    a.out_tok = out_tok;
    a.out_logq = out_logq;
    a.out_entropy = out_entropy;
    a.status = status;
    return dtype == SPEC_BF16 ? launch_fused_draw<__nv_bfloat16>(a, cs, tc, st)
                              : launch_fused_draw<float>(a, cs, tc, st);
  }
  // Larger rows: the row statistics, then the draw re-reading one row.
  DraftRows rows;
  rows.lg = lg;
  rows.ld = ld_bytes;
  rows.temperature = temperature;
  RsBuffers rb;
  rb.part = part;
  rb.mom = mom;
  rb.zero = nullptr;
  cudaError_t e = launch_row_stats(dtype, rows, B, V, rb, status, st);
  if (e != cudaSuccess) return e;
  DraftArgs a;
  a.B = B;
  a.V = V;
  a.ntiles = (V + kTileBytes / (dtype == SPEC_BF16 ? 2 : 4) - 1) /
             (kTileBytes / (dtype == SPEC_BF16 ? 2 : 4));
  a.lg = lg;
  a.ld = ld_bytes;
  a.temperature = temperature;
  a.seed = seed;
  a.seq_id = seq_id;
  a.round = round;
  a.pos = pos;
  a.part = part;
  a.mom = mom;
  a.out_tok = out_tok;
  a.out_logq = out_logq;
  a.out_entropy = out_entropy;
  a.status = status;
  return dtype == SPEC_BF16 ? launch_draw<__nv_bfloat16>(a, st) : launch_draw<float>(a, st);
}

}  // namespace specv
