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
// One launch when a cluster of up to 8 CTAs can hold a row in shared memory
// (draft_fused_kernel, 1 to 8 CTAs per row as launch_draft_step chooses: every logit read from HBM once, statistics and draw
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
#include "rowmath.cuh"

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
// 256-element tiles [r*tc, (r+1)*tc) -- in shared memory by bulk copies of
// kDfChunk bytes, each completing on its own mbarrier, so the row is read from
// HBM once and a warp starts on its tiles as soon as their chunk has landed.
// Per tile, in one pass: its largest logit m_t (and for a greedy row its
// first index), the sum S_t of 2^(x*c - M_t) with the tile's integral shift
// M_t = ceil(m_t * c_hi), and the first moment T_t = sum 2^(x*c - M_t) (x - m_t).
// The CTA rescales its tiles to its largest shift M_r by exact powers of two
// and sends (m_r, argmax, M_r, S_r, T_r) to every CTA of the cluster
// (distributed shared memory); after a cluster barrier each combines them in
// the same order -- the row's max, shift, partition, entropy and the draw
// target u * S -- and the CTA whose slice holds the target prefixes its tile
// sums and rescans one tile in shared memory, with that tile's own shift, for
// the token.
constexpr int kDfMaxCluster = 8;
constexpr int kDfSliceBytes = 100 * 1024;  // staged slice per CTA, at most
constexpr int kDfSmallSlice = 16;           // tiles: a slice this short is not split further
constexpr uint32_t kDfChunk = 32768;        // bytes per bulk copy (whole tiles)
constexpr int kDfMaxChunks = (kDfSliceBytes + (int)kDfChunk - 1) / (int)kDfChunk;
// Per tile of the slice: the scaled sum (double), then m_t, M_t, S_t, T_t.
constexpr size_t kDfTileBytes = sizeof(double) + 4 * sizeof(float);

struct DfPart {
  float m, M;
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
// A lane's 8 staged elements as four pairs, and their largest (-inf for
// masked entries, as staged).
__device__ __forceinline__ float lane_pairs(const __nv_bfloat16* xs, int i0, int n,
                                            float2 xp[4]) {
  if (i0 + 8 <= n) {
    const uint4 w = *reinterpret_cast<const uint4*>(xs + i0);
    xp[0] = make_float2(bf_lo(w.x), bf_hi(w.x));
    xp[1] = make_float2(bf_lo(w.y), bf_hi(w.y));
    xp[2] = make_float2(bf_lo(w.z), bf_hi(w.z));
    xp[3] = make_float2(bf_lo(w.w), bf_hi(w.w));
    return vec_max(w, (__nv_bfloat16*)nullptr);
  }
  float x[8];
  smem8(xs, i0, n, x);
  float m = -INFINITY;
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    xp[j] = make_float2(x[2 * j], x[2 * j + 1]);
    m = fmaxf(m, fmaxf(x[2 * j], x[2 * j + 1]));
  }
  return m;
}
__device__ __forceinline__ float lane_pairs(const float* xs, int i0, int n, float2 xp[4]) {
  float x[8];
  smem8(xs, i0, n, x);
  float m = -INFINITY;
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    xp[j] = make_float2(x[2 * j], x[2 * j + 1]);
    m = fmaxf(m, fmaxf(x[2 * j], x[2 * j + 1]));
  }
  return m;
}
// 2^k for an integer-valued k <= 0, built from its exponent bits (0 below
// the normal double range, where a term is negligible beside the largest).
__device__ __forceinline__ double pow2d(float k) {
  return k < -1022.0f ? 0.0 : __longlong_as_double((long long)(1023 + (int)k) << 52);
}

template <typename T>
__global__ void __launch_bounds__(kDecThreads, 2) draft_fused_kernel(DraftArgs A, int tc) {
  pdl_begin();
  asm volatile("barrier.cluster.arrive.relaxed;" ::: "memory");  // waited before remote writes
  cg::cluster_group cl = cg::this_cluster();
  const int rank = (int)cl.block_rank(), cs = (int)cl.num_blocks();
  extern __shared__ __align__(128) unsigned char dsm[];
  T* xs = reinterpret_cast<T*>(dsm);
  unsigned char* tiles = dsm + (size_t)tc * kResTile * sizeof(T);
  double* tsum = reinterpret_cast<double*>(tiles);           // S_t 2^(M_t - M_r)
  float* tm = reinterpret_cast<float*>(tsum + tc);           // m_t
  float* tM = tm + tc;                                       // M_t
  float* tS = tM + tc;                                       // S_t
  float* tT = tS + tc;                                       // T_t
  __shared__ __align__(8) uint64_t s_bar[kDfMaxChunks];
  __shared__ DfPart s_part[kDfMaxCluster];
  __shared__ float s_wm[kDecWarps];
  __shared__ int s_wi[kDecWarps];
  __shared__ DfPart s_mine;
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
  // The draw's uniform, formed now so that the combine does not wait for it.
  __shared__ float s_u;
  if (threadIdx.x == 0 && !greedy)
    s_u = spec_uniforms(A.seed, (uint32_t)A.seq_id[b], A.round, (uint32_t)A.pos[b], 0u).y;

  // Stage the slice: bulk copies of its 16-byte part in chunks of whole
  // tiles, plain loads of the rest (fewer than 16 bytes, at the slice's end).
  const uint32_t bytes = ((uint32_t)n * (uint32_t)sizeof(T)) & ~15u;
  const int nbulk = (int)(bytes / sizeof(T));
  const int nchunks = (int)((bytes + kDfChunk - 1) / kDfChunk);
  if (threadIdx.x == 0) {
    for (int c = 0; c < nchunks; ++c) mbar_init(&s_bar[c], 1);
    fence_barrier_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    const unsigned char* src = reinterpret_cast<const unsigned char*>(row + e0);
    for (int c = 0; c < nchunks; ++c) {
      const uint32_t o = (uint32_t)c * kDfChunk, len = min(kDfChunk, bytes - o);
      mbar_arrive_expect_tx(&s_bar[c], len);
      bulk_g2s(dsm + o, src + o, len, &s_bar[c]);
    }
  }
  for (int i = nbulk + (int)threadIdx.x; i < n; i += blockDim.x) xs[i] = row[e0 + i];
  __syncthreads();  // the plain-loaded end of the slice is in

  // One pass per tile as its chunk lands: the warp takes tiles warp, warp +
  // kDecWarps, ... in order, waiting for each chunk the first time it needs it.
  constexpr int kTilesPerChunk = (int)kDfChunk / (kResTile * (int)sizeof(T));
  int have = -1;  // chunks this warp has waited for
  bool late = false;
  float gv = -INFINITY;  // greedy rows: the warp's largest logit and its first index
  int gi = 0x7fffffff;
  for (int t = warp; t < nt; t += kDecWarps) {
    const int c = min(t / kTilesPerChunk, nchunks - 1);
    while (have < c) {
      ++have;
      if (!mbar_wait_bounded(&s_bar[have], 0, kWaitLimitNs)) {
        late = true;
        mbar_wait_bounded(&s_bar[have], 0, kWaitLimitNs);  // let the copy land before going on
      }
    }
    if (greedy) {
      float x[8];
      smem8(xs, t * kResTile + lane * 8, n, x);
      float v = -INFINITY;
      int i = 0x7fffffff;
#pragma unroll
      for (int e = 0; e < 8; ++e)
        if (x[e] > v) { v = x[e]; i = e0 + t * kResTile + lane * 8 + e; }
      warp_argmax(v, i);
      if (v > gv) { gv = v; gi = i; }  // tiles in index order: the first maximum stays
      continue;
    }
    float2 xp[4];
    const float tile_max = lane_pairs(xs, t * kResTile + lane * 8, n, xp);
    float lm;  // the tile's largest logit in every lane: one warp reduction (sm_100a)
    asm volatile("redux.sync.max.f32 %0, %1, 0xffffffff;" : "=f"(lm) : "f"(tile_max));
    float S = 0.0f, Tm = 0.0f, Mt = 0.0f;
    if (lm > -INFINITY && lm < INFINITY) {  // a finite element (the same in every lane)
      Mt = ceilf(lm * sc.hi);
      // Packed: two FMAs form each pair's exponents, one ex2 per element, the
      // sums and the first moment about lm (x - lm held at -FLT_MAX for a
      // masked entry, whose term 0 must contribute 0).
      const float2 chi2 = make_float2(sc.hi, sc.hi), clo2 = make_float2(sc.lo, sc.lo);
      const float2 nM2 = make_float2(-Mt, -Mt), nm2 = make_float2(-lm, -lm);
      float2 s2 = make_float2(0.0f, 0.0f), t2 = make_float2(0.0f, 0.0f);
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        float2 e = __ffma2_rn(xp[j], clo2, __ffma2_rn(xp[j], chi2, nM2));
        e = make_float2(ex2(e.x), ex2(e.y));
        s2 = __fadd2_rn(s2, e);
        float2 d = __fadd2_rn(xp[j], nm2);
        d = make_float2(fmaxf(d.x, -FLT_MAX), fmaxf(d.y, -FLT_MAX));
        t2 = __ffma2_rn(e, d, t2);
      }
      S = s2.x + s2.y;  // fp32 over the tile: 256 terms, each at most 1
      float mom = t2.x + t2.y;
#pragma unroll
      for (int o = 16; o; o >>= 1) {
        S += __shfl_xor_sync(0xffffffffu, S, o);
        mom += __shfl_xor_sync(0xffffffffu, mom, o);
      }
      Tm = mom;
    }
    if (lane == 0) {
      tm[t] = lm;
      tM[t] = Mt;
      tS[t] = S;
      tT[t] = Tm;
    }
  }
  if (late && lane == 0) set_status(A.status, SPEC_ETIMEOUT);
  if (greedy && lane == 0) { s_wm[warp] = gv; s_wi[warp] = gi; }
  __syncthreads();

  // The slice's summary (warp 0): largest logit, largest shift, and the tile
  // sums rescaled to it by exact powers of two.
  if (warp == 0) {
    DfPart me{-INFINITY, 0.0f, 0x7fffffff, 0.0, 0.0};
    if (greedy) {
      float v = lane < kDecWarps ? s_wm[lane] : -INFINITY;
      int i = lane < kDecWarps ? s_wi[lane] : 0x7fffffff;
      warp_argmax(v, i);
      me.m = v;
      me.amax = i;
    } else {
      float m = -INFINITY, M = -INFINITY;
      for (int t = lane; t < nt; t += 32) {
        m = fmaxf(m, tm[t]);
        if (tS[t] > 0.0f) M = fmaxf(M, tM[t]);
      }
#pragma unroll
      for (int o = 16; o; o >>= 1) {
        m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
        M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
      }
      double Sr = 0.0, Tr = 0.0;
      for (int t = lane; t < nt; t += 32) {
        double st = 0.0;
        if (tS[t] > 0.0f) {
          const double f = pow2d(tM[t] - M);
          st = (double)tS[t] * f;
          Tr += ((double)tT[t] + ((double)tm[t] - (double)m) * (double)tS[t]) * f;
        }
        tsum[t] = st;
        Sr += st;
      }
      me.m = m;
      me.M = M > -INFINITY ? M : 0.0f;
      me.S = warp_sum_d(Sr);
      me.T = warp_sum_d(Tr);
    }
    if (lane == 0) s_mine = me;
  }
  __syncthreads();

  // Every CTA's summary to every CTA, then the same combine everywhere.
  asm volatile("barrier.cluster.wait;" ::: "memory");
  if (threadIdx.x < cs) {
    DfPart* dst = cl.map_shared_rank(s_part, (unsigned)threadIdx.x);
    dst[rank] = s_mine;
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
      float Mc = -INFINITY;
      for (int r = 0; r < cs; ++r)
        if (s_part[r].S > 0.0) Mc = fmaxf(Mc, s_part[r].M);
      double f[kDfMaxCluster];
      double S = 0.0, Tm = 0.0;
      for (int r = 0; r < cs; ++r) {
        f[r] = 0.0;
        if (s_part[r].S > 0.0) {
          f[r] = pow2d(s_part[r].M - Mc);
          S += s_part[r].S * f[r];
          Tm += (s_part[r].T + ((double)s_part[r].m - (double)m) * s_part[r].S) * f[r];
        }
      }
      // Lt = Mc + log2 S; H = ln2 (Lt - c E[l]) with E[l] = m + Tm / S.
      const double Mcm = ((double)Mc - (double)m * (double)sc.hi) - (double)m * (double)sc.lo;
      const double l2S = log2(S);
      s_Lt = (double)Mc + l2S;
      s_H = kLn2 * (Mcm + l2S - sc.d * (Tm / S));
      const double target = (double)s_u * S;
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
  // lane, then a scan over the lanes), then the element, with the tile's own
  // shift and the same rescaling as its sum.
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
    const double ft = pow2d(tM[tile] - s_part[owner].M);
    float2 xp[4];
    lane_pairs(xs, tile * kResTile + lane * 8, n, xp);
    float w[8];
    {
      const float2 chi2 = make_float2(sc.hi, sc.hi), clo2 = make_float2(sc.lo, sc.lo);
      const float2 nM2 = make_float2(-tM[tile], -tM[tile]);
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const float2 e = __ffma2_rn(xp[j], clo2, __ffma2_rn(xp[j], chi2, nM2));
        w[2 * j] = ex2(e.x);
        w[2 * j + 1] = ex2(e.y);
      }
    }
    const double ls = lane_sum8(w) * ft;
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
        acc += (double)w[e] * ft;
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
  const size_t smem = (size_t)tc * kResTile * sizeof(T) + (size_t)tc * kDfTileBytes;
  const cudaError_t e = reserve_dyn_smem(k, smem);
  if (e != cudaSuccess) return e;
  return launch_pdl_cluster(k, dim3(cs, a.B), dim3(kDecThreads), smem, st, (unsigned)cs, a, tc);
}

cudaError_t launch_draft_step(int dtype, const unsigned char* lg, long long ld_bytes, int B, int V,
                              const float* temperature, uint64_t seed, const int32_t* seq_id,
                              uint32_t round, const int32_t* pos, Partial* part, double* mom,
                              int32_t* out_tok, double* out_logq, double* out_entropy,
                              int32_t* status, cudaStream_t st) {
  // One launch when a cluster of up to 8 CTAs holds the row in shared memory:
  // clusters of 1 or 2 CTAs when that slice fits and either the grid still
  // gives every SM a CTA or the slice is at most kDfSmallSlice tiles, else the
  // smallest of 4 and 8 that fits. (B200, bf16 rows: 256 x 32000 takes 14.2 us
  // per call with clusters of 1, 18.1 with 2, 26.2 with 4; 64 x 32000 10.3,
  // 8.2 and 7.6; 8 x 4096 6.0, 6.2 and 6.4; the same tokens at every size.)
  const int esz = dtype == SPEC_BF16 ? 2 : 4, nrt = residual_tiles(V);
  const int sms = sm_count();
  for (int cs = 1; cs <= kDfMaxCluster; cs *= 2) {
    const int tc = (nrt + cs - 1) / cs;
    if ((size_t)tc * kResTile * esz > (size_t)kDfSliceBytes) continue;
    if (cs < 4 && !((long long)B * cs >= sms || tc <= kDfSmallSlice)) continue;
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
