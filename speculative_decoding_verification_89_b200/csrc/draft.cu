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
// Two launches: the row-statistics kernel over the B rows (DraftRows, which
// also gathers the first moment sum 2^(l*c - M) * (l - m)), then one
// thread-block cluster per sequence that combines its row, and -- unless the
// sequence is greedy -- splits the row's 256-element tiles of p over the
// cluster, prefixes their sums in the leader and draws by inverse CDF with the
// lane-1 uniform of the Philox counter (seq_id, round, pos, 0).
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
  if (!temp_valid(Tb)) {  // the same verdict in every CTA of the cluster
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
  const ProbCoef kp = make_coef(st.Lt, sc);
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

template <typename T>
static cudaError_t launch_draw(const DraftArgs& a, cudaStream_t st) {
  auto k = draft_draw_kernel<T>;
  const size_t smem = 2 * (size_t)residual_tiles(a.V) * sizeof(double);
  const cudaError_t e = reserve_dyn_smem(k, smem);
  if (e != cudaSuccess) return e;
  return launch_pdl_cluster(k, dim3(kCluster, a.B), dim3(kDecThreads), smem, st, kCluster, a);
}

cudaError_t launch_draft_step(int dtype, const unsigned char* lg, long long ld_bytes, int B, int V,
                              const float* temperature, uint64_t seed, const int32_t* seq_id,
                              uint32_t round, const int32_t* pos, Partial* part, double* mom,
                              int32_t* out_tok, double* out_logq, double* out_entropy,
                              int32_t* status, cudaStream_t st) {
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
