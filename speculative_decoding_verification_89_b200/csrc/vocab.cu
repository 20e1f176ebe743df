// Vocabulary-parallel chain verification: each of R ranks holds one
// contiguous shard [v0, v0 + Vs) of every target and draft row (the output
// of a vocabulary-parallel LM head) and the check runs without gathering any
// row. Everything the check needs is a sum or a maximum over the vocabulary
// -- the partition functions, the argmax of greedy rows, the residual mass --
// or a single logit (the drafted token's), so per row and rank a 32-byte
// record suffices, and for the draw one mass per sequence and rank:
//
//   1. records (after the row-statistics kernel on the shard rows): the
//      shard's max, argmax, shifted sum and, where the shard holds it, the
//      drafted token's logit;                      -> all-gather (rank order)
//   2. decide: every rank combines the R records of each row (the same
//      arithmetic in every rank, so every rank reaches the same accepted
//      count a), writes the probabilities, and sums the draw weights
//      (max(0, p - q) at a rejection, p for the bonus token) over its shard
//      of the row pair at a;                       -> all-gather (rank order)
//   3. pick: every rank prefixes the R masses in rank order and finds the
//      shard holding u * Z; that rank alone draws inside its shard (the
//      single-GPU tile sums, prefix and rescan, with the target less the
//      masses of the shards before it); all ranks write the accepted drafts
//      and -1 at the drawn position unless they drew it.
//                                                  -> max-reduce of out_tok
//
// The exchanges between the launches are the caller's collectives (NCCL over
// NVLink in a multi-GPU job); together they carry 32 (2K+1) + 16 bytes plus
// 4 (K+1) bytes of tokens per sequence and rank, against 2 (2K+1) Vs bytes
// of logits each rank reads.
//
// Rules: speculative sampling as appealed to by HiSpec (gist.science summary
// of arXiv 2510.01336, section 2, "Verlustfreie Garantie"); the residual
// proportional to the target-minus-draft difference (Speculative Speculative
// Decoding summary, Technische Zusammenfassung 3.B). The split over the
// vocabulary changes the order of the sums only.
#include "draw.cuh"

namespace specv {

constexpr int kVpMaxRows = 2 * SPEC_MAX_K + 1;
constexpr int kVpRecWarps = 8;

// ---------------------------------------------------------------------------
// 1. Shard records
// ---------------------------------------------------------------------------
template <typename T>
__global__ void __launch_bounds__(kVpRecWarps * 32) vp_records_kernel(VpArgs A) {
  pdl_begin();
  const int lane = threadIdx.x & 31, K = A.K, per = 2 * K + 1;
  const long long r = (long long)blockIdx.x * kVpRecWarps + (threadIdx.x >> 5);
  if (r >= (long long)A.B * per) return;
  const int b = (int)(r / per), j = (int)(r - (long long)b * per);
  const float Tb = A.temperature[b];
  const bool greedy = (Tb == 0.0f);
  VpRow out{0.0, 0.0, -INFINITY, INT_MAX, 0.0f, 0};
  if (temp_valid(Tb) && (j <= K || !greedy)) {
    const float chi = greedy ? 0.0f : make_scale(Tb).hi;
    const Partial* p = A.part + r * A.ntiles;
    double s = 0.0;
    const RowFinal f = combine_row(p, A.ntiles, greedy, chi, lane, &s);
    bool bad = false;
    for (int t = lane; t < A.ntiles; t += 32) {
      const Partial q = p[t];
      bad |= isnan(q.m) || q.m == INFINITY || isnan(q.s) || q.s == INFINITY;
    }
    bad = __any_sync(0xffffffffu, bad);
    if (f.m > -INFINITY) {
      out.m = f.m;
      out.amax = A.v0 + f.amax;
      out.M = f.M;
      out.S = s;
    }
    if (bad || isnan(f.m)) out.flags |= kVpBad;
    if (!greedy && j != K) {  // the drafted token's logit, where this shard holds it
      const int jj = j < K ? j : j - K - 1;
      const int x = A.draft_tok[(size_t)b * K + jj];
      if (x >= A.v0 && x - A.v0 < A.Vs) {
        const T* row = j < K ? row_ptr<T>(A.tgt, A.ld_tgt, (long long)b * (K + 1) + j)
                             : row_ptr<T>(A.drf, A.ld_drf, (long long)b * K + jj);
        out.x = load_elem(row + (x - A.v0));
        out.flags |= kVpHasX;
      }
    }
  }
  if (lane == 0) A.rows[r] = out;
}

// ---------------------------------------------------------------------------
// 2. Combine, accept test, shard weights of the draw
// ---------------------------------------------------------------------------
struct VpShared {
  double M[kVpMaxRows], L[kVpMaxRows];
  float m[kVpMaxRows], x[kVpMaxRows];
  int amax[kVpMaxRows], flags[kVpMaxRows];  // bit 0: row ok; bit 1: x known
};

template <typename T>
__global__ void __launch_bounds__(kDecThreads) vp_decide_kernel(VpArgs A) {
  pdl_begin();
  __shared__ VpShared sh;
  __shared__ int s_a, s_bad;
  __shared__ float s_u;
  const int b = blockIdx.x, K = A.K, per = 2 * K + 1, B = A.B;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const float Tb = A.temperature[b];
  const bool greedy = (Tb == 0.0f);
  VpSeq* st = A.seq + b;
  if (!temp_valid(Tb)) {
    if (threadIdx.x == 0) {
      st->state = kVpSeqBad;
      A.mass[b] = VpMass{0.0, 0.0};
    }
    return;
  }
  const Scale sc = greedy ? Scale{0.f, 0.f, 0.0} : make_scale(Tb);
  auto rec = [&](int q, int r) -> const VpRow& {
    return A.rows_all[((size_t)q * B + b) * per + r];
  };
  // A warp per row: the rank records combined in rank order.
  for (int r = warp; r < per; r += kDecWarps) {
    if (greedy && r > K) {  // greedy checks read no draft row
      if (lane == 0) sh.flags[r] = 1;
      continue;
    }
    float mv = -INFINITY;
    int mi = INT_MAX, bad = 0;
    for (int q = lane; q < A.R; q += 32) {
      const VpRow& e = rec(q, r);
      if (e.m > mv || (e.m == mv && e.amax < mi)) { mv = e.m; mi = e.amax; }
      bad |= e.flags & kVpBad;
    }
    warp_argmax(mv, mi);
    bad = __any_sync(0xffffffffu, bad);
    bool ok = !bad && mv > -INFINITY && mv < INFINITY;
    double M = 0.0, L = 0.0;
    if (ok && !greedy) {
      M = (double)__fmul_rn(mv, sc.hi);
      double s = 0.0;
      for (int q = lane; q < A.R; q += 32) {
        const VpRow& e = rec(q, r);
        if (e.m > -INFINITY) s += e.S * exp2(e.M - M);
      }
      s = warp_sum_d(s);
      ok = (s > 0.0 && s < INFINITY);
      L = log2(s);
    }
    if (lane == 0) {
      int hx = 0;
      float xv = 0.0f;
      if (!greedy && r != K)
        for (int q = 0; q < A.R; ++q)
          if (rec(q, r).flags & kVpHasX) {
            hx = 1;
            xv = rec(q, r).x;
            break;
          }
      sh.M[r] = M;
      sh.L[r] = L;
      sh.m[r] = mv;
      sh.amax[r] = mi;
      sh.x[r] = xv;
      sh.flags[r] = (ok ? 1 : 0) | (hx ? 2 : 0);
    }
  }
  __syncthreads();
  double* diag = A.diag ? A.diag + (size_t)b * (4 * K + 2) : nullptr;
  // The accept test, a lane per position (warp 0).
  if (warp == 0) {
    int a = K, bad = 0;
    for (int r = lane; r < per; r += 32) bad |= !(sh.flags[r] & 1);
    for (int j0 = 0; j0 < K; j0 += 32) {
      const int j = j0 + lane;
      bool acc = true, badj = false;
      if (j < K) {
        const int x = A.draft_tok[(size_t)b * K + j];
        if (x < 0 || x >= A.V) {
          badj = true;
        } else if (greedy) {
          acc = (x == sh.amax[j]);
        } else if (!(sh.flags[j] & 2) || !(sh.flags[K + 1 + j] & 2)) {
          badj = true;  // no shard holds the drafted token
        } else {
          const double lp = (double)sh.x[j] * sc.d - (sh.M[j] + sh.L[j]);
          const double lq = (double)sh.x[K + 1 + j] * sc.d - (sh.M[K + 1 + j] + sh.L[K + 1 + j]);
          const float u = spec_uniforms(A.seed, (uint32_t)A.seq_id[b], A.round, (uint32_t)j, 1u).x;
          acc = (double)u < exp2(lp - lq);
          if (diag) {
            diag[2 * K + 1 + j] = exp2(lp);
            diag[3 * K + 1 + j] = exp2(lq);
          }
        }
      }
      if (__any_sync(0xffffffffu, badj)) bad = 1;
      const unsigned rej = __ballot_sync(0xffffffffu, j < K && !acc);
      if (rej && a == K) a = j0 + __ffs(rej) - 1;
    }
    bad = __any_sync(0xffffffffu, bad);
    if (lane == 0) {
      s_a = a;
      s_bad = bad;
      s_u = greedy ? 0.0f
                   : spec_uniforms(A.seed, (uint32_t)A.seq_id[b], A.round, (uint32_t)a, 1u).y;
    }
  }
  __syncthreads();
  const int a = s_a;
  if (s_bad || greedy) {
    if (threadIdx.x == 0) {
      st->a = a;
      st->state = s_bad ? kVpSeqBad : kVpSeqGreedy;
      st->tok = s_bad ? -1 : sh.amax[a];
      A.mass[b] = VpMass{0.0, 0.0};
    }
    return;
  }
  if (diag)
    for (int j = threadIdx.x; j < per; j += blockDim.x) diag[j] = (sh.M[j] + sh.L[j]) * kLn2;
  const double Lp = sh.M[a] + sh.L[a];
  const double Lq = a < K ? sh.M[K + 1 + a] + sh.L[K + 1 + a] : 0.0;
  const float mp = sh.m[a], mq = a < K ? sh.m[K + 1 + a] : 0.0f;
  const ProbCoef kp = make_coef(Lp, mp, sc), kq = make_coef(Lq, mq, sc);
  const T* prow = row_ptr<T>(A.tgt, A.ld_tgt, (long long)b * (K + 1) + a);
  const T* qrow = a < K ? row_ptr<T>(A.drf, A.ld_drf, (long long)b * K + a) : nullptr;
  const int nrt = residual_tiles(A.Vs);
  double* ts = A.tsum + (size_t)b * nrt;
  residual_tile_sums<T>(prow, qrow, A.Vs, kp, kq, 0, nrt, ts);
  __syncthreads();
  if (warp == 0) {
    double z = 0.0;
    for (int t = lane; t < nrt; t += 32) z += ts[t];
    z = warp_sum_d(z);
    if (lane == 0) {
      const VpRow& own = rec(A.rank, a);
      const double pm = own.m > -INFINITY ? own.S * exp2(own.M - Lp) : 0.0;
      A.mass[b] = VpMass{z, pm};
      // tok: the shard's own argmax of the target row, the token drawn if
      // this rank is chosen but its weights vanish in fp32.
      *st = VpSeq{Lp, Lq, mp, mq, s_u, a, kVpSeqDraw, own.amax};
    }
  }
}

// ---------------------------------------------------------------------------
// 3. The draw in the owning shard, outputs
// ---------------------------------------------------------------------------
template <typename T>
__global__ void __launch_bounds__(kDecThreads) vp_pick_kernel(VpArgs A) {
  pdl_begin();
  __shared__ int s_owner, s_usep;
  __shared__ double s_W, s_target;
  const int b = blockIdx.x, K = A.K, B = A.B;
  const VpSeq st = A.seq[b];
  int32_t* out = A.out_tok + (size_t)b * (K + 1);
  const int32_t* drafts = A.draft_tok + (size_t)b * K;
  double* diag = A.diag ? A.diag + (size_t)b * (4 * K + 2) : nullptr;
  if (st.state != kVpSeqDraw) {
    const bool bad = st.state == kVpSeqBad;
    const int a = bad ? -1 : st.a;
    for (int j = threadIdx.x; j <= K; j += blockDim.x)
      out[j] = j < a ? drafts[j] : (j == a ? st.tok : -1);
    if (diag)
      for (int j = threadIdx.x; j < 4 * K + 2; j += blockDim.x) diag[j] = dnan();
    if (threadIdx.x == 0) {
      A.accept_len[b] = a;
      if (bad) set_status(A.status, SPEC_EDEVICE);
    }
    return;
  }
  const int a = st.a;
  if (threadIdx.x == 0) {
    double Z = 0.0;
    for (int q = 0; q < A.R; ++q) Z += A.mass_all[(size_t)q * B + b].z;
    // p == q as computed leaves no residual: draw from p, as on one GPU.
    const int usep = !(Z > 0.0) && a < K;
    double W = Z;
    if (usep) {
      W = 0.0;
      for (int q = 0; q < A.R; ++q) W += A.mass_all[(size_t)q * B + b].p;
    }
    const double target = (double)st.u * W;
    // The last shard with mass whose prefix does not exceed the target.
    int owner = -1;
    double c = 0.0, cpre = 0.0;
    if (W > 0.0)
      for (int q = 0; q < A.R; ++q) {
        const VpMass& e = A.mass_all[(size_t)q * B + b];
        const double w = usep ? e.p : e.z;
        if (c <= target && w > 0.0) {
          owner = q;
          cpre = c;
        }
        c += w;
      }
    s_owner = owner;
    s_usep = usep;
    s_W = W;
    s_target = target - cpre;
  }
  __syncthreads();
  int tok = -1;
  if (s_owner == A.rank) {  // the same in every thread of the block
    const Scale sc = make_scale(A.temperature[b]);
    const ProbCoef kp = make_coef(st.Lp, st.mp, sc), kq = make_coef(st.Lq, st.mq, sc);
    const T* prow = row_ptr<T>(A.tgt, A.ld_tgt, (long long)b * (K + 1) + a);
    const T* qrow =
        (a < K && !s_usep) ? row_ptr<T>(A.drf, A.ld_drf, (long long)b * K + a) : nullptr;
    const int nrt = residual_tiles(A.Vs);
    double* ts = A.tsum + (size_t)b * nrt;
    if (s_usep) {
      residual_tile_sums<T>(prow, nullptr, A.Vs, kp, kq, 0, nrt, ts);
      __syncthreads();
    }
    double Zl;
    const int t = residual_pick<T>(prow, qrow, A.Vs, kp, kq, ts, A.pre + (size_t)b * nrt, nrt,
                                   st.u, &Zl, s_target);
    tok = t >= 0 ? A.v0 + t : st.tok;
  }
  for (int j = threadIdx.x; j <= K; j += blockDim.x)
    out[j] = j < a ? drafts[j] : (j == a ? tok : -1);
  if (threadIdx.x == 0) {
    A.accept_len[b] = a;
    if (diag) diag[4 * K + 1] = s_W;
  }
}

// ---------------------------------------------------------------------------
// Launchers
// ---------------------------------------------------------------------------
cudaError_t launch_vp_records(int dtype, const VpArgs& a, cudaStream_t st) {
  const long long rows = (long long)a.B * (2 * a.K + 1);
  if (rows == 0) return cudaSuccess;
  const dim3 grid((unsigned)((rows + kVpRecWarps - 1) / kVpRecWarps));
  if (dtype == SPEC_BF16)
    return launch_pdl(vp_records_kernel<__nv_bfloat16>, grid, dim3(kVpRecWarps * 32), 0, st, a);
  return launch_pdl(vp_records_kernel<float>, grid, dim3(kVpRecWarps * 32), 0, st, a);
}

cudaError_t launch_vp_decide(int dtype, const VpArgs& a, cudaStream_t st) {
  if (a.B == 0) return cudaSuccess;
  if (dtype == SPEC_BF16)
    return launch_pdl(vp_decide_kernel<__nv_bfloat16>, dim3(a.B), dim3(kDecThreads), 0, st, a);
  return launch_pdl(vp_decide_kernel<float>, dim3(a.B), dim3(kDecThreads), 0, st, a);
}

cudaError_t launch_vp_pick(int dtype, const VpArgs& a, cudaStream_t st) {
  if (a.B == 0) return cudaSuccess;
  if (dtype == SPEC_BF16)
    return launch_pdl(vp_pick_kernel<__nv_bfloat16>, dim3(a.B), dim3(kDecThreads), 0, st, a);
  return launch_pdl(vp_pick_kernel<float>, dim3(a.B), dim3(kDecThreads), 0, st, a);
}

}  // namespace specv
