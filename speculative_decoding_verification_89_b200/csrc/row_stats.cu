// Row statistics: for every logit row the verification needs, the maximum,
// its first index and the sum of exponentials at temperature T, as partial
// statistics over runs of consecutive vocabulary tiles.
//
// Step "temperature softmax over V" behind every check of HiSpec
// (gist.science summary of arXiv 2510.01336, section 2: the three exits L_d,
// L_i, L_f each give a token distribution; "Verlustfreie Garantie" compares
// them). p = softmax(l / T) needs max and sum over the whole vocabulary row.
//
// Design (B200): a persistent grid, one CTA of kRsWarps warps per SM. The
// rows that need statistics (not the draft rows of greedy sequences, not the
// slots outside a window) are first listed in shared memory; their
// (row, tile) items are then dealt out as one contiguous run per warp, so a
// warp changes row at most a few times. Each warp owns a ring of kRsStages
// tile buffers filled by 1-D bulk copies (TMA engine, no tensor map, no
// multicast) that complete on per-stage mbarriers. Per lane, the largest
// logit and the sum of 2^(l*c - M) are carried across the tiles of a row with
// an integral shift M that follows the lane's largest element (moved by exact
// powers of two), so a tile costs no warp shuffle and no division; the lanes
// are combined once per row run into one Partial at the run's first tile (its
// other tiles get empty partials).
#include "common.cuh"
#include "kernels.cuh"
#include "rowmath.cuh"

namespace specv {

// Limit of the waits for this kernel's tile copies: kWaitLimitNs unless a
// test has set another with spec_test_set_wait_limit_ns (0: one non-blocking
// test per wait, so a copy still in flight makes the wait run out). The
// drain of the copies in flight after a timeout always uses kWaitLimitNs.
__device__ unsigned long long g_rs_wait_limit_ns = kWaitLimitNs;

// A launch lists at most kMaxListRows rows (the host splits larger calls).
constexpr int kMaxListRows = 8192;
constexpr int kRsSmemTotal = kRsSmem + kMaxListRows * (int)sizeof(int);
static_assert(kRsSmemTotal <= 227 * 1024, "row list and ring exceed shared memory");

template <typename T, typename Rows>
__global__ void __launch_bounds__(kRsWarps * 32, 1)
    row_stats_kernel(Rows rows, int row_base, int nrows, int V, Partial* __restrict__ part,
                     double* __restrict__ mom, int32_t* status, int32_t* zero_word) {
  extern __shared__ __align__(128) unsigned char smem[];
  __shared__ int s_wsum[kRsWarps];
  constexpr int kVec = VecOf<T>::n;
  constexpr int kEpt = kTileBytes / (int)sizeof(T);     // elements per tile
  constexpr int kVpl = kTileBytes / 16 / 32;            // vectors per lane
  constexpr int kThreads = kRsWarps * 32;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  unsigned char* wbuf = smem + (size_t)warp * kRsStages * kTileBytes;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + (size_t)kRsWarps * kRsStages * kTileBytes) +
                   warp * kRsStages;
  int* s_list = reinterpret_cast<int*>(smem + kRsSmem);
  if (lane == 0) {
    for (int s = 0; s < kRsStages; ++s) mbar_init(&bars[s], 1);
    fence_barrier_init();
  }
  pdl_begin();
  if (zero_word && blockIdx.x == 0 && threadIdx.x == 0) *zero_word = 0;

  // The rows that need statistics: the early ones in order, then the late
  // ones in order. Each thread tests a contiguous run of at most 32 rows; a
  // block scan of the packed counts (early | late << 16) places them.
  int n_early = 0, n_late = 0;
  {
    const int per = (nrows + kThreads - 1) / kThreads;
    const int q0 = min(nrows, (int)threadIdx.x * per), q1 = min(nrows, q0 + per);
    uint32_t vmask = 0, lmask = 0;
    int cnt = 0;
    for (int q = q0; q < q1; ++q)
      if (rows.get(row_base + q).valid) {
        vmask |= 1u << (q - q0);
        if (rows.late(row_base + q)) {
          lmask |= 1u << (q - q0);
          cnt += 1 << 16;
        } else {
          cnt += 1;
        }
      }
    int incl = cnt;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += y;
    }
    if (lane == 31) s_wsum[warp] = incl;
    __syncthreads();
    int pos = incl - cnt, tot = 0;
    for (int w = 0; w < kRsWarps; ++w) {
      if (w < warp) pos += s_wsum[w];
      tot += s_wsum[w];
    }
    n_early = tot & 0xffff;
    n_late = tot >> 16;
    int pe = pos & 0xffff, pl = n_early + (pos >> 16);
    for (int q = q0; q < q1; ++q)
      if ((vmask >> (q - q0)) & 1u) s_list[((lmask >> (q - q0)) & 1u) ? pl++ : pe++] = q;
  }
  __syncthreads();

  // This warp's items: a contiguous share of the early rows' (listed row,
  // tile) items, then a contiguous share of the late rows' items.
  const int ntiles = (V + kEpt - 1) / kEpt;
  const int gw = blockIdx.x * kRsWarps + warp, nw = gridDim.x * kRsWarps;
  const long long ne = (long long)n_early * ntiles, nl = (long long)n_late * ntiles;
  const long long e0 = ne * gw / nw, e1 = ne * (gw + 1) / nw;
  const long long l0 = ne + nl * gw / nw, l1 = ne + nl * (gw + 1) / nw;
  struct Cursor {
    int k, t, left, seg;  // listed row, tile, items left in segment, segment
  };
  auto start = [&](Cursor& c, long long i, long long n, int seg) {
    c.k = (int)(i / ntiles);
    c.t = (int)(i - (long long)c.k * ntiles);
    c.left = (int)n;
    c.seg = seg;
  };
  auto begin = [&](Cursor& c) {
    start(c, e0, e1 - e0, 0);
    if (c.left == 0) start(c, l0, l1 - l0, 1);
  };
  auto advance = [&](Cursor& c) {
    if (++c.t == ntiles) { c.t = 0; ++c.k; }
    if (--c.left == 0 && c.seg == 0) start(c, l0, l1 - l0, 1);
  };
  // Streamed-once lines make room first when late rows are to stay in L2.
  const bool hint = n_late > 0;
  const uint64_t pol = l2_evict_first();

  // Producer: lane 0 issues the copies, every lane keeps the cursor.
  Cursor pc;
  begin(pc);
  int pk_row = -1;
  const unsigned char* pptr = nullptr;
  auto issue = [&](int st) {
    if (pc.k != pk_row) {
      pk_row = pc.k;
      pptr = rows.get(row_base + s_list[pc.k]).ptr;
    }
    if (lane == 0) {
      const int nel = min(kEpt, V - pc.t * kEpt);
      const uint32_t bytes = ((uint32_t)nel * sizeof(T)) & ~15u;
      fence_proxy_async_smem();  // the warp's reads of this stage come first
      mbar_arrive_expect_tx(&bars[st], bytes);
      const unsigned char* src = pptr + (size_t)pc.t * kTileBytes;
      if (bytes) {
        if (hint && pc.seg == 0)
          bulk_g2s_hint(wbuf + st * kTileBytes, src, bytes, &bars[st], pol);
        else
          bulk_g2s(wbuf + st * kTileBytes, src, bytes, &bars[st]);
      }
    }
    advance(pc);
  };
  int inflight = 0;
  for (int st = 0; st < kRsStages && pc.left > 0; ++st) {
    issue(st);
    ++inflight;
  }

  // Consumer state of the current row run (per lane).
  Cursor cc;
  begin(cc);
  bool fresh = true;  // the next item starts a row run
  uint32_t phase = 0;
  bool timed_out = false;
  int s = 0;  // stage of the item being consumed
  int row = 0, run_t0 = 0;
  const T* rptr = nullptr;
  bool greedy = false;
  float chi = 0.0f, clo = 0.0f;
  float mrun = -INFINITY;    // largest logit of the lane in the run
  float anchor = -INFINITY;  // the logit that set the shift
  float Msh = 0.0f;          // shift fl(anchor * chi)
  double acc = 0.0;          // sum of 2^(l*c - Msh) over the lane's elements
  double acc1 = 0.0;         // sum of 2^(l*c - Msh) * (l - anchor) (Rows::kEntropy)
  int gidx = 0x7fffffff;     // greedy rows: first index of mrun

  const uint64_t wait_limit = g_rs_wait_limit_ns;
  for (; cc.left > 0; s = (s + 1 == kRsStages) ? 0 : s + 1) {
    const bool ok = mbar_wait_bounded(&bars[s], (phase >> s) & 1u, wait_limit);
    if (__any_sync(0xffffffffu, !ok)) {
      timed_out = true;
      break;
    }
    phase ^= 1u << s;
    --inflight;

    const int ct = cc.t;
    if (fresh) {  // a row run starts
      fresh = false;
      row = row_base + s_list[cc.k];
      const RowRef ref = rows.get(row);
      rptr = reinterpret_cast<const T*>(ref.ptr);
      greedy = (ref.T == 0.0f);
      if (!greedy) {
        const Scale sc = make_scale(ref.T);
        chi = sc.hi;
        clo = sc.lo;
      }
      run_t0 = ct;
      mrun = anchor = -INFINITY;
      Msh = 0.0f;
      acc = 0.0;
      acc1 = 0.0;
      gidx = 0x7fffffff;
    }

    // The lane's vectors of the staged tile go to registers; the stage is
    // refilled before the arithmetic starts. Past the row's end the vectors
    // read as -inf; a tail of fewer than 16 bytes comes from global memory.
    const int nel = min(kEpt, V - ct * kEpt);
    const uint4* buf = reinterpret_cast<const uint4*>(wbuf + s * kTileBytes);
    uint4 x[kVpl];
    int nvec = kEpt / kVec, ntail = 0;
    float tailx = -INFINITY;
    if (nel == kEpt) {
#pragma unroll
      for (int i = 0; i < kVpl; ++i) x[i] = buf[lane + 32 * i];
    } else {
      nvec = (int)(((uint32_t)nel * sizeof(T)) >> 4);
      ntail = nel - nvec * kVec;
#pragma unroll
      for (int i = 0; i < kVpl; ++i) {
        const int v = lane + 32 * i;
        x[i] = v < nvec ? buf[v] : neg_inf_vec<T>();
      }
      if (lane < ntail) tailx = load_elem(rptr + (size_t)ct * kEpt + nvec * kVec + lane);
    }
    __syncwarp();
    if (pc.left > 0) {
      issue(s);
      ++inflight;
    }

    if (greedy) {
      // First index of the lane's largest element: vectors in index order,
      // strict comparisons keep the earliest.
      float tb = -INFINITY;
      int bv = -1;
#pragma unroll
      for (int i = 0; i < kVpl; ++i) {
        const float vm = vec_max(x[i], (T*)nullptr);
        if (vm > tb) { tb = vm; bv = i; }
      }
      if (tb > mrun) {
        uint4 w = x[0];
#pragma unroll
        for (int i = 1; i < kVpl; ++i)
          if (i == bv) w = x[i];
        int ef = 0;
#pragma unroll
        for (int e = kVec - 1; e >= 0; --e)
          if (vec_elem(w, e, (T*)nullptr) == tb) ef = e;
        mrun = tb;
        gidx = ct * kEpt + (lane + 32 * bv) * kVec + ef;
      }
      if (tailx > mrun) {
        mrun = tailx;
        gidx = ct * kEpt + nvec * kVec + lane;
      }
    } else {
      const float tm = fmaxf(regs_max<kVpl>(x, (T*)nullptr), tailx);
      if (tm > mrun) mrun = tm;
      // The lane's shift is an integer at or just above its largest scaled
      // element, moved (by an exact power of two) as soon as an element
      // passes it: the largest terms have exponents in (-1, 0], where fp32
      // rounds them least.
      const float Mn = ceilf(tm * chi);
      if (tm > -INFINITY && (!(anchor > -INFINITY) || Mn > Msh)) {
        if (acc != 0.0) {
          const double f = pow2i(Msh - Mn);
          if constexpr (Rows::kEntropy) acc1 = (acc1 + ((double)anchor - (double)tm) * acc) * f;
          acc *= f;
        }
        anchor = tm;
        Msh = Mn;
      }
      const bool has = anchor > -INFINITY;
      float a = 0.0f, a1s = 0.0f;
      if (__all_sync(0xffffffffu, !has || fabsf(Msh) < kFarShift)) {
        if (has) {
          const float2 chi2 = make_float2(chi, chi), clo2 = make_float2(clo, clo);
          const float2 nM2 = make_float2(-Msh, -Msh);
          float2 a0 = make_float2(0.0f, 0.0f), a1 = make_float2(0.0f, 0.0f);
          if constexpr (Rows::kEntropy) {
            const float2 nA2 = make_float2(-anchor, -anchor);
            float2 t0 = make_float2(0.0f, 0.0f);
#pragma unroll
            for (int i = 0; i < kVpl; ++i) {
              float2 t;
              a0 = __fadd2_rn(a0, vec_expsum_ent(x[i], chi2, clo2, nM2, nA2, &t, (T*)nullptr));
              t0 = __fadd2_rn(t0, t);
            }
            a1s = t0.x + t0.y;
          } else {
#pragma unroll
            for (int i = 0; i < kVpl; i += 2) {
              a0 = __fadd2_rn(a0, vec_expsum(x[i], chi2, clo2, nM2, (T*)nullptr));
              if (i + 1 < kVpl)
                a1 = __fadd2_rn(a1, vec_expsum(x[i + 1], chi2, clo2, nM2, (T*)nullptr));
            }
          }
          const float2 a2 = __fadd2_rn(a0, a1);
          a = a2.x + a2.y;
          if (lane < ntail) {
            const float e = term(tailx, chi, clo, -Msh);
            a += e;
            if constexpr (Rows::kEntropy) a1s += e * dev1(tailx, anchor);
          }
        }
      } else if (has) {
        const float rr = fmaf(anchor, chi, -Msh) + anchor * clo;
        if constexpr (Rows::kEntropy) {
#pragma unroll
          for (int i = 0; i < kVpl; ++i) {
#pragma unroll
            for (int e = 0; e < kVec; ++e) {
              const float xv = vec_elem(x[i], e, (T*)nullptr);
              const float te = term_far(xv, anchor, chi, clo, rr);
              a += te;
              a1s += te * dev1(xv, anchor);
            }
          }
        } else {
#pragma unroll
          for (int i = 0; i < kVpl; ++i) a += vec_expsum_far<T>(x[i], anchor, chi, clo, rr);
        }
        if (lane < ntail) {
          const float te = term_far(tailx, anchor, chi, clo, rr);
          a += te;
          if constexpr (Rows::kEntropy) a1s += te * dev1(tailx, anchor);
        }
      }
      acc += (double)a;
      if constexpr (Rows::kEntropy) acc1 += (double)a1s;
    }

    // End of the row, of a segment or of this warp's items: one Partial for
    // the run.
    const int t_last = ct, k_was = cc.k;
    advance(cc);
    if (cc.k != k_was || cc.left == 0) {
      fresh = true;
      Partial p;
      if (greedy) {
        float v = mrun;
        int i = gidx;
        warp_argmax(v, i);
        p.m = v;
        p.idx = i;
        p.s = 0.0;
      } else {
        float m = mrun;
#pragma unroll
        for (int o = 16; o; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
        double sl = 0.0, tl = 0.0;
        if (m > -INFINITY && m < INFINITY && acc != 0.0) {
          const double f = exp2((double)Msh - (double)__fmul_rn(m, chi));
          sl = acc * f;
          // moment about the run's maximum m
          if constexpr (Rows::kEntropy) tl = (acc1 + ((double)anchor - (double)m) * acc) * f;
        }
        p.m = m;
        p.idx = 0x7fffffff;
        p.s = warp_sum_d(sl);
        if constexpr (Rows::kEntropy) tl = warp_sum_d(tl);
        if (Rows::kEntropy && lane == 0) mom[(size_t)row * ntiles + run_t0] = tl;
      }
      Partial* prow = part + (size_t)row * ntiles;
      if (lane == 0) prow[run_t0] = p;
      for (int t = run_t0 + 1 + lane; t <= t_last; t += 32) {
        prow[t] = Partial{-INFINITY, 0x7fffffff, 0.0};
        if constexpr (Rows::kEntropy) mom[(size_t)row * ntiles + t] = 0.0;
      }
    }
  }

  if (timed_out) {
    if (lane == 0) set_status(status, SPEC_ETIMEOUT);
    // Let copies still in flight land before the CTA's shared memory goes:
    // stages s, s+1, ... hold the `inflight` copies not yet consumed.
    for (int j = 0; j < inflight; ++j) {
      const int q = (s + j) % kRsStages;
      mbar_wait_bounded(&bars[q], (phase >> q) & 1u, kWaitLimitNs);
    }
  }
}

// ----------------------------------------------------------------------------
// Launchers
// ----------------------------------------------------------------------------
template <typename T, typename Rows>
static cudaError_t launch_rs(const Rows& rows, int nrows, int V, Partial* part, double* mom,
                             int32_t* zero_word, int32_t* status, cudaStream_t st) {
  auto kern = row_stats_kernel<T, Rows>;
  {
    const cudaError_t e = reserve_dyn_smem(kern, (size_t)kRsSmemTotal);
    if (e != cudaSuccess) return e;
  }
  constexpr int kEpt = kTileBytes / (int)sizeof(T);
  const long long ntiles = (V + kEpt - 1) / kEpt;
  for (int r0 = 0; r0 < nrows; r0 += kMaxListRows) {
    const int n = nrows - r0 < kMaxListRows ? nrows - r0 : kMaxListRows;
    const long long items = (long long)n * ntiles;
    long long grid = sm_count();
    const long long need = (items + kRsWarps - 1) / kRsWarps;
    if (grid > need) grid = need;
    if (grid < 1) grid = 1;
    const cudaError_t e = launch_pdl(kern, dim3((unsigned)grid), dim3(kRsWarps * 32),
                                     (size_t)kRsSmemTotal, st, rows, r0, n, V, part, mom, status,
                                     zero_word);
    if (e != cudaSuccess) return e;
  }
  return cudaSuccess;
}

template <typename Rows>
cudaError_t launch_row_stats(int dtype, const Rows& rows, int nrows, int V, const RsBuffers& b,
                             int32_t* status, cudaStream_t st) {
  if (dtype == SPEC_BF16)
    return launch_rs<__nv_bfloat16>(rows, nrows, V, b.part, b.mom, b.zero, status, st);
  return launch_rs<float>(rows, nrows, V, b.part, b.mom, b.zero, status, st);
}

}  // namespace specv

#pragma GCC visibility push(default)
extern "C" int spec_test_set_wait_limit_ns(uint64_t ns) {
  const unsigned long long v = ns;
  const cudaError_t e = cudaMemcpyToSymbol(specv::g_rs_wait_limit_ns, &v, sizeof(v));
  if (e != cudaSuccess) return specv::record_cuda_status(e);
  return SPEC_OK;
}
#pragma GCC visibility pop

namespace specv {

template cudaError_t launch_row_stats<ChainRows>(int, const ChainRows&, int, int,
                                                 const RsBuffers&, int32_t*, cudaStream_t);
template cudaError_t launch_row_stats<Hier1Rows>(int, const Hier1Rows&, int, int,
                                                 const RsBuffers&, int32_t*, cudaStream_t);
template cudaError_t launch_row_stats<Hier2Rows>(int, const Hier2Rows&, int, int,
                                                 const RsBuffers&, int32_t*, cudaStream_t);
template cudaError_t launch_row_stats<DraftRows>(int, const DraftRows&, int, int,
                                                 const RsBuffers&, int32_t*, cudaStream_t);

}  // namespace specv
