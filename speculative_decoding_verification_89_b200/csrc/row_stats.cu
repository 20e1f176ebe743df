// Row statistics: for every logit row the verification needs, the running
// maximum, its first index and the sum of exponentials at temperature T,
// computed per 8 KiB vocabulary tile.
//
// Step "temperature softmax over V" behind every check of HiSpec
// (gist.science summary of arXiv 2510.01336, section 2: the three exits L_d,
// L_i, L_f each give a token distribution; "Verlustfreie Garantie" compares
// them). p = softmax(l / T) needs max and sum over the whole vocabulary row.
//
// Design (B200): a persistent grid; each warp owns a ring of kRsStages tile
// buffers in shared memory, filled by 1-D bulk copies (TMA engine, no tensor
// map, no multicast) that complete on per-stage mbarriers. A warp walks the
// (row, tile) items i = gw, gw + nw, ... so every SM streams; two passes over
// the staged tile (max with first index, then the sum of 2^((l - m) c)) and
// warp shuffles give one Partial per (row, tile). Rows that need no
// statistics (draft rows of greedy sequences, slots outside a window) are
// skipped without traffic.
#include "common.cuh"
#include "kernels.cuh"

namespace specv {

template <typename T> struct VecOf;
template <> struct VecOf<__nv_bfloat16> { static constexpr int n = 8; };
template <> struct VecOf<float> { static constexpr int n = 4; };

// Largest element of a 16-byte vector.
__device__ __forceinline__ float vec_max(uint4 w, __nv_bfloat16*) {
  __nv_bfloat162 a = __hmax2(*reinterpret_cast<__nv_bfloat162*>(&w.x),
                             *reinterpret_cast<__nv_bfloat162*>(&w.y));
  __nv_bfloat162 c = __hmax2(*reinterpret_cast<__nv_bfloat162*>(&w.z),
                             *reinterpret_cast<__nv_bfloat162*>(&w.w));
  a = __hmax2(a, c);
  return fmaxf(__low2float(a), __high2float(a));
}
__device__ __forceinline__ float vec_max(uint4 w, float*) {
  return fmaxf(fmaxf(__uint_as_float(w.x), __uint_as_float(w.y)),
               fmaxf(__uint_as_float(w.z), __uint_as_float(w.w)));
}
__device__ __forceinline__ float vec_elem(uint4 w, int e, __nv_bfloat16*) {
  const uint32_t word = e < 2 ? w.x : e < 4 ? w.y : e < 6 ? w.z : w.w;
  return (e & 1) ? bf_hi(word) : bf_lo(word);
}
__device__ __forceinline__ float vec_elem(uint4 w, int e, float*) {
  const uint32_t word = e == 0 ? w.x : e == 1 ? w.y : e == 2 ? w.z : w.w;
  return __uint_as_float(word);
}

// Largest element of a lane's register-resident vectors.
template <int kVpl>
__device__ __forceinline__ float regs_max(const uint4* x, __nv_bfloat16*) {
  __nv_bfloat162 m2 = __float2bfloat162_rn(-INFINITY);
#pragma unroll
  for (int i = 0; i < kVpl; ++i) {
    uint4 w = x[i];
    const __nv_bfloat162 a = __hmax2(*reinterpret_cast<__nv_bfloat162*>(&w.x),
                                     *reinterpret_cast<__nv_bfloat162*>(&w.y));
    const __nv_bfloat162 b = __hmax2(*reinterpret_cast<__nv_bfloat162*>(&w.z),
                                     *reinterpret_cast<__nv_bfloat162*>(&w.w));
    m2 = __hmax2(m2, __hmax2(a, b));
  }
  return fmaxf(__low2float(m2), __high2float(m2));
}
template <int kVpl>
__device__ __forceinline__ float regs_max(const uint4* x, float*) {
  float m = -INFINITY;
#pragma unroll
  for (int i = 0; i < kVpl; ++i) m = fmaxf(m, vec_max(x[i], (float*)nullptr));
  return m;
}

// Sum over one 16-byte vector of 2^(x*c - M) with c = chi + clo and M an
// exact fp32 shift: two packed FP32x2 FMAs per element pair form the
// exponent (the product x*chi - M is rounded once, relative to the small
// result), one MUFU ex2 per element, packed adds pairwise inside the vector.
__device__ __forceinline__ float2 expo2(float2 x, float2 chi, float2 clo, float2 nM) {
  return __ffma2_rn(x, clo, __ffma2_rn(x, chi, nM));
}
__device__ __forceinline__ float2 ex2x2(float2 a) { return make_float2(ex2(a.x), ex2(a.y)); }

__device__ __forceinline__ float2 vec_expsum(uint4 w, float2 chi, float2 clo, float2 nM,
                                             __nv_bfloat16*) {
  const float2 e0 = ex2x2(expo2(make_float2(bf_lo(w.x), bf_hi(w.x)), chi, clo, nM));
  const float2 e1 = ex2x2(expo2(make_float2(bf_lo(w.y), bf_hi(w.y)), chi, clo, nM));
  const float2 e2 = ex2x2(expo2(make_float2(bf_lo(w.z), bf_hi(w.z)), chi, clo, nM));
  const float2 e3 = ex2x2(expo2(make_float2(bf_lo(w.w), bf_hi(w.w)), chi, clo, nM));
  return __fadd2_rn(__fadd2_rn(e0, e1), __fadd2_rn(e2, e3));
}
__device__ __forceinline__ float2 vec_expsum(uint4 w, float2 chi, float2 clo, float2 nM, float*) {
  const float2 e0 =
      ex2x2(expo2(make_float2(__uint_as_float(w.x), __uint_as_float(w.y)), chi, clo, nM));
  const float2 e1 =
      ex2x2(expo2(make_float2(__uint_as_float(w.z), __uint_as_float(w.w)), chi, clo, nM));
  return __fadd2_rn(e0, e1);
}
// Scalar forms (one FMA pair per element): the same arithmetic without
// packing, for builds where pair formation costs more than it saves.
__device__ __forceinline__ float vec_expsum_s(uint4 w, float chi, float clo, float nM,
                                              __nv_bfloat16*) {
  const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
  float e[8];
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    const float lo = bf_lo(ws[q]), hi = bf_hi(ws[q]);
    e[2 * q] = ex2(fmaf(lo, clo, fmaf(lo, chi, nM)));
    e[2 * q + 1] = ex2(fmaf(hi, clo, fmaf(hi, chi, nM)));
  }
  return ((e[0] + e[1]) + (e[2] + e[3])) + ((e[4] + e[5]) + (e[6] + e[7]));
}
__device__ __forceinline__ float vec_expsum_s(uint4 w, float chi, float clo, float nM, float*) {
  float e[4];
  const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    const float x = __uint_as_float(ws[q]);
    e[q] = ex2(fmaf(x, clo, fmaf(x, chi, nM)));
  }
  return (e[0] + e[1]) + (e[2] + e[3]);
}

// Scalar form of one term (tail elements).
__device__ __forceinline__ float term(float x, float chi, float clo, float nM) {
  return ex2(fmaf(x, clo, fmaf(x, chi, nM)));
}

// Slow form for |M| >= 2^26, where 2^(m*c - M) itself could overflow:
// x*c - M = (x - m)*c + (m*chi - M) + m*clo with the product residual exact.
__device__ __forceinline__ float term_far(float x, float m, float chi, float clo, float rr) {
  const float d = x - m;
  return ex2(fmaf(d, chi, fmaf(d, clo, rr)));
}
template <typename T>
__device__ __forceinline__ float vec_expsum_far(uint4 w, float m, float chi, float clo, float rr);
template <>
__device__ __forceinline__ float vec_expsum_far<__nv_bfloat16>(uint4 w, float m, float chi,
                                                              float clo, float rr) {
  float s = 0.0f;
  const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
  for (int q = 0; q < 4; ++q)
    s += term_far(bf_lo(ws[q]), m, chi, clo, rr) + term_far(bf_hi(ws[q]), m, chi, clo, rr);
  return s;
}
template <>
__device__ __forceinline__ float vec_expsum_far<float>(uint4 w, float m, float chi, float clo,
                                                      float rr) {
  return (term_far(__uint_as_float(w.x), m, chi, clo, rr) +
          term_far(__uint_as_float(w.y), m, chi, clo, rr)) +
         (term_far(__uint_as_float(w.z), m, chi, clo, rr) +
          term_far(__uint_as_float(w.w), m, chi, clo, rr));
}

template <typename T, typename Rows>
__global__ void __launch_bounds__(kRsWarps * 32, 1)
    row_stats_kernel(Rows rows, int nrows, int V, Partial* __restrict__ part, int32_t* status) {
  extern __shared__ __align__(128) unsigned char smem[];
  constexpr int kVec = VecOf<T>::n;
  constexpr int kEpt = kTileBytes / (int)sizeof(T);     // elements per tile
  constexpr int kVpl = kTileBytes / 16 / 32;            // vectors per lane
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  grid_dependency_wait();

  unsigned char* wbuf = smem + (size_t)warp * kRsStages * kTileBytes;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + (size_t)kRsWarps * kRsStages * kTileBytes) +
                   warp * kRsStages;
  if (lane == 0) {
    for (int s = 0; s < kRsStages; ++s) mbar_init(&bars[s], 1);
    fence_barrier_init();
  }
  __syncwarp();

  const int ntiles = (V + kEpt - 1) / kEpt;
  const int gw = blockIdx.x * kRsWarps + warp;
  const int nw = gridDim.x * kRsWarps;
  const int dr = nw / ntiles, dt = nw - dr * ntiles;

  // Item cursors (row, tile) advanced by nw items at a time, skipping rows
  // that need no statistics.
  struct Cursor {
    int r, t;
  };
  auto advance = [&](Cursor& c) {
    c.t += dt;
    c.r += dr;
    if (c.t >= ntiles) { c.t -= ntiles; ++c.r; }
  };
  auto settle = [&](Cursor& c) {
    while (c.r < nrows && !rows.get(c.r).valid) advance(c);
  };
  auto issue = [&](int s, const Cursor& c) {
    const RowRef ref = rows.get(c.r);
    const int nel = min(kEpt, V - c.t * kEpt);
    const uint32_t bytes = ((uint32_t)nel * sizeof(T)) & ~15u;
    mbar_arrive_expect_tx(&bars[s], bytes);
    if (bytes) bulk_g2s(wbuf + s * kTileBytes, ref.ptr + (size_t)c.t * kTileBytes, bytes, &bars[s]);
  };

  Cursor prod{gw / ntiles, gw % ntiles};
  settle(prod);
  int inflight = 0;
  for (int s = 0; s < kRsStages && prod.r < nrows; ++s) {
    if (lane == 0) issue(s, prod);
    ++inflight;
    advance(prod);
    settle(prod);
  }
  Cursor cons{gw / ntiles, gw % ntiles};
  settle(cons);
  uint32_t phase = 0;
  bool timed_out = false;
  int s = 0;  // stage of the item being consumed

  // Hand stage s back to the copy engine with the next item of this warp.
  auto refill = [&](int st) {
    __syncwarp();
    if (prod.r < nrows) {
      if (lane == 0) {
        fence_proxy_async_smem();
        issue(st, prod);
      }
      ++inflight;
      advance(prod);
      settle(prod);
    }
  };

  for (; cons.r < nrows; s = (s + 1 == kRsStages) ? 0 : s + 1) {
    const bool ok = mbar_wait_bounded(&bars[s], (phase >> s) & 1u, kWaitLimitNs);
    if (__any_sync(0xffffffffu, !ok)) {
      timed_out = true;
      break;
    }
    phase ^= 1u << s;
    --inflight;

    const int r = cons.r, t = cons.t;
    const RowRef ref = rows.get(r);
    const bool greedy = (ref.T == 0.0f);
    float chi = 0.0f, clo = 0.0f;
    if (!greedy) {
      const Scale sc = make_scale(ref.T);
      chi = sc.hi;
      clo = sc.lo;
    }
    const int nel = min(kEpt, V - t * kEpt);
    const uint4* buf = reinterpret_cast<const uint4*>(wbuf + s * kTileBytes);
    float best = -INFINITY;
    int bidx = 0x7fffffff;
    double ssum = 0.0;

    if (nel == kEpt) {
      // Full tile: each lane's vectors go to registers once; the stage is
      // refilled before the arithmetic starts.
      uint4 x[kVpl];
#pragma unroll
      for (int i = 0; i < kVpl; ++i) x[i] = buf[lane + 32 * i];
      refill(s);
      if (greedy) {
        int bestv = -1;
#pragma unroll
        for (int i = 0; i < kVpl; ++i) {
          const float vm = vec_max(x[i], (T*)nullptr);
          if (vm > best) { best = vm; bestv = i; }
        }
        if (bestv >= 0) {
          uint4 w = x[0];
#pragma unroll
          for (int i = 1; i < kVpl; ++i)
            if (i == bestv) w = x[i];
#pragma unroll
          for (int e = kVec - 1; e >= 0; --e)
            if (vec_elem(w, e, (T*)nullptr) == best) bidx = (lane + 32 * bestv) * kVec + e;
        }
        warp_argmax(best, bidx);
      } else {
        best = regs_max<kVpl>(x, (T*)nullptr);
#pragma unroll
        for (int o = 16; o; o >>= 1) best = fmaxf(best, __shfl_xor_sync(0xffffffffu, best, o));
        if (best > -INFINITY && best < INFINITY) {
          const float M = __fmul_rn(best, chi);
          float a;
          if (fabsf(M) < 67108864.0f) {  // 2^26: 2^(m*c - M) <= 2^2
#if SPEC_RS_PACKED
            const float2 chi2 = make_float2(chi, chi), clo2 = make_float2(clo, clo);
            const float2 nM2 = make_float2(-M, -M);
            float2 acc = make_float2(0.0f, 0.0f);
#pragma unroll
            for (int i = 0; i < kVpl; ++i)
              acc = __fadd2_rn(acc, vec_expsum(x[i], chi2, clo2, nM2, (T*)nullptr));
            a = acc.x + acc.y;
#else
            float acc0 = 0.0f, acc1 = 0.0f;
#pragma unroll
            for (int i = 0; i < kVpl; i += 2) {
              acc0 += vec_expsum_s(x[i], chi, clo, -M, (T*)nullptr);
              if (i + 1 < kVpl) acc1 += vec_expsum_s(x[i + 1], chi, clo, -M, (T*)nullptr);
            }
            a = acc0 + acc1;
#endif
          } else {
            const float rr = fmaf(best, chi, -M) + best * clo;
            a = 0.0f;
#pragma unroll
            for (int i = 0; i < kVpl; ++i) a += vec_expsum_far<T>(x[i], best, chi, clo, rr);
          }
          ssum = warp_sum_d((double)a);
        }
      }
    } else {
      // Last, partial tile of a row: guarded loads and a scalar tail.
      const int nvec = (int)(((uint32_t)nel * sizeof(T)) >> 4);
      const int ntail = nel - nvec * kVec;
      const T* gtail = reinterpret_cast<const T*>(ref.ptr) + (size_t)t * kEpt + nvec * kVec;
      float tailx = -INFINITY;
      if (lane < ntail) tailx = load_elem(gtail + lane);
      if (greedy) {
        int bestv = -1;
        for (int i = 0; i < kVpl; ++i) {
          const int v = lane + 32 * i;
          if (v < nvec) {
            const float vm = vec_max(buf[v], (T*)nullptr);
            if (vm > best) { best = vm; bestv = v; }
          }
        }
        if (bestv >= 0) {
          const uint4 w = buf[bestv];
#pragma unroll
          for (int e = kVec - 1; e >= 0; --e)
            if (vec_elem(w, e, (T*)nullptr) == best) bidx = bestv * kVec + e;
        }
        if (tailx > best) { best = tailx; bidx = nvec * kVec + lane; }
        warp_argmax(best, bidx);
      } else {
        for (int i = 0; i < kVpl; ++i) {
          const int v = lane + 32 * i;
          if (v < nvec) best = fmaxf(best, vec_max(buf[v], (T*)nullptr));
        }
        best = fmaxf(best, tailx);
#pragma unroll
        for (int o = 16; o; o >>= 1) best = fmaxf(best, __shfl_xor_sync(0xffffffffu, best, o));
        if (best > -INFINITY && best < INFINITY) {
          const float M = __fmul_rn(best, chi);
          float a = 0.0f;
          if (fabsf(M) < 67108864.0f) {
            const float2 chi2 = make_float2(chi, chi), clo2 = make_float2(clo, clo);
            const float2 nM2 = make_float2(-M, -M);
            float2 acc = make_float2(0.0f, 0.0f);
            for (int i = 0; i < kVpl; ++i) {
              const int v = lane + 32 * i;
              if (v < nvec) acc = __fadd2_rn(acc, vec_expsum(buf[v], chi2, clo2, nM2, (T*)nullptr));
            }
            a = acc.x + acc.y;
            if (lane < ntail) a += term(tailx, chi, clo, -M);
          } else {
            const float rr = fmaf(best, chi, -M) + best * clo;
            for (int i = 0; i < kVpl; ++i) {
              const int v = lane + 32 * i;
              if (v < nvec) a += vec_expsum_far<T>(buf[v], best, chi, clo, rr);
            }
            if (lane < ntail) a += term_far(tailx, best, chi, clo, rr);
          }
          ssum = warp_sum_d((double)a);
        }
      }
      refill(s);
    }

    if (lane == 0) {
      Partial p;
      p.m = best;
      p.idx = bidx == 0x7fffffff ? bidx : t * kEpt + bidx;
      p.s = ssum;
      part[(size_t)r * ntiles + t] = p;
    }

    advance(cons);
    settle(cons);
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
  grid_dependents_launch();
}

// ----------------------------------------------------------------------------
// Launchers
// ----------------------------------------------------------------------------
static int rs_grid() {
  static int sms = 0;
  if (!sms) {
    int dev = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (sms <= 0) sms = 148;
  }
  return sms;
}

template <typename T, typename Rows>
static cudaError_t launch_rs(const Rows& rows, int nrows, int V, Partial* part, int32_t* status,
                             cudaStream_t st) {
  auto kern = row_stats_kernel<T, Rows>;
  static bool smem_set = false;  // once per instantiation (same on every B200)
  if (!smem_set) {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kRsSmem);
    if (e != cudaSuccess) {
      cudaGetLastError();  // do not leave the error pending for later calls
      return e;
    }
    smem_set = true;
  }
  constexpr int kEpt = kTileBytes / (int)sizeof(T);
  const long long items = (long long)nrows * ((V + kEpt - 1) / kEpt);
  if (items >= (1LL << 31)) return cudaErrorInvalidValue;
  long long grid = rs_grid();
  const long long need = (items + kRsWarps - 1) / kRsWarps;
  if (grid > need) grid = need;
  if (grid < 1) grid = 1;
  return launch_pdl(kern, dim3((unsigned)grid), dim3(kRsWarps * 32), kRsSmem, st, rows, nrows, V,
                    part, status);
}

template <typename Rows>
cudaError_t launch_row_stats(int dtype, const Rows& rows, int nrows, int V, const RsBuffers& b,
                             int32_t* status, cudaStream_t st) {
  if (dtype == SPEC_BF16)
    return launch_rs<__nv_bfloat16>(rows, nrows, V, b.part, status, st);
  return launch_rs<float>(rows, nrows, V, b.part, status, st);
}

template cudaError_t launch_row_stats<ChainRows>(int, const ChainRows&, int, int,
                                                 const RsBuffers&, int32_t*, cudaStream_t);
template cudaError_t launch_row_stats<Hier1Rows>(int, const Hier1Rows&, int, int,
                                                 const RsBuffers&, int32_t*, cudaStream_t);
template cudaError_t launch_row_stats<Hier2Rows>(int, const Hier2Rows&, int, int,
                                                 const RsBuffers&, int32_t*, cudaStream_t);

}  // namespace specv
