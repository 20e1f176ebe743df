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

// sum_e 2^((x_e - m) * c) over one vector; pairwise inside the vector.
__device__ __forceinline__ float term(float x, float m, float chi, float clo) {
  const float d = x - m;
  return ex2(fmaf(d, chi, d * clo));
}
__device__ __forceinline__ float vec_expsum(uint4 w, float m, float chi, float clo,
                                            __nv_bfloat16*) {
  const float e0 = term(bf_lo(w.x), m, chi, clo), e1 = term(bf_hi(w.x), m, chi, clo);
  const float e2 = term(bf_lo(w.y), m, chi, clo), e3 = term(bf_hi(w.y), m, chi, clo);
  const float e4 = term(bf_lo(w.z), m, chi, clo), e5 = term(bf_hi(w.z), m, chi, clo);
  const float e6 = term(bf_lo(w.w), m, chi, clo), e7 = term(bf_hi(w.w), m, chi, clo);
  return ((e0 + e1) + (e2 + e3)) + ((e4 + e5) + (e6 + e7));
}
__device__ __forceinline__ float vec_expsum(uint4 w, float m, float chi, float clo, float*) {
  const float e0 = term(__uint_as_float(w.x), m, chi, clo);
  const float e1 = term(__uint_as_float(w.y), m, chi, clo);
  const float e2 = term(__uint_as_float(w.z), m, chi, clo);
  const float e3 = term(__uint_as_float(w.w), m, chi, clo);
  return (e0 + e1) + (e2 + e3);
}

template <typename T, typename Rows>
__global__ void __launch_bounds__(kRsWarps * 32, 1)
    row_stats_kernel(Rows rows, int nrows, int V, Partial* __restrict__ part,
                     int* __restrict__ zero_words, int nzero, int32_t* status) {
  extern __shared__ __align__(128) unsigned char smem[];
  constexpr int kVec = VecOf<T>::n;
  constexpr int kEpt = kTileBytes / (int)sizeof(T);     // elements per tile
  constexpr int kVpl = kTileBytes / 16 / 32;            // vectors per lane
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  // Clear the decide kernels' arrival counters (stream-ordered before them).
  if (blockIdx.x == 0)
    for (int i = threadIdx.x; i < nzero; i += blockDim.x) zero_words[i] = 0;

  unsigned char* wbuf = smem + (size_t)warp * kRsStages * kTileBytes;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + (size_t)kRsWarps * kRsStages * kTileBytes) +
                   warp * kRsStages;
  if (lane == 0) {
    for (int s = 0; s < kRsStages; ++s) mbar_init(&bars[s], 1);
    fence_barrier_init();
  }
  __syncwarp();

  const int ntiles = (V + kEpt - 1) / kEpt;
  const long long nitems = (long long)nrows * ntiles;
  const long long gw = (long long)blockIdx.x * kRsWarps + warp;
  const long long nw = (long long)gridDim.x * kRsWarps;

  auto next_valid = [&](long long it) -> long long {
    for (; it < nitems; it += nw)
      if (rows.get((int)(it / ntiles)).valid) return it;
    return nitems;
  };
  auto issue = [&](int s, long long it) {
    const int r = (int)(it / ntiles), t = (int)(it - (long long)r * ntiles);
    const RowRef ref = rows.get(r);
    const int nel = min(kEpt, V - t * kEpt);
    const uint32_t bytes = ((uint32_t)nel * sizeof(T)) & ~15u;
    mbar_arrive_expect_tx(&bars[s], bytes);
    if (bytes) bulk_g2s(wbuf + s * kTileBytes, ref.ptr + (size_t)t * kTileBytes, bytes, &bars[s]);
  };

  long long prod = next_valid(gw);
  int inflight = 0;
  for (int s = 0; s < kRsStages && prod < nitems; ++s) {
    if (lane == 0) issue(s, prod);
    ++inflight;
    prod = next_valid(prod + nw);
  }
  long long cons = next_valid(gw);
  uint32_t phase = 0;
  bool timed_out = false;
  int k = 0;

  for (; cons < nitems; ++k) {
    const int s = k & (kRsStages - 1);
    const bool ok = mbar_wait_bounded(&bars[s], (phase >> s) & 1u, kWaitLimitNs);
    if (__any_sync(0xffffffffu, !ok)) {
      timed_out = true;
      break;
    }
    phase ^= 1u << s;
    --inflight;

    const int r = (int)(cons / ntiles), t = (int)(cons - (long long)r * ntiles);
    const RowRef ref = rows.get(r);
    const int nel = min(kEpt, V - t * kEpt);
    const int nvec = (int)(((uint32_t)nel * sizeof(T)) >> 4);
    const int ntail = nel - nvec * kVec;
    const uint4* buf = reinterpret_cast<const uint4*>(wbuf + s * kTileBytes);
    const T* gtail = reinterpret_cast<const T*>(ref.ptr) + (size_t)t * kEpt + nvec * kVec;

    // Pass 1: largest value and the first vector holding it.
    float best = -INFINITY;
    int bestv = -1;
#pragma unroll
    for (int i = 0; i < kVpl; ++i) {
      const int v = lane + 32 * i;
      if (v < nvec) {
        const float vm = vec_max(buf[v], (T*)nullptr);
        if (vm > best) { best = vm; bestv = v; }
      }
    }
    int bidx = 0x7fffffff;
    if (bestv >= 0) {
      const uint4 w = buf[bestv];
#pragma unroll
      for (int e = kVec - 1; e >= 0; --e)
        if (vec_elem(w, e, (T*)nullptr) == best) bidx = bestv * kVec + e;
    }
    float tailx = -INFINITY;
    if (lane < ntail) {
      tailx = load_elem(gtail + lane);
      if (tailx > best) { best = tailx; bidx = nvec * kVec + lane; }
    }
    warp_argmax(best, bidx);

    double ssum = 0.0;
    if (!ref.greedy && best > -INFINITY && best < INFINITY) {
      // Pass 2: sum of 2^((l - m) c) with m the tile maximum.
      float acc = 0.0f;
#pragma unroll
      for (int i = 0; i < kVpl; ++i) {
        const int v = lane + 32 * i;
        if (v < nvec) acc += vec_expsum(buf[v], best, ref.chi, ref.clo, (T*)nullptr);
      }
      if (lane < ntail) acc += term(tailx, best, ref.chi, ref.clo);
      ssum = warp_sum_d((double)acc);
    }
    if (lane == 0) {
      Partial p;
      p.m = best;
      p.idx = bidx == 0x7fffffff ? bidx : t * kEpt + bidx;
      p.s = ssum;
      part[(size_t)r * ntiles + t] = p;
    }

    // Every lane is done with stage s; refill it.
    __syncwarp();
    if (prod < nitems) {
      if (lane == 0) {
        fence_proxy_async_smem();
        issue(s, prod);
      }
      ++inflight;
      prod = next_valid(prod + nw);
    }
    cons = next_valid(cons + nw);
  }

  if (timed_out) {
    if (lane == 0) set_status(status, SPEC_ETIMEOUT);
    // Let copies still in flight land before the CTA's shared memory goes:
    // stages k, k+1, ... hold the `inflight` copies not yet consumed.
    for (int j = 0; j < inflight; ++j) {
      const int s = (k + j) & (kRsStages - 1);
      mbar_wait_bounded(&bars[s], (phase >> s) & 1u, kWaitLimitNs);
    }
  }
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
static cudaError_t launch_rs(const Rows& rows, int nrows, int V, Partial* part, int* zero_words,
                             int nzero, int32_t* status, cudaStream_t st) {
  auto kern = row_stats_kernel<T, Rows>;
  static bool smem_set = false;  // once per instantiation (same on every B200)
  if (!smem_set) {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kRsSmem);
    if (e != cudaSuccess) return e;
    smem_set = true;
  }
  constexpr int kEpt = kTileBytes / (int)sizeof(T);
  const long long items = (long long)nrows * ((V + kEpt - 1) / kEpt);
  long long grid = rs_grid();
  const long long need = (items + kRsWarps - 1) / kRsWarps;
  if (grid > need) grid = need;
  if (grid < 1) grid = 1;
  kern<<<(int)grid, kRsWarps * 32, kRsSmem, st>>>(rows, nrows, V, part, zero_words, nzero, status);
  return cudaGetLastError();
}

template <typename Rows>
cudaError_t launch_row_stats(int dtype, const Rows& rows, int nrows, int V, Partial* part,
                             int* zero_words, int nzero, int32_t* status, cudaStream_t st) {
  if (dtype == SPEC_BF16)
    return launch_rs<__nv_bfloat16>(rows, nrows, V, part, zero_words, nzero, status, st);
  return launch_rs<float>(rows, nrows, V, part, zero_words, nzero, status, st);
}

template cudaError_t launch_row_stats<ChainRows>(int, const ChainRows&, int, int, Partial*, int*,
                                                 int, int32_t*, cudaStream_t);
template cudaError_t launch_row_stats<Hier1Rows>(int, const Hier1Rows&, int, int, Partial*, int*,
                                                 int, int32_t*, cudaStream_t);
template cudaError_t launch_row_stats<Hier2Rows>(int, const Hier2Rows&, int, int, Partial*, int*,
                                                 int, int32_t*, cudaStream_t);

}  // namespace specv
