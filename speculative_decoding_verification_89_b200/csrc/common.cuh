// Device helpers shared by the kernels of libspecverify (sm_100a).
//
// Philox4x32-10: J. K. Salmon, M. A. Moraes, R. O. Dror, D. E. Shaw,
// "Parallel Random Numbers: As Easy as 1, 2, 3", SC'11 -- S-P network with the
// 4x32 multipliers and Weyl key increments of its table 2, ten rounds.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <mutex>

#include "../../include/spec_verify.h"

namespace specv {

// ----------------------------------------------------------------------------
// Constants and small structs
// ----------------------------------------------------------------------------
constexpr double kLog2e = 1.4426950408889634073599246810018921;  // 1/ln 2
constexpr double kLn2 = 0.6931471805599453094172321214581766;

// Row-statistics tiles: kTileBytes of one row, staged by one bulk copy into a
// per-warp ring of kRsStages buffers; one CTA of kRsWarps warps per SM.
#ifndef SPEC_RS_TILE
#define SPEC_RS_TILE 6144
#endif
#ifndef SPEC_RS_WARPS
#define SPEC_RS_WARPS 16
#endif
#ifndef SPEC_RS_STAGES
#define SPEC_RS_STAGES 2
#endif
constexpr int kTileBytes = SPEC_RS_TILE;
constexpr int kRsWarps = SPEC_RS_WARPS;
constexpr int kRsStages = SPEC_RS_STAGES;
constexpr int kRsSmem = kRsWarps * kRsStages * kTileBytes + kRsWarps * kRsStages * 8;
static_assert(kRsSmem <= 227 * 1024, "row-statistics ring exceeds shared memory");
static_assert(kTileBytes % 512 == 0, "a tile is a whole number of warp-wide 16-byte vectors");

// Residual tiles: 32 lanes x 8 elements.
constexpr int kResTile = 256;

// Statistics of a run of consecutive tiles of one row, stored at the run's
// first tile (the run's other tiles hold empty partials: m = -inf, s = 0):
// the run's largest raw logit m, its first index (greedy rows), and
// s = sum over the run of 2^(l*c - M), c = log2(e) / T, with the exact fp32
// shift M = fl(m * c_hi) (c_hi from make_scale; M is recomputed from m).
struct Partial {
  float m;
  int idx;
  double s;
};

// Final statistics of one row, written by the warp that completes the row's
// last tile: shift M = fl(m * c_hi) and L = log2 sum 2^(l*c - M) (so the
// row's log2-partition is M + L), raw max m, first argmax (greedy rows), ok.
struct RowFinal {
  double M, L;
  float m;
  int amax;
  int ok;
  int pad;
};

template <typename T> struct Elem;
template <> struct Elem<float> { static constexpr int kDtype = SPEC_F32; };
template <> struct Elem<__nv_bfloat16> { static constexpr int kDtype = SPEC_BF16; };

// Temperature scale c = log2(e) / T split as c_hi + c_lo (two floats) so the
// fp32 hot loop carries ~48 bits of the scale. c_hi is rounded toward zero
// and kept strictly below c, so c_lo > 0 and (-inf) * c_lo stays -inf.
struct Scale {
  float hi, lo;
  double d;
};
__device__ __forceinline__ Scale make_scale(float T) {
  Scale s;
  s.d = kLog2e / (double)T;
  s.hi = __double2float_rz(s.d);
  if ((double)s.hi == s.d) s.hi = nextafterf(s.hi, 0.0f);
  s.lo = (float)(s.d - (double)s.hi);
  return s;
}

// Accepted temperatures: 0 (greedy) or 1e-6 <= T <= 1e6.
constexpr float kTempMin = 1.0e-6f, kTempMax = 1.0e6f;
__device__ __forceinline__ bool temp_valid(float T) {
  return T == 0.0f || (T >= kTempMin && T <= kTempMax);  // false for NaN
}

// ----------------------------------------------------------------------------
// Element access
// ----------------------------------------------------------------------------
__device__ __forceinline__ float load_elem(const float* p) { return __ldg(p); }
__device__ __forceinline__ float load_elem(const __nv_bfloat16* p) {
  unsigned short h = __ldg(reinterpret_cast<const unsigned short*>(p));
  return __uint_as_float(((unsigned)h) << 16);
}
__device__ __forceinline__ float bf_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf_hi(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }

// 2^x with the hardware approximation (flushes subnormal results to zero).
__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// ----------------------------------------------------------------------------
// Philox4x32-10 and the uniform map
// ----------------------------------------------------------------------------
__device__ __forceinline__ uint4 philox4x32_10(uint4 c, uint32_t k0, uint32_t k1) {
  const uint32_t M0 = 0xD2511F53u, M1 = 0xCD9E8D57u;
  const uint32_t W0 = 0x9E3779B9u, W1 = 0xBB67AE85u;
#pragma unroll
  for (int r = 0; r < 10; ++r) {
    if (r) { k0 += W0; k1 += W1; }
    const uint32_t lo0 = M0 * c.x, hi0 = __umulhi(M0, c.x);
    const uint32_t lo1 = M1 * c.z, hi1 = __umulhi(M1, c.z);
    c = make_uint4(hi1 ^ c.y ^ k0, lo1, hi0 ^ c.w ^ k1, lo0);
  }
  return c;
}

// (2*(x >> 9) + 1) * 2^-24: odd multiple of 2^-24 in (0, 1), exact in fp32.
__device__ __forceinline__ float to_uniform(uint32_t x) {
  return (float)(2u * (x >> 9) + 1u) * 5.9604644775390625e-08f;
}

__device__ __forceinline__ float2 spec_uniforms(uint64_t seed, uint32_t seq, uint32_t rnd,
                                                uint32_t pos, uint32_t stage) {
  uint4 r = philox4x32_10(make_uint4(seq, rnd, pos, stage), (uint32_t)seed,
                          (uint32_t)(seed >> 32));
  return make_float2(to_uniform(r.x), to_uniform(r.y));
}

// ----------------------------------------------------------------------------
// Status word: first error wins.
// ----------------------------------------------------------------------------
__device__ __forceinline__ void set_status(int32_t* st, int code) {
  if (st) atomicCAS(reinterpret_cast<int*>(st), 0, code);
}

// ----------------------------------------------------------------------------
// Flags in global memory (device scope)
// ----------------------------------------------------------------------------
__device__ __forceinline__ int ld_acquire(const int* p) {
  int v;
  asm volatile("ld.acquire.gpu.global.b32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}
__device__ __forceinline__ void st_release(int* p, int v) {
  asm volatile("st.release.gpu.global.b32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}
__device__ __forceinline__ int ld_relaxed(const int* p) {
  int v;
  asm volatile("ld.relaxed.gpu.global.b32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}
__device__ __forceinline__ void fence_acq_rel() { asm volatile("fence.acq_rel.gpu;" ::: "memory"); }

// ----------------------------------------------------------------------------
// mbarrier + 1-D bulk copy (TMA without a tensor map, no multicast)
// ----------------------------------------------------------------------------
__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return (uint32_t)__cvta_generic_to_shared(p);
}
__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count));
}
__device__ __forceinline__ void fence_barrier_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}
__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}
__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)),
               "r"(bytes)
               : "memory");
}
__device__ __forceinline__ void bulk_g2s(void* dst, const void* src, uint32_t bytes,
                                         uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
          smem_u32(dst)),
      "l"(src), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}
// Same, with an L2 cache policy (l2_evict_first) for the copied lines.
__device__ __forceinline__ void bulk_g2s_hint(void* dst, const void* src, uint32_t bytes,
                                              uint64_t* bar, uint64_t policy) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint"
      " [%0], [%1], %2, [%3], %4;" ::"r"(smem_u32(dst)),
      "l"(src), "r"(bytes), "r"(smem_u32(bar)), "l"(policy)
      : "memory");
}
// L2 policy: lines go first when the cache needs room.
__device__ __forceinline__ uint64_t l2_evict_first() {
  uint64_t p;
  asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(p));
  return p;
}
__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}
__device__ __forceinline__ uint64_t globaltimer_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %globaltimer;" : "=l"(t));
  return t;
}
__device__ __forceinline__ bool mbar_test_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}
// Wait for a barrier phase, at most `limit_ns` nanoseconds. Returns false on
// timeout (the caller records SPEC_ETIMEOUT and winds down). A limit of 0
// makes the wait one non-blocking test.
__device__ __forceinline__ bool mbar_wait_bounded(uint64_t* bar, uint32_t parity,
                                                  uint64_t limit_ns) {
  if (limit_ns == 0) return mbar_test_wait(bar, parity);
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = globaltimer_ns();
  while (!mbar_try_wait(bar, parity)) {
    if (globaltimer_ns() - t0 > limit_ns) return false;
  }
  return true;
}
constexpr uint64_t kWaitLimitNs = 2000000000ull;  // 2 s

// ----------------------------------------------------------------------------
// Programmatic dependent launch: every kernel of the library is launched with
// programmatic stream serialization and starts with pdl_begin(): it waits for
// its stream predecessors before touching memory (griddepcontrol.wait returns
// once they have completed and their writes are visible) and at once lets its
// successor launch, so the successor's CTAs take SMs as this kernel's CTAs
// leave them and only wait for the completion (its own griddepcontrol.wait
// orders every memory access).
__device__ __forceinline__ void grid_dependency_wait() {
  asm volatile("griddepcontrol.wait;" ::: "memory");
}
__device__ __forceinline__ void grid_dependents_launch() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}
__device__ __forceinline__ void pdl_begin() {
  grid_dependency_wait();
  grid_dependents_launch();
}

// Device index of the calling thread (0 if the runtime cannot say).
static inline int current_device() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) {
    cudaGetLastError();
    dev = 0;
  }
  return dev;
}
constexpr int kMaxDevs = 64;  // per-device host caches

// Streaming multiprocessors of the current device (148 on a B200), looked up
// once per device.
static inline int sm_count() {
  static int sms[kMaxDevs];
  const int dev = current_device();
  int* slot = (dev >= 0 && dev < kMaxDevs) ? &sms[dev] : nullptr;
  if (slot && *slot > 0) return *slot;
  int v = 0;
  if (cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) {
    cudaGetLastError();
    v = 0;
  }
  v = v > 0 ? v : 148;
  if (slot) *slot = v;
  return v;
}

// Lets kernel `fn` launch with `bytes` of dynamic shared memory on the
// current device: a kernel whose static plus dynamic shared memory passes
// 48 KB needs the opt-in, which is a setting of the function on one device.
// The largest size granted so far is kept per (device, kernel), so the
// attribute is set only when a launch needs more than before (and never
// lowered under a concurrent caller).
static cudaError_t reserve_dyn_smem(const void* fn, size_t bytes) {
  static std::mutex mu;
  constexpr int kSlots = 256;
  static const void* fns[kSlots];
  static int devs[kSlots];
  static size_t granted[kSlots];
  static int n = 0;
  const int dev = current_device();
  std::lock_guard<std::mutex> lock(mu);
  int i = 0;
  while (i < n && !(fns[i] == fn && devs[i] == dev)) ++i;
  if (i < n && granted[i] >= bytes) return cudaSuccess;
  const cudaError_t e =
      cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
  if (e != cudaSuccess) {
    cudaGetLastError();
    return e;
  }
  if (i < n) {
    granted[i] = bytes;
  } else if (n < kSlots) {
    fns[n] = fn;
    devs[n] = dev;
    granted[n++] = bytes;
  }
  return cudaSuccess;
}
template <typename Kern>
static cudaError_t reserve_dyn_smem(Kern* fn, size_t bytes) {
  return reserve_dyn_smem(reinterpret_cast<const void*>(fn), bytes);
}

template <typename Kern, typename... Args>
static cudaError_t launch_pdl(Kern kern, dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                             Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  cudaError_t e = cudaLaunchKernelEx(&cfg, kern, args...);
  if (e != cudaSuccess) cudaGetLastError();
  return e;
}

// Same, for a grid of thread-block clusters of `cluster` CTAs along x.
template <typename Kern, typename... Args>
static cudaError_t launch_pdl_cluster(Kern kern, dim3 grid, dim3 block, size_t smem,
                                      cudaStream_t st, unsigned cluster, Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  attr[1].id = cudaLaunchAttributeClusterDimension;
  attr[1].val.clusterDim.x = cluster;
  attr[1].val.clusterDim.y = 1;
  attr[1].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  cudaError_t e = cudaLaunchKernelEx(&cfg, kern, args...);
  if (e != cudaSuccess) cudaGetLastError();
  return e;
}

// ----------------------------------------------------------------------------
// Warp reductions
// ----------------------------------------------------------------------------
__device__ __forceinline__ double warp_sum_d(double v) {
#pragma unroll
  for (int o = 16; o; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}
// (max value, smallest index among equal maxima); NaN never wins.
__device__ __forceinline__ void warp_argmax(float& v, int& i) {
#pragma unroll
  for (int o = 16; o; o >>= 1) {
    const float ov = __shfl_xor_sync(0xffffffffu, v, o);
    const int oi = __shfl_xor_sync(0xffffffffu, i, o);
    if (ov > v || (ov == v && oi < i)) { v = ov; i = oi; }
  }
}

}  // namespace specv
