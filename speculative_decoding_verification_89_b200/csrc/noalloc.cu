// Chain verification for callers that cannot allocate device memory.
//
// Some callers cannot call cudaMalloc, or any routine that allocates, at the
// point where they verify drafts: a serving process that fixes its memory
// budget at start-up and must not grow it, a plugin or custom-op host whose
// allocator belongs to someone else, or a hot loop that is not allowed to
// touch an allocator at all. For them this file adds one entry point,
// spec_verify_chain_noalloc, which does what spec_verify_chain does but takes
// its scratch memory from a fixed array compiled into the library instead of
// a workspace the caller provides.
//
// The array is a file-scope __device__ variable of SPEC_NOALLOC_SCRATCH_BYTES,
// so every GPU that loads the library keeps that much of its memory until the
// process exits. Host code cannot use the array's name as a device address:
// a call asks the runtime for the address (cudaGetSymbolAddress) with the
// device current, and keeps it per device and per CUDA context, so the
// lookup runs once per device (again only if the device's context was
// destroyed and re-created). A lookup that fails is not kept: the next call
// tries again. Make the first call on a device outside any stream capture.
// The array is shared by every call and keeps the previous call's contents;
// the per-call counters in it are cleared by the call's own first launch, and
// nothing else is read before it is written. Calls that overlap on the GPU
// (other streams, other threads) race on it.
#include <mutex>

#include "common.cuh"
#include "kernels.cuh"

namespace {

constexpr size_t kScratchBytes = SPEC_NOALLOC_SCRATCH_BYTES;
constexpr int kMaxDevices = 64;

__device__ __align__(256) unsigned char g_noalloc_scratch[kScratchBytes];

// Successful lookups only: the context they were made in and the address.
struct Slot {
  void* ctx;
  void* addr;
};
std::mutex g_mu;
Slot g_slot[kMaxDevices];
int g_fail_lookups = 0;  // test hook: lookups still to be refused

// cuCtxGetCurrent through the runtime's driver entry point (no link against
// the driver library); null if the driver does not provide it.
typedef int (*CtxGetCurrentFn)(void**);
CtxGetCurrentFn ctx_get_current() {
  static const CtxGetCurrentFn fn = [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q = cudaDriverEntryPointSymbolNotFound;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess) {
      cudaGetLastError();
      p = nullptr;
    }
    return reinterpret_cast<CtxGetCurrentFn>(p);
  }();
  return fn;
}

void* current_ctx() {
  const CtxGetCurrentFn fn = ctx_get_current();
  void* ctx = nullptr;
  if (!fn || fn(&ctx) != 0) return nullptr;
  return ctx;
}

// Device address of the scratch array on the current device.
cudaError_t scratch_address(void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  void* ctx = current_ctx();
  std::lock_guard<std::mutex> lock(g_mu);
  if (g_fail_lookups > 0) {
    --g_fail_lookups;
    return cudaErrorStreamCaptureUnsupported;  // what a lookup inside a capture returns
  }
  if (ctx && g_slot[dev].addr && g_slot[dev].ctx == ctx) {
    *out = g_slot[dev].addr;
    return cudaSuccess;
  }
  void* addr = nullptr;
  e = cudaGetSymbolAddress(&addr, g_noalloc_scratch);
  if (e != cudaSuccess) return e;  // nothing kept: the next call looks it up again
  ctx = current_ctx();             // the lookup made the device's context current
  if (ctx) g_slot[dev] = Slot{ctx, addr};
  *out = addr;
  return cudaSuccess;
}

}  // namespace

#pragma GCC visibility push(default)
extern "C" {

int spec_verify_chain_noalloc(const void* tgt, int64_t ld_tgt, const void* drf, int64_t ld_drf,
                              int dtype, int B, int K, int V, const int32_t* draft_tok,
                              const float* temperature, uint64_t seed, const int32_t* seq_id,
                              uint32_t round, int32_t* accept_len, int32_t* out_tok,
                              double* diag, int32_t* dev_status, void* stream) {
  const size_t need = spec_workspace_bytes(B, K, V, dtype, 0);
  if (need == 0) return SPEC_EINVAL;
  if (B == 0) return SPEC_OK;
  if (need > kScratchBytes) return SPEC_EWORKSPACE;
  void* ws = nullptr;
  const cudaError_t e = scratch_address(&ws);
  if (e != cudaSuccess) {
    cudaGetLastError();
    return specv::record_cuda_status(e);
  }
  return spec_verify_chain(tgt, ld_tgt, drf, ld_drf, dtype, B, K, V, draft_tok, temperature, seed,
                           seq_id, round, accept_len, out_tok, diag, dev_status, ws, need, stream);
}

int spec_noalloc_test_fail_lookups(int n) {
  if (n < 0) return SPEC_EINVAL;
  std::lock_guard<std::mutex> lock(g_mu);
  g_fail_lookups = n;
  for (int d = 0; d < kMaxDevices; ++d) g_slot[d] = Slot{nullptr, nullptr};
  return SPEC_OK;
}

}  // extern "C"
#pragma GCC visibility pop
