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
// process exits. Host code cannot use the array's name as a device address;
// the first call on each device, with that device current, asks the runtime
// for the address (cudaGetSymbolAddress) and keeps it, so make that first call
// outside any stream capture. The array is shared by every call and keeps the
// previous call's contents, none of which a later call reads before writing.
// Calls that overlap on the GPU (other streams, other threads) race on it.
#include <mutex>

#include "common.cuh"
#include "kernels.cuh"

namespace {

constexpr size_t kScratchBytes = SPEC_NOALLOC_SCRATCH_BYTES;
constexpr int kMaxDevices = 64;

__device__ __align__(256) unsigned char g_noalloc_scratch[kScratchBytes];

std::once_flag g_once[kMaxDevices];
void* g_addr[kMaxDevices];
cudaError_t g_err[kMaxDevices];

// Device address of the scratch array on the current device, looked up once
// per device.
cudaError_t scratch_address(void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::call_once(g_once[dev], [dev]() {
    g_err[dev] = cudaGetSymbolAddress(&g_addr[dev], g_noalloc_scratch);
  });
  *out = g_addr[dev];
  return g_err[dev];
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
  cudaError_t e = scratch_address(&ws);
  if (e != cudaSuccess) {
    cudaGetLastError();
    return SPEC_ECUDA;
  }
  return spec_verify_chain(tgt, ld_tgt, drf, ld_drf, dtype, B, K, V, draft_tok, temperature, seed,
                           seq_id, round, accept_len, out_tok, diag, dev_status, ws, need, stream);
}

}  // extern "C"
#pragma GCC visibility pop
