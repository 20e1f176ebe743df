// Paged-KV commit / rollback and pruning of the buffered rows.
//
// HiSpec (gist.science summary of arXiv 2510.01336), section 2: KV entries
// and hidden states are buffered while drafting and the entries of rejected
// tokens are dropped before the next phase ("Wiederverwendung von KV-Cache und
// versteckten Zustaenden"); paged attention with block tables lets every
// sequence accept its own number of tokens without padding ("Unterstuetzung
// fuer Batch-Inferenz").
//
// Two launches. (1) One CTA plans: it checks every sequence, the pool and the
// stack before anything changes, then frees table tails (sequences ascending,
// tails in ascending index, pushed) and allocates missing blocks (sequences
// ascending, popped), sets the lengths and the packed hidden-row offsets. The
// allocation order couples all sequences, hence the single CTA. (2) Many CTAs
// copy each kept token's staged K/V rows into its pool slot and its hidden
// row into the packed output (16-byte vectors, streaming hints).
#include "commit.cuh"

namespace specv {

__global__ void __launch_bounds__(kPlanThreads) commit_plan_kernel(CommitArgs a) {
  pdl_begin();
  extern __shared__ int s_seq[];
  plan_body(a, s_seq);
}

__global__ void __launch_bounds__(kCopyThreads) commit_copy_kernel(CommitArgs a) {
  pdl_begin();
  extern __shared__ int s_off[];
  copy_body(a, blockIdx.x, gridDim.x, s_off);
}

cudaError_t launch_commit_copy(const CommitArgs& a, cudaStream_t st) {
  if (a.B <= 0 || a.Kp1 <= 0 || !(a.kv_stage || a.hid_stage)) return cudaSuccess;
  const size_t smem = (2 * (size_t)a.B + 1) * sizeof(int);
  cudaError_t e = reserve_dyn_smem(commit_copy_kernel, smem);
  if (e != cudaSuccess) return e;
  return launch_pdl(commit_copy_kernel, dim3(sm_count() * kCopyCtasPerSm), dim3(kCopyThreads),
                    smem, st, a);
}

cudaError_t launch_commit(const CommitArgs& a, cudaStream_t st) {
  const size_t smem = 3 * (size_t)a.B * sizeof(int);
  cudaError_t e = reserve_dyn_smem(commit_plan_kernel, smem);
  if (e != cudaSuccess) return e;
  e = launch_pdl(commit_plan_kernel, dim3(1), dim3(kPlanThreads), smem, st, a);
  if (e != cudaSuccess) return e;
  return launch_commit_copy(a, st);
}

// ---------------------------------------------------------------------------
// Diagnostic: device Philox uniforms.
// ---------------------------------------------------------------------------
__global__ void philox_kernel(uint64_t seed, const uint32_t* ctr, int n, float* out) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= n) return;
  const float2 u = spec_uniforms(seed, ctr[4 * i], ctr[4 * i + 1], ctr[4 * i + 2], ctr[4 * i + 3]);
  out[2 * i] = u.x;
  out[2 * i + 1] = u.y;
}

cudaError_t launch_philox(uint64_t seed, const uint32_t* ctr, int n, float* out, cudaStream_t st) {
  if (n > 0) philox_kernel<<<(n + 255) / 256, 256, 0, st>>>(seed, ctr, n, out);
  return cudaGetLastError();
}

}  // namespace specv
