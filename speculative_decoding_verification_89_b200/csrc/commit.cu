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

// Limit of the planned copy launch's wait for the plan word: kWaitLimitNs
// unless a test has set another with spec_test_set_copy_wait_limit_ns (0:
// one poll, so a plan not yet written makes the wait run out).
__device__ unsigned long long g_copy_wait_limit_ns = kWaitLimitNs;

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

// The copy launch that follows a verify-and-commit decide launch: it does not
// wait for that launch to complete, only for its planner. It lets its own
// successors launch at once (they wait for its completion), waits -- one
// thread, bounded -- until the planner has published plan_flag, copies, and
// only then waits for the decide launch to complete, so nothing after it in
// the stream runs before the draws are written. Its CTAs run beside the
// decide launch's: this launch starts only once every CTA of that launch has
// started (programmatic launch), so the planner's CTA is resident while they
// wait.
__global__ void __launch_bounds__(kCopyThreads) commit_copy_planned_kernel(CommitArgs a,
                                                                           const int32_t* plan_flag) {
  grid_dependents_launch();
  __shared__ int s_go;
  if (threadIdx.x == 0) {
    int v = ld_relaxed(plan_flag);
    if (!v) {
      const uint64_t limit = g_copy_wait_limit_ns;
      const uint64_t t0 = globaltimer_ns();
      unsigned ns = 64;
      for (;;) {
        __nanosleep(ns);
        if (ns < 256) ns <<= 1;
        v = ld_relaxed(plan_flag);
        if (v || globaltimer_ns() - t0 > limit) break;
      }
    }
    if (v) fence_acq_rel();  // the planner's writes are visible from here on
    else set_status(a.status, SPEC_ETIMEOUT);
    s_go = v;
  }
  __syncthreads();
  if (s_go) {
    extern __shared__ int s_off[];
    copy_body(a, blockIdx.x, gridDim.x, s_off);
  }
  grid_dependency_wait();
}

cudaError_t launch_commit_copy_planned(const CommitArgs& a, const int32_t* plan_flag,
                                       cudaStream_t st) {
  const size_t smem = (2 * (size_t)a.B + 1) * sizeof(int);
  cudaError_t e = reserve_dyn_smem(commit_copy_planned_kernel, smem);
  if (e != cudaSuccess) return e;
  return launch_pdl(commit_copy_planned_kernel, dim3(sm_count() * kCopyCtasPerSmPlanned),
                    dim3(kCopyThreads), smem, st, a, plan_flag);
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

#pragma GCC visibility push(default)
extern "C" int spec_test_set_copy_wait_limit_ns(uint64_t ns) {
  const unsigned long long v = ns;
  const cudaError_t e = cudaMemcpyToSymbol(specv::g_copy_wait_limit_ns, &v, sizeof(v));
  if (e != cudaSuccess) return specv::record_cuda_status(e);
  return SPEC_OK;
}
#pragma GCC visibility pop
