// Saguaro sampling: the draft law with the speculation cache's tokens
// lowered.
//
// Speculative Speculative Decoding (gist.science summary of arXiv 2603.03251),
// Technische Zusammenfassung 3.B: the probabilities of the tokens held in the
// speculation cache are lowered a little in the draft, so the residual of a
// rejection -- proportional to the target-minus-draft difference -- lands on
// them more often. With the factor (1 - eps) on each cached token's draft
// probability, renormalised, the draft law at temperature T > 0 is the softmax
// of the logits with T ln(1 - eps) added to the cached tokens; this launch adds
// that shift in place to the drafting exit's rows, so the draft step and the
// check that follow use the lowered law as the draft law (and the check stays
// lossless). Greedy rows (T == 0) are left alone.
//
// The cache's tokens come as one list per sequence (lowered in each of its
// rows) or one list per row (the bonus tokens prepared for that position).
// One thread per (list, slot): an id outside [0, V) is padding, an id listed
// earlier in the same list is skipped, and the thread updates that token's
// logit in the rows its list covers. The shift is
// float32(T * ln(1 - eps)) added in float32 and rounded to the rows' type.
#include "common.cuh"
#include "kernels.cuh"

namespace specv {

template <typename T>
__device__ __forceinline__ void add_shift(T* p, float d);
template <>
__device__ __forceinline__ void add_shift<float>(float* p, float d) {
  *p = __fadd_rn(*p, d);
}
template <>
__device__ __forceinline__ void add_shift<__nv_bfloat16>(__nv_bfloat16* p, float d) {
  *p = __float2bfloat16_rn(__fadd_rn(__bfloat162float(*p), d));
}

template <typename T>
__global__ void saguaro_adjust_kernel(unsigned char* lg, long long ld_bytes, int B,
                                      int rows_per_seq, int V, const int32_t* cached,
                                      int n_cached, int per_row, double ln1m_eps,
                                      const float* temperature) {
  pdl_begin();
  const int sets = per_row ? rows_per_seq : 1;
  const long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= (long long)B * sets * n_cached) return;
  const long long set = i / n_cached;
  const int k = (int)(i - set * n_cached);
  const int b = (int)(set / sets), r0 = (int)(set - (long long)b * sets);
  const int32_t* ids = cached + set * n_cached;
  const int v = ids[k];
  if (v < 0 || v >= V) return;
  for (int j = 0; j < k; ++j)
    if (ids[j] == v) return;  // listed before: lowered once
  const float Tb = temperature[b];
  if (!(Tb > 0.0f) || !temp_valid(Tb)) return;
  const float d = (float)((double)Tb * ln1m_eps);
  const int r_end = per_row ? r0 + 1 : rows_per_seq;
  for (int r = per_row ? r0 : 0; r < r_end; ++r) {
    T* row = reinterpret_cast<T*>(lg + ((long long)b * rows_per_seq + r) * ld_bytes);
    add_shift<T>(row + v, d);
  }
}

cudaError_t launch_saguaro_adjust(int dtype, unsigned char* lg, long long ld_bytes, int B,
                                  int rows_per_seq, int V, const int32_t* cached, int n_cached,
                                  int per_row, double ln1m_eps, const float* temperature,
                                  cudaStream_t st) {
  const long long n = (long long)B * (per_row ? rows_per_seq : 1) * n_cached;
  if (n == 0 || rows_per_seq == 0) return cudaSuccess;
  const unsigned grid = (unsigned)((n + 255) / 256);
  if (dtype == SPEC_BF16)
    return launch_pdl(saguaro_adjust_kernel<__nv_bfloat16>, dim3(grid), dim3(256), 0, st, lg,
                      ld_bytes, B, rows_per_seq, V, cached, n_cached, per_row, ln1m_eps,
                      temperature);
  return launch_pdl(saguaro_adjust_kernel<float>, dim3(grid), dim3(256), 0, st, lg, ld_bytes, B,
                    rows_per_seq, V, cached, n_cached, per_row, ln1m_eps, temperature);
}

}  // namespace specv
