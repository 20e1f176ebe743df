// Per-element arithmetic of the row statistics, shared by the row-statistics
// kernel and the verification step kernel: the largest element of 16-byte
// vectors, and the sums of 2^(l*c - M) (c = log2(e) / T split as c_hi +
// c_lo, M an exact fp32 shift) one 16-byte vector at a time.
//
// Step "temperature softmax over V" behind every check of HiSpec
// (gist.science summary of arXiv 2510.01336, section 2: the three exits L_d,
// L_i, L_f each give a token distribution; "Verlustfreie Garantie" compares
// them).
#pragma once
#include <cfloat>

#include "common.cuh"

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
// x - a, held at -FLT_MAX for x = -inf (a masked or padded entry), whose term
// 2^(x*c - M) = 0 must then contribute 0, not 0 * -inf.
__device__ __forceinline__ float dev1(float x, float a) { return fmaxf(x - a, -FLT_MAX); }
__device__ __forceinline__ float2 dev2(float2 x, float2 nA) {
  const float2 d = __fadd2_rn(x, nA);
  return make_float2(fmaxf(d.x, -FLT_MAX), fmaxf(d.y, -FLT_MAX));
}

// Same, also returning the pairwise sums of 2^(x*c - M) * (x - a) (nA = -a),
// the first moment the entropy of the row's distribution needs.
__device__ __forceinline__ float2 vec_expsum_ent(uint4 w, float2 chi, float2 clo, float2 nM,
                                                 float2 nA, float2* mom, __nv_bfloat16*) {
  const float2 x0 = make_float2(bf_lo(w.x), bf_hi(w.x)), x1 = make_float2(bf_lo(w.y), bf_hi(w.y));
  const float2 x2 = make_float2(bf_lo(w.z), bf_hi(w.z)), x3 = make_float2(bf_lo(w.w), bf_hi(w.w));
  const float2 e0 = ex2x2(expo2(x0, chi, clo, nM)), e1 = ex2x2(expo2(x1, chi, clo, nM));
  const float2 e2 = ex2x2(expo2(x2, chi, clo, nM)), e3 = ex2x2(expo2(x3, chi, clo, nM));
  float2 t = __fmul2_rn(e0, dev2(x0, nA));
  t = __ffma2_rn(e1, dev2(x1, nA), t);
  t = __ffma2_rn(e2, dev2(x2, nA), t);
  *mom = __ffma2_rn(e3, dev2(x3, nA), t);
  return __fadd2_rn(__fadd2_rn(e0, e1), __fadd2_rn(e2, e3));
}
__device__ __forceinline__ float2 vec_expsum_ent(uint4 w, float2 chi, float2 clo, float2 nM,
                                                 float2 nA, float2* mom, float*) {
  const float2 x0 = make_float2(__uint_as_float(w.x), __uint_as_float(w.y));
  const float2 x1 = make_float2(__uint_as_float(w.z), __uint_as_float(w.w));
  const float2 e0 = ex2x2(expo2(x0, chi, clo, nM)), e1 = ex2x2(expo2(x1, chi, clo, nM));
  *mom = __ffma2_rn(e1, dev2(x1, nA), __fmul2_rn(e0, dev2(x0, nA)));
  return __fadd2_rn(e0, e1);
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

// 2^k as a double, exactly, for an integer-valued k <= 0 (0 below 2^-1022).
__device__ __forceinline__ double pow2i(float k) {
  const int e = (int)k;
  return e < -1022 ? 0.0 : __longlong_as_double((long long)(1023 + e) << 52);
}
constexpr float kFarShift = 67108864.0f;  // 2^26: beyond, 2^(m*c - M) itself may overflow

template <typename T> __device__ __forceinline__ uint4 neg_inf_vec();
template <> __device__ __forceinline__ uint4 neg_inf_vec<__nv_bfloat16>() {
  return make_uint4(0xff80ff80u, 0xff80ff80u, 0xff80ff80u, 0xff80ff80u);
}
template <> __device__ __forceinline__ uint4 neg_inf_vec<float>() {
  return make_uint4(0xff800000u, 0xff800000u, 0xff800000u, 0xff800000u);
}

}  // namespace specv
