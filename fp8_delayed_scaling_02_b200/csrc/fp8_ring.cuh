// FP8 casts, packed fp32x2 arithmetic and the delayed-scaling ring commit
// shared by the quantize and GEMM kernels (sm_100a).
//
// Cast: one fp32 multiply by the scale, rounded to nearest even, then the
// hardware round-to-nearest-even conversion with saturation to the largest
// finite value of the format.  Ring commit: the fold that ends every
// delayed-scaling call ("AstrAI commits, branch main, tests/extension", ring
// commit and snapshot commit) -- history[idx] = amax, idx advances, the next
// scale is FP8_MAX / max(history) when that maximum is positive and finite and
// the quotient is finite and positive (otherwise the scale is kept), and
// scale_inv is the inverse of the scale the call used.
#pragma once

#include <cuda_fp8.h>

#include "common.cuh"

namespace fp8ds {

// (a*s, b*s) with one packed fp32x2 multiply, each lane rounded to nearest
// even exactly as a scalar fp32 multiply (no contraction into anything else).
__device__ __forceinline__ void scale2(float& a, float& b, float s) {
  asm("{\n\t.reg .b64 ra, rs, rd;\n\t"
      "mov.b64 ra, {%0, %1};\n\t"
      "mov.b64 rs, {%2, %2};\n\t"
      "mul.rn.f32x2 rd, ra, rs;\n\t"
      "mov.b64 {%0, %1}, rd;\n\t}"
      : "+f"(a), "+f"(b)
      : "f"(s));
}

// (a*s + c, b*s + d) with one packed fp32x2 fused multiply-add: each lane
// is rounded once to nearest even, exactly as fmaf.
__device__ __forceinline__ void fma2(float& a, float& b, float s, float c, float d) {
  asm("{\n\t.reg .b64 ra, rs, rc, rd;\n\t"
      "mov.b64 ra, {%0, %1};\n\t"
      "mov.b64 rs, {%2, %2};\n\t"
      "mov.b64 rc, {%3, %4};\n\t"
      "fma.rn.f32x2 rd, ra, rs, rc;\n\t"
      "mov.b64 {%0, %1}, rd;\n\t}"
      : "+f"(a), "+f"(b)
      : "f"(s), "f"(c), "f"(d));
}

// fp8 codes of two already-scaled values packed low byte first.
template <int FMT>
__device__ __forceinline__ uint32_t cvt2(float lo, float hi) {
  return uint32_t(
      __nv_cvt_float2_to_fp8x2(make_float2(lo, hi), __NV_SATFINITE, FMT == FP8_E4M3 ? __NV_E4M3 : __NV_E5M2));
}

// Codes of v[0..3] * s in one word (v[0] in the low byte).
template <int FMT>
__device__ __forceinline__ uint32_t cvt4(float v0, float v1, float v2, float v3, float s) {
  scale2(v0, v1, s);
  scale2(v2, v3, s);
  return __byte_perm(cvt2<FMT>(v0, v1), cvt2<FMT>(v2, v3), 0x5410);
}

template <int FMT>
__device__ __forceinline__ uint32_t cvt_pair(float lo, float hi, float s) {
  scale2(lo, hi, s);
  return cvt2<FMT>(lo, hi);
}

template <int FMT>
__device__ __forceinline__ uint8_t cvt_one(float x, float s) {
  return uint8_t(__nv_cvt_float_to_fp8(__fmul_rn(x, s), __NV_SATFINITE,
                                       FMT == FP8_E4M3 ? __NV_E4M3 : __NV_E5M2));
}

// Commit amax `a` of one call to a ring.  `hist` holds the 16 history values
// as they were before the call (updated in place), `idx` the slot to write;
// history / idx_out / scale / scale_inv are the ring's words in global memory.
// s_used is the scale the call multiplied by.
template <int FMT>
__device__ __forceinline__ void ring_commit(float a, float* hist, int idx, float* history, int32_t* idx_out,
                                            float* scale, float* scale_inv, float s_used) {
  idx = ((idx % kHistoryLen) + kHistoryLen) % kHistoryLen;
  hist[idx] = a;
  float mx = 0.0f;
#pragma unroll
  for (int i = 0; i < kHistoryLen; ++i) mx = fmaxf(mx, hist[i]);
  history[idx] = a;
  *idx_out = (idx + 1) % kHistoryLen;
  const float fmax = FMT == FP8_E4M3 ? kE4M3Max : kE5M2Max;
  if (mx > 0.0f && isfinite(mx)) {
    const float c = __fdiv_rn(fmax, mx);
    if (isfinite(c) && c > 0.0f) *scale = c;
  }
  *scale_inv = __frcp_rn(s_used);
}

}  // namespace fp8ds
