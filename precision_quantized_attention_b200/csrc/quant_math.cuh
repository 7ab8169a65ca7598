// quant_math.cuh -- the per-tensor FP8 quantization arithmetic shared by the quantize kernels
// (quant.cu) and the GEMM epilogue that emits E4M3 codes (gemm_fp8.cu): the correctly rounded
// quotient x / s (the NVIDIA developer blog "Optimizing FLUX.1 Kontext for Image Editing with
// Low-Precision Quantization", "Workflow and quantization": per-tensor FP8 FakeQuantize, here
// code = e4m3(fl32(x / s)) with s = fl32(amax / 448)) and bf16 unpacking.
#pragma once
#include <cstdint>

#include "sm100_ptx.cuh"

namespace qattn {

// -------------------------------------------------------------------------------------------
// Correctly rounded x / s for a divisor shared by many elements (Markstein's theorem: with
// r = RN(1/s) and q0 = RN(x * r), which is within one ulp of x / s, the residual
// x - q0 * s is exact in one FMA and RN(q0 + residual * r) = RN(x / s)).  Three FMA-pipe
// instructions instead of a division; valid while s, r and the residual stay normal, which
// `markstein_ok` checks once per divisor (callers use __fdiv_rn otherwise).  Quotients so small
// that they leave the normal range map to a signed zero E4M3/E2M1 code either way.
// -------------------------------------------------------------------------------------------
__device__ __forceinline__ bool markstein_ok(float s) {
  const float a = fabsf(s);
  return a >= 0x1p-100f && a <= 0x1p+100f;
}

// s > 0, so RN(x / s) has the sign of x; copysign restores it where the correction step's
// sum of zeros would not (x = -0, or a quotient that underflows).
__device__ __forceinline__ float div_rn_by(float x, float s, float r) {
  const float q0 = __fmul_rn(x, r);
  const float e = __fmaf_rn(-q0, s, x);
  return copysignf(__fmaf_rn(e, r, q0), x);
}

// Two quotients at once with packed f32x2 arithmetic: lane by lane the operations and roundings
// of div_rn_by (q0 = RN(x r), e = RN(x - q0 s) exact, RN(q0 + e r)), so the results are
// identical, in three instructions for two elements.  Used by the FP4 block quantize, whose
// per-element quotients dominate its instruction count.
__device__ __forceinline__ void div2_rn_by(float x0, float x1, float s, float r, float& q0, float& q1) {
  float a, b;
  asm("{\n\t.reg .b64 x, q, e, rr, ns;\n\t"
      "mov.b64 x, {%2, %3};\n\t"
      "mov.b64 rr, {%4, %4};\n\t"
      "mov.b64 ns, {%5, %5};\n\t"
      "mul.rn.f32x2 q, x, rr;\n\t"
      "fma.rn.f32x2 e, q, ns, x;\n\t"
      "fma.rn.f32x2 q, e, rr, q;\n\t"
      "mov.b64 {%0, %1}, q;\n\t}"
      : "=f"(a), "=f"(b)
      : "f"(x0), "f"(x1), "f"(r), "f"(-s));
  q0 = copysignf(a, x0);
  q1 = copysignf(b, x1);
}

// -------------------------------------------------------------------------------------------
// Per-tensor FP8: s = fl32(amax / 448), code = e4m3(fl32(x / s)); amax == 0 gives s = 1.
// -------------------------------------------------------------------------------------------
__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

template <bool FAST>
__device__ __forceinline__ float div_s(float x, float s, float r) {
  return FAST ? div_rn_by(x, s, r) : __fdiv_rn(x, s);
}

template <bool FAST>
__device__ __forceinline__ uint32_t quant4_e4m3(uint32_t w0, uint32_t w1, float s, float r) {
  const uint32_t lo = cvt_e4m3x2(div_s<FAST>(bf16_lo(w0), s, r), div_s<FAST>(bf16_hi(w0), s, r));
  const uint32_t hi = cvt_e4m3x2(div_s<FAST>(bf16_lo(w1), s, r), div_s<FAST>(bf16_hi(w1), s, r));
  return lo | (hi << 16);
}

}  // namespace qattn
