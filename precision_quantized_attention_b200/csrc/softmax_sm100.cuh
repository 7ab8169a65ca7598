// softmax_sm100.cuh -- FP32 arithmetic of the attention softmax shared by the attention kernels:
// exact powers of two, the MUFU exp2, the FMA-pipe polynomial exp2 (packed f32x2), packed
// FMA/add helpers and the 128-score row maximum.
//
// The softmax computes p * 448 = 2^(S' - M + log2 448) for the base-2 scores S' and the
// integer running maximum M (NVIDIA developer blog "Optimizing FLUX.1 Kontext for Image Editing
// with Low-Precision Quantization", "Workflow and quantization", third SDPA bullet: softmax in
// FP32, no quantization at that stage).
#pragma once
#include <cuda_runtime.h>
#include <cstdint>

namespace qattn {

constexpr float LOG2E_F = 1.4426950408889634f;
constexpr float LOG2_448 = 8.807354922057604f;   // log2(448): p * 448 = 2^(S' - M + log2 448)

__device__ __forceinline__ float exp2_int(int k) {       // 2^k for k <= 0, exact (0 below 2^-126)
  return k < -126 ? 0.0f : __int_as_float((127 + k) << 23);
}

__device__ __forceinline__ float fast_exp2(float x) {    // MUFU ex2, flush-to-zero
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ float max3f(float a, float b, float c) {   // sm_100 3-input max
  float d;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}

// (d0, d1) = (a0 * b + c, a1 * b + c) with one packed f32x2 FMA.
__device__ __forceinline__ void ffma2_bc(float& d0, float& d1, float a0, float a1, float b, float c) {
  asm("{\n\t.reg .b64 ra, rb, rc, rd;\n\t"
      "mov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %4};\n\tmov.b64 rc, {%5, %5};\n\t"
      "fma.rn.f32x2 rd, ra, rb, rc;\n\tmov.b64 {%0, %1}, rd;\n\t}"
      : "=f"(d0), "=f"(d1)
      : "f"(a0), "f"(a1), "f"(b), "f"(c));
}

// (s0, s1) += (a0, a1) with one packed f32x2 add.
__device__ __forceinline__ void fadd2_acc(float& s0, float& s1, float a0, float a1) {
  asm("{\n\t.reg .b64 ra, rs;\n\t"
      "mov.b64 ra, {%2, %3};\n\tmov.b64 rs, {%0, %1};\n\t"
      "add.f32x2 rs, rs, ra;\n\tmov.b64 {%0, %1}, rs;\n\t}"
      : "+f"(s0), "+f"(s1)
      : "f"(a0), "f"(a1));
}

// 2^x on the FMA pipe for two values at once (packed f32x2), for x <= 9.  x is clamped at -125
// (2^-125 is far below the smallest E4M3 code of p * 448), split as x = n + f with
// n = round(x) (by adding and subtracting 1.5 * 2^23) and f in [-1/2, 1/2]; 2^f comes from a
// degree-5 minimax polynomial (relative error 2.1e-7 in binary32, fitted by
// csrc/fit_exp2_poly.py) and 2^n is added into the exponent field.
// Of every 8 pairs of scores, the pairs set in QATTN_POLY_MASK take the polynomial and the rest
// MUFU ex2; the default, pairs 1 and 5 (two of eight, spread apart in issue order), balances the
// two pipes.
#ifndef QATTN_POLY_MASK
#define QATTN_POLY_MASK 0x22
#endif
__device__ __forceinline__ constexpr bool poly_pair(int q) { return ((QATTN_POLY_MASK >> q) & 1) != 0; }
__device__ __forceinline__ void poly_exp2_x2(float x0, float x1, float& y0, float& y1) {
  x0 = fmaxf(x0, -125.0f);
  x1 = fmaxf(x1, -125.0f);
  float p0, p1, t0, t1;
  asm("{\n\t.reg .b64 x, t, n, f, p, m, nm, neg1, k;\n\t"
      "mov.b64 x, {%4, %5};\n\t"
      "mov.b64 m, {0f4B400000, 0f4B400000};\n\t"       // 1.5 * 2^23
      "mov.b64 nm, {0fCB400000, 0fCB400000};\n\t"
      "mov.b64 neg1, {0fBF800000, 0fBF800000};\n\t"
      "add.rn.f32x2 t, x, m;\n\t"                       // t = n + 1.5 * 2^23, n = round(x)
      "add.rn.f32x2 n, t, nm;\n\t"                      // n (exact)
      "fma.rn.f32x2 f, n, neg1, x;\n\t"                 // f = x - n (exact)
      "mov.b64 p, {0f3AAE0473, 0f3AAE0473};\n\t"        // c5
      "mov.b64 k, {0f3C1E8629, 0f3C1E8629};\n\t"        // c4
      "fma.rn.f32x2 p, p, f, k;\n\t"
      "mov.b64 k, {0f3D635B72, 0f3D635B72};\n\t"        // c3
      "fma.rn.f32x2 p, p, f, k;\n\t"
      "mov.b64 k, {0f3E75FC8C, 0f3E75FC8C};\n\t"        // c2
      "fma.rn.f32x2 p, p, f, k;\n\t"
      "mov.b64 k, {0f3F317214, 0f3F317214};\n\t"        // c1
      "fma.rn.f32x2 p, p, f, k;\n\t"
      "mov.b64 k, {0f3F800001, 0f3F800001};\n\t"        // c0
      "fma.rn.f32x2 p, p, f, k;\n\t"
      "mov.b64 {%0, %1}, p;\n\t"
      "mov.b64 {%2, %3}, t;\n\t}"
      : "=f"(p0), "=f"(p1), "=f"(t0), "=f"(t1)
      : "f"(x0), "f"(x1));
  // the low 9 bits of t hold n (two's complement); shifted into the exponent field they add n
  y0 = __int_as_float(__float_as_int(p0) + (__float_as_int(t0) << 23));
  y1 = __int_as_float(__float_as_int(p1) + (__float_as_int(t1) << 23));
}

// Row max of 64 scores: 8 independent chains of 3-input maxima, then a short tree.
__device__ __forceinline__ float rowmax64(const float (&s)[64]) {
  float m[8];
#pragma unroll
  for (int k = 0; k < 8; ++k) m[k] = max3f(s[k], s[k + 8], s[k + 16]);
#pragma unroll
  for (int i = 24; i < 56; i += 16) {
#pragma unroll
    for (int k = 0; k < 8; ++k) m[k] = max3f(m[k], s[i + k], s[i + 8 + k]);
  }
#pragma unroll
  for (int k = 0; k < 8; ++k) m[k] = fmaxf(m[k], s[56 + k]);
  return max3f(max3f(m[0], m[1], m[2]), max3f(m[3], m[4], m[5]), fmaxf(m[6], m[7]));
}

// Row max of 128 scores: 8 independent chains of 3-input maxima, then a short tree.
__device__ __forceinline__ float rowmax128(const float (&s)[128]) {
  float m[8];
#pragma unroll
  for (int k = 0; k < 8; ++k) m[k] = max3f(s[k], s[k + 8], s[k + 16]);
#pragma unroll
  for (int i = 24; i < 120; i += 16) {
#pragma unroll
    for (int k = 0; k < 8; ++k) m[k] = max3f(m[k], s[i + k], s[i + 8 + k]);
  }
#pragma unroll
  for (int k = 0; k < 8; ++k) m[k] = fmaxf(m[k], s[120 + k]);
  return max3f(max3f(m[0], m[1], m[2]), max3f(m[3], m[4], m[5]), fmaxf(m[6], m[7]));
}

// Test hook of the attention kernels: one row's P codes of a key step (word w: keys 4w..4w+3)
// and the integer maximum they are relative to, to the caller's buffers (codes + 128 * step,
// maxima + step).
__device__ __forceinline__ void capture_p_codes(uint8_t* codes, int* maxima, int step,
                                                const uint32_t (&pk)[32], float mx) {
  uint4* dst = reinterpret_cast<uint4*>(codes + static_cast<size_t>(step) * 128);
#pragma unroll
  for (int i = 0; i < 8; ++i) dst[i] = make_uint4(pk[4 * i], pk[4 * i + 1], pk[4 * i + 2], pk[4 * i + 3]);
  maxima[step] = static_cast<int>(mx);
}

}  // namespace qattn
