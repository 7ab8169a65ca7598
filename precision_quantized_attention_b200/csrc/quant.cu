// quant.cu -- HBM-bound calibration and FakeQuantize passes for Q, K and V.
//
// Method: NVIDIA developer blog "Optimizing FLUX.1 Kontext for Image Editing with Low-Precision
// Quantization", section "Workflow and quantization": Q, K, V are quantized per tensor to FP8
// or per block to FP4 (first SDPA bullet, Fig. 4), an extra FP8 quantize feeds BMM1 (second
// bullet), and scales come from post-training calibration (steps 3-4 of the flow), reduced here
// to max-calibration of the tensor in hand.
//
// Every kernel streams its input once with 16-byte loads over a grid sized to the SM count,
// and applies scales as correctly rounded binary32 quotients (Markstein's multiply-and-correct
// form for a shared divisor), so the codes are bit-identical to the definition (E4M3 / E2M1
// round-to-nearest-even with saturation, the hardware cvt forms).
#include <cuda_runtime.h>
#include <type_traits>
#include <cstdint>

#include "device_once.h"
#include "quant_math.cuh"
#include "launch.h"
#include "sm100_ptx.cuh"

namespace qattn {

// -------------------------------------------------------------------------------------------
// amax = max |x| over a bf16 tensor.  |x| of a bf16 is its bit pattern with the sign cleared,
// and for non-negative values (NaN and inf included) the integer order of those patterns is
// the numeric order, so the reduction runs on 16-bit integers (two per 32-bit word).
// The result is written as float bits with one atomicMax per CTA; the host zeroes it first.
// -------------------------------------------------------------------------------------------
__device__ __forceinline__ uint32_t absmax_word(uint32_t m2, uint32_t w) {
  return __vmaxu2(m2, w & 0x7FFF7FFFu);
}

__global__ void __launch_bounds__(256) k_amax_bf16(const uint4* __restrict__ xv, size_t nvec,
                                                   const uint16_t* __restrict__ xtail, int ntail,
                                                   unsigned* __restrict__ amax_bits,
                                                   int* __restrict__ err) {
  uint32_t m2 = 0;
  const size_t stride = static_cast<size_t>(gridDim.x) * blockDim.x;
  size_t i = static_cast<size_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  for (; i + 3 * stride < nvec; i += 4 * stride) {
    uint4 a = __ldcs(xv + i), b = __ldcs(xv + i + stride);
    uint4 c = __ldcs(xv + i + 2 * stride), d = __ldcs(xv + i + 3 * stride);
    m2 = absmax_word(m2, a.x); m2 = absmax_word(m2, a.y);
    m2 = absmax_word(m2, a.z); m2 = absmax_word(m2, a.w);
    m2 = absmax_word(m2, b.x); m2 = absmax_word(m2, b.y);
    m2 = absmax_word(m2, b.z); m2 = absmax_word(m2, b.w);
    m2 = absmax_word(m2, c.x); m2 = absmax_word(m2, c.y);
    m2 = absmax_word(m2, c.z); m2 = absmax_word(m2, c.w);
    m2 = absmax_word(m2, d.x); m2 = absmax_word(m2, d.y);
    m2 = absmax_word(m2, d.z); m2 = absmax_word(m2, d.w);
  }
  for (; i < nvec; i += stride) {
    uint4 a = __ldcs(xv + i);
    m2 = absmax_word(m2, a.x); m2 = absmax_word(m2, a.y);
    m2 = absmax_word(m2, a.z); m2 = absmax_word(m2, a.w);
  }
  uint32_t m = max(m2 & 0xFFFFu, m2 >> 16);
  if (blockIdx.x == 0 && static_cast<int>(threadIdx.x) < ntail)
    m = max(m, static_cast<uint32_t>(xtail[threadIdx.x]) & 0x7FFFu);
  m = __reduce_max_sync(0xFFFFFFFFu, m);
  __shared__ uint32_t warp_max[8];
  if ((threadIdx.x & 31) == 0) warp_max[threadIdx.x >> 5] = m;
  __syncthreads();
  if (threadIdx.x < 32) {
    m = threadIdx.x < (blockDim.x >> 5) ? warp_max[threadIdx.x] : 0u;
    m = __reduce_max_sync(0xFFFFFFFFu, m);
    if (threadIdx.x == 0) {
      if (m >= 0x7F80u) atomicExch(err, DEV_ERR_NONFINITE);
      atomicMax(amax_bits, m << 16);
    }
  }
}

// nloop: the element loop's bound in 8-element vectors, nvec except under the checked build's
// injection test (nvec + 1), where the bounds checks must stop the extra vector.
__global__ void __launch_bounds__(256) k_quant_fp8(const uint4* __restrict__ xv, size_t nvec,
                                                   size_t nloop,
                                                   const uint16_t* __restrict__ xtail, int ntail,
                                                   const float* __restrict__ amax_p,
                                                   uint2* __restrict__ outv,
                                                   uint8_t* __restrict__ outtail,
                                                   float* __restrict__ scale_out,
                                                   int* __restrict__ err) {
  const float amax = *amax_p;
  if (!(amax <= 3.402823466e38f)) {  // inf or NaN: nothing is written
    if (blockIdx.x == 0 && threadIdx.x == 0) atomicExch(err, DEV_ERR_NONFINITE);
    return;
  }
  const float s = (amax == 0.0f) ? 1.0f : __fdiv_rn(amax, 448.0f);
  if (blockIdx.x == 0 && threadIdx.x == 0) *scale_out = s;
  const float r = __frcp_rn(s);
  const size_t stride = static_cast<size_t>(gridDim.x) * blockDim.x;
  const size_t i0 = static_cast<size_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (markstein_ok(s)) {
    for (size_t i = i0; i < nloop; i += stride) {
      if (!QATTN_IN_BOUNDS(err, i < nvec)) continue;
      const uint4 a = __ldcs(xv + i);
      __stcs(outv + i, make_uint2(quant4_e4m3<true>(a.x, a.y, s, r), quant4_e4m3<true>(a.z, a.w, s, r)));
    }
  } else {
    for (size_t i = i0; i < nloop; i += stride) {
      if (!QATTN_IN_BOUNDS(err, i < nvec)) continue;
      const uint4 a = __ldcs(xv + i);
      __stcs(outv + i, make_uint2(quant4_e4m3<false>(a.x, a.y, s, r), quant4_e4m3<false>(a.z, a.w, s, r)));
    }
  }
  if (blockIdx.x == 0 && static_cast<int>(threadIdx.x) < ntail) {
    const float x = __uint_as_float(static_cast<uint32_t>(xtail[threadIdx.x]) << 16);
    outtail[threadIdx.x] = static_cast<uint8_t>(cvt_e4m3x2(__fdiv_rn(x, s), 0.0f) & 0xFFu);
  }
}

// -------------------------------------------------------------------------------------------
// Per-block FP4 (16 elements, E2M1 values, E4M3 block scale, FP32 tensor scale), fused with the
// per-tensor FP8 requantization of the dequantized values that feeds BMM1:
//   s_g = fl32(amax / 2688); s_b = e4m3(fl32(amax_b / fl32(6 s_g))); eff = fl32(val(s_b) s_g)
//   c = e2m1(fl32(x / eff)) (eff == 0: c = 0);  xhat = fl32(fl32(val(c) val(s_b)) s_g)
//   s8 = fl32(max|xhat| / 448), c8 = e4m3(fl32(xhat / s8)).
// max|xhat| needs no second pass: the block that holds the tensor amax gets s_b = 448 and code
// 6 (amax / fl32(6 s_g) rounds to 448 in E4M3 and amax / eff rounds to 6 in E2M1), and no
// other |xhat| can exceed fl32(fl32(6 * 448) * s_g), so max|xhat| = fl32(2688 * s_g).
// One thread per block: two 16-byte loads, an 8-byte packed store, the scale byte and a
// 16-byte store of FP8 codes.
// -------------------------------------------------------------------------------------------
// FP8 requant table of one tensor: for every E4M3 block-scale code b (0..127: block scales are
// never negative) and E2M1 magnitude m (0..7) the E4M3 code of the dequantized value over s8,
//   requant[8 b + m] = e4m3(fl32(fl32(fl32(val(m) * val(b)) * s_g) / s8)),
// in the same product order as the element-wise definition.  A negative E2M1 code gives the
// same code with the sign bit set: the products, the quotient and round-to-nearest-even are
// sign-symmetric, and -0 becomes 0x80.
// Per block-scale code the divisor of the block's E2M1 quotients is tabulated too:
//   er[b] = (eff, RN(1 / eff)), eff = fl32(val(b) * s_g),
// and the quotient that picks the block scale, amax_b / fl32(6 s_g), uses the tensor's
// RN(1 / fl32(6 s_g)) in Markstein's form (correctly rounded, as every quotient here).
// Built by the whole CTA (then synchronized).
struct Fp4Tables {
  uint2 requant[128];        // 8 requant codes (one per E2M1 magnitude) per block-scale code
  float2 er[128];            // (eff, RN(1 / eff)) per block-scale code
  float r_six;               // RN(1 / fl32(6 s_g))
  int fast_six;              // markstein_ok(fl32(6 s_g))
};

__device__ __forceinline__ void build_fp4_tables(Fp4Tables* tab, float sg, float six_sg, float s8) {
  const float r8 = __frcp_rn(s8);
  const bool fast8 = markstein_ok(s8);
  uint8_t* bytes = reinterpret_cast<uint8_t*>(tab->requant);
  for (int i = threadIdx.x; i < 1024; i += blockDim.x) {
    const float xh = __fmul_rn(__fmul_rn(e2m1_to_f32(static_cast<uint32_t>(i & 7)),
                                         e4m3_to_f32(static_cast<uint32_t>(i >> 3))), sg);
    const float d = fast8 ? div_rn_by(xh, s8, r8) : __fdiv_rn(xh, s8);
    bytes[i] = static_cast<uint8_t>(cvt_e4m3x2(d, 0.0f) & 0xFFu);
  }
  for (int b = threadIdx.x; b < 128; b += blockDim.x) {
    const float eff = __fmul_rn(e4m3_to_f32(static_cast<uint32_t>(b)), sg);
    tab->er[b] = make_float2(eff, eff != 0.0f ? __frcp_rn(eff) : 0.0f);
  }
  if (threadIdx.x == 0) {
    tab->r_six = __frcp_rn(six_sg);
    tab->fast_six = markstein_ok(six_sg) ? 1 : 0;
  }
}

// Four requant codes from four E2M1 codes packed as nibbles (low 16 bits of `nib4`) and the
// two bf16 words they came from: the magnitudes index the block's 8-entry table (one byte
// permute), and each code takes the sign of its input (the E2M1 code keeps the input's sign,
// -0 included).
__device__ __forceinline__ uint32_t requant4(uint2 t, uint32_t nib4, uint32_t w0, uint32_t w1) {
  return __byte_perm(t.x, t.y, nib4 & 0x7777u) | (__byte_perm(w0, w1, 0x7531u) & 0x80808080u);
}

// One 16-element block: E2M1 codes, E4M3 block scale and (optionally) the FP8 requant codes,
// the latter looked up in the tensor's tables.
__device__ __forceinline__ void fp4_block(uint4 a0, uint4 a1, size_t b, float six_sg,
                                          const Fp4Tables* __restrict__ tab,
                                          uint2* __restrict__ packed_out,
                                          uint8_t* __restrict__ bscale_out,
                                          uint4* __restrict__ codes8_out) {
  const uint32_t w[8] = {a0.x, a0.y, a0.z, a0.w, a1.x, a1.y, a1.z, a1.w};
  uint32_t am2 = 0;
#pragma unroll
  for (int i = 0; i < 8; ++i) am2 = absmax_word(am2, w[i]);
  const float amax_b = __uint_as_float(max(am2 & 0xFFFFu, am2 >> 16) << 16);
  const float qb = tab->fast_six ? div_rn_by(amax_b, six_sg, tab->r_six) : __fdiv_rn(amax_b, six_sg);
  const uint32_t sb = cvt_e4m3x2(qb, 0.0f) & 0xFFu;  // amax_b >= 0: sb < 128
  const float2 er = tab->er[sb & 0x7Fu];
  const float eff = er.x;
  uint32_t pk0 = 0, pk1 = 0;
  uint32_t c8[4] = {0u, 0u, 0u, 0u};
  if (eff != 0.0f) {
    const float r_eff = er.y;
    const bool fast_eff = markstein_ok(eff);
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const float x0 = bf16_lo(w[i]), x1 = bf16_hi(w[i]);
      float q0, q1;
      if (fast_eff) {
        div2_rn_by(x0, x1, eff, r_eff, q0, q1);
      } else {
        q0 = __fdiv_rn(x0, eff);
        q1 = __fdiv_rn(x1, eff);
      }
      const uint32_t byte = cvt_e2m1x2(q0, q1);
      if (i < 4) pk0 |= byte << (8 * i);
      else pk1 |= byte << (8 * (i - 4));
    }
    if (codes8_out) {
      const uint2 t = tab->requant[sb & 0x7Fu];
      c8[0] = requant4(t, pk0, w[0], w[1]);
      c8[1] = requant4(t, pk0 >> 16, w[2], w[3]);
      c8[2] = requant4(t, pk1, w[4], w[5]);
      c8[3] = requant4(t, pk1 >> 16, w[6], w[7]);
    }
  }
  __stcs(packed_out + b, make_uint2(pk0, pk1));
  bscale_out[b] = static_cast<uint8_t>(sb);
  if (codes8_out) __stcs(codes8_out + b, make_uint4(c8[0], c8[1], c8[2], c8[3]));
}

__global__ void __launch_bounds__(256) k_quant_fp4_block(
    const uint4* __restrict__ xv, size_t nblocks, const float* __restrict__ amax_p,
    uint2* __restrict__ packed_out, uint8_t* __restrict__ bscale_out,
    float* __restrict__ gscale_out, uint4* __restrict__ codes8_out,
    float* __restrict__ scale8_out, int* __restrict__ err) {
  const float amax = *amax_p;
  if (!(amax <= 3.402823466e38f)) {
    if (blockIdx.x == 0 && threadIdx.x == 0) atomicExch(err, DEV_ERR_NONFINITE);
    return;
  }
  const float sg = (amax == 0.0f) ? 1.0f : __fdiv_rn(amax, 2688.0f);
  const float six_sg = __fmul_rn(6.0f, sg);
  const float s8 = (amax == 0.0f) ? 1.0f : __fdiv_rn(__fmul_rn(2688.0f, sg), 448.0f);
  if (blockIdx.x == 0 && threadIdx.x == 0) {
    *gscale_out = sg;
    if (scale8_out) *scale8_out = s8;
  }
  __shared__ Fp4Tables tab;
  build_fp4_tables(&tab, sg, six_sg, s8);
  __syncthreads();
  const size_t stride = static_cast<size_t>(gridDim.x) * blockDim.x;
  for (size_t b = static_cast<size_t>(blockIdx.x) * blockDim.x + threadIdx.x; b < nblocks;
       b += stride)
    fp4_block(__ldcs(xv + 2 * b), __ldcs(xv + 2 * b + 1), b, six_sg, &tab, packed_out,
              bscale_out, codes8_out);
}

// -------------------------------------------------------------------------------------------
// Fused calibrate + quantize (one cooperative launch per tensor).  Every CTA reduces the amax of
// its contiguous chunk, publishes it with one max reduction into the workspace and arrives on a
// grid-wide counter; after the last arrival every CTA quantizes its chunk, which it just read
// and which is still in L2, so HBM sees the input once.  The spin on the counter is bounded by
// a global-timer limit (a launch that somehow is not co-resident records DEV_ERR_TIMEOUT and
// writes nothing).  Each CTA departs on a second counter when it is done; the last CTA to
// depart zeroes the workspace again, so it needs zeroing only before its first use and no reset
// launch precedes a call.
// -------------------------------------------------------------------------------------------
// The arrival counter has a 128-byte line of its own: the pollers read it while the other CTAs
// still publish their maxima into the first line.
struct FusedWorkspace {
  unsigned amax_bits;
  unsigned departed;
  unsigned pad0[30];
  unsigned arrived;
  unsigned pad1[31];
};
static_assert(sizeof(FusedWorkspace) <= 256, "fits QATTN_FUSED_WORKSPACE_BYTES");

__device__ __forceinline__ unsigned ld_acquire_gpu(const unsigned* p) {
  unsigned v;
  asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

// Reduces m over the CTA, publishes it, waits for every CTA; returns the tensor amax (as float
// bits) in every thread, or 0xFFFFFFFF after a timeout.  One thread per CTA publishes with a
// fire-and-forget max reduction and a releasing add on the arrival counter, then polls the
// counter with acquire loads and a short sleep between polls (444 pollers on one line would
// otherwise slow the arrivals down).
__device__ __forceinline__ unsigned grid_amax(uint32_t m, FusedWorkspace* ws, uint64_t limit_ns,
                                              int* err) {
  __shared__ uint32_t warp_max[32];
  __shared__ unsigned result;
  m = __reduce_max_sync(0xFFFFFFFFu, m);
  if ((threadIdx.x & 31) == 0) warp_max[threadIdx.x >> 5] = m;
  __syncthreads();
  if (threadIdx.x < 32) {
    m = threadIdx.x < (blockDim.x >> 5) ? warp_max[threadIdx.x] : 0u;
    m = __reduce_max_sync(0xFFFFFFFFu, m);
    if (threadIdx.x == 0) {
      asm volatile("red.relaxed.gpu.global.max.u32 [%0], %1;" ::"l"(&ws->amax_bits), "r"(m << 16)
                   : "memory");
      asm volatile("red.release.gpu.global.add.u32 [%0], 1;" ::"l"(&ws->arrived) : "memory");
      const uint64_t t0 = global_timer_ns();
      unsigned r = 0xFFFFFFFFu;
      while (true) {
        if (ld_acquire_gpu(&ws->arrived) >= gridDim.x) {
          r = ld_acquire_gpu(&ws->amax_bits);
          break;
        }
        if (global_timer_ns() - t0 > limit_ns) {
          atomicExch(err, DEV_ERR_TIMEOUT);
          break;
        }
        __nanosleep(32);
      }
      result = r;
    }
  }
  __syncthreads();
  return result;
}

// Called by every CTA once it no longer needs the workspace (at its end, off the critical path):
// when the last CTA departs, every CTA has read the amax, so it zeroes the workspace for the
// next call.
__device__ __forceinline__ void grid_depart(FusedWorkspace* ws) {
  if (threadIdx.x == 0) {
    unsigned old;
    asm volatile("atom.acq_rel.gpu.global.add.u32 %0, [%1], 1;"
                 : "=r"(old)
                 : "l"(&ws->departed)
                 : "memory");
    if (old == gridDim.x - 1) {
      ws->amax_bits = 0u;
      ws->arrived = 0u;
      ws->departed = 0u;
    }
  }
}

constexpr int FUSED_THREADS = 1024;    // one CTA per SM: fewer arrivals on the grid barrier
constexpr int FUSED_UNROLL = 4;       // independent 16-byte loads in flight per thread

// L2 eviction priorities: phase 1 marks the chunk evict-last so that it is still in L2 when
// phase 2 reads it back (evict-first, it is not needed afterwards).  Without the hint the L2
// does not keep a streamed tensor of tens of MB and phase 2 goes back to HBM.
__device__ __forceinline__ uint64_t l2_policy_evict_last() {
  uint64_t p;
  asm volatile("createpolicy.fractional.L2::evict_last.b64 %0, 1.0;" : "=l"(p));
  return p;
}
__device__ __forceinline__ uint64_t l2_policy_evict_first() {
  uint64_t p;
  asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(p));
  return p;
}
__device__ __forceinline__ uint4 ld_hint(const uint4* p, uint64_t pol) {
  uint4 v;
  asm volatile("ld.global.nc.L2::cache_hint.v4.u32 {%0, %1, %2, %3}, [%4], %5;"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p), "l"(pol));
  return v;
}

// Packed bf16 |x| maximum over the vectors [lo, hi) of this CTA's chunk (phase 1).
__device__ __forceinline__ uint32_t chunk_absmax(const uint4* __restrict__ xv, size_t lo,
                                                 size_t hi) {
  constexpr size_t T = FUSED_THREADS, U = FUSED_UNROLL;
  const uint64_t pol = l2_policy_evict_last();
  uint32_t m2 = 0;
  size_t i = lo + threadIdx.x;
  for (; i + (U - 1) * T < hi; i += U * T) {
    uint4 a[U];
#pragma unroll
    for (size_t u = 0; u < U; ++u) a[u] = ld_hint(xv + i + u * T, pol);
#pragma unroll
    for (size_t u = 0; u < U; ++u) {
      m2 = absmax_word(m2, a[u].x); m2 = absmax_word(m2, a[u].y);
      m2 = absmax_word(m2, a[u].z); m2 = absmax_word(m2, a[u].w);
    }
  }
  for (; i < hi; i += T) {
    const uint4 a = ld_hint(xv + i, pol);
    m2 = absmax_word(m2, a.x); m2 = absmax_word(m2, a.y);
    m2 = absmax_word(m2, a.z); m2 = absmax_word(m2, a.w);
  }
  return m2;
}

// FP8 codes of the vectors [lo, hi) (phase 2): the chunk comes back from L2.
template <bool FAST>
__device__ __forceinline__ void chunk_quant_fp8(const uint4* __restrict__ xv,
                                                uint2* __restrict__ outv, size_t lo, size_t hi,
                                                float s, float r) {
  constexpr size_t T = FUSED_THREADS, U = FUSED_UNROLL;
  const uint64_t pol = l2_policy_evict_first();
  size_t i = lo + threadIdx.x;
  for (; i + (U - 1) * T < hi; i += U * T) {
    uint4 a[U];
#pragma unroll
    for (size_t u = 0; u < U; ++u) a[u] = ld_hint(xv + i + u * T, pol);
#pragma unroll
    for (size_t u = 0; u < U; ++u)
      __stcs(outv + i + u * T, make_uint2(quant4_e4m3<FAST>(a[u].x, a[u].y, s, r),
                                          quant4_e4m3<FAST>(a[u].z, a[u].w, s, r)));
  }
  for (; i < hi; i += T) {
    const uint4 a = ld_hint(xv + i, pol);
    __stcs(outv + i, make_uint2(quant4_e4m3<FAST>(a.x, a.y, s, r), quant4_e4m3<FAST>(a.z, a.w, s, r)));
  }
}

__global__ void __launch_bounds__(FUSED_THREADS) k_calib_quant_fp8(
    const uint4* __restrict__ xv, size_t nvec, const uint16_t* __restrict__ xtail, int ntail,
    float* __restrict__ amax_out, uint2* __restrict__ outv, uint8_t* __restrict__ outtail,
    float* __restrict__ scale_out, FusedWorkspace* ws, uint64_t limit_ns, int* __restrict__ err) {
  // contiguous chunk per CTA (in 16-byte vectors)
  const size_t per = (nvec + gridDim.x - 1) / gridDim.x;
  const size_t lo = static_cast<size_t>(blockIdx.x) * per;
  const size_t hi = lo + per < nvec ? lo + per : nvec;
  const uint32_t m2 = chunk_absmax(xv, lo, hi);
  uint32_t m = max(m2 & 0xFFFFu, m2 >> 16);
  if (blockIdx.x == 0 && static_cast<int>(threadIdx.x) < ntail)
    m = max(m, static_cast<uint32_t>(xtail[threadIdx.x]) & 0x7FFFu);
  const unsigned bits = grid_amax(m, ws, limit_ns, err);
  if (bits == 0xFFFFFFFFu) {
    grid_depart(ws);
    return;
  }
  const float amax = __uint_as_float(bits);
  if (!(amax <= 3.402823466e38f)) {
    if (blockIdx.x == 0 && threadIdx.x == 0) {
      atomicExch(err, DEV_ERR_NONFINITE);
      *amax_out = amax;
    }
    grid_depart(ws);
    return;
  }
  const float s = (amax == 0.0f) ? 1.0f : __fdiv_rn(amax, 448.0f);
  if (blockIdx.x == 0 && threadIdx.x == 0) {
    *amax_out = amax;
    *scale_out = s;
  }
  const float r = __frcp_rn(s);
  if (markstein_ok(s))
    chunk_quant_fp8<true>(xv, outv, lo, hi, s, r);
  else
    chunk_quant_fp8<false>(xv, outv, lo, hi, s, r);
  if (blockIdx.x == 0 && static_cast<int>(threadIdx.x) < ntail) {
    const float x = __uint_as_float(static_cast<uint32_t>(xtail[threadIdx.x]) << 16);
    outtail[threadIdx.x] = static_cast<uint8_t>(cvt_e4m3x2(__fdiv_rn(x, s), 0.0f) & 0xFFu);
  }
  grid_depart(ws);
}

__global__ void __launch_bounds__(FUSED_THREADS) k_calib_quant_fp4_block(
    const uint4* __restrict__ xv, size_t nblocks, float* __restrict__ amax_out,
    uint2* __restrict__ packed_out, uint8_t* __restrict__ bscale_out,
    float* __restrict__ gscale_out, uint4* __restrict__ codes8_out,
    float* __restrict__ scale8_out, FusedWorkspace* ws, uint64_t limit_ns, int* __restrict__ err) {
  const size_t per = (nblocks + gridDim.x - 1) / gridDim.x;   // contiguous chunk of blocks
  const size_t lo = static_cast<size_t>(blockIdx.x) * per;
  const size_t hi = lo + per < nblocks ? lo + per : nblocks;
  const uint32_t m2 = chunk_absmax(xv, 2 * lo, 2 * hi);
  const unsigned bits = grid_amax(max(m2 & 0xFFFFu, m2 >> 16), ws, limit_ns, err);
  if (bits == 0xFFFFFFFFu) {
    grid_depart(ws);
    return;
  }
  const float amax = __uint_as_float(bits);
  if (!(amax <= 3.402823466e38f)) {
    if (blockIdx.x == 0 && threadIdx.x == 0) {
      atomicExch(err, DEV_ERR_NONFINITE);
      *amax_out = amax;
    }
    grid_depart(ws);
    return;
  }
  const float sg = (amax == 0.0f) ? 1.0f : __fdiv_rn(amax, 2688.0f);
  const float six_sg = __fmul_rn(6.0f, sg);
  const float s8 = (amax == 0.0f) ? 1.0f : __fdiv_rn(__fmul_rn(2688.0f, sg), 448.0f);
  if (blockIdx.x == 0 && threadIdx.x == 0) {
    *amax_out = amax;
    *gscale_out = sg;
    if (scale8_out) *scale8_out = s8;
  }
  __shared__ Fp4Tables tab;
  build_fp4_tables(&tab, sg, six_sg, s8);
  __syncthreads();
  const uint64_t pol = l2_policy_evict_first();
  size_t b = lo + threadIdx.x;
  for (; b + FUSED_THREADS < hi; b += 2 * FUSED_THREADS) {     // two blocks' loads in flight
    const uint4 a0 = ld_hint(xv + 2 * b, pol), a1 = ld_hint(xv + 2 * b + 1, pol);
    const uint4 c0 = ld_hint(xv + 2 * (b + FUSED_THREADS), pol);
    const uint4 c1 = ld_hint(xv + 2 * (b + FUSED_THREADS) + 1, pol);
    fp4_block(a0, a1, b, six_sg, &tab, packed_out, bscale_out, codes8_out);
    fp4_block(c0, c1, b + FUSED_THREADS, six_sg, &tab, packed_out, bscale_out, codes8_out);
  }
  for (; b < hi; b += FUSED_THREADS)
    fp4_block(ld_hint(xv + 2 * b, pol), ld_hint(xv + 2 * b + 1, pol), b, six_sg, &tab,
              packed_out, bscale_out, codes8_out);
  grid_depart(ws);
}

// -------------------------------------------------------------------------------------------
// Q, K and V in one cooperative launch.  Stage 0 reduces Q's amax; stage s = 1, 2 quantizes
// tensor s - 1 (its chunk comes back from L2, evict-first) while it reduces tensor s's amax from
// HBM (evict-last), so the L2-bound half of one tensor overlaps the HBM-bound half of the next;
// stage 3 quantizes V.  The stages are separated by grid barriers on one monotonic arrival
// counter.  No CTA leaves early: a tensor whose amax is not finite (or a barrier that timed
// out) only suppresses that tensor's writes, so every CTA arrives at every barrier.
// -------------------------------------------------------------------------------------------
constexpr int QKV = 3;

struct QkvWorkspace {
  unsigned amax_bits[4];
  unsigned departed;
  unsigned pad0[27];
  unsigned arrived;          // own 128-byte line
  unsigned pad1[31];
};
static_assert(sizeof(QkvWorkspace) <= 256, "fits QATTN_FUSED_WORKSPACE_BYTES");

struct QkvTensor {
  const uint4* x;            // n bf16 as 16-byte vectors
  uint8_t* codes8;           // n E4M3 codes (FP8 mode: the codes; FP4 mode: the requant codes)
  float* amax;
  float* scale8;             // dequantization multiplier of codes8
  uint2* e2m1;               // FP4 mode: n / 2 bytes of packed codes
  uint8_t* bscale;           // FP4 mode: n / 16 block scales
  float* gscale;             // FP4 mode: the FP32 tensor scale
};

struct QkvArgs {
  QkvTensor t[QKV];
  size_t n;                  // elements per tensor
  uint64_t limit_ns;
  int* err;
  QkvWorkspace* ws;
};

// CTA-reduce m, publish it into `slot`, arrive, wait until `target` arrivals; returns the
// published maximum (float bits) or 0xFFFFFFFF after a timeout.
__device__ __forceinline__ unsigned grid_stage(uint32_t m, unsigned* slot, unsigned* arrived,
                                               unsigned target, uint64_t limit_ns, int* err) {
  __shared__ uint32_t warp_max[32];
  __shared__ unsigned result;
  m = __reduce_max_sync(0xFFFFFFFFu, m);
  if ((threadIdx.x & 31) == 0) warp_max[threadIdx.x >> 5] = m;
  __syncthreads();
  if (threadIdx.x < 32) {
    m = threadIdx.x < (blockDim.x >> 5) ? warp_max[threadIdx.x] : 0u;
    m = __reduce_max_sync(0xFFFFFFFFu, m);
    if (threadIdx.x == 0) {
      asm volatile("red.relaxed.gpu.global.max.u32 [%0], %1;" ::"l"(slot), "r"(m << 16) : "memory");
      asm volatile("red.release.gpu.global.add.u32 [%0], 1;" ::"l"(arrived) : "memory");
      const uint64_t t0 = global_timer_ns();
      unsigned r = 0xFFFFFFFFu;
      while (true) {
        if (ld_acquire_gpu(arrived) >= target) {
          r = ld_acquire_gpu(slot);
          break;
        }
        if (global_timer_ns() - t0 > limit_ns) {
          atomicExch(err, DEV_ERR_TIMEOUT);
          break;
        }
        __nanosleep(32);
      }
      result = r;
    }
  }
  __syncthreads();
  return result;
}

__device__ __forceinline__ uint32_t fold_max(uint32_t m2) { return max(m2 & 0xFFFFu, m2 >> 16); }

// One FP8 stage over the vectors [lo, hi): quantize xp into op (when xp is set) and reduce the
// packed |x| maximum of xc (when xc is set).
template <bool FAST>
__device__ __forceinline__ uint32_t qkv_stage_fp8(const uint4* __restrict__ xp,
                                                  uint2* __restrict__ op, float s, float r,
                                                  const uint4* __restrict__ xc, size_t lo,
                                                  size_t hi) {
  constexpr size_t T = FUSED_THREADS, U = FUSED_UNROLL;
  const uint64_t pf = l2_policy_evict_first(), pl = l2_policy_evict_last();
  uint32_t m2 = 0;
  size_t i = lo + threadIdx.x;
  for (; i + (U - 1) * T < hi; i += U * T) {
    uint4 a[U], b[U];
    if (xc) {
#pragma unroll
      for (size_t u = 0; u < U; ++u) b[u] = ld_hint(xc + i + u * T, pl);
    }
    if (xp) {
#pragma unroll
      for (size_t u = 0; u < U; ++u) a[u] = ld_hint(xp + i + u * T, pf);
    }
    if (xc) {
#pragma unroll
      for (size_t u = 0; u < U; ++u) {
        m2 = absmax_word(m2, b[u].x); m2 = absmax_word(m2, b[u].y);
        m2 = absmax_word(m2, b[u].z); m2 = absmax_word(m2, b[u].w);
      }
    }
    if (xp) {
#pragma unroll
      for (size_t u = 0; u < U; ++u)
        __stcs(op + i + u * T, make_uint2(quant4_e4m3<FAST>(a[u].x, a[u].y, s, r),
                                          quant4_e4m3<FAST>(a[u].z, a[u].w, s, r)));
    }
  }
  for (; i < hi; i += T) {
    if (xc) {
      const uint4 b = ld_hint(xc + i, pl);
      m2 = absmax_word(m2, b.x); m2 = absmax_word(m2, b.y);
      m2 = absmax_word(m2, b.z); m2 = absmax_word(m2, b.w);
    }
    if (xp) {
      const uint4 a = ld_hint(xp + i, pf);
      __stcs(op + i, make_uint2(quant4_e4m3<FAST>(a.x, a.y, s, r), quant4_e4m3<FAST>(a.z, a.w, s, r)));
    }
  }
  return m2;
}

// One FP4 stage over the 16-element blocks [lo, hi): block-quantize xp into e2m1 / bscale /
// codes8 (when xp is set) and reduce the packed |x| maximum of xc (when xc is set).
__device__ __forceinline__ uint32_t qkv_stage_fp4(const uint4* __restrict__ xp,
                                                  uint2* __restrict__ e2m1,
                                                  uint8_t* __restrict__ bscale,
                                                  uint4* __restrict__ codes8,
                                                  float six_sg, const Fp4Tables* __restrict__ tab,
                                                  const uint4* __restrict__ xc, size_t lo,
                                                  size_t hi) {
  constexpr size_t T = FUSED_THREADS;
  const uint64_t pf = l2_policy_evict_first(), pl = l2_policy_evict_last();
  uint32_t m2 = 0;
  for (size_t b = lo + threadIdx.x; b < hi; b += T) {
    uint4 c0, c1, a0, a1;
    if (xc) {
      c0 = ld_hint(xc + 2 * b, pl);
      c1 = ld_hint(xc + 2 * b + 1, pl);
    }
    if (xp) {
      a0 = ld_hint(xp + 2 * b, pf);
      a1 = ld_hint(xp + 2 * b + 1, pf);
    }
    if (xc) {
      m2 = absmax_word(m2, c0.x); m2 = absmax_word(m2, c0.y);
      m2 = absmax_word(m2, c0.z); m2 = absmax_word(m2, c0.w);
      m2 = absmax_word(m2, c1.x); m2 = absmax_word(m2, c1.y);
      m2 = absmax_word(m2, c1.z); m2 = absmax_word(m2, c1.w);
    }
    if (xp) fp4_block(a0, a1, b, six_sg, tab, e2m1, bscale, codes8);
  }
  return m2;
}

template <int MODE>   // 0: per-tensor FP8, 1: FP4 blocks + FP8 requant
__global__ void __launch_bounds__(FUSED_THREADS) k_calib_quant_qkv(const QkvArgs a) {
  QkvWorkspace* ws = a.ws;
  // FP8 works on 16-byte vectors (a tail of n % 8 elements goes to CTA 0); FP4 on 16-element
  // blocks (n % 16 == 0)
  const size_t units = MODE == 0 ? a.n / 8 : a.n / 16;
  const int ntail = MODE == 0 ? static_cast<int>(a.n - units * 8) : 0;
  const size_t per = (units + gridDim.x - 1) / gridDim.x;
  const size_t lo = static_cast<size_t>(blockIdx.x) * per;
  const size_t hi = lo + per < units ? lo + per : units;
  const bool tail_thread = blockIdx.x == 0 && static_cast<int>(threadIdx.x) < ntail;
  auto tail_elem = [&](int i) {
    return reinterpret_cast<const uint16_t*>(a.t[i].x)[units * 8 + threadIdx.x];
  };

  uint32_t m = fold_max(MODE == 0 ? chunk_absmax(a.t[0].x, lo, hi)
                                  : chunk_absmax(a.t[0].x, 2 * lo, 2 * hi));
  if (tail_thread) m = max(m, static_cast<uint32_t>(tail_elem(0)) & 0x7FFFu);
  unsigned bits = grid_stage(m, &ws->amax_bits[0], &ws->arrived, gridDim.x, a.limit_ns, a.err);

#pragma unroll
  for (int st = 1; st <= QKV; ++st) {
    const int ip = st - 1;                          // tensor quantized in this stage
    const QkvTensor& tp = a.t[ip];
    const bool ok = bits < 0x7F800000u;             // finite amax (and no timeout)
    const float amax = __uint_as_float(bits);
    if (blockIdx.x == 0 && threadIdx.x == 0 && bits != 0xFFFFFFFFu) {
      *tp.amax = amax;
      if (!ok) atomicExch(a.err, DEV_ERR_NONFINITE);
    }
    const uint4* xc = st < QKV ? a.t[st].x : nullptr;
    uint32_t m2;
    if (MODE == 0) {
      const float s = (amax == 0.0f) ? 1.0f : __fdiv_rn(amax, 448.0f);
      const float r = __frcp_rn(s);
      if (ok && blockIdx.x == 0 && threadIdx.x == 0) *tp.scale8 = s;
      const uint4* xp = ok ? tp.x : nullptr;
      uint2* op = reinterpret_cast<uint2*>(tp.codes8);
      m2 = markstein_ok(s) ? qkv_stage_fp8<true>(xp, op, s, r, xc, lo, hi)
                           : qkv_stage_fp8<false>(xp, op, s, r, xc, lo, hi);
      if (ok && tail_thread) {
        const float x = __uint_as_float(static_cast<uint32_t>(tail_elem(ip)) << 16);
        tp.codes8[units * 8 + threadIdx.x] =
            static_cast<uint8_t>(cvt_e4m3x2(__fdiv_rn(x, s), 0.0f) & 0xFFu);
      }
    } else {
      const float sg = (amax == 0.0f) ? 1.0f : __fdiv_rn(amax, 2688.0f);
      const float six_sg = __fmul_rn(6.0f, sg);
      const float s8 = (amax == 0.0f) ? 1.0f : __fdiv_rn(__fmul_rn(2688.0f, sg), 448.0f);
      if (ok && blockIdx.x == 0 && threadIdx.x == 0) {
        *tp.gscale = sg;
        *tp.scale8 = s8;
      }
      __shared__ Fp4Tables tab;
      if (ok) {                                     // uniform over the grid
        build_fp4_tables(&tab, sg, six_sg, s8);
        __syncthreads();
      }
      m2 = qkv_stage_fp4(ok ? tp.x : nullptr, tp.e2m1, tp.bscale,
                         reinterpret_cast<uint4*>(tp.codes8), six_sg, &tab, xc, lo, hi);
    }
    if (st < QKV) {
      m = fold_max(m2);
      if (tail_thread) m = max(m, static_cast<uint32_t>(tail_elem(st)) & 0x7FFFu);
      bits = grid_stage(m, &ws->amax_bits[st], &ws->arrived, (st + 1) * gridDim.x, a.limit_ns,
                        a.err);
    }
  }
  // depart: the last CTA zeroes the workspace for the next call
  if (threadIdx.x == 0) {
    unsigned old;
    asm volatile("atom.acq_rel.gpu.global.add.u32 %0, [%1], 1;" : "=r"(old) : "l"(&ws->departed)
                 : "memory");
    if (old == gridDim.x - 1) {
      for (int i = 0; i < 4; ++i) ws->amax_bits[i] = 0u;
      ws->arrived = 0u;
      ws->departed = 0u;
    }
  }
}

// -------------------------------------------------------------------------------------------
// Q, K and V with given (static) scales in one launch: blockIdx.y picks the tensor, whose amax is
// an input (a calibration done earlier, as post-training quantization provides); each tensor
// gets exactly the results of k_quant_fp8 (MODE 0) or k_quant_fp4_block with the FP8 requant
// (MODE 1).  One streaming pass: read 2 B, write 1 B (FP8) or 1.5625 B (FP4) per element.
// -------------------------------------------------------------------------------------------
constexpr int STATIC_THREADS = 256;
constexpr int STATIC_UNROLL = 4;           // 16-byte loads in flight per thread (FP8)
#ifndef QATTN_STATIC_FP4_UNROLL
#define QATTN_STATIC_FP4_UNROLL 2
#endif
constexpr int STATIC_FP4_UNROLL = QATTN_STATIC_FP4_UNROLL;   // 16-element blocks in flight (FP4)

template <int MODE>
__global__ void __launch_bounds__(STATIC_THREADS) k_quant_qkv(const __grid_constant__ QkvArgs a) {
  const int ti = blockIdx.y;
  const QkvTensor tp = ti == 0 ? a.t[0] : (ti == 1 ? a.t[1] : a.t[2]);
  const float amax = *tp.amax;
  if (!(amax <= 3.402823466e38f)) {              // inf or NaN: nothing is written
    if (blockIdx.x == 0 && threadIdx.x == 0) atomicExch(a.err, DEV_ERR_NONFINITE);
    return;
  }
  const size_t T = static_cast<size_t>(gridDim.x) * STATIC_THREADS;
  const size_t i0 = static_cast<size_t>(blockIdx.x) * STATIC_THREADS + threadIdx.x;
  if (MODE == 0) {
    const size_t nvec = a.n / 8;
    const int ntail = static_cast<int>(a.n - nvec * 8);
    const float s = (amax == 0.0f) ? 1.0f : __fdiv_rn(amax, 448.0f);
    if (blockIdx.x == 0 && threadIdx.x == 0) *tp.scale8 = s;
    const float r = __frcp_rn(s);
    const uint4* xv = tp.x;
    uint2* ov = reinterpret_cast<uint2*>(tp.codes8);
    constexpr size_t U = STATIC_UNROLL;
    auto sweep = [&](auto fast) {
      constexpr bool FAST = decltype(fast)::value;
      size_t i = i0;
      for (; i + (U - 1) * T < nvec; i += U * T) {
        uint4 x[U];
#pragma unroll
        for (size_t u = 0; u < U; ++u) x[u] = __ldcs(xv + i + u * T);
#pragma unroll
        for (size_t u = 0; u < U; ++u)
          __stcs(ov + i + u * T, make_uint2(quant4_e4m3<FAST>(x[u].x, x[u].y, s, r),
                                            quant4_e4m3<FAST>(x[u].z, x[u].w, s, r)));
      }
      for (; i < nvec; i += T) {
        const uint4 x = __ldcs(xv + i);
        __stcs(ov + i, make_uint2(quant4_e4m3<FAST>(x.x, x.y, s, r), quant4_e4m3<FAST>(x.z, x.w, s, r)));
      }
    };
    if (markstein_ok(s)) sweep(std::true_type{});
    else sweep(std::false_type{});
    if (blockIdx.x == 0 && static_cast<int>(threadIdx.x) < ntail) {
      const uint16_t xb = reinterpret_cast<const uint16_t*>(xv)[nvec * 8 + threadIdx.x];
      const float x = __uint_as_float(static_cast<uint32_t>(xb) << 16);
      tp.codes8[nvec * 8 + threadIdx.x] = static_cast<uint8_t>(cvt_e4m3x2(__fdiv_rn(x, s), 0.0f) & 0xFFu);
    }
  } else {
    const size_t nblocks = a.n / 16;
    const float sg = (amax == 0.0f) ? 1.0f : __fdiv_rn(amax, 2688.0f);
    const float six_sg = __fmul_rn(6.0f, sg);
    const float s8 = (amax == 0.0f) ? 1.0f : __fdiv_rn(__fmul_rn(2688.0f, sg), 448.0f);
    if (blockIdx.x == 0 && threadIdx.x == 0) {
      *tp.gscale = sg;
      *tp.scale8 = s8;
    }
    __shared__ Fp4Tables tab;
    build_fp4_tables(&tab, sg, six_sg, s8);
    __syncthreads();
    const uint4* xv = tp.x;
    uint4* c8 = reinterpret_cast<uint4*>(tp.codes8);
    size_t b = i0;
    constexpr size_t UB = STATIC_FP4_UNROLL;
    for (; b + (UB - 1) * T < nblocks; b += UB * T) {   // UB blocks' loads in flight
      uint4 x0[UB], x1[UB];
#pragma unroll
      for (size_t u = 0; u < UB; ++u) {
        x0[u] = __ldcs(xv + 2 * (b + u * T));
        x1[u] = __ldcs(xv + 2 * (b + u * T) + 1);
      }
#pragma unroll
      for (size_t u = 0; u < UB; ++u) fp4_block(x0[u], x1[u], b + u * T, six_sg, &tab, tp.e2m1, tp.bscale, c8);
    }
    for (; b < nblocks; b += T)
      fp4_block(__ldcs(xv + 2 * b), __ldcs(xv + 2 * b + 1), b, six_sg, &tab, tp.e2m1, tp.bscale, c8);
  }
}

// -------------------------------------------------------------------------------------------
// Host launchers (called from the C-ABI layer, which validates arguments).
// -------------------------------------------------------------------------------------------
static int grid_for(size_t work_items, int num_sms) {
  const size_t per_cta = 256;
  size_t need = (work_items + per_cta - 1) / per_cta;
  size_t cap = static_cast<size_t>(num_sms) * 8;  // 8 CTAs of 256 threads fill an SM
  if (need < 1) need = 1;
  return static_cast<int>(need < cap ? need : cap);
}

cudaError_t launch_amax(const void* x, size_t n, float* amax, int* err, int num_sms,
                        cudaStream_t stream) {
  cudaError_t e = cudaMemsetAsync(amax, 0, sizeof(float), stream);
  if (e != cudaSuccess) return e;
  const size_t nvec = n / 8;
  const int ntail = static_cast<int>(n - nvec * 8);
  const uint16_t* xs = static_cast<const uint16_t*>(x);
  k_amax_bf16<<<grid_for(nvec / 4 + 1, num_sms), 256, 0, stream>>>(
      static_cast<const uint4*>(x), nvec, xs + nvec * 8, ntail, reinterpret_cast<unsigned*>(amax),
      err);
  return cudaGetLastError();
}

cudaError_t launch_quant_fp8(const void* x, size_t n, const float* amax, uint8_t* out,
                             float* scale, int* err, int num_sms, cudaStream_t stream,
                             int inject_oob) {
  const size_t nvec = n / 8;
  const int ntail = static_cast<int>(n - nvec * 8);
  const uint16_t* xs = static_cast<const uint16_t*>(x);
#ifndef QATTN_CHECKED
  inject_oob = 0;                  // only the checked build can stop the extra vector
#endif
  k_quant_fp8<<<grid_for(nvec, num_sms), 256, 0, stream>>>(
      static_cast<const uint4*>(x), nvec, nvec + (inject_oob ? 1 : 0), xs + nvec * 8, ntail, amax,
      reinterpret_cast<uint2*>(out), out + nvec * 8, scale, err);
  return cudaGetLastError();
}

cudaError_t launch_quant_fp4_block(const void* x, size_t n, const float* amax, uint8_t* packed,
                                   uint8_t* bscale, float* gscale, uint8_t* codes8, float* scale8,
                                   int* err, int num_sms, cudaStream_t stream) {
  const size_t nblocks = n / 16;
  k_quant_fp4_block<<<grid_for(nblocks, num_sms), 256, 0, stream>>>(
      static_cast<const uint4*>(x), nblocks, amax, reinterpret_cast<uint2*>(packed), bscale,
      gscale, reinterpret_cast<uint4*>(codes8), scale8, err);
  return cudaGetLastError();
}

// Co-resident CTAs per SM of a cooperative kernel with FUSED_THREADS threads (0 on error).
template <class K>
static int blocks_per_sm_of(K fn) {
  int n = 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, reinterpret_cast<const void*>(fn), FUSED_THREADS,
                                                    0) != cudaSuccess) {
    cudaGetLastError();
    return 0;
  }
  return n;
}

cudaError_t launch_calib_quant_fp8(const void* x, size_t n, float* amax, uint8_t* out,
                                   float* scale, void* workspace, uint64_t limit_ns, int* err,
                                   int num_sms, cudaStream_t stream) {
  static DeviceOnce occ;
  const int blocks_per_sm = occ.get([] { return blocks_per_sm_of(k_calib_quant_fp8); });
  if (blocks_per_sm < 1) return cudaErrorInvalidValue;
  const size_t nvec = n / 8;
  const int ntail = static_cast<int>(n - nvec * 8);
  size_t want = (nvec + FUSED_THREADS * 4 - 1) / (FUSED_THREADS * 4);   // >= 4 vectors/thread
  size_t cap = static_cast<size_t>(num_sms) * blocks_per_sm;
  unsigned grid = static_cast<unsigned>(want < 1 ? 1 : (want < cap ? want : cap));
  const uint4* xv = static_cast<const uint4*>(x);
  const uint16_t* xtail = static_cast<const uint16_t*>(x) + nvec * 8;
  uint2* outv = reinterpret_cast<uint2*>(out);
  uint8_t* outtail = out + nvec * 8;
  FusedWorkspace* ws = static_cast<FusedWorkspace*>(workspace);
  void* args[] = {(void*)&xv, (void*)&nvec, (void*)&xtail, (void*)&ntail, (void*)&amax,
                  (void*)&outv, (void*)&outtail, (void*)&scale, (void*)&ws, (void*)&limit_ns,
                  (void*)&err};
  return cudaLaunchCooperativeKernel((const void*)k_calib_quant_fp8, dim3(grid),
                                     dim3(FUSED_THREADS), args, 0, stream);
}

// tensors: x, codes8, amax, scale8, e2m1, bscale, gscale for each of Q, K, V (FP8 mode: the last
// three null).
cudaError_t launch_calib_quant_qkv(const void* const* x, uint8_t* const* codes8, float* const* amax,
                                   float* const* scale8, uint8_t* const* e2m1,
                                   uint8_t* const* bscale, float* const* gscale, size_t n, int mode,
                                   void* workspace, uint64_t limit_ns, int* err, int num_sms,
                                   cudaStream_t stream) {
  static DeviceOnce occ[2];
  const void* fn = mode == 0 ? (const void*)k_calib_quant_qkv<0> : (const void*)k_calib_quant_qkv<1>;
  const int bps_mode = occ[mode].get([fn] { return blocks_per_sm_of(fn); });
  if (bps_mode < 1) return cudaErrorInvalidValue;
  QkvArgs a;
  for (int i = 0; i < QKV; ++i) {
    a.t[i].x = static_cast<const uint4*>(x[i]);
    a.t[i].codes8 = codes8[i];
    a.t[i].amax = amax[i];
    a.t[i].scale8 = scale8[i];
    a.t[i].e2m1 = reinterpret_cast<uint2*>(e2m1[i]);
    a.t[i].bscale = bscale[i];
    a.t[i].gscale = gscale[i];
  }
  a.n = n;
  a.limit_ns = limit_ns;
  a.err = err;
  a.ws = static_cast<QkvWorkspace*>(workspace);
  const size_t units = mode == 0 ? n / 8 : n / 16;
  const size_t want = (units + FUSED_THREADS * 4 - 1) / (FUSED_THREADS * 4);
  const size_t cap = static_cast<size_t>(num_sms) * bps_mode;
  const unsigned grid = static_cast<unsigned>(want < 1 ? 1 : (want < cap ? want : cap));
  void* args[] = {(void*)&a};
  return cudaLaunchCooperativeKernel(fn, dim3(grid), dim3(FUSED_THREADS), args, 0, stream);
}

// Q, K, V with given amax values (io amax pointers are inputs); tensors: as launch_calib_quant_qkv.
cudaError_t launch_quant_qkv(const void* const* x, uint8_t* const* codes8, float* const* amax,
                             float* const* scale8, uint8_t* const* e2m1, uint8_t* const* bscale,
                             float* const* gscale, size_t n, int mode, int* err, int num_sms,
                             cudaStream_t stream) {
  QkvArgs a;
  for (int i = 0; i < QKV; ++i) {
    a.t[i].x = static_cast<const uint4*>(x[i]);
    a.t[i].codes8 = codes8[i];
    a.t[i].amax = amax[i];
    a.t[i].scale8 = scale8[i];
    a.t[i].e2m1 = reinterpret_cast<uint2*>(e2m1[i]);
    a.t[i].bscale = bscale[i];
    a.t[i].gscale = gscale[i];
  }
  a.n = n;
  a.limit_ns = 0;
  a.err = err;
  a.ws = nullptr;
  // per tensor: enough CTAs for four 16-byte vectors (FP8) or two blocks (FP4) per thread, at
  // most 4 CTAs of 256 threads per SM (3 tensors: 12 per SM)
  const size_t per_cta = mode == 0 ? static_cast<size_t>(STATIC_THREADS) * STATIC_UNROLL * 8
                                   : static_cast<size_t>(STATIC_THREADS) * STATIC_FP4_UNROLL * 16;
  size_t want = (n + per_cta - 1) / per_cta;
  const size_t cap = static_cast<size_t>(num_sms) * 4;
  if (want < 1) want = 1;
  const dim3 grid(static_cast<unsigned>(want < cap ? want : cap), QKV, 1);
  if (mode == 0)
    k_quant_qkv<0><<<grid, STATIC_THREADS, 0, stream>>>(a);
  else
    k_quant_qkv<1><<<grid, STATIC_THREADS, 0, stream>>>(a);
  return cudaGetLastError();
}

cudaError_t launch_calib_quant_fp4_block(const void* x, size_t n, float* amax, uint8_t* packed,
                                         uint8_t* bscale, float* gscale, uint8_t* codes8,
                                         float* scale8, void* workspace, uint64_t limit_ns,
                                         int* err, int num_sms, cudaStream_t stream) {
  static DeviceOnce occ;
  const int blocks_per_sm = occ.get([] { return blocks_per_sm_of(k_calib_quant_fp4_block); });
  if (blocks_per_sm < 1) return cudaErrorInvalidValue;
  const size_t nblocks = n / 16;
  size_t want = (nblocks + FUSED_THREADS * 2 - 1) / (FUSED_THREADS * 2);
  size_t cap = static_cast<size_t>(num_sms) * blocks_per_sm;
  unsigned grid = static_cast<unsigned>(want < 1 ? 1 : (want < cap ? want : cap));
  const uint4* xv = static_cast<const uint4*>(x);
  uint2* pk = reinterpret_cast<uint2*>(packed);
  uint4* c8 = reinterpret_cast<uint4*>(codes8);
  FusedWorkspace* ws = static_cast<FusedWorkspace*>(workspace);
  void* args[] = {(void*)&xv, (void*)&nblocks, (void*)&amax, (void*)&pk, (void*)&bscale,
                  (void*)&gscale, (void*)&c8, (void*)&scale8, (void*)&ws, (void*)&limit_ns,
                  (void*)&err};
  return cudaLaunchCooperativeKernel((const void*)k_calib_quant_fp4_block, dim3(grid),
                                     dim3(FUSED_THREADS), args, 0, stream);
}

}  // namespace qattn
