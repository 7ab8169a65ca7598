// attn_fwd.cu -- fused quantized attention forward for sm_100a (TMA + tcgen05 + TMEM).
//
// Method: NVIDIA developer blog "Optimizing FLUX.1 Kontext for Image Editing with Low-Precision
// Quantization", section "Workflow and quantization" and Fig. 4:
//   BMM1  S = Q8 K8^T in FP8 with higher-precision (FP32) accumulation   (second SDPA bullet)
//   softmax in FP32, no quantization at that stage                       (third bullet)
//   P requantized to per-tensor FP8, BMM2 O = P8 V8 in FP8                (fourth bullet, Fig. 4)
// over the full (non-causal) joint text + target + context token sequence.
//
// Readings taken where the blog is silent:
//   * P is quantized before normalization with the fixed per-tensor scale 1/448: the stored
//     value is e4m3(p * 448) with p = 2^(S' - M) in (0, 1]; the FP32 row sum l divides O after
//     BMM2.  (A single-pass kernel never holds the normalized P.)
//   * M is the running row max of the base-2 scores S' = S * s_q * s_k * sm_scale * log2(e),
//     rounded UP to an integer.  A rise of M rescales O and l by an exact power of two, and
//     E4M3 rounding commutes with power-of-two scaling in the normal range, so the result does
//     not depend on how keys are tiled.
//
// Kernel structure: one CTA (one per SM) per pair of 128-row Q tiles of one (sequence, head);
// keys advance in steps of BN = 64.
//   warp 1      TMA producer: both Q tiles once, then K and V tiles through separate rings.
//   warp 0      MMA issuer (one elected lane) and TMEM owner.  Each Q tile has two S buffers:
//               once P_t(j) is in TMEM (written over S_t(j)) it issues O_t += P_t(j) V_j (A
//               operand read from TMEM) and right behind it, in the same in-order tcgen05
//               stream, S_t(j+2) = Q_t K_{j+2}^T into that buffer, so the scores of the next
//               step are always computed while the softmax works on the current one.
//   warps 2-17  softmax, eight per Q tile: two threads per query row (TMEM lane), each with
//               half of the row's BN scores (16x32bx2 TMEM shapes), so every SM sub-partition
//               interleaves four softmax warps.  Each takes the row max (3-input maxima and
//               one shuffle) and computes p*448 = 2^(S' - M + log2 448) in FP32 (hardware ex2
//               for most pairs, a degree-5 polynomial on the FMA pipe for the rest), sums p in
//               packed f32x2 adds and converts to E4M3.  Once the previous P V has completed
//               it rescales its half of the O row on a rise of M, then writes its half of
//               P_t(j) with tcgen05.st.
//   K/V tiles are read by TMA once per CTA for both Q tiles.
// TMEM per Q tile: two S buffers (BN FP32 columns each; P of a step, 4 E4M3 per column, is
// written over its first BN/4 columns) and O (D columns).
// All waits are bounded (a global-timer limit); on expiry the CTA records a timeout in the
// library's error word, drains what it issued and exits.
#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <cstdint>

#include "sm100_ptx.cuh"

namespace qattn {

constexpr int BLOCK_M = 128;                 // query rows per tile (= TMEM lanes)
constexpr int NQ = 2;                        // query tiles per CTA
constexpr int KSTAGES = 6;
constexpr int VSTAGES = 6;
constexpr int NUM_SOFTMAX_WARPS = 8 * NQ;       // two warps per 32-lane quarter of each tile
// The MMA issuer and the TMA producer are the lowest-numbered warps: the warp schedulers favour
// older warps, and these two must not starve behind the four softmax warps of their sub-partition.
constexpr int WARP_MMA = 0;
constexpr int WARP_LOAD = 1;
constexpr int FIRST_SOFTMAX_WARP = 2;
constexpr int ATTN_THREADS = (NUM_SOFTMAX_WARPS + 2) * 32;
constexpr float LOG2E_F = 1.4426950408889634f;
constexpr float LOG2_448 = 8.807354922057604f;   // log2(448): p * 448 = 2^(S' - M + log2 448)

// Keys per step.  Per Q tile TMEM holds two S buffers (the scores of step j+1 are computed
// while the softmax works on step j; P of a step is written over its own S buffer) and O:
// 2 * 64 + 128 = 256 columns for D = 128, so both tiles fill the 512 columns.
template <int D>
struct KvStep {
  static constexpr int N = 64;
};

struct AttnArgs {
  int rows_per_slab;        // rows of one (b, h) slab in the tensor maps: L (dense) or T (varlen)
  int H;
  int L;                    // dense sequence length (unused for varlen)
  const int* cu_seqlens;    // varlen: device [nseq + 1]; nullptr for dense
  const float* s_q;
  const float* s_k;
  const float* s_v;
  float sm_scale;
  __nv_bfloat16* out;
  int* err;
  uint64_t timeout_ns;
  int inject_missing_q;     // fault injection for tests: the producer never loads Q
};

template <int D>
struct Smem {
  static constexpr int BN = KvStep<D>::N;
  static constexpr int TILE_Q = BLOCK_M * D;       // bytes (E4M3)
  static constexpr int TILE_KV = BN * D;
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_K = OFF_Q + NQ * TILE_Q;
  static constexpr int OFF_V = OFF_K + KSTAGES * TILE_KV;
  static constexpr int OFF_BAR = OFF_V + VSTAGES * TILE_KV;
  // barriers: q_full, k_full[KS], k_empty[KS], v_full[VS], v_empty[VS], s_full[NQ][2],
  // p_full[NQ][2], o_done[NQ][2], drain
  static constexpr int NBARS = 1 + 2 * KSTAGES + 2 * VSTAGES + 6 * NQ + 1;
  static constexpr int OFF_TMEM = OFF_BAR + 8 * NBARS;
  static constexpr int OFF_ABORT = OFF_TMEM + 4;
  static constexpr int BYTES = OFF_ABORT + 4;
  static constexpr int ALLOC = BYTES + 1024;       // slack for 1024-byte alignment
  static_assert(TILE_Q % 1024 == 0 && TILE_KV % 1024 == 0, "1024-byte aligned tiles");
};

template <int D>
struct TmemCols {
  static constexpr int BN = KvStep<D>::N;
  static constexpr uint32_t PER_TILE = 256;              // tile t uses [t * 256, t * 256 + 256)
  static constexpr uint32_t S = 0;                       // buffer b: [b * BN, b * BN + BN);
                                                         // P of that step: its first BN / 4
  static constexpr uint32_t O = 256 - D;                 // D columns, ending at the tile's end
  static constexpr uint32_t ALLOC = 512;
  static_assert(2 * BN <= O, "S buffers and O of one tile overlap");
};

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

// Packed f32x2 helpers.  Pairs live in 64-bit registers; constant pairs are built once per
// step (pair_of) so the inner loop issues only the arithmetic.
__device__ __forceinline__ uint64_t pair_of(float lo, float hi) {
  uint64_t r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
  return r;
}
__device__ __forceinline__ void unpair(uint64_t p, float& lo, float& hi) {
  asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(p));
}
__device__ __forceinline__ uint64_t ffma2(uint64_t a, uint64_t b, uint64_t c) {
  uint64_t d;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
  return d;
}
__device__ __forceinline__ uint64_t fadd2(uint64_t a, uint64_t b) {
  uint64_t d;
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}

// Four E4M3 codes in one word from four floats (first float in the low byte).
__device__ __forceinline__ uint32_t pack4_e4m3(float a, float b, float c, float d) {
  uint32_t r;
  asm("{\n\t.reg .b16 lo, hi;\n\t"
      "cvt.rn.satfinite.e4m3x2.f32 lo, %2, %1;\n\t"
      "cvt.rn.satfinite.e4m3x2.f32 hi, %4, %3;\n\t"
      "mov.b32 %0, {lo, hi};\n\t}"
      : "=r"(r)
      : "f"(a), "f"(b), "f"(c), "f"(d));
  return r;
}

// 2^x on the FMA pipe for two values at once, for x <= 9.  x is clamped at -125 (2^-125 is
// far below the smallest E4M3 code of p * 448), split as x = n + f with n = round(x) (by
// adding and subtracting 1.5 * 2^23) and f in [-1/2, 1/2]; 2^f comes from a degree-5 minimax
// polynomial (relative error 2.1e-7 in binary32, fitted by csrc/fit_exp2_poly.py) and 2^n is
// added into the exponent field.
#ifndef QATTN_POLY_PAIRS_PER_8
#define QATTN_POLY_PAIRS_PER_8 1       // of every 8 pairs of scores, this many take the polynomial
#endif
struct PolyConsts {
  uint64_t magic, neg_magic, neg_one, c5, c4, c3, c2, c1, c0;
  __device__ __forceinline__ PolyConsts()
      : magic(pair_of(12582912.0f, 12582912.0f)),      // 1.5 * 2^23
        neg_magic(pair_of(-12582912.0f, -12582912.0f)),
        neg_one(pair_of(-1.0f, -1.0f)),
        c5(pair_of(0x1.5c08e6p-10f, 0x1.5c08e6p-10f)),   // coefficients of the fit
        c4(pair_of(0x1.3d0c52p-7f, 0x1.3d0c52p-7f)),
        c3(pair_of(0x1.c6b6e4p-5f, 0x1.c6b6e4p-5f)),
        c2(pair_of(0x1.ebf918p-3f, 0x1.ebf918p-3f)),
        c1(pair_of(0x1.62e428p-1f, 0x1.62e428p-1f)),
        c0(pair_of(0x1.000002p+0f, 0x1.000002p+0f)) {}
};

__device__ __forceinline__ uint64_t poly_exp2_x2(uint64_t x, const PolyConsts& k) {
  float x0, x1;
  unpair(x, x0, x1);
  x = pair_of(fmaxf(x0, -125.0f), fmaxf(x1, -125.0f));
  const uint64_t t = fadd2(x, k.magic);                 // n + 1.5 * 2^23, n = round(x)
  const uint64_t n = fadd2(t, k.neg_magic);             // n (exact)
  const uint64_t f = ffma2(n, k.neg_one, x);            // x - n (exact)
  uint64_t p = ffma2(k.c5, f, k.c4);
  p = ffma2(p, f, k.c3);
  p = ffma2(p, f, k.c2);
  p = ffma2(p, f, k.c1);
  p = ffma2(p, f, k.c0);
  // the low 9 bits of each half of t hold n (two's complement): shifted into the exponent
  // field they add n
  float p0, p1, t0, t1;
  unpair(p, p0, p1);
  unpair(t, t0, t1);
  return pair_of(__int_as_float(__float_as_int(p0) + (__float_as_int(t0) << 23)),
                 __int_as_float(__float_as_int(p1) + (__float_as_int(t1) << 23)));
}

// Row max of N scores (N a multiple of 16): 8 independent chains of 3-input maxima, then a
// short tree.
template <int N>
__device__ __forceinline__ float rowmax(const float (&s)[N]) {
  float m[8];
#pragma unroll
  for (int k = 0; k < 8; ++k) m[k] = fmaxf(s[k], s[k + 8]);
#pragma unroll
  for (int i = 16; i + 16 <= N; i += 16) {
#pragma unroll
    for (int k = 0; k < 8; ++k) m[k] = max3f(m[k], s[i + k], s[i + 8 + k]);
  }
  return max3f(max3f(m[0], m[1], m[2]), max3f(m[3], m[4], m[5]), fmaxf(m[6], m[7]));
}

template <int D>
__global__ void __launch_bounds__(ATTN_THREADS, 1)
    k_attn_fp8_fwd(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                   const __grid_constant__ CUtensorMap tm_v, const AttnArgs args) {
  using SL = Smem<D>;
  using TC = TmemCols<D>;
  constexpr int BN = KvStep<D>::N;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_u32 = smem_u32(smem_raw);
  const uint32_t base_u32 = (raw_u32 + 1023u) & ~1023u;
  uint8_t* base = smem_raw + (base_u32 - raw_u32);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  // ---- which sequence and which rows -------------------------------------------------------
  const int qblk = blockIdx.x;                    // pair of Q tiles
  const int h = blockIdx.y;
  const int bz = blockIdx.z;                      // batch row (dense) or sequence (varlen)
  int seq_start, seq_len, slab;
  if (args.cu_seqlens) {
    seq_start = __ldg(args.cu_seqlens + bz);
    seq_len = __ldg(args.cu_seqlens + bz + 1) - seq_start;
    slab = h;
  } else {
    seq_start = 0;
    seq_len = args.L;
    slab = bz * args.H + h;
  }
  const int q_row0 = qblk * (NQ * BLOCK_M);
  if (q_row0 >= seq_len) return;                  // uniform over the CTA: nothing to do
  const int nkv = (seq_len + BN - 1) / BN;

  // ---- barriers --------------------------------------------------------------------------
  const uint32_t bar0 = base_u32 + SL::OFF_BAR;
  auto BAR = [&](int i) { return bar0 + 8u * static_cast<uint32_t>(i); };
  constexpr int B_QFULL = 0;
  constexpr int B_KFULL = 1, B_KEMPTY = B_KFULL + KSTAGES;
  constexpr int B_VFULL = B_KEMPTY + KSTAGES, B_VEMPTY = B_VFULL + VSTAGES;
  constexpr int B_SFULL = B_VEMPTY + VSTAGES;     // B_SFULL + 2 * t + buffer
  // Every per-step barrier exists once per S buffer (step j uses buffer j % 2 and phase j / 2):
  // the softmax may run up to one step ahead of the MMA issuer and waits on o_done only when
  // it rescales O (and before the epilogue), so one barrier per buffer keeps each waiter within
  // one phase of its barrier.
  constexpr int B_PFULL = B_SFULL + 2 * NQ;       // B_PFULL + 2 * t + buf
  constexpr int B_ODONE = B_PFULL + 2 * NQ;       // B_ODONE + 2 * t + buf
  constexpr int B_DRAIN = B_ODONE + 2 * NQ;
  constexpr int TILE_WARPS = NUM_SOFTMAX_WARPS / NQ;   // one arrive per softmax warp
  volatile int* abort_flag = reinterpret_cast<volatile int*>(base + SL::OFF_ABORT);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(base + SL::OFF_TMEM);

  if (threadIdx.x == 0) {
    mbar_init(BAR(B_QFULL), 1);
    for (int i = 0; i < KSTAGES; ++i) { mbar_init(BAR(B_KFULL + i), 1); mbar_init(BAR(B_KEMPTY + i), 1); }
    for (int i = 0; i < VSTAGES; ++i) { mbar_init(BAR(B_VFULL + i), 1); mbar_init(BAR(B_VEMPTY + i), 1); }
    for (int t = 0; t < NQ; ++t) {
      mbar_init(BAR(B_SFULL + 2 * t), 1);
      mbar_init(BAR(B_SFULL + 2 * t + 1), 1);
      mbar_init(BAR(B_PFULL + 2 * t), TILE_WARPS);
      mbar_init(BAR(B_PFULL + 2 * t + 1), TILE_WARPS);
      mbar_init(BAR(B_ODONE + 2 * t), 1);
      mbar_init(BAR(B_ODONE + 2 * t + 1), 1);
    }
    mbar_init(BAR(B_DRAIN), 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == WARP_MMA) {                         // whole warp: TMEM allocation
    tmem_alloc(base_u32 + SL::OFF_TMEM, TC::ALLOC);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint64_t tlim = args.timeout_ns;

  if (warp == WARP_LOAD) {
    // ======================= TMA producer (warp-wide loop, one elected lane issues) ============
    const uint32_t leader = elect_one();
    if (!args.inject_missing_q) {
      if (leader) {
        tma_prefetch_desc(&tm_q);
        tma_prefetch_desc(&tm_k);
        tma_prefetch_desc(&tm_v);
      }
      int nk = 0, nv = 0;                          // loads issued
      mbar_arrive_expect_tx_if(leader, BAR(B_QFULL), NQ * SL::TILE_Q);
      for (int t = 0; t < NQ; ++t)
        tma_load_3d_if(leader, base_u32 + SL::OFF_Q + t * SL::TILE_Q, &tm_q, BAR(B_QFULL), 0,
                       seq_start + q_row0 + t * BLOCK_M, slab);
      auto load_k = [&](int j) -> bool {
        const int s = j % KSTAGES;
        if (j >= KSTAGES &&
            !mbar_wait(BAR(B_KEMPTY + s), ((j / KSTAGES) - 1) & 1, tlim, abort_flag, args.err))
          return false;
        mbar_arrive_expect_tx_if(leader, BAR(B_KFULL + s), SL::TILE_KV);
        tma_load_3d_if(leader, base_u32 + SL::OFF_K + s * SL::TILE_KV, &tm_k, BAR(B_KFULL + s), 0,
                       seq_start + j * BN, slab);
        ++nk;
        return true;
      };
      auto load_v = [&](int j) -> bool {
        const int s = j % VSTAGES;
        if (j >= VSTAGES &&
            !mbar_wait(BAR(B_VEMPTY + s), ((j / VSTAGES) - 1) & 1, tlim, abort_flag, args.err))
          return false;
        mbar_arrive_expect_tx_if(leader, BAR(B_VFULL + s), SL::TILE_KV);
        tma_load_3d_if(leader, base_u32 + SL::OFF_V + s * SL::TILE_KV, &tm_v, BAR(B_VFULL + s), 0,
                       seq_start + j * BN, slab);
        ++nv;
        return true;
      };
      // order of use on the tensor pipe: K0, K1, V0, K2, V1, K3, ...: K runs two steps ahead
      bool ok = load_k(0);
      if (ok && nkv > 1) ok = load_k(1);
      for (int j = 0; ok && j < nkv; ++j) {
        ok = load_v(j);
        if (ok && j + 2 < nkv) ok = load_k(j + 2);
        ok = __all_sync(0xFFFFFFFFu, ok);
      }
      // drain: every issued load has landed before the CTA may exit (instant when healthy)
      mbar_drain(BAR(B_QFULL), 0, tlim);
      for (int j = nk - 1; j >= 0 && j >= nk - KSTAGES; --j)
        mbar_drain(BAR(B_KFULL + j % KSTAGES), (j / KSTAGES) & 1, tlim);
      for (int j = nv - 1; j >= 0 && j >= nv - VSTAGES; --j)
        mbar_drain(BAR(B_VFULL + j % VSTAGES), (j / VSTAGES) & 1, tlim);
    }
  } else if (warp == WARP_MMA) {
    // ======================= MMA issuer (warp-wide loop, one elected lane issues) =============
    const uint32_t leader = elect_one();
    constexpr uint32_t IDESC_S = idesc_e4m3_f32(BLOCK_M, BN, false);
    constexpr uint32_t IDESC_O = idesc_e4m3_f32(BLOCK_M, D, true);
    // Q, K: K-major rows of D bytes, swizzled in 8-row atoms (SBO = 8 rows); 32-byte K steps.
    constexpr uint32_t QK_LAYOUT = (D == 128) ? 2u : 4u;   // 128B / 64B swizzle
    constexpr uint32_t QK_SBO = 8 * D;
    // V: MN-major (D contiguous per key row), rows of D bytes, SBO = 8 key rows; a K step of
    // 32 keys advances 32 rows.
    constexpr uint32_t V_LAYOUT = QK_LAYOUT;
    constexpr uint32_t V_SBO = 8 * D;
    // Descriptors are built once; a step only adds (address >> 4) offsets to the low bits.
    const uint64_t desc_q0 = smem_desc(base_u32 + SL::OFF_Q, 16, QK_SBO, QK_LAYOUT);
    const uint64_t desc_k0 = smem_desc(base_u32 + SL::OFF_K, 16, QK_SBO, QK_LAYOUT);
    const uint64_t desc_v0 = smem_desc(base_u32 + SL::OFF_V, SL::TILE_KV, V_SBO, V_LAYOUT);
    auto bmm1 = [&](int t, int ks, int buf) {       // S_t(buffer) = Q_t K^T
      const uint64_t da = desc_q0 + static_cast<uint64_t>((t * SL::TILE_Q) >> 4);
      const uint64_t db = desc_k0 + static_cast<uint64_t>((ks * SL::TILE_KV) >> 4);
      const uint32_t d_tmem = tmem + t * TC::PER_TILE + TC::S + buf * BN;
#pragma unroll
      for (int kk = 0; kk < D / 32; ++kk)
        mma_f8_ss_if(leader, d_tmem, da + kk * 2, db + kk * 2, IDESC_S, kk > 0 ? 1u : 0u);
    };
    auto bmm2 = [&](int t, int vs, int buf, bool first) {   // O_t += P_t(buffer) V
      const uint64_t db = desc_v0 + static_cast<uint64_t>((vs * SL::TILE_KV) >> 4);
      const uint32_t d_tmem = tmem + t * TC::PER_TILE + TC::O;
      const uint32_t a_tmem = tmem + t * TC::PER_TILE + TC::S + buf * BN;
#pragma unroll
      for (int kk = 0; kk < BN / 32; ++kk)
        mma_f8_ts_if(leader, d_tmem, a_tmem + kk * 8, db + static_cast<uint64_t>((kk * 32 * D) >> 4),
                     IDESC_O, (!first || kk > 0) ? 1u : 0u);
    };
    // S of steps 0 and 1 into the two buffers of each tile.
    bool ok = mbar_wait(BAR(B_QFULL), 0, tlim, abort_flag, args.err);
    for (int jj = 0; jj < 2 && jj < nkv; ++jj) {
      ok = ok && mbar_wait(BAR(B_KFULL + jj), 0, tlim, abort_flag, args.err);
      ok = __all_sync(0xFFFFFFFFu, ok);
      if (!ok) break;
      tc_fence_after();
      for (int t = 0; t < NQ; ++t) {
        bmm1(t, jj, jj);
        mma_commit_if(leader, BAR(B_SFULL + 2 * t + jj));
      }
      mma_commit_if(leader, BAR(B_KEMPTY + jj));
    }
    // Step j: O_t += P_t(j) V_j, then S_t(j+2) into the buffer P_t(j) occupied (the in-order
    // tcgen05 stream reads P before it is overwritten).
    for (int j = 0; ok && j < nkv; ++j) {
      const int vs = j % VSTAGES;
      const int buf = j & 1;
      const bool more = j + 2 < nkv;
      const int ks = (j + 2) % KSTAGES;
      ok = mbar_wait(BAR(B_VFULL + vs), (j / VSTAGES) & 1, tlim, abort_flag, args.err);
      if (ok && more)
        ok = mbar_wait(BAR(B_KFULL + ks), ((j + 2) / KSTAGES) & 1, tlim, abort_flag, args.err);
      for (int t = 0; ok && t < NQ; ++t) {
        ok = mbar_wait(BAR(B_PFULL + 2 * t + buf), (j >> 1) & 1, tlim, abort_flag, args.err);
        if (!__all_sync(0xFFFFFFFFu, ok)) { ok = false; break; }
        tc_fence_after();
        bmm2(t, vs, buf, j == 0);
        mma_commit_if(leader, BAR(B_ODONE + 2 * t + buf));
        if (more) {
          bmm1(t, ks, buf);
          mma_commit_if(leader, BAR(B_SFULL + 2 * t + buf));
        }
      }
      ok = __all_sync(0xFFFFFFFFu, ok);
      if (ok) {
        mma_commit_if(leader, BAR(B_VEMPTY + vs));
        if (more) mma_commit_if(leader, BAR(B_KEMPTY + ks));
      }
    }
    // drain: all issued MMAs complete before TMEM is released
    mma_commit_if(leader, BAR(B_DRAIN));
    mbar_drain(BAR(B_DRAIN), 0, tlim);
  } else {
    // ======================= softmax warps =======================
    // Softmax warp w (index i = w - 2) handles tile t = (i / 4) % 2, TMEM lane quarter w % 4
    // (the quarter its SM sub-partition may access) and, within it, 16 lanes (i / 8 selects
    // which); with the
    // 16x32bx2 TMEM shapes, lanes 0-15 of the warp take the first half of every row's columns
    // and lanes 16-31 the second half, so a row's max and sum combine with one shuffle and
    // each sub-partition runs four softmax warps.
    constexpr int HN = BN / 2;                     // scores per thread and step
    constexpr int HD = D / 2;                      // O columns per thread
    const int si = warp - FIRST_SOFTMAX_WARP;      // 0..15; quarter, tile and half are unique
    const int quarter = warp & 3;
    const int t = (si >> 2) & 1;
    const int hs = si >> 3;
    const int ch = lane >> 4;                      // column half
    const int r = quarter * 32 + hs * 16 + (lane & 15);   // row within the Q tile
    const uint32_t trow = tmem + (static_cast<uint32_t>(quarter * 32 + hs * 16) << 16) +
                          t * TC::PER_TILE;
    const uint32_t tO = trow + TC::O;
    const float c = __ldg(args.s_q) * __ldg(args.s_k) * args.sm_scale * LOG2E_F;
    const PolyConsts pk_consts;
    float m_run = -INFINITY;                       // integer-valued running max (base 2)
    float l = 0.0f;                                // this thread's share of the sum of p * 448
    bool ok = true;
    auto load_o = [&](uint32_t (&v)[HD]) {
#pragma unroll
      for (int c4 = 0; c4 < HD / 32; ++c4) tmem_ld16x2_x32<HD>(tO + c4 * 32, v + c4 * 32);
      tmem_wait_ld();
    };
    for (int j = 0; j < nkv; ++j) {
      const uint32_t tS = trow + TC::S + (j & 1) * BN;   // S_t(j); later P_t(j)
      ok = mbar_wait(BAR(B_SFULL + 2 * t + (j & 1)), (j >> 1) & 1, tlim, abort_flag, args.err);
      if (!__all_sync(0xFFFFFFFFu, ok)) { ok = false; break; }
      tc_fence_after();
      float s[HN];
      {
        uint32_t sv[HN];
        if constexpr (HN % 32 == 0) {
#pragma unroll
          for (int c4 = 0; c4 < HN / 32; ++c4) tmem_ld16x2_x32<HN>(tS + c4 * 32, sv + c4 * 32);
        } else {
#pragma unroll
          for (int c4 = 0; c4 < HN / 16; ++c4) tmem_ld16x2_x16<HN>(tS + c4 * 16, sv + c4 * 16);
        }
        tmem_wait_ld();
#pragma unroll
        for (int i = 0; i < HN; ++i) s[i] = __uint_as_float(sv[i]);
      }
      const int kv_valid = seq_len - j * BN - ch * HN;   // this thread's keys inside the sequence
      if (kv_valid < HN) {
#pragma unroll
        for (int i = 0; i < HN; ++i)
          if (i >= kv_valid) s[i] = -INFINITY;
      }
      float mx = rowmax<HN>(s);
      mx = fmaxf(mx, __shfl_xor_sync(0xFFFFFFFFu, mx, 16));
      const float m_new = fmaxf(m_run, ceilf(mx * c));
      const float neg_off = LOG2_448 - m_new;
      const uint64_t c2 = pair_of(c, c), off2 = pair_of(neg_off, neg_off);
      uint64_t acc[4] = {0, 0, 0, 0};             // four pairs of partial sums (0.0f bits)
      uint32_t pk[HN / 4];
#pragma unroll
      for (int i = 0; i < HN; i += 16) {
        float p[16];
#pragma unroll
        for (int q = 0; q < 8; ++q) {
          const uint64_t x = ffma2(pair_of(s[i + 2 * q], s[i + 2 * q + 1]), c2, off2);
          uint64_t pp;
          if (q < QATTN_POLY_PAIRS_PER_8) {
            pp = poly_exp2_x2(x, pk_consts);
          } else {
            float x0, x1;
            unpair(x, x0, x1);
            pp = pair_of(fast_exp2(x0), fast_exp2(x1));
          }
          acc[q & 3] = fadd2(acc[q & 3], pp);
          unpair(pp, p[2 * q], p[2 * q + 1]);
        }
#pragma unroll
        for (int q = 0; q < 4; ++q)
          pk[i / 4 + q] = pack4_e4m3(p[4 * q], p[4 * q + 1], p[4 * q + 2], p[4 * q + 3]);
      }
      float r0, r1, r2, r3, r4, r5, r6, r7;
      unpair(acc[0], r0, r1);
      unpair(acc[1], r2, r3);
      unpair(acc[2], r4, r5);
      unpair(acc[3], r6, r7);
      const float rowsum = ((r0 + r1) + (r2 + r3)) + ((r4 + r5) + (r6 + r7));
      // A rise of the running max rescales this row of O by 2^-(rise); O must be quiescent, so
      // that (rare) case first waits for the previous P V.  P_t(j) itself goes to the buffer
      // that P V of step j-1 does not read, so the common case does not wait at all.
      const bool rise = j > 0 && m_new > m_run;   // same value in both threads of a row
      if (__any_sync(0xFFFFFFFFu, rise)) {
        ok = mbar_wait(BAR(B_ODONE + 2 * t + ((j - 1) & 1)), ((j - 1) >> 1) & 1, tlim, abort_flag,
                       args.err);
        if (!__all_sync(0xFFFFFFFFu, ok)) { ok = false; break; }
        tc_fence_after();
        const float f = rise ? exp2_int(static_cast<int>(m_run - m_new)) : 1.0f;
        uint32_t v[HD];
        load_o(v);
#pragma unroll
        for (int i = 0; i < HD; ++i) v[i] = __float_as_uint(__uint_as_float(v[i]) * f);
#pragma unroll
        for (int c4 = 0; c4 < HD / 32; ++c4) tmem_st16x2_x32<HD>(tO + c4 * 32, v + c4 * 32);
        l *= f;
      }
      l += rowsum;
      m_run = m_new;
      // P_t(j) over the first BN/4 columns of its S buffer: column c holds keys 4c..4c+3
      // (byte = key % 4); this thread's keys start at column ch * HN / 4
      static_assert(HN == 32, "P store covers 32 keys per thread");
      tmem_st16x2_x8<8>(tS, pk);
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(BAR(B_PFULL + 2 * t + (j & 1)));
    }
    if (ok) {
      // P V of the last step completes after every earlier one (in-order tcgen05 stream)
      ok = mbar_wait(BAR(B_ODONE + 2 * t + ((nkv - 1) & 1)), ((nkv - 1) >> 1) & 1, tlim,
                     abort_flag, args.err);
      const float l_row = l + __shfl_xor_sync(0xFFFFFFFFu, l, 16);
      if (__all_sync(0xFFFFFFFFu, ok)) {
        tc_fence_after();
        const int row = q_row0 + t * BLOCK_M + r;
        const bool valid = row < seq_len;
        const float scale = __ldg(args.s_v) / l_row;   // O = acc * s_v / 448 / (l / 448)
        uint32_t v[HD];
        load_o(v);
        __nv_bfloat16* orow = args.out +
                              (static_cast<size_t>(slab) * args.rows_per_slab + seq_start + row) * D +
                              ch * HD;
        uint32_t packed[HD / 2];
#pragma unroll
        for (int i = 0; i < HD / 2; ++i) {
          const __nv_bfloat162 b2 = __floats2bfloat162_rn(__uint_as_float(v[2 * i]) * scale,
                                                          __uint_as_float(v[2 * i + 1]) * scale);
          packed[i] = *reinterpret_cast<const uint32_t*>(&b2);
        }
        if (valid) {
          uint4* dst = reinterpret_cast<uint4*>(orow);
#pragma unroll
          for (int i = 0; i < HD / 8; ++i)
            dst[i] = make_uint4(packed[4 * i], packed[4 * i + 1], packed[4 * i + 2], packed[4 * i + 3]);
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == WARP_MMA) {
    tc_fence_after();
    tmem_dealloc(tmem, TC::ALLOC);
  }
}

// ---------------------------------------------------------------------------------------------
// Host side: tensor maps and launch
// ---------------------------------------------------------------------------------------------
using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                   const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                   const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

static EncodeTiledFn get_encode_fn() {
  static EncodeTiledFn fn = nullptr;
  if (!fn) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  }
  return fn;
}

// 3-D map over an E4M3 tensor viewed as [slabs][rows][D]: box = `box_rows` rows of one slab.
static bool make_map(CUtensorMap* map, const void* ptr, int D, int rows, int slabs, int box_rows) {
  EncodeTiledFn enc = get_encode_fn();
  if (!enc) return false;
  cuuint64_t dims[3] = {static_cast<cuuint64_t>(D), static_cast<cuuint64_t>(rows),
                        static_cast<cuuint64_t>(slabs)};
  cuuint64_t strides[2] = {static_cast<cuuint64_t>(D),
                           static_cast<cuuint64_t>(D) * static_cast<cuuint64_t>(rows)};
  cuuint32_t box[3] = {static_cast<cuuint32_t>(D), static_cast<cuuint32_t>(box_rows), 1u};
  cuuint32_t estr[3] = {1u, 1u, 1u};
  CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<void*>(ptr), dims, strides,
                   box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                   D == 128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

template <int D>
static cudaError_t launch_attn_d(const void* q8, const void* k8, const void* v8, const AttnArgs& a,
                                 int rows_per_slab, int slabs, dim3 grid, cudaStream_t stream) {
  CUtensorMap mq, mk, mv;
  constexpr int BN = KvStep<D>::N;
  if (!make_map(&mq, q8, D, rows_per_slab, slabs, BLOCK_M) ||
      !make_map(&mk, k8, D, rows_per_slab, slabs, BN) ||
      !make_map(&mv, v8, D, rows_per_slab, slabs, BN))
    return cudaErrorInvalidValue;
  static int configured_dev_mask = 0;   // bit per device id < 31
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 31 && !(configured_dev_mask & (1 << dev))) {
    cudaError_t e = cudaFuncSetAttribute(k_attn_fp8_fwd<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         Smem<D>::ALLOC);
    if (e != cudaSuccess) return e;
    configured_dev_mask |= 1 << dev;
  }
  k_attn_fp8_fwd<D><<<grid, ATTN_THREADS, Smem<D>::ALLOC, stream>>>(mq, mk, mv, a);
  return cudaGetLastError();
}

cudaError_t launch_attention(const uint8_t* q8, const uint8_t* k8, const uint8_t* v8, void* out,
                             int B, int H, int L, int D, const int* cu_seqlens, int nseq,
                             int max_seqlen, int total_tokens, const float* s_q, const float* s_k,
                             const float* s_v, float sm_scale, int* err, uint64_t timeout_ns,
                             int inject_missing_q, cudaStream_t stream) {
  AttnArgs a;
  const bool varlen = cu_seqlens != nullptr;
  a.rows_per_slab = varlen ? total_tokens : L;
  a.H = H;
  a.L = L;
  a.cu_seqlens = cu_seqlens;
  a.s_q = s_q;
  a.s_k = s_k;
  a.s_v = s_v;
  a.sm_scale = sm_scale;
  a.out = static_cast<__nv_bfloat16*>(out);
  a.err = err;
  a.timeout_ns = timeout_ns;
  a.inject_missing_q = inject_missing_q;
  const int slabs = varlen ? H : B * H;
  const int lmax = varlen ? max_seqlen : L;
  dim3 grid((lmax + NQ * BLOCK_M - 1) / (NQ * BLOCK_M), H, varlen ? nseq : B);
  if (D == 128) return launch_attn_d<128>(q8, k8, v8, a, a.rows_per_slab, slabs, grid, stream);
  return launch_attn_d<64>(q8, k8, v8, a, a.rows_per_slab, slabs, grid, stream);
}

}  // namespace qattn
