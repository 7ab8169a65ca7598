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
// Kernel structure: one CTA (one per SM) per pair of 128-row Q tiles of one (sequence, head).
//   warp 8      TMA producer: both Q tiles once, then K and V tiles through separate rings.
//   warp 9      MMA issuer (one elected thread) and TMEM owner.  Per KV tile j and Q tile t it
//               issues O_t += P_t(j) V_j (P read from tensor memory) and right behind it, in the
//               same in-order tcgen05 stream, S_t = Q_t K_{j+1}^T into the columns P_t(j)
//               occupied; one commit then tells softmax t that S_t(j+1) is ready and that O_t
//               holds every P_t V up to tile j.
//   warps 0-7   two softmax warpgroups, one per Q tile; thread = one query row = one TMEM lane.
//               Each reads its 128 scores with tcgen05.ld, takes the row max (3-input maxima)
//               and computes p*448 = 2^(S' - M + log2 448) in FP32 (hardware ex2 for most
//               pairs, a degree-5 polynomial on the FMA pipe for the rest), sums p in packed
//               f32x2 adds, converts to E4M3 and writes P_t(j) over S_t(j) with tcgen05.st.
//               On a rise of M it first rescales its O row in TMEM by 2^-(rise).
//   The two Q tiles alternate on the tensor pipe, so one tile's softmax overlaps the other
//   tile's MMAs; K/V tiles are read by TMA once per CTA for both Q tiles.
// TMEM: S_0/P_0, S_1/P_1 (128 FP32 columns each; P uses the first 32), O_0, O_1 (D columns).
// All waits are bounded (a global-timer limit); on expiry the CTA records a timeout in the
// library's error word, drains what it issued and exits.
//
// Grid: dense launches are 1-D.  With a workspace, the pairs left after the last full wave of
// one CTA per SM are split along the keys: each part CTA runs the same loop over its key range
// and writes its unnormalised O rows, integer running max and row sum; k_attn_combine merges
// the parts (exact power-of-two rescales) into the bf16 output.  Varlen launches keep a
// (pair, head, sequence) grid without splitting.
#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <cstdint>

#include "launch.h"
#include "sm100_ptx.cuh"

namespace qattn {

constexpr int BLOCK_M = 128;                 // query rows per tile (= TMEM lanes)
constexpr int BLOCK_N = 128;                 // keys per KV tile
constexpr int NQ = 2;                        // query tiles per CTA
constexpr int KSTAGES = 3;
constexpr int VSTAGES = 3;
constexpr int NUM_SOFTMAX_WARPS = 4 * NQ;
constexpr int WARP_LOAD = NUM_SOFTMAX_WARPS;
constexpr int WARP_MMA = NUM_SOFTMAX_WARPS + 1;
constexpr int ATTN_THREADS = (NUM_SOFTMAX_WARPS + 2) * 32;
constexpr float LOG2E_F = 1.4426950408889634f;
constexpr float LOG2_448 = 8.807354922057604f;   // log2(448): p * 448 = 2^(S' - M + log2 448)

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
  // Dense launches use a 1-D grid: CTAs [0, full_ctas) take one pair of Q tiles each; the pairs
  // after them (the last, partial wave) are split into nsplit parts along the keys, one CTA per
  // part, which writes unnormalised partial results for the combine kernel:
  //   part_o[(((tp * nsplit + part) * NQ + t) * BLOCK_M + row) * D + c]  (FP32, row-major)
  //   part_ml[((tp * nsplit + part) * NQ + t) * BLOCK_M + row] = (running max, row sum)
  // with tp the index of the pair among the split ones.
  int pairs_per_head;
  int full_ctas;
  int nsplit;
  int combine_pairs;        // number of split pairs (the combine kernel's work)
  float* part_o;
  float2* part_ml;
};

template <int D>
struct Smem {
  static constexpr int TILE_Q = BLOCK_M * D;       // bytes (E4M3)
  static constexpr int TILE_KV = BLOCK_N * D;
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_K = OFF_Q + NQ * TILE_Q;
  static constexpr int OFF_V = OFF_K + KSTAGES * TILE_KV;
  static constexpr int OFF_BAR = OFF_V + VSTAGES * TILE_KV;
  // barriers: q_full, k_full[KS], k_empty[KS], v_full[VS], v_empty[VS], s_full[NQ],
  // p_full[NQ], o_final[NQ], drain
  static constexpr int NBARS = 1 + 2 * KSTAGES + 2 * VSTAGES + 3 * NQ + 1;
  static constexpr int OFF_TMEM = OFF_BAR + 8 * NBARS;
  static constexpr int OFF_ABORT = OFF_TMEM + 4;
  static constexpr int BYTES = OFF_ABORT + 4;
  static constexpr int ALLOC = BYTES + 1024;       // slack for 1024-byte alignment
  static_assert(TILE_Q % 1024 == 0 && TILE_KV % 1024 == 0, "alignment");
};

template <int D>
struct TmemCols {
  static constexpr uint32_t S0 = 0;                      // S_t / P_t at t * BLOCK_N
  static constexpr uint32_t O0 = NQ * BLOCK_N;           // O_t at O0 + t * D
  static constexpr uint32_t USED = NQ * BLOCK_N + NQ * D;
  static constexpr uint32_t ALLOC = USED <= 256 ? 256 : 512;
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
// Of every 8 pairs of scores, pairs 1 and 5 take the polynomial and the rest MUFU ex2.  Two of
// eight balances the two pipes; spreading the two apart in issue order measured about 1.5%
// faster than giving the polynomial to pairs 0 and 1.
__device__ __forceinline__ constexpr bool poly_pair(int q) { return (q & 3) == 1; }
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

template <int D>
__global__ void __launch_bounds__(ATTN_THREADS, 1)
    k_attn_fp8_fwd(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                   const __grid_constant__ CUtensorMap tm_v, const AttnArgs args) {
  using SL = Smem<D>;
  using TC = TmemCols<D>;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_u32 = smem_u32(smem_raw);
  const uint32_t base_u32 = (raw_u32 + 1023u) & ~1023u;
  uint8_t* base = smem_raw + (base_u32 - raw_u32);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  // ---- which sequence and which rows -------------------------------------------------------
  int qblk, h, bz;                                // pair of Q tiles, head, batch row / sequence
  int part = 0, nparts = 1, split_pair = -1;
  if (args.cu_seqlens) {
    qblk = blockIdx.x;
    h = blockIdx.y;
    bz = blockIdx.z;
  } else {
    int pair = blockIdx.x;
    if (pair >= args.full_ctas) {                 // a part of a split pair
      const int u = pair - args.full_ctas;
      split_pair = u / args.nsplit;
      part = u % args.nsplit;
      nparts = args.nsplit;
      pair = args.full_ctas + split_pair;
    }
    qblk = pair % args.pairs_per_head;
    h = (pair / args.pairs_per_head) % args.H;
    bz = pair / (args.pairs_per_head * args.H);
  }
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
  // key steps [kv0, kv0 + nkv) of this CTA (all of them unless the pair is split)
  const int nkv_all = (seq_len + BLOCK_N - 1) / BLOCK_N;
  const int steps_per_part = (nkv_all + nparts - 1) / nparts;
  const int kv0 = part * steps_per_part;
  const int nkv = min(nkv_all, kv0 + steps_per_part) - kv0;   // >= 1: the host keeps parts
                                                               // shorter than the sequence

  // ---- barriers --------------------------------------------------------------------------
  const uint32_t bar0 = base_u32 + SL::OFF_BAR;
  auto BAR = [&](int i) { return bar0 + 8u * static_cast<uint32_t>(i); };
  constexpr int B_QFULL = 0;
  constexpr int B_KFULL = 1, B_KEMPTY = B_KFULL + KSTAGES;
  constexpr int B_VFULL = B_KEMPTY + KSTAGES, B_VEMPTY = B_VFULL + VSTAGES;
  constexpr int B_SFULL = B_VEMPTY + VSTAGES, B_PFULL = B_SFULL + NQ;
  constexpr int B_OFINAL = B_PFULL + NQ, B_DRAIN = B_OFINAL + NQ;
  volatile int* abort_flag = reinterpret_cast<volatile int*>(base + SL::OFF_ABORT);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(base + SL::OFF_TMEM);

  if (threadIdx.x == 0) {
    mbar_init(BAR(B_QFULL), 1);
    for (int i = 0; i < KSTAGES; ++i) { mbar_init(BAR(B_KFULL + i), 1); mbar_init(BAR(B_KEMPTY + i), 1); }
    for (int i = 0; i < VSTAGES; ++i) { mbar_init(BAR(B_VFULL + i), 1); mbar_init(BAR(B_VEMPTY + i), 1); }
    for (int t = 0; t < NQ; ++t) {
      mbar_init(BAR(B_SFULL + t), 1);
      mbar_init(BAR(B_PFULL + t), BLOCK_M);
      mbar_init(BAR(B_OFINAL + t), 1);
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
    // ======================= TMA producer =======================
    if (lane == 0 && !args.inject_missing_q) {
      tma_prefetch_desc(&tm_q);
      tma_prefetch_desc(&tm_k);
      tma_prefetch_desc(&tm_v);
      int nk = 0, nv = 0;                          // loads issued
      mbar_arrive_expect_tx(BAR(B_QFULL), NQ * SL::TILE_Q);
      for (int t = 0; t < NQ; ++t)
        tma_load_3d(base_u32 + SL::OFF_Q + t * SL::TILE_Q, &tm_q, BAR(B_QFULL), 0,
                    seq_start + q_row0 + t * BLOCK_M, slab);
      auto load_k = [&](int j) -> bool {
        const int s = j % KSTAGES;
        if (j >= KSTAGES &&
            !mbar_wait(BAR(B_KEMPTY + s), ((j / KSTAGES) - 1) & 1, tlim, abort_flag, args.err))
          return false;
        mbar_arrive_expect_tx(BAR(B_KFULL + s), SL::TILE_KV);
        tma_load_3d(base_u32 + SL::OFF_K + s * SL::TILE_KV, &tm_k, BAR(B_KFULL + s), 0,
                    seq_start + (kv0 + j) * BLOCK_N, slab);
        ++nk;
        return true;
      };
      auto load_v = [&](int j) -> bool {
        const int s = j % VSTAGES;
        if (j >= VSTAGES &&
            !mbar_wait(BAR(B_VEMPTY + s), ((j / VSTAGES) - 1) & 1, tlim, abort_flag, args.err))
          return false;
        mbar_arrive_expect_tx(BAR(B_VFULL + s), SL::TILE_KV);
        tma_load_3d(base_u32 + SL::OFF_V + s * SL::TILE_KV, &tm_v, BAR(B_VFULL + s), 0,
                    seq_start + (kv0 + j) * BLOCK_N, slab);
        ++nv;
        return true;
      };
      // order of use on the tensor pipe: K0, V0, K1, V1, ...; K runs one tile ahead
      bool ok = load_k(0);
      for (int j = 0; ok && j < nkv; ++j) {
        if (j + 1 < nkv) ok = load_k(j + 1);
        if (ok) ok = load_v(j);
      }
      // drain: every issued load has landed before the CTA may exit (instant when healthy)
      mbar_drain(BAR(B_QFULL), 0, tlim);
      for (int j = nk - 1; j >= 0 && j >= nk - KSTAGES; --j)
        mbar_drain(BAR(B_KFULL + j % KSTAGES), (j / KSTAGES) & 1, tlim);
      for (int j = nv - 1; j >= 0 && j >= nv - VSTAGES; --j)
        mbar_drain(BAR(B_VFULL + j % VSTAGES), (j / VSTAGES) & 1, tlim);
    }
  } else if (warp == WARP_MMA) {
    // ======================= MMA issuer =======================
    if (lane == 0) {
      constexpr uint32_t IDESC_S = idesc_e4m3_f32(BLOCK_M, BLOCK_N, false);
      constexpr uint32_t IDESC_O = idesc_e4m3_f32(BLOCK_M, D, true);
      // Q, K: K-major rows of D bytes, swizzled in 8-row atoms (SBO = 8 rows); 32-byte K steps.
      constexpr uint32_t QK_LAYOUT = (D == 128) ? 2u : 4u;   // 128B / 64B swizzle
      constexpr uint32_t QK_SBO = 8 * D;
      // V: MN-major (D contiguous per key row), rows of D bytes, SBO = 8 key rows; a K step
      // of 32 keys advances 32 rows.
      constexpr uint32_t V_LAYOUT = QK_LAYOUT;
      constexpr uint32_t V_SBO = 8 * D;
      auto bmm1 = [&](int t, int ks) {
        const uint32_t qa = base_u32 + SL::OFF_Q + t * SL::TILE_Q;
        const uint32_t kb = base_u32 + SL::OFF_K + ks * SL::TILE_KV;
#pragma unroll
        for (int kk = 0; kk < D / 32; ++kk) {
          const uint64_t da = smem_desc(qa + kk * 32, 16, QK_SBO, QK_LAYOUT);
          const uint64_t db = smem_desc(kb + kk * 32, 16, QK_SBO, QK_LAYOUT);
          mma_f8_ss(tmem + TC::S0 + t * BLOCK_N, da, db, IDESC_S, kk > 0 ? 1u : 0u);
        }
      };
      auto bmm2 = [&](int t, int vs, bool first) {
        const uint32_t vb = base_u32 + SL::OFF_V + vs * SL::TILE_KV;
#pragma unroll
        for (int kk = 0; kk < BLOCK_N / 32; ++kk) {
          const uint64_t db = smem_desc(vb + kk * 32 * D, SL::TILE_KV, V_SBO, V_LAYOUT);
          mma_f8_ts(tmem + TC::O0 + t * D, tmem + TC::S0 + t * BLOCK_N + kk * 8, db, IDESC_O,
                    (!first || kk > 0) ? 1u : 0u);
        }
      };
      bool ok = mbar_wait(BAR(B_QFULL), 0, tlim, abort_flag, args.err) &&
                mbar_wait(BAR(B_KFULL + 0), 0, tlim, abort_flag, args.err);
      if (ok) {
        tc_fence_after();
        for (int t = 0; t < NQ; ++t) {
          bmm1(t, 0);
          mma_commit(BAR(B_SFULL + t));
        }
        mma_commit(BAR(B_KEMPTY + 0));
      }
      for (int j = 0; ok && j < nkv; ++j) {
        const int vs = j % VSTAGES;
        const bool more = j + 1 < nkv;
        const int ks = (j + 1) % KSTAGES;
        ok = mbar_wait(BAR(B_VFULL + vs), (j / VSTAGES) & 1, tlim, abort_flag, args.err);
        if (ok && more)
          ok = mbar_wait(BAR(B_KFULL + ks), ((j + 1) / KSTAGES) & 1, tlim, abort_flag, args.err);
        for (int t = 0; ok && t < NQ; ++t) {
          ok = mbar_wait(BAR(B_PFULL + t), j & 1, tlim, abort_flag, args.err);
          if (!ok) break;
          tc_fence_after();
          bmm2(t, vs, j == 0);                     // reads P_t(j) from TMEM
          if (more) {
            bmm1(t, ks);                           // overwrites S_t / P_t after bmm2 read it
            mma_commit(BAR(B_SFULL + t));
          } else {
            mma_commit(BAR(B_OFINAL + t));
          }
        }
        if (ok) {
          mma_commit(BAR(B_VEMPTY + vs));
          if (more) mma_commit(BAR(B_KEMPTY + ks));
        }
      }
      // drain: all issued MMAs complete before TMEM is released
      mma_commit(BAR(B_DRAIN));
      mbar_drain(BAR(B_DRAIN), 0, tlim);
    }
  } else {
    // ======================= softmax warpgroups =======================
    const int t = warp >> 2;                       // Q tile of this warpgroup
    const int quarter = warp & 3;                  // TMEM lane quarter
    const int r = quarter * 32 + lane;             // row within the Q tile
    const uint32_t lane_off = static_cast<uint32_t>(quarter * 32) << 16;
    const uint32_t tS = tmem + lane_off + TC::S0 + t * BLOCK_N;
    const uint32_t tO = tmem + lane_off + TC::O0 + t * D;
    const float c = __ldg(args.s_q) * __ldg(args.s_k) * args.sm_scale * LOG2E_F;
    float m_run = -INFINITY;                       // integer-valued running max (base 2)
    float l = 0.0f;                                // running sum of p * 448
    bool ok = true;
    for (int j = 0; j < nkv; ++j) {
      // S_t(j) is in TMEM; BMM2 of tile j-1 has completed (it precedes in the MMA stream)
      ok = mbar_wait(BAR(B_SFULL + t), j & 1, tlim, abort_flag, args.err);
      if (!__all_sync(0xFFFFFFFFu, ok)) { ok = false; break; }
      tc_fence_after();
      float s[BLOCK_N];
      {
        uint32_t sv[BLOCK_N / 32][32];
#pragma unroll
        for (int c4 = 0; c4 < BLOCK_N / 32; ++c4) tmem_ld32(tS + c4 * 32, sv[c4]);
        tmem_wait_ld();
#pragma unroll
        for (int i = 0; i < BLOCK_N; ++i) s[i] = __uint_as_float(sv[i / 32][i % 32]);
      }
      const int kv_valid = seq_len - (kv0 + j) * BLOCK_N;  // keys of this tile in the sequence
      if (kv_valid < BLOCK_N) {
#pragma unroll
        for (int i = 0; i < BLOCK_N; ++i)
          if (i >= kv_valid) s[i] = -INFINITY;
      }
      const float m_new = fmaxf(m_run, ceilf(rowmax128(s) * c));
      const float neg_off = LOG2_448 - m_new;
      float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
      uint32_t pk[BLOCK_N / 4];
#pragma unroll
      for (int i = 0; i < BLOCK_N; i += 16) {
        float p[16];
#pragma unroll
        for (int q = 0; q < 8; ++q) {
          float x0, x1;
          ffma2_bc(x0, x1, s[i + 2 * q], s[i + 2 * q + 1], c, neg_off);
          if (poly_pair(q)) {
            poly_exp2_x2(x0, x1, p[2 * q], p[2 * q + 1]);
          } else {
            p[2 * q] = fast_exp2(x0);
            p[2 * q + 1] = fast_exp2(x1);
          }
        }
#pragma unroll
        for (int q = 0; q < 8; ++q) fadd2_acc(acc[2 * (q & 3)], acc[2 * (q & 3) + 1], p[2 * q], p[2 * q + 1]);
#pragma unroll
        for (int q = 0; q < 4; ++q)
          pk[i / 4 + q] = cvt_e4m3x2(p[4 * q], p[4 * q + 1]) | (cvt_e4m3x2(p[4 * q + 2], p[4 * q + 3]) << 16);
      }
      const float rowsum = ((acc[0] + acc[1]) + (acc[2] + acc[3])) + ((acc[4] + acc[5]) + (acc[6] + acc[7]));
      // A rise of the running max rescales this row of O (quiescent: its last BMM2 is done).
      if (j > 0) {
        const bool rise = m_new > m_run;
        if (__any_sync(0xFFFFFFFFu, rise)) {
          const float f = rise ? exp2_int(static_cast<int>(m_run - m_new)) : 1.0f;
          uint64_t f2;                             // packed f32x2 multiplies
          asm("mov.b64 %0, {%1, %1};" : "=l"(f2) : "f"(f));
#pragma unroll
          for (int c4 = 0; c4 < D / 32; ++c4) {
            uint32_t v[32];
            tmem_ld32(tO + c4 * 32, v);
            tmem_wait_ld();
#pragma unroll
            for (int i = 0; i < 32; i += 2) {
              uint64_t pr;
              asm("{\n\t.reg .b64 a;\n\tmov.b64 a, {%1, %2};\n\tmul.rn.f32x2 %0, a, %3;\n\t}"
                  : "=l"(pr) : "r"(v[i]), "r"(v[i + 1]), "l"(f2));
              asm("mov.b64 {%0, %1}, %2;" : "=r"(v[i]), "=r"(v[i + 1]) : "l"(pr));
            }
            tmem_st32(tO + c4 * 32, v);
          }
          l *= f;
        }
      }
      l += rowsum;
      m_run = m_new;
      // P_t(j) over the first 32 columns of S_t: column c holds keys 4c..4c+3 (byte = key % 4)
      tmem_st32(tS, pk);
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(BAR(B_PFULL + t));
    }
    if (ok) {
      ok = mbar_wait(BAR(B_OFINAL + t), 0, tlim, abort_flag, args.err);
      if (__all_sync(0xFFFFFFFFu, ok)) {
        tc_fence_after();
        const int row = q_row0 + t * BLOCK_M + r;
        const bool valid = row < seq_len;
        if (nparts > 1) {
          // partial result of this part: raw O row, running max and row sum
          const size_t slot = (static_cast<size_t>(split_pair) * nparts + part) * NQ + t;
          float4* po = reinterpret_cast<float4*>(args.part_o + (slot * BLOCK_M + r) * D);
#pragma unroll
          for (int c4 = 0; c4 < D / 32; ++c4) {
            uint32_t v[32];
            tmem_ld32(tO + c4 * 32, v);
            tmem_wait_ld();
#pragma unroll
            for (int i = 0; i < 8; ++i)
              po[c4 * 8 + i] = make_float4(__uint_as_float(v[4 * i]), __uint_as_float(v[4 * i + 1]),
                                           __uint_as_float(v[4 * i + 2]), __uint_as_float(v[4 * i + 3]));
          }
          args.part_ml[slot * BLOCK_M + r] = make_float2(m_run, l);
        } else {
        const float scale = __ldg(args.s_v) / l;   // O = acc * s_v / 448 / (l / 448)
        __nv_bfloat16* orow =
            args.out + (static_cast<size_t>(slab) * args.rows_per_slab + seq_start + row) * D;
#pragma unroll
        for (int c4 = 0; c4 < D / 32; ++c4) {
          uint32_t v[32];
          tmem_ld32(tO + c4 * 32, v);
          tmem_wait_ld();
          uint32_t packed[16];
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            const __nv_bfloat162 b2 = __floats2bfloat162_rn(__uint_as_float(v[2 * i]) * scale,
                                                            __uint_as_float(v[2 * i + 1]) * scale);
            packed[i] = *reinterpret_cast<const uint32_t*>(&b2);
          }
          if (valid) {
            uint4* dst = reinterpret_cast<uint4*>(orow + c4 * 32);
#pragma unroll
            for (int i = 0; i < 4; ++i)
              dst[i] = make_uint4(packed[4 * i], packed[4 * i + 1], packed[4 * i + 2], packed[4 * i + 3]);
          }
        }
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
// Combine of split pairs: one warp per output row (COMBINE_WARPS rows per CTA), each lane D / 32
// columns.  The parts' running maxima are integers, so each part is brought to the common
// maximum M by an exact power of two: O = sum_p 2^(m_p - M) O_p, l = sum_p 2^(m_p - M) l_p,
// out = O * s_v / l.
// ---------------------------------------------------------------------------------------------
constexpr int COMBINE_WARPS = 8;

template <int D>
__global__ void __launch_bounds__(COMBINE_WARPS * 32) k_attn_combine(const AttnArgs args) {
  constexpr int VEC = D / 32;                       // columns per lane: 4 or 2
  const int lane = threadIdx.x & 31;
  const int grow = blockIdx.x * COMBINE_WARPS + (threadIdx.x >> 5);   // row over all slots
  const int tp = grow / (NQ * BLOCK_M);
  const int t = (grow / BLOCK_M) % NQ;
  const int r = grow % BLOCK_M;
  if (tp >= args.combine_pairs) return;
  const int pair = args.full_ctas + tp;
  const int qblk = pair % args.pairs_per_head;
  const int h = (pair / args.pairs_per_head) % args.H;
  const int bz = pair / (args.pairs_per_head * args.H);
  const int row = qblk * (NQ * BLOCK_M) + t * BLOCK_M + r;
  if (row >= args.L) return;
  const int S = args.nsplit;
  auto slot = [&](int p) { return (static_cast<size_t>(tp) * S + p) * NQ + t; };
  float M = -INFINITY;
  for (int p = 0; p < S; ++p) M = fmaxf(M, args.part_ml[slot(p) * BLOCK_M + r].x);
  float l = 0.0f;
  float acc[VEC];
#pragma unroll
  for (int i = 0; i < VEC; ++i) acc[i] = 0.0f;
  for (int p = 0; p < S; ++p) {
    const float2 ml = args.part_ml[slot(p) * BLOCK_M + r];
    const float w = exp2_int(static_cast<int>(ml.x - M));
    l = fmaf(w, ml.y, l);
    const float* po = args.part_o + (slot(p) * BLOCK_M + r) * D + lane * VEC;
    if constexpr (VEC == 4) {
      const float4 o = *reinterpret_cast<const float4*>(po);
      acc[0] = fmaf(w, o.x, acc[0]); acc[1] = fmaf(w, o.y, acc[1]);
      acc[2] = fmaf(w, o.z, acc[2]); acc[3] = fmaf(w, o.w, acc[3]);
    } else {
      const float2 o = *reinterpret_cast<const float2*>(po);
      acc[0] = fmaf(w, o.x, acc[0]); acc[1] = fmaf(w, o.y, acc[1]);
    }
  }
  const float scale = __ldg(args.s_v) / l;
  __nv_bfloat16* orow =
      args.out + (static_cast<size_t>(bz * args.H + h) * args.L + row) * D + lane * VEC;
  uint32_t packed[VEC / 2];
#pragma unroll
  for (int i = 0; i < VEC / 2; ++i) {
    const __nv_bfloat162 b2 = __floats2bfloat162_rn(acc[2 * i] * scale, acc[2 * i + 1] * scale);
    packed[i] = *reinterpret_cast<const uint32_t*>(&b2);
  }
  if constexpr (VEC == 4)
    *reinterpret_cast<uint2*>(orow) = make_uint2(packed[0], packed[1]);
  else
    *reinterpret_cast<uint32_t*>(orow) = packed[0];
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

// 3-D map over an E4M3 tensor viewed as [slabs][rows][D]: box = one 128-row tile of one slab.
static bool make_map(CUtensorMap* map, const void* ptr, int D, int rows, int slabs) {
  EncodeTiledFn enc = get_encode_fn();
  if (!enc) return false;
  cuuint64_t dims[3] = {static_cast<cuuint64_t>(D), static_cast<cuuint64_t>(rows),
                        static_cast<cuuint64_t>(slabs)};
  cuuint64_t strides[2] = {static_cast<cuuint64_t>(D),
                           static_cast<cuuint64_t>(D) * static_cast<cuuint64_t>(rows)};
  cuuint32_t box[3] = {static_cast<cuuint32_t>(D), 128u, 1u};
  cuuint32_t estr[3] = {1u, 1u, 1u};
  CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<void*>(ptr), dims, strides,
                   box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                   D == 128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

template <int D>
static cudaError_t launch_attn_d(const void* q8, const void* k8, const void* v8, const AttnArgs& a,
                                 int rows_per_slab, int slabs, dim3 grid, int combine_ctas,
                                 cudaStream_t stream) {
  CUtensorMap mq, mk, mv;
  if (!make_map(&mq, q8, D, rows_per_slab, slabs) || !make_map(&mk, k8, D, rows_per_slab, slabs) ||
      !make_map(&mv, v8, D, rows_per_slab, slabs))
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
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess || combine_ctas == 0) return e;
  k_attn_combine<D><<<combine_ctas, COMBINE_WARPS * 32, 0, stream>>>(a);
  return cudaGetLastError();
}

// Split plan of a dense launch: pairs beyond the last full wave of num_sms CTAs (one CTA per
// SM) are split along the keys into the number of parts (2..4) that shortens that partial wave
// the most, if it shortens it to at most 0.8 of a full CTA's time; each part keeps at least two
// key steps.  bytes = the workspace the parts need (0: no split).
AttnSplitPlan plan_attention_split(int B, int H, int L, int D, int num_sms) {
  AttnSplitPlan p;
  p.pairs_per_head = (L + NQ * BLOCK_M - 1) / (NQ * BLOCK_M);
  const long long pairs = static_cast<long long>(p.pairs_per_head) * H * B;
  const int nkv = (L + BLOCK_N - 1) / BLOCK_N;
  const long long tail = num_sms > 0 ? pairs % num_sms : 0;
  p.nsplit = 1;
  double best = 1.0;
  for (int S = 2; tail > 0 && S <= 4; ++S) {
    if (nkv < 2 * S) break;
    const double tt = static_cast<double>((tail * S + num_sms - 1) / num_sms) / S;
    if (tt < best - 1e-9) {
      best = tt;
      p.nsplit = S;
    }
  }
  if (best > 0.8) p.nsplit = 1;
  p.tail = p.nsplit > 1 ? static_cast<int>(tail) : 0;
  p.full_ctas = static_cast<int>(pairs - p.tail);
  p.bytes = static_cast<size_t>(p.tail) * p.nsplit * NQ * BLOCK_M * (D + 2) * sizeof(float);
  return p;
}

cudaError_t launch_attention(const uint8_t* q8, const uint8_t* k8, const uint8_t* v8, void* out,
                             int B, int H, int L, int D, const int* cu_seqlens, int nseq,
                             int max_seqlen, int total_tokens, const float* s_q, const float* s_k,
                             const float* s_v, float sm_scale, int* err, uint64_t timeout_ns,
                             int inject_missing_q, void* workspace, size_t workspace_bytes,
                             int num_sms, cudaStream_t stream) {
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
  a.part_o = nullptr;
  a.part_ml = nullptr;
  a.combine_pairs = 0;
  const int slabs = varlen ? H : B * H;
  dim3 grid;
  int combine_ctas = 0;
  if (varlen) {
    a.pairs_per_head = 0;
    a.full_ctas = 0;
    a.nsplit = 1;
    grid = dim3((max_seqlen + NQ * BLOCK_M - 1) / (NQ * BLOCK_M), H, nseq);
  } else {
    AttnSplitPlan p = plan_attention_split(B, H, L, D, num_sms);
    if (workspace == nullptr || workspace_bytes < p.bytes) {   // no workspace: no split
      p.nsplit = 1;
      p.full_ctas += p.tail;
      p.tail = 0;
    }
    a.pairs_per_head = p.pairs_per_head;
    a.full_ctas = p.full_ctas;
    a.nsplit = p.nsplit;
    a.combine_pairs = p.tail;
    if (p.tail > 0) {
      const size_t o_elems = static_cast<size_t>(p.tail) * p.nsplit * NQ * BLOCK_M * D;
      a.part_o = static_cast<float*>(workspace);
      a.part_ml = reinterpret_cast<float2*>(a.part_o + o_elems);
      combine_ctas = p.tail * NQ * BLOCK_M / COMBINE_WARPS;
    }
    grid = dim3(p.full_ctas + p.tail * p.nsplit, 1, 1);
  }
  if (D == 128)
    return launch_attn_d<128>(q8, k8, v8, a, a.rows_per_slab, slabs, grid, combine_ctas, stream);
  return launch_attn_d<64>(q8, k8, v8, a, a.rows_per_slab, slabs, grid, combine_ctas, stream);
}

}  // namespace qattn
