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
// Kernel structure (one CTA per SM, persistent over nothing: one CTA per pair of 128-row Q tiles):
//   warp 8      TMA producer: Q tiles once, then K and V tiles through separate rings.
//   warp 9      MMA issuer (one thread) and TMEM owner: S_t = Q_t K_j^T for both tiles as
//               soon as the softmax of tile j-1 has read S_t, then O_t += P_t V_j.
//   warps 0-7   two softmax warpgroups, one per Q tile; thread = one query row = one TMEM lane.
//               Each reads its 128 scores with tcgen05.ld, computes the row max, the exp2 and
//               the row sum in FP32, converts p*448 to E4M3 and stores the row of P to shared
//               memory in the 128-byte-swizzled K-major layout BMM2 reads; on a rise of M it
//               rescales its O row in TMEM by 2^-(rise) first.
// TMEM: S_0, S_1 (128 FP32 columns each), O_0, O_1 (D columns each).
// All waits are bounded (a global-timer limit); on expiry the CTA records a timeout in the
// library's error word, drains what it issued and exits.
#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <cstdint>

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
};

template <int D>
struct Smem {
  static constexpr int TILE_Q = BLOCK_M * D;       // bytes (E4M3)
  static constexpr int TILE_KV = BLOCK_N * D;
  static constexpr int TILE_P = BLOCK_M * BLOCK_N;
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_K = OFF_Q + NQ * TILE_Q;
  static constexpr int OFF_V = OFF_K + KSTAGES * TILE_KV;
  static constexpr int OFF_P = OFF_V + VSTAGES * TILE_KV;
  static constexpr int OFF_BAR = OFF_P + NQ * TILE_P;
  // barriers: q_full, k_full[KS], k_empty[KS], v_full[VS], v_empty[VS], s_full[NQ],
  // s_free[NQ], p_full[NQ], o_done[NQ], drain
  static constexpr int NBARS = 1 + 2 * KSTAGES + 2 * VSTAGES + 4 * NQ + 1;
  static constexpr int OFF_TMEM = OFF_BAR + 8 * NBARS;
  static constexpr int OFF_ABORT = OFF_TMEM + 4;
  static constexpr int BYTES = OFF_ABORT + 4;
  static constexpr int ALLOC = BYTES + 1024;       // slack for 1024-byte alignment
  static_assert(TILE_Q % 1024 == 0 && TILE_KV % 1024 == 0 && TILE_P % 1024 == 0, "alignment");
};

template <int D>
struct TmemCols {
  static constexpr uint32_t S0 = 0;                      // S_t at t * BLOCK_N
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
  const int nkv = (seq_len + BLOCK_N - 1) / BLOCK_N;

  // ---- barriers --------------------------------------------------------------------------
  const uint32_t bar0 = base_u32 + SL::OFF_BAR;
  auto BAR = [&](int i) { return bar0 + 8u * static_cast<uint32_t>(i); };
  const int B_QFULL = 0;
  const int B_KFULL = 1, B_KEMPTY = B_KFULL + KSTAGES;
  const int B_VFULL = B_KEMPTY + KSTAGES, B_VEMPTY = B_VFULL + VSTAGES;
  const int B_SFULL = B_VEMPTY + VSTAGES, B_SFREE = B_SFULL + NQ;
  const int B_PFULL = B_SFREE + NQ, B_ODONE = B_PFULL + NQ;
  const int B_DRAIN = B_ODONE + NQ;
  volatile int* abort_flag = reinterpret_cast<volatile int*>(base + SL::OFF_ABORT);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(base + SL::OFF_TMEM);

  if (threadIdx.x == 0) {
    mbar_init(BAR(B_QFULL), 1);
    for (int i = 0; i < KSTAGES; ++i) { mbar_init(BAR(B_KFULL + i), 1); mbar_init(BAR(B_KEMPTY + i), 1); }
    for (int i = 0; i < VSTAGES; ++i) { mbar_init(BAR(B_VFULL + i), 1); mbar_init(BAR(B_VEMPTY + i), 1); }
    for (int t = 0; t < NQ; ++t) {
      mbar_init(BAR(B_SFULL + t), 1);
      mbar_init(BAR(B_SFREE + t), BLOCK_M);
      mbar_init(BAR(B_PFULL + t), BLOCK_M);
      mbar_init(BAR(B_ODONE + t), 1);
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
    if (lane == 0) {
      tma_prefetch_desc(&tm_q);
      tma_prefetch_desc(&tm_k);
      tma_prefetch_desc(&tm_v);
      bool ok = true;
      int nk = 0, nv = 0;                          // loads issued
      if (!args.inject_missing_q) {
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
                      seq_start + j * BLOCK_N, slab);
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
                      seq_start + j * BLOCK_N, slab);
          ++nv;
          return true;
        };
        ok = load_k(0);
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
      (void)ok;
    }
  } else if (warp == WARP_MMA) {
    // ======================= MMA issuer =======================
    if (lane == 0) {
      constexpr uint32_t IDESC_S = idesc_e4m3_f32(BLOCK_M, BLOCK_N, false);
      constexpr uint32_t IDESC_O = idesc_e4m3_f32(BLOCK_M, D, true);
      // Q, K: K-major rows of D bytes, swizzled in 8-row atoms (SBO = 8 rows).
      constexpr uint32_t QK_LAYOUT = (D == 128) ? 2u : 4u;   // 128B / 64B swizzle
      constexpr uint32_t QK_SBO = 8 * D;
      // P: K-major rows of 128 bytes (128 keys), 128B swizzle.
      // V: MN-major (D contiguous per key row), rows of D bytes, SBO = 8 key rows.
      constexpr uint32_t V_LAYOUT = QK_LAYOUT;
      constexpr uint32_t V_SBO = 8 * D;
      bool ok = mbar_wait(BAR(B_QFULL), 0, tlim, abort_flag, args.err);
      auto bmm1 = [&](int j) -> bool {
        const int s = j % KSTAGES;
        if (!mbar_wait(BAR(B_KFULL + s), (j / KSTAGES) & 1, tlim, abort_flag, args.err))
          return false;
        for (int t = 0; t < NQ; ++t) {
          if (j > 0 && !mbar_wait(BAR(B_SFREE + t), (j - 1) & 1, tlim, abort_flag, args.err))
            return false;
          tc_fence_after();
          const uint32_t qa = base_u32 + SL::OFF_Q + t * SL::TILE_Q;
          const uint32_t kb = base_u32 + SL::OFF_K + s * SL::TILE_KV;
#pragma unroll
          for (int kk = 0; kk < D / 32; ++kk) {
            const uint64_t da = smem_desc(qa + kk * 32, 16, QK_SBO, QK_LAYOUT);
            const uint64_t db = smem_desc(kb + kk * 32, 16, QK_SBO, QK_LAYOUT);
            mma_f8_ss(tmem + TC::S0 + t * BLOCK_N, da, db, IDESC_S, kk > 0 ? 1u : 0u);
          }
          mma_commit(BAR(B_SFULL + t));
        }
        mma_commit(BAR(B_KEMPTY + s));
        return true;
      };
      if (ok) ok = bmm1(0);
      for (int j = 0; ok && j < nkv; ++j) {
        if (j + 1 < nkv) ok = bmm1(j + 1);
        if (!ok) break;
        const int s = j % VSTAGES;
        ok = mbar_wait(BAR(B_VFULL + s), (j / VSTAGES) & 1, tlim, abort_flag, args.err);
        for (int t = 0; ok && t < NQ; ++t) {
          ok = mbar_wait(BAR(B_PFULL + t), j & 1, tlim, abort_flag, args.err);
          if (!ok) break;
          tc_fence_after();
          const uint32_t pa = base_u32 + SL::OFF_P + t * SL::TILE_P;
          const uint32_t vb = base_u32 + SL::OFF_V + s * SL::TILE_KV;
#pragma unroll
          for (int kk = 0; kk < BLOCK_N / 32; ++kk) {
            const uint64_t da = smem_desc(pa + kk * 32, 16, 1024, 2u);
            const uint64_t db = smem_desc(vb + kk * 32 * D, SL::TILE_KV, V_SBO, V_LAYOUT);
            mma_f8_ss(tmem + TC::O0 + t * D, da, db, IDESC_O, (j > 0 || kk > 0) ? 1u : 0u);
          }
          mma_commit(BAR(B_ODONE + t));
        }
        if (ok) mma_commit(BAR(B_VEMPTY + s));
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
    uint8_t* prow = base + SL::OFF_P + t * SL::TILE_P + r * BLOCK_N;
    const float c = __ldg(args.s_q) * __ldg(args.s_k) * args.sm_scale * LOG2E_F;
    float m_run = -INFINITY;                       // integer-valued running max (base 2)
    float l = 0.0f;                                // running sum of p * 448
    bool ok = true;
    for (int j = 0; j < nkv; ++j) {
      ok = mbar_wait(BAR(B_SFULL + t), j & 1, tlim, abort_flag, args.err);
      if (!__all_sync(0xFFFFFFFFu, ok)) { ok = false; break; }
      tc_fence_after();
      float s[BLOCK_N];
#pragma unroll
      for (int c4 = 0; c4 < BLOCK_N / 32; ++c4) {
        uint32_t v[32];
        tmem_ld32(tS + c4 * 32, v);
        tmem_wait_ld();
#pragma unroll
        for (int i = 0; i < 32; ++i) s[c4 * 32 + i] = __uint_as_float(v[i]);
      }
      tc_fence_before();
      mbar_arrive(BAR(B_SFREE + t));               // S_t may now be overwritten
      const int kv_valid = seq_len - j * BLOCK_N;  // keys of this tile inside the sequence
      if (kv_valid < BLOCK_N) {
#pragma unroll
        for (int i = 0; i < BLOCK_N; ++i)
          if (i >= kv_valid) s[i] = -INFINITY;
      }
      float mx = s[0];
#pragma unroll
      for (int i = 1; i < BLOCK_N; ++i) mx = fmaxf(mx, s[i]);
      const float m_new = fmaxf(m_run, ceilf(mx * c));
      const float neg_off = LOG2_448 - m_new;
      float rowsum = 0.0f;
      uint32_t pk[BLOCK_N / 4];
#pragma unroll
      for (int i = 0; i < BLOCK_N; i += 4) {
        const float p0 = fast_exp2(fmaf(s[i + 0], c, neg_off));
        const float p1 = fast_exp2(fmaf(s[i + 1], c, neg_off));
        const float p2 = fast_exp2(fmaf(s[i + 2], c, neg_off));
        const float p3 = fast_exp2(fmaf(s[i + 3], c, neg_off));
        rowsum += (p0 + p1) + (p2 + p3);
        pk[i / 4] = cvt_e4m3x2(p0, p1) | (cvt_e4m3x2(p2, p3) << 16);
      }
      // BMM2 of the previous tile must be done: it reads the P buffer and accumulates O.
      if (j > 0) {
        ok = mbar_wait(BAR(B_ODONE + t), (j - 1) & 1, tlim, abort_flag, args.err);
        if (!__all_sync(0xFFFFFFFFu, ok)) { ok = false; break; }
        tc_fence_after();
        const bool rise = m_new > m_run;
        if (__any_sync(0xFFFFFFFFu, rise)) {
          const float f = rise ? exp2_int(static_cast<int>(m_run - m_new)) : 1.0f;
#pragma unroll
          for (int c4 = 0; c4 < D / 32; ++c4) {
            uint32_t v[32];
            tmem_ld32(tO + c4 * 32, v);
            tmem_wait_ld();
#pragma unroll
            for (int i = 0; i < 32; ++i) v[i] = __float_as_uint(__uint_as_float(v[i]) * f);
            tmem_st32(tO + c4 * 32, v);
          }
          tmem_wait_st();
          l *= f;
        }
      }
      l += rowsum;
      m_run = m_new;
      // row r of P: 8 chunks of 16 bytes, chunk index XOR (r mod 8) (128-byte swizzle)
#pragma unroll
      for (int ch = 0; ch < BLOCK_N / 16; ++ch) {
        uint4* dst = reinterpret_cast<uint4*>(prow + ((ch ^ (r & 7)) << 4));
        *dst = make_uint4(pk[4 * ch], pk[4 * ch + 1], pk[4 * ch + 2], pk[4 * ch + 3]);
      }
      fence_proxy_async_smem();
      tc_fence_before();
      mbar_arrive(BAR(B_PFULL + t));
    }
    if (ok) {
      ok = mbar_wait(BAR(B_ODONE + t), (nkv - 1) & 1, tlim, abort_flag, args.err);
      if (__all_sync(0xFFFFFFFFu, ok)) {
        tc_fence_after();
        const int row = q_row0 + t * BLOCK_M + r;
        const bool valid = row < seq_len;
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
                                 int rows_per_slab, int slabs, dim3 grid, cudaStream_t stream) {
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
