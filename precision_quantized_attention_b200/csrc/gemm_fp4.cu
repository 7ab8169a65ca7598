// gemm_fp4.cu -- per-block FP4 GEMM (E2M1 values, an E4M3 scale per 16 elements, a per-tensor
// FP32 scale) for sm_100a: TMA + block-scaled tcgen05.mma (kind::mxf4nvf4) + TMEM.
//
// The linear layers of the transformer block in the blog's per-block FP4 post-training
// quantization (NVIDIA developer blog "Optimizing FLUX.1 Kontext for Image Editing with
// Low-Precision Quantization", "Workflow and quantization": the quant config takes per-tensor
// FP8 or per-block FP4; Fig. 3 puts the GEMMs and the SDPA at about 75 % of the block's time).
// Operands are in the format qattn_quantize_fp4_block writes: X [M, K] and W [N, K] as packed
// E2M1 codes (element 2i in the low nibble of byte i, rows K / 2 bytes long), E4M3 block scales
// [rows, K / 16] row-major (block b covers K elements 16 b .. 16 b + 15), and a per-tensor scale
// s_g.  Computed here:
//   Y[m, n] = bf16( (sum_k val(x[m,k]) val(sx[m,k/16]) val(w[n,k]) val(sw[n,k/16])) * fl32(sg_x sg_w) )
// with the block-scaled products accumulated in FP32 by the tensor cores.
//
// One persistent kernel, 320 threads, one SM per 128 x 128 output tile (m-fastest order):
//   warp 0      TMA producer: per 256-element (128-byte) K block the X tile (128 rows) and the W
//               tile (128 rows), 128-byte swizzle, and the rows' 16 block scales each (two
//               128 x 16-byte boxes of the row-major scale arrays), into a 6-stage ring.
//   warp 1      MMA issuer (one thread) and TMEM owner: four K = 64 block-scaled MMAs per K
//               block into one of two 128-column FP32 accumulators.
//   warps 2-5   epilogue: thread = output row = TMEM lane; 32 columns at a time, scaled by
//               sg_x sg_w, rounded to bf16, stored.
//   warps 6-9   scale factors: per K block, each warp copies the stage's block scales from
//               shared memory into its own lane quarter of a 6-stage TMEM ring (32 columns a
//               stage: X's, then W's), as the block-scaled MMA reads them: row r's four factors of
//               a K = 64 step form the word at lane r % 32, column (step * 4 + r / 32), replicated
//               in every lane quarter.
// The MMA commit of a K block frees both its shared-memory stage and its scale-factor stage.
// All waits are bounded (a global-timer limit).
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <cstdint>

#include "device_once.h"
#include "tensor_map.h"
#include "launch.h"
#include "sm100_ptx.cuh"

namespace qattn {

namespace gemm4 {
constexpr int BM = 128;                  // output rows per tile (= TMEM lanes)
constexpr int BN = 128;                  // output columns per tile (MMA N)
constexpr int BK = 256;                  // K elements per stage (128 bytes of E2M1 per row)
constexpr int BKB = BK / 2;              // bytes per row per stage
#ifndef QATTN_FP4_STAGES
#define QATTN_FP4_STAGES 6
#endif
constexpr int STAGES = QATTN_FP4_STAGES;
constexpr int THREADS = 320;
constexpr int WARP_LOAD = 0, WARP_MMA = 1, WARP_SF0 = 6;   // warps 2-5: epilogue
constexpr int TILE_A = BM * BKB;         // 16 KB
constexpr int TILE_B = BN * BKB;         // 16 KB
constexpr int OFF_A = 0;
constexpr int OFF_B = OFF_A + STAGES * TILE_A;
constexpr int TILE_SF = 128 * 16;        // 2 KB: 128 rows x 16 block scales
constexpr int OFF_SFX = OFF_B + STAGES * TILE_B;
constexpr int OFF_SFW = OFF_SFX + STAGES * TILE_SF;
constexpr int STAGE_TX = TILE_A + TILE_B + 2 * TILE_SF;
constexpr int OFF_BAR = OFF_SFW + STAGES * TILE_SF;
// barriers: full[STAGES] (TMA), sf_full[STAGES], empty[STAGES], acc_full[2], acc_empty[2], drain
constexpr int B_FULL = 0, B_SFFULL = STAGES, B_EMPTY = 2 * STAGES, B_ACCF = 3 * STAGES;
constexpr int B_ACCE = B_ACCF + 2, B_DRAIN = B_ACCE + 2, NBARS = B_DRAIN + 1;
constexpr int OFF_TMEM = OFF_BAR + 8 * NBARS;
constexpr int OFF_ABORT = OFF_TMEM + 4;
constexpr int BYTES = OFF_ABORT + 4;
constexpr int ALLOC = BYTES + 1024;      // slack for 1024-byte alignment
static_assert(TILE_A % 1024 == 0 && TILE_B % 1024 == 0, "alignment");
static_assert(ALLOC <= 227 * 1024, "shared memory per CTA");
// TMEM: accumulators at columns 0 and BN; scale-factor stage s at SF0 + 32 s (16 columns of X's
// factors, 16 of W's: K = 64 step kk, row group c = r / 32 in column kk * 4 + c)
constexpr uint32_t SF0 = 2 * BN;
constexpr uint32_t SF_COLS = 32;
constexpr uint32_t TMEM_COLS = 512;
static_assert(SF0 + STAGES * SF_COLS <= TMEM_COLS, "TMEM budget");
constexpr uint32_t IDESC = idesc_mxf4_e2m1(BM, BN);
}  // namespace gemm4

struct Gemm4Args {
  int M, N, K;
  const float* sg_x;
  const float* sg_w;
  __nv_bfloat16* y;
  int* err;
  uint64_t timeout_ns;
};

// 32 FP32 accumulator columns of one row, scaled, rounded to bf16 and stored (four 16-byte
// stores; y 16-byte aligned).
__device__ __forceinline__ void store_bf16_32(__nv_bfloat16* y, const uint32_t (&v)[32], float scale) {
  uint32_t packed[16];
#pragma unroll
  for (int e = 0; e < 16; ++e) {
    const __nv_bfloat162 b2 = __floats2bfloat162_rn(__uint_as_float(v[2 * e]) * scale,
                                                    __uint_as_float(v[2 * e + 1]) * scale);
    packed[e] = *reinterpret_cast<const uint32_t*>(&b2);
  }
  uint4* dst = reinterpret_cast<uint4*>(y);
#pragma unroll
  for (int e = 0; e < 4; ++e)
    dst[e] = make_uint4(packed[4 * e], packed[4 * e + 1], packed[4 * e + 2], packed[4 * e + 3]);
}

__global__ void __launch_bounds__(gemm4::THREADS, 1)
    k_gemm_fp4(const __grid_constant__ CUtensorMap tm_a, const __grid_constant__ CUtensorMap tm_b,
               const __grid_constant__ CUtensorMap tm_sa, const __grid_constant__ CUtensorMap tm_sb,
               const __grid_constant__ Gemm4Args args) {
  using namespace gemm4;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_u32 = smem_u32(smem_raw);
  const uint32_t base_u32 = (raw_u32 + 1023u) & ~1023u;
  uint8_t* base = smem_raw + (base_u32 - raw_u32);
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  const int tiles_m = (args.M + BM - 1) / BM;
  const int tiles = tiles_m * ((args.N + BN - 1) / BN);
  const int kblocks = args.K / BK;
  if (static_cast<int>(blockIdx.x) >= tiles) return;   // uniform over the CTA

  const uint32_t bar0 = base_u32 + OFF_BAR;
  auto BAR = [&](int i) { return bar0 + 8u * static_cast<uint32_t>(i); };
  volatile int* abort_flag = reinterpret_cast<volatile int*>(base + OFF_ABORT);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(base + OFF_TMEM);
  if (threadIdx.x == 0) {
    for (int i = 0; i < STAGES; ++i) {
      mbar_init(BAR(B_FULL + i), 1);
      mbar_init(BAR(B_SFFULL + i), 4);           // one arrival per scale-factor warp
      mbar_init(BAR(B_EMPTY + i), 1);
    }
    for (int b = 0; b < 2; ++b) { mbar_init(BAR(B_ACCF + b), 1); mbar_init(BAR(B_ACCE + b), 128); }
    mbar_init(BAR(B_DRAIN), 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == WARP_MMA) {
    tmem_alloc(base_u32 + OFF_TMEM, TMEM_COLS);
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
      tma_prefetch_desc(&tm_a);
      tma_prefetch_desc(&tm_b);
      tma_prefetch_desc(&tm_sa);
      tma_prefetch_desc(&tm_sb);
      int u = 0;                                   // K blocks issued (ring position)
      bool ok = true;
      for (int t = blockIdx.x; ok && t < tiles; t += gridDim.x) {
        const int m0 = (t % tiles_m) * BM, n0 = (t / tiles_m) * BN;
        (void)QATTN_IN_BOUNDS(args.err, m0 < args.M && n0 < args.N);
        for (int kb = 0; kb < kblocks; ++kb, ++u) {
          const int s = u % STAGES;
          if (u >= STAGES &&
              !mbar_wait(BAR(B_EMPTY + s), ((u / STAGES) - 1) & 1, tlim, abort_flag, args.err)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(BAR(B_FULL + s), STAGE_TX);
          tma_load_2d(base_u32 + OFF_A + s * TILE_A, &tm_a, BAR(B_FULL + s), kb * BKB, m0);
          tma_load_2d(base_u32 + OFF_B + s * TILE_B, &tm_b, BAR(B_FULL + s), kb * BKB, n0);
          tma_load_2d(base_u32 + OFF_SFX + s * TILE_SF, &tm_sa, BAR(B_FULL + s), kb * 16, m0);
          tma_load_2d(base_u32 + OFF_SFW + s * TILE_SF, &tm_sb, BAR(B_FULL + s), kb * 16, n0);
        }
      }
      // drain: every issued load has landed before the CTA may exit (instant when healthy)
      for (int j = u - 1; j >= 0 && j >= u - STAGES; --j)
        mbar_drain(BAR(B_FULL + j % STAGES), (j / STAGES) & 1, tlim);
    }
  } else if (warp >= WARP_SF0) {
    // ======================= scale factors into TMEM =======================
    // The stage's factors landed with its tiles (full barrier); the MMAs that read this TMEM
    // stage before completed before the producer could refill the shared-memory stage.
    const int quarter = warp & 3;                  // this warp's TMEM lane quarter
    const uint32_t lane_off = static_cast<uint32_t>(quarter * 32) << 16;
    int u = 0;
    bool ok = true;
    for (int t = blockIdx.x; ok && t < tiles; t += gridDim.x) {
      for (int kb = 0; kb < kblocks; ++kb, ++u) {
        const int s = u % STAGES;
        ok = mbar_wait(BAR(B_FULL + s), (u / STAGES) & 1, tlim, abort_flag, args.err);
        if (!__all_sync(0xFFFFFFFFu, ok)) { ok = false; break; }
        // row group c of the tile: rows 32 c + lane; 16 factors (16 bytes) of the K block each
        const uint32_t fx0 = base_u32 + OFF_SFX + s * TILE_SF + 16u * lane;
        const uint32_t fw0 = base_u32 + OFF_SFW + s * TILE_SF + 16u * lane;
        uint32_t v[32];
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          const uint4 fx = ld_shared_v4(fx0 + 512u * c), fw = ld_shared_v4(fw0 + 512u * c);
          v[c] = fx.x; v[4 + c] = fx.y; v[8 + c] = fx.z; v[12 + c] = fx.w;
          v[16 + c] = fw.x; v[20 + c] = fw.y; v[24 + c] = fw.z; v[28 + c] = fw.w;
        }
        tmem_st32(tmem + lane_off + SF0 + static_cast<uint32_t>(s) * SF_COLS, v);
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(BAR(B_SFFULL + s));
      }
    }
  } else if (warp == WARP_MMA) {
    // ======================= MMA issuer =======================
    if (lane == 0) {
      int u = 0, i = 0;                            // K blocks consumed; tiles of this CTA
      bool ok = true;
      for (int t = blockIdx.x; ok && t < tiles; t += gridDim.x, ++i) {
        const int ab = i & 1;                      // accumulator of this tile
        if (i >= 2)
          ok = mbar_wait(BAR(B_ACCE + ab), ((i >> 1) - 1) & 1, tlim, abort_flag, args.err);
        if (!ok) break;
        tc_fence_after();
        const uint32_t acc = tmem + static_cast<uint32_t>(ab * BN);
        for (int kb = 0; kb < kblocks; ++kb, ++u) {
          const int s = u % STAGES;
          ok = mbar_wait(BAR(B_FULL + s), (u / STAGES) & 1, tlim, abort_flag, args.err) &&
               mbar_wait(BAR(B_SFFULL + s), (u / STAGES) & 1, tlim, abort_flag, args.err);
          if (!ok) break;
          tc_fence_after();
          const uint32_t a_s = base_u32 + OFF_A + s * TILE_A;
          const uint32_t b_s = base_u32 + OFF_B + s * TILE_B;
          const uint32_t sf = tmem + SF0 + static_cast<uint32_t>(s) * SF_COLS;
#pragma unroll
          for (int kk = 0; kk < BK / 64; ++kk) {
            // K-major rows of 128 bytes, 128-byte swizzle, 8-row atoms (SBO 1024); a K = 64 step
            // is 32 bytes of packed E2M1
            const uint64_t da = smem_desc(a_s + kk * 32, 16, 1024, 2u);
            const uint64_t db = smem_desc(b_s + kk * 32, 16, 1024, 2u);
            mma_mxf4_ss(acc, da, db, IDESC, sf + kk * 4, sf + 16 + kk * 4, (kb > 0 || kk > 0) ? 1u : 0u);
          }
          mma_commit(BAR(B_EMPTY + s));           // stage and factors free once these complete
        }
        if (ok) mma_commit(BAR(B_ACCF + ab));     // accumulator complete
      }
      mma_commit(BAR(B_DRAIN));
      mbar_drain(BAR(B_DRAIN), 0, tlim);
    }
  } else {
    // ======================= epilogue warps =======================
    const int quarter = warp & 3;
    const int r = quarter * 32 + lane;             // row within the tile
    const uint32_t lane_off = static_cast<uint32_t>(quarter * 32) << 16;
    const float scale = __ldg(args.sg_x) * __ldg(args.sg_w);
    int i = 0;
    for (int t = blockIdx.x; t < tiles; t += gridDim.x, ++i) {
      const int ab = i & 1;
      const bool ok = mbar_wait(BAR(B_ACCF + ab), (i >> 1) & 1, tlim, abort_flag, args.err);
      if (!__all_sync(0xFFFFFFFFu, ok)) break;
      tc_fence_after();
      const int m = (t % tiles_m) * BM + r, n0 = (t / tiles_m) * BN;
      const uint32_t acc = tmem + lane_off + static_cast<uint32_t>(ab * BN);
#pragma unroll 1
      for (int c = 0; c < BN / 32; ++c) {
        uint32_t v[32];
        tmem_ld32(acc + c * 32, v);
        tmem_wait_ld();
        const size_t off = static_cast<size_t>(m) * args.N + n0 + c * 32;
        // N % 32 == 0: a 32-column chunk is all in or all out
        if (m < args.M && n0 + c * 32 < args.N &&
            QATTN_IN_BOUNDS(args.err, off + 32 <= static_cast<size_t>(args.M) * args.N))
          store_bf16_32(args.y + off, v, scale);
      }
      tc_fence_before();
      mbar_arrive(BAR(B_ACCE + ab));               // accumulator read out
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == WARP_MMA) {
    tc_fence_after();
    tmem_dealloc(tmem, TMEM_COLS);
  }
}

// ---------------------------------------------------------------------------------------------
// Pair kernel (M > 128): two SMs (a cluster of two CTAs) on one 256 x 192 output tile.
//
// One tcgen05.mma.cta_group::2.kind::mxf4nvf4 with M = 256, N = 192 reads 128 rows of X and 96
// rows of W from each CTA's shared memory and leaves 128 rows x 192 columns of the FP32 tile in
// each CTA's TMEM.  Each CTA's TMEM also holds the block scales of its own 128 rows of X and of
// all 192 rows of W (the MMA reads W's factors of the whole N = 192 from each CTA: N / 32 = 6
// consecutive columns per K = 64 step), in the one-SM layout.  Per K block an SM stages 28 KB
// of operands (not 32 KB as on one SM for a third less MMA work).  TMEM per CTA: two
// 192-column accumulators and a 3-slot factor ring of 40 columns (16 of X's factors, 24 of W's)
// fit in the 512 columns, which is why N is 192 and not 256; the shared-memory ring has 6
// stages, the factor ring 3 slots (slot u % 3 is refilled once the MMAs of step u - 3 completed).
//   warp 0 (both CTAs)  TMA producer: its halves of X and W counted on the leading CTA's `full`
//                       barrier; the block scales of its own X rows and of the tile's 192 W rows
//                       (two boxes, no pair form) on its own `sf_data` barrier.
//   warp 1              TMEM owner in both CTAs; in the leading CTA, one thread issues the MMAs
//                       and commits `empty` / `acc_full` to the barriers of both CTAs.
//   warps 2-5 (both)    epilogue of the CTA's 128 rows; each warp arrives once per tile on the
//                       leading CTA's `acc_empty` (8 arrivals release an accumulator).
//   warps 6-9 (both)    scale factors: once a stage's boxes landed and the factor slot is free,
//                       copy them into the CTA's TMEM ring and arrive on the leading CTA's
//                       `sf_full` (8 arrivals).
// Both CTAs reach the two cluster barriers (after set-up, before the TMEM free) on every path:
// every wait in between is bounded.
// ---------------------------------------------------------------------------------------------
namespace gemm4p {
#ifndef QATTN_FP4_PAIR_N
#define QATTN_FP4_PAIR_N 192
#endif
constexpr int BM = 256;                  // output rows per tile pair (128 per CTA)
constexpr int BN = QATTN_FP4_PAIR_N;     // output columns per tile (MMA N; BN / 2 W rows per CTA)
constexpr int BK = 256;                  // K elements per stage (128 bytes per row)
constexpr int BKB = BK / 2;
constexpr int STAGES = 6;                // shared-memory ring
constexpr int GW = BN / 32;              // W row groups per K = 64 step (TMEM columns of W's factors)
constexpr int THREADS = 320;
constexpr int WARP_LOAD = 0, WARP_MMA = 1, WARP_SF0 = 6;   // warps 2-5: epilogue
constexpr int ROWS_A = BM / 2, ROWS_B = BN / 2;             // operand rows per CTA
constexpr int TILE_A = ROWS_A * BKB;     // 16 KB
constexpr int TILE_B = ROWS_B * BKB;     // 12 KB
constexpr int TILE_SFA = ROWS_A * 16;    // 2 KB: this CTA's X rows' factors of the K block
constexpr int TILE_SFB = BN * 16;        // 3 KB: all of the tile's W rows' factors
constexpr int OFF_A = 0;
constexpr int OFF_B = OFF_A + STAGES * TILE_A;
constexpr int OFF_SFA = OFF_B + STAGES * TILE_B;
constexpr int OFF_SFB = OFF_SFA + STAGES * TILE_SFA;
constexpr int OFF_BAR = OFF_SFB + STAGES * TILE_SFB;
constexpr int B_FULL = 0, B_SFDATA = STAGES, B_SFFULL = 2 * STAGES, B_EMPTY = 3 * STAGES;
constexpr int B_ACCF = 4 * STAGES, B_ACCE = B_ACCF + 2, B_DRAIN = B_ACCE + 2, NBARS = B_DRAIN + 1;
constexpr int OFF_TMEM = OFF_BAR + 8 * NBARS;
constexpr int OFF_ABORT = OFF_TMEM + 4;
constexpr int BYTES = OFF_ABORT + 4;
constexpr int ALLOC = BYTES + 1024;
static_assert(TILE_A % 1024 == 0 && TILE_B % 1024 == 0 && OFF_SFA % 1024 == 0, "alignment");
static_assert(TILE_SFB % 128 == 0, "scale boxes stay 128-byte aligned");
static_assert(ALLOC <= 227 * 1024, "shared memory per CTA");
// factor slot f at SF0 + SF_COLS f: X's factors of step kk in column kk * 4 + c (c < 4), W's in
// column 16 + kk * GW + c (c < GW), c = row / 32
constexpr uint32_t SF0 = 2 * BN;
constexpr uint32_t SF_COLS = 16 + 4 * GW;
constexpr uint32_t TMEM_COLS = 512;
constexpr int SF_SLOTS = (TMEM_COLS - SF0) / SF_COLS < STAGES ? (TMEM_COLS - SF0) / SF_COLS : STAGES;
static_assert(SF_SLOTS >= 2 && SF0 + SF_SLOTS * SF_COLS <= TMEM_COLS, "TMEM budget");
static_assert(BN % 64 == 0 && BN <= 256, "W rows per CTA: whole 32-row groups");
static_assert(SF_COLS == 32 || SF_COLS == 40, "a slot is written with one 32-column store (+ 8)");
constexpr uint32_t STAGE_TX = 2u * (TILE_A + TILE_B);     // operand bytes of both CTAs per stage
constexpr uint32_t IDESC = idesc_mxf4_e2m1(BM, BN);
}  // namespace gemm4p

__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(gemm4p::THREADS, 1)
    k_gemm_fp4_pair(const __grid_constant__ CUtensorMap tm_a, const __grid_constant__ CUtensorMap tm_b,
                    const __grid_constant__ CUtensorMap tm_sa, const __grid_constant__ CUtensorMap tm_sb,
                    const __grid_constant__ Gemm4Args args) {
  using namespace gemm4p;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_u32 = smem_u32(smem_raw);
  const uint32_t base_u32 = (raw_u32 + 1023u) & ~1023u;   // the same offset in both CTAs
  uint8_t* base = smem_raw + (base_u32 - raw_u32);
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();                  // 0 leads the pair
  const bool leader = rank == 0;
  const int pair = static_cast<int>(blockIdx.x >> 1), npairs = static_cast<int>(gridDim.x >> 1);

  const int tiles_m = (args.M + BM - 1) / BM;
  const int tiles = tiles_m * ((args.N + BN - 1) / BN);   // the host launches <= tiles pairs
  const int kblocks = args.K / BK;

  const uint32_t bar0 = base_u32 + OFF_BAR;
  auto BAR = [&](int i) { return bar0 + 8u * static_cast<uint32_t>(i); };
  volatile int* abort_flag = reinterpret_cast<volatile int*>(base + OFF_ABORT);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(base + OFF_TMEM);
  if (threadIdx.x == 0) {
    for (int i = 0; i < STAGES; ++i) {
      mbar_init(BAR(B_FULL + i), 1);
      mbar_init(BAR(B_SFDATA + i), 1);
      mbar_init(BAR(B_SFFULL + i), 8);             // 4 factor warps x 2 CTAs (leading CTA's)
      mbar_init(BAR(B_EMPTY + i), 1);
    }
    for (int b = 0; b < 2; ++b) { mbar_init(BAR(B_ACCF + b), 1); mbar_init(BAR(B_ACCE + b), 8); }
    mbar_init(BAR(B_DRAIN), 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == WARP_MMA) {
    tmem_alloc_pair(base_u32 + OFF_TMEM, TMEM_COLS);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  cluster_sync();                      // barriers of both CTAs initialised, TMEM allocated
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint64_t tlim = args.timeout_ns;

  if (warp == WARP_LOAD) {
    // ======================= TMA producer (both CTAs) =======================
    if (lane == 0) {
      tma_prefetch_desc(&tm_a);
      tma_prefetch_desc(&tm_b);
      tma_prefetch_desc(&tm_sa);
      tma_prefetch_desc(&tm_sb);
      int u = 0;
      bool ok = true;
      for (int t = pair; ok && t < tiles; t += npairs) {
        const int m0 = (t % tiles_m) * BM + static_cast<int>(rank) * ROWS_A;
        const int n0 = (t / tiles_m) * BN + static_cast<int>(rank) * ROWS_B;
        (void)QATTN_IN_BOUNDS(args.err, (t % tiles_m) * BM < args.M && (t / tiles_m) * BN < args.N);
        for (int kb = 0; kb < kblocks; ++kb, ++u) {
          const int s = u % STAGES;
          if (u >= STAGES &&
              !mbar_wait(BAR(B_EMPTY + s), ((u / STAGES) - 1) & 1, tlim, abort_flag, args.err)) {
            ok = false;
            break;
          }
          if (leader) mbar_arrive_expect_tx(BAR(B_FULL + s), STAGE_TX);
          const uint32_t full_lead = mapa_shared(BAR(B_FULL + s), 0);
          tma_load_2d_pair(base_u32 + OFF_A + s * TILE_A, &tm_a, full_lead, kb * BKB, m0);
          tma_load_2d_pair(base_u32 + OFF_B + s * TILE_B, &tm_b, full_lead, kb * BKB, n0);
          mbar_arrive_expect_tx(BAR(B_SFDATA + s), TILE_SFA + TILE_SFB);
          tma_load_2d(base_u32 + OFF_SFA + s * TILE_SFA, &tm_sa, BAR(B_SFDATA + s), kb * 16, m0);
          tma_load_2d(base_u32 + OFF_SFB + s * TILE_SFB, &tm_sb, BAR(B_SFDATA + s), kb * 16,
                      (t / tiles_m) * BN);
        }
      }
      // the MMAs have released every stage this CTA filled: its loads have landed and no
      // commit from the leading CTA is still on its way here (instant when healthy)
      for (int j = u - 1; j >= 0 && j >= u - STAGES; --j) {
        mbar_drain(BAR(B_EMPTY + j % STAGES), (j / STAGES) & 1, tlim);
        mbar_drain(BAR(B_SFDATA + j % STAGES), (j / STAGES) & 1, tlim);
      }
    }
  } else if (warp >= WARP_SF0) {
    // ======================= scale factors into TMEM (both CTAs) =======================
    const int quarter = warp & 3;
    const uint32_t lane_off = static_cast<uint32_t>(quarter * 32) << 16;
    int u = 0;
    bool ok = true;
    for (int t = pair; ok && t < tiles; t += npairs) {
      for (int kb = 0; kb < kblocks; ++kb, ++u) {
        const int s = u % STAGES, f = u % SF_SLOTS;
        ok = mbar_wait(BAR(B_SFDATA + s), (u / STAGES) & 1, tlim, abort_flag, args.err);
        // factor slot f was last read by the MMAs of step u - SF_SLOTS: their commit arrived on
        // that step's `empty` barrier (in both CTAs)
        if (ok && u >= SF_SLOTS) {
          const int v = u - SF_SLOTS;
          ok = mbar_wait(BAR(B_EMPTY + v % STAGES), (v / STAGES) & 1, tlim, abort_flag, args.err);
        }
        if (!__all_sync(0xFFFFFFFFu, ok)) { ok = false; break; }
        // row group c: rows 32 c + lane of this CTA's X rows (c < 4) and of the W rows (c < GW)
        const uint32_t fa0 = base_u32 + OFF_SFA + s * TILE_SFA + 16u * lane;
        const uint32_t fb0 = base_u32 + OFF_SFB + s * TILE_SFB + 16u * lane;
        uint32_t v[40];                            // the slot's columns, in order (SF_COLS used)
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          const uint4 fa = ld_shared_v4(fa0 + 512u * c);
          v[c] = fa.x; v[4 + c] = fa.y; v[8 + c] = fa.z; v[12 + c] = fa.w;
        }
#pragma unroll
        for (int c = 0; c < GW; ++c) {
          const uint4 fb = ld_shared_v4(fb0 + 512u * c);
          v[16 + c] = fb.x; v[16 + GW + c] = fb.y; v[16 + 2 * GW + c] = fb.z; v[16 + 3 * GW + c] = fb.w;
        }
        const uint32_t slot = tmem + lane_off + SF0 + static_cast<uint32_t>(f) * SF_COLS;
        tmem_st32(slot, *reinterpret_cast<const uint32_t(*)[32]>(v));
        if constexpr (SF_COLS > 32) tmem_st8(slot + 32, *reinterpret_cast<const uint32_t(*)[8]>(v + 32));
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive_cluster(mapa_shared(BAR(B_SFFULL + s), 0));
      }
    }
  } else if (warp == WARP_MMA) {
    // ======================= MMA issuer (leading CTA) =======================
    if (leader && lane == 0) {
      const uint32_t peer = rank ^ 1u;
      int u = 0, i = 0;
      bool ok = true;
      for (int t = pair; ok && t < tiles; t += npairs, ++i) {
        const int ab = i & 1;
        if (i >= 2)
          ok = mbar_wait(BAR(B_ACCE + ab), ((i >> 1) - 1) & 1, tlim, abort_flag, args.err);
        if (!ok) break;
        tc_fence_after();
        const uint32_t acc = tmem + static_cast<uint32_t>(ab * BN);
        for (int kb = 0; kb < kblocks; ++kb, ++u) {
          const int s = u % STAGES;
          ok = mbar_wait(BAR(B_FULL + s), (u / STAGES) & 1, tlim, abort_flag, args.err) &&
               mbar_wait(BAR(B_SFFULL + s), (u / STAGES) & 1, tlim, abort_flag, args.err);
          if (!ok) break;
          tc_fence_after();
          const uint32_t a_s = base_u32 + OFF_A + s * TILE_A;
          const uint32_t b_s = base_u32 + OFF_B + s * TILE_B;
          const uint32_t sf = tmem + SF0 + static_cast<uint32_t>(u % SF_SLOTS) * SF_COLS;
#pragma unroll
          for (int kk = 0; kk < BK / 64; ++kk) {
            const uint64_t da = smem_desc(a_s + kk * 32, 16, 1024, 2u);
            const uint64_t db = smem_desc(b_s + kk * 32, 16, 1024, 2u);
            mma_mxf4_ss_pair(acc, da, db, IDESC, sf + kk * 4, sf + 16 + kk * GW,
                             (kb > 0 || kk > 0) ? 1u : 0u);
          }
          mma_commit_pair(BAR(B_EMPTY + s));                      // stage free in both CTAs
          mma_commit_pair(mapa_shared(BAR(B_EMPTY + s), peer));
        }
        if (ok) {
          mma_commit_pair(BAR(B_ACCF + ab));                      // accumulator complete
          mma_commit_pair(mapa_shared(BAR(B_ACCF + ab), peer));
        }
      }
      mma_commit_pair(BAR(B_DRAIN));
      mbar_drain(BAR(B_DRAIN), 0, tlim);
    }
  } else {
    // ======================= epilogue warps (both CTAs) =======================
    const int quarter = warp & 3;
    const int r = quarter * 32 + lane;
    const uint32_t lane_off = static_cast<uint32_t>(quarter * 32) << 16;
    const float scale = __ldg(args.sg_x) * __ldg(args.sg_w);
    int i = 0;
    for (int t = pair; t < tiles; t += npairs, ++i) {
      const int ab = i & 1;
      const bool ok = mbar_wait(BAR(B_ACCF + ab), (i >> 1) & 1, tlim, abort_flag, args.err);
      if (!__all_sync(0xFFFFFFFFu, ok)) break;
      tc_fence_after();
      const int m = (t % tiles_m) * BM + static_cast<int>(rank) * ROWS_A + r;
      const int n0 = (t / tiles_m) * BN;
      const uint32_t acc = tmem + lane_off + static_cast<uint32_t>(ab * BN);
#pragma unroll 1
      for (int c = 0; c < BN / 32; ++c) {
        uint32_t v[32];
        tmem_ld32(acc + c * 32, v);
        tmem_wait_ld();
        const size_t off = static_cast<size_t>(m) * args.N + n0 + c * 32;
        if (m < args.M && n0 + c * 32 < args.N &&
            QATTN_IN_BOUNDS(args.err, off + 32 <= static_cast<size_t>(args.M) * args.N))
          store_bf16_32(args.y + off, v, scale);
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(mapa_shared(BAR(B_ACCE + ab), 0));   // read out
    }
  }

  tc_fence_before();
  cluster_sync();                      // no MMA, load or arrival of either CTA is outstanding
  if (warp == WARP_MMA) {
    tc_fence_after();
    tmem_dealloc_pair(tmem, TMEM_COLS);
  }
}

// ---------------------------------------------------------------------------------------------
// Host side
// ---------------------------------------------------------------------------------------------

// Packed E2M1 [rows, K / 2 bytes]; box of `box_rows` rows x 128 bytes, 128-byte swizzle; reads
// past the last row return zeros.
static bool make_map_e2m1(CUtensorMap* map, const void* ptr, int rows, int K, int box_rows) {
  EncodeTiledFn enc = encode_tiled_fn();
  if (!enc) return false;
  cuuint64_t dims[2] = {static_cast<cuuint64_t>(K / 2), static_cast<cuuint64_t>(rows)};
  cuuint64_t strides[1] = {static_cast<cuuint64_t>(K / 2)};
  cuuint32_t box[2] = {static_cast<cuuint32_t>(gemm4::BKB), static_cast<cuuint32_t>(box_rows)};
  cuuint32_t estr[2] = {1u, 1u};
  return enc(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(ptr), dims, strides, box,
             estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Block scales [rows, K / 16] bytes, row-major; box of `box_rows` rows x 16 bytes (one K block's
// factors), no swizzle; rows past the last read as zeros.
static bool make_map_scales(CUtensorMap* map, const void* ptr, int rows, int K, int box_rows) {
  EncodeTiledFn enc = encode_tiled_fn();
  if (!enc) return false;
  cuuint64_t dims[2] = {static_cast<cuuint64_t>(K / 16), static_cast<cuuint64_t>(rows)};
  cuuint64_t strides[1] = {static_cast<cuuint64_t>(K / 16)};
  cuuint32_t box[2] = {16u, static_cast<cuuint32_t>(box_rows)};
  cuuint32_t estr[2] = {1u, 1u};
  return enc(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(ptr), dims, strides, box,
             estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
             CU_TENSOR_MAP_L2_PROMOTION_L2_128B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

cudaError_t launch_gemm_fp4(const uint8_t* x, const uint8_t* sx, const float* sg_x, const uint8_t* w,
                            const uint8_t* sw, const float* sg_w, void* y, int M, int N, int K,
                            int* err, uint64_t timeout_ns, int num_sms, cudaStream_t stream) {
  Gemm4Args a;
  a.M = M;
  a.N = N;
  a.K = K;
  a.sg_x = sg_x;
  a.sg_w = sg_w;
  a.y = static_cast<__nv_bfloat16*>(y);
  a.err = err;
  a.timeout_ns = timeout_ns;
  CUtensorMap ma, mb, msa, msb;
  if (M > gemm4::BM && num_sms >= 2) {
    // pairs of SMs on 256 x 192 tiles
    using namespace gemm4p;
    if (!make_map_e2m1(&ma, x, M, K, ROWS_A) || !make_map_e2m1(&mb, w, N, K, ROWS_B) ||
        !make_map_scales(&msa, sx, M, K, ROWS_A) || !make_map_scales(&msb, sw, N, K, BN))
      return cudaErrorInvalidValue;
    static DeviceOnce configured_pair;
    const int set = configured_pair.get([] {
      return static_cast<int>(cudaFuncSetAttribute(k_gemm_fp4_pair,
                                                   cudaFuncAttributeMaxDynamicSharedMemorySize, ALLOC));
    });
    if (set != static_cast<int>(cudaSuccess)) return static_cast<cudaError_t>(set);
    static DeviceOnce resident_pairs;
    const int resident = resident_pairs.get([num_sms] {
      cudaLaunchConfig_t cfg = {};
      cfg.gridDim = dim3(static_cast<unsigned>(num_sms & ~1));
      cfg.blockDim = dim3(THREADS);
      cfg.dynamicSmemBytes = ALLOC;
      int n = 0;
      if (cudaOccupancyMaxActiveClusters(&n, k_gemm_fp4_pair, &cfg) != cudaSuccess || n <= 0) {
        cudaGetLastError();
        n = num_sms / 2;
      }
      return n;
    });
    const int tiles = ((M + BM - 1) / BM) * ((N + BN - 1) / BN);
    const int pairs = tiles < resident ? tiles : resident;
    k_gemm_fp4_pair<<<2 * pairs, THREADS, ALLOC, stream>>>(ma, mb, msa, msb, a);
    return cudaGetLastError();
  }
  if (!make_map_e2m1(&ma, x, M, K, gemm4::BM) || !make_map_e2m1(&mb, w, N, K, gemm4::BN) ||
      !make_map_scales(&msa, sx, M, K, gemm4::BM) || !make_map_scales(&msb, sw, N, K, gemm4::BN))
    return cudaErrorInvalidValue;
  static DeviceOnce configured;
  const int set = configured.get([] {
    return static_cast<int>(cudaFuncSetAttribute(k_gemm_fp4, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                                 gemm4::ALLOC));
  });
  if (set != static_cast<int>(cudaSuccess)) return static_cast<cudaError_t>(set);
  const int tiles = ((M + gemm4::BM - 1) / gemm4::BM) * ((N + gemm4::BN - 1) / gemm4::BN);
  const int grid = tiles < num_sms ? tiles : num_sms;
  k_gemm_fp4<<<grid, gemm4::THREADS, gemm4::ALLOC, stream>>>(ma, mb, msa, msb, a);
  return cudaGetLastError();
}

}  // namespace qattn
