// gemm_fp8.cu -- FP8 (E4M3) GEMM with per-tensor scales for sm_100a (TMA + tcgen05 + TMEM).
//
// The transformer block around the quantized attention: the NVIDIA developer blog "Optimizing
// FLUX.1 Kontext for Image Editing with Low-Precision Quantization" quantizes the block's
// linear layers (QKV and output projections, MLP) to FP8 with the same per-tensor FakeQuantize
// as the attention inputs ("Workflow and quantization"; Fig. 3 puts the GEMMs and the SDPA at
// about 75 % of the transformer's time).  Computed here:
//   Y[m, n] = bf16( (sum_k val(A8[m, k]) * val(B8[n, k])) * fl32(s_a * s_b) )
// with A8 [M, K] the E4M3 activations and B8 [N, K] the E4M3 weights, both K-contiguous
// (Y = X W^T), the products accumulated in FP32 on the tensor cores.
//
// Two persistent kernels, both 192 threads with the roles below: `k_gemm_fp8_pair` (M > 128)
// pairs two SMs on each 256 x 256 tile (see its own comment); `k_gemm_fp8` (M <= 128) runs one
// SM per 128 x 256 tile:
//   warp 0      TMA producer: per 128 x 256 output tile and per 128-byte K block, the A tile
//               (128 rows) and the B tile (256 rows), 128-byte swizzle, into a 4-stage ring.
//   warp 1      MMA issuer (one thread) and TMEM owner: tcgen05.mma.cta_group::1.kind::f8f6f4,
//               M = 128, N = 256, four K = 32 steps per K block, into one of two 256-column
//               FP32 accumulators in TMEM, so the next tile's MMAs overlap this tile's epilogue.
//   warps 2-5   epilogue: thread = output row = TMEM lane; 32 columns at a time from TMEM,
//               scaled, rounded to bf16 and stored (16-byte stores).
// Output tiles are visited m-fastest (CTAs in flight share the weight tile, the activation
// matrix stays in L2).  All waits are bounded (a global-timer limit).
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <cstdint>

#include "device_once.h"
#include "tensor_map.h"
#include "quant_math.cuh"
#include "launch.h"
#include "sm100_ptx.cuh"

namespace qattn {

namespace gemm {
constexpr int BM = 128;                  // output rows per tile (= TMEM lanes)
constexpr int BN = 256;                  // output columns per tile (MMA N)
constexpr int BK = 128;                  // K elements (bytes) per stage
constexpr int STAGES = 4;
constexpr int THREADS = 192;
constexpr int WARP_LOAD = 0, WARP_MMA = 1;                  // warps 2-5: epilogue
constexpr int TILE_A = BM * BK;          // 16 KB
constexpr int TILE_B = BN * BK;          // 32 KB
constexpr int OFF_A = 0;
constexpr int OFF_B = OFF_A + STAGES * TILE_A;
constexpr int OFF_BAR = OFF_B + STAGES * TILE_B;
// barriers: full[STAGES], empty[STAGES], acc_full[2], acc_empty[2], drain
constexpr int NBARS = 2 * STAGES + 4 + 1;
constexpr int OFF_TMEM = OFF_BAR + 8 * NBARS;
constexpr int OFF_ABORT = OFF_TMEM + 4;
constexpr int BYTES = OFF_ABORT + 4;
constexpr int ALLOC = BYTES + 1024;      // slack for 1024-byte alignment
static_assert(TILE_A % 1024 == 0 && TILE_B % 1024 == 0, "alignment");
static_assert(ALLOC <= 227 * 1024, "shared memory per CTA");
constexpr uint32_t TMEM_COLS = 2 * BN;   // two accumulators
}  // namespace gemm

struct GemmArgs {
  int M, N, K;
  const float* s_a;
  const float* s_b;
  __nv_bfloat16* y;         // bf16 output, or nullptr (codes only)
  int* err;
  uint64_t timeout_ns;
  // optional per-tensor FP8 quantization of the bf16 output with a given (static) amax: codes
  // [M, N] = e4m3(fl32(y / s)), s = fl32(amax / 448) (amax == 0: s = 1) written to *scale_out
  uint8_t* codes;
  const float* amax;
  float* scale_out;
};

// Per-tensor scale of the epilogue's E4M3 codes from the given amax: (s, RN(1 / s), Markstein
// usable); ok = false (and a non-finite error recorded once) when the amax is not finite.
struct CodeScale {
  float s, r;
  bool fast, ok;
};
__device__ __forceinline__ CodeScale code_scale(const GemmArgs& a) {
  CodeScale cs{1.0f, 1.0f, true, false};
  if (!a.codes) return cs;
  const float amax = __ldg(a.amax);
  if (!(amax <= 3.402823466e38f)) {              // inf or NaN: no code is written
    if (blockIdx.x == 0 && threadIdx.x == 64) atomicExch(a.err, DEV_ERR_NONFINITE);
    return cs;
  }
  cs.s = amax == 0.0f ? 1.0f : __fdiv_rn(amax, 448.0f);
  cs.r = __frcp_rn(cs.s);
  cs.fast = markstein_ok(cs.s);
  cs.ok = true;
  if (blockIdx.x == 0 && threadIdx.x == 64) *a.scale_out = cs.s;
  return cs;
}

// Epilogue of 32 columns of one row: bf16 of acc * scale to y (if any) and, when the codes are
// requested, their E4M3 codes (the bf16 values quantized exactly as qattn_quantize_fp8 would).
__device__ __forceinline__ void epilogue32(const GemmArgs& a, const CodeScale& cs, const uint32_t (&v)[32],
                                           float scale, size_t off) {
  if (!QATTN_IN_BOUNDS(a.err, off + 32 <= static_cast<size_t>(a.M) * a.N)) return;
  uint32_t packed[16];
#pragma unroll
  for (int e = 0; e < 16; ++e) {
    const __nv_bfloat162 b2 = __floats2bfloat162_rn(__uint_as_float(v[2 * e]) * scale,
                                                    __uint_as_float(v[2 * e + 1]) * scale);
    packed[e] = *reinterpret_cast<const uint32_t*>(&b2);
  }
  if (a.y) {
    uint4* dst = reinterpret_cast<uint4*>(a.y + off);
#pragma unroll
    for (int e = 0; e < 4; ++e)
      dst[e] = make_uint4(packed[4 * e], packed[4 * e + 1], packed[4 * e + 2], packed[4 * e + 3]);
  }
  if (cs.ok) {
    uint32_t c[8];
    if (cs.fast) {
#pragma unroll
      for (int e = 0; e < 8; ++e) c[e] = quant4_e4m3<true>(packed[2 * e], packed[2 * e + 1], cs.s, cs.r);
    } else {
#pragma unroll
      for (int e = 0; e < 8; ++e) c[e] = quant4_e4m3<false>(packed[2 * e], packed[2 * e + 1], cs.s, cs.r);
    }
    uint4* dst = reinterpret_cast<uint4*>(a.codes + off);
    dst[0] = make_uint4(c[0], c[1], c[2], c[3]);
    dst[1] = make_uint4(c[4], c[5], c[6], c[7]);
  }
}

__global__ void __launch_bounds__(gemm::THREADS, 1)
    k_gemm_fp8(const __grid_constant__ CUtensorMap tm_a, const __grid_constant__ CUtensorMap tm_b,
               const __grid_constant__ GemmArgs args) {
  using namespace gemm;
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
  constexpr int B_FULL = 0, B_EMPTY = STAGES, B_ACCF = 2 * STAGES, B_ACCE = B_ACCF + 2;
  constexpr int B_DRAIN = B_ACCE + 2;
  volatile int* abort_flag = reinterpret_cast<volatile int*>(base + OFF_ABORT);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(base + OFF_TMEM);
  if (threadIdx.x == 0) {
    for (int i = 0; i < STAGES; ++i) { mbar_init(BAR(B_FULL + i), 1); mbar_init(BAR(B_EMPTY + i), 1); }
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
      int u = 0;                                   // K blocks issued (ring position)
      bool ok = true;
      for (int t = blockIdx.x; ok && t < tiles; t += gridDim.x) {
        const int m0 = (t % tiles_m) * BM, n0 = (t / tiles_m) * BN;
        // a tile starting past the output would be computed from zero fill: an index error
        (void)QATTN_IN_BOUNDS(args.err, m0 < args.M && n0 < args.N);
        for (int kb = 0; kb < kblocks; ++kb, ++u) {
          const int s = u % STAGES;
          if (u >= STAGES &&
              !mbar_wait(BAR(B_EMPTY + s), ((u / STAGES) - 1) & 1, tlim, abort_flag, args.err)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(BAR(B_FULL + s), TILE_A + TILE_B);
          tma_load_2d(base_u32 + OFF_A + s * TILE_A, &tm_a, BAR(B_FULL + s), kb * BK, m0);
          tma_load_2d(base_u32 + OFF_B + s * TILE_B, &tm_b, BAR(B_FULL + s), kb * BK, n0);
        }
      }
      // drain: every issued load has landed before the CTA may exit (instant when healthy)
      for (int j = u - 1; j >= 0 && j >= u - STAGES; --j)
        mbar_drain(BAR(B_FULL + j % STAGES), (j / STAGES) & 1, tlim);
    }
  } else if (warp == WARP_MMA) {
    // ======================= MMA issuer =======================
    if (lane == 0) {
      constexpr uint32_t IDESC = idesc_e4m3_f32(BM, BN, false);
      int u = 0, i = 0;                            // K blocks consumed; tiles of this CTA
      bool ok = true;
      for (int t = blockIdx.x; ok && t < tiles; t += gridDim.x, ++i) {
        const int ab = i & 1;                      // accumulator of this tile
        // the epilogue has read out the tile that used this accumulator two tiles ago
        if (i >= 2)
          ok = mbar_wait(BAR(B_ACCE + ab), ((i >> 1) - 1) & 1, tlim, abort_flag, args.err);
        if (!ok) break;
        tc_fence_after();
        const uint32_t acc = tmem + static_cast<uint32_t>(ab * BN);
        for (int kb = 0; kb < kblocks; ++kb, ++u) {
          const int s = u % STAGES;
          ok = mbar_wait(BAR(B_FULL + s), (u / STAGES) & 1, tlim, abort_flag, args.err);
          if (!ok) break;
          tc_fence_after();
          const uint32_t a_s = base_u32 + OFF_A + s * TILE_A;
          const uint32_t b_s = base_u32 + OFF_B + s * TILE_B;
#pragma unroll
          for (int kk = 0; kk < BK / 32; ++kk) {
            // K-major rows of 128 bytes, 128-byte swizzle, 8-row atoms (SBO 1024); 32-byte K steps
            const uint64_t da = smem_desc(a_s + kk * 32, 16, 1024, 2u);
            const uint64_t db = smem_desc(b_s + kk * 32, 16, 1024, 2u);
            mma_f8_ss(acc, da, db, IDESC, (kb > 0 || kk > 0) ? 1u : 0u);
          }
          mma_commit(BAR(B_EMPTY + s));           // stage free once these MMAs complete
        }
        if (ok) mma_commit(BAR(B_ACCF + ab));     // accumulator complete
      }
      mma_commit(BAR(B_DRAIN));
      mbar_drain(BAR(B_DRAIN), 0, tlim);
    }
  } else {
    // ======================= epilogue warps =======================
    const int quarter = warp & 3;                  // TMEM lane quarter of this warp
    const int r = quarter * 32 + lane;             // row within the tile
    const uint32_t lane_off = static_cast<uint32_t>(quarter * 32) << 16;
    const float scale = __ldg(args.s_a) * __ldg(args.s_b);
    const CodeScale cs = code_scale(args);
    int i = 0;
    for (int t = blockIdx.x; t < tiles; t += gridDim.x, ++i) {
      const int ab = i & 1;
      const bool ok = mbar_wait(BAR(B_ACCF + ab), (i >> 1) & 1, tlim, abort_flag, args.err);
      if (!__all_sync(0xFFFFFFFFu, ok)) break;
      tc_fence_after();
      const int m = (t % tiles_m) * BM + r, n0 = (t / tiles_m) * BN;
      const size_t row_off = static_cast<size_t>(m) * args.N + n0;
      const uint32_t acc = tmem + lane_off + static_cast<uint32_t>(ab * BN);
#pragma unroll 1
      for (int c = 0; c < BN / 32; ++c) {
        uint32_t v[32];
        tmem_ld32(acc + c * 32, v);
        tmem_wait_ld();
        if (m < args.M && n0 + c * 32 < args.N)     // N % 32 == 0: a chunk is all in or out
          epilogue32(args, cs, v, scale, row_off + c * 32);
      }
      tc_fence_before();
      mbar_arrive(BAR(B_ACCE + ab));               // accumulator read out
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == WARP_MMA) {
    tc_fence_after();
    tmem_dealloc(tmem, gemm::TMEM_COLS);
  }
}

// ---------------------------------------------------------------------------------------------
// Pair kernel: two SMs (a cluster of two CTAs) on one 256 x 256 output tile.
//
// One tcgen05.mma.cta_group::2 with M = 256, N = 256 reads 128 rows of A and 128 rows of B from
// each CTA's shared memory and leaves 128 rows x 256 columns of the FP32 tile in each CTA's TMEM.
// Per 128-byte K block an SM therefore stages 32 KB (not 48 KB as on one SM for the same MMA
// work), so six stages fit and cover more of the TMA refill latency.
//   warp 0 (both CTAs)  TMA producer for its own halves of A and B; completion is counted on the
//                       leading CTA's `full` barrier (64 KB per stage); waits on its own `empty`.
//   warp 1              TMEM owner in both CTAs; in the leading CTA, one thread issues the MMAs
//                       and commits `empty` / `acc_full` to the barriers of both CTAs.
//   warps 2-5 (both)    epilogue of the CTA's 128 rows; each warp arrives once per tile on the
//                       leading CTA's `acc_empty` (8 arrivals release an accumulator).
// Both CTAs reach the two cluster barriers (after set-up, before the TMEM free) on every path:
// every wait in between is bounded.
// ---------------------------------------------------------------------------------------------
namespace gemm2 {
constexpr int BM = 256;                  // output rows per tile pair (128 per CTA)
constexpr int BN = 256;                  // output columns per tile (MMA N; 128 B rows per CTA)
constexpr int BK = 128;
constexpr int STAGES = 6;
constexpr int THREADS = 192;
constexpr int WARP_LOAD = 0, WARP_MMA = 1;
constexpr int TILE_A = (BM / 2) * BK;    // 16 KB per CTA
constexpr int TILE_B = (BN / 2) * BK;    // 16 KB per CTA
constexpr int OFF_A = 0;
constexpr int OFF_B = OFF_A + STAGES * TILE_A;
constexpr int OFF_BAR = OFF_B + STAGES * TILE_B;
// barriers: full[STAGES] (leader), empty[STAGES], acc_full[2], acc_empty[2] (leader), drain
constexpr int NBARS = 2 * STAGES + 4 + 1;
constexpr int OFF_TMEM = OFF_BAR + 8 * NBARS;
constexpr int OFF_ABORT = OFF_TMEM + 4;
constexpr int BYTES = OFF_ABORT + 4;
constexpr int ALLOC = BYTES + 1024;
static_assert(TILE_A % 1024 == 0 && TILE_B % 1024 == 0, "alignment");
static_assert(ALLOC <= 227 * 1024, "shared memory per CTA");
constexpr uint32_t TMEM_COLS = 2 * BN;
constexpr uint32_t STAGE_TX = 2u * (TILE_A + TILE_B);   // bytes of both CTAs per stage
}  // namespace gemm2

__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(gemm2::THREADS, 1)
    k_gemm_fp8_pair(const __grid_constant__ CUtensorMap tm_a,
                    const __grid_constant__ CUtensorMap tm_b,
                    const __grid_constant__ GemmArgs args) {
  using namespace gemm2;
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
  constexpr int B_FULL = 0, B_EMPTY = STAGES, B_ACCF = 2 * STAGES, B_ACCE = B_ACCF + 2;
  constexpr int B_DRAIN = B_ACCE + 2;
  volatile int* abort_flag = reinterpret_cast<volatile int*>(base + OFF_ABORT);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(base + OFF_TMEM);
  if (threadIdx.x == 0) {
    for (int i = 0; i < STAGES; ++i) { mbar_init(BAR(B_FULL + i), 1); mbar_init(BAR(B_EMPTY + i), 1); }
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
      int u = 0;
      bool ok = true;
      for (int t = pair; ok && t < tiles; t += npairs) {
        const int m0 = (t % tiles_m) * BM + static_cast<int>(rank) * (BM / 2);
        const int n0 = (t / tiles_m) * BN + static_cast<int>(rank) * (BN / 2);
        // the pair's tile must start inside the output (a CTA's half may lie past it: zero fill)
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
          tma_load_2d_pair(base_u32 + OFF_A + s * TILE_A, &tm_a, full_lead, kb * BK, m0);
          tma_load_2d_pair(base_u32 + OFF_B + s * TILE_B, &tm_b, full_lead, kb * BK, n0);
        }
      }
      // the MMAs have released every stage this CTA filled: its loads have landed and no
      // commit from the leading CTA is still on its way here (instant when healthy)
      for (int j = u - 1; j >= 0 && j >= u - STAGES; --j)
        mbar_drain(BAR(B_EMPTY + j % STAGES), (j / STAGES) & 1, tlim);
    }
  } else if (warp == WARP_MMA) {
    // ======================= MMA issuer (leading CTA) =======================
    if (leader && lane == 0) {
      constexpr uint32_t IDESC = idesc_e4m3_f32(BM, BN, false);
      const uint32_t peer = rank ^ 1u;
      int u = 0, i = 0;
      bool ok = true;
      for (int t = pair; ok && t < tiles; t += npairs, ++i) {
        const int ab = i & 1;
        // both CTAs' epilogues have read out the tile that used this accumulator two tiles ago
        if (i >= 2)
          ok = mbar_wait(BAR(B_ACCE + ab), ((i >> 1) - 1) & 1, tlim, abort_flag, args.err);
        if (!ok) break;
        tc_fence_after();
        const uint32_t acc = tmem + static_cast<uint32_t>(ab * BN);
        for (int kb = 0; kb < kblocks; ++kb, ++u) {
          const int s = u % STAGES;
          ok = mbar_wait(BAR(B_FULL + s), (u / STAGES) & 1, tlim, abort_flag, args.err);
          if (!ok) break;
          tc_fence_after();
          const uint32_t a_s = base_u32 + OFF_A + s * TILE_A;
          const uint32_t b_s = base_u32 + OFF_B + s * TILE_B;
#pragma unroll
          for (int kk = 0; kk < BK / 32; ++kk) {
            const uint64_t da = smem_desc(a_s + kk * 32, 16, 1024, 2u);
            const uint64_t db = smem_desc(b_s + kk * 32, 16, 1024, 2u);
            mma_f8_ss_pair(acc, da, db, IDESC, (kb > 0 || kk > 0) ? 1u : 0u);
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
    const float scale = __ldg(args.s_a) * __ldg(args.s_b);
    const CodeScale cs = code_scale(args);
    int i = 0;
    for (int t = pair; t < tiles; t += npairs, ++i) {
      const int ab = i & 1;
      const bool ok = mbar_wait(BAR(B_ACCF + ab), (i >> 1) & 1, tlim, abort_flag, args.err);
      if (!__all_sync(0xFFFFFFFFu, ok)) break;
      tc_fence_after();
      const int m = (t % tiles_m) * BM + static_cast<int>(rank) * (BM / 2) + r;
      const int n0 = (t / tiles_m) * BN;
      const size_t row_off = static_cast<size_t>(m) * args.N + n0;
      const uint32_t acc = tmem + lane_off + static_cast<uint32_t>(ab * BN);
#pragma unroll 1
      for (int c = 0; c < BN / 32; ++c) {
        uint32_t v[32];
        tmem_ld32(acc + c * 32, v);
        tmem_wait_ld();
        if (m < args.M && n0 + c * 32 < args.N) epilogue32(args, cs, v, scale, row_off + c * 32);
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
    tmem_dealloc_pair(tmem, gemm2::TMEM_COLS);
  }
}

// ---------------------------------------------------------------------------------------------
// Host side
// ---------------------------------------------------------------------------------------------

// [rows, K] E4M3, K contiguous; box of `box_rows` rows x 128 bytes, 128-byte swizzle; reads past
// the last row return zeros.
static bool make_map_2d(CUtensorMap* map, const void* ptr, int rows, int K, int box_rows) {
  EncodeTiledFn enc = encode_tiled_fn();
  if (!enc) return false;
  cuuint64_t dims[2] = {static_cast<cuuint64_t>(K), static_cast<cuuint64_t>(rows)};
  cuuint64_t strides[1] = {static_cast<cuuint64_t>(K)};
  cuuint32_t box[2] = {static_cast<cuuint32_t>(gemm::BK), static_cast<cuuint32_t>(box_rows)};
  cuuint32_t estr[2] = {1u, 1u};
  return enc(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(ptr), dims, strides, box,
             estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Sets a kernel's dynamic-shared-memory size once per device (per call site's DeviceOnce).
static bool set_smem_once(DeviceOnce& once, const void* fn, int bytes) {
  return once.get([fn, bytes] {
    return static_cast<int>(cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes));
  }) == static_cast<int>(cudaSuccess);
}

// Largest number of pair clusters resident at once (one CTA per SM), per device.
static int pair_clusters_resident(int num_sms) {
  static DeviceOnce resident;
  return resident.get([num_sms] {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(num_sms & ~1));
    cfg.blockDim = dim3(gemm2::THREADS);
    cfg.dynamicSmemBytes = gemm2::ALLOC;
    int n = 0;
    if (cudaOccupancyMaxActiveClusters(&n, k_gemm_fp8_pair, &cfg) != cudaSuccess || n <= 0) {
      cudaGetLastError();
      n = num_sms / 2;
    }
    return n;
  });
}

// M <= 128 (one row tile) keeps the one-SM kernel: a 256-row pair tile would be half empty.
cudaError_t launch_gemm_fp8(const uint8_t* a8, const uint8_t* b8, void* y, int M, int N, int K,
                            const float* s_a, const float* s_b, int* err, uint64_t timeout_ns,
                            int num_sms, cudaStream_t stream, uint8_t* codes, const float* amax,
                            float* scale_out) {
  GemmArgs a;
  a.codes = codes;
  a.amax = amax;
  a.scale_out = scale_out;
  a.M = M;
  a.N = N;
  a.K = K;
  a.s_a = s_a;
  a.s_b = s_b;
  a.y = static_cast<__nv_bfloat16*>(y);
  a.err = err;
  a.timeout_ns = timeout_ns;
  CUtensorMap ma, mb;
  if (M > gemm::BM && num_sms >= 2) {
    static DeviceOnce configured;
    if (!make_map_2d(&ma, a8, M, K, gemm2::BM / 2) || !make_map_2d(&mb, b8, N, K, gemm2::BN / 2))
      return cudaErrorInvalidValue;
    if (!set_smem_once(configured, reinterpret_cast<const void*>(k_gemm_fp8_pair), gemm2::ALLOC))
      return cudaErrorInvalidValue;
    const int tiles = ((M + gemm2::BM - 1) / gemm2::BM) * ((N + gemm2::BN - 1) / gemm2::BN);
    const int resident = pair_clusters_resident(num_sms);
    const int pairs = tiles < resident ? tiles : resident;
    k_gemm_fp8_pair<<<2 * pairs, gemm2::THREADS, gemm2::ALLOC, stream>>>(ma, mb, a);
    return cudaGetLastError();
  }
  static DeviceOnce configured;
  if (!make_map_2d(&ma, a8, M, K, gemm::BM) || !make_map_2d(&mb, b8, N, K, gemm::BN))
    return cudaErrorInvalidValue;
  if (!set_smem_once(configured, reinterpret_cast<const void*>(k_gemm_fp8), gemm::ALLOC))
    return cudaErrorInvalidValue;
  const int tiles = ((M + gemm::BM - 1) / gemm::BM) * ((N + gemm::BN - 1) / gemm::BN);
  const int grid = tiles < num_sms ? tiles : num_sms;
  k_gemm_fp8<<<grid, gemm::THREADS, gemm::ALLOC, stream>>>(ma, mb, a);
  return cudaGetLastError();
}

}  // namespace qattn
