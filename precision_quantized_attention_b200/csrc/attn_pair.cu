// attn_pair.cu -- fused quantized attention forward for D = 128 on pairs of SMs (sm_100a:
// cluster of two CTAs, tcgen05.mma.cta_group::2, TMA, TMEM).  A variant of the one-SM kernel
// of attn_fwd.cu, selected with qattn_debug_use_pair_kernel; on B200 it measures about 6 %
// slower than that kernel at L = 8704 (its extra S buffers do not pay for the cross-CTA
// handshakes), so the one-SM kernel is the default.
//
// Method: NVIDIA developer blog "Optimizing FLUX.1 Kontext for Image Editing with Low-Precision
// Quantization", section "Workflow and quantization" and Fig. 4:
//   BMM1  S = Q8 K8^T in FP8 with higher-precision (FP32) accumulation   (second SDPA bullet)
//   softmax in FP32, no quantization at that stage                       (third bullet)
//   P requantized to per-tensor FP8, BMM2 O = P8 V8 in FP8                (fourth bullet, Fig. 4)
// over the full (non-causal) joint text + target + context token sequence.  The readings are
// those of the one-SM kernel in attn_fwd.cu: P = e4m3(p * 448), p = 2^(S' - M) in (0, 1] with M
// a maximum of the base-2 scores S' rounded up to an integer, and O divided by the
// FP32 row sum of the unquantized p after BMM2.
//
// Work unit: a pair of 128-row Q tiles of one (sequence, head), as in the one-SM kernel; here
// the two tiles run on the two CTAs of a cluster (CTA rank r holds rows 128 r .. 128 r + 127 of
// the pair).  One MMA instruction with M = 256 covers both tiles:
//   BMM1 (SS)  A = each CTA's Q tile, B = the key tile's 128 keys, of which each CTA's shared
//              memory holds 64 (rank 0 keys 0-63, rank 1 keys 64-127), so each SM stages half a
//              K tile per step; each CTA's TMEM receives S for its 128 rows and all 128 keys.
//   BMM2 (TS, block-scaled kind::mxf8f6f4)  A = P from each CTA's TMEM, B = the V tile, of which
//              each CTA holds 64 of the 128 D columns (MN-major), so again half a tile per SM.
// K/V therefore cross L2 and shared memory once per pair, as in the one-SM kernel.
//
// The point of the pair: each CTA's 512 TMEM columns hold O (128 columns) and THREE S buffers,
// so S for key steps s + 1 and s + 2 is computed while the softmax works on step s: the softmax
// never waits for its own P V and next Q K^T.  Two softmax warpgroups per CTA alternate key
// steps (warpgroup s % 2 takes step s), one thread per query row (= TMEM lane), so every SM
// sub-partition runs two softmax warps back to back.  Warps (384 threads):
//   0-3 / 4-7   softmax warpgroups 0 / 1: step s reads S from buffer s % 3 and writes P(s)
//               (E4M3) over its first 32 columns with BMM2's scale factors.
//   8           BMM1 issuer (leading CTA): S(s) = Q K(s)^T into buffer s % 3 once P(s - 3) V(s - 3)
//               has completed.
//   9           TMEM owner (both CTAs); BMM2 issuer (leading CTA): O += P(s) V(s).
//   11          TMA producer (both CTAs): its CTA's Q tile per segment, its halves of the K and
//               V tiles per step (one ring stage per step); bytes counted on the leading CTA's
//               barriers.  Warp 10 idles (a third warp on every sub-partition fits 168 registers).
// The issuer and producer loops run on the whole warp (warp-uniform values); one elected lane
// issues, and every commit arrives on the barrier of both CTAs (multicast).
// Maxima: P(s) is relative to its own tile's maximum mx(s), rounded up to an integer (p =
// 2^(S' - mx) in (0, 1]); O holds sum_s P(s) V 2^(mx(s) - M_ref): BMM2 multiplies each row of P(s)
// by 2^(mx(s) - M_ref) as an E8M0 scale factor, so no maximum is shared between steps except the
// reference M_ref, set by the segment's first tile.  Only a tile maximum more than 2^64 above
// M_ref (O could leave the FP32 range) rescales the row of O in TMEM (after the previous P V
// completed) and moves M_ref up; the warpgroup of step s - 1 publishes M_ref in shared memory
// after its exponentials and the one of step s reads it before writing its factor.  Each
// warpgroup keeps the row sum of its own steps relative to the largest tile maximum it has seen;
// the warpgroup of a segment's last step combines both (exact powers of two) and writes O.
// Relative to the running maximum of the one-SM kernel, the codes of P differ only in the E4M3
// subnormal range (rounding commutes with powers of two above it).
// All waits are bounded (a global-timer limit); on expiry a CTA records a timeout in the
// library's error word, drains what it issued and exits; both CTAs always meet at the final
// cluster barrier.
//
// Grid: dense launches are persistent (one cluster per two SMs), each cluster running the
// segment list of the one-SM kernel's schedule (whole pairs, then ranges of the tail pairs' key
// steps whose parts k_attn_combine merges); varlen launches keep a (pair, head, sequence) grid.
#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <cstdint>

#include "device_once.h"
#include "tensor_map.h"
#include "launch.h"
#include "sm100_ptx.cuh"
#include "softmax_sm100.cuh"

namespace qattn {

namespace pairk {
constexpr int D = 128;
constexpr int BLOCK_M = 128;                 // query rows per CTA (a pair covers 256)
constexpr int BLOCK_N = 128;                 // keys per step
constexpr int NSBUF = 3;                     // S buffers in TMEM
constexpr int STAGES = 6;                    // K/V ring: a stage holds one step's K and V halves
constexpr int NUM_SOFTMAX_WARPS = 8;         // warps 0-7
constexpr int WARP_BMM1 = 8;                 // issues S = Q K^T (leading CTA)
constexpr int WARP_MMA = 9;                  // TMEM owner; issues O += P V (leading CTA)
constexpr int WARP_LOAD = 11;                // TMA producer; warp 10 idles
constexpr int THREADS = 384;
constexpr int TILE_Q = BLOCK_M * D;          // 16 KB: 128 rows x 128 bytes
constexpr int TILE_KH = (BLOCK_N / 2) * D;   // 8 KB: 64 keys x 128 bytes (K-major)
constexpr int TILE_VH = BLOCK_N * (D / 2);   // 8 KB: 128 keys x 64 D columns (MN-major)
constexpr int OFF_Q = 0;                     // two buffers (segment i: i % 2)
constexpr int TILE_KV = TILE_KH + TILE_VH;   // 16 KB per stage
constexpr int OFF_KV = OFF_Q + 2 * TILE_Q;    // stage st: K half at OFF_KV + st * TILE_KV, V half after it
constexpr int OFF_BAR = OFF_KV + STAGES * TILE_KV;
// barriers: q_full[2] q_empty[2] kv_full[ST] kv_empty[ST] s_full[3]
// p_full[3] o_final[2] o_free pub[4] ep_ready[2][4] drain drain1.  A barrier a thread waits on by parity
// must never be two phases behind the phase it wants: the per-segment-parity o_final keeps that
// true although the softmax runs ahead of the MMAs.
constexpr int B_QFULL = 0, B_QEMPTY = 2, B_KVFULL = 4, B_KVEMPTY = B_KVFULL + STAGES;
constexpr int B_SFULL = B_KVEMPTY + STAGES, B_PFULL = B_SFULL + NSBUF;
constexpr int B_OFINAL = B_PFULL + NSBUF, B_OFREE = B_OFINAL + 2;
constexpr int B_PUB = B_OFREE + 1, B_EPREADY = B_PUB + 4, B_DRAIN = B_EPREADY + 8, B_DRAIN1 = B_DRAIN + 1;
constexpr int NBARS = B_DRAIN1 + 1;
constexpr int OFF_MREF = OFF_BAR + 8 * NBARS;          // float[128]: M_ref after the last published step
constexpr int OFF_STATS = OFF_MREF + 4 * BLOCK_M;      // float2[2][128]: (M, row sum) handoff
constexpr int OFF_TMEM = OFF_STATS + 2 * 8 * BLOCK_M;
constexpr int OFF_ABORT = OFF_TMEM + 4;
constexpr int BYTES = OFF_ABORT + 4;
constexpr int ALLOC = BYTES + 1024;          // slack for 1024-byte alignment
static_assert(TILE_Q % 1024 == 0 && TILE_KH % 1024 == 0 && TILE_VH % 1024 == 0, "alignment");
static_assert(STAGES >= NSBUF + 1, "the MMAs wait for step s + 3's K after releasing step s's stage");
static_assert(ALLOC <= 227 * 1024, "shared memory per CTA");
// TMEM columns: S buffers at 128 b (b = 0, 1, 2), O at 384; inside an S buffer P(s) takes the
// first 32 columns, BMM2's scale factors of P columns 64-67 and of V columns 96-99
constexpr uint32_t TM_O = NSBUF * BLOCK_N;
constexpr uint32_t TM_COLS = 512;
constexpr uint32_t SFA = 64, SFB = 96;
static_assert(TM_O + D <= TM_COLS, "TMEM budget");
constexpr uint32_t IDESC_S = idesc_e4m3_f32(2 * BLOCK_M, BLOCK_N, false);
}  // namespace pairk

struct PairArgs {
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
  int inject_missing_q;     // fault injection for tests: the producers never load anything
  uint8_t* dbg_p;           // test hook (see DebugHooks): P codes of one row, or nullptr
  int* dbg_m;
  int dbg_slab, dbg_row;
  // persistent schedule over pairs (dense), one entry per cluster: see k_attn_fp8_fwd's AttnArgs
  int pairs_per_head;
  int nkv;
  int ctas;                 // clusters G
  int whole;
  int tail_pairs;
  int tail_w;
  float* part_o;
  float2* part_ml;
  // extents for the checked build's index tests: slabs of the tensors, rows of partial results
  // the workspace holds, key steps the P-capture buffers hold
  int slabs;
  long long part_rows;
  int dbg_steps;
};

namespace {

// One unit of a cluster's work: key steps [kv0, kv1) of one pair of Q tiles (rows q_row0 ..
// q_row0 + 255 of the sequence), as in the one-SM kernel's schedule.
struct PSeg {
  int q_row0, seq_start, seq_len, slab;
  int kv0, kv1;
  int slot;                 // partial-result slot, or -1 when the segment covers the whole pair
};

__device__ __forceinline__ bool pair_segment(const PairArgs& a, int i, PSeg& s) {
  const int cl = static_cast<int>(blockIdx.x >> 1);            // cluster index
  int pair;
  if (a.cu_seqlens) {
    if (i > 0) return false;
    const int bz = blockIdx.z;
    s.seq_start = __ldg(a.cu_seqlens + bz);
    s.seq_len = __ldg(a.cu_seqlens + bz + 1) - s.seq_start;
    s.slab = blockIdx.y;
    s.q_row0 = cl * (2 * pairk::BLOCK_M);
    s.kv0 = 0;
    s.kv1 = (s.seq_len + pairk::BLOCK_N - 1) / pairk::BLOCK_N;
    s.slot = -1;
    return s.q_row0 < s.seq_len;
  }
  if (i < a.whole) {
    pair = cl + i * a.ctas;
    s.kv0 = 0;
    s.kv1 = a.nkv;
    s.slot = -1;
  } else {
    const int k = i - a.whole;                   // tail segment 0 or 1
    if (k > 1) return false;
    const long long end = static_cast<long long>(a.tail_pairs) * a.nkv;
    long long g0 = static_cast<long long>(cl) * a.tail_w;
    const long long g1 = min(g0 + a.tail_w, end);
    if (k == 1) g0 = (g0 / a.nkv + 1) * a.nkv;   // the second segment starts at a pair start
    if (g0 >= g1) return false;
    const int tp = static_cast<int>(g0 / a.nkv);
    s.kv0 = static_cast<int>(g0 - static_cast<long long>(tp) * a.nkv);
    s.kv1 = static_cast<int>(min(static_cast<long long>(a.nkv), s.kv0 + (g1 - g0)));
    s.slot = (s.kv0 == 0 && s.kv1 == a.nkv) ? -1 : 2 * cl + k;
    pair = a.whole * a.ctas + tp;
  }
  const int qblk = pair % a.pairs_per_head;
  const int h = (pair / a.pairs_per_head) % a.H;
  const int bz = pair / (a.pairs_per_head * a.H);
  s.seq_start = 0;
  s.seq_len = a.L;
  s.slab = bz * a.H + h;
  s.q_row0 = qblk * (2 * pairk::BLOCK_M);
  return true;
}

// Walks the cluster's key steps in order across its segments: global step index s, segment
// index seg, step j of the segment's n steps.
struct StepCursor {
  PSeg sg;
  int seg, j, n, s;
  bool valid;
  __device__ __forceinline__ void start(const PairArgs& a) {
    seg = 0;
    j = 0;
    s = 0;
    valid = pair_segment(a, 0, sg);
    n = valid ? sg.kv1 - sg.kv0 : 0;
  }
  __device__ __forceinline__ void next(const PairArgs& a) {
    ++s;
    if (++j == n) {
      ++seg;
      j = 0;
      valid = pair_segment(a, seg, sg);
      n = valid ? sg.kv1 - sg.kv0 : 0;
    }
  }
};

}  // namespace

// Test hook (see capture_p_codes), with the checked build's test of the step index.
__device__ __forceinline__ void capture_p_row(const PairArgs& args, int step, const uint32_t (&pk)[32],
                                           float mx) {
  if (!QATTN_IN_BOUNDS(args.err, step < args.dbg_steps)) return;
  capture_p_codes(args.dbg_p, args.dbg_m, step, pk, mx);
}

// Multiplies this thread's row of O (128 FP32 columns of its TMEM lane) by f, 8 columns at a
// time.  Out of line: only a rise of the row maximum past 2^64 over M_ref takes it.
__device__ __noinline__ void rescale_o_row(uint32_t t_o, float f) {
  tc_fence_after();
#pragma unroll 1
  for (int c8 = 0; c8 < pairk::D / 8; ++c8) {
    uint32_t v[8];
    tmem_ld8(t_o + c8 * 8, v);
    tmem_wait_ld();
#pragma unroll
    for (int i = 0; i < 8; ++i) v[i] = __float_as_uint(__uint_as_float(v[i]) * f);
    tmem_st8(t_o + c8 * 8, v);
  }
  tmem_wait_st();
}

// Writes this thread's row of a finished segment: O * f_ref is relative to the row maximum m_fin,
// l_tot the row sum of p * 448 relative to it.  A whole pair's row goes to the bf16 output
// (O * s_v / l); a cut pair's part goes to the workspace for k_attn_combine.  Out of line: once
// per segment, which keeps the per-step loop small.
__device__ __noinline__ void pair_epilogue(const PairArgs& args, const PSeg& sg, int rank, int r,
                                           uint32_t t_o, float f_ref, float m_fin, float l_tot) {
  constexpr int D = pairk::D;
  const int row = sg.q_row0 + rank * pairk::BLOCK_M + r;
  if (sg.slot >= 0) {
    if (!QATTN_IN_BOUNDS(args.err, (static_cast<long long>(sg.slot) * 2 + rank + 1) * pairk::BLOCK_M <=
                                       args.part_rows))
      return;
    const size_t slot = static_cast<size_t>(sg.slot) * 2 + rank;
    float4* po = reinterpret_cast<float4*>(args.part_o + (slot * pairk::BLOCK_M + r) * D);
#pragma unroll 1
    for (int c4 = 0; c4 < D / 32; ++c4) {
      uint32_t v[32];
      tmem_ld32(t_o + c4 * 32, v);
      tmem_wait_ld();
#pragma unroll
      for (int i = 0; i < 8; ++i)
        po[c4 * 8 + i] = make_float4(__uint_as_float(v[4 * i]) * f_ref, __uint_as_float(v[4 * i + 1]) * f_ref,
                                     __uint_as_float(v[4 * i + 2]) * f_ref, __uint_as_float(v[4 * i + 3]) * f_ref);
    }
    args.part_ml[slot * pairk::BLOCK_M + r] = make_float2(m_fin, l_tot);
    return;
  }
  const bool valid = row < sg.seq_len &&
                     QATTN_IN_BOUNDS(args.err, static_cast<long long>(sg.slab) * args.rows_per_slab +
                                                   sg.seq_start + row <
                                               static_cast<long long>(args.slabs) * args.rows_per_slab);
  const float scale = __ldg(args.s_v) / l_tot * f_ref;   // O = acc * s_v / 448 / (l / 448)
  __nv_bfloat16* orow =
      args.out + (static_cast<size_t>(sg.slab) * args.rows_per_slab + sg.seq_start + row) * D;
#pragma unroll 1
  for (int c4 = 0; c4 < D / 32; ++c4) {
    uint32_t v[32];
    tmem_ld32(t_o + c4 * 32, v);
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

__global__ void __cluster_dims__(2, 1, 1) __maxnreg__(168)
    k_attn_fp8_pair(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                    const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ PairArgs args) {
  using namespace pairk;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_u32 = smem_u32(smem_raw);
  const uint32_t base_u32 = (raw_u32 + 1023u) & ~1023u;   // the same offset in both CTAs
  uint8_t* base = smem_raw + (base_u32 - raw_u32);
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();                  // 0 leads the pair
  const bool leader = rank == 0;
  // Both CTAs of a cluster see the same segment list (uniform over the cluster), so an empty
  // one returns from both before any cluster-wide step.
  {
    PSeg s0;
    if (!pair_segment(args, 0, s0)) return;
  }

  const uint32_t bar0 = base_u32 + OFF_BAR;
  auto BAR = [&](int i) { return bar0 + 8u * static_cast<uint32_t>(i); };
  volatile int* abort_flag = reinterpret_cast<volatile int*>(base + OFF_ABORT);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(base + OFF_TMEM);
  if (threadIdx.x == 0) {
    for (int b = 0; b < 2; ++b) { mbar_init(BAR(B_QFULL + b), 1); mbar_init(BAR(B_QEMPTY + b), 1); }
    for (int i = 0; i < STAGES; ++i) { mbar_init(BAR(B_KVFULL + i), 1); mbar_init(BAR(B_KVEMPTY + i), 1); }
    for (int b = 0; b < NSBUF; ++b) {
      mbar_init(BAR(B_SFULL + b), 1);
      mbar_init(BAR(B_PFULL + b), 8);          // 4 softmax warps x 2 CTAs (leading CTA's)
    }
    for (int b = 0; b < 2; ++b) mbar_init(BAR(B_OFINAL + b), 1);      // segment i's O final, i % 2
    mbar_init(BAR(B_OFREE), 8);                // 4 epilogue warps x 2 CTAs (leading CTA's)
    for (int q = 0; q < 4; ++q) mbar_init(BAR(B_PUB + q), 32);
    for (int q = 0; q < 8; ++q) mbar_init(BAR(B_EPREADY + q), 32);
    mbar_init(BAR(B_DRAIN), 1);
    mbar_init(BAR(B_DRAIN1), 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == WARP_MMA) {                      // whole warp, both CTAs: TMEM of the pair
    tmem_alloc_pair(base_u32 + OFF_TMEM, TM_COLS);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  cluster_sync();                              // barriers of both CTAs initialised, TMEM allocated
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint64_t tlim = args.timeout_ns;

  if (warp == WARP_LOAD) {
    // ======================= TMA producer (both CTAs, whole warp) =======================
    // The warp runs the loop uniformly (waits by every lane); one elected lane issues.  Per step
    // s, in order: the Q tile of the segment (at its first step), then K and V halves of s into
    // stage s % STAGES once the MMAs released the step that used it before.
    if (!args.inject_missing_q) {
      const bool el = elect_one();
      if (el) {
        tma_prefetch_desc(&tm_q);
        tma_prefetch_desc(&tm_k);
        tma_prefetch_desc(&tm_v);
      }
      const int r = static_cast<int>(rank);
      bool ok = true;
      StepCursor lc;
      lc.start(args);
      while (ok && lc.valid) {
        // tiles starting past the sequence would load zeros: index errors (recorded; the loads
        // themselves stay in the tensor maps' bounds checking)
        (void)QATTN_IN_BOUNDS(args.err, (lc.sg.kv0 + lc.j) * BLOCK_N < lc.sg.seq_len);
        if (lc.j == 0) {
          (void)QATTN_IN_BOUNDS(args.err, lc.sg.q_row0 < lc.sg.seq_len && lc.sg.slab < args.slabs &&
                                              lc.sg.seq_start + lc.sg.seq_len <= args.rows_per_slab);
          const int i = lc.seg, b = i & 1;
          if (i >= 2 && !mbar_wait(BAR(B_QEMPTY + b), ((i >> 1) - 1) & 1, tlim, abort_flag, args.err)) {
            ok = false;
            break;
          }
          if (el) {
            if (leader) mbar_arrive_expect_tx(BAR(B_QFULL + b), 2 * TILE_Q);
            tma_load_3d_pair(base_u32 + OFF_Q + b * TILE_Q, &tm_q, mapa_shared(BAR(B_QFULL + b), 0), 0,
                             lc.sg.seq_start + lc.sg.q_row0 + r * BLOCK_M, lc.sg.slab);
          }
        }
        const int st = lc.s % STAGES;
        if (lc.s >= STAGES &&
            !mbar_wait(BAR(B_KVEMPTY + st), ((lc.s / STAGES) - 1) & 1, tlim, abort_flag, args.err)) {
          ok = false;
          break;
        }
        if (el) {
          const uint32_t full = mapa_shared(BAR(B_KVFULL + st), 0);
          const int key0 = lc.sg.seq_start + (lc.sg.kv0 + lc.j) * BLOCK_N;
          if (leader) mbar_arrive_expect_tx(BAR(B_KVFULL + st), 2 * TILE_KV);
          // K: keys 64 r .. 64 r + 63 of the step; V: D columns 64 r .. 64 r + 63 of all 128 keys
          tma_load_3d_pair(base_u32 + OFF_KV + st * TILE_KV, &tm_k, full, 0, key0 + r * (BLOCK_N / 2),
                           lc.sg.slab);
          tma_load_3d_pair(base_u32 + OFF_KV + st * TILE_KV + TILE_KH, &tm_v, full, r * (D / 2), key0,
                           lc.sg.slab);
        }
        lc.next(args);
      }
      // drain: the MMAs released every stage this CTA filled, so its loads have landed and no
      // commit from the leading CTA is still on its way here (instant when healthy)
      const int ns = lc.s, nq = lc.seg;
      for (int j = ns - 1; j >= 0 && j >= ns - STAGES; --j)
        mbar_drain(BAR(B_KVEMPTY + j % STAGES), (j / STAGES) & 1, tlim);
      for (int i = nq - 1; i >= 0 && i >= nq - 2; --i)
        mbar_drain(BAR(B_QEMPTY + (i & 1)), (i >> 1) & 1, tlim);
    }
  } else if (warp == WARP_BMM1) {
    // ======================= BMM1 issuer (leading CTA, whole warp) =======================
    // S(s) = Q K(s)^T into buffer s % 3 once P(s - 3) V(s - 3), which read P from that buffer,
    // has completed (its K/V stage release); loop warp-uniform, one elected lane issues.
    if (leader) {
      const bool el = elect_one();
      StepCursor bc;
      bc.start(args);
      bool ok = true;
      while (ok && bc.valid) {
        const int i = bc.seg, qb = i & 1, b = bc.s % NSBUF, st = bc.s % STAGES;
        if (bc.s >= NSBUF) {
          const int u = bc.s - NSBUF;
          ok = mbar_wait(BAR(B_KVEMPTY + u % STAGES), (u / STAGES) & 1, tlim, abort_flag, args.err);
        }
        if (ok && bc.j == 0) ok = mbar_wait(BAR(B_QFULL + qb), (i >> 1) & 1, tlim, abort_flag, args.err);
        if (ok) ok = mbar_wait(BAR(B_KVFULL + st), (bc.s / STAGES) & 1, tlim, abort_flag, args.err);
        if (!ok) break;
        tc_fence_after();
        // K-major rows of 128 bytes, 128-byte swizzle, 8-row atoms (SBO 1024); a 32-byte K step
        // adds 2 to the descriptor's start-address field (address >> 4)
        const uint64_t da = smem_desc(base_u32 + OFF_Q + qb * TILE_Q, 16, 1024, 2u);
        const uint64_t db = smem_desc(base_u32 + OFF_KV + st * TILE_KV, 16, 1024, 2u);
        if (el) {
#pragma unroll
          for (int kk = 0; kk < D / 32; ++kk)
            mma_f8_ss_pair(tmem + b * BLOCK_N, da + 2u * kk, db + 2u * kk, IDESC_S, kk > 0 ? 1u : 0u);
          mma_commit_pair_both(BAR(B_SFULL + b));
          if (bc.j == bc.n - 1) mma_commit_pair_both(BAR(B_QEMPTY + qb));   // last MMA reading Q buffer qb
        }
        __syncwarp();
        bc.next(args);
      }
      // drain: this thread's MMAs complete before TMEM is released
      if (el) mma_commit_pair(BAR(B_DRAIN1));
      __syncwarp();
      mbar_drain(BAR(B_DRAIN1), 0, tlim);
    }
  } else if (warp == WARP_MMA) {
    // ======================= BMM2 issuer (leading CTA, whole warp) =======================
    // O += P(s) V(s) once both CTAs' softmax wrote P(s); its commit releases the K/V stage of
    // step s (and with it S buffer s % 3 for BMM1(s + 3); and tells the softmax that O holds
    // every P V up to s).  Loop warp-uniform, one elected lane issues.
    if (leader) {
      const bool el = elect_one();
      StepCursor cc;
      cc.start(args);
      bool ok = true;
      while (ok && cc.valid) {
        const int b = cc.s % NSBUF, st = cc.s % STAGES;
        // P(s) written by both CTAs' softmax (V(s) landed with K(s), before BMM1(s))
        ok = mbar_wait(BAR(B_PFULL + b), (cc.s / NSBUF) & 1, tlim, abort_flag, args.err);
        // the first P V of a segment overwrites O: both CTAs have read out the previous one
        if (ok && cc.j == 0 && cc.seg > 0)
          ok = mbar_wait(BAR(B_OFREE), (cc.seg - 1) & 1, tlim, abort_flag, args.err);
        if (!ok) break;
        tc_fence_after();
        // O += (P(s) 2^(M(s) - M_ref)) V(s): E8M0 factors of P written by the softmax with P,
        // V's factors all 2^0; V MN-major, rows of 64 bytes (this CTA's D columns), 64-byte
        // swizzle, SBO = 8 key rows; a K step of 32 keys advances 32 rows (2 KB)
        const uint64_t dv = smem_desc(base_u32 + OFF_KV + st * TILE_KV + TILE_KH, TILE_VH, 8 * (D / 2), 4u);
        const uint32_t sb = tmem + b * BLOCK_N;
        if (el) {
#pragma unroll
          for (int kk = 0; kk < BLOCK_N / 32; ++kk)
            mma_mxf8_ts_pair(tmem + TM_O, sb + kk * 8, dv + static_cast<uint64_t>(kk * 32 * (D / 2) / 16),
                             idesc_mxf8_e4m3(2 * BLOCK_M, D, true, static_cast<uint32_t>(kk)),
                             sb + SFA, sb + SFB, (cc.j > 0 || kk > 0) ? 1u : 0u);
          mma_commit_pair_both(BAR(B_KVEMPTY + st));
          if (cc.j == cc.n - 1) mma_commit_pair_both(BAR(B_OFINAL + (cc.seg & 1)));
        }
        __syncwarp();
        cc.next(args);
      }
      // drain: all issued MMAs complete before TMEM is released
      if (el) mma_commit_pair(BAR(B_DRAIN));
      __syncwarp();
      mbar_drain(BAR(B_DRAIN), 0, tlim);
    }
  } else if (warp < NUM_SOFTMAX_WARPS) {
    // ======================= softmax warpgroups (both CTAs) =======================
    const int wg = warp >> 2;                      // takes the steps s with s % 2 == wg
    const int quarter = warp & 3;                  // TMEM lane quarter
    const int r = quarter * 32 + lane;             // row within this CTA's tile
    const uint32_t lane_off = static_cast<uint32_t>(quarter * 32) << 16;
    // this row's slot of the M_ref handoff and of the row-sum handoff (32-bit shared addresses)
    const uint32_t a_mref = base_u32 + OFF_MREF + 4u * r;
    const uint32_t a_stats = base_u32 + OFF_STATS + 8u * r;
    const float c = __ldg(args.s_q) * __ldg(args.s_k) * args.sm_scale * LOG2E_F;
    bool ok = true;
    int s0 = 0;                                    // global index of the segment's first step
    int k2 = 0;                                    // segments of two or more steps so far
    PSeg sg{};
    for (int seg = 0; ok && pair_segment(args, seg, sg); ++seg) {
      const int n = sg.kv1 - sg.kv0;
      float l = 0.0f;                              // this warpgroup's row sum of p * 448, relative
      float m_w = 0.0f;                            // to m_w, the largest tile maximum it has seen
      bool mine_before = false;
      float m_ref = 0.0f;
      const bool capture = args.dbg_p != nullptr && sg.slab == args.dbg_slab &&
                           sg.seq_start + sg.q_row0 + static_cast<int>(rank) * BLOCK_M + r == args.dbg_row;
      for (int j = (s0 & 1) == wg ? 0 : 1; j < n; j += 2) {
        const int s = s0 + j;
        const int b = s % NSBUF;
        const uint32_t tS = tmem + lane_off + b * BLOCK_N;
        ok = mbar_wait(BAR(B_SFULL + b), (s / NSBUF) & 1, tlim, abort_flag, args.err);
        if (!__all_sync(0xFFFFFFFFu, ok)) { ok = false; break; }
        tc_fence_after();
        float sc[BLOCK_N];
        {
          uint32_t sv[BLOCK_N / 32][32];
#pragma unroll
          for (int c4 = 0; c4 < BLOCK_N / 32; ++c4) tmem_ld32(tS + c4 * 32, sv[c4]);
          tmem_wait_ld();
#pragma unroll
          for (int i = 0; i < BLOCK_N; ++i) sc[i] = __uint_as_float(sv[i / 32][i % 32]);
        }
        // S is in registers: V's scale factors (all 2^0) can go into columns SFB..SFB + 3 now
        tmem_st4_same(tS + SFB, 0x7F7F7F7Fu);
        const int kv_valid = sg.seq_len - (sg.kv0 + j) * BLOCK_N;   // keys of this step in the sequence
        if (kv_valid < BLOCK_N) {
#pragma unroll
          for (int i = 0; i < BLOCK_N; ++i)
            if (i >= kv_valid) sc[i] = -INFINITY;
        }
        // P(s) relative to this tile's own maximum mx (an integer): p = 2^(S' - mx) in (0, 1]
        const float mx = ceilf(rowmax128(sc) * c);
        const float neg_off = LOG2_448 - mx;
        float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
        uint32_t pk[BLOCK_N / 4];
#pragma unroll
        for (int i = 0; i < BLOCK_N; i += 16) {
          float p[16];
#pragma unroll
          for (int q = 0; q < 8; ++q) {
            float x0, x1;
            ffma2_bc(x0, x1, sc[i + 2 * q], sc[i + 2 * q + 1], c, neg_off);
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
#ifndef QATTN_NO_CAPTURE_HOOK
        if (capture) capture_p_row(args, sg.kv0 + j, pk, mx);   // test hook: off unless a row is chosen
#endif
        // P(s) over the first 32 columns of the buffer (column c: keys 4c..4c+3)
        tmem_st32(tS, pk);
        // M_ref after step s - 1, published by the other warpgroup (waited on at every step so
        // that the barrier's phases stay in step order, also at a segment's first step)
        if (s > 0) {
          ok = mbar_wait(BAR(B_PUB + quarter), (s - 1) & 1, tlim, abort_flag, args.err);
          if (!__all_sync(0xFFFFFFFFu, ok)) { ok = false; break; }
        }
        bool far = false;
        if (j == 0) {
          m_ref = mx;                              // the segment's first tile sets M_ref
        } else {
          m_ref = ld_shared_f32(a_mref);
          // O holds sum P V 2^(mx - M_ref); past a gap of 2^64 O could leave the FP32 range:
          // this row of O is rescaled and M_ref moves up to mx
          far = mx - m_ref > 64.0f;
        }
        if (__any_sync(0xFFFFFFFFu, far)) {
          // O is quiescent once the previous step's P V completed (its commit released that
          // step's K/V stage); the next P V needs this step's P
          ok = mbar_wait(BAR(B_KVEMPTY + (s - 1) % STAGES), ((s - 1) / STAGES) & 1, tlim, abort_flag,
                         args.err);
          if (!__all_sync(0xFFFFFFFFu, ok)) { ok = false; break; }
          rescale_o_row(tmem + lane_off + TM_O, far ? exp2_int(static_cast<int>(m_ref - mx)) : 1.0f);
          if (far) m_ref = mx;
        }
        st_shared_f32(a_mref, m_ref);
        mbar_arrive(BAR(B_PUB + quarter));         // M_ref after step s published
        // BMM2's scale factor of this row: 2^(mx - M_ref) (E8M0, code 0 = 2^-127 at least) in
        // column SFA + quarter of its lane (the MMA reads row r's factor from lane r, column r / 32)
        const int gap = max(static_cast<int>(mx - m_ref), -127);
        tmem_st1(tS + SFA + quarter, static_cast<uint32_t>(127 + gap) * 0x01010101u);
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive_cluster(mapa_shared(BAR(B_PFULL + b), 0));
        // this warpgroup's row sum, relative to the largest tile maximum it has seen
        const float rowsum = ((acc[0] + acc[1]) + (acc[2] + acc[3])) + ((acc[4] + acc[5]) + (acc[6] + acc[7]));
        if (mine_before) {
          const float m_new = fmaxf(m_w, mx);
          l = l * exp2_int(static_cast<int>(m_w - m_new)) + rowsum * exp2_int(static_cast<int>(mx - m_new));
          m_w = m_new;
        } else {
          l = rowsum;
          m_w = mx;
        }
        mine_before = true;
        if (j == n - 2) {
          // hand this warpgroup's (m_w, row sum) to the warpgroup of the segment's last step
          st_shared_f32x2(a_stats + (k2 & 1) * (8u * BLOCK_M), m_w, l);
          mbar_arrive(BAR(B_EPREADY + (k2 & 1) * 4 + quarter));
        }
        if (j == n - 1) {
          // ---- epilogue of the segment: O is final once its last P V completed ----
          ok = mbar_wait(BAR(B_OFINAL + (seg & 1)), (seg >> 1) & 1, tlim, abort_flag, args.err);
          if (ok && n >= 2)
            ok = mbar_wait(BAR(B_EPREADY + (k2 & 1) * 4 + quarter), (k2 >> 1) & 1, tlim, abort_flag,
                           args.err);
          if (!__all_sync(0xFFFFFFFFu, ok)) { ok = false; break; }
          tc_fence_after();
          float m_fin = m_w, l_tot = l;
          if (n >= 2) {
            const float2 o = ld_shared_f32x2(a_stats + (k2 & 1) * (8u * BLOCK_M));   // other's (m_w, l)
            m_fin = fmaxf(m_w, o.x);
            l_tot = l * exp2_int(static_cast<int>(m_w - m_fin)) + o.y * exp2_int(static_cast<int>(o.x - m_fin));
          }
          pair_epilogue(args, sg, static_cast<int>(rank), r, tmem + lane_off + TM_O,
                        exp2_int(static_cast<int>(m_ref - m_fin)), m_fin, l_tot);
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive_cluster(mapa_shared(BAR(B_OFREE), 0));   // O read out
        }
      }
      if (!ok) break;
      if (n >= 2) ++k2;
      s0 += n;
    }
  }

  tc_fence_before();
  cluster_sync();                              // no MMA, load or arrival of either CTA is outstanding
  if (warp == WARP_MMA) {
    tc_fence_after();
    tmem_dealloc_pair(tmem, TM_COLS);
  }
}

// ---------------------------------------------------------------------------------------------
// Host side
// ---------------------------------------------------------------------------------------------

// 3-D map over an E4M3 tensor viewed as [slabs][rows][128]: box = box_inner bytes x box_rows rows
// of one slab, swizzle matching the inner box width (128 or 64 bytes).
static bool pair_map(CUtensorMap* map, const void* ptr, int rows, int slabs, int box_inner,
                     int box_rows) {
  EncodeTiledFn enc = encode_tiled_fn();
  if (!enc) return false;
  constexpr int D = pairk::D;
  cuuint64_t dims[3] = {static_cast<cuuint64_t>(D), static_cast<cuuint64_t>(rows),
                        static_cast<cuuint64_t>(slabs)};
  cuuint64_t strides[2] = {static_cast<cuuint64_t>(D),
                           static_cast<cuuint64_t>(D) * static_cast<cuuint64_t>(rows)};
  cuuint32_t box[3] = {static_cast<cuuint32_t>(box_inner), static_cast<cuuint32_t>(box_rows), 1u};
  cuuint32_t estr[3] = {1u, 1u, 1u};
  return enc(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<void*>(ptr), dims, strides, box,
             estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
             box_inner == 128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Pair clusters resident at once on the current device (one CTA per SM): the persistent grid.
// Sets the pair kernel's dynamic-shared-memory size on the current device (once per device).
static cudaError_t pair_smem_attribute() {
  static DeviceOnce attr;
  return static_cast<cudaError_t>(attr.get([] {
    return static_cast<int>(cudaFuncSetAttribute(k_attn_fp8_pair,
                                                 cudaFuncAttributeMaxDynamicSharedMemorySize,
                                                 pairk::ALLOC));
  }));
}

int attention_pair_units(int num_sms) {
  static DeviceOnce units;
  return units.get([num_sms] {
    int n = 0;
    if (pair_smem_attribute() == cudaSuccess) {
      cudaLaunchConfig_t cfg = {};
      cfg.gridDim = dim3(static_cast<unsigned>(num_sms & ~1));
      cfg.blockDim = dim3(pairk::THREADS);
      cfg.dynamicSmemBytes = pairk::ALLOC;
      if (cudaOccupancyMaxActiveClusters(&n, k_attn_fp8_pair, &cfg) != cudaSuccess) n = 0;
    }
    cudaGetLastError();
    if (n <= 0 || n > num_sms / 2) n = num_sms / 2;
    return n < 1 ? 1 : n;
  });
}

// Launch of the pair kernel (D = 128).  Dense: the schedule `plan` (planned for
// attention_pair_units clusters); varlen: grid of pairs x heads x sequences.
cudaError_t launch_attention_pair(const uint8_t* q8, const uint8_t* k8, const uint8_t* v8, void* out,
                                  int H, int L, const int* cu_seqlens, int nseq, int max_seqlen,
                                  int rows_per_slab, int slabs, const float* s_q, const float* s_k,
                                  const float* s_v, float sm_scale, int* err, uint64_t timeout_ns,
                                  const DebugHooks& dbg, const AttnSplitPlan* plan, void* workspace,
                                  cudaStream_t stream) {
  using namespace pairk;
  CUtensorMap mq, mk, mv;
  if (!pair_map(&mq, q8, rows_per_slab, slabs, D, BLOCK_M) ||
      !pair_map(&mk, k8, rows_per_slab, slabs, D, BLOCK_N / 2) ||
      !pair_map(&mv, v8, rows_per_slab, slabs, D / 2, BLOCK_N))
    return cudaErrorInvalidValue;
  const cudaError_t e = pair_smem_attribute();
  if (e != cudaSuccess) return e;
  PairArgs a;
  a.rows_per_slab = rows_per_slab;
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
  a.inject_missing_q = dbg.inject_missing_q;
  a.dbg_p = dbg.p_codes;
  a.dbg_m = dbg.p_maxima;
  a.dbg_slab = dbg.p_slab;
  a.dbg_row = dbg.p_row;
  a.pairs_per_head = plan ? plan->pairs_per_head : 0;
  a.nkv = plan ? plan->nkv : 0;
  a.ctas = plan ? plan->ctas : 0;
  a.whole = plan ? plan->whole : 0;
  a.tail_pairs = plan ? plan->tail_pairs : 0;
  a.tail_w = plan ? plan->tail_w : 1;
  a.part_o = nullptr;
  a.part_ml = nullptr;
  a.slabs = slabs;
  a.part_rows = 0;
  a.dbg_steps = ((cu_seqlens ? max_seqlen : L) + BLOCK_N - 1) / BLOCK_N;
  dim3 grid;
  if (cu_seqlens) {
    grid = dim3(2 * ((max_seqlen + 2 * BLOCK_M - 1) / (2 * BLOCK_M)), H, nseq);
  } else {
    if (plan->bytes > 0 && workspace) {
      const size_t o_elems = static_cast<size_t>(2) * plan->ctas * 2 * BLOCK_M * D;
      a.part_o = static_cast<float*>(workspace);
      a.part_ml = reinterpret_cast<float2*>(a.part_o + o_elems);
      a.part_rows = static_cast<long long>(2) * plan->ctas * 2 * BLOCK_M;
    }
    grid = dim3(2 * plan->ctas, 1, 1);
  }
  k_attn_fp8_pair<<<grid, THREADS, ALLOC, stream>>>(mq, mk, mv, a);
  return cudaGetLastError();
}

}  // namespace qattn
