// attn_fwd.cu -- fused quantized attention forward for sm_100a (TMA + tcgen05 + TMEM): the
// kernel of every launch (D = 64 and 128) unless the pair-of-SMs variant (attn_pair.cu) is
// selected for D = 128; the persistent schedule, the combine of cut pairs and the launch.
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
//     rounded UP to an integer.  P of a key tile is relative to the M of that tile; all
//     rescales are exact powers of two, and E4M3 rounding commutes with power-of-two scaling in
//     the normal range, so the result does not depend on how keys are tiled.
//
// Kernel structure: one CTA (one per SM) per pair of 128-row Q tiles of one (sequence, head).
//   warp 8      TMA producer: per segment both Q tiles, then K and V tiles through separate
//               rings.
//   warp 9      MMA issuer (one elected thread) and TMEM owner.  Per KV tile j and Q tile t it
//               issues O_t += P_t(j) V_j (P read from tensor memory; block-scaled MMA, see
//               below) and right behind it, in the
//               same in-order tcgen05 stream, S_t = Q_t K_{j+1}^T into the columns P_t(j)
//               occupied; one commit then tells softmax t that S_t(j+1) is ready and that O_t
//               holds every P_t V up to tile j.
//   warps 0-7   two softmax warpgroups, one per Q tile; thread = one query row = one TMEM lane.
//               Each reads its 128 scores with tcgen05.ld, takes the row max (3-input maxima)
//               and computes p*448 = 2^(S' - M + log2 448) in FP32 (hardware ex2 for most
//               pairs, a degree-5 polynomial on the FMA pipe for the rest), sums p in packed
//               f32x2 adds, converts to E4M3 and writes P_t(j) over S_t(j) with tcgen05.st.
//   O_t is kept relative to a reference max M_ref per row (the row's first M): BMM2 multiplies
//   each row of P_t(j) by 2^(M - M_ref) as an E8M0 block scale factor (kind::mxf8f6f4), which
//   the softmax writes next to P, so a rise of M costs no pass over O.  Only when M - M_ref
//   would pass 64 (O could leave the FP32 range) does the softmax rescale its O row in TMEM and
//   move M_ref up; the epilogue applies the last 2^(M_ref - M).
//   The two Q tiles alternate on the tensor pipe, so one tile's softmax overlaps the other
//   tile's MMAs; K/V tiles are read by TMA once per CTA for both Q tiles.
// TMEM: S_0/P_0, S_1/P_1 (128 FP32 columns each; P uses the first 32, BMM2's scale factors
// columns 64-67 and 96-99), O_0, O_1 (D columns).
// All waits are bounded (a global-timer limit); on expiry the CTA records a timeout in the
// library's error word, drains what it issued and exits.
//
// Grid: dense launches are persistent, one CTA per SM.  Each CTA runs a list of segments (key
// ranges of one pair of Q tiles): an equal share of whole pairs, then, with a workspace, a
// contiguous range of the remaining pairs' key steps laid end to end, so that every CTA runs
// the same number of key steps.  A segment that covers part of a pair writes its unnormalised
// O rows, integer running max and row sum; k_attn_combine merges the parts (exact power-of-two
// rescales) into the bf16 output.  Between segments Q is double-buffered, and the first P V of
// a segment waits until the softmax has read out the previous segment's O.  Varlen launches
// keep a (pair, head, sequence) grid, one segment per CTA.
#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <cstdint>

#include "device_once.h"
#include "tensor_map.h"
#include "launch.h"
#include "sm100_ptx.cuh"
#include "softmax_sm100.cuh"

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
  // Dense launches are persistent: G = ctas CTAs, at most one per SM.  CTA c runs, in order,
  // the pairs of Q tiles c, c + G, ..., c + (whole - 1) G whole, and then the key steps
  // [c * tail_w, (c + 1) * tail_w) of the tail: the pairs from whole * G on, their key steps
  // laid end to end.  A tail range is at most one pair long, so a CTA has at most two tail
  // segments; one that covers only part of a pair writes unnormalised partial results to slot
  // 2c (the CTA's first tail segment) or 2c + 1 (its second), for the combine kernel:
  //   part_o[((slot * NQ + t) * BLOCK_M + row) * D + c]   (FP32, row-major)
  //   part_ml[(slot * NQ + t) * BLOCK_M + row] = (running max, row sum)
  int pairs_per_head;
  int nkv;                  // key steps of a pair (dense)
  int ctas;                 // G
  int whole;                // whole pairs per CTA
  int tail_pairs;
  int tail_w;               // tail key steps per CTA, 1..nkv (nkv: no pair is cut)
  float* part_o;
  float2* part_ml;
  // extents for the checked build's index tests: slabs of the tensors (the output has
  // slabs * rows_per_slab rows) and rows of partial results the workspace holds
  int slabs;
  long long part_rows;
  // test hook (DebugHooks): P codes and maxima of one query row, or dbg_p == nullptr
  uint8_t* dbg_p;
  int* dbg_m;
  int dbg_slab, dbg_row, dbg_steps;
};

// One unit of a CTA's work: key steps [kv0, kv1) of one pair of Q tiles.
struct Seg {
  int q_row0, seq_start, seq_len, slab;
  int kv0, kv1;
  int slot;                 // partial-result slot, or -1 when the segment covers the whole pair
};

// The i-th segment of this CTA (false when it has no more).  Varlen launches keep one pair per
// CTA (grid = pairs x heads x sequences); dense ones follow the persistent schedule above.
__device__ __forceinline__ bool get_segment(const AttnArgs& a, int i, Seg& s) {
  int pair;
  if (a.cu_seqlens) {
    if (i > 0) return false;
    const int bz = blockIdx.z;
    s.seq_start = __ldg(a.cu_seqlens + bz);
    s.seq_len = __ldg(a.cu_seqlens + bz + 1) - s.seq_start;
    s.slab = blockIdx.y;
    s.q_row0 = blockIdx.x * (NQ * BLOCK_M);
    s.kv0 = 0;
    s.kv1 = (s.seq_len + BLOCK_N - 1) / BLOCK_N;
    s.slot = -1;
    return s.q_row0 < s.seq_len;
  }
  const int c = blockIdx.x;
  if (i < a.whole) {
    pair = c + i * a.ctas;
    s.kv0 = 0;
    s.kv1 = a.nkv;
    s.slot = -1;
  } else {
    const int k = i - a.whole;                   // tail segment 0 or 1
    if (k > 1) return false;
    const long long end = static_cast<long long>(a.tail_pairs) * a.nkv;
    long long g0 = static_cast<long long>(c) * a.tail_w;
    const long long g1 = min(g0 + a.tail_w, end);
    if (k == 1) g0 = (g0 / a.nkv + 1) * a.nkv;   // the second segment starts at a pair start
    if (g0 >= g1) return false;
    const int tp = static_cast<int>(g0 / a.nkv);
    s.kv0 = static_cast<int>(g0 - static_cast<long long>(tp) * a.nkv);
    s.kv1 = static_cast<int>(min(static_cast<long long>(a.nkv), s.kv0 + (g1 - g0)));
    s.slot = (s.kv0 == 0 && s.kv1 == a.nkv) ? -1 : 2 * c + k;
    pair = a.whole * a.ctas + tp;
  }
  const int qblk = pair % a.pairs_per_head;
  const int h = (pair / a.pairs_per_head) % a.H;
  const int bz = pair / (a.pairs_per_head * a.H);
  s.seq_start = 0;
  s.seq_len = a.L;
  s.slab = bz * a.H + h;
  s.q_row0 = qblk * (NQ * BLOCK_M);
  return true;
}

template <int D>
struct Smem {
  static constexpr int TILE_Q = BLOCK_M * D;       // bytes (E4M3)
  static constexpr int TILE_KV = BLOCK_N * D;
  static constexpr int OFF_Q = 0;                  // two buffers of NQ tiles (segment i: i % 2)
  static constexpr int OFF_K = OFF_Q + 2 * NQ * TILE_Q;
  static constexpr int OFF_V = OFF_K + KSTAGES * TILE_KV;
  static constexpr int OFF_BAR = OFF_V + VSTAGES * TILE_KV;
  // barriers: q_full[2], q_empty[2], k_full[KS], k_empty[KS], v_full[VS], v_empty[VS],
  // s_full[NQ], p_full[NQ], o_final[NQ], o_free[NQ], drain
  static constexpr int NBARS = 4 + 2 * KSTAGES + 2 * VSTAGES + 4 * NQ + 1;
  static constexpr int OFF_TMEM = OFF_BAR + 8 * NBARS;
  static constexpr int OFF_ABORT = OFF_TMEM + 4;
  static constexpr int BYTES = OFF_ABORT + 4;
  static constexpr int ALLOC = BYTES + 1024;       // slack for 1024-byte alignment
  static_assert(TILE_Q % 1024 == 0 && TILE_KV % 1024 == 0, "alignment");
  static_assert(ALLOC <= 227 * 1024, "shared memory per CTA");
};

template <int D>
struct TmemCols {
  static constexpr uint32_t S0 = 0;                      // S_t / P_t at t * BLOCK_N
  static constexpr uint32_t O0 = NQ * BLOCK_N;           // O_t at O0 + t * D
  // BMM2's E8M0 scale factors (4 columns each), written with P_t inside S_t past P_t's 32
  // columns (S_t is not read again before the next S_t = Q_t K^T overwrites it)
  static constexpr uint32_t SFA = 64, SFB = 96;
  static constexpr uint32_t USED = NQ * BLOCK_N + NQ * D;
  static constexpr uint32_t ALLOC = USED <= 256 ? 256 : 512;
};

// CAPTURE: the instance with the P-code test hook (launched only while a capture is armed); the
// instance without it is the one every other launch runs, so the hook costs nothing there.
template <int D, bool CAPTURE>
__global__ void __launch_bounds__(ATTN_THREADS, 1)
    k_attn_fp8_fwd(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                   const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ AttnArgs args) {
  using SL = Smem<D>;
  using TC = TmemCols<D>;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_u32 = smem_u32(smem_raw);
  const uint32_t base_u32 = (raw_u32 + 1023u) & ~1023u;
  uint8_t* base = smem_raw + (base_u32 - raw_u32);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  {
    Seg s0;
    if (!get_segment(args, 0, s0)) return;        // uniform over the CTA: nothing to do
  }

  // ---- barriers --------------------------------------------------------------------------
  // Phases run on across segments: the K/V rings count loads, s_full / p_full count key steps,
  // o_final / o_free count segments, q_full / q_empty count the uses of each Q buffer.
  const uint32_t bar0 = base_u32 + SL::OFF_BAR;
  auto BAR = [&](int i) { return bar0 + 8u * static_cast<uint32_t>(i); };
  constexpr int B_QFULL = 0, B_QEMPTY = 2;
  constexpr int B_KFULL = 4, B_KEMPTY = B_KFULL + KSTAGES;
  constexpr int B_VFULL = B_KEMPTY + KSTAGES, B_VEMPTY = B_VFULL + VSTAGES;
  constexpr int B_SFULL = B_VEMPTY + VSTAGES, B_PFULL = B_SFULL + NQ;
  constexpr int B_OFINAL = B_PFULL + NQ, B_OFREE = B_OFINAL + NQ, B_DRAIN = B_OFREE + NQ;
  volatile int* abort_flag = reinterpret_cast<volatile int*>(base + SL::OFF_ABORT);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(base + SL::OFF_TMEM);

  if (threadIdx.x == 0) {
    for (int b = 0; b < 2; ++b) { mbar_init(BAR(B_QFULL + b), 1); mbar_init(BAR(B_QEMPTY + b), 1); }
    for (int i = 0; i < KSTAGES; ++i) { mbar_init(BAR(B_KFULL + i), 1); mbar_init(BAR(B_KEMPTY + i), 1); }
    for (int i = 0; i < VSTAGES; ++i) { mbar_init(BAR(B_VFULL + i), 1); mbar_init(BAR(B_VEMPTY + i), 1); }
    for (int t = 0; t < NQ; ++t) {
      mbar_init(BAR(B_SFULL + t), 1);
      mbar_init(BAR(B_PFULL + t), BLOCK_M);
      mbar_init(BAR(B_OFINAL + t), 1);
      mbar_init(BAR(B_OFREE + t), BLOCK_M);
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
      int nk = 0, nv = 0, nseg = 0;                // loads issued (K, V tiles; Q buffers)
      Seg sg{};
      auto load_k = [&](int kv) -> bool {
        const int s = nk % KSTAGES;
        if (nk >= KSTAGES &&
            !mbar_wait(BAR(B_KEMPTY + s), ((nk / KSTAGES) - 1) & 1, tlim, abort_flag, args.err))
          return false;
        // a tile starting past the sequence would load zeros: an index error (recorded; the
        // load itself stays in the tensor map's bounds checking)
        (void)QATTN_IN_BOUNDS(args.err, kv * BLOCK_N < sg.seq_len);
        mbar_arrive_expect_tx(BAR(B_KFULL + s), SL::TILE_KV);
        tma_load_3d(base_u32 + SL::OFF_K + s * SL::TILE_KV, &tm_k, BAR(B_KFULL + s), 0,
                    sg.seq_start + kv * BLOCK_N, sg.slab);
        ++nk;
        return true;
      };
      auto load_v = [&](int kv) -> bool {
        const int s = nv % VSTAGES;
        if (nv >= VSTAGES &&
            !mbar_wait(BAR(B_VEMPTY + s), ((nv / VSTAGES) - 1) & 1, tlim, abort_flag, args.err))
          return false;
        (void)QATTN_IN_BOUNDS(args.err, kv * BLOCK_N < sg.seq_len);
        mbar_arrive_expect_tx(BAR(B_VFULL + s), SL::TILE_KV);
        tma_load_3d(base_u32 + SL::OFF_V + s * SL::TILE_KV, &tm_v, BAR(B_VFULL + s), 0,
                    sg.seq_start + kv * BLOCK_N, sg.slab);
        ++nv;
        return true;
      };
      bool ok = true;
      for (int i = 0; ok && get_segment(args, i, sg); ++i) {
        // Q buffer i % 2: free once the MMAs of segment i - 2 that read it have completed
        const int b = i & 1;
        if (i >= 2 && !mbar_wait(BAR(B_QEMPTY + b), ((i >> 1) - 1) & 1, tlim, abort_flag, args.err))
          break;
        (void)QATTN_IN_BOUNDS(args.err, sg.q_row0 < sg.seq_len && sg.slab < args.slabs &&
                                            sg.seq_start + sg.seq_len <= args.rows_per_slab);
        mbar_arrive_expect_tx(BAR(B_QFULL + b), NQ * SL::TILE_Q);
        for (int t = 0; t < NQ; ++t)
          tma_load_3d(base_u32 + SL::OFF_Q + (b * NQ + t) * SL::TILE_Q, &tm_q, BAR(B_QFULL + b), 0,
                      sg.seq_start + sg.q_row0 + t * BLOCK_M, sg.slab);
        ++nseg;
        // order of use on the tensor pipe: K0, V0, K1, V1, ...; K runs one tile ahead
        const int n = sg.kv1 - sg.kv0;
        ok = load_k(sg.kv0);
        for (int j = 0; ok && j < n; ++j) {
          if (j + 1 < n) ok = load_k(sg.kv0 + j + 1);
          if (ok) ok = load_v(sg.kv0 + j);
        }
      }
      // drain: every issued load has landed before the CTA may exit (instant when healthy)
      for (int i = nseg - 1; i >= 0 && i >= nseg - 2; --i)
        mbar_drain(BAR(B_QFULL + (i & 1)), (i >> 1) & 1, tlim);
      for (int j = nk - 1; j >= 0 && j >= nk - KSTAGES; --j)
        mbar_drain(BAR(B_KFULL + j % KSTAGES), (j / KSTAGES) & 1, tlim);
      for (int j = nv - 1; j >= 0 && j >= nv - VSTAGES; --j)
        mbar_drain(BAR(B_VFULL + j % VSTAGES), (j / VSTAGES) & 1, tlim);
    }
  } else if (warp == WARP_MMA) {
    // ======================= MMA issuer =======================
    if (lane == 0) {
      constexpr uint32_t IDESC_S = idesc_e4m3_f32(BLOCK_M, BLOCK_N, false);
      // Q, K: K-major rows of D bytes, swizzled in 8-row atoms (SBO = 8 rows); 32-byte K steps.
      constexpr uint32_t QK_LAYOUT = (D == 128) ? 2u : 4u;   // 128B / 64B swizzle
      constexpr uint32_t QK_SBO = 8 * D;
      // V: MN-major (D contiguous per key row), rows of D bytes, SBO = 8 key rows; a K step
      // of 32 keys advances 32 rows.
      constexpr uint32_t V_LAYOUT = QK_LAYOUT;
      constexpr uint32_t V_SBO = 8 * D;
      auto bmm1 = [&](int t, int qb, int ks) {
        const uint32_t qa = base_u32 + SL::OFF_Q + (qb * NQ + t) * SL::TILE_Q;
        const uint32_t kb = base_u32 + SL::OFF_K + ks * SL::TILE_KV;
#pragma unroll
        for (int kk = 0; kk < D / 32; ++kk) {
          const uint64_t da = smem_desc(qa + kk * 32, 16, QK_SBO, QK_LAYOUT);
          const uint64_t db = smem_desc(kb + kk * 32, 16, QK_SBO, QK_LAYOUT);
          mma_f8_ss(tmem + TC::S0 + t * BLOCK_N, da, db, IDESC_S, kk > 0 ? 1u : 0u);
        }
      };
      // O_t += (P_t 2^(M - M_ref)) V: the per-row power of two rides on BMM2 as an E8M0 scale
      // factor of P, written by the softmax with P; V's factors are all 2^0
      auto bmm2 = [&](int t, int vs, bool first) {
        const uint32_t vb = base_u32 + SL::OFF_V + vs * SL::TILE_KV;
        const uint32_t sfa = tmem + TC::S0 + t * BLOCK_N + TC::SFA;
        const uint32_t sfb = tmem + TC::S0 + t * BLOCK_N + TC::SFB;
#pragma unroll
        for (int kk = 0; kk < BLOCK_N / 32; ++kk) {
          const uint64_t db = smem_desc(vb + kk * 32 * D, SL::TILE_KV, V_SBO, V_LAYOUT);
          mma_mxf8_ts(tmem + TC::O0 + t * D, tmem + TC::S0 + t * BLOCK_N + kk * 8, db,
                      idesc_mxf8_e4m3(BLOCK_M, D, true, static_cast<uint32_t>(kk)), sfa, sfb,
                      (!first || kk > 0) ? 1u : 0u);
        }
      };
      int nk = 0, nv = 0, step = 0;               // K, V tiles consumed; key steps before this segment
      bool ok = true;
      Seg sg{};
      for (int i = 0; ok && get_segment(args, i, sg); ++i) {
        const int qb = i & 1;
        const int n = sg.kv1 - sg.kv0;
        // S_t of the segment's first key step (S_t is free: the last P V of the previous
        // segment, which read P_t from it, precedes in the MMA stream)
        ok = mbar_wait(BAR(B_QFULL + qb), (i >> 1) & 1, tlim, abort_flag, args.err) &&
             mbar_wait(BAR(B_KFULL + nk % KSTAGES), (nk / KSTAGES) & 1, tlim, abort_flag, args.err);
        if (!ok) break;
        tc_fence_after();
        for (int t = 0; t < NQ; ++t) {
          bmm1(t, qb, nk % KSTAGES);
          mma_commit(BAR(B_SFULL + t));
        }
        mma_commit(BAR(B_KEMPTY + nk % KSTAGES));
        ++nk;
        // the first P V of this segment overwrites O_t: softmax t has read out the last one
        for (int t = 0; ok && i > 0 && t < NQ; ++t)
          ok = mbar_wait(BAR(B_OFREE + t), (i - 1) & 1, tlim, abort_flag, args.err);
        const int pbase = step & 1;
        for (int j = 0; ok && j < n; ++j) {
          const int vs = nv % VSTAGES;
          const bool more = j + 1 < n;
          const int ks = nk % KSTAGES;
          ok = mbar_wait(BAR(B_VFULL + vs), (nv / VSTAGES) & 1, tlim, abort_flag, args.err);
          if (ok && more)
            ok = mbar_wait(BAR(B_KFULL + ks), (nk / KSTAGES) & 1, tlim, abort_flag, args.err);
          for (int t = 0; ok && t < NQ; ++t) {
            ok = mbar_wait(BAR(B_PFULL + t), pbase ^ (j & 1), tlim, abort_flag, args.err);
            if (!ok) break;
            tc_fence_after();
            bmm2(t, vs, j == 0);                   // reads P_t from TMEM
            if (more) {
              bmm1(t, qb, ks);                     // overwrites S_t / P_t after bmm2 read it
              mma_commit(BAR(B_SFULL + t));
            } else {
              mma_commit(BAR(B_OFINAL + t));
            }
          }
          if (ok) {
            mma_commit(BAR(B_VEMPTY + vs));
            ++nv;
            if (more) {
              mma_commit(BAR(B_KEMPTY + ks));
              ++nk;
            }
          }
        }
        if (ok) mma_commit(BAR(B_QEMPTY + qb));   // every MMA reading Q buffer qb is issued
        step += n;
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
    bool ok = true;
    int step = 0;                                  // key steps of the earlier segments
    Seg sg{};
    for (int seg = 0; ok && get_segment(args, seg, sg); ++seg) {
    const int n = sg.kv1 - sg.kv0;
    float m_run = -INFINITY;                       // integer-valued running max (base 2)
    float m_ref = 0.0f;                            // O_t holds sum_j P(j) V 2^(m_j - m_ref)
    float l = 0.0f;                                // running sum of p * 448 (relative to m_run)
    for (int j = 0; j < n; ++j) {
      // S_t(j) is in TMEM; BMM2 of tile j-1 has completed (it precedes in the MMA stream)
      ok = mbar_wait(BAR(B_SFULL + t), (step + j) & 1, tlim, abort_flag, args.err);
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
      const int kv_valid = sg.seq_len - (sg.kv0 + j) * BLOCK_N;  // keys of this tile in the sequence
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
      if constexpr (CAPTURE) {                                                  // test hook
        if (sg.slab == args.dbg_slab && sg.seq_start + sg.q_row0 + t * BLOCK_M + r == args.dbg_row &&
            QATTN_IN_BOUNDS(args.err, sg.kv0 + j < args.dbg_steps))
          capture_p_codes(args.dbg_p, args.dbg_m, sg.kv0 + j, pk, m_new);
      }
      const float rowsum = ((acc[0] + acc[1]) + (acc[2] + acc[3])) + ((acc[4] + acc[5]) + (acc[6] + acc[7]));
      // P(j) is relative to m_new and enters O scaled by 2^(m_new - m_ref) (BMM2's scale factor),
      // so a rise of the running max leaves O alone.  Only a gap beyond 2^64, which could carry
      // O past the FP32 range, rescales this row of O (quiescent: its last BMM2 is done) and
      // moves m_ref up.
      if (j == 0) {
        m_ref = m_new;
      } else {
        l *= exp2_int(static_cast<int>(m_run - m_new));
        const bool far = m_new - m_ref > 64.0f;
        if (__any_sync(0xFFFFFFFFu, far)) {
          const float f = far ? exp2_int(static_cast<int>(m_ref - m_new)) : 1.0f;
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
          if (far) m_ref = m_new;
        }
      }
      l += rowsum;
      m_run = m_new;
      // P_t(j) over the first 32 columns of S_t: column c holds keys 4c..4c+3 (byte = key % 4).
      // BMM2's scale factors: the MMA reads row r's factor of P from lane r, column r / 32 of
      // the SFA block (one byte per 32 keys), so each thread writes only that column of its own
      // lane: its row's 2^(m_new - m_ref) (E8M0 code 127 + gap) in all four bytes.  V's block
      // (2^0, code 127) is read by every lane quarter for all D columns: four columns per lane.
      tmem_st32(tS, pk);
      tmem_st1(tS + TC::SFA + quarter, (127u + static_cast<uint32_t>(m_new - m_ref)) * 0x01010101u);
      tmem_st4_same(tS + TC::SFB, 0x7F7F7F7Fu);
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(BAR(B_PFULL + t));
    }
    if (!ok) break;
    {
      ok = mbar_wait(BAR(B_OFINAL + t), seg & 1, tlim, abort_flag, args.err);
      if (!__all_sync(0xFFFFFFFFu, ok)) { ok = false; break; }
      {
        tc_fence_after();
        const int row = sg.q_row0 + t * BLOCK_M + r;
        const bool valid = row < sg.seq_len;
        const float f_ref = exp2_int(static_cast<int>(m_ref - m_run));   // O relative to m_run
        if (sg.slot >= 0 && QATTN_IN_BOUNDS(args.err, (static_cast<long long>(sg.slot) * NQ + t + 1) *
                                                          BLOCK_M <= args.part_rows)) {
          // partial result of this segment: raw O row, running max and row sum
          const size_t slot = static_cast<size_t>(sg.slot) * NQ + t;
          float4* po = reinterpret_cast<float4*>(args.part_o + (slot * BLOCK_M + r) * D);
#pragma unroll
          for (int c4 = 0; c4 < D / 32; ++c4) {
            uint32_t v[32];
            tmem_ld32(tO + c4 * 32, v);
            tmem_wait_ld();
#pragma unroll
            for (int i = 0; i < 8; ++i)
              po[c4 * 8 + i] = make_float4(__uint_as_float(v[4 * i]) * f_ref, __uint_as_float(v[4 * i + 1]) * f_ref,
                                           __uint_as_float(v[4 * i + 2]) * f_ref, __uint_as_float(v[4 * i + 3]) * f_ref);
          }
          args.part_ml[slot * BLOCK_M + r] = make_float2(m_run, l);
        } else if (sg.slot < 0) {
        const float scale = __ldg(args.s_v) / l * f_ref;   // O = acc * s_v / 448 / (l / 448)
        __nv_bfloat16* orow =
            args.out + (static_cast<size_t>(sg.slab) * args.rows_per_slab + sg.seq_start + row) * D;
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
          if (valid && QATTN_IN_BOUNDS(args.err, static_cast<long long>(sg.slab) * args.rows_per_slab +
                                                     sg.seq_start + row < static_cast<long long>(args.slabs) * args.rows_per_slab)) {
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
    mbar_arrive(BAR(B_OFREE + t));                 // O_t is read out: the next segment may overwrite it
    step += n;
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
// Combine of the tail pairs the persistent schedule cut: one warp per output row (COMBINE_WARPS
// rows per CTA), each lane D / 32 columns.  Tail pair tp spans the key steps
// [tp * nkv, (tp + 1) * nkv) of the tail, so its parts are those of CTAs
// c_first = tp * nkv / tail_w .. c_last = ((tp + 1) * nkv - 1) / tail_w; CTA c's part sits in
// slot 2c + 1 if the CTA started in an earlier pair, else in slot 2c.  The parts' running maxima
// are integers, so each part is brought to the common maximum M by an exact power of two:
// O = sum_p 2^(m_p - M) O_p, l = sum_p 2^(m_p - M) l_p, out = O * s_v / l.
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
  if (tp >= args.tail_pairs) return;
  const long long W = args.tail_w, nkv = args.nkv, g0 = tp * nkv;
  const int c_first = static_cast<int>(g0 / W);
  const int c_last = static_cast<int>((g0 + nkv - 1) / W);
  if (c_first == c_last) return;                  // one CTA ran the whole pair and wrote it
  const int pair = args.whole * args.ctas + tp;
  const int qblk = pair % args.pairs_per_head;
  const int h = (pair / args.pairs_per_head) % args.H;
  const int bz = pair / (args.pairs_per_head * args.H);
  const int row = qblk * (NQ * BLOCK_M) + t * BLOCK_M + r;
  if (row >= args.L) return;
  auto slot = [&](int c) {
    return static_cast<size_t>(2 * c + (c * W < g0 ? 1 : 0)) * NQ + t;
  };
  if (!QATTN_IN_BOUNDS(args.err, c_first >= 0 && c_last < args.ctas &&
                                     static_cast<long long>(slot(c_last) + 1) * BLOCK_M <= args.part_rows &&
                                     static_cast<long long>(bz * args.H + h) < args.slabs))
    return;
  float M = -INFINITY;
  for (int c = c_first; c <= c_last; ++c) M = fmaxf(M, args.part_ml[slot(c) * BLOCK_M + r].x);
  float l = 0.0f;
  float acc[VEC];
#pragma unroll
  for (int i = 0; i < VEC; ++i) acc[i] = 0.0f;
  for (int c = c_first; c <= c_last; ++c) {
    const float2 ml = args.part_ml[slot(c) * BLOCK_M + r];
    const float w = exp2_int(static_cast<int>(ml.x - M));
    l = fmaf(w, ml.y, l);
    const float* po = args.part_o + (slot(c) * BLOCK_M + r) * D + lane * VEC;
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

// 3-D map over an E4M3 tensor viewed as [slabs][rows][D]: box = one 128-row tile of one slab.
static bool make_map(CUtensorMap* map, const void* ptr, int D, int rows, int slabs) {
  EncodeTiledFn enc = encode_tiled_fn();
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
  static DeviceOnce smem_attr;                  // per device and per D, set once (both instances)
  const cudaError_t ea = static_cast<cudaError_t>(smem_attr.get([] {
    cudaError_t e0 = cudaFuncSetAttribute(k_attn_fp8_fwd<D, false>,
                                          cudaFuncAttributeMaxDynamicSharedMemorySize, Smem<D>::ALLOC);
    if (e0 == cudaSuccess)
      e0 = cudaFuncSetAttribute(k_attn_fp8_fwd<D, true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                Smem<D>::ALLOC);
    return static_cast<int>(e0);
  }));
  if (ea != cudaSuccess) return ea;
  if (a.dbg_p != nullptr)
    k_attn_fp8_fwd<D, true><<<grid, ATTN_THREADS, Smem<D>::ALLOC, stream>>>(mq, mk, mv, a);
  else
    k_attn_fp8_fwd<D, false><<<grid, ATTN_THREADS, Smem<D>::ALLOC, stream>>>(mq, mk, mv, a);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess || combine_ctas == 0) return e;
  k_attn_combine<D><<<combine_ctas, COMBINE_WARPS * 32, 0, stream>>>(a);
  return cudaGetLastError();
}

// Persistent plan of a dense launch: ctas = one CTA per SM (fewer when the work is small); each
// CTA takes `whole` whole pairs, and the key steps of the remaining tail pairs, laid end to end,
// are cut into equal contiguous ranges of tail_w steps, one per CTA, so every CTA runs the same
// number of key steps to within one range.  A range is at least a quarter of a pair (a cut pair
// has a handful of parts at most) and at most one pair; when the even share would be 0.8 of a
// pair or more, or would save fewer than 4 key steps, the tail pairs stay whole (one per CTA).
// bytes = the workspace the cut pairs' partial results need (0: no pair is cut).
#ifndef QATTN_TAIL_MIN_DIV
#define QATTN_TAIL_MIN_DIV 4        // a tail range is at least 1/QATTN_TAIL_MIN_DIV of a pair
#endif
AttnSplitPlan plan_attention_split(int B, int H, int L, int D, int num_sms) {
  AttnSplitPlan p;
  p.pairs_per_head = (L + NQ * BLOCK_M - 1) / (NQ * BLOCK_M);
  const long long pairs = static_cast<long long>(p.pairs_per_head) * H * B;
  p.nkv = (L + BLOCK_N - 1) / BLOCK_N;
  const long long steps = pairs * p.nkv;
  const int wmin = (p.nkv + QATTN_TAIL_MIN_DIV - 1) / QATTN_TAIL_MIN_DIV;
  const long long want = (steps + wmin - 1) / wmin;
  p.ctas = static_cast<int>(want < num_sms ? want : num_sms);
  if (p.ctas < 1) p.ctas = 1;
  p.whole = static_cast<int>(pairs / p.ctas);
  p.tail_pairs = static_cast<int>(pairs - static_cast<long long>(p.whole) * p.ctas);
  const long long even =
      (static_cast<long long>(p.tail_pairs) * p.nkv + p.ctas - 1) / p.ctas;
  p.tail_w = p.tail_pairs > 0 ? static_cast<int>(even > wmin ? even : wmin) : p.nkv;
  // cutting costs partial results and a combine launch: worth it only when it shortens the
  // tail to less than 0.8 of a whole pair and by at least 4 key steps
  if (p.tail_w * 5 >= p.nkv * 4 || p.nkv - p.tail_w < 4) p.tail_w = p.nkv;
  if (p.tail_w == p.nkv && p.whole == 0) {      // fewer pairs than CTAs: one CTA per pair
    p.ctas = p.tail_pairs;
    p.whole = 1;
    p.tail_pairs = 0;
  }
  p.bytes = p.tail_w < p.nkv
                ? static_cast<size_t>(2) * p.ctas * NQ * BLOCK_M * (D + 2) * sizeof(float)
                : 0;
  return p;
}

AttnSplitPlan attention_plan(int B, int H, int L, int D, int num_sms, bool pair) {
  return plan_attention_split(B, H, L, D, (D == 128 && pair) ? attention_pair_units(num_sms) : num_sms);
}

cudaError_t launch_attention(const uint8_t* q8, const uint8_t* k8, const uint8_t* v8, void* out,
                             int B, int H, int L, int D, const int* cu_seqlens, int nseq,
                             int max_seqlen, int total_tokens, const float* s_q, const float* s_k,
                             const float* s_v, float sm_scale, int* err, uint64_t timeout_ns,
                             const DebugHooks& dbg, void* workspace, size_t workspace_bytes,
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
  a.inject_missing_q = dbg.inject_missing_q;
  a.part_o = nullptr;
  a.part_ml = nullptr;
  a.part_rows = 0;
  a.dbg_p = dbg.p_codes;
  a.dbg_m = dbg.p_maxima;
  a.dbg_slab = dbg.p_slab;
  a.dbg_row = dbg.p_row;
  a.dbg_steps = ((varlen ? max_seqlen : L) + BLOCK_N - 1) / BLOCK_N;
  a.pairs_per_head = 0;
  a.nkv = 0;
  a.ctas = 0;
  a.whole = 0;
  a.tail_pairs = 0;
  a.tail_w = 1;
  const int slabs = varlen ? H : B * H;
  const bool pair = D == 128 && dbg.attn_pair != 0;   // the pair-of-SMs variant, when selected
  a.slabs = slabs;
  dim3 grid;
  int combine_ctas = 0;
  AttnSplitPlan p{};
  if (varlen) {
    grid = dim3((max_seqlen + NQ * BLOCK_M - 1) / (NQ * BLOCK_M), H, nseq);
  } else {
    p = attention_plan(B, H, L, D, num_sms, pair);
    if (workspace == nullptr || workspace_bytes < p.bytes) {   // no workspace: no pair is cut
      p.tail_w = p.nkv;
      p.bytes = 0;
    }
    a.pairs_per_head = p.pairs_per_head;
    a.nkv = p.nkv;
    a.ctas = p.ctas;
    a.whole = p.whole;
    a.tail_pairs = p.tail_pairs;
    a.tail_w = p.tail_w;
    if (p.bytes > 0) {
      const size_t o_elems = static_cast<size_t>(2) * p.ctas * NQ * BLOCK_M * D;
      a.part_o = static_cast<float*>(workspace);
      a.part_ml = reinterpret_cast<float2*>(a.part_o + o_elems);
      a.part_rows = static_cast<long long>(2) * p.ctas * NQ * BLOCK_M;
      combine_ctas = p.tail_pairs * NQ * BLOCK_M / COMBINE_WARPS;
    }
    grid = dim3(p.ctas, 1, 1);
  }
  if (pair) {
    // pairs of SMs: the two Q tiles of a pair on the two CTAs of a cluster (attn_pair.cu)
    cudaError_t e = launch_attention_pair(q8, k8, v8, out, H, L, cu_seqlens, nseq, max_seqlen,
                                          a.rows_per_slab, slabs, s_q, s_k, s_v, sm_scale, err,
                                          timeout_ns, dbg, varlen ? nullptr : &p,
                                          a.part_o, stream);
    if (e != cudaSuccess || combine_ctas == 0) return e;
    k_attn_combine<128><<<combine_ctas, COMBINE_WARPS * 32, 0, stream>>>(a);
    return cudaGetLastError();
  }
  if (D == 128)
    return launch_attn_d<128>(q8, k8, v8, a, a.rows_per_slab, slabs, grid, combine_ctas, stream);
  return launch_attn_d<64>(q8, k8, v8, a, a.rows_per_slab, slabs, grid, combine_ctas, stream);
}

}  // namespace qattn
