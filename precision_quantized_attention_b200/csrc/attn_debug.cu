// attn_debug.cu -- the attention with P quantization switched off, a debug path.
//
// The method's BMM2 reads P as E4M3 codes (NVIDIA developer blog "Optimizing FLUX.1 Kontext for
// Image Editing with Low-Precision Quantization", "Workflow and quantization", fourth SDPA bullet
// and Fig. 4).  With QATTN_FLAG_P_UNQUANTIZED in the mode, the forward calls run this kernel
// instead: the same Q, K, V codes and scales, the same FP32 softmax with the integer row maximum,
// but P stays FP32 and BMM2 accumulates p * v in FP32:
//   S'_j = fl32(acc_j * c)   acc_j = sum_d val(q_d) val(k_jd) in FP32,  c = s_q s_k sm_scale log2 e
//   M    = ceil(max_j S'_j),  p_j = 2^fl32(S'_j - M),  l = sum_j p_j
//   O_d  = (sum_j p_j val(v_jd)) * s_v / l
// It separates the error of the P quantization from the rest (the tensor quantization and the
// FP32 softmax).  A plain CUDA-core kernel, not tuned: two passes over the keys (the first finds
// M, the second forms p, l and O), 16 query rows per block, keys staged 32 at a time in shared
// memory as FP32 values.
#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <cstdint>

#include "launch.h"
#include "sm100_ptx.cuh"
#include "softmax_sm100.cuh"

namespace qattn {

namespace dbgk {
constexpr int QR = 16;        // query rows per block (4 per warp)
constexpr int KT = 32;        // keys per tile (one per lane)
constexpr int THREADS = 128;
}  // namespace dbgk

struct PlainArgs {
  const uint8_t* q8;
  const uint8_t* k8;
  const uint8_t* v8;
  __nv_bfloat16* out;
  int rows_per_slab;        // L (dense) or the packed token count (varlen)
  int L;                    // dense sequence length
  const int* cu_seqlens;    // varlen: device [nseq + 1]; nullptr for dense
  const float* s_q;
  const float* s_k;
  const float* s_v;
  float sm_scale;
};

template <int D>
__global__ void __launch_bounds__(dbgk::THREADS) k_attn_p_unquantized(const PlainArgs a) {
  using namespace dbgk;
  constexpr int CPL = D / 32;                       // output columns per lane
  __shared__ float sq[QR][D];
  __shared__ float sk[KT][D + 1];
  __shared__ float sv[KT][D];
  __shared__ float sp[QR][KT];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int slab = blockIdx.y;
  int seq_start = 0, seq_len = a.L;
  if (a.cu_seqlens) {
    seq_start = __ldg(a.cu_seqlens + blockIdx.z);
    seq_len = __ldg(a.cu_seqlens + blockIdx.z + 1) - seq_start;
  }
  const int row0 = blockIdx.x * QR;
  if (row0 >= seq_len) return;
  const size_t base = (static_cast<size_t>(slab) * a.rows_per_slab + seq_start) * D;
  const float c = __ldg(a.s_q) * __ldg(a.s_k) * a.sm_scale * LOG2E_F;

  for (int i = threadIdx.x; i < QR * D; i += THREADS) {
    const int r = i / D, d = i % D;
    sq[r][d] = row0 + r < seq_len ? e4m3_to_f32(a.q8[base + static_cast<size_t>(row0 + r) * D + d]) : 0.0f;
  }
  auto load_tile = [&](int key0, bool with_v) {
    for (int i = threadIdx.x; i < KT * D; i += THREADS) {
      const int j = i / D, d = i % D;
      const bool in = key0 + j < seq_len;
      const size_t off = base + static_cast<size_t>(key0 + j) * D + d;
      sk[j][d] = in ? e4m3_to_f32(a.k8[off]) : 0.0f;
      if (with_v) sv[j][d] = in ? e4m3_to_f32(a.v8[off]) : 0.0f;
    }
  };
  // S' of key `key` (this lane's key of the tile) for the warp's row r
  auto score = [&](int r) {
    float acc = 0.0f;
#pragma unroll 8
    for (int d = 0; d < D; ++d) acc = __fmaf_rn(sq[r][d], sk[lane][d], acc);
    return __fmul_rn(acc, c);
  };

  // pass 1: the row maxima
  float mrow[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
  for (int key0 = 0; key0 < seq_len; key0 += KT) {
    __syncthreads();
    load_tile(key0, false);
    __syncthreads();
    if (key0 + lane < seq_len) {
#pragma unroll
      for (int i = 0; i < 4; ++i) mrow[i] = fmaxf(mrow[i], score(warp * 4 + i));
    }
  }
  float M[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    float m = mrow[i];
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xFFFFFFFFu, m, o));
    M[i] = ceilf(m);
  }

  // pass 2: p, the row sums and P V
  float lpart[4] = {0.f, 0.f, 0.f, 0.f};
  float o[4][CPL];
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int k = 0; k < CPL; ++k) o[i][k] = 0.0f;
  for (int key0 = 0; key0 < seq_len; key0 += KT) {
    __syncthreads();
    load_tile(key0, true);
    __syncthreads();
    const bool in = key0 + lane < seq_len;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float p = in ? exp2f(__fsub_rn(score(warp * 4 + i), M[i])) : 0.0f;
      lpart[i] += p;
      sp[warp * 4 + i][lane] = p;
    }
    __syncwarp();
#pragma unroll 4
    for (int j = 0; j < KT; ++j) {
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const float p = sp[warp * 4 + i][j];
#pragma unroll
        for (int k = 0; k < CPL; ++k) o[i][k] = __fmaf_rn(p, sv[j][lane + 32 * k], o[i][k]);
      }
    }
    __syncwarp();
  }
  const float s_v = __ldg(a.s_v);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    float l = lpart[i];
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) l += __shfl_xor_sync(0xFFFFFFFFu, l, off);
    const int row = row0 + warp * 4 + i;
    if (row < seq_len) {
      const float scale = s_v / l;
#pragma unroll
      for (int k = 0; k < CPL; ++k)
        a.out[base + static_cast<size_t>(row) * D + lane + 32 * k] = __float2bfloat16_rn(o[i][k] * scale);
    }
  }
}

cudaError_t launch_attention_p_unquantized(const uint8_t* q8, const uint8_t* k8, const uint8_t* v8,
                                           void* out, int B, int H, int L, int D,
                                           const int* cu_seqlens, int nseq, int max_seqlen,
                                           int total_tokens, const float* s_q, const float* s_k,
                                           const float* s_v, float sm_scale, cudaStream_t stream) {
  PlainArgs a;
  a.q8 = q8;
  a.k8 = k8;
  a.v8 = v8;
  a.out = static_cast<__nv_bfloat16*>(out);
  const bool varlen = cu_seqlens != nullptr;
  a.rows_per_slab = varlen ? total_tokens : L;
  a.L = L;
  a.cu_seqlens = cu_seqlens;
  a.s_q = s_q;
  a.s_k = s_k;
  a.s_v = s_v;
  a.sm_scale = sm_scale;
  const int rows = varlen ? max_seqlen : L;
  const dim3 grid((rows + dbgk::QR - 1) / dbgk::QR, varlen ? H : B * H, varlen ? nseq : 1);
  if (D == 128)
    k_attn_p_unquantized<128><<<grid, dbgk::THREADS, 0, stream>>>(a);
  else
    k_attn_p_unquantized<64><<<grid, dbgk::THREADS, 0, stream>>>(a);
  return cudaGetLastError();
}

}  // namespace qattn
