// launch.h -- host-side launchers of the kernels in quant.cu and attn_fwd.cu, called by the C ABI
// layer (qattn_api.cu) after it has validated the arguments.  Internal to the library.
#pragma once

#include <cuda_runtime.h>

#include <cstddef>
#include <cstdint>

namespace qattn {

cudaError_t launch_amax(const void* x, size_t n, float* amax, int* err, int num_sms,
                        cudaStream_t stream);
cudaError_t launch_quant_fp8(const void* x, size_t n, const float* amax, uint8_t* out,
                             float* scale, int* err, int num_sms, cudaStream_t stream,
                             int inject_oob = 0);
cudaError_t launch_quant_fp4_block(const void* x, size_t n, const float* amax, uint8_t* packed,
                                   uint8_t* bscale, float* gscale, uint8_t* codes8, float* scale8,
                                   int* err, int num_sms, cudaStream_t stream);
cudaError_t launch_calib_quant_fp8(const void* x, size_t n, float* amax, uint8_t* out,
                                   float* scale, void* workspace, uint64_t limit_ns, int* err,
                                   int num_sms, cudaStream_t stream);
cudaError_t launch_calib_quant_fp4_block(const void* x, size_t n, float* amax, uint8_t* packed,
                                         uint8_t* bscale, float* gscale, uint8_t* codes8,
                                         float* scale8, void* workspace, uint64_t limit_ns,
                                         int* err, int num_sms, cudaStream_t stream);
cudaError_t launch_calib_quant_qkv(const void* const* x, uint8_t* const* codes8, float* const* amax,
                                   float* const* scale8, uint8_t* const* e2m1,
                                   uint8_t* const* bscale, float* const* gscale, size_t n, int mode,
                                   void* workspace, uint64_t limit_ns, int* err, int num_sms,
                                   cudaStream_t stream);

cudaError_t launch_quant_qkv(const void* const* x, uint8_t* const* codes8, float* const* amax,
                             float* const* scale8, uint8_t* const* e2m1, uint8_t* const* bscale,
                             float* const* gscale, size_t n, int mode, int* err, int num_sms,
                             cudaStream_t stream);

// Y[M, N] (bf16) = (A8[M, K] B8[N, K]^T) * s_a * s_b; K % 128 == 0, N % 32 == 0.  y may be null
// when codes are requested; codes (optional): the E4M3 codes of the bf16 Y under the given amax
// (scale s = amax / 448 written to *scale_out).
cudaError_t launch_gemm_fp8(const uint8_t* a8, const uint8_t* b8, void* y, int M, int N, int K,
                            const float* s_a, const float* s_b, int* err, uint64_t timeout_ns,
                            int num_sms, cudaStream_t stream, uint8_t* codes = nullptr,
                            const float* amax = nullptr, float* scale_out = nullptr);

// Test hooks of the attention launches (all off by default): inject_missing_q makes the producer
// never load anything (every wait then runs into its limit); p_codes != null makes the D = 128
// kernel copy, for the query row p_row of slab p_slab (row index within the slab's rows), the
// 128 E4M3 codes of P of every key step into p_codes[step * 128 + key] and the step's integer
// tile maximum into p_maxima[step].
struct DebugHooks {
  int inject_missing_q = 0;
  int attn_pair = 0;               // D = 128 launches run the pair-of-SMs kernel (attn_pair.cu)
  int inject_oob = 0;              // checked build only: qattn_quantize_fp8 loops one vector past n
  uint8_t* p_codes = nullptr;
  int* p_maxima = nullptr;
  int p_slab = -1;
  int p_row = -1;
};

// Per-block FP4 GEMM (gemm_fp4.cu): Y [M, N] bf16 = X W^T from packed E2M1 codes, E4M3 block
// scales (one per 16 K elements, row-major) and per-tensor scales.  K % 256 == 0, N % 32 == 0.
cudaError_t launch_gemm_fp4(const uint8_t* x, const uint8_t* sx, const float* sg_x, const uint8_t* w,
                            const uint8_t* sw, const float* sg_w, void* y, int M, int N, int K,
                            int* err, uint64_t timeout_ns, int num_sms, cudaStream_t stream);

// The attention with P left unquantized (QATTN_FLAG_P_UNQUANTIZED, a debug path; attn_debug.cu):
// dense (cu_seqlens == nullptr: B, H, L) or varlen (cu_seqlens, nseq, max_seqlen, total_tokens, H).
cudaError_t launch_attention_p_unquantized(const uint8_t* q8, const uint8_t* k8, const uint8_t* v8,
                                           void* out, int B, int H, int L, int D,
                                           const int* cu_seqlens, int nseq, int max_seqlen,
                                           int total_tokens, const float* s_q, const float* s_k,
                                           const float* s_v, float sm_scale, cudaStream_t stream);

// Persistent schedule of a dense attention launch (see plan_attention_split in attn_fwd.cu):
// ctas CTAs, `whole` whole pairs each, then tail ranges of tail_w key steps; bytes = workspace
// the cut tail pairs need (0: no pair is cut).
struct AttnSplitPlan {
  int pairs_per_head, nkv, ctas, whole, tail_pairs, tail_w;
  size_t bytes;
};
AttnSplitPlan plan_attention_split(int B, int H, int L, int D, int num_sms);

// Units of the persistent dense grid on the current device: SMs for the one-SM kernel,
// resident pair clusters for the pair kernel (D = 128, when selected); and the plan the launch
// uses for them.
int attention_pair_units(int num_sms);
AttnSplitPlan attention_plan(int B, int H, int L, int D, int num_sms, bool pair);

// The D = 128 pair kernel (attn_pair.cu): dense with `plan` (workspace may be null when the plan
// cuts no pair), or varlen with plan == nullptr.
cudaError_t launch_attention_pair(const uint8_t* q8, const uint8_t* k8, const uint8_t* v8, void* out,
                                  int H, int L, const int* cu_seqlens, int nseq, int max_seqlen,
                                  int rows_per_slab, int slabs, const float* s_q, const float* s_k,
                                  const float* s_v, float sm_scale, int* err, uint64_t timeout_ns,
                                  const DebugHooks& dbg, const AttnSplitPlan* plan, void* workspace,
                                  cudaStream_t stream);

// workspace may be null (no split); it is used only when workspace_bytes covers the plan.
cudaError_t launch_attention(const uint8_t* q8, const uint8_t* k8, const uint8_t* v8, void* out,
                             int B, int H, int L, int D, const int* cu_seqlens, int nseq,
                             int max_seqlen, int total_tokens, const float* s_q, const float* s_k,
                             const float* s_v, float sm_scale, int* err, uint64_t timeout_ns,
                             const DebugHooks& dbg, void* workspace, size_t workspace_bytes,
                             int num_sms, cudaStream_t stream);

}  // namespace qattn
