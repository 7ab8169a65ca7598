/*
 * qattn.h -- C ABI of libqattn, quantized scaled-dot-product attention for NVIDIA B200 (sm_100a).
 *
 * The operation is the quantized SDPA of the FLUX.1 Kontext transformer as described in the
 * NVIDIA developer blog "Optimizing FLUX.1 Kontext for Image Editing with Low-Precision
 * Quantization", section "Workflow and quantization" (the four SDPA bullets and Fig. 4):
 *   1. Q, K, V are FakeQuantized to per-tensor FP8 (E4M3), or to per-block FP4 (E2M1 values
 *      with E4M3 block scales and an FP32 tensor scale) followed by an extra per-tensor FP8
 *      quantize, because BMM1's inputs are FP8 in both modes;
 *   2. BMM1 = Q K^T in FP8 with FP32 accumulation;
 *   3. softmax in FP32, unquantized;
 *   4. P requantized to per-tensor FP8 (scale 1/448), BMM2 = P V in FP8.
 * Scales come from max-calibration of the tensor in hand (the blog's post-training
 * calibration step reduced to one tensor), or are given (static scales, qattn_quantize_qkv).
 * The block's linear layers around the attention (the blog quantizes them with the same
 * schemes) are here too: qattn_gemm_fp8 / qattn_gemm_fp8_e4m3 (per-tensor FP8) and
 * qattn_gemm_fp4 (per-block FP4).
 *
 * Conventions for every entry point:
 *   - Pointers named *_dev or tensor data are DEVICE pointers on the current CUDA device; the
 *     caller owns and allocates every buffer.  The library keeps no state besides one device
 *     error word per device, cached kernel attributes, the 256-byte static workspace of
 *     qattn_calibrate_quantize_fp8_noalloc and the settings of the qattn_debug_* hooks.
 *   - Work is enqueued on `stream` (0 = legacy default stream) and is asynchronous: scales and
 *     amax stay in device memory, nothing synchronizes with the host.  qattn_get_error() is the
 *     only call that synchronizes.
 *   - Argument errors are detected on the host before anything is launched and returned as
 *     QATTN_ERR_INVALID_ARG / QATTN_ERR_UNSUPPORTED; launch failures as QATTN_ERR_CUDA.  Errors
 *     found on the device (non-finite input, a timed-out wait, and in the checked build an
 *     index outside its buffer) are recorded in the device error word and reported by
 *     qattn_get_error().
 *   - Tensors are contiguous.  bf16 inputs are 16-byte aligned; E4M3 code buffers are 16-byte
 *     aligned (the attention kernel reads them with TMA).
 *   - Only sm_100 devices are supported (QATTN_ERR_UNSUPPORTED otherwise).
 */
#ifndef QATTN_H_
#define QATTN_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define QATTN_API __attribute__((visibility("default")))
#else
#define QATTN_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st* qattn_stream_t; /* a cudaStream_t */

typedef enum {
  QATTN_OK = 0,
  QATTN_ERR_INVALID_ARG = 1,
  QATTN_ERR_UNSUPPORTED = 2,
  QATTN_ERR_CUDA = 3,
  QATTN_ERR_NONFINITE = 4,
  QATTN_ERR_TIMEOUT = 5,
  /* checked build only (libqattn_checked.so): a kernel found an index outside its buffer and
   * skipped that access; the results are then incomplete */
  QATTN_ERR_BOUNDS = 6
} qattn_status;

typedef enum {
  QATTN_MODE_FP8 = 0,
  QATTN_MODE_FP4 = 1,
  /* Debug switch of the attention calls (qattn_forward, _ws, _varlen), OR'ed into the mode: P is
   * not quantized.  The same codes, scales and FP32 softmax with the integer row maximum M, but
   * BMM2 takes P in FP32: O = (sum_j p_j val(v_j)) * s_v / l with p_j = 2^fl32(S'_j - M) (the
   * blog's steps without the fourth SDPA bullet's P quantization), from a plain CUDA-core
   * kernel, not the tensor-core path: for isolating the error the P codes add.  The workspace
   * of qattn_forward_ws is not used. */
  QATTN_FLAG_P_UNQUANTIZED = 0x100
} qattn_mode;

/* Per-tensor dequantization multipliers of the E4M3 inputs of qattn_forward: value of an
 * element = val(code) * (*s).  All three are device pointers to one float each, as written by
 * qattn_quantize_fp8 (scale_dev) or qattn_quantize_fp4_block (scale8_dev). */
typedef struct {
  const float* s_q;
  const float* s_k;
  const float* s_v;
} qattn_scales;

/* Calibration: *amax_dev = max |x| over n bf16 elements, exactly.
 * Blog, "Workflow and quantization", flow steps 3-4 (post-training calibration), applied to the
 * tensor in hand.  x_bf16: device, n elements, 16-byte aligned.  amax_dev: device float, set to
 * 0 and then reduced into (so it must not be shared by concurrent calls).  A non-finite element
 * records QATTN_ERR_NONFINITE in the error word (amax is then inf or NaN). */
QATTN_API qattn_status qattn_calibrate_amax(const void* x_bf16, size_t n, float* amax_dev,
                                  qattn_stream_t stream);

/* Per-tensor FP8 FakeQuantize (blog, "Workflow and quantization", first SDPA bullet, Fig. 4):
 *   s = fl32(amax / 448) (s = 1 when amax == 0);  out[i] = e4m3(fl32(x[i] / s))
 * with round-to-nearest-even, saturation to +-448 and the sign kept.  x_bf16: device [n],
 * 16-byte aligned.  amax_dev: device float from qattn_calibrate_amax.  out_e4m3: device [n]
 * bytes, 8-byte aligned.  scale_dev: device float, receives s (the dequantization multiplier).
 * A non-finite amax records QATTN_ERR_NONFINITE and writes nothing. */
QATTN_API qattn_status qattn_quantize_fp8(const void* x_bf16, size_t n, const float* amax_dev,
                                uint8_t* out_e4m3, float* scale_dev, qattn_stream_t stream);

/* Per-block FP4 FakeQuantize fused with the per-tensor FP8 quantize of the dequantized values
 * (blog, "Workflow and quantization", first and second SDPA bullets; Fig. 4 "inputs quantized
 * with per-block FP4").  Blocks are 16 consecutive elements (along D of a [.., D] tensor):
 *   s_g  = fl32(amax / 2688)                        -> *gscale_dev
 *   s_b  = e4m3(fl32(amax_b / fl32(6 * s_g)))       -> blk_scale_e4m3[n / 16]
 *   c    = e2m1(fl32(x / fl32(val(s_b) * s_g)))     -> out_e2m1[n / 2] (element 2i in the low
 *                                                      nibble of byte i); 0 if that scale is 0
 *   xhat = fl32(fl32(val(c) * val(s_b)) * s_g)
 *   s8   = fl32(max|xhat| / 448)                    -> *scale8_dev
 *   c8   = e4m3(fl32(xhat / s8))                    -> out_e4m3_requant[n]
 * x_bf16: device [n], n % 16 == 0, 16-byte aligned.  out_e2m1 8-byte aligned,
 * out_e4m3_requant 16-byte aligned.  out_e4m3_requant and scale8_dev may both be NULL (FP4
 * codes only).  Non-finite amax: QATTN_ERR_NONFINITE recorded, nothing written. */
QATTN_API qattn_status qattn_quantize_fp4_block(const void* x_bf16, size_t n, const float* amax_dev,
                                      uint8_t* out_e2m1, uint8_t* blk_scale_e4m3,
                                      float* gscale_dev, uint8_t* out_e4m3_requant,
                                      float* scale8_dev, qattn_stream_t stream);

/* Bytes of device workspace the fused calibrate+quantize calls need (16-byte aligned). */
#define QATTN_FUSED_WORKSPACE_BYTES 256

/* Fused calibration + per-tensor FP8 FakeQuantize: the result of qattn_calibrate_amax followed by
 * qattn_quantize_fp8 (same definitions, same codes), computed by one cooperative kernel that
 * reads x from HBM once (the second pass reads it back from L2).  amax_dev receives the amax,
 * scale_dev the dequantization multiplier s.  workspace_dev: caller-owned device scratch of at
 * least QATTN_FUSED_WORKSPACE_BYTES bytes, 16-byte aligned, ZERO-FILLED before its first use;
 * every call that completes leaves it zero-filled again (after a call reported
 * QATTN_ERR_TIMEOUT, zero it again).  Calls that share a workspace must not overlap on the
 * device (stream order is enough; concurrent streams race).  n >= 1, x_bf16 16-byte aligned,
 * out_e4m3 8-byte aligned.  Non-finite input: QATTN_ERR_NONFINITE recorded, amax written, codes
 * and scale not written. */
QATTN_API qattn_status qattn_calibrate_quantize_fp8(const void* x_bf16, size_t n, float* amax_dev,
                                                    uint8_t* out_e4m3, float* scale_dev,
                                                    void* workspace_dev, size_t workspace_bytes,
                                                    qattn_stream_t stream);

/* Fused calibration + per-block FP4 FakeQuantize with the FP8 requant (the result of
 * qattn_calibrate_amax followed by qattn_quantize_fp4_block), one cooperative kernel; workspace
 * rules as for qattn_calibrate_quantize_fp8.  n % 16 == 0. */
QATTN_API qattn_status qattn_calibrate_quantize_fp4_block(
    const void* x_bf16, size_t n, float* amax_dev, uint8_t* out_e2m1, uint8_t* blk_scale_e4m3,
    float* gscale_dev, uint8_t* out_e4m3_requant, float* scale8_dev, void* workspace_dev,
    size_t workspace_bytes, qattn_stream_t stream);

/* Inputs and outputs of one tensor for qattn_calibrate_quantize_qkv (all device pointers).
 * FP8 mode: out_e4m3 receives the codes and scale_dev the multiplier s (as qattn_quantize_fp8);
 * out_e2m1, blk_scale_e4m3 and gscale_dev are ignored.  FP4 mode: the outputs of
 * qattn_quantize_fp4_block, out_e4m3 / scale_dev being the FP8 requant codes and multiplier. */
typedef struct {
  const void* x_bf16;        /* n bf16, 16-byte aligned */
  uint8_t* out_e4m3;         /* n bytes; 8-byte aligned (FP8) or 16-byte aligned (FP4) */
  float* amax_dev;           /* 1 float */
  float* scale_dev;          /* 1 float */
  uint8_t* out_e2m1;         /* FP4: n / 2 bytes, 8-byte aligned */
  uint8_t* blk_scale_e4m3;   /* FP4: n / 16 bytes */
  float* gscale_dev;         /* FP4: 1 float */
} qattn_quant_io;

/* Calibration + FakeQuantize of Q, K and V (three tensors of n elements each; io is a HOST
 * array of three descriptors, read during the call) in one cooperative kernel: each tensor gets
 * exactly the results of qattn_calibrate_amax followed by qattn_quantize_fp8 (mode FP8) or
 * qattn_quantize_fp4_block with the FP8 requant (mode FP4).  The kernel staggers the tensors:
 * while it quantizes one (read back from L2) it reduces the next one's amax from HBM.
 * Workspace rules as for qattn_calibrate_quantize_fp8 (QATTN_FUSED_WORKSPACE_BYTES, zero-filled
 * before first use, left zero-filled).  FP4 mode needs n % 16 == 0.  A tensor with a non-finite
 * element gets its amax written and nothing else; QATTN_ERR_NONFINITE is recorded; the other
 * tensors are still quantized. */
QATTN_API qattn_status qattn_calibrate_quantize_qkv(const qattn_quant_io* io, size_t n,
                                                    qattn_mode mode, void* workspace_dev,
                                                    size_t workspace_bytes, qattn_stream_t stream);

/* FakeQuantize of Q, K and V with GIVEN scales, in one launch: io[i].amax_dev is an INPUT here
 * (the amax of a calibration done earlier, as the blog's post-training quantization produces),
 * and each tensor gets exactly the results of qattn_quantize_fp8 (mode FP8) or
 * qattn_quantize_fp4_block with the FP8 requant (mode FP4) for that amax; the other io fields
 * are as for qattn_calibrate_quantize_qkv (io: HOST array of three descriptors, read during the
 * call).  No calibration pass and no workspace: one streaming read of each input.  FP4 mode
 * needs n % 16 == 0.  A non-finite amax writes nothing for that tensor and records
 * QATTN_ERR_NONFINITE. */
QATTN_API qattn_status qattn_quantize_qkv(const qattn_quant_io* io, size_t n, qattn_mode mode,
                                          qattn_stream_t stream);

/* FP8 GEMM of the transformer block's quantized linear layers (QKV and output projections,
 * MLP; the blog quantizes them with the same per-tensor FP8 FakeQuantize, "Workflow and
 * quantization"): Y = X W^T with X8 [M, K] and W8 [N, K] E4M3 codes (K contiguous, row-major),
 *   y_bf16[m, n] = bf16( (sum_k val(a8[m, k]) * val(b8[n, k])) * fl32(s_a * s_b) ),
 * products accumulated in FP32 on the tensor cores.  s_a_dev, s_b_dev: device floats (the
 * dequantization multipliers, e.g. from qattn_quantize_fp8).  Needs K % 128 == 0 and
 * N % 32 == 0 (M arbitrary); a8, b8, y_bf16 16-byte aligned; y_bf16 is [M, N] row-major.
 * M > 128 runs on pairs of SMs (256 x 256 tiles, one MMA over both SMs), M <= 128 on one SM per
 * 128 x 256 tile; both give the same result for every element (the same FP32 products are summed
 * in the same K order). */
QATTN_API qattn_status qattn_gemm_fp8(const uint8_t* a8, const uint8_t* b8, void* y_bf16, int M,
                                      int N, int K, const float* s_a_dev, const float* s_b_dev,
                                      qattn_stream_t stream);

/* The same GEMM with the per-tensor FP8 FakeQuantize of its output fused into the epilogue, for
 * a projection whose output goes straight to the quantized attention (the value projection: no
 * RoPE or normalization lies between it and SDPA).  The scale is static, from a given amax (the
 * blog's post-training calibration, "Workflow and quantization", flow steps 3-4):
 *   s = fl32(amax / 448) (amax == 0: s = 1), written to *scale_out_dev;
 *   codes_out[m, n] = e4m3(fl32(y[m, n] / s)), y[m, n] the bf16 value qattn_gemm_fp8 computes,
 * i.e. exactly what qattn_quantize_fp8(y, amax) would write from that bf16 output (round to
 * nearest even, saturating; values above the amax saturate).  y_bf16 may be null (codes only)
 * or receive the bf16 output as well.  codes_out: [M, N] bytes, 16-byte aligned; amax_dev,
 * scale_out_dev: device floats.  A non-finite amax writes no code and records
 * QATTN_ERR_NONFINITE (qattn_get_error).  Other requirements as qattn_gemm_fp8. */
QATTN_API qattn_status qattn_gemm_fp8_e4m3(const uint8_t* a8, const uint8_t* b8, void* y_bf16,
                                           uint8_t* codes_out, int M, int N, int K,
                                           const float* s_a_dev, const float* s_b_dev,
                                           const float* amax_dev, float* scale_out_dev,
                                           qattn_stream_t stream);

/* The block's linear layers in the per-block FP4 format (the blog's per-block FP4 quant config,
 * "Workflow and quantization"; Fig. 3): Y = X W^T with
 *   Y[m, n] = bf16((sum_k val(x[m,k]) val(sx[m,k/16]) val(w[n,k]) val(sw[n,k/16])) * sg_x * sg_w)
 * on block-scaled FP4 tensor cores (FP32 accumulation).  X [M, K] and W [N, K] as
 * qattn_quantize_fp4_block writes them: x_e2m1 / w_e2m1 packed E2M1 codes, rows of K / 2 bytes
 * (element 2i in the low nibble of byte i); x_bscale / w_bscale E4M3 block scales, [rows, K / 16]
 * row-major (block b covers K elements 16 b .. 16 b + 15, codes 0x00..0x7E); sg_x_dev /
 * sg_w_dev one-element device FP32 per-tensor scales; y_bf16 [M, N] row-major.  All device,
 * caller-owned, 16-byte aligned (the scales 4-byte); M >= 1, N >= 32 with N % 32 == 0,
 * K >= 256 with K % 256 == 0, else QATTN_ERR_INVALID_ARG.  Timeouts of the kernel's bounded
 * waits are reported by qattn_get_error. */
QATTN_API qattn_status qattn_gemm_fp4(const uint8_t* x_e2m1, const uint8_t* x_bscale,
                                      const float* sg_x_dev, const uint8_t* w_e2m1,
                                      const uint8_t* w_bscale, const float* sg_w_dev, void* y_bf16,
                                      int M, int N, int K, qattn_stream_t stream);

/* qattn_calibrate_quantize_fp8 without a caller workspace (the blog has no counterpart: this is
 * a calling convention, not part of the method).  For callers that cannot supply a scratch
 * buffer -- C code with no device allocator at the call site, or a runtime whose device memory
 * is planned ahead and must not allocate on the hot path.  The call allocates nothing: the
 * workspace is a static QATTN_FUSED_WORKSPACE_BYTES-byte device array inside the library (one
 * per device), cleared with a memset on `stream` before the kernel.  The workspace need does not
 * grow with n, so no size is rejected on its account; the argument rules and results are those
 * of qattn_calibrate_quantize_fp8.  The FIRST call on each device looks the array's address up
 * (cudaGetSymbolAddress, with that device current); make that first call before any stream
 * capture.  All calls on one device share the array: calls that overlap on the device (other
 * streams, other host threads without ordering) race and give wrong results. */
QATTN_API qattn_status qattn_calibrate_quantize_fp8_noalloc(const void* x_bf16, size_t n,
                                                            float* amax_dev, uint8_t* out_e4m3,
                                                            float* scale_dev,
                                                            qattn_stream_t stream);

/* Quantized attention forward, full (non-causal) attention over [B, H, L, D] (blog, "Workflow
 * and quantization", SDPA bullets 2-4 and Fig. 4):
 *   S' = (Q8 K8^T) * s_q * s_k * sm_scale * log2(e)   FP8 MMA, FP32 accumulation
 *   M  = ceil(running row max of S')                  power-of-two running max
 *   p  = 2^(S' - M),  l = sum p                       FP32
 *   P8 = e4m3(p * 448)                                per-tensor scale 1/448
 *   O  = (P8 V8) * s_v / 448 / l                      FP8 MMA, FP32 accumulation -> bf16
 * q8, k8, v8: device E4M3 codes [B, H, L, D] (row-major, 16-byte aligned).  out_bf16: device
 * [B, H, L, D] bf16.  D must be 64 or 128; B, H, L >= 1.  mode records whether the codes came
 * from the FP8 or the FP4 path (both feed BMM1 with E4M3 codes).  sm_scale > 0 (1/sqrt(D) in
 * the model). */
QATTN_API qattn_status qattn_forward(const uint8_t* q8, const uint8_t* k8, const uint8_t* v8,
                           void* out_bf16, int B, int H, int L, int D,
                           const qattn_scales* scales, float sm_scale, qattn_mode mode,
                           qattn_stream_t stream);

/* qattn_forward with a caller workspace that lets the kernel balance its work across SMs: the
 * attention kernel is persistent (one CTA per SM); after an equal share of whole Q-tile pairs
 * per CTA, the key steps of the remaining pairs are cut into equal contiguous ranges, one per
 * CTA.  A range that covers part of a pair writes its unnormalised FP32 partial O, running row
 * maximum and row sum to the workspace, and a combine kernel merges the parts.  The maxima are
 * integers (power-of-two running max), so merging rescales by exact powers of two and the result
 * equals the uncut one up to FP32 summation order.  workspace_dev: device, 16-byte aligned, at
 * least qattn_forward_workspace_bytes(B, H, L, D) bytes, no initial contents needed; NULL = no
 * pair is cut (exactly qattn_forward).  Calls sharing a workspace must not overlap on the
 * device. */
QATTN_API qattn_status qattn_forward_ws(const uint8_t* q8, const uint8_t* k8, const uint8_t* v8,
                                        void* out_bf16, int B, int H, int L, int D,
                                        const qattn_scales* scales, float sm_scale,
                                        qattn_mode mode, void* workspace_dev,
                                        size_t workspace_bytes, qattn_stream_t stream);

/* Workspace bytes qattn_forward_ws uses for this shape on the current device (0: no pair of
 * this shape is cut, or the arguments or device are not supported). */
QATTN_API size_t qattn_forward_workspace_bytes(int B, int H, int L, int D);

/* Same over a packed batch of variable-length sequences ([1, H, T, D] with sequence s at token
 * rows [cu_seqlens[s], cu_seqlens[s+1]) of every head; attention stays inside a sequence).
 * cu_seqlens_dev: device int32 [nseq + 1], non-decreasing from 0 to total_tokens; max_seqlen:
 * the largest cu_seqlens[s+1] - cu_seqlens[s] (a larger value only costs idle CTAs; a smaller
 * one leaves rows unwritten).  The host does not read cu_seqlens_dev. */
QATTN_API qattn_status qattn_forward_varlen(const uint8_t* q8, const uint8_t* k8, const uint8_t* v8,
                                  void* out_bf16, const int* cu_seqlens_dev, int nseq,
                                  int max_seqlen, int total_tokens, int H, int D,
                                  const qattn_scales* scales, float sm_scale, qattn_mode mode,
                                  qattn_stream_t stream);

/* Synchronizes `stream`, then returns and clears the current device's error word: QATTN_OK,
 * QATTN_ERR_NONFINITE, QATTN_ERR_TIMEOUT or (checked build) QATTN_ERR_BOUNDS (or QATTN_ERR_CUDA
 * if the synchronization failed). */
QATTN_API qattn_status qattn_get_error(qattn_stream_t stream);

/* Human-readable name of a status code (static storage). */
QATTN_API const char* qattn_status_str(qattn_status status);

/* The CUDA runtime error (a cudaError_t value) behind the last QATTN_ERR_CUDA that a call of
 * this library returned on the calling host thread, or 0 if none has.  Argument checks and
 * device error words do not change it.  Lets a caller report which CUDA call failed. */
QATTN_API int qattn_last_cuda_error(void);

/* How this library was built: bit 0 set for the checked build (libqattn_checked.so, compiled
 * with QATTN_CHECKED), in which every kernel tests the global-memory indices it computes (output
 * rows, workspace slots, tile and TMA coordinates, element and block indices) against the
 * extents of its buffers, records QATTN_ERR_BOUNDS in the error word on a miss and skips that
 * access instead of trapping.  No device needed. */
QATTN_API int qattn_build_info(void);

/* Test hook of the checked build, not part of the method: with enable != 0 the next
 * qattn_quantize_fp8 launches run their element loop one 8-element vector past n (as an index
 * bug would), so the bounds checks must catch the extra vector, record QATTN_ERR_BOUNDS and skip
 * it; the first n codes are still written.  The normal build has no such switch: there it
 * returns QATTN_ERR_UNSUPPORTED and changes nothing. */
QATTN_API qattn_status qattn_debug_inject_oob(int enable);

/* Test hooks, not part of the method.  qattn_debug_set_wait_timeout_ns sets the limit after
 * which a wait inside the attention kernel gives up (default 2 s; 0 restores the default).
 * qattn_debug_inject_missing_q(1) makes the next attention launches never load Q, so every
 * wait of the kernel runs into that limit and the kernel reports QATTN_ERR_TIMEOUT instead of
 * hanging. */
QATTN_API void qattn_debug_set_wait_timeout_ns(uint64_t ns);
QATTN_API void qattn_debug_inject_missing_q(int enable);

/* Kernel choice for D = 128, not part of the method: with enable != 0 the next D = 128 attention
 * launches run the pair-of-SMs kernel (two CTAs of a cluster per pair of Q tiles, cta_group::2
 * MMAs, three S buffers in TMEM) instead of the default one-SM kernel; enable = 0 restores the
 * default.  Same results up to FP32 summation order; the default is the faster one on B200.
 * qattn_forward_workspace_bytes covers both. */
QATTN_API void qattn_debug_use_pair_kernel(int enable);

/* Test hook, not part of the method: with enable != 0 the next attention launches copy,
 * for query row `row` (row index within the slab's rows: the token index for dense launches,
 * the packed token index for varlen) of slab `slab` (b * H + h; the head for varlen), the E4M3
 * codes of P of every key step s into codes_dev[s * 128 + key] (key within the step) and the
 * integer maximum they are relative to (base-2 units; P(s) = e4m3(2^(S' - max) * 448)): the
 * running row maximum after step s in the one-SM kernel, step s's own tile maximum in the pair
 * kernel, into maxima_dev[s].
 * codes_dev: device, 16-byte aligned, ceil(L / 128) * 128 bytes; maxima_dev: device int32,
 * ceil(L / 128) entries; both caller-owned and written only by launches made while enabled.
 * enable = 0 turns it off (the pointers are forgotten); with it off nothing of the launches
 * changes.  QATTN_ERR_INVALID_ARG for null or misaligned buffers or negative indices. */
QATTN_API qattn_status qattn_debug_capture_p_row(int enable, int slab, int row, uint8_t* codes_dev,
                                                 int* maxima_dev);

/* Host-only view of the persistent schedule qattn_forward_ws runs for a dense (B, H, L, D) on a
 * GPU with num_sms SMs (no device needed): plan[0..5] = pairs of Q tiles per head, key steps
 * per pair, CTAs, whole pairs per CTA, tail pairs, tail key steps per CTA (== key steps per pair
 * when no pair is cut); *workspace_bytes = qattn_forward_workspace_bytes on such a GPU.  CTA c
 * runs pairs c, c + CTAs, ... (the whole ones), then tail key steps [c * tail_w, (c + 1) * tail_w)
 * of the tail pairs laid end to end.  QATTN_ERR_INVALID_ARG for a shape the forward rejects. */
QATTN_API qattn_status qattn_debug_attention_plan(int B, int H, int L, int D, int num_sms,
                                                  int* plan, size_t* workspace_bytes);

#ifdef __cplusplus
}
#endif

#endif /* QATTN_H_ */
