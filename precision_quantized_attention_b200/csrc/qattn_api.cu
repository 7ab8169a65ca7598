// qattn_api.cu -- the C ABI (include/qattn.h): argument checks, device checks, launches.
#include <cuda_runtime.h>
#include <cstdint>
#include <mutex>

#include "launch.h"
#include "qattn.h"
#include "sm100_ptx.cuh"


// The device error word (one per device that loads the library).
static __device__ int g_qattn_error = 0;

namespace {

constexpr int kMaxDevices = 64;
constexpr uint64_t kDefaultTimeoutNs = 2000000000ull;

struct DeviceInfo {
  cudaError_t setup = cudaSuccess;   // error of the set-up below, if any
  bool supported = false;
  int num_sms = 0;
  int* err = nullptr;
};
DeviceInfo g_dev[kMaxDevices];
std::once_flag g_dev_once[kMaxDevices];
uint64_t g_timeout_ns = kDefaultTimeoutNs;
qattn::DebugHooks g_dbg;          // test hooks (qattn_debug_*)

thread_local int t_last_cuda_error = 0;   // qattn_last_cuda_error: per calling host thread

qattn_status from_cuda(cudaError_t e) {
  if (e == cudaSuccess) return QATTN_OK;
  t_last_cuda_error = static_cast<int>(e);
  return QATTN_ERR_CUDA;
}

// Per-device set-up on first use, once per device and thread-safe (std::call_once): capability
// check, SM count, device address of the error word.  Callers on other threads wait for it.
qattn_status device_info(DeviceInfo** out) {
  int dev = 0;
  const cudaError_t ge = cudaGetDevice(&dev);
  if (ge != cudaSuccess) return from_cuda(ge);
  if (dev < 0 || dev >= kMaxDevices) return QATTN_ERR_CUDA;
  DeviceInfo& d = g_dev[dev];
  std::call_once(g_dev_once[dev], [&d, dev] {
    int major = 0, minor = 0, sms = 0;
    cudaError_t e = cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev);
    if (e == cudaSuccess) e = cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev);
    if (e == cudaSuccess) e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    d.supported = e == cudaSuccess && major == 10 && minor == 0;
    d.num_sms = sms;
    if (e == cudaSuccess && d.supported) {
      void* p = nullptr;
      e = cudaGetSymbolAddress(&p, g_qattn_error);
      d.err = static_cast<int*>(p);
    }
    d.setup = e;
  });
  if (d.setup != cudaSuccess) return from_cuda(d.setup);
  if (!d.supported) return QATTN_ERR_UNSUPPORTED;
  *out = &d;
  return QATTN_OK;
}

bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }


qattn_status check_attention_common(const uint8_t* q8, const uint8_t* k8, const uint8_t* v8,
                                    const void* out, int H, int D, const qattn_scales* sc,
                                    float sm_scale, qattn_mode mode) {
  if (!q8 || !k8 || !v8 || !out || !sc || !sc->s_q || !sc->s_k || !sc->s_v)
    return QATTN_ERR_INVALID_ARG;
  if (!aligned(q8, 16) || !aligned(k8, 16) || !aligned(v8, 16) || !aligned(out, 16))
    return QATTN_ERR_INVALID_ARG;
  if (H < 1 || !(sm_scale > 0.0f) || !(sm_scale < 3.0e38f)) return QATTN_ERR_INVALID_ARG;
  if (D != 64 && D != 128) return QATTN_ERR_UNSUPPORTED;
  const int base = static_cast<int>(mode) & ~static_cast<int>(QATTN_FLAG_P_UNQUANTIZED);
  if (base != QATTN_MODE_FP8 && base != QATTN_MODE_FP4) return QATTN_ERR_INVALID_ARG;
  return QATTN_OK;
}

bool p_unquantized(qattn_mode mode) {
  return (static_cast<int>(mode) & static_cast<int>(QATTN_FLAG_P_UNQUANTIZED)) != 0;
}

}  // namespace

extern "C" {

qattn_status qattn_calibrate_amax(const void* x_bf16, size_t n, float* amax_dev,
                                  qattn_stream_t stream) {
  if (!x_bf16 || !amax_dev || n == 0 || !aligned(x_bf16, 16) || !aligned(amax_dev, 4))
    return QATTN_ERR_INVALID_ARG;
  DeviceInfo* d = nullptr;
  qattn_status st = device_info(&d);
  if (st != QATTN_OK) return st;
  return from_cuda(qattn::launch_amax(x_bf16, n, amax_dev, d->err, d->num_sms,
                                      reinterpret_cast<cudaStream_t>(stream)));
}

qattn_status qattn_quantize_fp8(const void* x_bf16, size_t n, const float* amax_dev,
                                uint8_t* out_e4m3, float* scale_dev, qattn_stream_t stream) {
  if (!x_bf16 || !amax_dev || !out_e4m3 || !scale_dev || n == 0) return QATTN_ERR_INVALID_ARG;
  if (!aligned(x_bf16, 16) || !aligned(out_e4m3, 8) || !aligned(amax_dev, 4) ||
      !aligned(scale_dev, 4))
    return QATTN_ERR_INVALID_ARG;
  DeviceInfo* d = nullptr;
  qattn_status st = device_info(&d);
  if (st != QATTN_OK) return st;
  return from_cuda(qattn::launch_quant_fp8(x_bf16, n, amax_dev, out_e4m3, scale_dev, d->err,
                                           d->num_sms, reinterpret_cast<cudaStream_t>(stream),
                                           g_dbg.inject_oob));
}

qattn_status qattn_quantize_fp4_block(const void* x_bf16, size_t n, const float* amax_dev,
                                      uint8_t* out_e2m1, uint8_t* blk_scale_e4m3,
                                      float* gscale_dev, uint8_t* out_e4m3_requant,
                                      float* scale8_dev, qattn_stream_t stream) {
  if (!x_bf16 || !amax_dev || !out_e2m1 || !blk_scale_e4m3 || !gscale_dev || n == 0 ||
      n % 16 != 0)
    return QATTN_ERR_INVALID_ARG;
  if ((out_e4m3_requant == nullptr) != (scale8_dev == nullptr)) return QATTN_ERR_INVALID_ARG;
  if (!aligned(x_bf16, 16) || !aligned(out_e2m1, 8) || !aligned(amax_dev, 4) ||
      !aligned(gscale_dev, 4) || (out_e4m3_requant && !aligned(out_e4m3_requant, 16)) ||
      (scale8_dev && !aligned(scale8_dev, 4)))
    return QATTN_ERR_INVALID_ARG;
  DeviceInfo* d = nullptr;
  qattn_status st = device_info(&d);
  if (st != QATTN_OK) return st;
  return from_cuda(qattn::launch_quant_fp4_block(x_bf16, n, amax_dev, out_e2m1, blk_scale_e4m3,
                                                 gscale_dev, out_e4m3_requant, scale8_dev, d->err,
                                                 d->num_sms,
                                                 reinterpret_cast<cudaStream_t>(stream)));
}

qattn_status qattn_calibrate_quantize_fp8(const void* x_bf16, size_t n, float* amax_dev,
                                          uint8_t* out_e4m3, float* scale_dev,
                                          void* workspace_dev, size_t workspace_bytes,
                                          qattn_stream_t stream) {
  if (!x_bf16 || !amax_dev || !out_e4m3 || !scale_dev || !workspace_dev || n == 0)
    return QATTN_ERR_INVALID_ARG;
  if (workspace_bytes < QATTN_FUSED_WORKSPACE_BYTES || !aligned(workspace_dev, 16))
    return QATTN_ERR_INVALID_ARG;
  if (!aligned(x_bf16, 16) || !aligned(out_e4m3, 8) || !aligned(amax_dev, 4) ||
      !aligned(scale_dev, 4))
    return QATTN_ERR_INVALID_ARG;
  DeviceInfo* d = nullptr;
  qattn_status st = device_info(&d);
  if (st != QATTN_OK) return st;
  return from_cuda(qattn::launch_calib_quant_fp8(x_bf16, n, amax_dev, out_e4m3, scale_dev,
                                                 workspace_dev, g_timeout_ns, d->err, d->num_sms,
                                                 reinterpret_cast<cudaStream_t>(stream)));
}

qattn_status qattn_calibrate_quantize_fp4_block(const void* x_bf16, size_t n, float* amax_dev,
                                                uint8_t* out_e2m1, uint8_t* blk_scale_e4m3,
                                                float* gscale_dev, uint8_t* out_e4m3_requant,
                                                float* scale8_dev, void* workspace_dev,
                                                size_t workspace_bytes, qattn_stream_t stream) {
  if (!x_bf16 || !amax_dev || !out_e2m1 || !blk_scale_e4m3 || !gscale_dev || !workspace_dev ||
      n == 0 || n % 16 != 0)
    return QATTN_ERR_INVALID_ARG;
  if ((out_e4m3_requant == nullptr) != (scale8_dev == nullptr)) return QATTN_ERR_INVALID_ARG;
  if (workspace_bytes < QATTN_FUSED_WORKSPACE_BYTES || !aligned(workspace_dev, 16))
    return QATTN_ERR_INVALID_ARG;
  if (!aligned(x_bf16, 16) || !aligned(out_e2m1, 8) || !aligned(amax_dev, 4) ||
      !aligned(gscale_dev, 4) || (out_e4m3_requant && !aligned(out_e4m3_requant, 16)) ||
      (scale8_dev && !aligned(scale8_dev, 4)))
    return QATTN_ERR_INVALID_ARG;
  DeviceInfo* d = nullptr;
  qattn_status st = device_info(&d);
  if (st != QATTN_OK) return st;
  return from_cuda(qattn::launch_calib_quant_fp4_block(
      x_bf16, n, amax_dev, out_e2m1, blk_scale_e4m3, gscale_dev, out_e4m3_requant, scale8_dev,
      workspace_dev, g_timeout_ns, d->err, d->num_sms, reinterpret_cast<cudaStream_t>(stream)));
}

qattn_status qattn_calibrate_quantize_qkv(const qattn_quant_io* io, size_t n, qattn_mode mode,
                                          void* workspace_dev, size_t workspace_bytes,
                                          qattn_stream_t stream) {
  if (!io || n == 0 || !workspace_dev) return QATTN_ERR_INVALID_ARG;
  if (mode != QATTN_MODE_FP8 && mode != QATTN_MODE_FP4) return QATTN_ERR_INVALID_ARG;
  if (mode == QATTN_MODE_FP4 && n % 16 != 0) return QATTN_ERR_INVALID_ARG;
  if (workspace_bytes < QATTN_FUSED_WORKSPACE_BYTES || !aligned(workspace_dev, 16))
    return QATTN_ERR_INVALID_ARG;
  const void* x[3];
  uint8_t *c8[3], *e2m1[3], *bs[3];
  float *am[3], *sc[3], *gs[3];
  for (int i = 0; i < 3; ++i) {
    const qattn_quant_io& t = io[i];
    if (!t.x_bf16 || !t.out_e4m3 || !t.amax_dev || !t.scale_dev) return QATTN_ERR_INVALID_ARG;
    if (!aligned(t.x_bf16, 16) || !aligned(t.amax_dev, 4) || !aligned(t.scale_dev, 4) ||
        !aligned(t.out_e4m3, mode == QATTN_MODE_FP4 ? 16 : 8))
      return QATTN_ERR_INVALID_ARG;
    if (mode == QATTN_MODE_FP4 && (!t.out_e2m1 || !t.blk_scale_e4m3 || !t.gscale_dev ||
                                   !aligned(t.out_e2m1, 8) || !aligned(t.gscale_dev, 4)))
      return QATTN_ERR_INVALID_ARG;
    x[i] = t.x_bf16;
    c8[i] = t.out_e4m3;
    am[i] = t.amax_dev;
    sc[i] = t.scale_dev;
    e2m1[i] = mode == QATTN_MODE_FP4 ? t.out_e2m1 : nullptr;
    bs[i] = mode == QATTN_MODE_FP4 ? t.blk_scale_e4m3 : nullptr;
    gs[i] = mode == QATTN_MODE_FP4 ? t.gscale_dev : nullptr;
  }
  DeviceInfo* d = nullptr;
  qattn_status st = device_info(&d);
  if (st != QATTN_OK) return st;
  return from_cuda(qattn::launch_calib_quant_qkv(x, c8, am, sc, e2m1, bs, gs, n,
                                                 mode == QATTN_MODE_FP4 ? 1 : 0, workspace_dev,
                                                 g_timeout_ns, d->err, d->num_sms,
                                                 reinterpret_cast<cudaStream_t>(stream)));
}

qattn_status qattn_quantize_qkv(const qattn_quant_io* io, size_t n, qattn_mode mode,
                                qattn_stream_t stream) {
  if (!io || n == 0) return QATTN_ERR_INVALID_ARG;
  if (mode != QATTN_MODE_FP8 && mode != QATTN_MODE_FP4) return QATTN_ERR_INVALID_ARG;
  if (mode == QATTN_MODE_FP4 && n % 16 != 0) return QATTN_ERR_INVALID_ARG;
  const void* x[3];
  uint8_t *c8[3], *e2m1[3], *bs[3];
  float *am[3], *sc[3], *gs[3];
  for (int i = 0; i < 3; ++i) {
    const qattn_quant_io& t = io[i];
    if (!t.x_bf16 || !t.out_e4m3 || !t.amax_dev || !t.scale_dev) return QATTN_ERR_INVALID_ARG;
    if (!aligned(t.x_bf16, 16) || !aligned(t.amax_dev, 4) || !aligned(t.scale_dev, 4) ||
        !aligned(t.out_e4m3, mode == QATTN_MODE_FP4 ? 16 : 8))
      return QATTN_ERR_INVALID_ARG;
    if (mode == QATTN_MODE_FP4 && (!t.out_e2m1 || !t.blk_scale_e4m3 || !t.gscale_dev ||
                                   !aligned(t.out_e2m1, 8) || !aligned(t.gscale_dev, 4)))
      return QATTN_ERR_INVALID_ARG;
    x[i] = t.x_bf16;
    c8[i] = t.out_e4m3;
    am[i] = t.amax_dev;
    sc[i] = t.scale_dev;
    e2m1[i] = mode == QATTN_MODE_FP4 ? t.out_e2m1 : nullptr;
    bs[i] = mode == QATTN_MODE_FP4 ? t.blk_scale_e4m3 : nullptr;
    gs[i] = mode == QATTN_MODE_FP4 ? t.gscale_dev : nullptr;
  }
  DeviceInfo* d = nullptr;
  qattn_status st = device_info(&d);
  if (st != QATTN_OK) return st;
  return from_cuda(qattn::launch_quant_qkv(x, c8, am, sc, e2m1, bs, gs, n,
                                           mode == QATTN_MODE_FP4 ? 1 : 0, d->err, d->num_sms,
                                           reinterpret_cast<cudaStream_t>(stream)));
}

qattn_status qattn_gemm_fp8(const uint8_t* a8, const uint8_t* b8, void* y_bf16, int M, int N,
                            int K, const float* s_a_dev, const float* s_b_dev,
                            qattn_stream_t stream) {
  if (!a8 || !b8 || !y_bf16 || !s_a_dev || !s_b_dev) return QATTN_ERR_INVALID_ARG;
  if (M < 1 || N < 32 || K < 128 || N % 32 != 0 || K % 128 != 0) return QATTN_ERR_INVALID_ARG;
  if (!aligned(a8, 16) || !aligned(b8, 16) || !aligned(y_bf16, 16) || !aligned(s_a_dev, 4) ||
      !aligned(s_b_dev, 4))
    return QATTN_ERR_INVALID_ARG;
  DeviceInfo* d = nullptr;
  qattn_status st = device_info(&d);
  if (st != QATTN_OK) return st;
  return from_cuda(qattn::launch_gemm_fp8(a8, b8, y_bf16, M, N, K, s_a_dev, s_b_dev, d->err,
                                          g_timeout_ns, d->num_sms,
                                          reinterpret_cast<cudaStream_t>(stream)));
}

qattn_status qattn_gemm_fp8_e4m3(const uint8_t* a8, const uint8_t* b8, void* y_bf16,
                                 uint8_t* codes_out, int M, int N, int K, const float* s_a_dev,
                                 const float* s_b_dev, const float* amax_dev, float* scale_out_dev,
                                 qattn_stream_t stream) {
  if (!a8 || !b8 || !codes_out || !s_a_dev || !s_b_dev || !amax_dev || !scale_out_dev)
    return QATTN_ERR_INVALID_ARG;
  if (M < 1 || N < 32 || K < 128 || N % 32 != 0 || K % 128 != 0) return QATTN_ERR_INVALID_ARG;
  if (!aligned(a8, 16) || !aligned(b8, 16) || (y_bf16 && !aligned(y_bf16, 16)) ||
      !aligned(codes_out, 16) || !aligned(s_a_dev, 4) || !aligned(s_b_dev, 4) ||
      !aligned(amax_dev, 4) || !aligned(scale_out_dev, 4))
    return QATTN_ERR_INVALID_ARG;
  DeviceInfo* d = nullptr;
  qattn_status st = device_info(&d);
  if (st != QATTN_OK) return st;
  return from_cuda(qattn::launch_gemm_fp8(a8, b8, y_bf16, M, N, K, s_a_dev, s_b_dev, d->err,
                                          g_timeout_ns, d->num_sms,
                                          reinterpret_cast<cudaStream_t>(stream), codes_out,
                                          amax_dev, scale_out_dev));
}

qattn_status qattn_gemm_fp4(const uint8_t* x_e2m1, const uint8_t* x_bscale, const float* sg_x_dev,
                           const uint8_t* w_e2m1, const uint8_t* w_bscale, const float* sg_w_dev,
                           void* y_bf16, int M, int N, int K, qattn_stream_t stream) {
  if (!x_e2m1 || !x_bscale || !sg_x_dev || !w_e2m1 || !w_bscale || !sg_w_dev || !y_bf16)
    return QATTN_ERR_INVALID_ARG;
  if (M < 1 || N < 32 || K < 256 || N % 32 != 0 || K % 256 != 0) return QATTN_ERR_INVALID_ARG;
  if (!aligned(x_e2m1, 16) || !aligned(w_e2m1, 16) || !aligned(x_bscale, 16) ||
      !aligned(w_bscale, 16) || !aligned(y_bf16, 16) || !aligned(sg_x_dev, 4) || !aligned(sg_w_dev, 4))
    return QATTN_ERR_INVALID_ARG;
  DeviceInfo* d = nullptr;
  qattn_status st = device_info(&d);
  if (st != QATTN_OK) return st;
  return from_cuda(qattn::launch_gemm_fp4(x_e2m1, x_bscale, sg_x_dev, w_e2m1, w_bscale, sg_w_dev,
                                          y_bf16, M, N, K, d->err, g_timeout_ns, d->num_sms,
                                          reinterpret_cast<cudaStream_t>(stream)));
}

qattn_status qattn_forward_ws(const uint8_t* q8, const uint8_t* k8, const uint8_t* v8,
                              void* out_bf16, int B, int H, int L, int D,
                              const qattn_scales* scales, float sm_scale, qattn_mode mode,
                              void* workspace_dev, size_t workspace_bytes, qattn_stream_t stream) {
  qattn_status st = check_attention_common(q8, k8, v8, out_bf16, H, D, scales, sm_scale, mode);
  if (st != QATTN_OK) return st;
  if (B < 1 || L < 1) return QATTN_ERR_INVALID_ARG;
  if (B > 65535 || H > 65535) return QATTN_ERR_UNSUPPORTED;
  if (static_cast<int64_t>(B) * H * L * D >= (int64_t(1) << 40)) return QATTN_ERR_UNSUPPORTED;
  if (workspace_dev != nullptr && !aligned(workspace_dev, 16)) return QATTN_ERR_INVALID_ARG;
  DeviceInfo* d = nullptr;
  st = device_info(&d);
  if (st != QATTN_OK) return st;
  if (workspace_dev != nullptr &&
      workspace_bytes < qattn::attention_plan(B, H, L, D, d->num_sms, g_dbg.attn_pair != 0).bytes)
    return QATTN_ERR_INVALID_ARG;
  if (p_unquantized(mode)) {
    if (static_cast<int64_t>(B) * H > 65535) return QATTN_ERR_UNSUPPORTED;
    return from_cuda(qattn::launch_attention_p_unquantized(
        q8, k8, v8, out_bf16, B, H, L, D, nullptr, 0, L, L, scales->s_q, scales->s_k, scales->s_v,
        sm_scale, reinterpret_cast<cudaStream_t>(stream)));
  }
  return from_cuda(qattn::launch_attention(q8, k8, v8, out_bf16, B, H, L, D, nullptr, 0, L, L,
                                           scales->s_q, scales->s_k, scales->s_v, sm_scale,
                                           d->err, g_timeout_ns, g_dbg,
                                           workspace_dev, workspace_bytes, d->num_sms,
                                           reinterpret_cast<cudaStream_t>(stream)));
}

qattn_status qattn_forward(const uint8_t* q8, const uint8_t* k8, const uint8_t* v8,
                           void* out_bf16, int B, int H, int L, int D,
                           const qattn_scales* scales, float sm_scale, qattn_mode mode,
                           qattn_stream_t stream) {
  return qattn_forward_ws(q8, k8, v8, out_bf16, B, H, L, D, scales, sm_scale, mode, nullptr, 0,
                          stream);
}

size_t qattn_forward_workspace_bytes(int B, int H, int L, int D) {
  if (B < 1 || H < 1 || L < 1 || (D != 64 && D != 128)) return 0;
  DeviceInfo* d = nullptr;
  if (device_info(&d) != QATTN_OK) return 0;
  // enough for either D = 128 kernel, so a workspace stays valid if the variant is switched
  const size_t one_sm = qattn::attention_plan(B, H, L, D, d->num_sms, false).bytes;
  const size_t pair = D == 128 ? qattn::attention_plan(B, H, L, D, d->num_sms, true).bytes : 0;
  return one_sm > pair ? one_sm : pair;
}

qattn_status qattn_forward_varlen(const uint8_t* q8, const uint8_t* k8, const uint8_t* v8,
                                  void* out_bf16, const int* cu_seqlens_dev, int nseq,
                                  int max_seqlen, int total_tokens, int H, int D,
                                  const qattn_scales* scales, float sm_scale, qattn_mode mode,
                                  qattn_stream_t stream) {
  qattn_status st = check_attention_common(q8, k8, v8, out_bf16, H, D, scales, sm_scale, mode);
  if (st != QATTN_OK) return st;
  if (!cu_seqlens_dev || !aligned(cu_seqlens_dev, 4) || nseq < 1 || max_seqlen < 1 ||
      total_tokens < 1 || max_seqlen > total_tokens)
    return QATTN_ERR_INVALID_ARG;
  if (nseq > 65535 || H > 65535) return QATTN_ERR_UNSUPPORTED;
  DeviceInfo* d = nullptr;
  st = device_info(&d);
  if (st != QATTN_OK) return st;
  if (p_unquantized(mode))
    return from_cuda(qattn::launch_attention_p_unquantized(
        q8, k8, v8, out_bf16, 1, H, 0, D, cu_seqlens_dev, nseq, max_seqlen, total_tokens,
        scales->s_q, scales->s_k, scales->s_v, sm_scale, reinterpret_cast<cudaStream_t>(stream)));
  return from_cuda(qattn::launch_attention(q8, k8, v8, out_bf16, 1, H, 0, D, cu_seqlens_dev,
                                           nseq, max_seqlen, total_tokens, scales->s_q,
                                           scales->s_k, scales->s_v, sm_scale, d->err,
                                           g_timeout_ns, g_dbg, nullptr, 0,
                                           d->num_sms, reinterpret_cast<cudaStream_t>(stream)));
}

qattn_status qattn_get_error(qattn_stream_t stream) {
  DeviceInfo* d = nullptr;
  qattn_status st = device_info(&d);
  if (st != QATTN_OK) return st;
  if (cudaStreamSynchronize(reinterpret_cast<cudaStream_t>(stream)) != cudaSuccess)
    return QATTN_ERR_CUDA;
  int word = 0;
  if (cudaMemcpyFromSymbol(&word, g_qattn_error, sizeof(int)) != cudaSuccess) return QATTN_ERR_CUDA;
  if (word != 0) {
    const int zero = 0;
    if (cudaMemcpyToSymbol(g_qattn_error, &zero, sizeof(int)) != cudaSuccess)
      return QATTN_ERR_CUDA;
  }
  switch (word) {
    case 0: return QATTN_OK;
    case qattn::DEV_ERR_NONFINITE: return QATTN_ERR_NONFINITE;
    case qattn::DEV_ERR_TIMEOUT: return QATTN_ERR_TIMEOUT;
    case qattn::DEV_ERR_BOUNDS: return QATTN_ERR_BOUNDS;
    default: return QATTN_ERR_CUDA;
  }
}

int qattn_last_cuda_error(void) { return t_last_cuda_error; }

const char* qattn_status_str(qattn_status status) {
  switch (status) {
    case QATTN_OK: return "QATTN_OK";
    case QATTN_ERR_INVALID_ARG: return "QATTN_ERR_INVALID_ARG";
    case QATTN_ERR_UNSUPPORTED: return "QATTN_ERR_UNSUPPORTED";
    case QATTN_ERR_CUDA: return "QATTN_ERR_CUDA";
    case QATTN_ERR_NONFINITE: return "QATTN_ERR_NONFINITE";
    case QATTN_ERR_TIMEOUT: return "QATTN_ERR_TIMEOUT";
    case QATTN_ERR_BOUNDS: return "QATTN_ERR_BOUNDS";
  }
  return "QATTN_ERR_UNKNOWN";
}

void qattn_debug_set_wait_timeout_ns(uint64_t ns) {
  g_timeout_ns = ns ? ns : kDefaultTimeoutNs;
}

void qattn_debug_inject_missing_q(int enable) { g_dbg.inject_missing_q = enable ? 1 : 0; }

void qattn_debug_use_pair_kernel(int enable) { g_dbg.attn_pair = enable ? 1 : 0; }

int qattn_build_info(void) {
#ifdef QATTN_CHECKED
  return 1;
#else
  return 0;
#endif
}

qattn_status qattn_debug_inject_oob(int enable) {
#ifdef QATTN_CHECKED
  g_dbg.inject_oob = enable ? 1 : 0;
  return QATTN_OK;
#else
  (void)enable;
  return QATTN_ERR_UNSUPPORTED;
#endif
}

qattn_status qattn_debug_capture_p_row(int enable, int slab, int row, uint8_t* codes_dev,
                                       int* maxima_dev) {
  if (!enable) {
    g_dbg.p_codes = nullptr;
    g_dbg.p_maxima = nullptr;
    g_dbg.p_slab = g_dbg.p_row = -1;
    return QATTN_OK;
  }
  if (!codes_dev || !maxima_dev || !aligned(codes_dev, 16) || !aligned(maxima_dev, 4) || slab < 0 ||
      row < 0)
    return QATTN_ERR_INVALID_ARG;
  g_dbg.p_codes = codes_dev;
  g_dbg.p_maxima = maxima_dev;
  g_dbg.p_slab = slab;
  g_dbg.p_row = row;
  return QATTN_OK;
}

qattn_status qattn_debug_attention_plan(int B, int H, int L, int D, int num_sms, int* plan,
                                        size_t* workspace_bytes) {
  if (B < 1 || H < 1 || L < 1 || (D != 64 && D != 128) || num_sms < 1 || !plan ||
      !workspace_bytes)
    return QATTN_ERR_INVALID_ARG;
  const qattn::AttnSplitPlan p = qattn::plan_attention_split(B, H, L, D, num_sms);
  plan[0] = p.pairs_per_head;
  plan[1] = p.nkv;
  plan[2] = p.ctas;
  plan[3] = p.whole;
  plan[4] = p.tail_pairs;
  plan[5] = p.tail_w;
  *workspace_bytes = p.bytes;
  return QATTN_OK;
}

}  // extern "C"
