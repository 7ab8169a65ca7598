"""ctypes binding of libqattn (include/qattn.h): argument marshalling only.

Every entry point has the C name without the ``qattn_`` prefix, takes torch CUDA tensors for
the device buffers, enqueues on torch's current CUDA stream and raises ``QattnError`` on a
non-OK status.  There is no fallback: if the shared library is missing, loading fails loudly.
"""
from __future__ import annotations

import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
# QATTN_DEBUG=1 selects the checked build (device bounds checks that record QATTN_ERR_BOUNDS)
CHECKED = os.environ.get("QATTN_DEBUG") == "1"
LIB_PATH = os.path.join(_HERE, "libqattn_checked.so" if CHECKED else "libqattn.so")

OK, ERR_INVALID_ARG, ERR_UNSUPPORTED, ERR_CUDA, ERR_NONFINITE, ERR_TIMEOUT, ERR_BOUNDS = range(7)
MODE_FP8, MODE_FP4 = 0, 1
FLAG_P_UNQUANTIZED = 0x100   # OR into the mode of forward(): P stays FP32 (debug path)

# every symbol the header declares
EXPORTS = (
    "qattn_calibrate_amax", "qattn_quantize_fp8", "qattn_quantize_fp4_block", "qattn_forward",
    "qattn_forward_varlen", "qattn_get_error", "qattn_calibrate_quantize_fp8",
    "qattn_calibrate_quantize_fp4_block", "qattn_calibrate_quantize_fp8_noalloc",
    "qattn_calibrate_quantize_qkv", "qattn_quantize_qkv", "qattn_forward_ws", "qattn_gemm_fp8",
    "qattn_gemm_fp8_e4m3", "qattn_gemm_fp4",
    "qattn_status_str", "qattn_last_cuda_error",
    "qattn_forward_workspace_bytes",
    "qattn_debug_set_wait_timeout_ns", "qattn_debug_inject_missing_q", "qattn_debug_capture_p_row",
    "qattn_debug_attention_plan", "qattn_build_info", "qattn_debug_inject_oob",
    "qattn_debug_use_pair_kernel",
)
_RETURNS_STATUS = EXPORTS[:15]
FUSED_WORKSPACE_BYTES = 256     # QATTN_FUSED_WORKSPACE_BYTES


class QattnError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        msg = f"{what}: {status_str(status)} ({status})"
        if status == ERR_CUDA:
            msg += f", cudaError_t {load().qattn_last_cuda_error()}"
        super().__init__(msg)


class QuantIO(ctypes.Structure):
    """qattn_quant_io: one tensor's device buffers for calibrate_quantize_qkv."""
    _fields_ = [("x_bf16", ctypes.c_void_p), ("out_e4m3", ctypes.c_void_p),
                ("amax_dev", ctypes.c_void_p), ("scale_dev", ctypes.c_void_p),
                ("out_e2m1", ctypes.c_void_p), ("blk_scale_e4m3", ctypes.c_void_p),
                ("gscale_dev", ctypes.c_void_p)]


class _Scales(ctypes.Structure):
    _fields_ = [("s_q", ctypes.c_void_p), ("s_k", ctypes.c_void_p), ("s_v", ctypes.c_void_p)]


_lib = None


def load() -> ctypes.CDLL:
    """Load libqattn.so (built in-tree by ``python -m precision_quantized_attention_b200.build``)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"{LIB_PATH} is missing: build it with "
                          "`python -m precision_quantized_attention_b200.build"
                          + (" --checked`" if CHECKED else "`"))
    lib = ctypes.CDLL(LIB_PATH)
    P, S, I, F = ctypes.c_void_p, ctypes.c_size_t, ctypes.c_int, ctypes.c_float
    lib.qattn_calibrate_amax.argtypes = [P, S, P, P]
    lib.qattn_quantize_fp8.argtypes = [P, S, P, P, P, P]
    lib.qattn_quantize_fp4_block.argtypes = [P, S, P, P, P, P, P, P, P]
    lib.qattn_calibrate_quantize_fp8.argtypes = [P, S, P, P, P, P, S, P]
    lib.qattn_calibrate_quantize_fp4_block.argtypes = [P, S, P, P, P, P, P, P, P, S, P]
    lib.qattn_calibrate_quantize_fp8_noalloc.argtypes = [P, S, P, P, P, P]
    lib.qattn_calibrate_quantize_qkv.argtypes = [ctypes.POINTER(QuantIO), S, I, P, S, P]
    lib.qattn_quantize_qkv.argtypes = [ctypes.POINTER(QuantIO), S, I, P]
    lib.qattn_gemm_fp8.argtypes = [P, P, P, I, I, I, P, P, P]
    lib.qattn_gemm_fp8_e4m3.argtypes = [P, P, P, P, I, I, I, P, P, P, P, P]
    lib.qattn_gemm_fp4.argtypes = [P, P, P, P, P, P, P, I, I, I, P]
    lib.qattn_forward.argtypes = [P, P, P, P, I, I, I, I, ctypes.POINTER(_Scales), F, I, P]
    lib.qattn_forward_varlen.argtypes = [P, P, P, P, P, I, I, I, I, I, ctypes.POINTER(_Scales),
                                         F, I, P]
    lib.qattn_forward_ws.argtypes = [P, P, P, P, I, I, I, I, ctypes.POINTER(_Scales), F, I, P, S, P]
    lib.qattn_forward_workspace_bytes.argtypes = [I, I, I, I]
    lib.qattn_forward_workspace_bytes.restype = S
    lib.qattn_get_error.argtypes = [P]
    lib.qattn_status_str.argtypes = [I]
    lib.qattn_status_str.restype = ctypes.c_char_p
    lib.qattn_last_cuda_error.argtypes = []
    lib.qattn_last_cuda_error.restype = I
    lib.qattn_debug_set_wait_timeout_ns.argtypes = [ctypes.c_uint64]
    lib.qattn_debug_set_wait_timeout_ns.restype = None
    lib.qattn_debug_inject_missing_q.argtypes = [I]
    lib.qattn_debug_inject_missing_q.restype = None
    lib.qattn_debug_use_pair_kernel.argtypes = [I]
    lib.qattn_debug_use_pair_kernel.restype = None
    lib.qattn_build_info.argtypes = []
    lib.qattn_build_info.restype = I
    lib.qattn_debug_inject_oob.argtypes = [I]
    lib.qattn_debug_inject_oob.restype = I
    lib.qattn_debug_capture_p_row.argtypes = [I, I, I, P, P]
    lib.qattn_debug_capture_p_row.restype = I
    lib.qattn_debug_attention_plan.argtypes = [I, I, I, I, I, ctypes.POINTER(I),
                                              ctypes.POINTER(S)]
    lib.qattn_debug_attention_plan.restype = I
    for name in _RETURNS_STATUS:
        getattr(lib, name).restype = I
    _lib = lib
    return lib


def status_str(status: int) -> str:
    return load().qattn_status_str(int(status)).decode()


def _check(status: int, what: str):
    if status != OK:
        raise QattnError(status, what)


def _stream(stream=None):
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def _dev(t: torch.Tensor | None, dtype=None, what="tensor"):
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError(f"{what} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{what} must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise ValueError(f"{what} must be {dtype}, got {t.dtype}")
    return ctypes.c_void_p(t.data_ptr())


def calibrate_amax(x: torch.Tensor, amax: torch.Tensor, stream=None):
    _check(load().qattn_calibrate_amax(_dev(x, torch.bfloat16, "x"), x.numel(),
                                       _dev(amax, torch.float32, "amax"), _stream(stream)),
           "qattn_calibrate_amax")


def quantize_fp8(x: torch.Tensor, amax: torch.Tensor, out: torch.Tensor, scale: torch.Tensor,
                 stream=None):
    if out.numel() != x.numel():
        raise ValueError("out must have x.numel() bytes")
    _check(load().qattn_quantize_fp8(_dev(x, torch.bfloat16, "x"), x.numel(),
                                     _dev(amax, torch.float32, "amax"),
                                     _dev(out, torch.uint8, "out"),
                                     _dev(scale, torch.float32, "scale"), _stream(stream)),
           "qattn_quantize_fp8")


def quantize_fp4_block(x: torch.Tensor, amax: torch.Tensor, out_e2m1: torch.Tensor,
                       blk_scale: torch.Tensor, gscale: torch.Tensor,
                       out_e4m3_requant: torch.Tensor | None = None,
                       scale8: torch.Tensor | None = None, stream=None):
    n = x.numel()
    if out_e2m1.numel() != n // 2 or blk_scale.numel() != n // 16:
        raise ValueError("out_e2m1 needs n/2 bytes and blk_scale n/16 bytes")
    if out_e4m3_requant is not None and out_e4m3_requant.numel() != n:
        raise ValueError("out_e4m3_requant needs n bytes")
    _check(load().qattn_quantize_fp4_block(
        _dev(x, torch.bfloat16, "x"), n, _dev(amax, torch.float32, "amax"),
        _dev(out_e2m1, torch.uint8, "out_e2m1"), _dev(blk_scale, torch.uint8, "blk_scale"),
        _dev(gscale, torch.float32, "gscale"),
        _dev(out_e4m3_requant, torch.uint8, "out_e4m3_requant"),
        _dev(scale8, torch.float32, "scale8"), _stream(stream)), "qattn_quantize_fp4_block")


def new_workspace(device="cuda") -> torch.Tensor:
    """A zero-filled workspace for the fused calibrate+quantize calls."""
    return torch.zeros(FUSED_WORKSPACE_BYTES, dtype=torch.uint8, device=device)


def calibrate_quantize_fp8(x: torch.Tensor, amax: torch.Tensor, out: torch.Tensor,
                           scale: torch.Tensor, workspace: torch.Tensor, stream=None):
    if out.numel() != x.numel():
        raise ValueError("out must have x.numel() bytes")
    _check(load().qattn_calibrate_quantize_fp8(
        _dev(x, torch.bfloat16, "x"), x.numel(), _dev(amax, torch.float32, "amax"),
        _dev(out, torch.uint8, "out"), _dev(scale, torch.float32, "scale"),
        _dev(workspace, torch.uint8, "workspace"), workspace.numel(), _stream(stream)),
        "qattn_calibrate_quantize_fp8")


def calibrate_quantize_fp8_noalloc(x: torch.Tensor, amax: torch.Tensor, out: torch.Tensor,
                                   scale: torch.Tensor, stream=None):
    """calibrate_quantize_fp8 with the library's static workspace (no caller buffer)."""
    if out.numel() != x.numel():
        raise ValueError("out must have x.numel() bytes")
    _check(load().qattn_calibrate_quantize_fp8_noalloc(
        _dev(x, torch.bfloat16, "x"), x.numel(), _dev(amax, torch.float32, "amax"),
        _dev(out, torch.uint8, "out"), _dev(scale, torch.float32, "scale"), _stream(stream)),
        "qattn_calibrate_quantize_fp8_noalloc")


def calibrate_quantize_fp4_block(x: torch.Tensor, amax: torch.Tensor, out_e2m1: torch.Tensor,
                                 blk_scale: torch.Tensor, gscale: torch.Tensor,
                                 out_e4m3_requant: torch.Tensor | None,
                                 scale8: torch.Tensor | None, workspace: torch.Tensor,
                                 stream=None):
    n = x.numel()
    if out_e2m1.numel() != n // 2 or blk_scale.numel() != n // 16:
        raise ValueError("out_e2m1 needs n/2 bytes and blk_scale n/16 bytes")
    if out_e4m3_requant is not None and out_e4m3_requant.numel() != n:
        raise ValueError("out_e4m3_requant needs n bytes")
    _check(load().qattn_calibrate_quantize_fp4_block(
        _dev(x, torch.bfloat16, "x"), n, _dev(amax, torch.float32, "amax"),
        _dev(out_e2m1, torch.uint8, "out_e2m1"), _dev(blk_scale, torch.uint8, "blk_scale"),
        _dev(gscale, torch.float32, "gscale"),
        _dev(out_e4m3_requant, torch.uint8, "out_e4m3_requant"),
        _dev(scale8, torch.float32, "scale8"), _dev(workspace, torch.uint8, "workspace"),
        workspace.numel(), _stream(stream)), "qattn_calibrate_quantize_fp4_block")


def _qkv_io(xs, amax, codes8, scale8, mode, e2m1, bscale, gscale):
    n = xs[0].numel()
    if any(x.numel() != n for x in xs):
        raise ValueError("Q, K and V must have the same number of elements")
    for t, nm in ((amax, "amax"), (scale8, "scale8")):
        if t.numel() != 3 or t.dtype != torch.float32 or not t.is_contiguous():
            raise ValueError(f"{nm} must be a contiguous float32 tensor of 3 elements")
    if mode == MODE_FP4 and (e2m1 is None or bscale is None or gscale is None or gscale.numel() != 3):
        raise ValueError("FP4 mode needs e2m1, bscale and a 3-element gscale")
    io = (QuantIO * 3)()
    for i in range(3):
        if codes8[i].numel() != n:
            raise ValueError("codes8 tensors need n bytes")
        io[i].x_bf16 = _dev(xs[i], torch.bfloat16, "x").value
        io[i].out_e4m3 = _dev(codes8[i], torch.uint8, "codes8").value
        io[i].amax_dev = amax.data_ptr() + 4 * i
        io[i].scale_dev = scale8.data_ptr() + 4 * i
        if mode == MODE_FP4:
            if e2m1[i].numel() != n // 2 or bscale[i].numel() != n // 16:
                raise ValueError("e2m1 needs n/2 bytes and bscale n/16 bytes")
            io[i].out_e2m1 = _dev(e2m1[i], torch.uint8, "e2m1").value
            io[i].blk_scale_e4m3 = _dev(bscale[i], torch.uint8, "bscale").value
            io[i].gscale_dev = gscale.data_ptr() + 4 * i
    return io, n


def calibrate_quantize_qkv(xs, amax, codes8, scale8, workspace, mode: int = MODE_FP8,
                           e2m1=None, bscale=None, gscale=None, stream=None):
    """Q, K, V in one launch.  xs: three bf16 tensors of n elements; amax, scale8 (and gscale
    in FP4 mode): float32 tensors of 3 elements (one per tensor); codes8, e2m1, bscale: lists of
    three uint8 tensors."""
    io, n = _qkv_io(xs, amax, codes8, scale8, mode, e2m1, bscale, gscale)
    _check(load().qattn_calibrate_quantize_qkv(io, n, int(mode), _dev(workspace, torch.uint8, "workspace"),
                                               workspace.numel(), _stream(stream)),
           "qattn_calibrate_quantize_qkv")


def quantize_qkv(xs, amax, codes8, scale8, mode: int = MODE_FP8, e2m1=None, bscale=None,
                 gscale=None, stream=None):
    """Q, K, V with given scales in one launch: amax (float32, 3 elements) is an input, the
    other arguments as for calibrate_quantize_qkv (no workspace)."""
    io, n = _qkv_io(xs, amax, codes8, scale8, mode, e2m1, bscale, gscale)
    _check(load().qattn_quantize_qkv(io, n, int(mode), _stream(stream)), "qattn_quantize_qkv")


def gemm_fp8(a8, b8, y, s_a, s_b, stream=None):
    """y [M, N] bf16 = (a8 [M, K] b8 [N, K]^T) * s_a * s_b (E4M3 codes, K contiguous; s_a, s_b
    one-element float32 device tensors).  K % 128 == 0, N % 32 == 0."""
    if a8.dim() != 2 or b8.dim() != 2 or a8.shape[1] != b8.shape[1]:
        raise ValueError("a8 [M, K] and b8 [N, K] with the same K")
    M, K = a8.shape
    N = b8.shape[0]
    if tuple(y.shape) != (M, N):
        raise ValueError("y must be [M, N]")
    _check(load().qattn_gemm_fp8(_dev(a8, torch.uint8, "a8"), _dev(b8, torch.uint8, "b8"),
                                 _dev(y, torch.bfloat16, "y"), M, N, K,
                                 _dev(s_a, torch.float32, "s_a"), _dev(s_b, torch.float32, "s_b"),
                                 _stream(stream)), "qattn_gemm_fp8")


def gemm_fp8_e4m3(a8, b8, codes, s_a, s_b, amax, scale_out, y=None, stream=None):
    """The FP8 GEMM with its bf16 output quantized to E4M3 in the epilogue under a static amax:
    codes [M, N] uint8 = e4m3(y / s), s = amax / 448 written to scale_out (one-element float32
    device tensors); y [M, N] bf16 optional.  K % 128 == 0, N % 32 == 0."""
    if a8.dim() != 2 or b8.dim() != 2 or a8.shape[1] != b8.shape[1]:
        raise ValueError("a8 [M, K] and b8 [N, K] with the same K")
    M, K = a8.shape
    N = b8.shape[0]
    if tuple(codes.shape) != (M, N) or (y is not None and tuple(y.shape) != (M, N)):
        raise ValueError("codes (and y) must be [M, N]")
    _check(load().qattn_gemm_fp8_e4m3(_dev(a8, torch.uint8, "a8"), _dev(b8, torch.uint8, "b8"),
                                      None if y is None else _dev(y, torch.bfloat16, "y"),
                                      _dev(codes, torch.uint8, "codes"), M, N, K,
                                      _dev(s_a, torch.float32, "s_a"), _dev(s_b, torch.float32, "s_b"),
                                      _dev(amax, torch.float32, "amax"),
                                      _dev(scale_out, torch.float32, "scale_out"), _stream(stream)),
           "qattn_gemm_fp8_e4m3")


def gemm_fp4(x_e2m1, x_bscale, sg_x, w_e2m1, w_bscale, sg_w, y, stream=None):
    """Per-block FP4 GEMM, Y = X W^T: x_e2m1 uint8 [M, K/2] packed E2M1, x_bscale uint8 [M, K/16]
    E4M3 block scales, sg_x float32 [1] per-tensor scale (W likewise with N rows); y bf16 [M, N].
    K % 256 == 0, N % 32 == 0."""
    M, N = y.shape
    K = 2 * x_e2m1.shape[-1]
    if (tuple(x_e2m1.shape) != (M, K // 2) or tuple(w_e2m1.shape) != (N, K // 2) or
            tuple(x_bscale.shape) != (M, K // 16) or tuple(w_bscale.shape) != (N, K // 16)):
        raise ValueError("x_e2m1 [M, K/2], x_bscale [M, K/16], w_e2m1 [N, K/2], w_bscale [N, K/16]")
    _check(load().qattn_gemm_fp4(_dev(x_e2m1, torch.uint8, "x_e2m1"), _dev(x_bscale, torch.uint8, "x_bscale"),
                                 _dev(sg_x, torch.float32, "sg_x"), _dev(w_e2m1, torch.uint8, "w_e2m1"),
                                 _dev(w_bscale, torch.uint8, "w_bscale"), _dev(sg_w, torch.float32, "sg_w"),
                                 _dev(y, torch.bfloat16, "y"), M, N, K, _stream(stream)), "qattn_gemm_fp4")


def _scales(s_q, s_k, s_v):
    return _Scales(_dev(s_q, torch.float32, "s_q").value, _dev(s_k, torch.float32, "s_k").value,
                   _dev(s_v, torch.float32, "s_v").value)


def forward_workspace_bytes(B: int, H: int, L: int, D: int) -> int:
    """Bytes of the workspace forward() uses to cut its tail pairs (0: none needed)."""
    return int(load().qattn_forward_workspace_bytes(int(B), int(H), int(L), int(D)))


def forward(q8, k8, v8, out, s_q, s_k, s_v, sm_scale: float, mode: int = MODE_FP8, stream=None,
            workspace: torch.Tensor | None = None):
    """q8, k8, v8: uint8 E4M3 codes [B, H, L, D]; out: bf16 [B, H, L, D].  With a workspace of
    forward_workspace_bytes(B, H, L, D) bytes (uint8 CUDA tensor) the persistent kernel cuts the
    pairs left after an equal share of whole pairs per SM along the keys (qattn_forward_ws);
    without one, qattn_forward."""
    B, H, L, D = q8.shape
    for t, nm in ((k8, "k8"), (v8, "v8"), (out, "out")):
        if tuple(t.shape) != (B, H, L, D):
            raise ValueError(f"{nm} shape {tuple(t.shape)} != {(B, H, L, D)}")
    sc = _scales(s_q, s_k, s_v)
    args = (_dev(q8, torch.uint8, "q8"), _dev(k8, torch.uint8, "k8"), _dev(v8, torch.uint8, "v8"),
            _dev(out, torch.bfloat16, "out"), B, H, L, D, ctypes.byref(sc), float(sm_scale),
            int(mode))
    if workspace is None:
        _check(load().qattn_forward(*args, _stream(stream)), "qattn_forward")
    else:
        _check(load().qattn_forward_ws(*args, _dev(workspace, torch.uint8, "workspace"),
                                       workspace.numel(), _stream(stream)), "qattn_forward_ws")


def forward_varlen(q8, k8, v8, out, cu_seqlens: torch.Tensor, max_seqlen: int, s_q, s_k, s_v,
                   sm_scale: float, mode: int = MODE_FP4, stream=None):
    """q8, k8, v8: uint8 [1, H, T, D]; cu_seqlens: int32 CUDA tensor [nseq + 1]."""
    _, H, T, D = q8.shape
    sc = _scales(s_q, s_k, s_v)
    _check(load().qattn_forward_varlen(
        _dev(q8, torch.uint8, "q8"), _dev(k8, torch.uint8, "k8"), _dev(v8, torch.uint8, "v8"),
        _dev(out, torch.bfloat16, "out"), _dev(cu_seqlens, torch.int32, "cu_seqlens"),
        cu_seqlens.numel() - 1, int(max_seqlen), T, H, D, ctypes.byref(sc), float(sm_scale),
        int(mode), _stream(stream)), "qattn_forward_varlen")


def get_error(stream=None) -> int:
    """Synchronizes the stream; returns (and clears) the device error word as a status."""
    return int(load().qattn_get_error(_stream(stream)))


def debug_set_wait_timeout_ns(ns: int):
    load().qattn_debug_set_wait_timeout_ns(int(ns))


def debug_inject_missing_q(enable: bool):
    load().qattn_debug_inject_missing_q(1 if enable else 0)


def debug_use_pair_kernel(enable: bool):
    """D = 128 attention on the pair-of-SMs kernel instead of the default one-SM kernel."""
    load().qattn_debug_use_pair_kernel(1 if enable else 0)


def build_info() -> int:
    """Bit 0: the loaded library is the checked build (QATTN_DEBUG=1)."""
    return int(load().qattn_build_info())


def debug_inject_oob(enable: bool):
    """Checked build only: the next quantize_fp8 launches loop one 8-element vector past n, which
    the device bounds checks must stop (QATTN_ERR_BOUNDS).  Raises QattnError in the normal build."""
    _check(load().qattn_debug_inject_oob(1 if enable else 0), "qattn_debug_inject_oob")


def debug_capture_p_row(enable: bool, slab: int = 0, row: int = 0, codes: torch.Tensor = None,
                        maxima: torch.Tensor = None):
    """Test hook: the next attention launches copy row `row` of slab `slab`'s P codes
    (uint8 [steps * 128]) and the integer maxima they are relative to (int32 [steps]) into the
    given device tensors."""
    if not enable:
        _check(load().qattn_debug_capture_p_row(0, 0, 0, None, None), "qattn_debug_capture_p_row")
        return
    assert codes.is_cuda and codes.dtype == torch.uint8 and maxima.is_cuda and maxima.dtype == torch.int32
    _check(load().qattn_debug_capture_p_row(1, slab, row, codes.data_ptr(), maxima.data_ptr()),
           "qattn_debug_capture_p_row")


def debug_attention_plan(B: int, H: int, L: int, D: int, num_sms: int) -> dict:
    """The persistent schedule of a dense forward on a GPU with num_sms SMs (host only)."""
    plan = (ctypes.c_int * 6)()
    nbytes = ctypes.c_size_t(0)
    _check(load().qattn_debug_attention_plan(int(B), int(H), int(L), int(D), int(num_sms), plan,
                                             ctypes.byref(nbytes)), "qattn_debug_attention_plan")
    keys = ("pairs_per_head", "nkv", "ctas", "whole", "tail_pairs", "tail_w")
    return dict(zip(keys, list(plan)), workspace_bytes=int(nbytes.value))
