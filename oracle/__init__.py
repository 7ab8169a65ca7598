"""CPU oracle for quantized scaled-dot-product attention -- TEST INFRASTRUCTURE ONLY.

Only the test suite, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline leg may
import this package.  The CUDA library never loads it and shares no code with it.

The arithmetic lives in ``qattn_oracle.c`` (plain C, FP64/FP32, OpenMP over query rows); this
module compiles it with gcc on first use and marshals numpy arrays.  The method is the one the
NVIDIA developer blog "Optimizing FLUX.1 Kontext for Image Editing with Low-Precision
Quantization" describes in "Workflow and quantization" (SDPA bullets and Fig. 4): FakeQuantize
Q, K, V to per-tensor FP8 or per-block FP4, FP8 BMM1 with higher-precision accumulation, FP32
softmax, per-tensor FP8 P, FP8 BMM2.

``attention_fp64`` is the unquantized closed form softmax(Q K^T * sm_scale) V in FP64 (numpy
matmul as a library primitive), used to pin the oracle's attention and to report the
quantized path's error against unquantized attention.  ``gemm_e4m3`` is the plain definition of
the block's FP8 linear layers (same blog, same section: the GEMMs are quantized like the
attention inputs), also in FP64.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "qattn_oracle.c")
_LIB_PATH = os.path.join(_HERE, "_build", "liboracle.so")
_lock = threading.Lock()
_lib = None

FP32 = 1          # round scores / probabilities / row sum to binary32 (the FP32 softmax)
QUANT_P = 2       # quantize P to E4M3 with per-tensor scale 1/448 (before normalization)
FIG4_LITERAL = 4  # quantize the normalized probability instead (reported, not gated)
METHOD = FP32 | QUANT_P

OK, ERR_INVALID, ERR_NONFINITE = 0, 1, 4


def build(force: bool = False) -> str:
    """Compile the oracle with gcc (-O2, OpenMP, no fast-math).  Returns the .so path."""
    os.makedirs(os.path.dirname(_LIB_PATH), exist_ok=True)
    stale = (not os.path.exists(_LIB_PATH)
             or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC))
    if force or stale:
        tmp = _LIB_PATH + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-std=c11",
                               "-fno-fast-math", "-ffp-contract=off", "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    with _lock:
        if _lib is None:
            lib = ctypes.CDLL(build())
            P = ctypes.c_void_p
            i64, f32, f64, i32 = ctypes.c_int64, ctypes.c_float, ctypes.c_double, ctypes.c_int
            lib.orc_bf16_to_float.argtypes = [ctypes.c_uint16]
            lib.orc_bf16_to_float.restype = f32
            lib.orc_e4m3_to_float.argtypes = [ctypes.c_uint8]
            lib.orc_e4m3_to_float.restype = f32
            lib.orc_e4m3_from_float.argtypes = [f32]
            lib.orc_e4m3_from_float.restype = ctypes.c_uint8
            lib.orc_e2m1_to_float.argtypes = [ctypes.c_uint8]
            lib.orc_e2m1_to_float.restype = f32
            lib.orc_e2m1_from_float.argtypes = [f32]
            lib.orc_e2m1_from_float.restype = ctypes.c_uint8
            lib.orc_amax_bf16.argtypes = [P, i64, P]
            lib.orc_amax_bf16.restype = i32
            lib.orc_quantize_fp8.argtypes = [P, i64, f32, P, P]
            lib.orc_quantize_fp8.restype = i32
            lib.orc_quantize_fp4_block.argtypes = [P, i64, f32, P, P, P, P, P]
            lib.orc_quantize_fp4_block.restype = i32
            lib.orc_dequant_fp4_block.argtypes = [P, P, f32, i64, P]
            lib.orc_dequant_fp4_block.restype = None
            att = [P, P, P, i32, i32, i64, i32, P, i32, f64, f64, f64, f64, i32, P, i64, P, P]
            lib.orc_attention_values.argtypes = att
            lib.orc_attention_values.restype = i32
            lib.orc_attention_e4m3.argtypes = att
            lib.orc_attention_e4m3.restype = i32
            lib.orc_p_row_detail.argtypes = [P, P, i32, i32, i64, i32, P, i32, f64, f64, f64, i64,
                                             P, P, P, P, P, P, P]
            lib.orc_p_row_detail.restype = i64
            lib.orc_num_threads.argtypes = []
            lib.orc_num_threads.restype = i32
            _lib = lib
    return _lib


def _ptr(a: np.ndarray):
    assert a.flags["C_CONTIGUOUS"]
    return a.ctypes.data_as(ctypes.c_void_p)


def _bits(x) -> np.ndarray:
    """bf16 input as a contiguous uint16 array (accepts a CPU torch bf16 tensor or uint16)."""
    if hasattr(x, "view") and hasattr(x, "dtype") and str(x.dtype) == "torch.bfloat16":
        import torch
        return x.contiguous().view(torch.int16).numpy().view(np.uint16).reshape(-1)
    a = np.ascontiguousarray(x)
    assert a.dtype == np.uint16
    return a.reshape(-1)


def num_threads() -> int:
    return int(_load().orc_num_threads())


# --- scalar codecs -------------------------------------------------------------------------
def bf16_to_float(bits: int) -> float:
    return float(_load().orc_bf16_to_float(bits))


def e4m3_to_float(code: int) -> float:
    return float(_load().orc_e4m3_to_float(code))


def e4m3_from_float(x: float) -> int:
    return int(_load().orc_e4m3_from_float(x))


def e2m1_to_float(code: int) -> float:
    return float(_load().orc_e2m1_to_float(code))


def e2m1_from_float(x: float) -> int:
    return int(_load().orc_e2m1_from_float(x))


def e4m3_table() -> np.ndarray:
    """Values of all 256 E4M3 codes (NaN for 0x7F / 0xFF)."""
    return np.array([e4m3_to_float(c) for c in range(256)], dtype=np.float64)


# --- tensor ops -----------------------------------------------------------------------------
def amax(x) -> tuple[int, float]:
    b = _bits(x)
    out = np.zeros(1, dtype=np.float32)
    rc = _load().orc_amax_bf16(_ptr(b), b.size, _ptr(out))
    return rc, float(out[0])


def quantize_fp8(x, amax_value: float):
    """Returns (codes uint8 [n], scale float32)."""
    b = _bits(x)
    codes = np.empty(b.size, dtype=np.uint8)
    s = np.zeros(1, dtype=np.float32)
    rc = _load().orc_quantize_fp8(_ptr(b), b.size, np.float32(amax_value), _ptr(codes), _ptr(s))
    if rc != OK:
        raise ValueError(f"orc_quantize_fp8 failed with status {rc}")
    return codes, np.float32(s[0])


def quantize_fp4_block(x, amax_value: float, requant: bool = True):
    """Returns (packed uint8 [n/2], block scales uint8 [n/16], s_g, codes8 uint8 [n], s8)."""
    b = _bits(x)
    n = b.size
    packed = np.empty(n // 2, dtype=np.uint8)
    bscale = np.empty(n // 16, dtype=np.uint8)
    sg = np.zeros(1, dtype=np.float32)
    codes8 = np.empty(n, dtype=np.uint8) if requant else None
    s8 = np.zeros(1, dtype=np.float32)
    rc = _load().orc_quantize_fp4_block(
        _ptr(b), n, np.float32(amax_value), _ptr(packed), _ptr(bscale), _ptr(sg),
        _ptr(codes8) if requant else None, _ptr(s8) if requant else None)
    if rc != OK:
        raise ValueError(f"orc_quantize_fp4_block failed with status {rc}")
    return packed, bscale, np.float32(sg[0]), codes8, np.float32(s8[0])


def dequant_fp4_block(packed, bscale, sg, n) -> np.ndarray:
    out = np.empty(n, dtype=np.float32)
    _load().orc_dequant_fp4_block(_ptr(np.ascontiguousarray(packed)),
                                  _ptr(np.ascontiguousarray(bscale)), np.float32(sg), n, _ptr(out))
    return out


def _cu(cu_seqlens, T):
    if cu_seqlens is None:
        return np.array([0, T], dtype=np.int64)
    return np.ascontiguousarray(np.asarray(cu_seqlens, dtype=np.int64))


def attention_values(q, k, v, s_q=1.0, s_k=1.0, s_v=1.0, sm_scale=None, flags=METHOD,
                     cu_seqlens=None, rows=None) -> np.ndarray:
    """Oracle attention over values q, k, v: float arrays [B, H, T, D]."""
    q = np.ascontiguousarray(q, dtype=np.float64)
    k = np.ascontiguousarray(k, dtype=np.float64)
    v = np.ascontiguousarray(v, dtype=np.float64)
    B, H, T, D = q.shape
    sm = 1.0 / np.sqrt(D) if sm_scale is None else sm_scale
    cu = _cu(cu_seqlens, T)
    r = None if rows is None else np.ascontiguousarray(np.asarray(rows, dtype=np.int64))
    nrows = B * H * T if r is None else r.size
    out = np.empty((nrows, D), dtype=np.float64)
    rc = _load().orc_attention_values(_ptr(q), _ptr(k), _ptr(v), B, H, T, D, _ptr(cu),
                                      cu.size - 1, s_q, s_k, s_v, sm, flags,
                                      None if r is None else _ptr(r), nrows, _ptr(out), None)
    if rc != OK:
        raise ValueError(f"orc_attention_values failed with status {rc}")
    return out if r is not None else out.reshape(B, H, T, D)


def attention_e4m3(q8, k8, v8, shape, s_q, s_k, s_v, sm_scale=None, flags=METHOD,
                   cu_seqlens=None, rows=None, with_ambiguity=False):
    """Oracle attention over E4M3 codes (uint8 arrays of B*H*T*D) with per-tensor scales.

    with_ambiguity=True also returns, per output, the largest change that choosing the other
    code of an ambiguous P decision can make (P codes whose FP32 rounding boundary lies within
    the accumulation-order uncertainty of the score; see the C source)."""
    B, H, T, D = shape
    sm = 1.0 / np.sqrt(D) if sm_scale is None else sm_scale
    q8, k8, v8 = (np.ascontiguousarray(a, dtype=np.uint8).reshape(-1) for a in (q8, k8, v8))
    assert q8.size == k8.size == v8.size == B * H * T * D
    cu = _cu(cu_seqlens, T)
    r = None if rows is None else np.ascontiguousarray(np.asarray(rows, dtype=np.int64))
    nrows = B * H * T if r is None else r.size
    out = np.empty((nrows, D), dtype=np.float64)
    amb = np.empty((nrows, D), dtype=np.float64) if with_ambiguity else None
    rc = _load().orc_attention_e4m3(_ptr(q8), _ptr(k8), _ptr(v8), B, H, T, D, _ptr(cu),
                                    cu.size - 1, float(s_q), float(s_k), float(s_v), sm, flags,
                                    None if r is None else _ptr(r), nrows, _ptr(out),
                                    _ptr(amb) if with_ambiguity else None)
    if rc != OK:
        raise ValueError(f"orc_attention_e4m3 failed with status {rc}")
    if r is None:
        out = out.reshape(B, H, T, D)
        amb = amb.reshape(B, H, T, D) if with_ambiguity else None
    return (out, amb) if with_ambiguity else out


def p_row_detail(q8, k8, shape, s_q, s_k, row, sm_scale=None, cu_seqlens=None):
    """The method's P decisions for one query row (row = (b * H + h) * T + t) over E4M3 codes:
    per key of its sequence the E4M3 code of p * 448, x = S' - M (base-2 score minus the integer
    row max), the accumulation-order radius delta of S' and the codes lo, hi of
    2^(x -+ delta) * 448 (the range of codes another FP32 summation order may give; see
    orc_p_row_detail in the C source); and M and the FP32 row sum l of the unquantized p.
    Returns (codes, x, delta, lo, hi, M, l)."""
    B, H, T, D = shape
    sm = 1.0 / np.sqrt(D) if sm_scale is None else sm_scale
    q8, k8 = (np.ascontiguousarray(a, dtype=np.uint8).reshape(-1) for a in (q8, k8))
    cu = _cu(cu_seqlens, T)
    code = np.empty(T, dtype=np.uint8)
    x = np.empty(T, dtype=np.float64)
    delta = np.empty(T, dtype=np.float64)
    lo = np.empty(T, dtype=np.uint8)
    hi = np.empty(T, dtype=np.uint8)
    M = ctypes.c_double()
    l = ctypes.c_double()
    n = _load().orc_p_row_detail(_ptr(q8), _ptr(k8), B, H, T, D, _ptr(cu), cu.size - 1, float(s_q),
                                 float(s_k), sm, int(row), _ptr(code), _ptr(x), _ptr(delta),
                                 _ptr(lo), _ptr(hi), ctypes.byref(M), ctypes.byref(l))
    if n < 0:
        raise ValueError(f"orc_p_row_detail failed with status {n}")
    return code[:n], x[:n], delta[:n], lo[:n], hi[:n], M.value, l.value


def attention_fp64(q, k, v, sm_scale=None, cu_seqlens=None) -> np.ndarray:
    """Unquantized closed form softmax(q k^T * sm_scale) v per sequence, FP64 throughout."""
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    B, H, T, D = q.shape
    sm = 1.0 / np.sqrt(D) if sm_scale is None else sm_scale
    cu = _cu(cu_seqlens, T)
    out = np.empty_like(q)
    for s in range(cu.size - 1):
        a, b = int(cu[s]), int(cu[s + 1])
        logits = np.einsum("bhid,bhjd->bhij", q[:, :, a:b], k[:, :, a:b]) * sm
        logits -= logits.max(axis=-1, keepdims=True)
        w = np.exp(logits)
        w /= w.sum(axis=-1, keepdims=True)
        out[:, :, a:b] = np.einsum("bhij,bhjd->bhid", w, v[:, :, a:b])
    return out


# --- the whole method, from bf16 inputs --------------------------------------------------------
def quantize_tensor(x, mode: str):
    """FakeQuantize one bf16 tensor for BMM input: returns (e4m3 codes [n], scale, extras)."""
    rc, a = amax(x)
    if rc != OK:
        raise ValueError("non-finite input")
    if mode == "fp8":
        codes, s = quantize_fp8(x, a)
        return codes, s, {"amax": a}
    if mode == "fp4":
        packed, bscale, sg, codes8, s8 = quantize_fp4_block(x, a)
        return codes8, s8, {"amax": a, "packed": packed, "bscale": bscale, "sg": sg}
    raise ValueError(mode)


def method_forward(q, k, v, mode="fp8", sm_scale=None, cu_seqlens=None, rows=None,
                   flags=METHOD, with_ambiguity=False):
    """The quantized SDPA from bf16 inputs [B, H, T, D] (CPU torch bf16 tensors)."""
    shape = tuple(q.shape)
    q8, sq, _ = quantize_tensor(q, mode)
    k8, sk, _ = quantize_tensor(k, mode)
    v8, sv, _ = quantize_tensor(v, mode)
    return attention_e4m3(q8, k8, v8, shape, sq, sk, sv, sm_scale, flags, cu_seqlens, rows,
                          with_ambiguity)


def e2m1_table() -> np.ndarray:
    """Values of the 16 E2M1 codes."""
    return np.array([e2m1_to_float(c) for c in range(16)], dtype=np.float64)


def unpack_e2m1(packed, k: int) -> np.ndarray:
    """E2M1 codes [rows, k] from their packed form [rows, k / 2]: element 2i in the low nibble of
    byte i, element 2i + 1 in the high nibble (the layout quantize_fp4_block writes)."""
    p = np.asarray(packed, dtype=np.uint8).reshape(-1, k // 2)
    codes = np.empty((p.shape[0], k), dtype=np.uint8)
    codes[:, 0::2] = p & 0x0F
    codes[:, 1::2] = p >> 4
    return codes


def gemm_fp4_block(a_packed, a_bscale, sg_a, b_packed, b_bscale, sg_b, k: int, rows=None):
    """The per-block FP4 linear layer, Y = X W^T, as its plain definition in FP64.  X [M, k] and
    W [N, k] are in the per-block FP4 format of quantize_fp4_block: packed E2M1 codes [rows, k/2],
    E4M3 block scales [rows, k/16] (block b covers columns 16 b .. 16 b + 15) and a per-tensor
    FP32 scale s_g;
        Y[m, n] = (sum_k val(a[m, k]) val(sa[m, k/16]) val(b[n, k]) val(sb[n, k/16])) sg_a sg_b,
    the per-tensor scales applied once to the block-scaled dot product (as a block-scaled tensor
    core GEMM does), not through the FP32-rounded per-element dequantization of
    dequant_fp4_block.  numpy matmul as the library primitive; the block-scaled values are exact
    in FP64.  rows: optional row indices of Y.  Returns (Y, bound), bound[m, n] = sum_k |terms|,
    the scale an FP32 accumulation error is relative to."""
    t2, t8 = e2m1_table(), e4m3_table()
    a = t2[unpack_e2m1(a_packed, k)] * np.repeat(t8[np.asarray(a_bscale, np.uint8).reshape(-1, k // 16)], 16, axis=1)
    b = t2[unpack_e2m1(b_packed, k)] * np.repeat(t8[np.asarray(b_bscale, np.uint8).reshape(-1, k // 16)], 16, axis=1)
    if rows is not None:
        a = a[np.asarray(rows)]
    g = float(np.float32(sg_a)) * float(np.float32(sg_b))
    return (a @ b.T) * g, (np.abs(a) @ np.abs(b).T) * abs(g)


def gemm_e4m3(a8, b8, s_a, s_b, rows=None):
    """The FP8 linear layer, Y = X W^T, as its plain definition in FP64: a8 [M, K] and b8 [N, K]
    E4M3 codes (uint8), s_a, s_b their per-tensor dequantization multipliers;
    Y[m, n] = sum_k (val(a8[m, k]) s_a) (val(b8[n, k]) s_b).  numpy matmul as the library
    primitive.  rows: optional row indices of Y to compute.  Returns (Y, bound) with
    bound[m, n] = sum_k |val(a8[m, k]) s_a| |val(b8[n, k]) s_b|, the scale of the terms that an
    FP32 accumulation error is relative to."""
    tab = e4m3_table()
    a8 = np.asarray(a8)
    if rows is not None:
        a8 = a8[np.asarray(rows)]
    a = tab[a8] * float(s_a)
    b = tab[np.asarray(b8)] * float(s_b)
    return a @ b.T, np.abs(a) @ np.abs(b).T
