"""The C ABI without a GPU: the library loads, exports every symbol include/qattn.h declares,
and rejects bad arguments on the host before touching the device."""
import ctypes
import os
import re

import pytest

from precision_quantized_attention_b200 import _lib

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    with open(os.path.join(ROOT, "include", "qattn.h")) as f:
        text = f.read()
    return sorted(set(re.findall(r"QATTN_API\s+[\w\s\*]+?\b(qattn_\w+)\s*\(", text)))


def test_header_declares_the_exported_set():
    assert _declared() == sorted(_lib.EXPORTS)


def test_library_loads_and_exports_every_declared_symbol():
    lib = _lib.load()
    for name in _declared():
        assert hasattr(lib, name), name
    assert _lib.status_str(5) == "QATTN_ERR_TIMEOUT"
    assert _lib.status_str(42) == "QATTN_ERR_UNKNOWN"


def test_oracle_is_not_linked_into_the_product():
    lib = _lib.load()
    with pytest.raises(AttributeError):
        getattr(lib, "orc_attention_e4m3")


FAKE = ctypes.c_void_p(0x10000)       # aligned, never dereferenced: checks come first
MISALIGNED = ctypes.c_void_p(0x10001)


def test_host_side_argument_errors():
    lib = _lib.load()
    s0 = ctypes.c_void_p(0)
    assert lib.qattn_calibrate_amax(None, 16, FAKE, s0) == _lib.ERR_INVALID_ARG
    assert lib.qattn_calibrate_amax(MISALIGNED, 16, FAKE, s0) == _lib.ERR_INVALID_ARG
    assert lib.qattn_calibrate_amax(FAKE, 0, FAKE, s0) == _lib.ERR_INVALID_ARG
    assert lib.qattn_quantize_fp8(FAKE, 16, FAKE, None, FAKE, s0) == _lib.ERR_INVALID_ARG
    # FP4 needs n % 16 == 0 and both-or-neither of the requant outputs
    assert lib.qattn_quantize_fp4_block(FAKE, 24, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, s0) == _lib.ERR_INVALID_ARG
    assert lib.qattn_quantize_fp4_block(FAKE, 32, FAKE, FAKE, FAKE, FAKE, FAKE, None, s0) == _lib.ERR_INVALID_ARG
    # fused calibrate+quantize: workspace present, large enough and aligned
    W = _lib.FUSED_WORKSPACE_BYTES
    cq8 = lib.qattn_calibrate_quantize_fp8
    assert cq8(FAKE, 16, FAKE, FAKE, FAKE, None, W, s0) == _lib.ERR_INVALID_ARG
    assert cq8(FAKE, 16, FAKE, FAKE, FAKE, FAKE, W - 1, s0) == _lib.ERR_INVALID_ARG
    assert cq8(FAKE, 16, FAKE, FAKE, FAKE, ctypes.c_void_p(0x10008), W, s0) == _lib.ERR_INVALID_ARG
    assert cq8(FAKE, 0, FAKE, FAKE, FAKE, FAKE, W, s0) == _lib.ERR_INVALID_ARG
    assert cq8(MISALIGNED, 16, FAKE, FAKE, FAKE, FAKE, W, s0) == _lib.ERR_INVALID_ARG
    cq4 = lib.qattn_calibrate_quantize_fp4_block
    assert cq4(FAKE, 24, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, W, s0) == _lib.ERR_INVALID_ARG
    assert cq4(FAKE, 32, FAKE, FAKE, FAKE, FAKE, None, FAKE, FAKE, W, s0) == _lib.ERR_INVALID_ARG
    assert cq4(FAKE, 32, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 16, s0) == _lib.ERR_INVALID_ARG
    na = lib.qattn_calibrate_quantize_fp8_noalloc
    assert na(None, 16, FAKE, FAKE, FAKE, s0) == _lib.ERR_INVALID_ARG
    assert na(FAKE, 0, FAKE, FAKE, FAKE, s0) == _lib.ERR_INVALID_ARG
    assert na(MISALIGNED, 16, FAKE, FAKE, FAKE, s0) == _lib.ERR_INVALID_ARG
    qkv = lib.qattn_calibrate_quantize_qkv
    io = (_lib.QuantIO * 3)(*[_lib.QuantIO(0x10000, 0x10000, 0x10000, 0x10000, 0x10000, 0x10000,
                                           0x10000) for _ in range(3)])
    assert qkv(None, 16, 0, FAKE, W, s0) == _lib.ERR_INVALID_ARG
    assert qkv(io, 0, 0, FAKE, W, s0) == _lib.ERR_INVALID_ARG
    assert qkv(io, 16, 2, FAKE, W, s0) == _lib.ERR_INVALID_ARG            # bad mode
    assert qkv(io, 24, 1, FAKE, W, s0) == _lib.ERR_INVALID_ARG            # FP4 needs n % 16 == 0
    assert qkv(io, 16, 0, FAKE, W - 1, s0) == _lib.ERR_INVALID_ARG
    io[1].x_bf16 = 0x10001                                                # misaligned input
    assert qkv(io, 16, 0, FAKE, W, s0) == _lib.ERR_INVALID_ARG
    io[1].x_bf16 = 0x10000
    io[2].out_e2m1 = None                                                 # FP4 output missing
    assert qkv(io, 32, 1, FAKE, W, s0) == _lib.ERR_INVALID_ARG
    sq = lib.qattn_quantize_qkv                                           # given scales
    io[2].out_e2m1 = 0x10000
    assert sq(None, 16, 0, s0) == _lib.ERR_INVALID_ARG
    assert sq(io, 0, 0, s0) == _lib.ERR_INVALID_ARG
    assert sq(io, 16, 2, s0) == _lib.ERR_INVALID_ARG                      # bad mode
    assert sq(io, 24, 1, s0) == _lib.ERR_INVALID_ARG                      # FP4 needs n % 16 == 0
    io[0].amax_dev = None                                                 # the scales are inputs
    assert sq(io, 16, 0, s0) == _lib.ERR_INVALID_ARG
    io[0].amax_dev = 0x10000
    io[1].out_e4m3 = 0x10004                                              # codes not 8-byte aligned
    assert sq(io, 16, 0, s0) == _lib.ERR_INVALID_ARG
    sc = _lib._Scales(0x10000, 0x10000, 0x10000)
    fws = lib.qattn_forward_ws
    assert fws(FAKE, FAKE, FAKE, FAKE, 1, 1, 16, 64, ctypes.byref(sc), 0.1, 0, MISALIGNED, 1 << 20,
               s0) == _lib.ERR_INVALID_ARG                            # misaligned workspace
    assert fws(FAKE, FAKE, FAKE, FAKE, 1, 1, 16, 96, ctypes.byref(sc), 0.1, 0, FAKE, 1 << 20,
               s0) == _lib.ERR_UNSUPPORTED
    assert lib.qattn_forward_workspace_bytes(1, 1, 16, 96) == 0          # D not supported
    assert lib.qattn_forward_workspace_bytes(1, 0, 16, 64) == 0
    fwd = lib.qattn_forward
    # maximum sizes: B*H*L*D >= 2^40 elements and B or H > 65535 are refused on the host
    assert fwd(FAKE, FAKE, FAKE, FAKE, 1, 65535, 1 << 20, 128, ctypes.byref(sc), 0.1, 0,
               s0) == _lib.ERR_UNSUPPORTED
    assert fwd(FAKE, FAKE, FAKE, FAKE, 70000, 1, 16, 64, ctypes.byref(sc), 0.1, 0,
               s0) == _lib.ERR_UNSUPPORTED
    assert fwd(FAKE, FAKE, FAKE, FAKE, 1, 1, 16, 96, ctypes.byref(sc), 0.1, 0, s0) == _lib.ERR_UNSUPPORTED
    assert fwd(FAKE, FAKE, FAKE, FAKE, 1, 1, 0, 64, ctypes.byref(sc), 0.1, 0, s0) == _lib.ERR_INVALID_ARG
    assert fwd(FAKE, FAKE, FAKE, FAKE, 1, 1, 16, 64, ctypes.byref(sc), -1.0, 0, s0) == _lib.ERR_INVALID_ARG
    assert fwd(FAKE, FAKE, FAKE, FAKE, 1, 1, 16, 64, ctypes.byref(sc), 0.1, 7, s0) == _lib.ERR_INVALID_ARG
    assert fwd(MISALIGNED, FAKE, FAKE, FAKE, 1, 1, 16, 64, ctypes.byref(sc), 0.1, 0, s0) == _lib.ERR_INVALID_ARG
    assert fwd(FAKE, FAKE, FAKE, FAKE, 1, 1, 16, 64, None, 0.1, 0, s0) == _lib.ERR_INVALID_ARG
    bad = _lib._Scales(0x10000, 0, 0x10000)
    assert fwd(FAKE, FAKE, FAKE, FAKE, 1, 1, 16, 64, ctypes.byref(bad), 0.1, 0, s0) == _lib.ERR_INVALID_ARG
    vl = lib.qattn_forward_varlen
    assert vl(FAKE, FAKE, FAKE, FAKE, None, 2, 8, 16, 1, 64, ctypes.byref(sc), 0.1, 1, s0) == _lib.ERR_INVALID_ARG
    assert vl(FAKE, FAKE, FAKE, FAKE, FAKE, 2, 32, 16, 1, 64, ctypes.byref(sc), 0.1, 1, s0) == _lib.ERR_INVALID_ARG


def test_gemm_argument_errors():
    """qattn_gemm_fp8 refuses on the host, before any launch: null or misaligned buffers, K not
    a multiple of the 128-byte K block, N not a multiple of the 32-column epilogue chunk."""
    lib = _lib.load()
    g = lib.qattn_gemm_fp8
    s0 = ctypes.c_void_p(0)
    ok = (FAKE, FAKE, FAKE, 256, 256, 256, FAKE, FAKE, s0)

    def call(**kw):
        a = list(ok)
        for i, name in enumerate(("a8", "b8", "y", "M", "N", "K", "s_a", "s_b")):
            if name in kw:
                a[i] = kw[name]
        return g(*a)

    for kw in ({"a8": None}, {"b8": None}, {"y": None}, {"s_a": None}, {"s_b": None},
               {"a8": MISALIGNED}, {"b8": MISALIGNED}, {"y": MISALIGNED},
               {"s_a": ctypes.c_void_p(0x10002)}, {"M": 0}, {"N": 16}, {"N": 48}, {"K": 64},
               {"K": 200}):
        assert call(**kw) == _lib.ERR_INVALID_ARG, kw


def test_gemm_e4m3_argument_errors():
    """qattn_gemm_fp8_e4m3 refuses on the host, before any launch: null codes, amax or scale
    output, misaligned buffers (a null y is allowed: codes only), and the shapes qattn_gemm_fp8
    refuses."""
    lib = _lib.load()
    g = lib.qattn_gemm_fp8_e4m3
    s0 = ctypes.c_void_p(0)
    names = ("a8", "b8", "y", "codes", "M", "N", "K", "s_a", "s_b", "amax", "scale")
    ok = (FAKE, FAKE, FAKE, FAKE, 256, 256, 256, FAKE, FAKE, FAKE, FAKE, s0)

    def call(**kw):
        a = list(ok)
        for i, name in enumerate(names):
            if name in kw:
                a[i] = kw[name]
        return g(*a)

    for kw in ({"a8": None}, {"b8": None}, {"codes": None}, {"s_a": None}, {"s_b": None},
               {"amax": None}, {"scale": None}, {"codes": MISALIGNED}, {"y": MISALIGNED},
               {"amax": ctypes.c_void_p(0x10002)}, {"M": 0}, {"N": 48}, {"K": 200}):
        assert call(**kw) == _lib.ERR_INVALID_ARG, kw


def test_checked_build_exports_the_same_symbols_and_says_so():
    """libqattn_checked.so (QATTN_DEBUG=1) is the same C ABI compiled with device bounds checks:
    it exports every declared symbol, reports bit 0 in qattn_build_info, accepts the overrun
    injection and names QATTN_ERR_BOUNDS; the normal build reports 0 and refuses the injection."""
    from precision_quantized_attention_b200 import build
    path = build.build(checked=True)             # a no-op when it is up to date
    checked = ctypes.CDLL(path)
    for name in _declared():
        assert hasattr(checked, name), name
    checked.qattn_status_str.restype = ctypes.c_char_p
    assert checked.qattn_build_info() == 1
    assert checked.qattn_debug_inject_oob(0) == _lib.OK
    assert checked.qattn_status_str(_lib.ERR_BOUNDS) == b"QATTN_ERR_BOUNDS"
    normal = _lib.load()
    if not _lib.CHECKED:
        assert normal.qattn_build_info() == 0
        assert normal.qattn_debug_inject_oob(1) == _lib.ERR_UNSUPPORTED


def test_p_unquantized_flag_is_validated_on_the_host():
    """QATTN_FLAG_P_UNQUANTIZED combines with either mode; other high bits are refused, and the
    flag's own limit (B * H grid rows <= 65535) is checked on the host."""
    lib = _lib.load()
    s0 = ctypes.c_void_p(0)
    sc = _lib._Scales(0x10000, 0x10000, 0x10000)
    fwd = lib.qattn_forward
    flag = _lib.FLAG_P_UNQUANTIZED
    assert fwd(FAKE, FAKE, FAKE, FAKE, 1, 1, 16, 64, ctypes.byref(sc), 0.1, 0x200, s0) == _lib.ERR_INVALID_ARG
    assert fwd(FAKE, FAKE, FAKE, FAKE, 1, 1, 16, 64, ctypes.byref(sc), 0.1, flag | 2, s0) == _lib.ERR_INVALID_ARG
    assert fwd(FAKE, FAKE, FAKE, FAKE, 1, 1, 0, 64, ctypes.byref(sc), 0.1, flag, s0) == _lib.ERR_INVALID_ARG
    assert fwd(FAKE, FAKE, FAKE, FAKE, 1, 1, 16, 96, ctypes.byref(sc), 0.1, flag | 1, s0) == _lib.ERR_UNSUPPORTED
    if not _gpu():
        return
    assert fwd(FAKE, FAKE, FAKE, FAKE, 300, 300, 16, 64, ctypes.byref(sc), 0.1, flag, s0) == _lib.ERR_UNSUPPORTED


def _gpu():
    import torch
    return torch.cuda.is_available()


def test_gemm_fp4_argument_errors():
    lib = _lib.load()
    s0 = ctypes.c_void_p(0)
    g = lib.qattn_gemm_fp4
    ok = (FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE)
    assert g(None, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 128, 128, 256, s0) == _lib.ERR_INVALID_ARG
    assert g(*ok, 128, 128, 128, s0) == _lib.ERR_INVALID_ARG           # K < 256
    assert g(*ok, 128, 128, 384, s0) == _lib.ERR_INVALID_ARG           # K % 256 != 0
    assert g(*ok, 128, 48, 256, s0) == _lib.ERR_INVALID_ARG            # N % 32 != 0
    assert g(*ok, 0, 128, 256, s0) == _lib.ERR_INVALID_ARG
    assert g(FAKE, MISALIGNED, FAKE, FAKE, FAKE, FAKE, FAKE, 128, 128, 256, s0) == _lib.ERR_INVALID_ARG
