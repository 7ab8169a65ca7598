"""Pins for the oracle's number formats, calibration and FakeQuantize (CPU only).

The blog ("Workflow and quantization", Fig. 4) names per-tensor FP8 and per-block FP4
FakeQuantize but not the encodings; the pins therefore come from the format definitions
(golden points from the OCP specifications), from an independent library conversion
(ml_dtypes, round-to-nearest-even) and from brute force.
"""
import os

import ml_dtypes
import numpy as np
import pytest
import torch

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "format_points.txt")


def _golden():
    rows = []
    with open(GOLDEN) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            fmt, code, val = line.split()
            rows.append((fmt, int(code, 16), float(val)))
    return rows


def test_golden_format_points():
    rows = _golden()
    assert len(rows) >= 20
    for fmt, code, val in rows:
        dec = oracle.e4m3_to_float(code) if fmt == "e4m3" else oracle.e2m1_to_float(code)
        enc = oracle.e4m3_from_float(val) if fmt == "e4m3" else oracle.e2m1_from_float(val)
        assert dec == val and np.signbit(dec) == np.signbit(val), (fmt, hex(code), dec, val)
        assert enc == code, (fmt, val, hex(enc), hex(code))


def test_e4m3_decode_all_codes_vs_library():
    codes = np.arange(256, dtype=np.uint8)
    ref = codes.view(ml_dtypes.float8_e4m3fn).astype(np.float64)
    mine = oracle.e4m3_table()
    nan = np.isnan(ref)
    assert np.array_equal(nan, np.isnan(mine)) and nan.sum() == 2
    assert np.array_equal(ref[~nan], mine[~nan])
    assert np.array_equal(np.signbit(ref[~nan]), np.signbit(mine[~nan]))


def test_e4m3_roundtrip_and_midpoints():
    vals = oracle.e4m3_table()
    finite = [c for c in range(256) if not np.isnan(vals[c])]
    for c in finite:
        assert oracle.e4m3_from_float(float(vals[c])) == c
    # every midpoint between neighbouring positive codes rounds to the even code (ties-to-even)
    pos = sorted(c for c in finite if c < 0x80)
    for lo, hi in zip(pos[:-1], pos[1:]):
        mid = np.float32((vals[lo] + vals[hi]) / 2)
        assert float(mid) == (vals[lo] + vals[hi]) / 2          # midpoint exact in binary32
        want = lo if lo % 2 == 0 else hi
        assert oracle.e4m3_from_float(float(mid)) == want, (lo, hi, float(mid))
        assert oracle.e4m3_from_float(float(-mid)) == (want | 0x80)
        below = np.nextafter(mid, np.float32(0))
        above = np.nextafter(mid, np.float32(1e9))
        assert oracle.e4m3_from_float(float(below)) == lo
        assert oracle.e4m3_from_float(float(above)) == hi


def test_e4m3_encode_random_vs_library():
    rng = np.random.default_rng(7)
    x = np.concatenate([
        rng.uniform(-463.0, 463.0, 20000),
        rng.uniform(-0.02, 0.02, 20000),                    # subnormal band and below
        rng.standard_normal(20000) * 30.0,
    ]).astype(np.float32)
    x = x[np.abs(x) < 464.0]                                # the library turns overflow into NaN
    ref = x.astype(ml_dtypes.float8_e4m3fn).view(np.uint8)
    mine = np.array([oracle.e4m3_from_float(float(v)) for v in x], dtype=np.uint8)
    assert np.array_equal(ref, mine)


def test_e4m3_saturation_subnormals_and_signed_zero():
    f = oracle.e4m3_from_float
    assert f(448.0001) == 0x7E and f(464.0) == 0x7E and f(480.0) == 0x7E and f(1e6) == 0x7E
    assert f(-1e30) == 0xFE and f(float("inf")) == 0x7E and f(float("-inf")) == 0xFE
    assert f(2.0 ** -9) == 0x01
    assert f(2.0 ** -10) == 0x00                  # tie between 0 and 2^-9 -> even (0)
    assert f(1.5 * 2.0 ** -10) == 0x01
    assert f(3.0 * 2.0 ** -10) == 0x02            # tie between 2^-9 and 2^-8 -> even code 2
    assert f(-0.0) == 0x80 and f(0.0) == 0x00
    assert f(-(2.0 ** -11)) == 0x80               # negative underflow keeps its sign
    assert f(0.9375 * 2.0 ** -6) == 0x08          # rounds up out of the subnormal band


def test_e2m1_all_codes_vs_library_and_brute_force():
    codes = np.arange(16, dtype=np.uint8)
    ref = codes.view(ml_dtypes.float4_e2m1fn).astype(np.float64)
    mine = np.array([oracle.e2m1_to_float(int(c)) for c in codes])
    assert np.array_equal(ref, mine) and np.array_equal(np.signbit(ref), np.signbit(mine))
    grid = mine[:8]
    # brute force: nearest grid value, ties to the even code; saturate above 6
    xs = np.concatenate([np.arange(0, 7.01, 0.03125), [0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0, 6.1]])
    for x in xs:
        d = np.abs(grid - x)
        best = np.flatnonzero(d == d.min())
        want = int(best[0]) if len(best) == 1 else int(best[best % 2 == 0][0])
        if x > 6.0:
            want = 7
        assert oracle.e2m1_from_float(float(x)) == want, x
        assert oracle.e2m1_from_float(float(-x)) == (want | 8), x
    # the library agrees on a random sample (it saturates too)
    rng = np.random.default_rng(3)
    x = rng.uniform(-8, 8, 5000).astype(np.float32)
    lib = x.astype(ml_dtypes.float4_e2m1fn).view(np.uint8)
    mine = np.array([oracle.e2m1_from_float(float(v)) for v in x], dtype=np.uint8)
    assert np.array_equal(lib, mine)
    # the tie points of the blueprint's list
    expect = {0.25: 0, 0.75: 2, 1.25: 2, 1.75: 4, 2.5: 4, 3.5: 6, 5.0: 6, 6.1: 7}
    for x, c in expect.items():
        assert oracle.e2m1_from_float(x) == c, x


def _bf16(a) -> torch.Tensor:
    return torch.as_tensor(np.asarray(a, dtype=np.float32)).to(torch.bfloat16)


def _f32(t: torch.Tensor) -> np.ndarray:
    return t.float().numpy().reshape(-1)


def test_amax_exact_and_nonfinite():
    x = torch.randn(10007, generator=torch.Generator().manual_seed(1)).to(torch.bfloat16)
    rc, a = oracle.amax(x)
    assert rc == oracle.OK and a == float(np.max(np.abs(_f32(x))))
    for bad in (float("inf"), float("nan"), float("-inf")):
        y = x.clone()
        y[5000] = bad
        rc, _ = oracle.amax(y)
        assert rc == oracle.ERR_NONFINITE
    rc, a = oracle.amax(torch.zeros(64, dtype=torch.bfloat16))
    assert rc == oracle.OK and a == 0.0


def _fp8_independent(x: torch.Tensor):
    """FP8 per-tensor quantize by library routines: binary32 arithmetic in numpy and the
    ml_dtypes RNE conversion, with saturation applied before the conversion."""
    xf = _f32(x)
    amax = np.float32(np.max(np.abs(xf)))
    s = np.float32(1.0) if amax == 0 else np.float32(amax / np.float32(448.0))
    y = (xf / s).astype(np.float32)
    y = np.clip(y, np.float32(-448.0), np.float32(448.0))
    return y.astype(ml_dtypes.float8_e4m3fn).view(np.uint8), s


@pytest.mark.parametrize("n,scale", [(4096, 1.0), (12345, 37.5), (2048, 1e-3), (999, 3e4)])
def test_quantize_fp8_vs_independent(n, scale):
    g = torch.Generator().manual_seed(n)
    x = (torch.randn(n, generator=g) * scale).to(torch.bfloat16)
    _, a = oracle.amax(x)
    codes, s = oracle.quantize_fp8(x, a)
    ref_codes, ref_s = _fp8_independent(x)
    assert s == ref_s
    assert np.array_equal(codes, ref_codes)
    # the element holding the amax maps to the top code
    i = int(np.argmax(np.abs(_f32(x))))
    assert codes[i] & 0x7F == 0x7E


def test_quantize_fp8_zero_tensor():
    codes, s = oracle.quantize_fp8(torch.zeros(32, dtype=torch.bfloat16), 0.0)
    assert s == 1.0 and np.all(codes == 0)


def _fp4_independent(x: torch.Tensor):
    """FP4 block quantize + FP8 requant by library routines (numpy binary32, ml_dtypes RNE)."""
    xf = _f32(x).astype(np.float32)
    f32 = np.float32
    amax = f32(np.max(np.abs(xf)))
    sg = f32(1.0) if amax == 0 else f32(amax / f32(2688.0))
    six = f32(f32(6.0) * sg)
    blocks = xf.reshape(-1, 16)
    amax_b = np.max(np.abs(blocks), axis=1).astype(np.float32)
    r = np.clip((amax_b / six).astype(np.float32), f32(-448), f32(448))
    sb = r.astype(ml_dtypes.float8_e4m3fn)
    sb_code = sb.view(np.uint8)
    eff = (sb.astype(np.float32) * sg).astype(np.float32)
    with np.errstate(divide="ignore", invalid="ignore"):
        y = (blocks / eff[:, None]).astype(np.float32)
    c = y.astype(ml_dtypes.float4_e2m1fn)
    c = np.where(eff[:, None] == 0, np.zeros_like(c), c)
    code = c.view(np.uint8).reshape(-1) & 0xF
    packed = (code[0::2] | (code[1::2] << 4)).astype(np.uint8)
    xhat = ((c.astype(np.float32) * sb.astype(np.float32)[:, None]).astype(np.float32) * sg)
    xhat = xhat.astype(np.float32).reshape(-1)
    m = f32(np.max(np.abs(xhat)))
    s8 = f32(1.0) if m == 0 else f32(m / f32(448.0))
    c8 = np.clip((xhat / s8).astype(np.float32), f32(-448), f32(448)).astype(ml_dtypes.float8_e4m3fn)
    return packed, sb_code, sg, c8.view(np.uint8), s8, xhat


@pytest.mark.parametrize("n,scale", [(4096, 1.0), (16 * 777, 12.0), (2048, 1e-2)])
def test_quantize_fp4_vs_independent(n, scale):
    g = torch.Generator().manual_seed(n + 1)
    x = (torch.randn(n, generator=g) * scale).to(torch.bfloat16)
    # a block of tiny values makes some block scales round to zero or subnormal
    x[:16] = x[:16] * 1e-4
    _, a = oracle.amax(x)
    packed, bscale, sg, c8, s8 = oracle.quantize_fp4_block(x, a)
    r_packed, r_bscale, r_sg, r_c8, r_s8, xhat = _fp4_independent(x)
    assert sg == r_sg and s8 == r_s8
    assert np.array_equal(bscale, r_bscale)
    assert np.array_equal(packed, r_packed)
    assert np.array_equal(c8, r_c8)
    mine_xhat = oracle.dequant_fp4_block(packed, bscale, sg, n)
    assert np.array_equal(mine_xhat, xhat)
    # closed form of the requant scale: max|xhat| = fl32(2688 * s_g)
    assert np.float32(np.max(np.abs(mine_xhat))) == np.float32(np.float32(2688.0) * sg)
    assert s8 == np.float32(np.float32(np.float32(2688.0) * sg) / np.float32(448.0))


def test_fp4_packing_order_and_amax_block():
    x = np.zeros(32, dtype=np.float32)
    x[0] = 6.0      # element 0 -> low nibble of byte 0
    x[3] = -3.0     # element 3 -> high nibble of byte 1
    x[17] = 1.0     # second block
    t = _bf16(x)
    _, a = oracle.amax(t)
    packed, bscale, sg, c8, s8 = oracle.quantize_fp4_block(t, a)
    assert sg == np.float32(np.float32(6.0) / np.float32(2688.0))
    assert bscale[0] == 0x7E                          # block holding amax gets scale 448
    assert packed[0] == 0x07 and packed[1] == (0xD << 4)   # -3.0 is code 0xD
    assert c8[0] == 0x7E                              # the amax element requantizes to 448


def test_fp4_error_bound():
    """|x - xhat| is at most half a grid step of the block (times 1 + 2^-3 for the scale
    rounding), the defining property of round-to-nearest on the scaled grid."""
    g = torch.Generator().manual_seed(11)
    x = torch.randn(16 * 512, generator=g).to(torch.bfloat16)
    _, a = oracle.amax(x)
    packed, bscale, sg, _, _ = oracle.quantize_fp4_block(x, a)
    xhat = oracle.dequant_fp4_block(packed, bscale, sg, x.numel()).reshape(-1, 16)
    xf = _f32(x).reshape(-1, 16)
    eff = np.array([oracle.e4m3_to_float(int(c)) for c in bscale]) * float(sg)
    # grid step is at most 2 (between 4 and 6) in units of eff; inside [0, 4] it is <= 1
    err = np.abs(xf - xhat)
    assert np.all(err <= eff[:, None] * 1.0 + 1e-12)
    # values that do not saturate are within half the local step
    assert np.all(np.abs(xf) <= eff[:, None] * 6.0 * (1 + 2.0 ** -3))
