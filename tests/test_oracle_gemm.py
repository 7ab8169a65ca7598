"""Pins of the oracle's FP8 linear layer (gemm_e4m3) against what the definition fixes: a
brute-force triple loop on a tiny case, a constant-code case with a closed form, and exact
linearity in each scale (powers of two)."""
import numpy as np

import oracle


def _codes(rng, shape):
    c = rng.integers(0, 256, size=shape, dtype=np.uint8)
    c[(c & 0x7F) == 0x7F] = 0x38               # no NaN codes
    return c


def test_gemm_matches_a_triple_loop():
    rng = np.random.default_rng(5)
    a8, b8 = _codes(rng, (3, 5)), _codes(rng, (4, 5))
    y, bound = oracle.gemm_e4m3(a8, b8, 0.5, 0.25)
    for m in range(3):
        for n in range(4):
            want = sum(oracle.e4m3_to_float(int(a8[m, k])) * 0.5 *
                       oracle.e4m3_to_float(int(b8[n, k])) * 0.25 for k in range(5))
            mag = sum(abs(oracle.e4m3_to_float(int(a8[m, k])) * 0.5 *
                          oracle.e4m3_to_float(int(b8[n, k])) * 0.25) for k in range(5))
            assert y[m, n] == want and bound[m, n] == mag


def test_gemm_constant_codes_closed_form():
    # code 0x38 is 1.0, code 0x40 is 2.0: every output is K * 1 * 2 * s_a * s_b
    K = 384
    y, _ = oracle.gemm_e4m3(np.full((7, K), 0x38, np.uint8), np.full((9, K), 0x40, np.uint8), 3.0, 0.125)
    assert np.all(y == K * 2.0 * 3.0 * 0.125)


def test_gemm_is_linear_in_each_scale_and_rows_select():
    rng = np.random.default_rng(6)
    a8, b8 = _codes(rng, (6, 256)), _codes(rng, (32, 256))
    y1, _ = oracle.gemm_e4m3(a8, b8, 1.0, 1.0)
    y2, _ = oracle.gemm_e4m3(a8, b8, 4.0, 0.5)
    assert np.array_equal(y2, 2.0 * y1)        # powers of two: exact in FP64
    y3, _ = oracle.gemm_e4m3(a8, b8, 1.0, 1.0, rows=[4, 1])
    assert np.array_equal(y3, y1[[4, 1]])


# --- the per-block FP4 linear layer (gemm_fp4_block) ----------------------------------------
def _fp4(rng, rows, k):
    """Random packed E2M1 codes and E4M3 block scales (finite, non-negative scale codes)."""
    packed = rng.integers(0, 256, size=(rows, k // 2), dtype=np.uint8)
    bscale = rng.integers(0, 0x7F, size=(rows, k // 16), dtype=np.uint8)
    return packed, bscale


def test_fp4_gemm_matches_a_triple_loop_over_nibbles():
    """Independent restatement: nibbles unpacked by hand (element 2i low, 2i + 1 high), each
    element's block scale looked up as bscale[k // 16], scalar codecs."""
    rng = np.random.default_rng(11)
    K = 32
    ap, ab = _fp4(rng, 3, K)
    bp, bb = _fp4(rng, 4, K)
    y, bound = oracle.gemm_fp4_block(ap, ab, np.float32(0.75), bp, bb, np.float32(0.5), K)
    for m in range(3):
        for n in range(4):
            want = mag = 0.0
            for k in range(K):
                ca = (int(ap[m, k // 2]) >> (4 * (k % 2))) & 0xF
                cb = (int(bp[n, k // 2]) >> (4 * (k % 2))) & 0xF
                t = (oracle.e2m1_to_float(ca) * oracle.e4m3_to_float(int(ab[m, k // 16])) *
                     oracle.e2m1_to_float(cb) * oracle.e4m3_to_float(int(bb[n, k // 16])))
                want += t
                mag += abs(t)
            assert abs(y[m, n] - want * 0.375) <= 1e-12 * mag and abs(bound[m, n] - mag * 0.375) <= 1e-12 * mag


def test_fp4_gemm_constant_codes_closed_form():
    # E2M1 code 0x2 is 1.0 (byte 0x22: both nibbles); E4M3 scale codes 0x38 = 1 and 0x40 = 2
    K = 256
    y, _ = oracle.gemm_fp4_block(np.full((5, K // 2), 0x22, np.uint8), np.full((5, K // 16), 0x38, np.uint8),
                                 np.float32(3.0), np.full((6, K // 2), 0x22, np.uint8),
                                 np.full((6, K // 16), 0x40, np.uint8), np.float32(0.125), K)
    assert np.all(y == K * 2.0 * 3.0 * 0.125)


def test_fp4_gemm_nibble_order_and_block_placement():
    """Only the low nibbles set (value 1.5 = code 0x3): Y counts the even columns alone; only
    block 2 scaled (the others 0): Y sums columns 32..47 alone.  A swapped nibble order or a
    block size other than 16 fails one of the two."""
    K = 64
    ones_b = np.full((1, K // 2), 0x22, np.uint8)                 # W = 1.0 everywhere
    scale1 = np.full((1, K // 16), 0x38, np.uint8)
    low = np.full((1, K // 2), 0x03, np.uint8)                    # even k: 1.5, odd k: 0
    y, _ = oracle.gemm_fp4_block(low, scale1, np.float32(1), ones_b, scale1, np.float32(1), K)
    assert y[0, 0] == 1.5 * (K // 2)
    a = np.zeros((1, K // 2), np.uint8)
    a[0, 20] = 0x40                                               # k = 41 (high nibble of byte 20): 2.0
    a[0, 3] = 0x04                                                # k = 6 (block 0): 2.0, scaled to 0
    ab = np.zeros((1, K // 16), np.uint8)
    ab[0, 2] = 0x48                                               # block 2 (k 32..47): scale 4
    y, _ = oracle.gemm_fp4_block(a, ab, np.float32(1), ones_b, scale1, np.float32(1), K)
    assert y[0, 0] == 2.0 * 4.0


def test_fp4_gemm_agrees_with_the_quantizer_and_its_dequantization():
    """X and W quantized by quantize_fp4_block: the GEMM equals dequant(X) dequant(W)^T up to the
    FP32 rounding that dequant_fp4_block applies per element (relative 2^-24 each), and is linear
    in the per-tensor scales."""
    import torch
    g = torch.Generator().manual_seed(3)
    M, N, K = 4, 5, 128
    x = torch.randn(M, K, generator=g).to(torch.bfloat16)
    w = torch.randn(N, K, generator=g).to(torch.bfloat16)
    xp, xb, xs, _, _ = oracle.quantize_fp4_block(x.reshape(-1), float(x.abs().max()), requant=False)
    wp, wb, ws, _, _ = oracle.quantize_fp4_block(w.reshape(-1), float(w.abs().max()), requant=False)
    y, bound = oracle.gemm_fp4_block(xp, xb, xs, wp, wb, ws, K)
    xd = oracle.dequant_fp4_block(xp, xb, xs, M * K).astype(np.float64).reshape(M, K)
    wd = oracle.dequant_fp4_block(wp, wb, ws, N * K).astype(np.float64).reshape(N, K)
    assert np.all(np.abs(y - xd @ wd.T) <= 2.0 ** -22 * bound)
    y2, _ = oracle.gemm_fp4_block(xp, xb, xs * np.float32(4), wp, wb, ws * np.float32(0.5), K)
    assert np.array_equal(y2, 2.0 * y)
    y3, _ = oracle.gemm_fp4_block(xp, xb, xs, wp, wb, ws, K, rows=[3, 0])
    assert np.array_equal(y3, y[[3, 0]])


def test_unpack_reads_the_quantizers_layout_element_by_element():
    """unpack_e2m1 puts each code at the column the quantizer took it from: the unpacked values
    times their block scale and s_g equal dequant_fp4_block's element-wise values (which follow
    the packing order pinned with the codecs) to FP32 rounding.  A nibble swap moves values
    between neighbouring columns and fails.  (Inside the GEMM both operands share the layout,
    so the swap alone would not change Y: this pin is where the order is fixed.)"""
    import torch
    g = torch.Generator().manual_seed(8)
    R, K = 3, 64
    x = torch.randn(R, K, generator=g).to(torch.bfloat16)
    xp, xb, xs, _, _ = oracle.quantize_fp4_block(x.reshape(-1), float(x.abs().max()), requant=False)
    vals = (oracle.e2m1_table()[oracle.unpack_e2m1(xp, K)] *
            np.repeat(oracle.e4m3_table()[xb.reshape(R, K // 16)], 16, axis=1) * float(xs))
    want = oracle.dequant_fp4_block(xp, xb, xs, R * K).astype(np.float64).reshape(R, K)
    assert np.all(np.abs(vals - want) <= 2.0 ** -23 * np.abs(want))
    assert np.count_nonzero(vals[:, 0::2] != vals[:, 1::2]) > 0    # the test can see a swap
