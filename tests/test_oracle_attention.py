"""Pins for the oracle's quantized attention (CPU only).

The method (NVIDIA blog "Optimizing FLUX.1 Kontext for Image Editing with Low-Precision
Quantization", "Workflow and quantization", Fig. 4): FP8 BMM1 with higher-precision
accumulation, FP32 softmax, P requantized to per-tensor FP8, FP8 BMM2.  The pages print no
worked example, so the attention is pinned by
  - the unquantized closed form softmax(Q K^T * sm_scale) V in FP64 (oracle flags = 0),
  - a hand-computed case whose every intermediate is exactly representable,
  - invariants: uniform V, single key, one dominant key, key permutation, row sampling,
    varlen == separate dense calls.
"""
import numpy as np
import pytest
import torch

import oracle
import workloads


def _rand(shape, seed, scale=1.0):
    return np.random.default_rng(seed).standard_normal(shape) * scale


@pytest.mark.parametrize("B,H,T,D", [(1, 1, 1, 64), (1, 2, 7, 64), (2, 3, 16, 64), (1, 1, 13, 128)])
def test_exact_mode_matches_closed_form(B, H, T, D):
    q, k, v = (_rand((B, H, T, D), s) for s in (1, 2, 3))
    sm = 1.0 / np.sqrt(D)
    got = oracle.attention_values(q, k, v, sm_scale=sm, flags=0)
    want = oracle.attention_fp64(q, k, v, sm_scale=sm)
    assert np.max(np.abs(got - want)) <= 1e-12


def test_exact_mode_with_scales_matches_closed_form():
    q, k, v = (_rand((1, 2, 9, 64), s) for s in (4, 5, 6))
    sq, sk, sv, sm = 0.37, 2.5, 0.011, 0.125
    got = oracle.attention_values(q, k, v, sq, sk, sv, sm, flags=0)
    want = oracle.attention_fp64(q * sq, k * sk, v * sv, sm_scale=sm)
    assert np.max(np.abs(got - want)) <= 1e-12 * np.max(np.abs(want)) + 1e-15


def test_fp32_softmax_close_to_closed_form():
    q, k, v = (_rand((1, 2, 64, 64), s) for s in (7, 8, 9))
    got = oracle.attention_values(q, k, v, flags=oracle.FP32)
    want = oracle.attention_fp64(q, k, v)
    rel = np.linalg.norm(got - want) / np.linalg.norm(want)
    assert rel < 1e-6


def test_hand_computed_two_keys():
    """S' (base-2 score) = acc * sm_scale * log2(e); choose q, k so that S' is {M, M-1}
    exactly: then p = {1, 1/2}, l = 3/2, P8 = {448, 224} (exact E4M3 codes 0x7E and 0x76),
    O = (448 v0 + 224 v1) * s_v / 448 / 1.5."""
    D = 64
    log2e = 1.4426950408889634
    sm = 1.0 / log2e          # makes S' = acc exactly in the FP64 path
    q = np.zeros((1, 1, 2, D))
    k = np.zeros((1, 1, 2, D))
    v = np.zeros((1, 1, 2, D))
    q[0, 0, 0, 0] = 3.0       # row 0: acc = 3 * k_j0
    k[0, 0, 0, 0] = 1.0       # key 0: acc = 3 -> S' = 3 -> M = 3, p = 1
    k[0, 0, 1, 0] = 2.0 / 3.0  # key 1: acc = 2 -> S' = 2, p = 1/2
    v[0, 0, 0, :] = 0.5
    v[0, 0, 1, :] = -0.25
    q[0, 0, 1, 0] = 0.0       # row 1: both scores 0 -> p = {1, 1}, l = 2
    out = oracle.attention_values(q, k, v, 1.0, 1.0, 1.0, sm, flags=oracle.QUANT_P)
    want0 = (448 * 0.5 + 224 * (-0.25)) / 448 / 1.5      # = 0.25
    want1 = (448 * 0.5 + 448 * (-0.25)) / 448 / 2.0      # = 0.125
    assert np.allclose(out[0, 0, 0], want0, rtol=0, atol=1e-15)
    assert np.allclose(out[0, 0, 1], want1, rtol=0, atol=1e-15)
    assert oracle.e4m3_from_float(224.0) == 0x76


def test_uniform_v():
    B, H, T, D = 1, 2, 40, 64
    q, k = _rand((B, H, T, D), 10, 3.0), _rand((B, H, T, D), 11, 3.0)
    vrow = _rand((D,), 12)
    v = np.broadcast_to(vrow, (B, H, T, D)).copy()
    exact = oracle.attention_values(q, k, v, flags=0)
    assert np.max(np.abs(exact - vrow)) <= 1e-14
    fp32 = oracle.attention_values(q, k, v, flags=oracle.FP32)
    assert np.max(np.abs(fp32 / vrow - 1)) <= 1e-6
    quant = oracle.attention_values(q, k, v, flags=oracle.METHOD)
    # sum of quantized P differs from l by at most one E4M3 half-ulp (2^-4) per element
    assert np.max(np.abs(quant / vrow - 1)) <= 2.0 ** -4


def test_single_key():
    q, k, v = (_rand((1, 1, 1, 64), s) for s in (13, 14, 15))
    exact = oracle.attention_values(q, k, v, flags=0)[0, 0, 0]
    assert np.allclose(exact, v[0, 0, 0], rtol=1e-15, atol=0)
    quant = oracle.attention_values(q, k, v, flags=oracle.METHOD)[0, 0, 0]
    assert np.max(np.abs(quant / v[0, 0, 0] - 1)) <= 2.0 ** -4


def test_dominant_key():
    T, D = 50, 64
    q, k, v = (_rand((1, 1, T, D), s, 0.1) for s in (16, 17, 18))
    q[0, 0, 5] = 4.0
    k[0, 0, 33] = 4.0          # q5 . k33 = 16 * 64 -> all other weights vanish
    out = oracle.attention_values(q, k, v, flags=oracle.METHOD)
    assert np.max(np.abs(out[0, 0, 5] - v[0, 0, 33])) <= 2.0 ** -4 * np.max(np.abs(v[0, 0, 33]))


def test_key_permutation_invariance_is_exact():
    """The power-of-two row max makes the result independent of key order: permuting keys
    and values together changes nothing, bit for bit (both BMM sums are exact in FP64)."""
    B, H, T, D = 1, 2, 300, 64
    x = torch.randn(3, B, H, T, D, generator=torch.Generator().manual_seed(5)).to(torch.bfloat16)
    q8, sq, _ = oracle.quantize_tensor(x[0], "fp8")
    k8, sk, _ = oracle.quantize_tensor(x[1], "fp8")
    v8, sv, _ = oracle.quantize_tensor(x[2], "fp8")
    shape = (B, H, T, D)
    base = oracle.attention_e4m3(q8, k8, v8, shape, sq, sk, sv)
    perm = np.random.default_rng(1).permutation(T)
    k8p = k8.reshape(shape)[:, :, perm].copy()
    v8p = v8.reshape(shape)[:, :, perm].copy()
    permuted = oracle.attention_e4m3(q8, k8p, v8p, shape, sq, sk, sv)
    assert np.array_equal(base, permuted)


def test_row_sampling_matches_full():
    w = workloads.custom("t", "fp8", 2, 3, 77, 64, seed=21)
    q, k, v = workloads.make_qkv(w)
    full = oracle.method_forward(q, k, v, "fp8")
    rows = workloads.sample_rows(w, per_head=9).numpy()
    part = oracle.method_forward(q, k, v, "fp8", rows=rows)
    assert np.array_equal(part, full.reshape(-1, w.D)[rows])


def test_varlen_equals_separate_dense_calls():
    lens = [5, 17, 1, 40]
    w = workloads.custom("v", "fp8", None, 2, None, 64, seed=22, varlen_lens=lens)
    q, k, v = workloads.make_qkv(w)
    q8, sq, _ = oracle.quantize_tensor(q, "fp8")
    k8, sk, _ = oracle.quantize_tensor(k, "fp8")
    v8, sv, _ = oracle.quantize_tensor(v, "fp8")
    shape = w.shape
    packed = oracle.attention_e4m3(q8, k8, v8, shape, sq, sk, sv, cu_seqlens=w.cu_seqlens)
    cu = w.cu_seqlens
    for s in range(len(lens)):
        a, b = cu[s], cu[s + 1]
        sub = lambda c: c.reshape(shape)[:, :, a:b].copy()
        dense = oracle.attention_e4m3(sub(q8), sub(k8), sub(v8), (1, 2, b - a, 64), sq, sk, sv)
        assert np.array_equal(packed[:, :, a:b], dense)


def test_quantized_error_against_unquantized_is_small():
    """FP8 FakeQuantize of Q, K, V and P keeps the output close to FP64 attention (a few
    percent relative L2 for N(0,1) inputs: E4M3 carries 3 mantissa bits)."""
    w = workloads.custom("e", "fp8", 1, 2, 256, 64, seed=23)
    q, k, v = workloads.make_qkv(w)
    got = oracle.method_forward(q, k, v, "fp8")
    want = oracle.attention_fp64(q.double().numpy(), k.double().numpy(), v.double().numpy())
    rel = np.linalg.norm(got - want) / np.linalg.norm(want)
    assert 1e-3 < rel < 0.08
    got4 = oracle.method_forward(q, k, v, "fp4")
    rel4 = np.linalg.norm(got4 - want) / np.linalg.norm(want)
    assert rel < rel4 < 0.4           # FP4 inputs lose more than FP8 inputs


def test_fig4_literal_variant_is_close():
    w = workloads.custom("f", "fp8", 1, 2, 128, 64, seed=24)
    q, k, v = workloads.make_qkv(w)
    a = oracle.method_forward(q, k, v, "fp8")
    b = oracle.method_forward(q, k, v, "fp8", flags=oracle.FP32 | oracle.FIG4_LITERAL)
    rel = np.linalg.norm(a - b) / np.linalg.norm(a)
    assert 0 < rel < 0.1


def test_invalid_arguments():
    q = np.zeros((1, 1, 4, 64))
    with pytest.raises(ValueError):
        oracle.attention_values(q, q, q, cu_seqlens=[0, 3])          # does not end at T
    with pytest.raises(ValueError):
        oracle.attention_values(q, q, q, cu_seqlens=[0, 2, 2, 4])    # empty sequence


def _method_fp32_accumulation(q8, k8, v8, shape, sq, sk, sv, sm, order):
    """The method with BMM1 accumulated in binary32 in a given order of the D terms (what a
    tensor core with an FP32 accumulator may do), the rest as the oracle: used to check that
    the oracle's ambiguity bound covers accumulation-order effects."""
    import ml_dtypes
    B, H, T, D = shape
    val = lambda c: c.reshape(shape).view(ml_dtypes.float8_e4m3fn).astype(np.float32)
    q, k, v = val(q8), val(k8), val(v8)
    c32 = np.float32(float(sq) * float(sk) * sm * 1.4426950408889634)
    out = np.empty(shape)
    for b in range(B):
        for h in range(H):
            acc = np.zeros((T, T), dtype=np.float32)
            for d in order:
                acc = (acc + np.outer(q[b, h, :, d], k[b, h, :, d]).astype(np.float32)).astype(np.float32)
            s = (acc * c32).astype(np.float32)
            m = np.ceil(s.max(axis=1, keepdims=True).astype(np.float64))
            p = np.exp2((s - m).astype(np.float32).astype(np.float64)).astype(np.float32)
            l = p.astype(np.float64).sum(axis=1, keepdims=True).astype(np.float32)
            p8 = (p * np.float32(448)).astype(np.float32)
            p8 = np.clip(p8, 0, 448).astype(ml_dtypes.float8_e4m3fn).astype(np.float64)
            out[b, h] = (p8 @ v[b, h].astype(np.float64)) * float(sv) / 448.0 / l.astype(np.float64)
    return out


def test_ambiguity_bound_covers_fp32_accumulation_orders():
    """Outputs of the method with BMM1 accumulated in FP32 in several term orders stay within
    the oracle's ambiguity bound (plus bf16-free float noise); the outlier structure makes rows
    peaked, which is where ambiguous P codes matter."""
    w = workloads.custom("amb", "fp8", 1, 2, 96, 64, seed=31, outliers=4)
    q, k, v = workloads.make_qkv(w)
    q8, sq, _ = oracle.quantize_tensor(q, "fp8")
    k8, sk, _ = oracle.quantize_tensor(k, "fp8")
    v8, sv, _ = oracle.quantize_tensor(v, "fp8")
    want, amb = oracle.attention_e4m3(q8, k8, v8, w.shape, sq, sk, sv, w.sm_scale,
                                      with_ambiguity=True)
    assert amb.shape == want.shape and np.all(amb >= 0)
    rng = np.random.default_rng(0)
    worst, flips = 0.0, 0
    for order in (range(64), range(63, -1, -1), rng.permutation(64), rng.permutation(64)):
        got = _method_fp32_accumulation(q8, k8, v8, w.shape, sq, sk, sv, w.sm_scale, list(order))
        # beyond the bound only FP32 noise of the unquantized row sum is left (~1e-5 relative
        # for scores of magnitude ~60 in base-2 units)
        excess = np.abs(got - want) - amb - 1e-4 * np.abs(want)
        worst = max(worst, float(excess.max()))
        flips += int(np.sum(np.abs(got - want) > 1e-3))
    assert worst <= 1e-6
    assert np.max(amb) > 0          # the peaked rows do contain undecided P codes


def test_ambiguity_is_zero_without_p_quantization_and_small_otherwise():
    w = workloads.custom("amb2", "fp8", 1, 2, 128, 64, seed=32)
    q, k, v = workloads.make_qkv(w)
    out, amb = oracle.method_forward(q, k, v, "fp8", with_ambiguity=True)
    assert np.mean(amb) < 1e-3 * np.mean(np.abs(out))
    q8, sq, _ = oracle.quantize_tensor(q, "fp8")
    _, amb0 = oracle.attention_e4m3(q8, q8, q8, w.shape, sq, sq, sq, flags=oracle.FP32,
                                    with_ambiguity=True)
    assert np.all(amb0 == 0)


def test_p_row_detail_rebuilds_the_row_and_its_ambiguity():
    """oracle.p_row_detail gives one row's P codes, x = S' - M, the radius delta and the code
    range [lo, hi]; from them the row's output (sum_j val(code_j) v_j * s_v / 448 / l) and its
    ambiguity bound (sum_j max|val(lo or hi) - val(code)| |v_j| * s_v / 448 / l) are rebuilt
    and must equal attention_e4m3's, on peaked rows (outlier channels) and plain ones."""
    tbl = oracle.e4m3_table().astype(np.float64)
    for outliers, seed in ((4, 33), (0, 34)):
        w = workloads.custom("detail", "fp8", 1, 2, 300, 64, seed=seed, outliers=outliers)
        q, k, v = workloads.make_qkv(w)
        q8, sq, _ = oracle.quantize_tensor(q, "fp8")
        k8, sk, _ = oracle.quantize_tensor(k, "fp8")
        v8, sv, _ = oracle.quantize_tensor(v, "fp8")
        B, H, T, D = w.shape
        rows = [0, 17, 299, T + 5, 2 * T - 1]
        want, amb = oracle.attention_e4m3(q8, k8, v8, w.shape, sq, sk, sv, w.sm_scale, rows=rows,
                                          with_ambiguity=True)
        V = tbl[v8.reshape(B * H, T, D)]
        for i, row in enumerate(rows):
            code, x, delta, lo, hi, M, l = oracle.p_row_detail(q8, k8, w.shape, sq, sk, row, w.sm_scale)
            assert code.shape == (T,) and M == np.ceil(M) and np.all(x <= 0) and np.all(delta > 0)
            # the code is e4m3 of fl32(2^fl32(x)) * 448, within its own range
            p = np.exp2(x.astype(np.float32)).astype(np.float32)
            assert np.array_equal(code, np.array([oracle.e4m3_from_float(float(np.float32(pi * 448.0)))
                                                  for pi in p], dtype=np.uint8))
            assert np.all(tbl[lo] <= tbl[code]) and np.all(tbl[code] <= tbl[hi])
            post = np.float64(sv) / 448.0 / l
            vv = V[row // T]
            np.testing.assert_allclose((tbl[code] @ vv) * post, want[i], rtol=1e-12, atol=1e-15)
            a = np.maximum(np.abs(tbl[lo] - tbl[code]), np.abs(tbl[hi] - tbl[code]))
            np.testing.assert_allclose((a @ np.abs(vv)) * post, amb[i], rtol=1e-12, atol=1e-15)
