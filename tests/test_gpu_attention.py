"""GPU quantized attention vs the oracle (element by element, same seeded inputs).

Small shapes are compared on every output; the full-size workloads (the ones the bench times,
in the same launch configuration) on a seeded sample of query rows that the oracle computes one
by one.  Bar: relative L2 error <= 1e-2 and max abs error <= 3e-2 on unit-variance V.
"""
import numpy as np
import pytest
import torch

import oracle
import precision_quantized_attention_b200 as qa
import workloads
from parity import assert_close, compare, gpu_path, oracle_path

pytestmark = pytest.mark.gpu

SMALL = [
    # name, mode, B, H, L, D
    ("L1", "fp8", 1, 2, 1, 64),
    ("L7", "fp8", 2, 3, 7, 128),
    ("L128", "fp8", 1, 2, 128, 128),
    ("L129", "fp8", 1, 2, 129, 64),
    ("L256", "fp8", 1, 2, 256, 64),
    ("L300_B2", "fp8", 2, 3, 300, 128),
    ("L513", "fp4", 1, 2, 513, 128),
    ("L1000", "fp8", 1, 1, 1000, 64),
    ("L777_fp4", "fp4", 2, 1, 777, 64),
]


@pytest.mark.parametrize("name,mode,B,H,L,D", SMALL)
def test_small_shapes_all_rows(name, mode, B, H, L, D):
    w = workloads.custom(name, mode, B, H, L, D, seed=100 + L)
    q, k, v = workloads.make_qkv(w)
    path = gpu_path(w, q, k, v)
    got = path.out.float().cpu().numpy()
    want = oracle_path(w, q, k, v)
    rel, mx = assert_close(got, want, name)
    print(f"{name}: rel-L2 {rel:.2e} max-abs {mx:.2e}")


def test_small_workload_and_error_vs_unquantized():
    w = workloads.WORKLOADS["small_fp8"]
    q, k, v = workloads.make_qkv(w)
    path = gpu_path(w, q, k, v)
    got = path.out.float().cpu().numpy()
    want = oracle_path(w, q, k, v)
    rel, mx = assert_close(got, want, "small_fp8")
    ref = oracle.attention_fp64(q.double().numpy(), k.double().numpy(), v.double().numpy(),
                                sm_scale=w.sm_scale)
    rel_fp, _ = compare(got, ref)
    print(f"small_fp8: vs oracle rel-L2 {rel:.2e} max-abs {mx:.2e}; vs FP64 unquantized {rel_fp:.2e}")
    assert rel_fp < 0.1


@pytest.mark.parametrize("lens", [[1, 5, 200, 129], [300, 128, 7], [513]])
def test_varlen_small_all_rows(lens):
    w = workloads.custom("vl", "fp8", None, 3, None, 128, seed=7, varlen_lens=lens)
    q, k, v = workloads.make_qkv(w)
    path = gpu_path(w, q, k, v)
    got = path.out.float().cpu().numpy()
    want = oracle_path(w, q, k, v)
    assert_close(got, want, f"varlen {lens}")


@pytest.mark.parametrize("wname", ["gen_fp8", "edit_fp8", "edit_fp4", "varlen_fp4"])
def test_full_size_workloads_sampled_rows(wname):
    w = workloads.WORKLOADS[wname]
    q, k, v = workloads.make_qkv(w)
    path = gpu_path(w, q, k, v)
    rows = workloads.sample_rows(w, per_head=256 if not w.varlen else 64).numpy()
    got = path.out.float().reshape(-1, w.D)[torch.as_tensor(rows, device=path.out.device)].cpu().numpy()
    want, amb = oracle_path(w, q, k, v, rows=rows, with_ambiguity=True)
    rel, mx = assert_close(got, want, wname, amb=amb)
    per_row = np.linalg.norm(got - want, axis=1) / np.maximum(np.linalg.norm(want, axis=1), 1e-30)
    flagged = int(np.sum(np.abs(got - want).max(axis=1) > 3e-2))
    print(f"{wname}: {rows.size} rows, rel-L2 {rel:.2e} max-abs {mx:.2e}, worst row rel "
          f"{per_row.max():.2e}, rows past 3e-2 explained by ambiguous P codes: {flagged}")


def test_output_is_deterministic():
    w = workloads.custom("det", "fp8", 1, 4, 1024, 128, seed=3)
    q, k, v = workloads.make_qkv(w)
    a = gpu_path(w, q, k, v).out.clone()
    b = gpu_path(w, q, k, v).out.clone()
    assert torch.equal(a, b)


def test_wait_timeout_reports_error_and_context_survives():
    """A launch whose Q tile is never loaded: every wait runs into its (short) limit, the kernel
    records QATTN_ERR_TIMEOUT and exits; afterwards the context still works."""
    w = workloads.custom("to", "fp8", 1, 1, 128, 64, seed=5)
    q, k, v = workloads.make_qkv(w)
    path = qa.QuantizedAttention(w.shape, "fp8")
    path.quantize(q.cuda(), k.cuda(), v.cuda())
    assert qa.get_error() == 0
    qa._lib.debug_set_wait_timeout_ns(50_000_000)
    qa._lib.debug_inject_missing_q(True)
    try:
        path.attend()
        status = qa.get_error()
    finally:
        qa._lib.debug_inject_missing_q(False)
        qa._lib.debug_set_wait_timeout_ns(0)
    assert status == qa._lib.ERR_TIMEOUT
    out = gpu_path(w, q, k, v).out.float().cpu().numpy()
    assert_close(out, oracle_path(w, q, k, v), "after timeout")


# (1, 160, 1024, 64): four whole pairs per CTA (Q buffers reused), then a tail cut into
# ranges of 3 key steps
@pytest.mark.parametrize("B,H,L,D", [(1, 2, 1000, 128), (2, 3, 777, 64), (1, 160, 1024, 64),
                                     (1, 24, 8704, 128)])
def test_cut_tail_pairs_match_uncut_and_oracle(B, H, L, D):
    """With a workspace the persistent schedule cuts the tail pairs (those left after an equal
    share of whole pairs per CTA) along the keys and the combine kernel merges the parts; the
    result equals the launch without a workspace (tail pairs whole) up to FP32 summation order
    and meets the oracle bar."""
    w = workloads.custom("split", "fp8", B, H, L, D, seed=40 + L)
    q, k, v = workloads.make_qkv(w)
    path = gpu_path(w, q, k, v)
    nbytes = qa.forward_workspace_bytes(B, H, L, D)
    assert nbytes > 0 and path.attn_workspace is not None        # these shapes do split
    split = path.out.clone()
    path.attend()                                                # same again: reusable workspace
    assert torch.equal(path.out, split)
    s = [path.scale[i:i + 1] for i in range(3)]
    plain = torch.empty_like(path.out)
    qa.forward(path.codes[0], path.codes[1], path.codes[2], plain, *s, w.sm_scale)
    assert qa.get_error() == 0
    # the two differ only by FP32 summation order: at most one bf16 rounding step apart
    excess = ((split.float() - plain.float()).abs() - plain.float().abs() * 2.0 ** -7 - 1e-3)
    assert excess.max().item() <= 0.0
    rows = workloads.sample_rows(w, per_head=64).numpy() if L > 2000 else None
    want = oracle_path(w, q, k, v, rows=rows)
    got = split.float().reshape(-1, D)
    got = (got[torch.as_tensor(rows, device=got.device)] if rows is not None else got).cpu().numpy()
    assert_close(got.reshape(want.shape), want, f"split B{B} H{H} L{L} D{D}")


@pytest.mark.parametrize("L,D", [(8704, 128), (1000, 64)])
def test_zero_queries_give_the_mean_of_v(L, D):
    """Degenerate case checked on every row at full size: Q = 0 makes every score 0, so every P
    code is e4m3(448) = 448 exactly and each output row is the mean of the dequantized V rows of
    its head (up to FP32 summation and the bf16 output rounding)."""
    w = workloads.custom("zeroq", "fp8", 1, 24 if L > 2000 else 3, L, D, seed=21)
    q, k, v = workloads.make_qkv(w)
    q = torch.zeros_like(q)
    path = gpu_path(w, q, k, v)
    codes, s_v, _ = oracle.quantize_tensor(v, "fp8")
    v_deq = torch.from_numpy(codes.reshape(v.shape)).view(torch.float8_e4m3fn).double() * s_v
    want = v_deq.mean(dim=2, keepdim=True).expand_as(v_deq)             # [B, H, L, D]
    got = path.out.double().cpu()
    err = (got - want).abs() - want.abs() * 2.0 ** -8 - 1e-6            # bf16 rounding allowance
    assert err.max().item() <= 0.0


def test_power_of_two_scaling_of_v_scales_the_output_exactly():
    """Full size: V * 2^3 has the same E4M3 codes and an 8x scale, so every bf16 output is
    exactly 8x the unscaled one (bit-exact check of the whole path on every row)."""
    w = workloads.WORKLOADS["edit_fp8"]
    q, k, v = workloads.make_qkv(w)
    a = gpu_path(w, q, k, v).out.clone()
    b = gpu_path(w, q, k, (v.float() * 8.0).to(torch.bfloat16)).out
    assert torch.equal(b, a * 8)


def test_key_permutation_changes_only_the_summation_order():
    """Permuting the keys (K and V rows together) leaves the method's result unchanged: with the
    power-of-two running max the per-key P codes do not depend on the key order, so the GPU
    outputs differ only by FP32 summation order (one bf16 step at most)."""
    w = workloads.custom("perm", "fp8", 1, 4, 2000, 128, seed=31, outliers=4)
    q, k, v = workloads.make_qkv(w)
    perm = torch.randperm(w.L, generator=torch.Generator().manual_seed(5))
    a = gpu_path(w, q, k, v).out.float()
    b = gpu_path(w, q, k[:, :, perm], v[:, :, perm]).out.float()
    excess = (a - b).abs() - a.abs() * 2.0 ** -7 - 1e-3
    assert excess.max().item() <= 0.0


def _dequantized(x, mode):
    """The BMM operand the method feeds to BMM2: val(code) * scale, per element (oracle)."""
    codes, s, _ = oracle.quantize_tensor(x, mode)
    return (oracle.e4m3_table()[codes] * np.float64(s)).reshape(tuple(x.shape))


def _p_code_bound(L):
    """Relative bound on sum_j val(c_j)/448 / l - 1: E4M3 rounds each normal p*448 within
    2^-4 of it (3 fraction bits); each subnormal code is off by at most 2^-10 absolute, against
    l*448 >= 224 (the row maximum of p is above 1/2); plus bf16 output rounding and FP32 sums."""
    return 2.0 ** -4 + L * 2.0 ** -10 / 224.0 + 2.0 ** -8


@pytest.mark.parametrize("mode,D", [("fp8", 128), ("fp8", 64), ("fp4", 128)])
def test_uniform_v_gives_v_within_the_p_code_bound(mode, D):
    # every key of a head carries the same V row, so O = v8 * (sum_j val(c_j) / 448) / l
    B, H, L = 1, 3, 700
    w = workloads.custom(f"uniform_v_{mode}_{D}", mode, B, H, L, D, seed=31)
    q, k, v = workloads.make_qkv(w)
    v = v[:, :, :1, :].expand(B, H, L, D).contiguous()
    path = gpu_path(w, q, k, v)
    got = path.out.float().cpu().numpy()
    assert_close(got, oracle_path(w, q, k, v), f"uniform V {mode} D={D}")
    v8 = _dequantized(v, mode)[:, :, :1, :]
    dev = np.abs(got - v8) / np.maximum(np.abs(v8), 1e-30)
    bound = _p_code_bound(L)
    assert float(dev[np.abs(np.broadcast_to(v8, got.shape)) > 0].max()) <= bound, dev.max()


def test_dominant_key_gives_its_v_row():
    # all queries point along (1, ..., 1); key j* = 3 * (1, ..., 1) scores ~48 binades above the
    # rest, whose p * 448 then round to the zero code: every output row is v8[j*] * val(c)/448/p
    B, H, L, D, jstar = 1, 2, 300, 128, 217
    w = workloads.custom("dominant_key", "fp8", B, H, L, D, seed=32)
    q, k, v = workloads.make_qkv(w)
    q = (1.0 + 0.1 * q.float()).to(torch.bfloat16)
    k = k.clone()
    k[:, :, jstar, :] = 3.0
    path = gpu_path(w, q, k, v)
    got = path.out.float().cpu().numpy()
    assert_close(got, oracle_path(w, q, k, v), "dominant key")
    v8 = _dequantized(v, "fp8")[:, :, jstar:jstar + 1, :]
    # per element: one code's rounding (<= 2^-4 relative) plus bf16 output rounding
    excess = np.abs(got - v8) - (2.0 ** -4 + 2.0 ** -8) * np.abs(v8)
    assert float(excess.max()) <= 1e-6, excess.max()


def test_large_and_staggered_rises_of_the_row_max():
    """Rows whose max jumps by 50-85 binades at the second key tile and then rises a few
    binades per tile, the jump differing from row to row: rows past 64 binades rescale O in
    tensor memory, the others carry the gap in BMM2's per-row scale factor, and neighbouring
    rows (same lane quarter) carry different factors."""
    B, H, L, D = 1, 2, 640, 128
    w = workloads.custom("rises", "fp8", B, H, L, D, seed=41)
    q, k, v = workloads.make_qkv(w)
    a = torch.tensor([1.0, 1.2, 0.8, 1.1, 0.9, 1.3, 0.7, 1.05])[torch.arange(L) % 8]
    q = (a[None, None, :, None] * (1.0 + 0.05 * q.float())).to(torch.bfloat16)
    b = torch.tensor([0.0, 4.0, 4.2, 4.5, 4.8])[torch.arange(L) // 128]   # per key tile
    k = (b[None, None, :, None] + 0.1 * k.float()).to(torch.bfloat16)
    path = gpu_path(w, q, k, v)
    got = path.out.float().cpu().numpy()
    rel, mx = assert_close(got, oracle_path(w, q, k, v), "staggered rises")
    print(f"staggered rises: rel-L2 {rel:.2e} max-abs {mx:.2e}")


def _p_unquantized(path, w):
    """The debug switch: the same codes and scales through the attention with P left FP32."""
    out = torch.empty_like(path.out)
    s = path.scale
    mode = (qa.MODE_FP8 if w.mode == "fp8" else qa.MODE_FP4) | qa._lib.FLAG_P_UNQUANTIZED
    if w.varlen:
        qa.forward_varlen(path.codes[0], path.codes[1], path.codes[2], out, path.cu,
                          path.max_seqlen, s[0:1], s[1:2], s[2:3], w.sm_scale, mode)
    else:
        qa.forward(path.codes[0], path.codes[1], path.codes[2], out, s[0:1], s[1:2], s[2:3],
                   w.sm_scale, mode)
    assert qa.get_error() == 0
    return out.float().cpu().numpy().reshape(-1, w.D)


@pytest.mark.parametrize("name,mode,B,H,L,D,lens", [
    ("dense300", "fp8", 2, 3, 300, 128, None), ("dense129_d64", "fp8", 1, 2, 129, 64, None),
    ("dense1000_fp4", "fp4", 1, 2, 1000, 128, None), ("varlen", "fp8", None, 3, None, 128, [1, 200, 129])])
def test_p_unquantized_switch_matches_the_oracle_without_p_quantization(name, mode, B, H, L, D, lens):
    """QATTN_FLAG_P_UNQUANTIZED runs the method with P left in FP32; it must equal the oracle's
    FP32-softmax attention without P quantization (flag FP32 only) on the same codes and scales,
    within the bf16 rounding of the output (2^-8 relative) plus FP32 accumulation noise; and the
    quantized-P output must differ from it by the (small) error of the P codes alone."""
    w = workloads.custom(name, mode, B, H, L, D, seed=41, varlen_lens=lens)
    q, k, v = workloads.make_qkv(w)
    path = gpu_path(w, q, k, v)
    got = _p_unquantized(path, w)
    sc = [float(x) for x in path.scale.cpu()]
    want = oracle.attention_e4m3(path.codes[0].cpu().numpy(), path.codes[1].cpu().numpy(),
                                 path.codes[2].cpu().numpy(), w.shape, *sc, sm_scale=w.sm_scale,
                                 flags=oracle.FP32, cu_seqlens=w.cu_seqlens).reshape(-1, w.D)
    bound = 2.0 ** -8 * np.abs(want) + 1e-5 * np.abs(want).max()
    excess = np.abs(got - want) - bound
    assert excess.max() <= 0.0, f"{name}: worst excess {excess.max():.3e}"
    quantized = path.out.float().cpu().numpy().reshape(-1, w.D)
    rel_p, _ = compare(quantized, want)
    print(f"{name}: error of the P codes alone (rel-L2) {rel_p:.2e}")
    assert 0.0 < rel_p < 3e-2


# --- the pair-of-SMs variant of the D = 128 kernel (qattn_debug_use_pair_kernel) -------------
@pytest.fixture
def pair_kernel():
    qa._lib.debug_use_pair_kernel(True)
    try:
        yield
    finally:
        qa._lib.debug_use_pair_kernel(False)


@pytest.mark.parametrize("name,mode,B,H,L,D", [c for c in SMALL if c[5] == 128])
def test_pair_kernel_small_shapes_all_rows(pair_kernel, name, mode, B, H, L, D):
    test_small_shapes_all_rows(name, mode, B, H, L, D)


@pytest.mark.parametrize("lens", [[1, 5, 200, 129], [513]])
def test_pair_kernel_varlen_small_all_rows(pair_kernel, lens):
    test_varlen_small_all_rows(lens)


def test_pair_kernel_cut_tail_pairs_match_uncut_and_oracle(pair_kernel):
    test_cut_tail_pairs_match_uncut_and_oracle(1, 24, 8704, 128)


def test_pair_kernel_equals_the_one_sm_kernel_on_the_editing_workload():
    """Both D = 128 kernels compute the same method: on edit_fp8 their outputs differ only by
    FP32 summation order and the E4M3 subnormal-range codes of the pair kernel's per-tile
    maxima (reading 7)."""
    w = workloads.WORKLOADS["edit_fp8"]
    q, k, v = workloads.make_qkv(w)
    path = gpu_path(w, q, k, v)
    one = path.out.float().clone()
    qa._lib.debug_use_pair_kernel(True)
    try:
        path.attend()
        assert qa.get_error() == 0
    finally:
        qa._lib.debug_use_pair_kernel(False)
    two = path.out.float()
    rel = float((two - one).norm() / one.norm())
    print(f"pair vs one-SM kernel: rel-L2 {rel:.2e}, max-abs {float((two - one).abs().max()):.2e}")
    assert rel < 1e-3
