"""GPU calibration and quantize kernels vs the oracle: bit-exact codes, scales and amax."""
import numpy as np
import pytest
import torch

import oracle
import precision_quantized_attention_b200 as qa
import workloads

pytestmark = pytest.mark.gpu


def _u8(t):
    return t.cpu().numpy().reshape(-1)


def _inputs():
    g = torch.Generator().manual_seed(99)
    cases = {
        "tiny_tail": torch.randn(37, generator=g),
        "tail_7": torch.randn(8 * 1000 + 7, generator=g) * 3.0,
        "subnormal_heavy": torch.randn(16 * 4096, generator=g) * 1e-3,
        "wide_range": torch.randn(16 * 5000, generator=g) * torch.exp(torch.randn(16 * 5000, generator=g) * 3),
        "zeros": torch.zeros(16 * 64),
        "neg_zero": -torch.zeros(16 * 64),
    }
    x = torch.randn(16 * 1024, generator=g)
    x[:16] *= 1e-6          # a block whose E4M3 scale underflows
    x[100] = -0.0
    cases["mixed_blocks"] = x
    # scales outside [2^-100, 2^100] take the division path, inside the multiply-and-correct one
    cases["scale_tiny"] = torch.randn(16 * 2048, generator=g) * 1e-35
    cases["scale_huge"] = torch.randn(16 * 2048, generator=g) * 1e33
    cases["scale_large_fast"] = torch.randn(16 * 2048, generator=g) * 1e29
    cases["uniform_grid"] = (torch.arange(16 * 4096, dtype=torch.float32) - 32768.0) / 97.0
    return {k: v.to(torch.bfloat16) for k, v in cases.items()}


@pytest.mark.parametrize("name", list(_inputs().keys()))
def test_amax_and_fp8_bit_exact(name):
    x = _inputs()[name]
    xd = x.cuda()
    amax = torch.zeros(1, device="cuda")
    scale = torch.zeros(1, device="cuda")
    codes = torch.empty(x.numel(), dtype=torch.uint8, device="cuda")
    qa.calibrate_amax(xd, amax)
    qa.quantize_fp8(xd, amax, codes, scale)
    assert qa.get_error() == 0
    rc, a = oracle.amax(x)
    assert rc == 0 and float(amax.item()) == a
    want, s = oracle.quantize_fp8(x, a)
    assert np.float32(scale.item()) == s
    assert np.array_equal(_u8(codes), want)


@pytest.mark.parametrize("name", [k for k in _inputs() if k not in ("tiny_tail", "tail_7")])
def test_fp4_block_bit_exact(name):
    x = _inputs()[name]
    n = x.numel()
    xd = x.cuda()
    amax = torch.zeros(1, device="cuda")
    packed = torch.empty(n // 2, dtype=torch.uint8, device="cuda")
    bscale = torch.empty(n // 16, dtype=torch.uint8, device="cuda")
    gscale = torch.zeros(1, device="cuda")
    c8 = torch.empty(n, dtype=torch.uint8, device="cuda")
    s8 = torch.zeros(1, device="cuda")
    qa.calibrate_amax(xd, amax)
    qa.quantize_fp4_block(xd, amax, packed, bscale, gscale, c8, s8)
    assert qa.get_error() == 0
    _, a = oracle.amax(x)
    w_packed, w_bscale, w_sg, w_c8, w_s8 = oracle.quantize_fp4_block(x, a)
    assert np.float32(gscale.item()) == w_sg
    assert np.float32(s8.item()) == w_s8
    assert np.array_equal(_u8(bscale), w_bscale)
    assert np.array_equal(_u8(packed), w_packed)
    assert np.array_equal(_u8(c8), w_c8)


@pytest.mark.parametrize("wname", ["small_fp8", "gen_fp8", "edit_fp8", "edit_fp4"])
def test_workload_tensors_bit_exact(wname):
    """Full-size workload tensors (the shapes the bench times): every code and scale matches."""
    w = workloads.WORKLOADS[wname]
    q, k, v = workloads.make_qkv(w)
    path = qa.QuantizedAttention(w.shape, w.mode, sm_scale=w.sm_scale)
    path.quantize(q.cuda(), k.cuda(), v.cuda())
    assert qa.get_error() == 0
    for i, x in enumerate((q, k, v)):
        codes, s, extra = oracle.quantize_tensor(x, w.mode)
        assert float(path.amax[i].item()) == extra["amax"]
        assert np.float32(path.scale[i].item()) == s
        assert np.array_equal(_u8(path.codes[i]), codes)
        if w.mode == "fp4":
            assert np.array_equal(_u8(path.e2m1[i]), extra["packed"])
            assert np.array_equal(_u8(path.bscale[i]), extra["bscale"])
            assert np.float32(path.gscale[i].item()) == extra["sg"]


def test_nonfinite_input_is_reported():
    x = torch.randn(4096).to(torch.bfloat16)
    x[1234] = float("nan")
    xd = x.cuda()
    amax = torch.zeros(1, device="cuda")
    scale = torch.full((1,), -1.0, device="cuda")
    codes = torch.full((4096,), 0x55, dtype=torch.uint8, device="cuda")
    qa.calibrate_amax(xd, amax)
    qa.quantize_fp8(xd, amax, codes, scale)
    assert qa.get_error() == qa._lib.ERR_NONFINITE
    assert scale.item() == -1.0 and int(codes[0].item()) == 0x55     # nothing written
    assert qa.get_error() == 0                                        # the word was cleared


@pytest.mark.parametrize("name", list(_inputs().keys()))
def test_fused_calibrate_quantize_fp8_bit_exact(name):
    """One cooperative launch gives the amax, scale and codes of calibrate + quantize; twice in a
    row on one workspace, which each call leaves zero-filled."""
    x = _inputs()[name]
    xd = x.cuda()
    ws = qa.new_workspace()
    _, a = oracle.amax(x)
    want, s = oracle.quantize_fp8(x, a)
    for _ in range(2):
        amax = torch.full((1,), -1.0, device="cuda")
        scale = torch.zeros(1, device="cuda")
        codes = torch.full((x.numel(),), 0x55, dtype=torch.uint8, device="cuda")
        qa.calibrate_quantize_fp8(xd, amax, codes, scale, ws)
        assert qa.get_error() == 0
        assert float(amax.item()) == a
        assert np.float32(scale.item()) == s
        assert np.array_equal(_u8(codes), want)
        assert int(ws.count_nonzero().item()) == 0


@pytest.mark.parametrize("name", [k for k in _inputs() if k not in ("tiny_tail", "tail_7")])
def test_fused_calibrate_quantize_fp4_block_bit_exact(name):
    x = _inputs()[name]
    n = x.numel()
    xd = x.cuda()
    ws = qa.new_workspace()
    _, a = oracle.amax(x)
    w_packed, w_bscale, w_sg, w_c8, w_s8 = oracle.quantize_fp4_block(x, a)
    for requant in (True, False):
        amax = torch.zeros(1, device="cuda")
        packed = torch.empty(n // 2, dtype=torch.uint8, device="cuda")
        bscale = torch.empty(n // 16, dtype=torch.uint8, device="cuda")
        gscale = torch.zeros(1, device="cuda")
        c8 = torch.empty(n, dtype=torch.uint8, device="cuda") if requant else None
        s8 = torch.zeros(1, device="cuda") if requant else None
        qa.calibrate_quantize_fp4_block(xd, amax, packed, bscale, gscale, c8, s8, ws)
        assert qa.get_error() == 0
        assert float(amax.item()) == a
        assert np.float32(gscale.item()) == w_sg
        assert np.array_equal(_u8(bscale), w_bscale)
        assert np.array_equal(_u8(packed), w_packed)
        if requant:
            assert np.float32(s8.item()) == w_s8
            assert np.array_equal(_u8(c8), w_c8)
        assert int(ws.count_nonzero().item()) == 0


def test_fused_matches_separate_calls_on_a_large_tensor():
    """Many CTAs (grid at the co-residency cap), every code equal to the two-call path."""
    g = torch.Generator().manual_seed(5)
    x = (torch.randn(24 * 4096 * 128, generator=g) * 2.0).to(torch.bfloat16).cuda()
    x[7_000_001] = -300.0                          # the amax sits in one CTA's chunk
    ws = qa.new_workspace()
    a1, s1, c1 = torch.zeros(1, device="cuda"), torch.zeros(1, device="cuda"), torch.empty_like(x, dtype=torch.uint8)
    a2, s2, c2 = torch.zeros(1, device="cuda"), torch.zeros(1, device="cuda"), torch.empty_like(x, dtype=torch.uint8)
    qa.calibrate_amax(x, a1)
    qa.quantize_fp8(x, a1, c1, s1)
    qa.calibrate_quantize_fp8(x, a2, c2, s2, ws)
    assert qa.get_error() == 0
    assert float(a2.item()) == 300.0 == float(a1.item())
    assert float(s2.item()) == float(s1.item())
    assert torch.equal(c1, c2)


def test_fused_nonfinite_input_is_reported():
    x = torch.randn(4096 * 16).to(torch.bfloat16)
    x[40000] = float("inf")
    xd = x.cuda()
    ws = qa.new_workspace()
    amax = torch.zeros(1, device="cuda")
    scale = torch.full((1,), -1.0, device="cuda")
    codes = torch.full((x.numel(),), 0x55, dtype=torch.uint8, device="cuda")
    qa.calibrate_quantize_fp8(xd, amax, codes, scale, ws)
    assert qa.get_error() == qa._lib.ERR_NONFINITE
    assert float(amax.item()) == float("inf")
    assert scale.item() == -1.0 and int(codes[0].item()) == 0x55     # nothing written
    assert int(ws.count_nonzero().item()) == 0
    # the workspace is usable again right away
    x[40000] = 1.0
    qa.calibrate_quantize_fp8(x.cuda(), amax, codes, scale, ws)
    assert qa.get_error() == 0
    _, a = oracle.amax(x)
    want, s = oracle.quantize_fp8(x, a)
    assert np.array_equal(_u8(codes), want) and np.float32(scale.item()) == s


def _qkv_inputs(n, seed, scales=(1.0, 3.0, 1e-2)):
    g = torch.Generator().manual_seed(seed)
    return [(torch.randn(n, generator=g) * sc).to(torch.bfloat16) for sc in scales]


@pytest.mark.parametrize("n", [37, 8 * 1000 + 7, 16 * 4096, 24 * 4096 * 128 + 3])
def test_qkv_fp8_bit_exact(n):
    """Q, K, V in one staggered launch: every tensor's amax, scale and codes are the oracle's;
    twice in a row on one workspace."""
    xs = _qkv_inputs(n, seed=n % 1000)
    xd = [x.cuda() for x in xs]
    ws = qa.new_workspace()
    for _ in range(2):
        amax = torch.full((3,), -1.0, device="cuda")
        scale = torch.zeros(3, device="cuda")
        codes = [torch.full((n,), 0x55, dtype=torch.uint8, device="cuda") for _ in range(3)]
        qa.calibrate_quantize_qkv(xd, amax, codes, scale, ws)
        assert qa.get_error() == 0
        for i, x in enumerate(xs):
            _, a = oracle.amax(x)
            want, s = oracle.quantize_fp8(x, a)
            assert float(amax[i].item()) == a
            assert np.float32(scale[i].item()) == s
            assert np.array_equal(_u8(codes[i]), want), i
        assert int(ws.count_nonzero().item()) == 0


@pytest.mark.parametrize("n", [16 * 64, 16 * 4097, 24 * 4096 * 128])
def test_qkv_fp4_bit_exact(n):
    xs = _qkv_inputs(n, seed=7 + n % 1000, scales=(1.0, 1e-3, 40.0))
    xs[0][:16] = xs[0][:16] * 1e-6                  # a block whose E4M3 scale underflows
    xd = [x.cuda() for x in xs]
    ws = qa.new_workspace()
    amax, scale, gscale = (torch.zeros(3, device="cuda") for _ in range(3))
    codes = [torch.empty(n, dtype=torch.uint8, device="cuda") for _ in range(3)]
    e2m1 = [torch.empty(n // 2, dtype=torch.uint8, device="cuda") for _ in range(3)]
    bscale = [torch.empty(n // 16, dtype=torch.uint8, device="cuda") for _ in range(3)]
    qa.calibrate_quantize_qkv(xd, amax, codes, scale, ws, qa.MODE_FP4, e2m1, bscale, gscale)
    assert qa.get_error() == 0
    for i, x in enumerate(xs):
        _, a = oracle.amax(x)
        w_packed, w_bscale, w_sg, w_c8, w_s8 = oracle.quantize_fp4_block(x, a)
        assert float(amax[i].item()) == a
        assert np.float32(gscale[i].item()) == w_sg
        assert np.float32(scale[i].item()) == w_s8
        assert np.array_equal(_u8(bscale[i]), w_bscale)
        assert np.array_equal(_u8(e2m1[i]), w_packed)
        assert np.array_equal(_u8(codes[i]), w_c8)
    assert int(ws.count_nonzero().item()) == 0


def test_qkv_matches_single_tensor_kernel():
    n = 24 * 2048 * 128
    xs = [x.cuda() for x in _qkv_inputs(n, seed=3)]
    ws = qa.new_workspace()
    amax, scale = torch.zeros(3, device="cuda"), torch.zeros(3, device="cuda")
    codes = [torch.empty(n, dtype=torch.uint8, device="cuda") for _ in range(3)]
    qa.calibrate_quantize_qkv(xs, amax, codes, scale, ws)
    for i, x in enumerate(xs):
        a1, s1 = torch.zeros(1, device="cuda"), torch.zeros(1, device="cuda")
        c1 = torch.empty(n, dtype=torch.uint8, device="cuda")
        qa.calibrate_quantize_fp8(x, a1, c1, s1, ws)
        assert float(a1.item()) == float(amax[i].item())
        assert float(s1.item()) == float(scale[i].item())
        assert torch.equal(c1, codes[i])
    assert qa.get_error() == 0


def test_qkv_nonfinite_tensor_is_reported_and_the_others_are_quantized():
    n = 16 * 4096
    xs = _qkv_inputs(n, seed=11)
    xs[1][777] = float("nan")
    xd = [x.cuda() for x in xs]
    ws = qa.new_workspace()
    amax = torch.zeros(3, device="cuda")
    scale = torch.full((3,), -1.0, device="cuda")
    codes = [torch.full((n,), 0x55, dtype=torch.uint8, device="cuda") for _ in range(3)]
    qa.calibrate_quantize_qkv(xd, amax, codes, scale, ws)
    assert qa.get_error() == qa._lib.ERR_NONFINITE
    assert np.isnan(amax[1].item()) and scale[1].item() == -1.0
    assert int(codes[1][0].item()) == 0x55                        # K: nothing written
    for i in (0, 2):
        _, a = oracle.amax(xs[i])
        want, s = oracle.quantize_fp8(xs[i], a)
        assert np.array_equal(_u8(codes[i]), want) and np.float32(scale[i].item()) == s
    assert int(ws.count_nonzero().item()) == 0


# ---- given (static) scales: qattn_quantize_qkv ----------------------------------------------

def _given(xs, factors):
    """float32 amax values to quantize with: the data's amax times a factor."""
    return [float(np.float32(oracle.amax(x)[1] * f)) for x, f in zip(xs, factors)]


@pytest.mark.parametrize("n", [37, 8 * 1000 + 7, 24 * 4096 * 128 + 3])
def test_static_qkv_fp8_bit_exact(n):
    """Given scales below (codes saturate), at and above the data's amax: every tensor's scale
    and codes are the oracle's quantize for that amax, and the amax is left as given."""
    xs = _qkv_inputs(n, seed=20 + n % 1000)
    given = _given(xs, (0.5, 1.0, 2.0))
    amax = torch.tensor(given, dtype=torch.float32, device="cuda")
    scale = torch.zeros(3, device="cuda")
    codes = [torch.full((n,), 0x55, dtype=torch.uint8, device="cuda") for _ in range(3)]
    qa.quantize_qkv([x.cuda() for x in xs], amax, codes, scale)
    assert qa.get_error() == 0
    for i, x in enumerate(xs):
        want, s = oracle.quantize_fp8(x, given[i])
        assert float(amax[i].item()) == given[i]
        assert np.float32(scale[i].item()) == s
        assert np.array_equal(_u8(codes[i]), want), i


@pytest.mark.parametrize("n", [16 * 64, 24 * 4096 * 128])
def test_static_qkv_fp4_bit_exact(n):
    """FP4 blocks with given scales at and below the data's amax (there the requant scale's
    closed form fl32(2688 s_g) / 448 is what the oracle finds by brute force: the block holding
    the data's maximum saturates to scale 448 and code 6)."""
    xs = _qkv_inputs(n, seed=30 + n % 1000, scales=(1.0, 1e-3, 40.0))
    given = _given(xs, (1.0, 0.5, 0.25))
    amax = torch.tensor(given, dtype=torch.float32, device="cuda")
    scale, gscale = torch.zeros(3, device="cuda"), torch.zeros(3, device="cuda")
    codes = [torch.empty(n, dtype=torch.uint8, device="cuda") for _ in range(3)]
    e2m1 = [torch.empty(n // 2, dtype=torch.uint8, device="cuda") for _ in range(3)]
    bscale = [torch.empty(n // 16, dtype=torch.uint8, device="cuda") for _ in range(3)]
    qa.quantize_qkv([x.cuda() for x in xs], amax, codes, scale, qa.MODE_FP4, e2m1, bscale, gscale)
    assert qa.get_error() == 0
    for i, x in enumerate(xs):
        w_packed, w_bscale, w_sg, w_c8, w_s8 = oracle.quantize_fp4_block(x, given[i])
        assert np.float32(gscale[i].item()) == w_sg
        assert np.float32(scale[i].item()) == w_s8
        assert np.array_equal(_u8(bscale[i]), w_bscale)
        assert np.array_equal(_u8(e2m1[i]), w_packed)
        assert np.array_equal(_u8(codes[i]), w_c8)


@pytest.mark.parametrize("mode", ["fp8", "fp4"])
def test_static_path_with_the_calibrated_amax_equals_the_calibrated_path(mode):
    w = workloads.custom("static", mode, 1, 3, 700, 128, seed=21)
    q, k, v = (t.cuda() for t in workloads.make_qkv(w))
    dyn = qa.QuantizedAttention(w.shape, mode)
    dyn(q, k, v)
    assert qa.get_error() == 0
    stat = qa.QuantizedAttention(w.shape, mode, static_amax=dyn.amax.tolist())
    stat(q, k, v)
    assert qa.get_error() == 0
    assert torch.equal(stat.scale, dyn.scale)
    for i in range(3):
        assert torch.equal(stat.codes[i], dyn.codes[i])
    assert torch.equal(stat.out, dyn.out)


def test_static_nonfinite_amax_writes_nothing_for_that_tensor():
    n = 8 * 4096
    xs = _qkv_inputs(n, seed=12)
    given = _given(xs, (1.0, 1.0, 1.0))
    amax = torch.tensor([given[0], float("inf"), given[2]], dtype=torch.float32, device="cuda")
    scale = torch.full((3,), -1.0, device="cuda")
    codes = [torch.full((n,), 0x55, dtype=torch.uint8, device="cuda") for _ in range(3)]
    qa.quantize_qkv([x.cuda() for x in xs], amax, codes, scale)
    assert qa.get_error() == qa._lib.ERR_NONFINITE
    assert scale[1].item() == -1.0 and int(codes[1].count_nonzero().item()) == n
    assert int((codes[1] == 0x55).sum().item()) == n
    for i in (0, 2):
        want, s = oracle.quantize_fp8(xs[i], given[i])
        assert np.array_equal(_u8(codes[i]), want) and np.float32(scale[i].item()) == s
