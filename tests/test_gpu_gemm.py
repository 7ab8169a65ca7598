"""GPU FP8 GEMM (the block's quantized linear layers) vs the oracle's FP64 definition.

Inputs are seeded E4M3 codes drawn on the host (every finite code, both signs) with
per-tensor multipliers; the bar follows from the arithmetic: the products are exact, their FP32
accumulation is off by at most K * 2^-24 of the sum of |terms|, and the bf16 output rounding by
2^-9 of the value (2^-8 allowed, covering the rounding of s_a * s_b)."""
import numpy as np
import pytest
import torch

import oracle
import precision_quantized_attention_b200 as qa

pytestmark = pytest.mark.gpu


def _codes(rng, shape):
    c = rng.integers(0, 256, size=shape, dtype=np.uint8)
    c[(c & 0x7F) == 0x7F] ^= 0x01               # no NaN codes (0x7F -> 0x7E)
    return c


def _run(M, N, K, seed, s_a=0.01, s_b=0.002):
    rng = np.random.default_rng(seed)
    a8, b8 = _codes(rng, (M, K)), _codes(rng, (N, K))
    sa = torch.tensor([s_a], dtype=torch.float32, device="cuda")
    sb = torch.tensor([s_b], dtype=torch.float32, device="cuda")
    y = torch.full((M, N), float("nan"), dtype=torch.bfloat16, device="cuda")
    qa.gemm_fp8(torch.from_numpy(a8).cuda(), torch.from_numpy(b8).cuda(), y, sa, sb)
    assert qa.get_error() == 0
    return a8, b8, np.float32(s_a), np.float32(s_b), y


def _check(got, want, bound, K):
    excess = np.abs(got.astype(np.float64) - want) - (2.0 ** -8 * np.abs(want) + K * 2.0 ** -24 * bound)
    assert np.isfinite(got).all()
    assert excess.max() <= 0.0, f"worst excess {excess.max():.3e}"


@pytest.mark.parametrize("M,N,K", [(1, 32, 128), (128, 1056, 512),            # one-SM kernel
                                   (129, 288, 256), (130, 288, 256), (300, 512, 384),
                                   (257, 96, 1024), (2560, 2080, 256)])        # SM pairs
def test_small_shapes_all_elements(M, N, K):
    """Ragged row tiles, a partial column tile (N not a multiple of 256) and several K blocks.
    M <= 128 runs on one SM per tile; larger M on pairs of SMs with 256-row tiles, where the
    second CTA of a pair may hold a single valid row (M = 129) or no valid column of B
    (N = 96), and where a pair runs more than one tile (2560 x 2080: 90 tiles of 256 x 256)."""
    a8, b8, sa, sb, y = _run(M, N, K, seed=M + N + K)
    want, bound = oracle.gemm_e4m3(a8, b8, sa, sb)
    _check(y.float().cpu().numpy(), want, bound, K)


@pytest.mark.parametrize("M,N,K", [(8704, 9216, 3072), (8704, 3072, 3072), (8704, 12288, 3072),
                                   (8704, 3072, 12288)])
def test_kontext_block_shapes_sampled_rows(M, N, K):
    """The joint sequence (512 text + 4096 target + 4096 context tokens) through the block's QKV
    projection (3072 -> 3 x 3072) and the MLP (3072 -> 12288 -> 3072): every column of 64
    seeded rows, first and last row included."""
    a8, b8, sa, sb, y = _run(M, N, K, seed=K)
    rows = np.unique(np.concatenate([[0, M - 1], np.random.default_rng(1).integers(0, M, 62)]))
    want, bound = oracle.gemm_e4m3(a8, b8, sa, sb, rows=rows)
    got = y[torch.as_tensor(rows, device="cuda")].float().cpu().numpy()
    _check(got, want, bound, K)


def test_repeatable_and_scales_applied():
    a8, b8, sa, sb, y = _run(384, 512, 512, seed=9)
    y2 = torch.empty_like(y)
    qa.gemm_fp8(torch.from_numpy(a8).cuda(), torch.from_numpy(b8).cuda(), y2,
                torch.tensor([sa * 2], device="cuda"), torch.tensor([sb], device="cuda"))
    assert qa.get_error() == 0
    assert torch.equal(y2.float(), (y.float() * 2))   # a power of two: exact in bf16


def _fused(M, N, K, seed, amax_factor=1.0, with_y=True):
    """gemm_fp8_e4m3 on seeded codes; amax = amax_factor * max |bf16 y| of the plain GEMM (a
    static calibration).  Returns (a8, b8, s_a, s_b, y of the plain GEMM, y of the fused call or
    None, codes, scale, amax)."""
    a8, b8, sa, sb, y = _run(M, N, K, seed)
    amax = float(y.float().abs().max().item()) * amax_factor
    codes = torch.full((M, N), 0x55, dtype=torch.uint8, device="cuda")
    scale = torch.zeros(1, device="cuda")
    y2 = torch.full((M, N), float("nan"), dtype=torch.bfloat16, device="cuda") if with_y else None
    qa.gemm_fp8_e4m3(torch.from_numpy(a8).cuda(), torch.from_numpy(b8).cuda(), codes,
                     torch.tensor([sa], device="cuda"), torch.tensor([sb], device="cuda"),
                     torch.tensor([amax], dtype=torch.float32, device="cuda"), scale, y=y2)
    assert qa.get_error() == 0
    return a8, b8, sa, sb, y, y2, codes, scale, np.float32(amax)


@pytest.mark.parametrize("M,N,K,amax_factor", [(100, 288, 256, 1.0),       # one-SM kernel
                                               (130, 288, 256, 1.0), (300, 512, 384, 0.5),
                                               (2560, 2080, 256, 2.0)])    # SM pairs
def test_fused_e4m3_codes_are_the_quantized_bf16_output(M, N, K, amax_factor):
    """The codes of gemm_fp8_e4m3 are exactly oracle.quantize_fp8 of the GEMM's own bf16 output
    under the given amax (also when the amax is below the output's maximum: saturation), the
    written scale is the oracle's, the bf16 output of the fused call equals the plain GEMM's,
    and that bf16 output meets the oracle's GEMM bound."""
    a8, b8, sa, sb, y, y2, codes, scale, amax = _fused(M, N, K, seed=M * 7 + N, amax_factor=amax_factor)
    assert torch.equal(y2, y)
    want_codes, want_scale = oracle.quantize_fp8(y.cpu().reshape(-1), float(amax))
    assert np.array_equal(codes.cpu().numpy().reshape(-1), want_codes)
    assert np.float32(scale.item()) == want_scale
    want, bound = oracle.gemm_e4m3(a8, b8, sa, sb)
    _check(y.float().cpu().numpy(), want, bound, K)
    # codes only (no bf16 output): the same codes
    _, _, _, _, _, _, codes2, _, _ = _fused(M, N, K, seed=M * 7 + N, amax_factor=amax_factor, with_y=False)
    assert torch.equal(codes2, codes)


def test_fused_e4m3_value_projection_against_the_oracle_bf16_path():
    """The value projection of the joint sequence (8704 tokens, 3072 -> 3072): the fused codes
    equal the quantized GPU bf16 output everywhere, and differ from the quantized oracle bf16
    output only where the FP32 accumulation order tipped a bf16 rounding (a few in a million)."""
    M, N, K = 8704, 3072, 3072
    a8, b8, sa, sb, y, _, codes, scale, amax = _fused(M, N, K, seed=21, with_y=False)
    want_codes, _ = oracle.quantize_fp8(y.cpu().reshape(-1), float(amax))
    assert np.array_equal(codes.cpu().numpy().reshape(-1), want_codes)
    rows = np.unique(np.concatenate([[0, M - 1], np.random.default_rng(2).integers(0, M, 62)]))
    want, _ = oracle.gemm_e4m3(a8, b8, sa, sb, rows=rows)
    want_bf16 = torch.from_numpy(want.astype(np.float32)).to(torch.bfloat16)
    orc_codes, _ = oracle.quantize_fp8(want_bf16.reshape(-1), float(amax))
    got = codes.cpu().numpy()[rows].reshape(-1)
    assert np.mean(got != orc_codes) < 1e-4


def test_fused_e4m3_nonfinite_amax_writes_no_code():
    a8, b8, sa, sb, y = _run(130, 288, 256, seed=5)
    codes = torch.full((130, 288), 0x55, dtype=torch.uint8, device="cuda")
    qa.gemm_fp8_e4m3(torch.from_numpy(a8).cuda(), torch.from_numpy(b8).cuda(), codes,
                     torch.tensor([sa], device="cuda"), torch.tensor([sb], device="cuda"),
                     torch.tensor([float("inf")], device="cuda"), torch.zeros(1, device="cuda"))
    assert qa.get_error() == qa._lib.ERR_NONFINITE
    assert bool((codes == 0x55).all())


# --- per-block FP4 GEMM (kind::mxf4nvf4) vs oracle.gemm_fp4_block ---------------------------
def _fp4_operands(rng, rows, K):
    """Random packed E2M1 codes (all 16 codes) and E4M3 block scales (every finite non-negative
    code 0x00..0x7E, subnormals included)."""
    return (rng.integers(0, 256, size=(rows, K // 2), dtype=np.uint8),
            rng.integers(0, 0x7F, size=(rows, K // 16), dtype=np.uint8))


def _run_fp4(M, N, K, seed, sg_x=0.01, sg_w=0.002):
    rng = np.random.default_rng(seed)
    (xp, xb), (wp, wb) = _fp4_operands(rng, M, K), _fp4_operands(rng, N, K)
    y = torch.full((M, N), float("nan"), dtype=torch.bfloat16, device="cuda")
    dev = lambda a: torch.from_numpy(a).cuda()
    qa.gemm_fp4(dev(xp), dev(xb), torch.tensor([sg_x], device="cuda"), dev(wp), dev(wb),
                torch.tensor([sg_w], device="cuda"), y)
    assert qa.get_error() == 0
    return (xp, xb, np.float32(sg_x), wp, wb, np.float32(sg_w)), y


@pytest.mark.parametrize("M,N,K", [(1, 32, 256), (128, 128, 256), (130, 288, 512), (300, 512, 768),
                                   (257, 96, 1024), (2560, 2080, 256)])
def test_fp4_small_shapes_all_elements(M, N, K):
    """Ragged row and column tiles (N not a multiple of 128), one and several 256-element K
    blocks, several tiles per SM (2560 x 2080: 340 tiles of 128 x 128); the bar of the FP8 GEMM:
    FP32 accumulation (K * 2^-24 of the sum of |terms|) plus the bf16 rounding (2^-8)."""
    ops, y = _run_fp4(M, N, K, seed=M + 3 * N + K)
    want, bound = oracle.gemm_fp4_block(*ops, K)
    _check(y.float().cpu().numpy(), want, bound, K)


@pytest.mark.parametrize("M,N,K", [(8704, 9216, 3072), (8704, 3072, 3072), (8704, 12288, 3072),
                                   (8704, 3072, 12288)])
def test_fp4_kontext_block_shapes_sampled_rows(M, N, K):
    ops, y = _run_fp4(M, N, K, seed=K + 1)
    rows = np.unique(np.concatenate([[0, M - 1], np.random.default_rng(3).integers(0, M, 62)]))
    want, bound = oracle.gemm_fp4_block(*ops, K, rows=rows)
    _check(y[torch.as_tensor(rows, device="cuda")].float().cpu().numpy(), want, bound, K)


def test_fp4_gemm_of_operands_quantized_on_the_gpu():
    """bf16 X and W through qattn_quantize_fp4_block (bit-exact with the oracle's quantizer),
    then the FP4 GEMM: within the accumulation bar of the oracle on those codes, and near the
    bf16 product (the FP4 quantization error of Gaussian data, about 10 % per element)."""
    g = torch.Generator().manual_seed(2)
    M, N, K = 300, 256, 512
    x = torch.randn(M, K, generator=g).to(torch.bfloat16).cuda()
    w = torch.randn(N, K, generator=g).to(torch.bfloat16).cuda()
    ops = []
    for t in (x, w):
        rows = t.shape[0]
        amax = torch.zeros(1, device="cuda")
        qa.calibrate_amax(t.reshape(-1), amax)
        e2m1 = torch.empty(rows * K // 2, dtype=torch.uint8, device="cuda")
        bs = torch.empty(rows * K // 16, dtype=torch.uint8, device="cuda")
        sg = torch.zeros(1, device="cuda")
        qa.quantize_fp4_block(t.reshape(-1), amax, e2m1, bs, sg)
        ops.append((e2m1.reshape(rows, K // 2), bs.reshape(rows, K // 16), sg))
    y = torch.empty(M, N, dtype=torch.bfloat16, device="cuda")
    qa.gemm_fp4(*ops[0], *ops[1], y)
    assert qa.get_error() == 0
    host = [a.cpu().numpy() for o in ops for a in o]
    want, bound = oracle.gemm_fp4_block(host[0], host[1], host[2][0], host[3], host[4], host[5][0], K)
    got = y.float().cpu().numpy()
    _check(got, want, bound, K)
    ref = (x.float() @ w.float().T).cpu().numpy()
    rel = np.linalg.norm(got - ref) / np.linalg.norm(ref)
    print(f"FP4 GEMM vs the bf16 product: rel-L2 {rel:.3f}")
    assert rel < 0.25
