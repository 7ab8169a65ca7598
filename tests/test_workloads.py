"""The seeded input recipe: Kontext joint-sequence sizes, determinism, and the structure the
workloads put on N(0, 1) draws (text rows scaled, Q/K outlier channels shared per head),
checked statistically on the CPU."""
import torch

import workloads


def test_kontext_sequence_sizes_and_flops():
    assert workloads.image_tokens(1024, 1024) == 4096
    assert workloads.image_tokens(1024, 768) == 3072
    assert workloads.image_tokens(512, 512) == 1024
    W = workloads.WORKLOADS
    assert W["edit_fp8"].L == 8704 and W["gen_fp8"].L == 4608
    vl = W["varlen_fp4"]
    assert vl.cu_seqlens == [0, 8704, 17408, 22016, 27648] and vl.T == 27648
    assert vl.shape == (1, 24, 27648, 128)
    # algorithmic FLOPs 4 H D sum(L^2): 9.309e11 at L=8704, 2.513e12 for the varlen batch
    assert abs(W["edit_fp8"].flops - 4 * 24 * 128 * 8704 ** 2) == 0
    assert round(W["edit_fp8"].flops / 1e11, 3) == 9.309
    assert round(vl.flops / 1e12, 3) == 2.513
    assert W["small_fp8"].sm_scale == 0.125


def test_inputs_are_deterministic_bf16():
    w = workloads.custom("det", "fp8", 2, 3, 100, 64, seed=7, outliers=2)
    a, b = workloads.make_qkv(w), workloads.make_qkv(w)
    for x, y in zip(a, b):
        assert x.dtype == torch.bfloat16 and tuple(x.shape) == (2, 3, 100, 64)
        assert torch.equal(x, y)
    other = workloads.make_qkv(workloads.custom("det", "fp8", 2, 3, 100, 64, seed=8, outliers=2))
    assert not torch.equal(a[0], other[0])


def test_outlier_channels_shared_by_q_and_k():
    w = workloads.custom("outl", "fp8", 1, 3, 4096, 128, seed=11, outliers=4)
    q, k, v = (t.float() for t in workloads.make_qkv(w))
    for h in range(w.H):
        rq = q[0, h].pow(2).mean(0).sqrt()          # RMS per channel
        rk = k[0, h].pow(2).mean(0).sqrt()
        rv = v[0, h].pow(2).mean(0).sqrt()
        big_q = set(torch.nonzero(rq > 5).flatten().tolist())
        big_k = set(torch.nonzero(rk > 5).flatten().tolist())
        assert len(big_q) == 4 and big_q == big_k
        assert ((rq[list(big_q)] - 10).abs() < 0.5).all()
        assert (rv < 1.2).all()                     # V keeps unit variance


def test_text_rows_scaled():
    w = workloads.custom("text", "fp8", 1, 2, 1536, 64, seed=12, text_scale=2.0)
    q, k, v = (t.float() for t in workloads.make_qkv(w))
    for x in (q, k, v):
        text = x[0, :, :512].pow(2).mean().sqrt()
        rest = x[0, :, 512:].pow(2).mean().sqrt()
        assert abs(text - 2.0) < 0.05 and abs(rest - 1.0) < 0.05
