"""The checked build (libqattn_checked.so, loaded under QATTN_DEBUG=1): device bounds checks
that record QATTN_ERR_BOUNDS and skip the access instead of trapping.

Run normally, this file re-runs the small-shape GPU parity tests in a child process with
QATTN_DEBUG=1 (the checked kernels must give the same bit-exact or within-bound results and
report no error), including the overrun-injection test below, which only the checked build can
run: its quantize loop goes one vector past the buffer and the checks must stop it.  The
buffers of that test are padded, so even a failed check could not touch memory outside them."""
import os
import subprocess
import sys

import numpy as np
import pytest
import torch

import oracle
import precision_quantized_attention_b200 as qa
from precision_quantized_attention_b200 import _lib

pytestmark = pytest.mark.gpu
ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.mark.skipif(not _lib.CHECKED, reason="runs in the checked build (QATTN_DEBUG=1)")
def test_injected_overrun_is_stopped_and_reported():
    assert qa._lib.build_info() & 1
    n = 8 * 1000 + 3                              # 1000 vectors and a 3-element tail
    g = torch.Generator().manual_seed(5)
    x = torch.randn(n + 64, generator=g).to(torch.bfloat16).cuda()
    codes = torch.full((n + 64,), 0x5A, dtype=torch.uint8, device="cuda")
    amax = torch.zeros(1, device="cuda")
    scale = torch.zeros(1, device="cuda")
    qa.calibrate_amax(x[:n], amax)
    qa._lib.debug_inject_oob(True)
    try:
        qa.quantize_fp8(x[:n], amax, codes[:n], scale)
    finally:
        qa._lib.debug_inject_oob(False)
    assert qa.get_error() == _lib.ERR_BOUNDS
    want, want_scale = oracle.quantize_fp8(x[:n].cpu(), float(amax.item()))
    assert np.array_equal(codes[:n].cpu().numpy(), want)
    assert bool((codes[n:] == 0x5A).all())       # the extra vector was not written
    assert np.float32(scale.item()) == want_scale
    # the context is intact: the same call without the injection reports nothing
    qa.quantize_fp8(x[:n], amax, codes[:n], scale)
    assert qa.get_error() == _lib.OK


@pytest.mark.skipif(_lib.CHECKED, reason="the normal build")
def test_normal_build_has_no_injection_switch():
    assert qa._lib.build_info() == 0
    with pytest.raises(qa.QattnError) as e:
        qa._lib.debug_inject_oob(True)
    assert e.value.status == _lib.ERR_UNSUPPORTED


@pytest.mark.skipif(_lib.CHECKED, reason="starts the checked-build run")
def test_small_parity_suites_pass_in_the_checked_build():
    from precision_quantized_attention_b200 import build
    build.build(checked=True)
    env = dict(os.environ, QATTN_DEBUG="1")
    cmd = [sys.executable, "-m", "pytest", "-q", "-x", "-m", "gpu", "-p", "no:cacheprovider",
           "tests/test_gpu_checked.py", "tests/test_gpu_quant.py", "tests/test_gpu_gemm.py",
           "tests/test_gpu_attention.py", "-k", "not full_size and not kontext and not workload"]
    r = subprocess.run(cmd, cwd=ROOT, env=env, capture_output=True, text=True, timeout=1500)
    tail = (r.stdout + r.stderr)[-4000:]
    assert r.returncode == 0, tail
    assert " passed" in r.stdout and "error" not in r.stdout.splitlines()[-1], tail
