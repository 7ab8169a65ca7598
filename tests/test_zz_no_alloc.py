"""qattn_calibrate_quantize_fp8_noalloc through the C ABI: the same amax, scale and codes as
qattn_calibrate_quantize_fp8 with a caller workspace, on two calls in a row.  The file is
collected last (its name), so the static workspace is checked after every other test used the
library; one test repeats the check in a fresh Python process, where the first call on the
device looks the static array up."""
import os
import subprocess
import sys

import numpy as np
import pytest
import torch

import oracle
import precision_quantized_attention_b200 as qa

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CASES = [(11, 24 * 4096 * 128, 2.0), (12, 8 * 1000 + 7, 1e-3), (13, 37, 30.0)]


def _tensor(seed, n, scale):
    g = torch.Generator().manual_seed(seed)
    return (torch.randn(n, generator=g) * scale).to(torch.bfloat16)


def check_noalloc_against_workspace_entry(seed, n, scale):
    x = _tensor(seed, n, scale)
    xd = x.cuda()
    ws = qa.new_workspace()
    a_ref, s_ref = torch.zeros(1, device="cuda"), torch.zeros(1, device="cuda")
    c_ref = torch.empty(n, dtype=torch.uint8, device="cuda")
    qa.calibrate_quantize_fp8(xd, a_ref, c_ref, s_ref, ws)
    assert qa.get_error() == 0
    for _ in range(2):
        a, s = torch.full((1,), -1.0, device="cuda"), torch.zeros(1, device="cuda")
        c = torch.full((n,), 0x55, dtype=torch.uint8, device="cuda")
        qa._lib.calibrate_quantize_fp8_noalloc(xd, a, c, s)
        assert qa.get_error() == 0
        assert float(a.item()) == float(a_ref.item())
        assert float(s.item()) == float(s_ref.item())
        assert torch.equal(c, c_ref)
    # and both agree with the oracle (bit-exact codes)
    _, amax = oracle.amax(x)
    want, scale_want = oracle.quantize_fp8(x, amax)
    assert np.array_equal(c_ref.cpu().numpy(), want) and np.float32(s_ref.item()) == scale_want


@pytest.mark.parametrize("seed,n,scale", CASES)
def test_noalloc_matches_workspace_entry_twice(seed, n, scale):
    check_noalloc_against_workspace_entry(seed, n, scale)


def test_noalloc_first_use_in_a_fresh_process():
    """The no-allocation call made first, in a process that has not used the library yet."""
    code = ("import sys; sys.path.insert(0, %r); sys.path.insert(0, %r)\n"
            "import test_zz_no_alloc as t\n"
            "for case in t.CASES: t.check_noalloc_against_workspace_entry(*case)\n"
            "print('fresh process ok')\n") % (ROOT, os.path.join(ROOT, "tests"))
    r = subprocess.run([sys.executable, "-c", code], cwd=ROOT, capture_output=True, text=True,
                       timeout=600)
    assert r.returncode == 0 and "fresh process ok" in r.stdout, r.stdout[-2000:] + r.stderr[-4000:]
