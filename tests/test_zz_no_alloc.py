"""qattn_calibrate_quantize_fp8_noalloc through the C ABI: the same amax, scale and codes as
qattn_calibrate_quantize_fp8 with a caller workspace, on two calls in a row.  Collected last
(file name), and also run alone in a fresh process, so that the static workspace is checked
both on first use and after every other test used the library."""
import numpy as np
import pytest
import torch

import oracle
import precision_quantized_attention_b200 as qa

pytestmark = pytest.mark.gpu


def _tensor(seed, n, scale):
    g = torch.Generator().manual_seed(seed)
    return (torch.randn(n, generator=g) * scale).to(torch.bfloat16)


@pytest.mark.parametrize("seed,n,scale", [(11, 24 * 4096 * 128, 2.0), (12, 8 * 1000 + 7, 1e-3),
                                          (13, 37, 30.0)])
def test_noalloc_matches_workspace_entry_twice(seed, n, scale):
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
