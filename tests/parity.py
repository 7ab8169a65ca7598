"""Shared helpers of the parity tests: run the CUDA path and the oracle on the same inputs."""
from __future__ import annotations

import numpy as np
import torch

import oracle
import workloads

# Tolerances of the quantized attention against the oracle, on unit-variance V.
REL_L2_TOL = 1e-2
MAX_ABS_TOL = 3e-2


def gpu_path(w: workloads.Workload, q, k, v):
    """Runs amax -> quantize -> attention through the C ABI on cuda:0.  Returns the
    QuantizedAttention object (codes, scales, output stay on the device)."""
    import precision_quantized_attention_b200 as qa
    qa_ = qa.QuantizedAttention(w.shape, w.mode, cu_seqlens=w.cu_seqlens, sm_scale=w.sm_scale)
    qd, kd, vd = (t.cuda() for t in (q, k, v))
    qa_(qd, kd, vd)
    status = qa.get_error()
    assert status == 0, f"device error word {status}"
    torch.cuda.synchronize()
    return qa_


def oracle_path(w: workloads.Workload, q, k, v, rows=None, with_ambiguity=False):
    return oracle.method_forward(q, k, v, w.mode, sm_scale=w.sm_scale, cu_seqlens=w.cu_seqlens,
                                 rows=rows, with_ambiguity=with_ambiguity)


def compare(gpu_out: np.ndarray, want: np.ndarray):
    diff = gpu_out.astype(np.float64) - want
    rel = float(np.linalg.norm(diff) / max(np.linalg.norm(want), 1e-300))
    mx = float(np.max(np.abs(diff))) if diff.size else 0.0
    return rel, mx


def assert_close(gpu_out, want, what="", amb=None):
    """rel-L2 <= 1e-2 over everything; |diff| <= 3e-2 per output, beyond the oracle's
    ambiguity bound `amb` when given (outputs whose P codes the method leaves undecided at
    FP32 accumulation precision may move by that much, see oracle.attention_e4m3)."""
    rel, mx = compare(gpu_out, want)
    assert rel <= REL_L2_TOL, f"{what}: rel-L2 {rel:.3e}"
    if amb is None:
        assert mx <= MAX_ABS_TOL, f"{what}: max-abs {mx:.3e}"
    else:
        excess = np.abs(gpu_out.astype(np.float64) - want) - amb
        worst = float(excess.max()) if excess.size else 0.0
        assert worst <= MAX_ABS_TOL, f"{what}: max-abs beyond ambiguity {worst:.3e} (raw {mx:.3e})"
    return rel, mx
