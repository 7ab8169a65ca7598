"""Quantized scaled-dot-product attention for NVIDIA B200 (sm_100a).

The method is the quantized SDPA of the FLUX.1 Kontext transformer in the NVIDIA developer blog
"Optimizing FLUX.1 Kontext for Image Editing with Low-Precision Quantization" ("Workflow and
quantization", Fig. 4): Q, K, V FakeQuantized to per-tensor FP8 or per-block FP4, FP8 BMM1 with
FP32 accumulation, FP32 softmax, P requantized to per-tensor FP8, FP8 BMM2.

All arithmetic runs in the CUDA kernels of ``libqattn.so`` behind the C ABI of
``include/qattn.h``; this package only marshals arguments (``_lib``) and keeps the device
buffers of one call together (``QuantizedAttention``).  Build the library with
``python -m precision_quantized_attention_b200.build``.
"""
from __future__ import annotations

import torch

from . import _lib
from ._lib import (MODE_FP4, MODE_FP8, QattnError, calibrate_amax, calibrate_quantize_fp4_block,
                   calibrate_quantize_fp8, calibrate_quantize_qkv, forward, forward_varlen,
                   forward_workspace_bytes, get_error, new_workspace, quantize_fp4_block,
                   quantize_fp8, quantize_qkv, gemm_fp4, gemm_fp8, gemm_fp8_e4m3)

__all__ = ["QuantizedAttention", "calibrate_amax", "quantize_fp8", "quantize_fp4_block",
           "calibrate_quantize_fp8", "calibrate_quantize_fp4_block", "calibrate_quantize_qkv",
           "quantize_qkv", "gemm_fp8", "gemm_fp8_e4m3", "gemm_fp4",
           "new_workspace", "forward", "forward_workspace_bytes",
           "forward_varlen", "get_error", "QattnError", "MODE_FP8", "MODE_FP4"]


class QuantizedAttention:
    """The whole hot path for one shape: calibrate+quantize of Q, K, V (one launch) -> fused
    attention.

    Holds the device buffers (codes, scales, FP4 side outputs, output, the calibration
    workspace) so repeated calls allocate nothing.  Calls on one object must not overlap on
    the device (they share the buffers and the workspace); stream order is enough.  ``mode`` is
    "fp8" or "fp4".  For varlen, pass ``cu_seqlens`` (list of ints) and q, k, v of shape
    [1, H, T, D].  With ``static_amax`` (three floats: the amax of Q, K and V from an earlier
    calibration) the calls skip calibration and quantize with those scales in one streaming
    pass; ``amax`` then holds them.
    """

    def __init__(self, shape, mode: str = "fp8", cu_seqlens=None, sm_scale: float | None = None,
                 device="cuda", static_amax=None):
        B, H, T, D = shape
        self.shape = tuple(shape)
        self.mode = mode
        self.sm_scale = float(sm_scale) if sm_scale is not None else D ** -0.5
        n = B * H * T * D
        dev = torch.device(device)
        u8 = dict(dtype=torch.uint8, device=dev)
        f32 = dict(dtype=torch.float32, device=dev)
        self.codes = [torch.empty(shape, **u8) for _ in range(3)]
        self.amax = torch.zeros(3, **f32)
        self.static = static_amax is not None
        if self.static:
            vals = [float(a) for a in static_amax]
            if len(vals) != 3:
                raise ValueError("static_amax needs three values (Q, K, V)")
            self.amax.copy_(torch.tensor(vals, dtype=torch.float32))
        self.scale = torch.zeros(3, **f32)          # per-tensor E4M3 dequant multipliers
        if mode == "fp4":
            if n % 16:
                raise ValueError("FP4 block quantization needs numel % 16 == 0")
            self.e2m1 = [torch.empty(n // 2, **u8) for _ in range(3)]
            self.bscale = [torch.empty(n // 16, **u8) for _ in range(3)]
            self.gscale = torch.zeros(3, **f32)
        elif mode != "fp8":
            raise ValueError(mode)
        self.out = torch.empty(shape, dtype=torch.bfloat16, device=dev)
        self.workspace = new_workspace(dev)
        self.varlen = cu_seqlens is not None
        # attention workspace: lets a dense launch cut its tail pairs so that every SM runs the
        # same number of key steps (none for varlen)
        nbytes = 0 if self.varlen else forward_workspace_bytes(B, H, T, D)
        self.attn_workspace = torch.empty(nbytes, dtype=torch.uint8, device=dev) if nbytes else None
        if self.varlen:
            if B != 1:
                raise ValueError("varlen tensors are [1, H, T, D]")
            self.cu = torch.tensor(list(cu_seqlens), dtype=torch.int32, device=dev)
            self.max_seqlen = max(b - a for a, b in zip(cu_seqlens[:-1], cu_seqlens[1:]))

    def quantize(self, q, k, v, stream=None):
        """Calibrate and FakeQuantize Q, K and V in one launch (with static scales: quantize
        only)."""
        if self.static:
            extra = (self.e2m1, self.bscale, self.gscale) if self.mode == "fp4" else ()
            quantize_qkv((q, k, v), self.amax, self.codes, self.scale,
                         MODE_FP4 if self.mode == "fp4" else MODE_FP8, *extra, stream=stream)
        elif self.mode == "fp8":
            calibrate_quantize_qkv((q, k, v), self.amax, self.codes, self.scale, self.workspace,
                                   MODE_FP8, stream=stream)
        else:
            calibrate_quantize_qkv((q, k, v), self.amax, self.codes, self.scale, self.workspace,
                                   MODE_FP4, self.e2m1, self.bscale, self.gscale, stream=stream)

    def attend(self, stream=None):
        mode = MODE_FP8 if self.mode == "fp8" else MODE_FP4
        s = [self.scale[i:i + 1] for i in range(3)]
        if self.varlen:
            forward_varlen(self.codes[0], self.codes[1], self.codes[2], self.out, self.cu,
                           self.max_seqlen, *s, self.sm_scale, mode, stream)
        else:
            forward(self.codes[0], self.codes[1], self.codes[2], self.out, *s, self.sm_scale,
                    mode, stream, workspace=self.attn_workspace)
        return self.out

    def __call__(self, q, k, v, stream=None):
        self.quantize(q, k, v, stream)
        return self.attend(stream)
