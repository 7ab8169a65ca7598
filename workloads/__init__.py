"""Seeded synthetic inputs shaped like the FLUX.1 Kontext joint attention sequence.

This module only draws random numbers and arranges them; it holds none of the quantized
attention's arithmetic, so both the CPU oracle's tests and the CUDA path's tests and bench can
use it without sharing method code.

Token counts follow the Kontext layout (VAE latent at 1/8 resolution cut into 2x2 patches, so
one token per 16x16 pixels; 512 text tokens; text || target image || context image concatenated
along the sequence axis):
  1024x1024 image -> 4096 tokens, 1024x768 -> 3072, 512x512 -> 1024.
Inputs are post-RoPE Q, K, V in bf16, [B, H, L, D] (varlen: [1, H, T, D] with cu_seqlens).
"""
from __future__ import annotations

import dataclasses
import math

import torch

TEXT_TOKENS = 512


def image_tokens(width: int, height: int) -> int:
    """Tokens of one image: VAE downsamples by 8, then 2x2 patches -> one token per 16x16 px."""
    return (width // 16) * (height // 16)


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    mode: str                 # "fp8" or "fp4"
    B: int
    H: int
    D: int
    seqlens: tuple            # one entry per sequence; dense workloads have B equal entries
    varlen: bool = False
    text_scale: float = 1.0   # multiply rows [0, 512) of each sequence of Q, K, V
    outliers: int = 0         # per head, this many channels of Q and K scaled by outlier_scale
    outlier_scale: float = 10.0
    seed: int = 0             # seeds: Q = 1000*seed, K = +1, V = +2, outlier channels = +3

    @property
    def T(self) -> int:
        return sum(self.seqlens) if self.varlen else self.seqlens[0]

    @property
    def L(self) -> int:
        return max(self.seqlens)

    @property
    def sm_scale(self) -> float:
        return 1.0 / math.sqrt(self.D)

    @property
    def cu_seqlens(self):
        if not self.varlen:
            return None
        cu = [0]
        for s in self.seqlens:
            cu.append(cu[-1] + s)
        return cu

    @property
    def shape(self):
        return (1 if self.varlen else self.B, self.H, self.T, self.D)

    @property
    def flops(self) -> float:
        """Algorithmic FLOPs of BMM1 + BMM2: 4 * H * D * sum(L_i^2) (times B for dense)."""
        per = sum(s * s for s in self.seqlens) if self.varlen else self.B * self.seqlens[0] ** 2
        return 4.0 * self.H * self.D * per


KONTEXT_TARGET = image_tokens(1024, 1024)        # 4096
KONTEXT_CONTEXT = image_tokens(1024, 1024)       # 4096
L_GEN = TEXT_TOKENS + KONTEXT_TARGET                              # 4608
L_EDIT = TEXT_TOKENS + KONTEXT_TARGET + KONTEXT_CONTEXT           # 8704
L_MIXED_A = TEXT_TOKENS + image_tokens(1024, 768) + image_tokens(512, 512)   # 4608
L_MIXED_B = TEXT_TOKENS + image_tokens(1024, 1024) + image_tokens(512, 512)  # 5632

WORKLOADS = {
    "small_fp8": Workload("small_fp8", "fp8", 1, 2, 64, (256,), seed=1),
    "gen_fp8": Workload("gen_fp8", "fp8", 1, 24, 128, (L_GEN,), text_scale=2.0, seed=2),
    "edit_fp8": Workload("edit_fp8", "fp8", 1, 24, 128, (L_EDIT,), outliers=4, seed=3),
    "edit_fp4": Workload("edit_fp4", "fp4", 1, 24, 128, (L_EDIT,), outliers=4, seed=4),
    "varlen_fp4": Workload("varlen_fp4", "fp4", 4, 24, 128,
                           (L_EDIT, L_EDIT, L_MIXED_A, L_MIXED_B), varlen=True, seed=5),
}


def _randn(shape, seed):
    g = torch.Generator(device="cpu")
    g.manual_seed(seed)
    return torch.randn(shape, generator=g, dtype=torch.float32)


def make_qkv(w: Workload):
    """Returns CPU bf16 tensors q, k, v of w.shape, drawn iid N(0, 1) from fixed seeds and
    given the workload's structure (text-row scaling, shared Q/K outlier channels)."""
    shape = w.shape
    base = 1000 * w.seed
    q = _randn(shape, base + 0)
    k = _randn(shape, base + 1)
    v = _randn(shape, base + 2)
    if w.text_scale != 1.0:
        starts = [0] if not w.varlen else w.cu_seqlens[:-1]
        for s0 in starts:
            for t in (q, k, v):
                t[:, :, s0:s0 + TEXT_TOKENS] *= w.text_scale
    if w.outliers:
        g = torch.Generator(device="cpu")
        g.manual_seed(base + 3)
        for h in range(w.H):
            ch = torch.randperm(w.D, generator=g)[: w.outliers]
            q[:, h, :, ch] *= w.outlier_scale
            k[:, h, :, ch] *= w.outlier_scale
    return q.to(torch.bfloat16), k.to(torch.bfloat16), v.to(torch.bfloat16)


def custom(name, mode, B, H, L, D, seed, varlen_lens=None, **kw) -> Workload:
    """A parity-test workload of arbitrary (small) shape."""
    if varlen_lens is not None:
        return Workload(name, mode, len(varlen_lens), H, D, tuple(varlen_lens), varlen=True,
                        seed=seed, **kw)
    return Workload(name, mode, B, H, D, (L,), seed=seed, **kw)


def sample_rows(w: Workload, per_head: int, seed: int = 12345):
    """Row ids r = (b*H + h)*T + t of a seeded random sample: per (batch row, head), per
    sequence, `per_head` query rows spread over the sequence, always including its first and
    last row."""
    g = torch.Generator(device="cpu")
    g.manual_seed(seed)
    B = w.shape[0]
    T = w.T
    starts = [0] if not w.varlen else w.cu_seqlens[:-1]
    rows = []
    for b in range(B):
        for h in range(w.H):
            for si, s0 in enumerate(starts):
                n = w.seqlens[si] if w.varlen else w.seqlens[0]
                k = min(per_head, n)
                pick = torch.randperm(n, generator=g)[:k].tolist()
                pick = sorted(set(pick) | {0, n - 1})
                rows.extend(((b * w.H + h) * T + s0 + t) for t in pick)
    return torch.tensor(sorted(rows), dtype=torch.int64)
