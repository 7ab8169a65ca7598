"""Error study of the quantized SDPA: relative L2 error of the output against unquantized FP64
attention, for the pieces of the method the blog ("Optimizing FLUX.1 Kontext for Image Editing
with Low-Precision Quantization", "Workflow and quantization", Fig. 4) combines:

  gpu_fp8      the method with per-tensor FP8 inputs (libqattn on the GPU)
  gpu_fp4      the method with per-block FP4 inputs + FP8 requant (libqattn on the GPU)
  orc_fp8      the oracle's FP8 method (cross-check of gpu_fp8)
  orc_fp8_noP  FP8 inputs, FP32 softmax, P left unquantized (isolates the P quantization)
  orc_fp8_fig4 FP8 inputs, the normalized P quantized with scale 1/448 (literal Fig. 4 reading)

over sequence lengths and outlier-channel strength, on seeded synthetic inputs shaped like the
joint text + image sequence (rows sampled per head; every output row depends on all keys).

    python tests/error_study.py [--heads 4] [--rows 128]

Prints a markdown table.  Needs a GPU for the gpu_* columns.
"""
from __future__ import annotations

import argparse
import os
import sys

import numpy as np
import torch

HERE = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, os.path.dirname(HERE))
sys.path.insert(0, HERE)

import oracle  # noqa: E402
import workloads  # noqa: E402


def rel_l2(got: np.ndarray, ref: np.ndarray) -> float:
    return float(np.linalg.norm(got - ref) / np.linalg.norm(ref))


def study(L: int, outliers: int, heads: int, rows_per_head: int, seed: int):
    import precision_quantized_attention_b200 as qa
    from parity import gpu_path
    res = {}
    for mode in ("fp8", "fp4"):
        w = workloads.custom(f"err_{mode}", mode, 1, heads, L, 128, seed=seed, outliers=outliers)
        q, k, v = workloads.make_qkv(w)
        rows = workloads.sample_rows(w, per_head=min(rows_per_head, L)).numpy()
        if mode == "fp8":
            ref = oracle.attention_values(q.double().numpy(), k.double().numpy(),
                                          v.double().numpy(), sm_scale=w.sm_scale, flags=0,
                                          rows=rows)
            res["orc_fp8"] = rel_l2(oracle.method_forward(q, k, v, "fp8", w.sm_scale, rows=rows), ref)
            res["orc_fp8_noP"] = rel_l2(oracle.method_forward(q, k, v, "fp8", w.sm_scale, rows=rows,
                                                              flags=oracle.FP32), ref)
            res["orc_fp8_fig4"] = rel_l2(
                oracle.method_forward(q, k, v, "fp8", w.sm_scale, rows=rows,
                                      flags=oracle.FP32 | oracle.QUANT_P | oracle.FIG4_LITERAL), ref)
        path = gpu_path(w, q, k, v)
        got = path.out.float().reshape(-1, 128)[torch.as_tensor(rows, device=path.out.device)]
        res[f"gpu_{mode}"] = rel_l2(got.cpu().numpy().astype(np.float64), ref)
        del path
    return res


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--heads", type=int, default=4)
    ap.add_argument("--rows", type=int, default=128)
    args = ap.parse_args()
    cols = ["gpu_fp8", "gpu_fp4", "orc_fp8", "orc_fp8_noP", "orc_fp8_fig4"]
    print(f"rel-L2 error vs unquantized FP64 attention; {args.heads} heads, {args.rows} sampled "
          f"rows per head, D=128, oracle threads {oracle.num_threads()}\n")
    print("| L | outlier channels (x10) | " + " | ".join(cols) + " |")
    print("|---|---|" + "---|" * len(cols))
    for L in (1024, 4608, 8704):
        for outliers in (0, 4):
            r = study(L, outliers, args.heads, args.rows, seed=50 + L % 97 + outliers)
            print(f"| {L} | {outliers} | " + " | ".join(f"{r[c]:.2e}" for c in cols) + " |",
                  flush=True)


if __name__ == "__main__":
    main()
