"""Error study of the quantized SDPA: relative L2 error of the output against unquantized FP64
attention, for the pieces of the method the blog ("Optimizing FLUX.1 Kontext for Image Editing
with Low-Precision Quantization", "Workflow and quantization", Fig. 4; its Figs. 6-7 compare the
precisions by image quality, which these synthetic inputs stand in for) combines:

  gpu_fp8      the method with per-tensor FP8 inputs (libqattn on the GPU)
  gpu_fp4      the method with per-block FP4 inputs + FP8 requant (libqattn on the GPU)
  orc_fp8      the oracle's FP8 method (cross-check of gpu_fp8)
  orc_fp4      the oracle's FP4 method (cross-check of gpu_fp4)
  orc_fp8_noP  FP8 inputs, FP32 softmax, P left unquantized (isolates the P quantization)
  orc_fp8_fig4 FP8 inputs, the normalized P quantized with scale 1/448 (literal Fig. 4 reading)

along three axes of the seeded synthetic joint text + image sequence: the sequence length (with
and without outlier channels), the scale of the text rows (x1, x2, x4), and the outlier channels
of Q and K (0, 4 or 8 per head, scaled x3, x10 or x30).  Rows are sampled per head; every output
row depends on all keys.  gpu_vs_orc_* is the GPU output's rel-L2 distance from the oracle's
output of the same method (tests/test_gpu_error_study.py asserts it on a reduced grid).

    python tests/error_study.py [--heads 4] [--rows 128]

Prints markdown tables.  Needs a GPU for the gpu_* columns.
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

COLS = ["gpu_fp8", "gpu_fp4", "orc_fp8", "orc_fp4", "orc_fp8_noP", "orc_fp8_fig4",
        "gpu_vs_orc_fp8", "gpu_vs_orc_fp4"]


def rel_l2(got: np.ndarray, ref: np.ndarray) -> float:
    return float(np.linalg.norm(got - ref) / np.linalg.norm(ref))


def study(L: int, heads: int, rows_per_head: int, seed: int, outliers: int = 0,
          outlier_scale: float = 10.0, text_scale: float = 1.0) -> dict:
    """The columns of COLS for one point of the grid."""
    from parity import gpu_path
    res = {}
    for mode in ("fp8", "fp4"):
        w = workloads.custom(f"err_{mode}", mode, 1, heads, L, 128, seed=seed, outliers=outliers,
                             outlier_scale=outlier_scale, text_scale=text_scale)
        q, k, v = workloads.make_qkv(w)
        rows = workloads.sample_rows(w, per_head=min(rows_per_head, L)).numpy()
        ref = oracle.attention_values(q.double().numpy(), k.double().numpy(), v.double().numpy(),
                                      sm_scale=w.sm_scale, flags=0, rows=rows)
        orc = oracle.method_forward(q, k, v, mode, w.sm_scale, rows=rows)
        res[f"orc_{mode}"] = rel_l2(orc, ref)
        if mode == "fp8":
            res["orc_fp8_noP"] = rel_l2(oracle.method_forward(q, k, v, "fp8", w.sm_scale, rows=rows,
                                                              flags=oracle.FP32), ref)
            res["orc_fp8_fig4"] = rel_l2(
                oracle.method_forward(q, k, v, "fp8", w.sm_scale, rows=rows,
                                      flags=oracle.FP32 | oracle.QUANT_P | oracle.FIG4_LITERAL), ref)
        path = gpu_path(w, q, k, v)
        got = path.out.float().reshape(-1, 128)[torch.as_tensor(rows, device=path.out.device)]
        got = got.cpu().numpy().astype(np.float64).reshape(orc.shape)
        res[f"gpu_{mode}"] = rel_l2(got, ref)
        res[f"gpu_vs_orc_{mode}"] = rel_l2(got, orc)
        del path
    return res


# the grid of the full study: (label, L, study keyword arguments)
GRID_LENGTH = [(f"L={L}, {o} outlier ch x10", L, {"outliers": o}) for L in (1024, 4608, 8704)
               for o in (0, 4)]
GRID_TEXT = [(f"L=4608, text rows x{t:g}", 4608, {"text_scale": t}) for t in (1.0, 2.0, 4.0)]
GRID_OUTLIERS = [(f"L=4608, {o} outlier ch x{s:g}", 4608, {"outliers": o, "outlier_scale": s})
                 for o in (4, 8) for s in (3.0, 10.0, 30.0)] + [("L=4608, no outliers", 4608, {})]


def table(title, grid, heads, rows, cols=COLS):
    print(f"\n{title}\n")
    print("| case | " + " | ".join(cols) + " |")
    print("|---|" + "---|" * len(cols))
    for label, L, kw in grid:
        r = study(L, heads, rows, seed=50 + L % 97 + int(kw.get("outliers", 0)), **kw)
        print(f"| {label} | " + " | ".join(f"{r[c]:.2e}" for c in cols) + " |", flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--heads", type=int, default=4)
    ap.add_argument("--rows", type=int, default=128)
    args = ap.parse_args()
    print(f"rel-L2 error vs unquantized FP64 attention; {args.heads} heads, {args.rows} sampled "
          f"rows per head, D=128, oracle threads {oracle.num_threads()}")
    table("Sequence length", GRID_LENGTH, args.heads, args.rows)
    table("Text-row scaling (no outliers)", GRID_TEXT, args.heads, args.rows)
    table("Outlier channels of Q and K", GRID_OUTLIERS, args.heads, args.rows)


if __name__ == "__main__":
    main()
