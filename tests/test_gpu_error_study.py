"""The error study's GPU columns against the oracle (tests/error_study.py): on a reduced grid of
the study's three axes (sequence length with and without outlier channels, text-row scaling,
outlier strength), the GPU output equals the oracle's output of the same method (FP8 and FP4
mode) within the parity bar, while both differ from unquantized attention by the amounts the
study reports; and the study's structural facts hold: FP4 blocks err more than per-tensor FP8 on
plain inputs, and quantizing P adds error on top of FP8 inputs."""
import pytest

from error_study import study

pytestmark = pytest.mark.gpu

GRID = [
    ("length 1024, plain", 1024, {}),
    ("length 4608, 4 channels x10", 4608, {"outliers": 4}),
    ("text rows x4", 2048, {"text_scale": 4.0}),
    ("8 channels x30", 2048, {"outliers": 8, "outlier_scale": 30.0}),
    ("4 channels x3", 2048, {"outliers": 4, "outlier_scale": 3.0}),
]


@pytest.mark.parametrize("label,L,kw", GRID, ids=[g[0] for g in GRID])
def test_gpu_matches_oracle_on_the_error_study_grid(label, L, kw):
    r = study(L, heads=2, rows_per_head=32, seed=70 + L % 97, **kw)
    print(label, {k: f"{v:.2e}" for k, v in r.items()})
    assert r["gpu_vs_orc_fp8"] <= 1e-2 and r["gpu_vs_orc_fp4"] <= 1e-2
    # the GPU's distance from unquantized attention is the oracle's, up to that agreement
    assert abs(r["gpu_fp8"] - r["orc_fp8"]) <= 1e-2 and abs(r["gpu_fp4"] - r["orc_fp4"]) <= 1e-2
    if not kw:
        assert r["orc_fp4"] > r["orc_fp8"]           # 16-element FP4 blocks vs per-tensor FP8
        assert r["orc_fp8"] > r["orc_fp8_noP"]       # P quantization adds to the input error
