"""The algorithmic bytes and flops bench.py divides by (the roofline numerators) against the sizes of the
arrays the layer really holds and against each other. No GPU."""

import os
import sys

import numpy as np
import pytest

from bit_routed_expert_sigmoid_b200 import synthetic as S

sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
import bench  # noqa: E402


@pytest.mark.parametrize("fmt", ["int4", "nvfp4"])
def test_expert_and_layer_bytes_match_the_arrays(fmt):
    L = S.make_layer(32, fmt)
    assert bench.expert_bytes(fmt) == S.expert_nbytes(L)
    n_active, T = 7, 8
    arrays = n_active * S.expert_nbytes(L) + L["sh_gu"].nbytes + L["sh_dn"].nbytes + L["router_w"].nbytes
    x_y = 2 * T * bench.H * 2
    assert bench.algorithmic_bytes(32, fmt, T, n_active) == arrays + x_y


@pytest.mark.parametrize("fmt", ["int4", "nvfp4"])
def test_routed_stage_weights_match_the_arrays(fmt):
    L = S.make_layer(32, fmt)
    E, T, K, n = 32, 2048, 6, 5
    gu_w = (L["gu_codes"].nbytes + L["gu_scales"].nbytes + (L["gu_tscale"].nbytes if fmt == "nvfp4" else 0)) // E
    dn_w = (L["dn_codes"].nbytes + L["dn_scales"].nbytes + (L["dn_tscale"].nbytes if fmt == "nvfp4" else 0)) // E
    P = T * K
    assert bench.stage_bytes("gu_routed", E, fmt, T, K, n) == n * gu_w + P * bench.H * 2 + P * bench.I * 2
    assert bench.stage_bytes("dn_routed", E, fmt, T, K, n) == n * dn_w + P * bench.I * 2 + P * bench.H * 2


def test_flops_add_up():
    T, K, E = 2048, 6, 256
    parts = (bench.stage_flops("gu_routed", E, T, K) + bench.stage_flops("dn_routed", E, T, K)
             + bench.stage_flops("gu_shared", E, T, K) + bench.stage_flops("dn_shared", E, T, K) // 2)
    assert bench.grouped_gemm_flops(T, K) == parts
    # 2 flops per multiply-add over every (token, slot) of the routed experts' three projections
    assert bench.stage_flops("gu_routed", E, T, K) == 2 * T * K * (2 * bench.I) * bench.H


@pytest.mark.parametrize("fmt", ["int4", "nvfp4"])
def test_quant_bytes_per_weight(fmt):
    rows, cols = 64, 2048
    codes = rows * cols // 2
    scales = rows * (cols // 128) * 2 if fmt == "int4" else rows * (cols // 16)
    reads = 2 * rows * cols * (1 if fmt == "int4" else 2)        # NVFP4 reads the input twice (amax pass)
    assert bench.quant_bytes_per_weight(fmt) * rows * cols == pytest.approx(reads + codes + scales)
    assert np.isclose(bench.quant_bytes_per_weight("int4"), 2.515625)


def test_w4a4_stage_bytes_match_the_arrays():
    # W4A4: the routed stages read the NVFP4 weight arrays and the NVFP4 activation rows (codes, block
    # scales, one fp32 tensor scale per row); gate|up writes fp32 h, down reads h's NVFP4 rows and writes fp16 o
    L = S.make_layer(32, "nvfp4")
    E, T, K, n = 32, 2048, 6, 5
    P = T * K
    gu_w = (L["gu_codes"].nbytes + L["gu_scales"].nbytes + L["gu_tscale"].nbytes) // E
    dn_w = (L["dn_codes"].nbytes + L["dn_scales"].nbytes + L["dn_tscale"].nbytes) // E
    xa = P * (bench.H // 2 + bench.H // 16 + 4)
    ha = P * (bench.I // 2 + bench.I // 16 + 4)
    assert bench.stage_bytes("gu_routed", E, "nvfp4", T, K, n, w4a4=True) == n * gu_w + xa + P * bench.I * 4
    assert bench.stage_bytes("dn_routed", E, "nvfp4", T, K, n, w4a4=True) == n * dn_w + ha + P * bench.H * 2
    assert bench.stage_bytes("hq", E, "nvfp4", T, K, n, w4a4=True) == P * bench.I * 4 + ha
    # the other stages are those of the 16-bit-activation path
    for st in ("router_logits", "topk", "permute", "gu_shared", "dn_shared", "combine"):
        assert bench.stage_bytes(st, E, "nvfp4", T, K, n, w4a4=True) == bench.stage_bytes(st, E, "nvfp4", T, K, n)


def test_prefill_roofline_picks_the_slower_roofline():
    peaks = {"hbm_gbs": 6554.6, "bf16_tflops": 1657.2, "source": "measured"}
    E, T, n = 256, 2048, 256
    # W4A4 gate|up at T = 2048: 341 MB at 6.55 TB/s (52 µs) against 51.5 GFLOP at 4 x 1657 TF (7.8 µs): HBM
    r = bench.prefill_roofline("gu_routed", 0.0663, E, "nvfp4", T, n, peaks, "prefill_nvfp4_w4a4", True)
    assert r["bound"] == "hbm" and r["unit"] == "GB/s" and r["peak"] == peaks["hbm_gbs"]
    assert r["achieved"] == pytest.approx(bench.stage_bytes("gu_routed", E, "nvfp4", T, 6, n, True) / 66.3e-6 / 1e9, rel=1e-3)
    assert r["frac"] == pytest.approx(r["achieved"] / peaks["hbm_gbs"], rel=1e-3)
    # with a hypothetical HBM ten times faster the FP4 tensor time is the larger: tensor, peak = 4 x bf16
    fast = dict(peaks, hbm_gbs=65546.0)
    r = bench.prefill_roofline("gu_routed", 0.0663, E, "nvfp4", T, n, fast, "prefill_nvfp4_w4a4", True)
    assert r["bound"] == "tensor" and r["peak"] == pytest.approx(4 * peaks["bf16_tflops"], rel=1e-3)
    # W4A16: always the bf16 tensor peak (fp16 MMAs at the bf16 rate)
    r = bench.prefill_roofline("gu_routed", 0.12, E, "int4", T, n, peaks, "prefill_int4", False)
    assert r["bound"] == "tensor" and r["peak"] == peaks["bf16_tflops"]
    assert r["achieved"] == pytest.approx(bench.stage_flops("gu_routed", E, T, 6) / 0.12e-3 / 1e12, rel=1e-3)
