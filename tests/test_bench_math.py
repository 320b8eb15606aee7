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
