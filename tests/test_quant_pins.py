"""Pins of the weight-preparation oracle (int4 g128 with rotation, NVFP4) against definitions that are
not the oracle itself: the dense Hadamard of the layer oracle, exact round-to-nearest bounds, exactly
representable fixed points, torch's float8 conversion and brute force over the E2M1 grid."""

import math

import numpy as np
import pytest

from bit_routed_expert_sigmoid_b200 import synthetic as S
from oracle import flint_moe_ref as R
from oracle import quant_ref as Q

torch = pytest.importorskip("torch")


def bf16(x):
    return S.f32_to_bf16_bits(np.asarray(x, dtype=np.float32))


def test_int4_brute_force_nearest_code():
    # every code is the integer c in [-8, 7] nearest to r / s (ties to the even c), found by trying all 16
    rng = np.random.default_rng(1)
    w = bf16(rng.standard_normal((9, 256)) * 0.03)
    for rotate in (True, False):
        out = Q.quantize_int4_g128(w, rotate=rotate)
        r = R.rotate_segments(R.bf16_to_f64(w)) if rotate else R.bf16_to_f64(w)
        s = np.repeat(R.bf16_to_f64(out["scales"]), 128, axis=1)
        cands = np.arange(-8, 8)
        dist = np.abs(r[..., None] - cands * s[..., None])
        best = dist.min(-1, keepdims=True)
        tie = np.where(dist == best, cands, 99)
        even = np.where(tie % 2 == 0, tie, 99).min(-1)
        want = np.where((tie < 99).sum(-1) > 1, even, np.where(tie < 99, tie, 99).min(-1))
        np.testing.assert_array_equal(R.int4_values(out["codes"]), want)


def test_int4_scale_is_bf16_of_max_over_7():
    rng = np.random.default_rng(9)
    w = bf16(rng.standard_normal((4, 512)) * 0.05)
    out = Q.quantize_int4_g128(w, rotate=True)
    r = R.rotate_segments(R.bf16_to_f64(w)).reshape(4, 4, 128)
    m = np.abs(r).max(-1) / 7.0
    want = torch.from_numpy(m).to(torch.float32).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    # torch rounds through fp32 first; the two roundings agree unless m/7 sits within 2^-24 of a
    # bf16 midpoint, which these draws do not
    assert np.all(Q.int4_margins(w, True)["scale"] > 2.0 ** -20)
    np.testing.assert_array_equal(out["scales"], want)


def test_int4_margins_mark_the_rounding_boundaries():
    # a group with max 7 * 2^-4 (scale 2^-4 exactly) and values at, near and far from half-steps
    vals = np.zeros((1, 128))
    vals[0, 0] = 7 * 2.0 ** -4
    vals[0, 1] = 2.5 * 2.0 ** -4                      # exactly half-way: margin 0, ties to even (2)
    vals[0, 2] = 3.0 * 2.0 ** -4                      # an integer: margin 0.5
    vals[0, 3] = -1.5 * 2.0 ** -4                     # half-way, negative: ties to even (-2)
    w = bf16(vals)
    mg = Q.int4_margins(w, rotate=False)
    np.testing.assert_allclose(mg["code"][0, :4], [0.5, 0.0, 0.5, 0.0])
    out = Q.quantize_int4_g128(w, rotate=False)
    assert R.int4_values(out["codes"])[0, :4].tolist() == [7, 2, 3, -2]


def test_int4_fixed_points_unrotated():
    # W = q * 2^k with max |q| = 7 in every group: the scale is 2^k exactly and the codes are q
    rng = np.random.default_rng(2)
    q = rng.integers(-7, 8, size=(5, 256))
    q[:, 0] = 7
    q[:, 128] = -7
    k = rng.integers(-12, 4, size=(5, 2))
    w = q * np.exp2(np.repeat(k, 128, axis=1))
    out = Q.quantize_int4_g128(bf16(w), rotate=False)
    np.testing.assert_array_equal(R.bf16_to_f64(out["scales"]), np.exp2(k))
    np.testing.assert_array_equal(R.int4_values(out["codes"]), q)


@pytest.mark.parametrize("rotate", [True, False])
def test_int4_round_to_nearest_bound(rotate):
    rng = np.random.default_rng(3)
    w = bf16(rng.standard_normal((6, 1024)) * 0.02)
    out = Q.quantize_int4_g128(w, rotate=rotate)
    wf = R.bf16_to_f64(w)
    target = R.rotate_segments(wf) if rotate else wf                      # fp64, dense Hadamard
    deq = R.dequant_int4(out["codes"], out["scales"])                     # the layer's decoder
    s = np.repeat(R.bf16_to_f64(out["scales"]), 128, axis=1)
    m = np.repeat(np.abs(target).reshape(6, 8, 128).max(-1), 128, axis=1)
    # half a step, up to the fp64 rounding of r / s
    assert np.all(np.abs(deq - target) <= s / 2 * (1 + 2.0 ** -50) + 2.0 ** -60 * m)
    assert np.all(np.abs(R.int4_values(out["codes"])) <= 7)


def test_int4_zero_group():
    w = np.zeros((2, 256), np.uint16)
    w[1, 200] = bf16([0.5])[0]
    out = Q.quantize_int4_g128(w, rotate=False)
    assert out["scales"][0, 0] == 0 and out["scales"][0, 1] == 0 and out["scales"][1, 0] == 0
    assert np.all(out["codes"][0] == 0) and np.all(out["codes"][1, :64] == 0)
    assert R.int4_values(out["codes"])[1, 200] == 7


def test_rotation_lowers_error_on_outliers():
    # Gaussian rows with a few large outliers per group: the rotation spreads an outlier over the
    # group, so the group scale no longer wastes the code range on it
    rng = np.random.default_rng(4)
    w = rng.standard_normal((64, 2048)) * 0.02
    idx = rng.integers(0, 2048, size=(64, 24))
    np.put_along_axis(w, idx, rng.choice([-1, 1], size=idx.shape) * 0.6, axis=1)
    wb = bf16(w)
    wf = R.bf16_to_f64(wb)

    def rel_err(rotate):
        out = Q.quantize_int4_g128(wb, rotate=rotate)
        deq = R.dequant_int4(out["codes"], out["scales"])
        back = R.rotate_segments(deq) if rotate else deq                  # Hn is its own inverse
        return np.linalg.norm(back - wf) / np.linalg.norm(wf)

    assert rel_err(True) < 0.5 * rel_err(False)


def test_e2m1_rounding_brute_force():
    rng = np.random.default_rng(5)
    grid = np.array([0, 0.5, 1, 1.5, 2, 3, 4, 6])
    mids = (grid[1:] + grid[:-1]) / 2
    x = np.concatenate([rng.uniform(-8, 8, 4000), mids, -mids, grid, -grid, [7.0, 1e9, -1e9]]).astype(np.float32)
    got = Q.e2m1_rne(x)
    mag = np.abs(x.astype(np.float64))
    dist = np.abs(mag[:, None] - grid[None, :])
    best = dist.min(1, keepdims=True)
    cand = np.where(dist == best, np.arange(8)[None, :], 99)
    even = np.where(cand % 2 == 0, cand, 99).min(1)
    want = np.where((cand < 99).sum(1) > 1, even, cand.min(1))
    np.testing.assert_array_equal(got & 0x7, want)
    np.testing.assert_array_equal(got >> 3, np.signbit(x).astype(np.uint8))


def test_e4m3_rounding_matches_torch():
    rng = np.random.default_rng(6)
    x = np.concatenate([
        np.exp2(rng.uniform(-12, np.log2(448.0), 20000)),
        R.e4m3fn_to_f64(np.arange(0x7F)),                   # every finite non-negative code
        [0.0, 2.0 ** -10, 2.0 ** -9 * 0.5, 2.0 ** -9 * 1.5],
    ]).astype(np.float32)
    want = torch.from_numpy(x).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    np.testing.assert_array_equal(Q.e4m3_rne_pos(x), want)
    assert Q.e4m3_rne_pos(np.float32([448.0, 460.0, 1e6])).tolist() == [0x7E] * 3


def test_nvfp4_fixed_points():
    # amax = 6 * 448 * 2^-10, so ts = 2^-10 exactly; every block holds +-6 and its scale is an E4M3
    # value, so the block scale, the codes and the tensor scale come back exactly
    rng = np.random.default_rng(7)
    N, K = 4, 64
    sb = rng.integers(0x20, 0x7E, size=(N, K // 16))
    sb[0, 0] = 0x7E                                                        # 448: the Linear's amax
    sv = R.e4m3fn_to_f64(sb)
    codes = rng.integers(0, 16, size=(N, K))
    codes[:, ::16] = 0x7                                                    # +6 in every block
    ts = 2.0 ** -10
    w = R.e2m1_to_f64(codes) * np.repeat(sv, 16, axis=1) * ts
    out = Q.quantize_nvfp4(bf16(w))
    assert float(out["tscale"]) == ts
    np.testing.assert_array_equal(out["scales"], sb)
    # -0 is stored as the sign-only code 8; compare values
    np.testing.assert_array_equal(R.e2m1_to_f64(R.unpack_nibbles(out["codes"])), R.e2m1_to_f64(codes))


def test_nvfp4_round_to_nearest_bound():
    rng = np.random.default_rng(8)
    w = bf16(rng.standard_normal((8, 512)) * np.exp2(rng.uniform(-6, 2, (8, 1))))
    out = Q.quantize_nvfp4(w)
    wf = R.bf16_to_f64(w)
    deq = R.dequant_nvfp4(out["codes"], out["scales"], out["tscale"])
    d = np.repeat(R.e4m3fn_to_f64(out["scales"]), 16, axis=1) * float(out["tscale"])
    x = np.abs(wf) / d
    half_step = np.where(x <= 2, 0.25, np.where(x <= 4, 0.5, 1.0))       # E2M1 grid spacing / 2
    assert np.all(np.abs(deq - wf) <= (half_step * (1 + 1e-6)) * d)
    # every block scale keeps its block inside the E2M1 range
    assert np.all(x <= 6.0 * (1 + 2.0 ** -3))


def test_nvfp4_zero_linear():
    out = Q.quantize_nvfp4(np.zeros((2, 32), np.uint16))
    assert float(out["tscale"]) == 1.0
    assert np.all(out["scales"] == 0) and np.all(out["codes"] == 0)


def test_nvfp4_margins_mark_the_rounding_boundaries():
    # ts = 2^-10 (amax 6 * 448 * 2^-10); block 0 has scale 448 -> d = 448 * 2^-10; 1.25 d is an E2M1
    # midpoint (margin 0, rounds to the even code 1.0), 1.5 d a grid value
    d = 448 * 2.0 ** -10
    w = np.zeros((1, 32))
    w[0, 0] = 6 * d
    w[0, 1] = 1.25 * d
    w[0, 2] = 1.5 * d
    wb = bf16(w)
    mg = Q.nvfp4_margins(wb)
    assert mg["code"][0, 1] == 0.0 and mg["code"][0, 2] > 0.1
    out = Q.quantize_nvfp4(wb)
    assert R.e2m1_to_f64(R.unpack_nibbles(out["codes"]))[0, :3].tolist() == [6.0, 1.0, 1.5]
    assert mg["scale"][0, 0] > 0.01                 # 448 is an E4M3 value, far from a midpoint
