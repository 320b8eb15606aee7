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


def test_inv_sqrt128_is_nearest_f32():
    c = float(Q.F32_INV_SQRT128)
    exact = 1.0 / math.sqrt(128.0)
    up = float(np.nextafter(Q.F32_INV_SQRT128, np.float32(1)))
    dn = float(np.nextafter(Q.F32_INV_SQRT128, np.float32(0)))
    assert abs(c - exact) < abs(up - exact) and abs(c - exact) < abs(dn - exact)


def test_butterfly_matches_dense_hadamard():
    rng = np.random.default_rng(1)
    v = rng.standard_normal((7, 512)).astype(np.float32)
    got = Q.fwht128_f32(v).astype(np.float64)
    ref = R.rotate_segments(v.astype(np.float64))
    # 7 butterfly stages and one multiplication, each rounding by at most half an fp32 ulp of a
    # partial sum bounded by the segment's L1 norm
    l1 = np.abs(v.reshape(7, 4, 128)).sum(-1, keepdims=True)
    bound = np.repeat(l1, 128, axis=-1).reshape(7, 512) * 8 * 2.0 ** -24 / math.sqrt(128) + 1e-30
    assert np.all(np.abs(got - ref) <= bound)
    # the normalised transform is its own inverse
    np.testing.assert_allclose(Q.fwht128_f32(Q.fwht128_f32(v)), v, rtol=0, atol=1e-5)


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
    # half a step, plus the fp32 rotation and division errors (a few ulp of the group maximum)
    assert np.all(np.abs(deq - target) <= s / 2 + 2.0 ** -18 * m)
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
    np.testing.assert_array_equal(got >> 3, (x.view(np.uint32) >> 31).astype(np.uint8))


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
