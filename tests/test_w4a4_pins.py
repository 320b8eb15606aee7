"""Pins of the oracle's W4A4 activation quantiser (quantize_act_nvfp4: NVFP4 per row, fp32 decisions)
against definitions that are not the quantiser itself: the fp64 round-to-nearest NVFP4 quantiser of the
weight-preparation oracle row by row, torch's float8 conversion, brute force over the E2M1 grid, exact
fixed points and the half-step error bound; and of the W4A4 layer against its own structure."""

import numpy as np
import pytest

from bit_routed_expert_sigmoid_b200 import synthetic as S
from oracle import flint_moe_ref as R
from oracle import quant_ref as Q

torch = pytest.importorskip("torch")


def rows(n, k, seed):
    rng = np.random.default_rng(seed)
    v = rng.standard_normal((n, k)) * np.exp2(rng.uniform(-8, 4, (n, 1)))
    v[0, :] = 0.0
    v[1, 16:32] = 0.0
    return v.astype(np.float32)


def test_matches_the_fp64_quantiser_away_from_boundaries():
    v = rows(40, 512, 1)
    bf = S.f32_to_bf16_bits(v)                        # quant_ref takes bf16 rows: compare on bf16 values
    vb = R.bf16_to_f64(bf).astype(np.float32)
    q = R.quantize_act_nvfp4(vb)
    n_ok = 0
    for i in range(v.shape[0]):
        ref = Q.quantize_nvfp4(bf[i:i + 1])
        mg = Q.nvfp4_margins(bf[i:i + 1])
        assert q["ts"][i] == ref["tscale"]
        ok_b = mg["scale"][0] > 2.0 ** -20
        np.testing.assert_array_equal(q["scales"][i][ok_b], ref["scales"][0][ok_b])
        ok = (mg["code"][0] > 2.0 ** -19) & np.repeat(ok_b, 16)
        got = R.e2m1_to_f64(q["codes"][i])
        want = R.e2m1_to_f64(R.unpack_nibbles(ref["codes"])[0])
        np.testing.assert_array_equal(got[ok], want[ok])
        n_ok += ok.sum()
    assert n_ok > 0.97 * v.size


def test_e2m1_brute_force_and_e4m3_against_torch():
    rng = np.random.default_rng(2)
    grid = np.array([0, 0.5, 1, 1.5, 2, 3, 4, 6])
    a = np.concatenate([rng.uniform(0, 8, 5000), (grid[1:] + grid[:-1]) / 2, grid, [7.0, 100.0]])
    got = R._e2m1_nearest_even(a)
    dist = np.abs(a[:, None] - grid[None, :])
    best = dist.min(1, keepdims=True)
    cand = np.where(dist == best, np.arange(8), 99)
    even = np.where(cand % 2 == 0, cand, 99).min(1)
    np.testing.assert_array_equal(got, np.where((cand < 99).sum(1) > 1, even, cand.min(1)))
    x = np.concatenate([np.exp2(rng.uniform(-12, np.log2(448.0), 20000)), R.e4m3fn_to_f64(np.arange(0x7F))])
    x = x.astype(np.float32)
    want = torch.from_numpy(x).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    np.testing.assert_array_equal(R._e4m3_nearest_even_pos(x), want)


def test_fixed_points_and_bounds():
    # rows built as e2m1 x E4M3 x 2^-8 with a +-6 in every block and one block at scale 448: amax is
    # 6 * 448 * 2^-8, so ts = 2^-8 exactly and every code and block scale comes back
    rng = np.random.default_rng(3)
    n, k = 6, 128
    sb = rng.integers(0x20, 0x7E, size=(n, k // 16))
    sb[:, 0] = 0x7E
    codes = rng.integers(0, 16, size=(n, k))
    codes[:, ::16] = 7
    v = (R.e2m1_to_f64(codes) * np.repeat(R.e4m3fn_to_f64(sb), 16, axis=1) * 2.0 ** -8).astype(np.float32)
    q = R.quantize_act_nvfp4(v)
    assert np.all(q["ts"] == np.float32(2.0 ** -8))
    np.testing.assert_array_equal(q["scales"], sb)
    np.testing.assert_array_equal(q["values"], v.astype(np.float64))
    # random rows: within half a grid step of the block's scale; an all-zero row gives ts = 1, codes 0
    v = rows(30, 256, 4)
    q = R.quantize_act_nvfp4(v)
    d = np.repeat(R.e4m3fn_to_f64(q["scales"]), 16, axis=1) * q["ts"].astype(np.float64)[:, None]
    x = np.abs(v.astype(np.float64)) / np.where(d > 0, d, 1)
    half = np.where(x <= 2, 0.25, np.where(x <= 4, 0.5, 1.0))
    assert np.all(np.abs(q["values"] - v) <= half * d * (1 + 1e-6) + 1e-30)
    assert q["ts"][0] == 1.0 and np.all(q["codes"][0] == 0)


def test_w4a4_layer_structure():
    # with W4A4 the routed experts see quantised inputs: each permuted row's input is its token's
    # quantised x, the routing is that of W4A16, y differs from W4A16; the option is refused for the
    # rotated int4 format
    L = S.make_layer(32, "nvfp4", H=256, I=128, Is=64)
    x = S.make_x(5, H=256)
    a = R.moe_forward(L, x, w4a4=True, keep=True)
    b = R.moe_forward(L, x, keep=True)
    np.testing.assert_array_equal(a["ids"], b["ids"])                 # routing is untouched
    xq = R.quantize_act_nvfp4(R.bf16_to_f64(x).astype(np.float32))["values"]
    np.testing.assert_array_equal(a["x_in"][0], xq[a["perm"][0] // 6])
    assert not np.allclose(a["y"], b["y"])
    with pytest.raises(ValueError):
        R.moe_forward(S.make_layer(32, "int4", H=256, I=128, Is=64), x, w4a4=True)


def test_w4a4_on_grid_inputs_matches_w4a16_up_to_the_down_input():
    # token rows that already lie on the per-row NVFP4 grid are quantised to themselves: each row is
    # E2M1 code x E4M3 block scale x 2^-8 with a +-6 in every block and one block at scale 448, so the
    # row's tensor scale is exactly 2^-8 and every block scale and code comes back (and such values are
    # exact in bf16). The W4A4 layer's routed inputs, gate|up and SwiGLU outputs are then those of the
    # 16-bit-activation layer bit for bit; only the down input differs (h is quantised, x was not)
    # (kekzle/Flint-NVFP4, evaluation table: W4A4 quantises the activations of the same NVFP4 weights)
    L = S.make_layer(32, "nvfp4", H=256, I=128, Is=64)
    rng = np.random.default_rng(7)
    T, H = 7, 256
    sb = rng.integers(0x20, 0x7E, size=(T, H // 16))
    sb[:, 0] = 0x7E
    codes = rng.integers(0, 16, size=(T, H))
    codes[:, ::16] = 7
    v = R.e2m1_to_f64(codes) * np.repeat(R.e4m3fn_to_f64(sb), 16, axis=1) * 2.0 ** -8
    x_bits = S.f32_to_bf16_bits(v.astype(np.float32))
    np.testing.assert_array_equal(R.bf16_to_f64(x_bits), v)
    a = R.moe_forward(L, x_bits, w4a4=True, keep=True)
    b = R.moe_forward(L, x_bits, keep=True)
    np.testing.assert_array_equal(a["ids"], b["ids"])
    np.testing.assert_array_equal(a["x_in"], b["x_in"])
    np.testing.assert_array_equal(a["h"], b["h"])
    assert not np.array_equal(a["h_in"], b["h_in"])
    np.testing.assert_array_equal(a["ys"], b["ys"])
