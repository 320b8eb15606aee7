"""Pins the fp64 oracle to facts that do not come from the oracle itself: closed forms, invariants
of the mathematics, library routines for special cases, hand-derived format tables and brute force
on tiny inputs. A plausible slip anywhere in the oracle (a dropped term, a wrong sign or index, a
transposed operand, a missing rotation) fails at least one of these."""

import itertools
import math
import os

import numpy as np
import pytest

from bit_routed_expert_sigmoid_b200 import synthetic as S
from oracle import flint_moe_ref as R

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _small_layer(E=8, fmt="int4", H=256, I=128, Is=64, seed=5):
    return S.make_layer(E, fmt, H=H, I=I, Is=Is, seed=seed)


# ----------------------------------------------------------------------------- Hadamard

def test_hadamard_involution_and_symmetry():
    Hn = R.hadamard_normalized(128)
    np.testing.assert_allclose(Hn @ Hn, np.eye(128), atol=1e-13)
    np.testing.assert_array_equal(Hn, Hn.T)


def test_hadamard_matches_scipy_sylvester():
    scipy_linalg = pytest.importorskip("scipy.linalg")
    np.testing.assert_allclose(R.hadamard_normalized(128), scipy_linalg.hadamard(128) / math.sqrt(128),
                               rtol=0, atol=1e-15)


def test_rotate_segments_is_blockdiagonal():
    rng = np.random.default_rng(0)
    v = rng.standard_normal((3, 512))
    Hn = R.hadamard_normalized(128)
    ref = np.concatenate([v[:, 128 * j:128 * (j + 1)] @ Hn for j in range(4)], axis=1)
    np.testing.assert_allclose(R.rotate_segments(v), ref, atol=1e-13)
    # an impulse in segment 2 stays in segment 2 and spreads with magnitude 1/sqrt(128)
    e = np.zeros(512)
    e[256 + 5] = 1.0
    r = R.rotate_segments(e)
    assert np.all(r[:256] == 0) and np.all(r[384:] == 0)
    np.testing.assert_allclose(np.abs(r[256:384]), 1 / math.sqrt(128), atol=1e-15)
    np.testing.assert_allclose(R.rotate_segments(R.rotate_segments(v)), v, atol=1e-13)


# ----------------------------------------------------------------------------- formats

def _read_table(name):
    rows = []
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.split("#")[0].strip()
            if line:
                rows.append(line.split())
    return rows


def test_int4_golden_bytes():
    rows = _read_table("int4_bytes.txt")
    codes = np.array([[int(r[0], 16) for r in rows]], dtype=np.uint8)
    want = np.array([[int(v) for r in rows for v in (r[1], r[2])]])
    np.testing.assert_array_equal(R.int4_values(codes), want)


def test_int4_dequant_scale_per_group_of_128():
    N, K = 3, 512
    codes = np.full((N, K // 2), 0x11, dtype=np.uint8)          # every code is +1
    scales = np.array([[0x3F80, 0x4000, 0x3E80, 0xBF00]] * N, dtype=np.uint16)   # 1, 2, 0.25, -0.5
    W = R.dequant_int4(codes, scales)
    want = np.repeat(np.array([1.0, 2.0, 0.25, -0.5]), 128)
    np.testing.assert_array_equal(W, np.tile(want, (N, 1)))
    codes[:, :] = 0x88                                          # every code is -8
    np.testing.assert_array_equal(R.dequant_int4(codes, scales), -8 * np.tile(want, (N, 1)))
    # the tensor scale multiplies everything (exact f32 value of the stored scale)
    np.testing.assert_array_equal(R.dequant_int4(codes, scales, np.float32(0.5)), -4 * np.tile(want, (N, 1)))


def test_int4_layer_size_matches_the_container():
    # Aijuus/flint-w4exp, model summary: the routed experts (47 MoE blocks x 256) take ~18.2 GiB at
    # four bits with a bf16 scale per 128 of K. Our storage layout reproduces that size exactly.
    L = _small_layer(E=2, H=2048, I=512, Is=8)
    per_expert = S.expert_nbytes(L)
    assert per_expert == 3 * 2048 * 512 // 2 + (3 * 2048 * 512 // 128) * 2 == 1_622_016
    gib = 47 * 256 * per_expert / 2 ** 30
    assert abs(gib - 18.2) < 0.05


def test_e2m1_table():
    rows = _read_table("e2m1_values.txt")
    codes = np.array([int(r[0]) for r in rows])
    want = np.array([float(r[1]) for r in rows])
    got = R.e2m1_to_f64(codes)
    np.testing.assert_array_equal(got, want)
    np.testing.assert_array_equal(np.signbit(got[8:]), True)


def test_e4m3_matches_torch_float8_e4m3fn():
    torch = pytest.importorskip("torch")
    b = np.arange(256, dtype=np.uint8)
    ref = torch.from_numpy(b).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    got = R.e4m3fn_to_f64(b)
    np.testing.assert_array_equal(np.isnan(got), np.isnan(ref))
    m = ~np.isnan(ref)
    np.testing.assert_array_equal(got[m], ref[m])


def test_nvfp4_value_is_code_times_block_scale_times_tensor_scale():
    # kekzle/Flint-NVFP4, lm_head row: the BF16 weight is code x block scale x tensor scale.
    e2m1 = {c: float(v) for c, v in ((int(r[0]), r[1]) for r in _read_table("e2m1_values.txt"))}
    ts = np.float32(0.01)
    for e in range(-4, 3):
        sbyte = (e + 7) << 3
        codes = np.array([[lo | (hi << 4) for lo in range(16) for hi in range(16)]], dtype=np.uint8)
        scales = np.full((1, codes.shape[1] * 2 // 16), sbyte, dtype=np.uint8)
        W = R.dequant_nvfp4(codes, scales, ts)
        want = []
        for lo in range(16):
            for hi in range(16):
                want += [e2m1[lo] * 2.0 ** e * float(ts), e2m1[hi] * 2.0 ** e * float(ts)]
        np.testing.assert_array_equal(W[0], np.array(want))
    # block scales apply per 16 columns
    codes = np.full((1, 16), 0x22, dtype=np.uint8)                  # every value 1.0
    scales = np.array([[0x38, 0x40]], dtype=np.uint8)               # e4m3 1.0, 2.0
    W = R.dequant_nvfp4(codes, scales, np.float32(1.0))
    np.testing.assert_array_equal(W[0], np.repeat([1.0, 2.0], 16))


def test_bf16_decode_matches_torch():
    torch = pytest.importorskip("torch")
    bits = np.arange(0, 65536, 7, dtype=np.uint16)
    ref = torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).to(torch.float64).numpy()
    got = R.bf16_to_f64(bits)
    m = ~np.isnan(ref)
    np.testing.assert_array_equal(np.isnan(got), ~m)
    np.testing.assert_array_equal(got[m], ref[m])


def test_generator_bf16_rounding_matches_torch():
    torch = pytest.importorskip("torch")
    v = np.random.default_rng(3).standard_normal(100000).astype(np.float32) * 3
    ref = torch.from_numpy(v).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    np.testing.assert_array_equal(S.f32_to_bf16_bits(v), ref)


# ----------------------------------------------------------------------------- router

def test_router_brute_force_subsets():
    rng = np.random.default_rng(11)
    for _ in range(200):
        E = 4
        logits = rng.standard_normal((1, E)) * 3
        for k in (1, 2, 3):
            r = R.route(logits, top_k=k)
            s = 1 / (1 + np.exp(-logits[0]))
            best = max(itertools.combinations(range(E), k), key=lambda c: sum(s[list(c)]))
            assert tuple(r["ids"][0]) == tuple(sorted(best))
            tot = sum(s[list(best)])
            np.testing.assert_allclose(r["w"][0], s[list(sorted(best))] / max(tot, 2 ** -14), rtol=1e-15)


def test_router_selects_top_raw_logits_no_bias():
    # sigmoid is increasing, so an unbiased router picks the largest logits
    rng = np.random.default_rng(12)
    logits = rng.standard_normal((50, 256))
    r = R.route(logits, top_k=6)
    want = np.sort(np.argsort(-logits, axis=1, kind="stable")[:, :6], axis=1)
    np.testing.assert_array_equal(r["ids"], want)
    np.testing.assert_allclose(r["w"].sum(axis=1), 1.0, rtol=1e-14)


def test_router_all_equal_logits_take_lowest_ids():
    r = R.route(np.zeros((3, 32)), top_k=6)
    np.testing.assert_array_equal(r["ids"], np.tile(np.arange(6), (3, 1)))
    np.testing.assert_allclose(r["w"], 1 / 6, rtol=1e-15)
    assert np.all(r["gap"] == 0)


def test_router_floor_is_active_for_tiny_scores():
    logits = np.full((1, 16), -30.0)
    logits[0, 3] = -29.0
    r = R.route(logits, top_k=6)
    s = 1 / (1 + math.exp(30.0))
    assert 6 * s < 2 ** -14
    assert r["ids"][0, 0] == 0 and 3 in r["ids"][0]
    np.testing.assert_allclose(r["w"][0][r["ids"][0] != 3], s / 2 ** -14, rtol=1e-12)
    assert r["w"][0].sum() < 1e-6


def test_permutation_matches_library_stable_sort():
    rng = np.random.default_rng(13)
    T, K, E = 37, 6, 16
    ids = np.sort(np.stack([rng.choice(E, K, replace=False) for _ in range(T)]), axis=1)
    pm = R.permutation(ids, E)
    flat = ids.reshape(-1)
    tok = np.repeat(np.arange(T), K)
    order = np.lexsort((tok, flat))                     # primary: expert, secondary: token
    np.testing.assert_array_equal(pm["perm"], order)
    np.testing.assert_array_equal(pm["counts"], np.bincount(flat, minlength=E))
    np.testing.assert_array_equal(pm["offsets"], np.concatenate([[0], np.cumsum(np.bincount(flat, minlength=E))]))
    for p, j in enumerate(pm["perm"]):
        assert pm["inv"][j // K, j % K] == p


# ----------------------------------------------------------------------------- experts

def test_silu_closed_forms():
    assert R.silu(0.0) == 0.0
    np.testing.assert_allclose(R.silu(math.log(3)), 0.75 * math.log(3), rtol=1e-15)
    np.testing.assert_allclose(R.silu(-math.log(3)), -0.25 * math.log(3), rtol=1e-15)


def test_swiglu_mlp_closed_form():
    H, I = 128, 128
    x = np.zeros((1, H))
    x[0, 0] = math.log(3)
    Wg = np.zeros((I, H)); Wg[0, 0] = 1.0
    Wu = np.zeros((I, H)); Wu[0, 0] = 2.0
    Wd = np.zeros((H, I)); Wd[7, 0] = -1.0          # output lands in column 7: catches a transposed W_down
    out = R.swiglu_mlp(x, Wg, Wu, Wd, rotated=False)["out"]
    want = np.zeros((1, H)); want[0, 7] = -1.5 * math.log(3) ** 2
    np.testing.assert_allclose(out, want, atol=1e-15)


def test_rotated_storage_equals_unrotated_weights():
    # The int4 codes store W * blockdiag(Hn); rotating x and h with the same normalised Hn must
    # reproduce the plain MLP of the unrotated W, because Hn * Hn = I.
    rng = np.random.default_rng(14)
    H, I = 256, 256
    W_g, W_u = rng.standard_normal((I, H)) * 0.05, rng.standard_normal((I, H)) * 0.05
    W_d = rng.standard_normal((H, I)) * 0.05
    x = rng.standard_normal((5, H))
    stored = [R.rotate_segments(W) for W in (W_g, W_u, W_d)]       # W @ blockdiag(Hn), Hn symmetric
    a = R.swiglu_mlp(x, *stored, rotated=True)["out"]
    b = R.swiglu_mlp(x, W_g, W_u, W_d, rotated=False)["out"]
    np.testing.assert_allclose(a, b, rtol=1e-12, atol=1e-12)
    # and skipping either rotation breaks it
    xr = R.rotate_segments(x)
    g = xr @ stored[0].T
    u = xr @ stored[1].T
    wrong = (R.silu(g) * u) @ stored[2].T
    assert np.abs(wrong - b).max() > 1e-3


# ----------------------------------------------------------------------------- whole layer

def test_identical_experts_reduce_to_one_mlp():
    L = _small_layer(E=8)
    rng = np.random.default_rng(15)
    W = [rng.standard_normal((128, 256)) * 0.05, rng.standard_normal((128, 256)) * 0.05,
         rng.standard_normal((256, 128)) * 0.05]
    x = S.make_x(9, H=256)
    out = R.moe_forward(L, x, expert_override=lambda e: W)
    xf = R.bf16_to_f64(x)
    mlp = R.swiglu_mlp(xf, *W, rotated=True)["out"]
    Sg, Su, Sd = R.shared_weights(L)
    shared = R.swiglu_mlp(xf, Sg, Su, Sd, rotated=False)["out"]
    np.testing.assert_allclose(out["y"], mlp + shared, rtol=1e-12, atol=1e-12)


def test_zero_experts_leave_the_shared_expert():
    L = _small_layer(E=8)
    x = S.make_x(4, H=256)
    Z = [np.zeros((128, 256)), np.zeros((128, 256)), np.zeros((256, 128))]
    out = R.moe_forward(L, x, expert_override=lambda e: Z)
    xf = R.bf16_to_f64(x)
    # shared expert by hand, with the un-fused halves of the gate|up bank
    Sgu = R.bf16_to_f64(L["sh_gu"])
    g, u = xf @ Sgu[:64].T, xf @ Sgu[64:].T
    want = (g / (1 + np.exp(-g)) * u) @ R.bf16_to_f64(L["sh_dn"]).T
    np.testing.assert_allclose(out["y"], want, rtol=1e-12, atol=1e-14)


def test_top1_layer_is_that_expert_plus_shared():
    L = _small_layer(E=8)
    x = S.make_x(6, H=256)
    out = R.moe_forward(L, x, top_k=1)
    xf = R.bf16_to_f64(x)
    Sg, Su, Sd = R.shared_weights(L)
    for t in range(6):
        e = out["ids"][t, 0]
        assert out["w"][t, 0] == 1.0
        mlp = R.swiglu_mlp(xf[t:t + 1], *R.expert_weights(L, e), rotated=True)["out"][0]
        sh = R.swiglu_mlp(xf[t:t + 1], Sg, Su, Sd, rotated=False)["out"][0]
        np.testing.assert_allclose(out["y"][t], mlp + sh, rtol=1e-12, atol=1e-14)


def test_token_order_equivariance_and_expert_relabeling():
    L = _small_layer(E=8)
    x = S.make_x(10, H=256)
    base = R.moe_forward(L, x)
    p = np.random.default_rng(16).permutation(10)
    np.testing.assert_allclose(R.moe_forward(L, x[p])["y"], base["y"][p], rtol=1e-13, atol=1e-15)
    # relabel experts: permute router rows and expert banks together
    q = np.random.default_rng(17).permutation(8)
    L2 = dict(L)
    for k in ("router_w", "gu_codes", "gu_scales", "dn_codes", "dn_scales"):
        L2[k] = L[k][q]
    np.testing.assert_allclose(R.moe_forward(L2, x)["y"], base["y"], rtol=1e-13, atol=1e-15)


def test_nvfp4_layer_uses_no_rotation():
    L = _small_layer(E=8, fmt="nvfp4")
    x = S.make_x(3, H=256)
    out = R.moe_forward(L, x, keep=True)
    np.testing.assert_allclose(out["x_in"][0], R.bf16_to_f64(x)[out["perm"][0] // 6], rtol=0, atol=0)


def test_redraw_tables_leave_no_near_tie():
    for E in (32, 256):
        L = S.make_layer(E, H=2048, I=128, Is=8)          # router rows do not depend on I / Is
        x = S.make_workload_x(2048 if E == 256 else 4096, E)
        assert R.router_gap(L, x).min() >= 1e-4


def test_rmsnorm_closed_forms():
    # a constant row c has mean square c^2: every element becomes c / sqrt(c^2 + eps)
    eps = 1e-6
    for c in (-3.0, 0.5, 7.25):
        row = np.full((1, 2048), c)
        np.testing.assert_allclose(R.rmsnorm(row, eps), c / math.sqrt(c * c + eps), rtol=1e-15)
    # the two-element row (3, 4): mean square 12.5
    np.testing.assert_allclose(R.rmsnorm(np.array([[3.0, 4.0]]), 0.0), [[3 / math.sqrt(12.5), 4 / math.sqrt(12.5)]])
    # without eps the result has unit mean square and is invariant to positive scaling, odd in x
    rng = np.random.default_rng(5)
    x = rng.standard_normal((4, 2048))
    z = R.rmsnorm(x, 0.0)
    np.testing.assert_allclose(np.mean(z * z, axis=-1), 1.0, rtol=1e-12)
    np.testing.assert_allclose(R.rmsnorm(37.5 * x, 0.0), z, rtol=1e-12)
    np.testing.assert_allclose(R.rmsnorm(-x, 0.0), -z, rtol=1e-12)


def test_f64_to_bf16_rounding_matches_torch():
    torch = pytest.importorskip("torch")
    rng = np.random.default_rng(6)
    x = np.concatenate([rng.standard_normal(20000) * 10.0 ** rng.integers(-6, 6, 20000),
                        [0.0, -0.0, 1.0, 1.00390625, 1.0 + 2.0 ** -8, 1.0 + 3 * 2.0 ** -9]])
    ref = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    np.testing.assert_array_equal(R.f64_to_bf16_bits(x), ref)


@pytest.mark.parametrize("top_k", [2, 3])
def test_combine_pairs_each_weight_with_its_own_expert(top_k):
    """The weighted combine, recomputed without the oracle's routing, permutation or rotation: a toy
    int4 layer (E = 4, H = 256, I = 128) whose four experts differ, routed by brute force over every
    k-subset, weighted through an explicit [T][E] routing matrix and summed by einsum. A weight paired
    with the wrong slot (for example weights left in score order while the ids are sorted by id)
    changes y here, because the experts and the weights all differ (midagedev/bloomery issue #632:
    unbiased sigmoid top-k with the SelectedSumFloor; NInfer README, "What is inside": scores
    renormalised)."""
    scipy_linalg = pytest.importorskip("scipy.linalg")
    E, H, I, Is, T = 4, 256, 128, 64, 24
    L = S.make_layer(E, "int4", H=H, I=I, Is=Is, seed=21)
    x_bits = S.make_x(T, H=H)
    out = R.moe_forward(L, x_bits, top_k=top_k)

    x = (x_bits.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    # unrotated fp64 weights: the stored W_q times blockdiag(Hs), Hs from scipy's Sylvester matrix
    Hs = scipy_linalg.hadamard(128) / math.sqrt(128)

    def unrotate(Wq):
        return np.concatenate([Wq[:, 128 * j:128 * (j + 1)] @ Hs for j in range(Wq.shape[1] // 128)], axis=1)

    Wg = np.stack([unrotate(R.dequant_int4(L["gu_codes"][e, :I], L["gu_scales"][e, :I])) for e in range(E)])
    Wu = np.stack([unrotate(R.dequant_int4(L["gu_codes"][e, I:], L["gu_scales"][e, I:])) for e in range(E)])
    Wd = np.stack([unrotate(R.dequant_int4(L["dn_codes"][e], L["dn_scales"][e])) for e in range(E)])

    # brute-force routing: the k-subset whose every score beats every score outside it
    logits = x @ ((L["router_w"].astype(np.uint32) << 16).view(np.float32).astype(np.float64)).T
    s = 1.0 / (1.0 + np.exp(-logits))
    Rm = np.zeros((T, E))
    for t in range(T):
        sel = [c for c in itertools.combinations(range(E), top_k)
               if min(s[t, list(c)]) > max(s[t, [e for e in range(E) if e not in c]])]
        assert len(sel) == 1
        c = list(sel[0])
        Rm[t, c] = s[t, c] / max(s[t, c].sum(), 2.0 ** -14)
        # the oracle's slot k carries the weight of the expert in slot k
        np.testing.assert_array_equal(out["ids"][t], sorted(c))
        np.testing.assert_allclose(out["w"][t], Rm[t, out["ids"][t]], rtol=1e-14)
    assert np.all(np.abs(np.diff(np.sort(Rm, axis=1), axis=1))[:, -top_k + 1:] > 1e-6)   # weights differ

    silu = lambda z: z / (1.0 + np.exp(-z))  # noqa: E731
    G = np.einsum("eih,th->eti", Wg, x)
    U = np.einsum("eih,th->eti", Wu, x)
    O = np.einsum("ehi,eti->eth", Wd, silu(G) * U)
    routed = np.einsum("te,eth->th", Rm, O)
    Sgu = (L["sh_gu"].astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    Sdn = (L["sh_dn"].astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    shared = (silu(x @ Sgu[:Is].T) * (x @ Sgu[Is:].T)) @ Sdn.T
    np.testing.assert_allclose(out["y"], routed + shared, rtol=1e-11, atol=1e-13)
    # the experts differ enough that pairing a weight with a neighbouring slot is visible
    assert np.abs(O[0] - O[1]).max() > 1e-3


def test_stack_step_residual_identities():
    """x_next = x + layer(bf16(rmsnorm(x))): a layer whose weights are all zero leaves the residual exactly
    as it was; with eps = 0 the normalised input, and so the layer output, is the same for x and for any
    positive multiple of x (closed forms of the residual + RMSNorm glue between stacked layers)."""
    L = _small_layer(E=8)
    Lz = dict(L)
    for k in ("gu_codes", "dn_codes", "sh_gu", "sh_dn"):
        Lz[k] = np.zeros_like(L[k])
    rng = np.random.default_rng(9)
    x = rng.standard_normal((5, 256)) * 1.26
    st = R.stack_step(Lz, x)
    np.testing.assert_array_equal(st["y"], 0.0)
    np.testing.assert_array_equal(st["x_next"], x)
    a = R.stack_step(L, x, eps=0.0)
    b = R.stack_step(L, 8.0 * x, eps=0.0)     # a power of two keeps rmsnorm's fp64 result bit-identical
    np.testing.assert_array_equal(a["z"], b["z"])
    np.testing.assert_array_equal(a["y"], b["y"])
    np.testing.assert_array_equal(b["x_next"], 8.0 * x + a["y"])
    assert np.abs(a["y"]).max() > 0


def test_routed_scale_scales_only_the_routed_sum():
    """y = routed_scale * sum_k w_k o_k + shared: scale 0 leaves the shared expert alone, and the routed
    part is linear in the scale while the routing is untouched."""
    L = _small_layer(E=8)
    x = S.make_x(6, H=256)
    one = R.moe_forward(L, x)
    zero = R.moe_forward(L, x, routed_scale=0.0)
    half = R.moe_forward(L, x, routed_scale=0.5)
    np.testing.assert_array_equal(zero["y"], one["ys"])
    np.testing.assert_array_equal(half["ids"], one["ids"])
    np.testing.assert_allclose(half["y"] - half["ys"], 0.5 * (one["y"] - one["ys"]), rtol=1e-12, atol=1e-15)
    assert np.abs(one["y"] - one["ys"]).max() > 1e-3
