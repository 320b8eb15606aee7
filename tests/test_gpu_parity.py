"""Parity of the CUDA layer (through the C ABI) against the fp64 oracle on seeded workloads."""

import numpy as np
import pytest

from bit_routed_expert_sigmoid_b200 import synthetic as S
from oracle import flint_moe_ref as R
from tests import parity as PT

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():  # collected on CPU-only machines, skipped there
    pytest.skip("no CUDA device", allow_module_level=True)

from bit_routed_expert_sigmoid_b200 import binding as B  # noqa: E402
from bit_routed_expert_sigmoid_b200.layer import FlintMoELayer, x_to_device, y_to_host_bits  # noqa: E402

_LAYERS = {}


def layer(E, fmt, skew=False):
    key = (E, fmt, skew)
    if key not in _LAYERS:
        _LAYERS[key] = S.make_layer(E, fmt, skew=skew)
    return _LAYERS[key]


def run(L, x_bits, top_k=6, t_max=None, flags=0):
    T = x_bits.shape[0]
    dev = FlintMoELayer(L, t_max=t_max or T, top_k=top_k, flags=flags)
    xd = x_to_device(x_bits)
    y = dev.forward(xd)
    torch.cuda.synchronize()
    return dev, xd, y


def full_check(L, x_bits, top_k=6, keep=False):
    T = x_bits.shape[0]
    ref = R.moe_forward(L, x_bits, top_k=top_k, keep=keep)
    dev, xd, y = run(L, x_bits, top_k=top_k)
    PT.check_routing(dev.routing(T), ref, T, top_k)
    st = PT.compare_y(y_to_host_bits(y), ref["y"])
    assert st["finite"]
    assert st["violations"] == 0, st
    assert dev.error_word() == 0
    return dev, xd, y, ref, st


@pytest.mark.parametrize("fmt", ["int4", "nvfp4"])
def test_tiny_layer(fmt):
    # E=32 routed experts, T=8 tokens
    L = layer(32, fmt)
    x = S.make_workload_x(8, 32)
    full_check(L, x)


@pytest.mark.parametrize("T", [1, 2, 4, 8])
def test_decode_int4_full_layer(T):
    L = layer(256, "int4")
    full_check(L, S.make_workload_x(T, 256))


@pytest.mark.parametrize("T", [1, 8])
def test_decode_nvfp4_full_layer(T):
    L = layer(256, "nvfp4")
    full_check(L, S.make_workload_x(T, 256))


@pytest.mark.parametrize("fmt,T", [("int4", 9), ("nvfp4", 9), ("int4", 37), ("nvfp4", 37), ("int4", 300)])
def test_ragged_token_counts(fmt, T):
    # T = 9 is the smallest batch of the tensor-core path (one row per expert for most experts)
    L = layer(256, fmt)
    full_check(L, S.make_workload_x(T, 256))


def test_prefill_int4_full_size():
    L = layer(256, "int4")
    full_check(L, S.make_workload_x(2048, 256))


def test_prefill_int4_skewed_loads():
    L = layer(256, "int4", skew=True)
    x = S.make_workload_x(2048, 256, skew=True)
    dev, xd, y, ref, st = full_check(L, x)
    counts = np.diff(ref["offsets"])
    assert counts.max() > 300 and (counts == 0).any()          # skewed: hot and idle experts


def test_prefill_nvfp4_full_size():
    L = layer(256, "nvfp4")
    full_check(L, S.make_workload_x(2048, 256))


def test_permutation_spans_rounds():
    # T*K = 18000 (token, slot) pairs: 18 CTAs of the counting sort (1024 pairs each, the last one
    # ragged) and more than one round (16384 ids) of its histogram loop; the permutation is rebuilt
    # from the device's ids by the oracle
    L = layer(32, "int4")
    T = 3000
    x = S.make_workload_x(T, 32)
    dev, xd, y, ref, st = full_check(L, x)
    r = dev.routing(T)
    pr = R.permutation(r["ids"].cpu().numpy(), 32)
    np.testing.assert_array_equal(r["offsets"].cpu().numpy(), pr["offsets"])
    np.testing.assert_array_equal(r["perm"].cpu().numpy(), pr["perm"])


def test_top1_routing():
    L = layer(32, "int4")
    x = S.make_x(16)
    ref = R.moe_forward(L, x, top_k=1)
    keep = ref["gap"] >= 1e-4
    dev, xd, y = run(L, x, top_k=1)
    r = dev.routing(16)
    np.testing.assert_array_equal(r["ids"].cpu().numpy()[keep], ref["ids"][keep])
    np.testing.assert_array_equal(r["w"].cpu().numpy(), 1.0)
    st = PT.compare_y(y_to_host_bits(y)[keep], ref["y"][keep])
    assert st["violations"] == 0, st


def test_all_tokens_on_six_experts():
    # router column 0 strongly prefers experts 0..5, so each of them receives every token (several
    # token chunks per expert) and the other experts receive none
    L = dict(layer(256, "int4"))
    rw = L["router_w"].copy()
    rw[:, 0] = S.f32_to_bf16_bits(np.where(np.arange(256) < 6, 8.0, -8.0).astype(np.float32))
    L["router_w"] = rw
    x = S.make_x(64, skew=True)                                 # x[:, 0] = 1
    dev, xd, y, ref, st = full_check(L, x)
    np.testing.assert_array_equal(np.diff(ref["offsets"])[:6], 64)


@pytest.mark.parametrize("T", [8, 64])
def test_exact_tie_goes_to_lower_id(T):
    # router rows 9 and 12 are identical, so their logits are equal bit for bit on every path; with
    # experts 0..4 far above and the rest far below, the sixth pick is a tie between 9 and 12 for
    # every token and must go to the lower id (T = 8: decode kernels; T = 64: tensor-core router and
    # the top-k kernel of the prefill path)
    L = dict(layer(32, "int4"))
    rw = L["router_w"].copy()
    rw[12] = rw[9]
    col = np.full(32, -16.0, np.float32)
    col[:5] = 16.0
    col[9] = col[12] = 4.0
    rw[:, 0] = S.f32_to_bf16_bits(col)
    L["router_w"] = rw
    x = S.make_x(T, skew=True)                                  # x[:, 0] = 1
    ref = R.moe_forward(L, x)
    expect = np.tile(np.array([0, 1, 2, 3, 4, 9], np.int32), (T, 1))
    np.testing.assert_array_equal(ref["ids"], expect)
    assert np.all(ref["gap"] == 0.0)                            # the tie is exact in the oracle too
    dev, xd, y = run(L, x)
    np.testing.assert_array_equal(dev.routing(T)["ids"].cpu().numpy(), expect)
    st = PT.compare_y(y_to_host_bits(y), ref["y"])
    assert st["finite"] and st["violations"] == 0, st
    assert dev.error_word() == 0


def test_intermediates_router_logits_and_rotation():
    L = layer(256, "int4")
    T = 8
    x = S.make_workload_x(T, 256)
    ref = R.moe_forward(L, x, keep=True)
    dev, xd, y = run(L, x)
    logits = dev.intermediate(B.FLINT_BUF_LOGITS, T).cpu().numpy()
    np.testing.assert_allclose(logits, ref["logits"], rtol=0, atol=2e-5)
    xq = dev.intermediate(B.FLINT_BUF_XQ, T).cpu().numpy().astype(np.float64)
    xr = R.rotate_segments(R.bf16_to_f64(x))
    np.testing.assert_allclose(PT.xq_natural_order(xq, True), xr, rtol=2 ** -11, atol=1e-6)
    ys = dev.intermediate(B.FLINT_BUF_YS, T).cpu().numpy()
    np.testing.assert_allclose(ys, ref["ys"], rtol=1e-4, atol=1e-4 * np.abs(ref["ys"]).max())


@pytest.mark.parametrize("fmt,T", [("int4", 300), ("nvfp4", 37), ("nvfp4", 200), ("int4", 8), ("nvfp4", 8)])
def test_deterministic_across_runs(fmt, T):
    # every sum has a fixed order, so repeated forwards agree bit for bit (a race in a kernel shows here
    # as run-to-run differences, often before it breaks the tolerance)
    L = layer(256, fmt)
    x = S.make_workload_x(T, 256)
    dev = FlintMoELayer(L, t_max=T)
    xd = x_to_device(x)
    ys = [dev.forward(xd).clone() for _ in range(4)]
    torch.cuda.synchronize()
    for y in ys[1:]:
        assert torch.equal(ys[0].view(torch.int16), y.view(torch.int16))
    dev.close()


def test_forward_host_matches_device_forward():
    L = layer(256, "int4")
    T = 8
    x = S.make_workload_x(T, 256)
    dev = FlintMoELayer(L, t_max=T)
    y_dev = dev.forward(x_to_device(x))
    xh = torch.from_numpy(x.view(np.int16)).pin_memory()
    yh = torch.empty((T, 2048), dtype=torch.int16).pin_memory()
    dev.forward_host(xh, yh)
    torch.cuda.synchronize()
    assert torch.equal(yh, y_dev.view(torch.int16).cpu())


def test_argument_errors_on_device():
    L = layer(32, "int4")
    dev = FlintMoELayer(L, t_max=8)
    xd = x_to_device(S.make_x(8))
    y = torch.empty((8, 2048), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(B.FlintError) as e:
        B.flint_moe_forward(dev.handle, xd.data_ptr(), 9, y.data_ptr(), 0)
    assert e.value.status == B.FLINT_ERR_INVALID_ARG
    with pytest.raises(B.FlintError):
        B.flint_moe_forward(dev.handle, xd.data_ptr() + 2, 4, y.data_ptr(), 0)
    B.flint_moe_forward(dev.handle, xd.data_ptr(), 0, y.data_ptr(), 0)      # T = 0 is a no-op
    torch.cuda.synchronize()


def _logit_gap(L, x, top_k=6):
    """fp64 gap between the top_k-th and next logit of every token (the selection is unique above the
    fp32 error of the logits, ~1e-5 here)."""
    lg = np.sort(R.bf16_to_f64(x) @ R.bf16_to_f64(L["router_w"]).T, axis=1)[:, ::-1]
    return lg[:, top_k - 1] - lg[:, top_k]


@pytest.mark.parametrize("T", [8, 40])
def test_selected_sum_floor_is_applied(T):
    # every logit near -20 (x[:, 0] = 1 carries a per-expert bias in router column 0), so the six
    # selected sigmoid scores sum to ~1e-8, far below 2^-14: the weights are s / 2^-14, not s / sum
    # (midagedev/bloomery issue #632, host-policy comment: SelectedSumFloor); T = 8 takes the decode
    # kernel, T = 40 the tensor-core path
    L = dict(layer(32, "int4"))
    rw = L["router_w"].copy()
    rw[:, 0] = S.f32_to_bf16_bits((-18.0 - 0.375 * np.arange(32)).astype(np.float32))
    L["router_w"] = rw
    x = S.make_x(T, skew=True)
    ref = R.moe_forward(L, x)
    s_sel = np.take_along_axis(ref["scores"], ref["ids"].astype(np.int64), axis=1)
    assert np.all(s_sel.sum(axis=1) < 2.0 ** -14)
    np.testing.assert_allclose(ref["w"], s_sel / 2.0 ** -14, rtol=1e-12)
    keep = _logit_gap(L, x) >= 1e-3
    assert keep.sum() >= T // 2
    dev, xd, y = run(L, x)
    r = dev.routing(T)
    np.testing.assert_array_equal(r["ids"].cpu().numpy()[keep], ref["ids"][keep])
    # w = s / 2^-14 with s = sigmoid(logit) ~ e^logit: its relative error is the absolute error of the
    # fp32 logit (sums of 2048 exact products near -20, a few 2^-19)
    np.testing.assert_allclose(r["w"].cpu().numpy()[keep], ref["w"][keep], rtol=1e-4)
    assert float(r["w"].cpu().numpy().sum(axis=1).max()) < 0.1        # the floor, not a renormalisation to 1
    st = PT.compare_y(y_to_host_bits(y), ref["y"])
    assert st["finite"] and st["violations"] == 0, st
    assert dev.error_word() == 0


@pytest.mark.parametrize("fmt,T", [("int4", 8), ("nvfp4", 8), ("int4", 40), ("nvfp4", 40)])
def test_routed_scale_half(fmt, T):
    L = layer(32, fmt)
    x = S.make_workload_x(T, 32)
    ref = R.moe_forward(L, x, routed_scale=0.5)
    dev = FlintMoELayer(L, t_max=T, routed_scale=0.5)
    y = dev.forward(x_to_device(x))
    torch.cuda.synchronize()
    PT.check_routing(dev.routing(T), ref, T, 6)
    st = PT.compare_y(y_to_host_bits(y), ref["y"])
    assert st["finite"] and st["violations"] == 0, st
    # and it is not the scale-1 layer
    ref1 = R.moe_forward(L, x)
    assert np.abs(ref1["y"] - ref["y"]).max() > 0.1
    dev.close()


@pytest.mark.parametrize("T", [8, 300])
def test_debug_checks_stay_clear_on_a_valid_forward(T):
    # FLINT_FLAG_DEBUG_CHECKS turns on the device-side range checks of ids and offsets; on a valid
    # forward the error word stays 0 and the output is unchanged
    L = layer(256, "int4")
    x = S.make_workload_x(T, 256)
    ref = R.moe_forward(L, x)
    dev, xd, y = run(L, x, flags=B.FLINT_FLAG_DEBUG_CHECKS)
    PT.check_routing(dev.routing(T), ref, T, 6)
    st = PT.compare_y(y_to_host_bits(y), ref["y"])
    assert st["finite"] and st["violations"] == 0, st
    assert dev.error_word() == 0
    dev2, _, y2 = run(L, x)
    assert torch.equal(y.view(torch.int16), y2.view(torch.int16))


def test_decode_top8_most_active_experts():
    # top-8 at T = 8: 64 (token, slot) pairs, the most the decode kernel takes; ~57 distinct experts,
    # so four routed gate|up tiles per warp and nine phase-C items per warp on 148 SMs
    L = layer(256, "int4")
    x = S.make_x(8, redraws=S.redraw_table(256))
    ref = R.moe_forward(L, x, top_k=8)
    keep = ref["gap"] >= 1e-4
    dev, xd, y = run(L, x, top_k=8)
    r = dev.routing(8)
    np.testing.assert_array_equal(r["ids"].cpu().numpy()[keep], ref["ids"][keep])
    st = PT.compare_y(y_to_host_bits(y)[keep], ref["y"][keep])
    assert st["finite"] and st["violations"] == 0, st
    assert dev.error_word() == 0


def test_prefill_nvfp4_skewed_loads():
    L = layer(256, "nvfp4", skew=True)
    x = S.make_workload_x(2048, 256, skew=True)
    dev, xd, y, ref, st = full_check(L, x)
    counts = np.diff(ref["offsets"])
    assert counts.max() > 300 and (counts == 0).any()
