"""W4A4 prefill (NVFP4 weights; the routed experts' inputs x and h quantised to NVFP4 per row; the
routed projections as block-scaled FP4 MMAs) against the oracle, stage by stage on the device's own
inputs, then end to end:

* activation quantiser: bit-exact (codes, E4M3 block scales, fp32 tensor scales) against the oracle's
  quantiser on the same fp32 rows: x (bf16 -> fp32 is exact) and the device's own h
* gate|up: the device's h against silu(g) u from the device's quantised x and the dequantised
  weights, in fp64; the fp32 accumulation is bounded by (terms) x 2^-24 x sum |x||w| (recursive
  summation), the fast silu by a few ulp
* down: the device's o against (device's quantised h) @ W_down^T in fp64, plus half an fp16 ulp
* end to end: y against the oracle's W4A4 layer with the layer's output tolerance; the oracle
  quantises h from fp64 while the device quantises its fp32 h, so a code may differ where h lies
  within fp32 rounding of a rounding boundary
"""

import numpy as np
import pytest

from bit_routed_expert_sigmoid_b200 import synthetic as S
from oracle import flint_moe_ref as R
from tests import parity as PT

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():
    pytest.skip("no CUDA device", allow_module_level=True)

from bit_routed_expert_sigmoid_b200 import binding as B  # noqa: E402
from bit_routed_expert_sigmoid_b200.layer import FlintMoELayer, x_to_device, y_to_host_bits  # noqa: E402

K = 6
_LAYERS = {}


def layer(E, skew=False):
    if (E, skew) not in _LAYERS:
        _LAYERS[(E, skew)] = S.make_layer(E, "nvfp4", skew=skew)
    return _LAYERS[(E, skew)]


def run(L, x_bits, t_max=None):
    T = x_bits.shape[0]
    dev = FlintMoELayer(L, t_max=t_max or T, top_k=K, flags=B.FLINT_FLAG_W4A4)
    y = dev.forward(x_to_device(x_bits))
    torch.cuda.synchronize()
    assert dev.error_word() == 0
    return dev, y


def fetch(dev, T):
    names = {"xa": B.FLINT_BUF_XA, "xa_sf": B.FLINT_BUF_XA_SF, "xa_ts": B.FLINT_BUF_XA_TS, "h": B.FLINT_BUF_H,
             "ha": B.FLINT_BUF_HA, "ha_sf": B.FLINT_BUF_HA_SF, "ha_ts": B.FLINT_BUF_HA_TS, "o": B.FLINT_BUF_O}
    out = {k: dev.intermediate(v, T).cpu().numpy() for k, v in names.items()}
    r = dev.routing(T)
    out["perm"] = r["perm"].cpu().numpy()
    out["offsets"] = r["offsets"].cpu().numpy()
    return out


def values(codes, sf, ts):
    """NVFP4 rows -> fp64 (e2m1 x E4M3 x tensor scale)."""
    return (R.e2m1_to_f64(R.unpack_nibbles(codes)) * np.repeat(R.e4m3fn_to_f64(sf), 16, axis=1)
            * ts.astype(np.float64)[:, None])


def check_quantiser(src_f32, codes, sf, ts, rows):
    q = R.quantize_act_nvfp4(src_f32[rows])
    np.testing.assert_array_equal(ts[rows], q["ts"])
    np.testing.assert_array_equal(sf[rows], q["scales"])
    np.testing.assert_array_equal(R.unpack_nibbles(codes[rows]), q["codes"])


def check_stages(L, x_bits, d, experts):
    """Quantisers on every permuted row; the two projections on the rows of `experts`."""
    P = d["perm"].shape[0]
    tok = d["perm"] // K
    x32 = R.bf16_to_f64(x_bits).astype(np.float32)
    allr = np.arange(P)
    check_quantiser(x32[tok], d["xa"], d["xa_sf"], d["xa_ts"], allr)
    check_quantiser(d["h"], d["ha"], d["ha_sf"], d["ha_ts"], allr)
    xv = values(d["xa"], d["xa_sf"], d["xa_ts"])
    hv = values(d["ha"], d["ha_sf"], d["ha_ts"])
    eps32 = 2.0 ** -24
    n_checked = 0
    for e in experts:
        lo, hi = int(d["offsets"][e]), int(d["offsets"][e + 1])
        if lo == hi:
            continue
        Wg, Wu, Wd = R.expert_weights(L, e)
        g, u = xv[lo:hi] @ Wg.T, xv[lo:hi] @ Wu.T
        ag, au = np.abs(xv[lo:hi]) @ np.abs(Wg).T, np.abs(xv[lo:hi]) @ np.abs(Wu).T
        sg = R.silu(g)
        h_ref = sg * u
        tol = (L["H"] * eps32) * (1.1 * np.abs(u) * ag + np.abs(sg) * au) + 1e-5 * np.abs(h_ref) + 1e-30
        err = np.abs(d["h"][lo:hi] - h_ref)
        assert np.all(err <= tol), (e, float(np.max(err / tol)))
        # typical error far inside the bound: a misplaced block scale would show here first
        assert np.sqrt(np.mean(err ** 2)) <= 1e-5 * np.sqrt(np.mean(h_ref ** 2)) + 1e-30, e
        o_ref = hv[lo:hi] @ Wd.T
        ao = np.abs(hv[lo:hi]) @ np.abs(Wd).T
        half_ulp = np.abs(o_ref) * 2.0 ** -11 + 2.0 ** -25
        err = np.abs(d["o"][lo:hi].astype(np.float64) - o_ref)
        assert np.all(err <= half_ulp + (L["I"] * eps32) * ao * 1.01), (e, float(np.max(err - half_ulp)))
        n_checked += hi - lo
    return n_checked


def test_w4a4_small_layer_all_stages_and_output():
    # E=32, T=100: ~19 rows per expert (single ragged chunks); token 3 has four all-zero 16-blocks
    # (block scale 0: codes carry the sign only)
    L = layer(32)
    x = S.make_workload_x(100, 32)
    x[3, :64] = 0
    dev, y = run(L, x)
    d = fetch(dev, 100)
    assert check_stages(L, x, d, range(32)) == 600
    assert np.all(d["xa_sf"][np.nonzero(d["perm"] // K == 3)[0], :4] == 0)
    ref = R.moe_forward(L, x, top_k=K, w4a4=True)
    PT.check_routing(dev.routing(100), ref, 100, K)
    st = PT.compare_y(y_to_host_bits(y), ref["y"])
    assert st["finite"] and st["violations"] == 0, st
    # W4A4 differs from the 16-bit-activation layer (the quantisation is really applied)
    ref16 = R.moe_forward(L, x, top_k=K)
    assert np.max(np.abs(ref["y"] - ref16["y"])) > 10 * PT.y_tolerance(ref["y"])[0]
    dev.close()


def test_w4a4_all_zero_token():
    # an all-zero token: tensor scale 1, zero codes and scales, a finite output; its routing is a tie
    # among all experts, so only the device's own permutation is used
    L = layer(32)
    x = S.make_workload_x(16, 32)
    x[5] = 0
    dev, y = run(L, x)
    d = fetch(dev, 16)
    rows = np.nonzero(d["perm"] // K == 5)[0]
    assert len(rows) == K
    assert np.all(d["xa_ts"][rows] == 1.0) and np.all(d["xa_sf"][rows] == 0) and np.all(d["xa"][rows] == 0)
    assert np.all(d["ha_ts"][rows] == 1.0) and np.all(d["ha"][rows] == 0)
    x32 = R.bf16_to_f64(x).astype(np.float32)
    check_quantiser(x32[d["perm"] // K], d["xa"], d["xa_sf"], d["xa_ts"], np.arange(16 * K))
    assert torch.isfinite(y.float()).all()
    dev.close()


def test_w4a4_multi_chunk_experts():
    # T=700 over E=32: every expert has two or three 64-row chunks, the last one ragged
    L = layer(32)
    T = 700
    x = S.make_workload_x(T, 32)
    dev, y = run(L, x)
    d = fetch(dev, T)
    counts = np.diff(d["offsets"])
    assert counts.max() > 128 and np.any((counts % 64) != 0)
    assert check_stages(L, x, d, range(32)) == T * K
    ref = R.moe_forward(L, x, top_k=K, w4a4=True)
    st = PT.compare_y(y_to_host_bits(y), ref["y"])
    assert st["finite"] and st["violations"] == 0, st
    dev.close()


def test_w4a4_full_size_workload_sampled():
    # E=256, T=2048 (the prefill workload, launch configuration of the benchmark): quantisers on every
    # row, projections on the largest and a spread of other experts, y on sampled tokens
    L = layer(256)
    T = 2048
    x = S.make_workload_x(T, 256)
    dev, y = run(L, x)
    d = fetch(dev, T)
    counts = np.diff(d["offsets"])
    experts = sorted({int(np.argmax(counts))} | set(range(0, 256, 37)))
    assert check_stages(L, x, d, experts) > 0
    sample = np.array([0, 1, 777, 1500, 2046, 2047])
    ref = R.moe_forward(L, x[sample], top_k=K, w4a4=True)
    st = PT.compare_y(y_to_host_bits(y)[sample], ref["y"])
    assert st["finite"] and st["violations"] == 0, st
    dev.close()


def test_w4a4_smallest_batch_in_a_larger_handle():
    # T = 9, the smallest batch of the tensor-core path (mostly one-row chunks), on a handle sized for
    # 300 tokens (chunk numbering and atom arrays larger than used)
    L = layer(256)
    T = 9
    x = S.make_workload_x(T, 256)
    dev, y = run(L, x, t_max=300)
    d = fetch(dev, T)
    active = np.nonzero(np.diff(d["offsets"]))[0]
    assert check_stages(L, x, d, active) == T * K
    ref = R.moe_forward(L, x, top_k=K, w4a4=True)
    PT.check_routing(dev.routing(T), ref, T, K)
    st = PT.compare_y(y_to_host_bits(y), ref["y"])
    assert st["finite"] and st["violations"] == 0, st
    dev.close()


def test_w4a4_skewed_loads_sampled():
    # skewed router (hot experts with up to ~800 rows: 13 chunks of 64, and idle experts): quantisers on
    # every row, projections of the hottest and of a few other experts, y on sampled tokens
    L = layer(256, skew=True)
    T = 2048
    x = S.make_workload_x(T, 256, skew=True)
    dev, y = run(L, x)
    d = fetch(dev, T)
    counts = np.diff(d["offsets"])
    assert counts.max() > 640 and (counts == 0).any()
    experts = sorted({int(np.argmax(counts))} | {int(e) for e in np.nonzero(counts)[0][::40]})
    assert check_stages(L, x, d, experts) > counts.max()
    sample = np.array([0, 5, 1024, 2047])
    ref = R.moe_forward(L, x[sample], top_k=K, w4a4=True)
    st = PT.compare_y(y_to_host_bits(y)[sample], ref["y"])
    assert st["finite"] and st["violations"] == 0, st
    dev.close()


def test_w4a4_is_deterministic():
    # repeated forwards agree bit for bit: y, and the gate|up output h before its quantisation
    L = layer(256)
    T = 200
    x = x_to_device(S.make_workload_x(T, 256))
    dev = FlintMoELayer(L, t_max=T, flags=B.FLINT_FLAG_W4A4)
    runs = []
    for _ in range(3):
        y = dev.forward(x).clone()
        runs.append((y.view(torch.int16), dev.intermediate(B.FLINT_BUF_H, T)))
    torch.cuda.synchronize()
    for y, h in runs[1:]:
        assert torch.equal(runs[0][0], y) and torch.equal(runs[0][1], h)
    dev.close()


def test_w4a4_leaves_decode_unchanged():
    # T <= 8 runs the decode kernel with 16-bit activations, with or without the flag
    L = layer(32)
    x = S.make_workload_x(5, 32)
    a = FlintMoELayer(L, t_max=5, flags=B.FLINT_FLAG_W4A4)
    b = FlintMoELayer(L, t_max=5)
    ya, yb = a.forward(x_to_device(x)), b.forward(x_to_device(x))
    torch.cuda.synchronize()
    assert torch.equal(ya, yb)
    a.close()
    b.close()


def test_w4a4_is_refused_for_int4():
    # the configuration check rejects it (no workspace size), so no handle can be made
    cfg = B.flint_moe_cfg(hidden=2048, n_experts=32, top_k=K, inter=512, inter_shared=1024,
                          fmt=B.FLINT_W_INT4_G128_FWHT128, t_max=16, routed_scale=1.0, norm_floor=2.0 ** -14,
                          flags=B.FLINT_FLAG_W4A4, n_slots=0)
    assert B.flint_moe_workspace_size(cfg) == 0
    cfg.fmt = B.FLINT_W_NVFP4
    assert B.flint_moe_workspace_size(cfg) > 0
