"""Weight preparation on the GPU (through the C ABI) against the CPU oracle, which rounds the exact fp64
quantities to nearest: codes, scales and tensor scales equal everywhere except where the exact value
lies within the kernels' fp32 error of a rounding boundary (counted, bounded, and there off by one
step at most), and a layer built from the GPU's output running through the forward against the
oracle."""

import numpy as np
import pytest

from bit_routed_expert_sigmoid_b200 import synthetic as S
from oracle import flint_moe_ref as R
from oracle import quant_ref as Q
from tests import parity as PT

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():  # collected on CPU-only machines, skipped there
    pytest.skip("no CUDA device", allow_module_level=True)

from bit_routed_expert_sigmoid_b200 import binding as B  # noqa: E402
from bit_routed_expert_sigmoid_b200.layer import FlintMoELayer, x_to_device, y_to_host_bits  # noqa: E402


def dev_u16(a):
    return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).cuda()


def gpu_int4(w, rotate):
    rows, cols = w.shape[0] * (w.shape[1] if w.ndim == 3 else 1), w.shape[-1]
    wd = dev_u16(w.reshape(rows, cols))
    codes = torch.empty((rows, cols // 2), dtype=torch.uint8, device="cuda")
    scales = torch.empty((rows, cols // 128), dtype=torch.int16, device="cuda")
    B.flint_quantize_int4_g128(wd.data_ptr(), rows, cols, rotate, codes.data_ptr(), scales.data_ptr(), 0)
    torch.cuda.synchronize()
    return codes.cpu().numpy(), scales.cpu().numpy().view(np.uint16)


def gpu_nvfp4(w):
    n, rows, cols = w.shape
    wd = dev_u16(w)
    codes = torch.empty((n, rows, cols // 2), dtype=torch.uint8, device="cuda")
    scales = torch.empty((n, rows, cols // 16), dtype=torch.uint8, device="cuda")
    ts = torch.empty((n,), dtype=torch.float32, device="cuda")
    B.flint_quantize_nvfp4(wd.data_ptr(), n, rows, cols, codes.data_ptr(), scales.data_ptr(), ts.data_ptr(), 0)
    torch.cuda.synchronize()
    return codes.cpu().numpy(), scales.cpu().numpy(), ts.cpu().numpy()


def rows_with_structure(rows, cols, seed):
    # normal rows with outliers, an all-zero group, a row of exact ties and a range of magnitudes
    rng = np.random.default_rng(seed)
    w = rng.standard_normal((rows, cols)) * np.exp2(rng.uniform(-10, 3, (rows, 1)))
    idx = rng.integers(0, cols, (rows, 4))
    np.put_along_axis(w, idx, rng.choice([-40.0, 40.0], idx.shape) * np.abs(w).mean(1, keepdims=True), axis=1)
    w[1, 128:256] = 0.0
    w[2] = np.where(np.arange(cols) % 2, 0.75, -0.75)
    return S.f32_to_bf16_bits(w.astype(np.float32))


def check_int4(w, rotate, codes, scales):
    """GPU int4 codes and scales against the fp64 oracle. The kernels rotate in fp32 (seven butterfly
    stages and a multiplication by fp32 2^-3.5: error at most 10 * 2^-24 of the segment's L1 norm over
    sqrt(128)) and divide as one fp32 product with a rounded reciprocal (2^-22 relative); a decision
    whose exact value is closer than that to its boundary may go either way."""
    ref = Q.quantize_int4_g128(w, rotate=rotate)
    mg = Q.int4_margins(w, rotate=rotate)
    wf = R.bf16_to_f64(w)
    N, K = wf.shape
    l1 = np.abs(wf).reshape(N, K // 128, 128).sum(-1)
    err_r = 10 * 2.0 ** -24 * l1 / np.sqrt(128) if rotate else np.zeros_like(l1)
    m = np.abs(ref["rotated"]).reshape(N, K // 128, 128).max(-1)
    s = R.bf16_to_f64(ref["scales"])
    with np.errstate(divide="ignore", invalid="ignore"):
        amb_g = mg["scale"] < np.where(m > 0, err_r / m, 0) + 2.0 ** -22
        tol = np.repeat(np.where(s > 0, err_r / s, 0), 128, axis=1) + 2.0 ** -21 * np.abs(mg["ratio"]) + 2.0 ** -40
    amb_e = (mg["code"] < tol) | np.repeat(amb_g, 128, axis=1)
    sd = np.abs(scales.astype(np.int64) - ref["scales"].astype(np.int64))
    assert np.all(sd[~amb_g] == 0) and np.all(sd <= 1)
    cg, cr = R.int4_values(codes), R.int4_values(ref["codes"])
    assert np.all(cg[~amb_e] == cr[~amb_e])
    assert np.all(np.abs(cg - cr)[~np.repeat(amb_g, 128, axis=1)] <= 1)
    # exact ties (the exact quotient is a half-integer) may go either way under any fp32 arithmetic;
    # the other ambiguous positions are counted and bounded, so that the comparison covers at least
    # 95 % of the codes (bf16 weights put many quotients within a few fp32 ulps of a boundary: the
    # test matrices hold rows of ties on purpose, and random bf16 weights give ~1e-3 of them)
    ties = mg["code"] == 0
    n_near = int((amb_e & ~ties).sum())
    assert n_near <= max(16, 0.05 * amb_e.size), n_near
    return {"exact_ties": int(ties.sum()), "near_boundary": n_near, "ambiguous_groups": int(amb_g.sum()),
            "differing_codes": int((cg != cr).sum())}


def check_nvfp4(w, codes, scales, ts):
    """GPU NVFP4 codes, block scales and tensor scale against the fp64 oracle. The kernels form 6 ts,
    the block quotient, d = sb ts and 1/d in fp32, each within 2^-24 relative; decisions closer than
    2^-22 (block scales: two roundings) or 2^-21 (codes: three) to their boundary may go either way."""
    ref = Q.quantize_nvfp4(w)
    mg = Q.nvfp4_margins(w)
    assert ts == ref["tscale"]
    amb_b = mg["scale"] < 2.0 ** -22
    amb_e = (mg["code"] < 2.0 ** -21) | np.repeat(amb_b, 16, axis=1)
    assert np.all(scales[~amb_b] == ref["scales"][~amb_b])
    vg = R.e2m1_to_f64(R.unpack_nibbles(codes))
    vr = R.e2m1_to_f64(R.unpack_nibbles(ref["codes"]))
    assert np.all(vg[~amb_e] == vr[~amb_e])
    ties = mg["code"] == 0
    n_near = int((amb_e & ~ties).sum())
    assert n_near <= max(16, 0.05 * amb_e.size), n_near
    return {"exact_ties": int(ties.sum()), "near_boundary": n_near, "ambiguous_blocks": int(amb_b.sum()),
            "differing_codes": int((vg != vr).sum())}


@pytest.mark.parametrize("rotate", [True, False])
@pytest.mark.parametrize("rows,cols", [(37, 2048), (300, 512)])
def test_int4_matches_round_to_nearest(rows, cols, rotate):
    w = rows_with_structure(rows, cols, seed=rows + cols)
    codes, scales = gpu_int4(w, rotate)
    st = check_int4(w, rotate, codes, scales)
    print("int4", rows, cols, rotate, st)


@pytest.mark.parametrize("n,rows,cols", [(3, 64, 512), (2, 5, 2048)])
def test_nvfp4_matches_round_to_nearest(n, rows, cols):
    w = np.stack([rows_with_structure(rows, cols, seed=11 * i + cols) for i in range(n)])
    w[-1] = 0                                                             # an all-zero Linear
    codes, scales, ts = gpu_nvfp4(w)
    for i in range(n):
        st = check_nvfp4(w[i], codes[i], scales[i], ts[i])
        print("nvfp4", i, rows, cols, st)


@pytest.mark.parametrize("fmt", ["int4", "nvfp4"])
def test_layer_from_quantised_weights(fmt):
    # bf16 master weights of E = 32 experts -> the GPU quantiser -> a layer; its forward agrees with the
    # oracle's forward on the GPU-quantised weights (whose codes are checked against round-to-nearest first)
    E, I, H = 32, 512, 2048
    m = S.make_master_weights(E, outliers=2)
    L = dict(S.make_layer(E, fmt))
    if fmt == "int4":
        gc, gs = gpu_int4(m["gu"], True)
        dc, ds = gpu_int4(m["dn"], True)
        check_int4(m["gu"][:2].reshape(-1, H), True, gc[:4 * I], gs[:4 * I])
        check_int4(m["dn"][:2].reshape(-1, I), True, dc[:2 * H], ds[:2 * H])
        L.update(gu_codes=gc.reshape(E, 2 * I, H // 2), gu_scales=gs.reshape(E, 2 * I, H // 128),
                 dn_codes=dc.reshape(E, H, I // 2), dn_scales=ds.reshape(E, H, I // 128))
    else:
        gc, gs, gt = gpu_nvfp4(m["gu"].reshape(2 * E, I, H))
        dc, ds, dt = gpu_nvfp4(m["dn"])
        for i in (0, 1, 2 * E - 1):
            check_nvfp4(m["gu"].reshape(2 * E, I, H)[i], gc[i], gs[i], gt[i])
        L.update(gu_codes=gc.reshape(E, 2 * I, H // 2), gu_scales=gs.reshape(E, 2 * I, H // 16),
                 gu_tscale=gt.reshape(E, 2), dn_codes=dc, dn_scales=ds, dn_tscale=dt)
    # the quantised weights reproduce the master weights up to the formats' rounding
    g, u, d = R.expert_weights(L, 3)
    master = R.bf16_to_f64(m["gu"][3, :I])
    back = R.rotate_segments(g) if fmt == "int4" else g
    assert np.linalg.norm(back - master) / np.linalg.norm(master) < 0.15
    for T in (8, 40):
        x = S.make_workload_x(T, E)
        ref = R.moe_forward(L, x)
        keep = ref["gap"] >= 1e-4
        dev = FlintMoELayer(L, t_max=T)
        y = dev.forward(x_to_device(x))
        torch.cuda.synchronize()
        np.testing.assert_array_equal(dev.routing(T)["ids"].cpu().numpy()[keep], ref["ids"][keep])
        st = PT.compare_y(y_to_host_bits(y)[keep], ref["y"][keep])
        assert st["finite"] and st["violations"] == 0, (T, st)
        assert dev.error_word() == 0
        dev.close()


def test_quantise_rejects_bad_arguments():
    w = torch.zeros((4, 256), dtype=torch.int16, device="cuda")
    c = torch.zeros((4, 128), dtype=torch.uint8, device="cuda")
    s = torch.zeros((4, 16), dtype=torch.int16, device="cuda")
    with pytest.raises(B.FlintError):
        B.flint_quantize_int4_g128(w.data_ptr(), 4, 200, True, c.data_ptr(), s.data_ptr(), 0)   # cols % 128
    with pytest.raises(B.FlintError):
        B.flint_quantize_nvfp4(w.data_ptr() + 2, 1, 4, 256, c.data_ptr(), s.data_ptr(), s.data_ptr(), 0)  # w unaligned
