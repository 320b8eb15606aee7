"""Weight preparation on the GPU (through the C ABI) against the CPU oracle: codes, scales and tensor
scales bit for bit (every decision is fp32 in the same order on both sides), and a layer built from
the GPU's output running through the forward against the oracle."""

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


@pytest.mark.parametrize("rotate", [True, False])
@pytest.mark.parametrize("rows,cols", [(37, 2048), (300, 512)])
def test_int4_bit_exact(rows, cols, rotate):
    w = rows_with_structure(rows, cols, seed=rows + cols)
    codes, scales = gpu_int4(w, rotate)
    ref = Q.quantize_int4_g128(w, rotate=rotate)
    np.testing.assert_array_equal(scales, ref["scales"])
    np.testing.assert_array_equal(codes, ref["codes"])


@pytest.mark.parametrize("n,rows,cols", [(3, 64, 512), (2, 5, 2048)])
def test_nvfp4_bit_exact(n, rows, cols):
    w = np.stack([rows_with_structure(rows, cols, seed=11 * i + cols) for i in range(n)])
    w[-1] = 0                                                             # an all-zero Linear
    codes, scales, ts = gpu_nvfp4(w)
    for i in range(n):
        ref = Q.quantize_nvfp4(w[i])
        assert ts[i] == ref["tscale"], i
        np.testing.assert_array_equal(scales[i], ref["scales"])
        np.testing.assert_array_equal(codes[i], ref["codes"])


@pytest.mark.parametrize("fmt", ["int4", "nvfp4"])
def test_layer_from_quantised_weights(fmt):
    # bf16 master weights of E = 32 experts -> the GPU quantiser -> a layer; its forward agrees with the
    # oracle's forward on the oracle-quantised weights (which are the same codes, checked first)
    E, I, H = 32, 512, 2048
    m = S.make_master_weights(E, outliers=2)
    L = dict(S.make_layer(E, fmt))
    if fmt == "int4":
        gc, gs = gpu_int4(m["gu"], True)
        dc, ds = gpu_int4(m["dn"], True)
        rg = Q.quantize_int4_g128(m["gu"].reshape(-1, H), rotate=True)
        rd = Q.quantize_int4_g128(m["dn"].reshape(-1, I), rotate=True)
        np.testing.assert_array_equal(gc, rg["codes"])
        np.testing.assert_array_equal(dc, rd["codes"])
        L.update(gu_codes=gc.reshape(E, 2 * I, H // 2), gu_scales=gs.reshape(E, 2 * I, H // 128),
                 dn_codes=dc.reshape(E, H, I // 2), dn_scales=ds.reshape(E, H, I // 128))
    else:
        gc, gs, gt = gpu_nvfp4(m["gu"].reshape(2 * E, I, H))
        dc, ds, dt = gpu_nvfp4(m["dn"])
        for i in (0, 1, 2 * E - 1):
            np.testing.assert_array_equal(gc[i], Q.quantize_nvfp4(m["gu"].reshape(2 * E, I, H)[i])["codes"])
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
