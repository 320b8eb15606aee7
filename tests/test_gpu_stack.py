"""Layer stack on the GPU (through the C ABI): the residual + RMSNorm glue kernel against the oracle,
every layer of a 3-layer stack against the oracle on the device's own layer inputs, and the native
stack entry point against the same sequence of public calls."""

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
from bit_routed_expert_sigmoid_b200.layer import FlintMoEStack, y_to_host_bits  # noqa: E402

EPS = 1e-6
H = 2048


def bf16_ulp_diff(a_bits: np.ndarray, b_bits: np.ndarray) -> np.ndarray:
    """Distance in bf16 ulps between two arrays of bf16 bit patterns of the same sign."""
    return np.abs(a_bits.astype(np.int32) - b_bits.astype(np.int32))


@pytest.mark.parametrize("with_y,with_z", [(True, True), (False, True), (True, False)])
def test_residual_rmsnorm_kernel(with_y, with_z):
    rng = np.random.default_rng(11)
    T = 37
    x0 = (rng.standard_normal((T, H)) * 10.0 ** rng.uniform(-2, 2, (T, 1))).astype(np.float32)
    yb = S.f32_to_bf16_bits(rng.standard_normal((T, H)).astype(np.float32))
    x = torch.from_numpy(x0).cuda()
    y = torch.from_numpy(yb.view(np.int16)).cuda() if with_y else None
    z = torch.empty((T, H), dtype=torch.int16, device="cuda") if with_z else None
    B.flint_residual_rmsnorm(x.data_ptr(), y.data_ptr() if with_y else 0, T, EPS, z.data_ptr() if with_z else 0, 0)
    torch.cuda.synchronize()
    x_ref = x0 + R.bf16_to_f64(yb).astype(np.float32) if with_y else x0     # one fp32 add per element
    np.testing.assert_array_equal(x.cpu().numpy(), x_ref)
    if with_z:
        z_ref = R.f64_to_bf16_bits(R.rmsnorm(x_ref.astype(np.float64), EPS))
        zd = z.cpu().numpy().view(np.uint16)
        d = bf16_ulp_diff(zd, z_ref)
        assert d.max() <= 1                        # the fp32 kernel and the fp64 oracle round alike,
        assert np.mean(d == 0) > 0.995             # except next to a rounding boundary


def test_stack_of_three_layers():
    E, T, n = 32, 8, 3
    layers = [S.make_layer(E, "int4", seed=1000 + l) for l in range(n)]
    x0 = R.bf16_to_f64(S.make_workload_x(T, E)).astype(np.float32)          # residual starts at the input
    st = FlintMoEStack(layers, t_max=T, eps=EPS)
    x = torch.from_numpy(x0.copy()).cuda()
    z = torch.empty((T, H), dtype=torch.int16, device="cuda")
    y = torch.empty((T, H), dtype=torch.bfloat16, device="cuda")
    for l, L in enumerate(layers):
        # the public calls the stack entry point makes: residual add + norm, then the layer
        B.flint_residual_rmsnorm(x.data_ptr(), y.data_ptr() if l else 0, T, EPS, z.data_ptr(), 0)
        B.flint_moe_forward(st.layers[l].handle, z.data_ptr(), T, y.data_ptr(), 0)
        torch.cuda.synchronize()
        z_bits = z.cpu().numpy().view(np.uint16)
        ref = R.moe_forward(L, z_bits)
        keep = ref["gap"] >= 1e-4                  # tokens whose top-6 is not a near tie
        assert keep.sum() >= T - 1
        stats = PT.compare_y(y_to_host_bits(y)[keep], ref["y"][keep])
        assert stats["finite"] and stats["violations"] == 0, (l, stats)
        ids = st.layers[l].routing(T)["ids"].cpu().numpy()
        np.testing.assert_array_equal(ids[keep], ref["ids"][keep])
    B.flint_residual_rmsnorm(x.data_ptr(), y.data_ptr(), T, EPS, 0, 0)
    # the native entry point runs the same kernels in the same order: bit-identical residual
    xs = torch.from_numpy(x0.copy()).cuda()
    st.forward(xs)
    torch.cuda.synchronize()
    assert torch.equal(xs, x)
    assert all(layer.error_word() == 0 for layer in st.layers)
    st.close()


def test_stack_rejects_bad_arguments():
    L = S.make_layer(32, "int4", seed=1000)
    st = FlintMoEStack([L], t_max=8)
    x = torch.zeros((16, H), dtype=torch.float32, device="cuda")
    with pytest.raises(B.FlintError):                                   # T above the layer's t_max
        B.flint_moe_stack_forward([st.layers[0].handle], x.data_ptr(), 16, EPS, st.z.data_ptr(), st.y.data_ptr(), 0)
    with pytest.raises(B.FlintError):                                   # z and y must differ
        B.flint_moe_stack_forward([st.layers[0].handle], x.data_ptr(), 8, EPS, st.z.data_ptr(), st.z.data_ptr(), 0)
    with pytest.raises(B.FlintError):                                   # eps must be positive
        B.flint_residual_rmsnorm(x.data_ptr(), 0, 8, 0.0, st.z.data_ptr(), 0)
    st.close()


def test_stack_of_four_full_layers_matches_the_oracle_chain():
    # four E = 256 int4 layers through the native stack entry point, against the oracle's own chain
    # x <- x + layer(bf16(rmsnorm(x))) in fp64 (each layer fed the oracle's residual, not the
    # device's): the residual after the last layer agrees within the sum of the layers' output
    # tolerances, and every layer picks the oracle's experts wherever its top-6 is not a near tie
    E, T, n = 256, 8, 4
    layers = [S.make_layer(E, "int4", seed=1000 + l) for l in range(n)]
    x0 = R.bf16_to_f64(S.make_workload_x(T, E)).astype(np.float32)
    st = FlintMoEStack(layers, t_max=T, eps=EPS)
    xs = torch.from_numpy(x0.copy()).cuda()
    st.forward(xs)
    torch.cuda.synchronize()
    x_ref = x0.astype(np.float64)
    tol = np.zeros((T, H))
    for l, L in enumerate(layers):
        step = R.stack_step(L, x_ref, eps=EPS)
        ref = R.moe_forward(L, step["z"])
        keep = ref["gap"] >= 1e-4
        assert keep.sum() >= T - 2
        ids = st.layers[l].routing(T)["ids"].cpu().numpy()
        np.testing.assert_array_equal(ids[keep], ref["ids"][keep])
        tol += PT.y_tolerance(step["y"])[1]
        x_ref = step["x_next"]
    err = np.abs(xs.cpu().numpy().astype(np.float64) - x_ref)
    assert np.all(err <= tol + 2.0 ** -20 * np.abs(x_ref)), float((err / tol).max())
    assert all(layer.error_word() == 0 for layer in st.layers)
    st.close()
