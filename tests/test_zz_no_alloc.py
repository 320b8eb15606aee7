"""flint_moe_route_noalloc: routing for callers that cannot allocate device memory (for example a
plug-in whose host owns the allocator). Its logits scratch is a fixed device array inside the library
instead of a caller workspace; its results must equal the
oracle's routing and the routing that flint_moe_forward produces through the existing entry points,
call after call (ids exactly, weights to fp32 rounding: the two entry points form the same fp32 logits
from exact bf16 products but sum them in different orders).

This file is collected last on purpose, so that a run stopping at its first failure has already run
every other test."""

import numpy as np
import pytest

from oracle import flint_moe_ref as R

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():
    pytest.skip("no CUDA device", allow_module_level=True)

from bit_routed_expert_sigmoid_b200 import binding as B  # noqa: E402
from bit_routed_expert_sigmoid_b200 import synthetic as S  # noqa: E402
from bit_routed_expert_sigmoid_b200.layer import FlintMoELayer, x_to_device  # noqa: E402


def test_noalloc_routing_matches_the_forward_routing_on_consecutive_calls():
    E, K = 256, 6
    L = S.make_layer(E, "int4")
    layer = FlintMoELayer(L, t_max=64)
    stream = torch.cuda.current_stream().cuda_stream
    redraws = S.redraw_table(E)
    # two calls in a row, different batches (the second one smaller than the first)
    for T, first in ((48, 0), (7, 100)):
        x = x_to_device(S.make_x(T, redraws=redraws, first_row=first))
        layer.forward(x)
        want = layer.routing(T)
        ids = torch.full((T, K), -1, dtype=torch.int32, device="cuda")
        w = torch.full((T, K), -1.0, dtype=torch.float32, device="cuda")
        B.flint_moe_route_noalloc(x.data_ptr(), layer.tensors["router_w"].data_ptr(), T, E, K, 2.0 ** -14,
                                  ids.data_ptr(), w.data_ptr(), stream)
        torch.cuda.synchronize()
        # the oracle's routing on fp64 logits (the redraw table keeps every 6th/7th gap >= 1e-4)
        xb = x.cpu().view(torch.int16).numpy().view(np.uint16)
        ref = R.route(R.bf16_to_f64(xb) @ R.bf16_to_f64(L["router_w"]).T, K)
        assert np.all(ref["gap"] >= 1e-4)
        np.testing.assert_array_equal(ids.cpu().numpy(), ref["ids"])
        np.testing.assert_allclose(w.cpu().numpy(), ref["w"], rtol=2e-6, atol=1e-7)
        np.testing.assert_array_equal(ids.cpu().numpy(), want["ids"].cpu().numpy())
        np.testing.assert_allclose(w.cpu().numpy(), want["w"].cpu().numpy(), rtol=2e-6, atol=1e-7)
    layer.close()


def test_noalloc_rejects_sizes_beyond_its_scratch():
    E = 256
    L = S.make_layer(32, "int4")
    rw = torch.from_numpy(L["router_w"].view(np.int16)).cuda()
    x = torch.zeros((65, 2048), dtype=torch.bfloat16, device="cuda")
    ids = torch.empty((65, 6), dtype=torch.int32, device="cuda")
    w = torch.empty((65, 6), dtype=torch.float32, device="cuda")
    with pytest.raises(B.FlintError) as e:
        B.flint_moe_route_noalloc(x.data_ptr(), rw.data_ptr(), 65, 32, 6, 2.0 ** -14, ids.data_ptr(), w.data_ptr())
    assert e.value.status == B.FLINT_ERR_INVALID_ARG
    with pytest.raises(B.FlintError):
        B.flint_moe_route_noalloc(x.data_ptr(), rw.data_ptr(), 8, 2 * E, 6, 2.0 ** -14, ids.data_ptr(), w.data_ptr())
