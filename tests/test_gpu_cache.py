"""Host-resident routed experts with a device cache of hot experts (flint_moe_forward_cached) and the
forward on a given routing (flint_moe_forward_routed), through the C ABI, against the fp64 oracle.
The routed weights live in page-locked host memory; the device holds a few expert slots."""

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


def expert_bytes(L):
    return S.expert_nbytes(L)


@pytest.mark.parametrize("fmt,E,n_slots,T", [("int4", 32, 16, 2), ("nvfp4", 32, 24, 2), ("int4", 256, 64, 8)])
def test_cached_decode_matches_the_oracle_over_a_stream_of_batches(fmt, E, n_slots, T):
    L = S.make_layer(E, fmt)
    dev = FlintMoELayer(L, t_max=T, n_slots=n_slots)
    redraws = S.redraw_table(E)
    seen, distinct_total, misses_expected = set(), 0, None
    for step, first in enumerate((0, 0, 40, 80, 0, 120)):
        x = S.make_x(T, redraws=redraws, first_row=first)
        ref = R.moe_forward(L, x)
        y = dev.forward(x_to_device(x))
        torch.cuda.synchronize()
        PT.check_routing(dev.routing(T), ref, T, 6)
        st = PT.compare_y(y_to_host_bits(y), ref["y"])
        assert st["finite"] and st["violations"] == 0, (step, st)
        distinct_total += len(set(ref["ids"].reshape(-1).tolist()))
        seen |= set(ref["ids"].reshape(-1).tolist())
    stats = dev.cache_stats()
    assert stats["hits"] + stats["misses"] == distinct_total
    assert stats["hits"] > 0                                        # repeated batches hit the cache
    assert stats["misses"] >= min(len(seen), n_slots)               # every expert was loaded once at least
    assert stats["bytes"] == stats["misses"] * expert_bytes(L)
    assert dev.error_word() == 0
    dev.close()


def test_cached_prefill_and_capacity():
    # T = 40 on the tensor-core path with a slot per expert; with too few slots the call is refused
    E, T = 32, 40
    L = S.make_layer(E, "int4")
    x = S.make_workload_x(T, E)
    ref = R.moe_forward(L, x)
    dev = FlintMoELayer(L, t_max=T, n_slots=E)
    y = dev.forward(x_to_device(x))
    torch.cuda.synchronize()
    PT.check_routing(dev.routing(T), ref, T, 6)
    st = PT.compare_y(y_to_host_bits(y), ref["y"])
    assert st["finite"] and st["violations"] == 0, st
    dev.close()
    small = FlintMoELayer(L, t_max=T, n_slots=8)
    with pytest.raises(B.FlintError) as e:
        small.forward(x_to_device(x))
    assert e.value.status == B.FLINT_ERR_UNSUPPORTED
    # a cache handle takes no other forward
    with pytest.raises(B.FlintError):
        xd = x_to_device(x[:4])
        yd = torch.empty((4, 2048), dtype=torch.bfloat16, device="cuda")
        B.flint_moe_forward(small.handle, xd.data_ptr(), 4, yd.data_ptr(), 0)
    small.close()


@pytest.mark.parametrize("T", [8, 40])
def test_forward_on_a_given_routing(T):
    # the oracle's routing handed in: the layer reproduces the oracle's output on it, on the decode
    # kernel (T = 8) and the tensor-core path (T = 40)
    E = 32
    L = S.make_layer(E, "int4")
    x = S.make_workload_x(T, E)
    ref = R.moe_forward(L, x)
    dev = FlintMoELayer(L, t_max=T)
    ids = torch.from_numpy(ref["ids"].astype(np.int32)).cuda()
    w = torch.from_numpy(ref["w"].astype(np.float32)).cuda()
    y = dev.forward_routed(x_to_device(x), ids, w)
    torch.cuda.synchronize()
    st = PT.compare_y(y_to_host_bits(y), ref["y"])
    assert st["finite"] and st["violations"] == 0, st
    r = dev.routing(T)
    np.testing.assert_array_equal(r["ids"].cpu().numpy(), ref["ids"])
    np.testing.assert_array_equal(r["offsets"].cpu().numpy(), ref["offsets"])
    dev.close()
