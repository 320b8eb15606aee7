"""The C-ABI library loads, exports every entry point include/flint_moe.h declares, and rejects bad
arguments on the host before touching a device. No GPU needed."""

import ctypes
import os
import re

import pytest

from bit_routed_expert_sigmoid_b200 import binding as B

HEADER_DIR = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "include")


def declared_functions():
    names = set()
    for fn in os.listdir(HEADER_DIR):
        if not fn.endswith(".h"):
            continue
        src = open(os.path.join(HEADER_DIR, fn)).read()
        src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
        for m in re.finditer(r"\b(flint_\w+)\s*\(", src):
            names.add(m.group(1))
    return sorted(names)


def test_every_declared_symbol_is_exported():
    names = declared_functions()
    assert "flint_moe_forward" in names and "flint_moe_create" in names
    lib = B.library_handle()
    for n in names:
        assert hasattr(lib, n), n
    assert set(B.EXPORTS) <= set(names)


def _cfg(**kw):
    base = dict(hidden=2048, n_experts=256, top_k=6, inter=512, inter_shared=1024, fmt=0, t_max=64,
                routed_scale=1.0, norm_floor=2.0 ** -14, flags=0)
    base.update(kw)
    return B.flint_moe_cfg(**base)


def test_workspace_size_rules():
    assert B.flint_moe_workspace_size(_cfg()) > 0
    small, big = B.flint_moe_workspace_size(_cfg(t_max=8)), B.flint_moe_workspace_size(_cfg(t_max=2048))
    assert 0 < small < big
    for bad in (dict(hidden=4096), dict(inter=256), dict(n_experts=48), dict(n_experts=512), dict(top_k=0),
                dict(top_k=9), dict(t_max=0), dict(fmt=7), dict(norm_floor=0.0), dict(n_experts=32, top_k=8)):
        cfg = _cfg(**bad)
        ok = bad == dict(n_experts=32, top_k=8)
        assert (B.flint_moe_workspace_size(cfg) > 0) == ok, bad


def test_w4a4_configuration_rules():
    # W4A4 is an NVFP4 mode: refused for int4 and for expert-cache handles; it adds the NVFP4 activation
    # rows of x and h, their scale atoms per 64-row chunk, the chunk positions and numbering, and the
    # weight scales as atoms (all 256-byte aligned pieces of the workspace)
    W = B.FLINT_FLAG_W4A4
    assert B.flint_moe_workspace_size(_cfg(fmt=B.FLINT_W_INT4_G128_FWHT128, flags=W)) == 0
    assert B.flint_moe_workspace_size(_cfg(fmt=B.FLINT_W_NVFP4, flags=W, n_slots=64)) == 0
    T, K, E, H, I = 2048, 6, 256, 2048, 512
    plain = B.flint_moe_workspace_size(_cfg(fmt=B.FLINT_W_NVFP4, t_max=T))
    w4 = B.flint_moe_workspace_size(_cfg(fmt=B.FLINT_W_NVFP4, t_max=T, flags=W))
    P = T * K
    chunks = (P + 63) // 64 + E
    al = lambda n: (n + 255) // 256 * 256  # noqa: E731
    extra = (al(P * H // 2) + al(P * H // 16) + al(P * 4) + al(P * I // 2) + al(P * I // 16) + al(P * 4)
             + al(P * 4) + al(E * 4) + al(chunks * (H // 64) * 512) + al(chunks * (I // 64) * 512)
             + al(E * (2 * I // 128) * (H // 64) * 512) + al(E * (H // 128) * (I // 64) * 512))
    assert w4 - plain == extra
    # the debug-check flag changes nothing in the workspace
    assert B.flint_moe_workspace_size(_cfg(fmt=B.FLINT_W_NVFP4, t_max=T, flags=B.FLINT_FLAG_DEBUG_CHECKS)) == plain


def test_create_rejects_bad_pointers_without_a_device():
    cfg = _cfg()
    w = B.flint_moe_weights(*([0x1000] * 9))
    h = ctypes.c_void_p()
    ws = B.flint_moe_workspace_size(cfg)
    # null / misaligned weights
    w0 = B.flint_moe_weights(*([0] * 9))
    assert B.raw_status("flint_moe_create", ctypes.byref(cfg), ctypes.byref(w0), ctypes.c_void_p(0x100000),
                        ctypes.c_size_t(ws), ctypes.byref(h)) == B.FLINT_ERR_INVALID_ARG
    w1 = B.flint_moe_weights(*([0x1008] * 9))
    assert B.raw_status("flint_moe_create", ctypes.byref(cfg), ctypes.byref(w1), ctypes.c_void_p(0x100000),
                        ctypes.c_size_t(ws), ctypes.byref(h)) == B.FLINT_ERR_INVALID_ARG
    # workspace too small / misaligned / missing
    for ptr, size in ((0x100000, ws - 1), (0x100010, ws), (0, ws)):
        assert B.raw_status("flint_moe_create", ctypes.byref(cfg), ctypes.byref(w), ctypes.c_void_p(ptr),
                            ctypes.c_size_t(size), ctypes.byref(h)) == B.FLINT_ERR_WORKSPACE
    # nvfp4 needs tensor scales
    wn = B.flint_moe_weights(0x1000, 0x1000, 0x1000, None, 0x1000, 0x1000, None, 0x1000, 0x1000)
    cfgn = _cfg(fmt=1)
    assert B.raw_status("flint_moe_create", ctypes.byref(cfgn), ctypes.byref(wn), ctypes.c_void_p(0x100000),
                        ctypes.c_size_t(B.flint_moe_workspace_size(cfgn)), ctypes.byref(h)) == B.FLINT_ERR_INVALID_ARG
    # unsupported width
    cfgu = _cfg(hidden=1024)
    assert B.raw_status("flint_moe_create", ctypes.byref(cfgu), ctypes.byref(w), ctypes.c_void_p(0x100000),
                        ctypes.c_size_t(ws), ctypes.byref(h)) == B.FLINT_ERR_UNSUPPORTED


def test_calls_on_a_null_handle_fail_cleanly():
    V = ctypes.c_void_p
    assert B.raw_status("flint_moe_forward", V(0), V(0x1000), 1, V(0x2000), V(0)) == B.FLINT_ERR_INVALID_ARG
    assert B.raw_status("flint_moe_forward_host", V(0), V(0x1000), 1, V(0x2000), V(0)) == B.FLINT_ERR_INVALID_ARG
    assert B.raw_status("flint_moe_routing", V(0), V(0), V(0), V(0), V(0), V(0)) == B.FLINT_ERR_INVALID_ARG
    assert B.raw_status("flint_moe_destroy", V(0)) == B.FLINT_OK
    with pytest.raises(B.FlintError):
        B.flint_moe_forward(0, 0x1000, 1, 0x2000)


def test_stack_entry_points_check_arguments_on_the_host():
    V, F = ctypes.c_void_p, ctypes.c_float
    # residual + norm: negative T, non-positive eps, misaligned or missing residual -> rejected before a launch
    assert B.raw_status("flint_residual_rmsnorm", V(0x1000), V(0), -1, F(1e-6), V(0x2000), V(0)) == B.FLINT_ERR_INVALID_ARG
    assert B.raw_status("flint_residual_rmsnorm", V(0x1000), V(0), 4, F(0.0), V(0x2000), V(0)) == B.FLINT_ERR_INVALID_ARG
    assert B.raw_status("flint_residual_rmsnorm", V(0x1004), V(0), 4, F(1e-6), V(0x2000), V(0)) == B.FLINT_ERR_INVALID_ARG
    assert B.raw_status("flint_residual_rmsnorm", V(0), V(0), 4, F(1e-6), V(0x2000), V(0)) == B.FLINT_ERR_INVALID_ARG
    assert B.raw_status("flint_residual_rmsnorm", V(0), V(0), 0, F(1e-6), V(0), V(0)) == B.FLINT_OK      # T = 0: no-op
    # stack: no layers, a null layer handle
    arr = (ctypes.c_void_p * 2)(None, None)
    assert B.raw_status("flint_moe_stack_forward", None, 1, V(0x1000), 4, F(1e-6), V(0x2000), V(0x3000), V(0)) == \
        B.FLINT_ERR_INVALID_ARG
    assert B.raw_status("flint_moe_stack_forward", arr, 0, V(0x1000), 4, F(1e-6), V(0x2000), V(0x3000), V(0)) == \
        B.FLINT_ERR_INVALID_ARG
    assert B.raw_status("flint_moe_stack_forward", arr, 2, V(0x1000), 4, F(1e-6), V(0x2000), V(0x3000), V(0)) == \
        B.FLINT_ERR_INVALID_ARG


def test_status_strings():
    for s in range(7):
        assert B.flint_moe_status_string(s)
    assert "unknown" in B.flint_moe_status_string(99)


def test_quantiser_entry_points_check_arguments_on_the_host():
    V, LL = ctypes.c_void_p, ctypes.c_longlong
    q4 = "flint_quantize_int4_g128"
    bad = [
        (V(0x1000), LL(4), 200, 1, V(0x2000), V(0x3000), V(0)),        # cols not a multiple of 128
        (V(0x1000), LL(-1), 256, 1, V(0x2000), V(0x3000), V(0)),       # negative rows
        (V(0x1000), LL(4), 256, 2, V(0x2000), V(0x3000), V(0)),        # rotate is 0 or 1
        (V(0x1008), LL(4), 256, 1, V(0x2000), V(0x3000), V(0)),        # w not 16-byte aligned
        (V(0x1000), LL(4), 256, 1, V(0x2001), V(0x3000), V(0)),        # codes not 2-byte aligned
        (V(0), LL(4), 256, 1, V(0x2000), V(0x3000), V(0)),             # null input
    ]
    for args in bad:
        assert B.raw_status(q4, *args) == B.FLINT_ERR_INVALID_ARG, args
    assert B.raw_status(q4, V(0), LL(0), 256, 1, V(0), V(0), V(0)) == B.FLINT_OK       # rows = 0: no-op
    nv = "flint_quantize_nvfp4"
    bad = [
        (V(0x1000), 2, 4, 24, V(0x2000), V(0x3000), V(0x4000), V(0)),  # cols not a multiple of 16
        (V(0x1000), -1, 4, 32, V(0x2000), V(0x3000), V(0x4000), V(0)), # negative count
        (V(0x1000), 70000, 4, 32, V(0x2000), V(0x3000), V(0x4000), V(0)),  # more Linears than one grid row holds
        (V(0x1000), 2, 0, 32, V(0x2000), V(0x3000), V(0x4000), V(0)),  # empty Linears
        (V(0x1000), 2, 4, 32, V(0x2004), V(0x3000), V(0x4000), V(0)),  # codes not 8-byte aligned
        (V(0x1000), 2, 4, 32, V(0x2000), V(0x3000), V(0x4002), V(0)),  # tscale not 4-byte aligned
        (V(0x1000), 2, 4, 32, V(0x2000), V(0x3000), V(0), V(0)),       # no tscale
    ]
    for args in bad:
        assert B.raw_status(nv, *args) == B.FLINT_ERR_INVALID_ARG, args
    assert B.raw_status(nv, V(0), 0, 4, 32, V(0), V(0), V(0), V(0)) == B.FLINT_OK     # no Linears: no-op
