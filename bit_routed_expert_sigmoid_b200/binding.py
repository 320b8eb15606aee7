"""ctypes binding of libflint_moe.so (include/flint_moe.h): argument marshalling only.

Every function here forwards to the C entry point of the same name. Pointers are plain integers
(device addresses, e.g. torch's tensor.data_ptr(), or host addresses for *_host arguments);
streams are cudaStream_t handles as integers (torch.cuda.Stream.cuda_stream). A non-OK status
raises FlintError. Importing this module fails loudly when the library has not been built: there
is no other implementation to fall back to.
"""

from __future__ import annotations

import ctypes
import os

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libflint_moe.so")

FLINT_OK = 0
FLINT_ERR_INVALID_ARG = 1
FLINT_ERR_UNSUPPORTED = 2
FLINT_ERR_CUDA = 3
FLINT_ERR_WORKSPACE = 4
FLINT_ERR_DEVICE_CHECK = 5
FLINT_ERR_TIMEOUT = 6

FLINT_W_INT4_G128_FWHT128 = 0
FLINT_W_NVFP4 = 1
FLINT_FLAG_DEBUG_CHECKS = 0x1
FLINT_FLAG_W4A4 = 0x2

FLINT_BUF_LOGITS = 0
FLINT_BUF_XQ = 1
FLINT_BUF_YS = 2
FLINT_BUF_XA = 3
FLINT_BUF_XA_SF = 4
FLINT_BUF_XA_TS = 5
FLINT_BUF_H = 6
FLINT_BUF_HA = 7
FLINT_BUF_HA_SF = 8
FLINT_BUF_HA_TS = 9
FLINT_BUF_O = 10

EXPORTS = (
    "flint_moe_workspace_size", "flint_moe_create", "flint_moe_forward", "flint_moe_forward_host",
    "flint_moe_routing", "flint_moe_intermediate", "flint_moe_error_word", "flint_moe_destroy",
    "flint_moe_status_string", "flint_moe_set_stage_events", "flint_moe_stage_count", "flint_moe_stage_name",
    "flint_moe_route_noalloc", "flint_residual_rmsnorm", "flint_moe_stack_forward",
    "flint_quantize_int4_g128", "flint_quantize_nvfp4",
)


class FlintError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {flint_moe_status_string(status)} (status {status})")


class flint_moe_cfg(ctypes.Structure):
    _fields_ = [("hidden", ctypes.c_int), ("n_experts", ctypes.c_int), ("top_k", ctypes.c_int),
                ("inter", ctypes.c_int), ("inter_shared", ctypes.c_int), ("fmt", ctypes.c_int),
                ("t_max", ctypes.c_int), ("routed_scale", ctypes.c_float), ("norm_floor", ctypes.c_float),
                ("flags", ctypes.c_uint), ("n_slots", ctypes.c_int)]


class flint_moe_weights(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in ("router_w", "gu_codes", "gu_scales", "gu_tscale", "dn_codes",
                                                "dn_scales", "dn_tscale", "sh_gu", "sh_dn")]


def _load():
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"{LIB_PATH} is missing: build it with `python -m bit_routed_expert_sigmoid_b200.build` "
                          "(the Flint MoE layer has no implementation other than its CUDA kernels)")
    lib = ctypes.CDLL(LIB_PATH)
    P, I, S, V = ctypes.POINTER, ctypes.c_int, ctypes.c_size_t, ctypes.c_void_p
    sig = {
        "flint_moe_workspace_size": (S, [P(flint_moe_cfg)]),
        "flint_moe_create": (I, [P(flint_moe_cfg), P(flint_moe_weights), V, S, P(V)]),
        "flint_moe_forward": (I, [V, V, I, V, V]),
        "flint_moe_forward_host": (I, [V, V, I, V, V]),
        "flint_moe_forward_routed": (I, [V, V, I, V, V, V, V]),
        "flint_cache_create": (I, [V, P(flint_moe_weights), P(V)]),
        "flint_cache_destroy": (I, [V]),
        "flint_cache_stats": (I, [V, P(ctypes.c_longlong), P(ctypes.c_longlong), P(ctypes.c_longlong)]),
        "flint_moe_forward_cached": (I, [V, V, V, I, V, V]),
        "flint_cache_plan": (I, [I, I, P(I), P(I), P(ctypes.c_ulonglong), ctypes.c_ulonglong, P(I), I, P(I)]),
        "flint_moe_routing": (I, [V, V, V, V, V, V]),
        "flint_moe_intermediate": (I, [V, I, V, S, V]),
        "flint_moe_error_word": (I, [V, P(ctypes.c_uint)]),
        "flint_moe_destroy": (I, [V]),
        "flint_moe_status_string": (ctypes.c_char_p, [I]),
        "flint_moe_set_stage_events": (I, [V, P(V), I]),
        "flint_moe_stage_count": (I, [V, I]),
        "flint_moe_stage_name": (ctypes.c_char_p, [V, I, I]),
        "flint_moe_route_noalloc": (I, [V, V, I, I, I, ctypes.c_float, V, V, V]),
        "flint_residual_rmsnorm": (I, [V, V, I, ctypes.c_float, V, V]),
        "flint_moe_stack_forward": (I, [P(V), I, V, I, ctypes.c_float, V, V, V]),
        "flint_quantize_int4_g128": (I, [V, ctypes.c_longlong, I, I, V, V, V]),
        "flint_quantize_nvfp4": (I, [V, I, I, I, V, V, V, V]),
    }
    for name, (res, args) in sig.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    return lib


_lib = _load()


def _check(status: int, where: str) -> None:
    if status != FLINT_OK:
        raise FlintError(status, where)


def flint_moe_status_string(status: int) -> str:
    return _lib.flint_moe_status_string(int(status)).decode()


def flint_moe_workspace_size(cfg: flint_moe_cfg) -> int:
    return int(_lib.flint_moe_workspace_size(ctypes.byref(cfg)))


def flint_moe_create(cfg: flint_moe_cfg, weights: flint_moe_weights, workspace: int, workspace_bytes: int) -> int:
    h = ctypes.c_void_p()
    _check(_lib.flint_moe_create(ctypes.byref(cfg), ctypes.byref(weights), ctypes.c_void_p(workspace),
                                 ctypes.c_size_t(workspace_bytes), ctypes.byref(h)), "flint_moe_create")
    return h.value


def flint_moe_forward(h: int, x: int, T: int, y: int, stream: int = 0) -> None:
    _check(_lib.flint_moe_forward(ctypes.c_void_p(h), ctypes.c_void_p(x), int(T), ctypes.c_void_p(y),
                                  ctypes.c_void_p(stream)), "flint_moe_forward")


def flint_moe_forward_routed(h: int, x: int, T: int, ids: int, w: int, y: int, stream: int = 0) -> None:
    _check(_lib.flint_moe_forward_routed(ctypes.c_void_p(h), ctypes.c_void_p(x), int(T), ctypes.c_void_p(ids),
                                         ctypes.c_void_p(w), ctypes.c_void_p(y), ctypes.c_void_p(stream)),
           "flint_moe_forward_routed")


def flint_cache_create(layer: int, host: flint_moe_weights) -> int:
    c = ctypes.c_void_p()
    _check(_lib.flint_cache_create(ctypes.c_void_p(layer), ctypes.byref(host), ctypes.byref(c)), "flint_cache_create")
    return c.value


def flint_cache_destroy(c: int) -> None:
    _check(_lib.flint_cache_destroy(ctypes.c_void_p(c)), "flint_cache_destroy")


def flint_cache_stats(c: int) -> tuple:
    h, m, b = ctypes.c_longlong(), ctypes.c_longlong(), ctypes.c_longlong()
    _check(_lib.flint_cache_stats(ctypes.c_void_p(c), ctypes.byref(h), ctypes.byref(m), ctypes.byref(b)),
           "flint_cache_stats")
    return h.value, m.value, b.value


def flint_moe_forward_cached(h: int, c: int, x: int, T: int, y: int, stream: int = 0) -> None:
    _check(_lib.flint_moe_forward_cached(ctypes.c_void_p(h), ctypes.c_void_p(c), ctypes.c_void_p(x), int(T),
                                         ctypes.c_void_p(y), ctypes.c_void_p(stream)), "flint_moe_forward_cached")


def flint_cache_plan(E: int, S: int, slot_of, expert_of, last_use, tick: int, ids, loads) -> int:
    """Host-only replacement rule (no CUDA): numpy int32 slot_of [E], expert_of [S], uint64 last_use [S]
    (updated in place), int32 ids [P], int32 loads [2S] (out). Returns the number of misses or -1."""
    P_ = ctypes.POINTER
    return int(_lib.flint_cache_plan(int(E), int(S), slot_of.ctypes.data_as(P_(ctypes.c_int)),
                                     expert_of.ctypes.data_as(P_(ctypes.c_int)),
                                     last_use.ctypes.data_as(P_(ctypes.c_ulonglong)), ctypes.c_ulonglong(tick),
                                     ids.ctypes.data_as(P_(ctypes.c_int)), int(ids.size),
                                     loads.ctypes.data_as(P_(ctypes.c_int))))


def flint_moe_forward_host(h: int, x_host: int, T: int, y_host: int, stream: int = 0) -> None:
    _check(_lib.flint_moe_forward_host(ctypes.c_void_p(h), ctypes.c_void_p(x_host), int(T), ctypes.c_void_p(y_host),
                                       ctypes.c_void_p(stream)), "flint_moe_forward_host")


def flint_moe_routing(h: int, ids: int = 0, w: int = 0, offsets: int = 0, perm: int = 0, stream: int = 0) -> None:
    _check(_lib.flint_moe_routing(ctypes.c_void_p(h), ctypes.c_void_p(ids), ctypes.c_void_p(w),
                                  ctypes.c_void_p(offsets), ctypes.c_void_p(perm), ctypes.c_void_p(stream)),
           "flint_moe_routing")


def flint_moe_intermediate(h: int, which: int, dst: int, nbytes: int, stream: int = 0) -> None:
    _check(_lib.flint_moe_intermediate(ctypes.c_void_p(h), int(which), ctypes.c_void_p(dst), ctypes.c_size_t(nbytes),
                                       ctypes.c_void_p(stream)), "flint_moe_intermediate")


def flint_moe_error_word(h: int) -> int:
    out = ctypes.c_uint(0)
    _check(_lib.flint_moe_error_word(ctypes.c_void_p(h), ctypes.byref(out)), "flint_moe_error_word")
    return int(out.value)


def flint_residual_rmsnorm(x: int, y: int, T: int, eps: float, z: int, stream: int = 0) -> None:
    _check(_lib.flint_residual_rmsnorm(ctypes.c_void_p(x), ctypes.c_void_p(y), int(T), ctypes.c_float(eps),
                                       ctypes.c_void_p(z), ctypes.c_void_p(stream)), "flint_residual_rmsnorm")


def flint_moe_stack_forward(handles, x: int, T: int, eps: float, z: int, y: int, stream: int = 0) -> None:
    arr = (ctypes.c_void_p * len(handles))(*handles)
    _check(_lib.flint_moe_stack_forward(arr, len(handles), ctypes.c_void_p(x), int(T), ctypes.c_float(eps),
                                        ctypes.c_void_p(z), ctypes.c_void_p(y), ctypes.c_void_p(stream)),
           "flint_moe_stack_forward")


def flint_quantize_int4_g128(w: int, rows: int, cols: int, rotate: bool, codes: int, scales: int,
                             stream: int = 0) -> None:
    _check(_lib.flint_quantize_int4_g128(ctypes.c_void_p(w), int(rows), int(cols), 1 if rotate else 0,
                                         ctypes.c_void_p(codes), ctypes.c_void_p(scales), ctypes.c_void_p(stream)),
           "flint_quantize_int4_g128")


def flint_quantize_nvfp4(w: int, n_mats: int, rows: int, cols: int, codes: int, scales: int, tscale: int,
                         stream: int = 0) -> None:
    _check(_lib.flint_quantize_nvfp4(ctypes.c_void_p(w), int(n_mats), int(rows), int(cols), ctypes.c_void_p(codes),
                                     ctypes.c_void_p(scales), ctypes.c_void_p(tscale), ctypes.c_void_p(stream)),
           "flint_quantize_nvfp4")


def flint_moe_destroy(h: int) -> None:
    _check(_lib.flint_moe_destroy(ctypes.c_void_p(h)), "flint_moe_destroy")


def flint_moe_set_stage_events(h: int, events) -> None:
    """events: sequence of cudaEvent_t handles (ints), or None to stop recording."""
    if events is None:
        _check(_lib.flint_moe_set_stage_events(ctypes.c_void_p(h), None, 0), "flint_moe_set_stage_events")
        return
    arr = (ctypes.c_void_p * len(events))(*events)
    _check(_lib.flint_moe_set_stage_events(ctypes.c_void_p(h), arr, len(events)), "flint_moe_set_stage_events")


def flint_moe_stage_count(h: int, T: int) -> int:
    return int(_lib.flint_moe_stage_count(ctypes.c_void_p(h), int(T)))


def flint_moe_stage_name(h: int, T: int, i: int) -> str:
    r = _lib.flint_moe_stage_name(ctypes.c_void_p(h), int(T), int(i))
    return r.decode() if r else ""


def flint_moe_route_noalloc(x: int, router_w: int, T: int, n_experts: int, top_k: int, norm_floor: float,
                            ids: int, w: int, stream: int = 0) -> None:
    """Routing (ids, w) for T <= 64 tokens using the library's fixed device scratch array instead of
    a workspace: for callers that cannot allocate device memory."""
    _check(_lib.flint_moe_route_noalloc(ctypes.c_void_p(x), ctypes.c_void_p(router_w), int(T), int(n_experts),
                                        int(top_k), ctypes.c_float(norm_floor), ctypes.c_void_p(ids),
                                        ctypes.c_void_p(w), ctypes.c_void_p(stream)), "flint_moe_route_noalloc")


def raw_status(name: str, *args) -> int:
    """Calls an entry point and returns its status code without raising (for argument-check tests)."""
    return int(getattr(_lib, name)(*args))


def library_handle():
    return _lib
