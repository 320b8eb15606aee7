"""PyTorch plumbing around the C ABI: device buffers for one layer's weights and workspace.

PyTorch only allocates device memory and provides streams here; every step of the forward runs in
the library's CUDA kernels (binding.flint_moe_forward).
"""

from __future__ import annotations

import numpy as np
import torch

from . import binding as B

H, I, IS = 2048, 512, 1024


def _to_device(a, device):
    if a is None:
        return None
    a = np.ascontiguousarray(a)
    if a.dtype == np.uint16:
        a = a.view(np.int16)
    return torch.from_numpy(a).to(device)


# W4A4 intermediates (permuted rows): columns per row (0: one value per row) and dtype
_W4A4_BUFS = {B.FLINT_BUF_XA: (H // 2, torch.uint8), B.FLINT_BUF_XA_SF: (H // 16, torch.uint8),
              B.FLINT_BUF_XA_TS: (0, torch.float32), B.FLINT_BUF_H: (I, torch.float32),
              B.FLINT_BUF_HA: (I // 2, torch.uint8), B.FLINT_BUF_HA_SF: (I // 16, torch.uint8),
              B.FLINT_BUF_HA_TS: (0, torch.float32), B.FLINT_BUF_O: (H, torch.float16)}


class FlintMoELayer:
    """One Flint MoE layer resident on a CUDA device.

    L is a dict of host arrays in the C-ABI storage layout (see synthetic.make_layer). The weights
    are copied to the device once; the handle borrows them and the workspace."""

    def __init__(self, L: dict, t_max: int, *, top_k: int = 6, device="cuda", flags: int = 0,
                 routed_scale: float = 1.0, norm_floor: float = 2.0 ** -14, n_slots: int = 0):
        self.device = torch.device(device)
        self.E = int(L["E"])
        self.top_k = top_k
        self.t_max = t_max
        self.n_slots = n_slots
        fmt = B.FLINT_W_INT4_G128_FWHT128 if L["fmt"] == "int4" else B.FLINT_W_NVFP4
        self.cfg = B.flint_moe_cfg(hidden=L["H"], n_experts=self.E, top_k=top_k, inter=L["I"],
                                   inter_shared=L["Is"], fmt=fmt, t_max=t_max, routed_scale=routed_scale,
                                   norm_floor=norm_floor, flags=flags, n_slots=n_slots)
        routed = ("gu_codes", "gu_scales", "gu_tscale", "dn_codes", "dn_scales", "dn_tscale")
        if n_slots > 0:
            # routed experts in page-locked host memory; the device holds n_slots expert slots
            self.host = {k: (torch.from_numpy(np.ascontiguousarray(L[k]).view(
                np.int16 if L[k].dtype == np.uint16 else L[k].dtype)).pin_memory() if L.get(k) is not None else None)
                for k in routed}
            self.tensors = {k: _to_device(L.get(k), self.device) for k in ("router_w", "sh_gu", "sh_dn")}
            for k, v in self.host.items():
                self.tensors[k] = (torch.zeros((n_slots,) + tuple(v.shape[1:]), dtype=v.dtype, device=self.device)
                                   if v is not None else None)
        else:
            self.tensors = {k: _to_device(L.get(k), self.device)
                            for k in ("router_w", "sh_gu", "sh_dn") + routed}
        ptr = {k: (v.data_ptr() if v is not None else None) for k, v in self.tensors.items()}
        self.weights = B.flint_moe_weights(**ptr)
        self.ws_bytes = B.flint_moe_workspace_size(self.cfg)
        if self.ws_bytes == 0:
            raise ValueError("configuration rejected by flint_moe_workspace_size")
        self.workspace = torch.empty(self.ws_bytes + 256, dtype=torch.uint8, device=self.device)
        base = self.workspace.data_ptr()
        self.ws_ptr = (base + 255) // 256 * 256
        self.handle = B.flint_moe_create(self.cfg, self.weights, self.ws_ptr, self.ws_bytes)
        self.cache = None
        if n_slots > 0:
            hp = {k: (v.data_ptr() if v is not None else None) for k, v in self.host.items()}
            self.host_weights = B.flint_moe_weights(**hp)
            self.cache = B.flint_cache_create(self.handle, self.host_weights)

    def weight_bytes(self) -> int:
        return sum(v.numel() * v.element_size() for v in self.tensors.values() if v is not None)

    def forward(self, x: torch.Tensor, y: torch.Tensor | None = None, stream=None) -> torch.Tensor:
        """x: [T][H] bf16 (or int16 bit patterns) on the device. Returns y [T][H] bf16."""
        T = x.shape[0]
        if y is None:
            y = torch.empty((T, H), dtype=torch.bfloat16, device=self.device)
        s = (stream or torch.cuda.current_stream(self.device)).cuda_stream
        if self.cache is not None:
            B.flint_moe_forward_cached(self.handle, self.cache, x.data_ptr(), T, y.data_ptr(), s)
        else:
            B.flint_moe_forward(self.handle, x.data_ptr(), T, y.data_ptr(), s)
        return y

    def forward_routed(self, x: torch.Tensor, ids: torch.Tensor, w: torch.Tensor, y: torch.Tensor | None = None,
                       stream=None) -> torch.Tensor:
        """Forward on a given routing: ids int32 [T][top_k] (ascending per token), w f32 [T][top_k]."""
        T = x.shape[0]
        if y is None:
            y = torch.empty((T, H), dtype=torch.bfloat16, device=self.device)
        s = (stream or torch.cuda.current_stream(self.device)).cuda_stream
        B.flint_moe_forward_routed(self.handle, x.data_ptr(), T, ids.data_ptr(), w.data_ptr(), y.data_ptr(), s)
        return y

    def cache_stats(self) -> dict:
        h, m, b = B.flint_cache_stats(self.cache)
        return {"hits": h, "misses": m, "bytes": b}

    def forward_host(self, x_host: torch.Tensor, y_host: torch.Tensor, stream=None) -> None:
        """x_host, y_host: [T][H] 16-bit host tensors (pinned for asynchronous copies)."""
        s = (stream or torch.cuda.current_stream(self.device)).cuda_stream
        B.flint_moe_forward_host(self.handle, x_host.data_ptr(), x_host.shape[0], y_host.data_ptr(), s)

    def routing(self, T: int) -> dict:
        K = self.top_k
        out = {"ids": torch.empty((T, K), dtype=torch.int32, device=self.device),
               "w": torch.empty((T, K), dtype=torch.float32, device=self.device),
               "offsets": torch.empty((self.E + 1,), dtype=torch.int32, device=self.device),
               "perm": torch.empty((T * K,), dtype=torch.int32, device=self.device)}
        s = torch.cuda.current_stream(self.device).cuda_stream
        B.flint_moe_routing(self.handle, out["ids"].data_ptr(), out["w"].data_ptr(), out["offsets"].data_ptr(),
                            out["perm"].data_ptr(), s)
        return out

    def intermediate(self, which: int, T: int) -> torch.Tensor:
        if which == B.FLINT_BUF_LOGITS:
            t = torch.empty((T, self.E), dtype=torch.float32, device=self.device)
        elif which == B.FLINT_BUF_XQ:
            t = torch.empty((T, H), dtype=torch.float16, device=self.device)
        elif which == B.FLINT_BUF_YS:
            t = torch.empty((T, H), dtype=torch.float32, device=self.device)
        elif which in _W4A4_BUFS:
            P = T * self.top_k
            cols, dtype = _W4A4_BUFS[which]
            t = torch.empty((P, cols) if cols else (P,), dtype=dtype, device=self.device)
        else:
            raise ValueError(which)
        s = torch.cuda.current_stream(self.device).cuda_stream
        B.flint_moe_intermediate(self.handle, which, t.data_ptr(), t.numel() * t.element_size(), s)
        return t

    def error_word(self) -> int:
        return B.flint_moe_error_word(self.handle)

    def close(self) -> None:
        if getattr(self, "cache", None):
            B.flint_cache_destroy(self.cache)
            self.cache = None
        if getattr(self, "handle", None):
            B.flint_moe_destroy(self.handle)
            self.handle = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


class FlintMoEStack:
    """A stack of Flint MoE layers on one device, run on an fp32 residual stream:
    for each layer, z = bf16(rmsnorm(x)); x += layer(z) (flint_moe_stack_forward)."""

    def __init__(self, layers, t_max: int, *, eps: float = 1e-6, device="cuda", **kw):
        """layers: an iterable of host weight dicts; each is copied to the device as it comes, so a
        generator keeps at most one layer on the host."""
        self.device = torch.device(device)
        self.eps = float(eps)
        self.t_max = t_max
        self.layers = [FlintMoELayer(L, t_max=t_max, device=device, **kw) for L in layers]
        self.z = torch.empty((t_max, H), dtype=torch.bfloat16, device=self.device)
        self.y = torch.empty((t_max, H), dtype=torch.bfloat16, device=self.device)

    def weight_bytes(self) -> int:
        return sum(layer.weight_bytes() for layer in self.layers)

    def forward(self, x: torch.Tensor, stream=None) -> torch.Tensor:
        """x: [T][H] fp32 residual on the device, updated in place and returned."""
        T = x.shape[0]
        s = (stream or torch.cuda.current_stream(self.device)).cuda_stream
        B.flint_moe_stack_forward([layer.handle for layer in self.layers], x.data_ptr(), T, self.eps,
                                  self.z.data_ptr(), self.y.data_ptr(), s)
        return x

    def close(self) -> None:
        for layer in self.layers:
            layer.close()


def x_to_device(x_bits: np.ndarray, device="cuda") -> torch.Tensor:
    """bf16 bit patterns [T][H] (uint16) -> device bf16 tensor."""
    return torch.from_numpy(np.ascontiguousarray(x_bits).view(np.int16)).to(device).view(torch.bfloat16)


def y_to_host_bits(y: torch.Tensor) -> np.ndarray:
    return y.view(torch.int16).cpu().numpy().view(np.uint16)
