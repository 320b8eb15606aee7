"""Seeded synthetic inputs for one Flint MoE layer (weights and activations).

This module draws random numbers and encodes them into the storage formats the
layer consumes; it computes nothing the layer computes. It is shared by the
CUDA path's tests and benchmark and by the CPU oracle's tests, so that both
sides see byte-identical inputs.

Workload recipe (shapes from the Flint model cards; distributions chosen to
match the statistics the pages quote):

* hidden H = 2048, routed experts E (256 for the full layer, 32 for the tiny
  case), SwiGLU width I = 512, shared-expert width Is = 1024
  (Aijuus/flint-w4exp, model summary; WaveCut/Flint-UD-Q4_K_XL-NInfer-v3,
  "What is inside").
* activations x ~ N(0, 1.26^2) in bf16: the residual entering a late MoE block
  has rms 1.26 (Aijuus/flint-w4exp, "Why the linears stay bf16").
* router rows W_r ~ N(0, 0.02^2) in bf16 (the routers are bf16 in the
  checkpoint: kekzle/Flint-NVFP4, "What is in the files").
* int4 experts: two's-complement codes uniform in [-8, 7], two per byte (low
  nibble = even K index), one bf16 scale 0.004*(1+U[0,1)) per 128 of K
  (Aijuus/flint-w4exp, "weights" row: codes i4, group 128, bf16 scale).
* NVFP4 experts: E2M1 codes uniform over all 16 patterns, two per byte (low
  nibble = even column), one E4M3 block scale 2^U{-4..2} per 16 columns and an
  F32 tensor scale 0.01 per Linear (kekzle/Flint-NVFP4, "What is in the
  files", Layout row).
* shared expert gate|up [2*Is][H] and down [H][Is] ~ N(0, 0.02^2) in bf16.
* skewed-load variant: a per-expert router bias b_e ~ N(0, 1) folded into the
  data (x[:, 0] := 1 and W_r[e, 0] := bf16(b_e)), so the layer itself stays
  unbiased.

Every component draws from its own counter-keyed PCG64 stream, so the router
and shared expert are identical across weight formats. Token row r of x comes
from stream (SEED_X, r, d) where d is that row's redraw count; the redraw
table (rows whose 6th/7th sigmoid-score gap is under 1e-4 are redrawn) is
data shipped with this package (redraws.json).
"""

from __future__ import annotations

import numpy as np

SEED_WEIGHTS = 0
SEED_X = 1
SEED_SKEW = 2

H_DEFAULT = 2048
I_DEFAULT = 512
IS_DEFAULT = 1024
X_STD = 1.26
W_STD = 0.02

FMT_INT4 = "int4"
FMT_NVFP4 = "nvfp4"

# stream tags, one per component
_TAG_ROUTER, _TAG_GU_CODES, _TAG_GU_SCALES, _TAG_DN_CODES, _TAG_DN_SCALES, _TAG_SH_GU, _TAG_SH_DN = range(7)
_TAG_MASTER_GU, _TAG_MASTER_DN, _TAG_MASTER_OUT = range(7, 10)


def _rng(*key: int) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(list(key)))


def f32_to_bf16_bits(a) -> np.ndarray:
    """Round float32 values to bf16 (round to nearest even); returns uint16 bit patterns."""
    u = np.ascontiguousarray(a, dtype=np.float32).view(np.uint32).astype(np.uint64)
    r = (u + 0x7FFF + ((u >> 16) & 1)) >> 16
    return r.astype(np.uint16)


def _bf16_normal(rng: np.random.Generator, shape, std: float) -> np.ndarray:
    return f32_to_bf16_bits(rng.standard_normal(size=shape, dtype=np.float32) * np.float32(std))


def make_layer(E: int, fmt: str = FMT_INT4, *, H: int = H_DEFAULT, I: int = I_DEFAULT,
               Is: int = IS_DEFAULT, seed: int = SEED_WEIGHTS, skew: bool = False) -> dict:
    """Draw one layer's weights in the C-ABI storage layout (all row-major [out][in]).

    Returns a dict of numpy arrays:
      router_w  u16 (bf16) [E][H]
      gu_codes  u8 [E][2I][H/2]          gate rows 0..I-1 then up rows I..2I-1
      gu_scales int4: u16 (bf16) [E][2I][H/128]; nvfp4: u8 (E4M3) [E][2I][H/16]
      gu_tscale nvfp4: f32 [E][2] (gate, up); int4: None
      dn_codes  u8 [E][H][I/2]
      dn_scales int4: u16 (bf16) [E][H][I/128]; nvfp4: u8 (E4M3) [E][H][I/16]
      dn_tscale nvfp4: f32 [E]; int4: None
      sh_gu     u16 (bf16) [2*Is][H]      gate rows then up rows
      sh_dn     u16 (bf16) [H][Is]
    """
    if fmt not in (FMT_INT4, FMT_NVFP4):
        raise ValueError(f"unknown weight format {fmt!r}")
    if H % 128 or I % 128 or Is % 8:
        raise ValueError("H and I must be multiples of 128")
    L = {"fmt": fmt, "E": E, "H": H, "I": I, "Is": Is}
    router = _bf16_normal(_rng(seed, _TAG_ROUTER), (E, H), W_STD)
    if skew:
        b = _rng(SEED_SKEW, seed).standard_normal(size=E, dtype=np.float32)
        router[:, 0] = f32_to_bf16_bits(b)
    L["router_w"] = router
    L["skew"] = bool(skew)

    L["gu_codes"] = _rng(seed, _TAG_GU_CODES).integers(0, 256, size=(E, 2 * I, H // 2), dtype=np.uint8)
    L["dn_codes"] = _rng(seed, _TAG_DN_CODES).integers(0, 256, size=(E, H, I // 2), dtype=np.uint8)
    if fmt == FMT_INT4:
        def scales(tag, shape):
            u = _rng(seed, tag).random(size=shape)
            return f32_to_bf16_bits((0.004 * (1.0 + u)).astype(np.float32))
        L["gu_scales"] = scales(_TAG_GU_SCALES, (E, 2 * I, H // 128))
        L["dn_scales"] = scales(_TAG_DN_SCALES, (E, H, I // 128))
        L["gu_tscale"] = None
        L["dn_tscale"] = None
    else:
        def scales(tag, shape):
            e = _rng(seed, tag).integers(-4, 3, size=shape)          # 2^e, e in {-4..2}
            return ((e + 7) << 3).astype(np.uint8)                    # E4M3: exponent field e+7, mantissa 0
        L["gu_scales"] = scales(_TAG_GU_SCALES, (E, 2 * I, H // 16))
        L["dn_scales"] = scales(_TAG_DN_SCALES, (E, H, I // 16))
        L["gu_tscale"] = np.full((E, 2), 0.01, dtype=np.float32)
        L["dn_tscale"] = np.full((E,), 0.01, dtype=np.float32)

    L["sh_gu"] = _bf16_normal(_rng(seed, _TAG_SH_GU), (2 * Is, H), W_STD)
    L["sh_dn"] = _bf16_normal(_rng(seed, _TAG_SH_DN), (H, Is), W_STD)
    return L


def make_master_weights(E: int, *, H: int = H_DEFAULT, I: int = I_DEFAULT, seed: int = SEED_WEIGHTS,
                        outliers: int = 0) -> dict:
    """bf16 expert weights before quantisation (the input of the weight-preparation entry points):
    gu u16 [E][2I][H] (gate rows then up rows) and dn u16 [E][H][I], normal with std W_STD; with
    `outliers` > 0 that many entries per row are set to +-30 W_STD (heavy-tailed rows)."""
    out = {}
    for name, tag, shape in (("gu", _TAG_MASTER_GU, (E, 2 * I, H)), ("dn", _TAG_MASTER_DN, (E, H, I))):
        w = _rng(seed, tag).standard_normal(size=shape, dtype=np.float32) * np.float32(W_STD)
        if outliers:
            r = _rng(seed, _TAG_MASTER_OUT, tag)
            idx = r.integers(0, shape[-1], size=shape[:-1] + (outliers,))
            val = r.choice(np.float32([-30.0, 30.0]), size=idx.shape) * np.float32(W_STD)
            np.put_along_axis(w, idx, val, axis=-1)
        out[name] = f32_to_bf16_bits(w)
    return out


def x_row(r: int, d: int, H: int = H_DEFAULT, skew: bool = False) -> np.ndarray:
    """Token row r, draw d, as bf16 bits [H]."""
    v = _rng(SEED_X, r, d).standard_normal(size=H, dtype=np.float32) * np.float32(X_STD)
    row = f32_to_bf16_bits(v)
    if skew:
        row[0] = 0x3F80          # bf16 1.0 carries the folded router bias
    return row


def make_x(T: int, *, H: int = H_DEFAULT, skew: bool = False, redraws: dict | None = None,
           first_row: int = 0) -> np.ndarray:
    """Activations as bf16 bits [T][H]; row t is token row first_row+t.

    `redraws` maps a token row index to the number of times it is redrawn."""
    redraws = redraws or {}
    out = np.empty((T, H), dtype=np.uint16)
    for t in range(T):
        r = first_row + t
        out[t] = x_row(r, int(redraws.get(r, 0)), H, skew)
    return out


def layer_nbytes(L: dict) -> int:
    """Bytes of all weight arrays of a layer."""
    n = 0
    for k in ("router_w", "gu_codes", "gu_scales", "gu_tscale", "dn_codes", "dn_scales", "dn_tscale",
              "sh_gu", "sh_dn"):
        if L.get(k) is not None:
            n += L[k].nbytes
    return n


def expert_nbytes(L: dict) -> int:
    """Bytes one routed expert streams (codes, scales and tensor scales of gate|up and down)."""
    E = L["E"]
    n = (L["gu_codes"].nbytes + L["gu_scales"].nbytes + L["dn_codes"].nbytes + L["dn_scales"].nbytes) // E
    if L.get("gu_tscale") is not None:
        n += (L["gu_tscale"].nbytes + L["dn_tscale"].nbytes) // E
    return n


def redraw_table(E: int, seed: int = SEED_WEIGHTS, skew: bool = False) -> dict:
    """Redraw counts per token row for the router drawn with (E, seed, skew), from the table shipped
    with this package (redraws.json beside this module; written by tests/golden/make_redraws.py)."""
    import json
    import os
    path = os.path.join(os.path.dirname(os.path.abspath(__file__)), "redraws.json")
    with open(path) as f:
        tab = json.load(f)["tables"]
    key = f"E{E}_seed{seed}" + ("_skew" if skew else "")
    if key not in tab:
        raise KeyError(f"no redraw table for {key}")
    return {int(k): v for k, v in tab[key]["redraws"].items()}


def make_workload_x(T: int, E: int, *, seed: int = SEED_WEIGHTS, skew: bool = False, H: int = H_DEFAULT):
    """Activations of the standard workloads: rows 0..T-1 with the committed redraws applied."""
    return make_x(T, H=H, skew=skew, redraws=redraw_table(E, seed, skew))
