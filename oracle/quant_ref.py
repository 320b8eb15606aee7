"""CPU oracle of the weight preparation that produces the layer's routed-expert formats from bf16
weights: round-to-nearest int4 with one bf16 scale per 128 of K, stored against the 128-wide
Hadamard rotation, and NVFP4 (E2M1 codes, E4M3 scale per 16, F32 scale per Linear).

TEST INFRASTRUCTURE ONLY. Nothing on the product path may import or call this module; it exists so
that tests can check the CUDA quantisers against a plain restatement. It shares no code with the
CUDA library.

What the pages fix, and the readings taken where they are silent:

* int4 (Aijuus/flint-w4exp, summary table, weights row: codes i4, group 128, bf16 scale,
  128-wide Hadamard (fwht128) rotation; the container is produced from the bf16 checkpoint by a
  round-to-nearest conversion, same page, "Serving it" and the 11.7 % error paragraph). The stored
  matrix is the rotated one, W_q = W blockdiag(Hn) with Hn = H_128 / sqrt(128), so the quantiser
  rotates every 128-segment of a row and rounds the result. Readings: the scale is symmetric,
  s = bf16(max |r| / 7) (codes -7..7, -8 unused), and a code is rint(r * (1/s)) clamped to [-8, 7],
  with 1/s the correctly rounded fp32 reciprocal (the quotient formed as one multiplication).
* NVFP4 (kekzle/Flint-NVFP4, "What is in the files": E2M1 codes two per byte, an E4M3 scale per 16
  columns, an F32 tensor scale per Linear; value = code x block scale x tensor scale). Readings:
  tensor scale = amax / (6 * 448), the largest magnitude of the Linear over the largest products of
  the two formats; block scale = E4M3(block amax / (6 * tensor scale)), rounded to nearest even and
  saturated at 448; code = E2M1(w * (1 / (block scale * tensor scale))), nearest grid value, ties
  to the even code, saturated at 6, sign from the sign bit of the product (the reciprocal correctly
  rounded in fp32, so the quotient is one multiplication). An all-zero Linear gets tensor scale 1.

Precision. A quantiser decides integers (codes) from floating point, so this oracle takes every
decision in the precision the kernels use, IEEE fp32 with round-to-nearest for each operation, and
in the same order: the rotation is the Sylvester butterfly by stages h = 1, 2, 4, ..., 64, pairs
(i, i + h) with i & h = 0 becoming (v_i + v_i+h, v_i - v_i+h), then one multiplication by the fp32
nearest to 2^-3.5. Independently of that order, tests compare the butterfly with the dense Hn of the
layer oracle and the codes with exact round-to-nearest bounds.
"""

from __future__ import annotations

import numpy as np

from oracle import flint_moe_ref as R

GROUP = 128
BLOCK = 16
F32_INV_SQRT128 = np.uint32(0x3DB504F3).view(np.float32)   # fp32 nearest to 2^-3.5
E2M1_MAX = 6.0
E4M3_MAX = 448.0


def bf16_to_f32(bits) -> np.ndarray:
    """bf16 bit patterns -> float32 (exact)."""
    return (np.asarray(bits, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


def f32_to_bf16_rne(x) -> np.ndarray:
    """float32 -> bf16 bit patterns, round to nearest even (finite inputs)."""
    u = np.asarray(x, dtype=np.float32).view(np.uint32).astype(np.uint64)
    r = (u + 0x7FFF + ((u >> 16) & 1)) >> 16
    return r.astype(np.uint16)


# ----------------------------------------------------------------------------------------------
# int4 g128 with rotation
# ----------------------------------------------------------------------------------------------

def fwht128_f32(v: np.ndarray) -> np.ndarray:
    """Normalised Sylvester FWHT of every 128-segment of the last axis, in fp32, butterfly order
    h = 1, 2, ..., 64, then one multiplication by fp32(2^-3.5)."""
    v = np.array(v, dtype=np.float32)
    n = v.shape[-1]
    assert n % GROUP == 0
    seg = v.reshape(v.shape[:-1] + (n // GROUP, GROUP))
    h = 1
    while h < GROUP:
        s = seg.reshape(seg.shape[:-1] + (GROUP // (2 * h), 2, h))
        a = s[..., 0, :].copy()
        b = s[..., 1, :].copy()
        s[..., 0, :] = a + b            # float32 + float32: one IEEE rounding
        s[..., 1, :] = a - b
        seg = s.reshape(seg.shape)
        h *= 2
    return (seg * F32_INV_SQRT128).reshape(v.shape)


def quantize_int4_g128(w_bf16, rotate: bool = True) -> dict:
    """bf16 matrix [N][K] (bit patterns) -> {codes u8 [N][K/2], scales bf16 bits [N][K/128]}.
    r = the rotated row (or the row itself); per 128-group: s = bf16(max|r| / 7) and
    c = clamp(rint(r * fp32(1/s)), -8, 7), two's complement, low nibble = even K index; s = 0 gives c = 0."""
    w = bf16_to_f32(w_bf16)
    N, K = w.shape
    assert K % GROUP == 0
    r = fwht128_f32(w) if rotate else w
    g = r.reshape(N, K // GROUP, GROUP)
    m = np.max(np.abs(g), axis=-1)                                   # exact
    sb = f32_to_bf16_rne(m / np.float32(7.0))                        # fp32 division, then bf16
    s = bf16_to_f32(sb)
    with np.errstate(divide="ignore", invalid="ignore"):
        rs = np.float32(1.0) / s                                     # correctly rounded reciprocal
        q = np.rint(g * rs[..., None])                               # fp32 product, ties to even
    q = np.where(s[..., None] > 0, q, 0.0)
    q = np.clip(q, -8, 7).astype(np.int64).reshape(N, K)
    nib = (q & 0xF).astype(np.uint8)
    codes = (nib[:, 0::2] | (nib[:, 1::2] << 4)).astype(np.uint8)
    return {"codes": codes, "scales": sb, "rotated": r}


# ----------------------------------------------------------------------------------------------
# NVFP4
# ----------------------------------------------------------------------------------------------

_E2M1_MID = np.array([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0], dtype=np.float64)   # between grid values


def e2m1_rne(x) -> np.ndarray:
    """float32 -> E2M1 nibble: nearest of 0, .5, 1, 1.5, 2, 3, 4, 6 (ties to the even code,
    saturating at 6); sign bit 3 from the sign bit of x."""
    x = np.asarray(x, dtype=np.float32)
    a = np.abs(x).astype(np.float64)
    code = np.zeros(a.shape, dtype=np.int64)
    for i, mid in enumerate(_E2M1_MID):
        # code i + 1 once a passes the midpoint; exactly at the midpoint only if i + 1 is even
        up = (a > mid) | ((a == mid) & ((i + 1) % 2 == 0))
        code = np.where(up, i + 1, code)
    sign = (x.view(np.uint32) >> 31).astype(np.int64)
    return (code | (sign << 3)).astype(np.uint8)


def e4m3_rne_pos(x) -> np.ndarray:
    """Non-negative float32 -> E4M3 (fn) byte, round to nearest even, saturating at 448."""
    x = np.asarray(x, dtype=np.float64)             # fp32 values, exact in fp64
    out = np.zeros(x.shape, dtype=np.int64)
    sat = x >= E4M3_MAX
    sub = x < 2.0 ** -6
    q_sub = np.rint(x * 2.0 ** 9)                   # subnormal step 2^-9; q = 8 is 2^-6, code 0x08
    with np.errstate(divide="ignore"):
        e = np.floor(np.log2(np.where(sub | sat, 1.0, x)))
    # correct a floor(log2) that lands one off at an exact power of two
    m = np.where(sub | sat, 1.0, x) / np.exp2(e)
    e = np.where(m >= 2.0, e + 1, np.where(m < 1.0, e - 1, e))
    m = np.where(sub | sat, 1.0, x) / np.exp2(e)
    q = np.rint(m * 8.0)                            # 8..16
    e = np.where(q == 16, e + 1, e)
    q = np.where(q == 16, 8, q)
    normal = ((e.astype(np.int64) + 7) << 3) | (q.astype(np.int64) - 8)
    normal = np.minimum(normal, 0x7E)
    out = np.where(sub, q_sub.astype(np.int64), normal)
    out = np.where(sat, 0x7E, out)
    return out.astype(np.uint8)


def quantize_nvfp4(w_bf16) -> dict:
    """bf16 Linear [N][K] (bit patterns) -> {codes u8 [N][K/2], scales e4m3 [N][K/16], tscale f32}.
    fp32 throughout: ts = amax / 2688 (1 for an all-zero Linear); per 16-block sb = E4M3(bm / (6 ts))
    with 6 ts one fp32 product; d = value(sb) * ts; code = E2M1(w * fp32(1/d)) (0 where d = 0)."""
    w = bf16_to_f32(w_bf16)
    N, K = w.shape
    assert K % BLOCK == 0
    amax = np.float32(np.max(np.abs(w))) if w.size else np.float32(0)
    ts = np.float32(amax / np.float32(E2M1_MAX * E4M3_MAX)) if amax > 0 else np.float32(1.0)
    blk = w.reshape(N, K // BLOCK, BLOCK)
    bm = np.max(np.abs(blk), axis=-1)
    six_ts = np.float32(np.float32(E2M1_MAX) * ts)
    sb = e4m3_rne_pos(bm / six_ts)                                    # fp32 division
    sv = R.e4m3fn_to_f64(sb).astype(np.float32)                       # exact
    d = (sv * ts).astype(np.float32)                                  # fp32 product
    with np.errstate(divide="ignore", invalid="ignore"):
        rd = np.float32(1.0) / d                                      # correctly rounded reciprocal
        x = blk * rd[..., None]                                       # fp32 product
    x = np.where(d[..., None] > 0, x, np.float32(0.0)).astype(np.float32)
    nib = e2m1_rne(x).reshape(N, K)
    codes = (nib[:, 0::2] | (nib[:, 1::2] << 4)).astype(np.uint8)
    return {"codes": codes, "scales": sb, "tscale": np.float32(ts)}
