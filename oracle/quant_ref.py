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
  s = bf16(max |r| / 7) (codes -7..7, -8 unused), and a code is the integer nearest to r / s
  (ties to even), clamped to [-8, 7].
* NVFP4 (kekzle/Flint-NVFP4, "What is in the files": E2M1 codes two per byte, an E4M3 scale per 16
  columns, an F32 tensor scale per Linear; value = code x block scale x tensor scale). Readings:
  tensor scale = F32(amax / (6 * 448)), the largest magnitude of the Linear over the largest
  products of the two formats; block scale = E4M3(block amax / (6 * tensor scale)), rounded to
  nearest even and saturated at 448; code = E2M1(w / (block scale * tensor scale)), nearest grid
  value, ties to the even code, saturated at 6, sign from the sign of w. An all-zero Linear gets
  tensor scale 1.

Precision. Every quantity is formed in fp64 from the exact bf16 inputs, with the dense Hadamard
matrix of the layer oracle, and rounded once to its storage format; a quotient is a plain fp64
division. This is the definition, not the arithmetic of any kernel: a kernel that forms the same
quantities in fp32 can land on the other side of a rounding boundary where the exact value lies
within its fp32 error of that boundary, and the tests count and bound those positions separately
(`int4_margins`, `nvfp4_margins` below give the distance of every decision from its boundary).
"""

from __future__ import annotations

import numpy as np

from oracle import flint_moe_ref as R

GROUP = 128
BLOCK = 16
E2M1_MAX = 6.0
E4M3_MAX = 448.0
E2M1_GRID = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0])


# ----------------------------------------------------------------------------------------------
# int4 g128 with rotation
# ----------------------------------------------------------------------------------------------

def int4_target(w_bf16, rotate: bool = True) -> np.ndarray:
    """fp64 matrix the int4 codes approximate: each 128-segment of a row times Hn (dense), or the
    row itself."""
    w = R.bf16_to_f64(w_bf16)
    assert w.shape[-1] % GROUP == 0
    return R.rotate_segments(w) if rotate else w


def quantize_int4_g128(w_bf16, rotate: bool = True) -> dict:
    """bf16 matrix [N][K] (bit patterns) -> {codes u8 [N][K/2], scales bf16 bits [N][K/128], rotated}.
    r = the rotated row (or the row itself), fp64; per 128-group: s = bf16(max|r| / 7) and
    c = clamp(nearest integer to r / s, ties to even, -8, 7), two's complement, low nibble = even K
    index; s = 0 gives c = 0."""
    r = int4_target(w_bf16, rotate)
    N, K = r.shape
    g = r.reshape(N, K // GROUP, GROUP)
    m = np.max(np.abs(g), axis=-1)
    sb = R.f64_to_bf16_bits(m / 7.0)
    s = R.bf16_to_f64(sb)
    with np.errstate(divide="ignore", invalid="ignore"):
        q = np.rint(g / s[..., None])                                 # numpy rint: ties to even
    q = np.where(s[..., None] > 0, q, 0.0)
    q = np.clip(q, -8, 7).astype(np.int64).reshape(N, K)
    nib = (q & 0xF).astype(np.uint8)
    codes = (nib[:, 0::2] | (nib[:, 1::2] << 4)).astype(np.uint8)
    return {"codes": codes, "scales": sb, "rotated": r}


def _bf16_midpoint_distance(v: np.ndarray) -> np.ndarray:
    """Relative distance of positive v from the nearest point half-way between two bf16 values."""
    v = np.asarray(v, dtype=np.float64)
    m, e = np.frexp(np.where(v > 0, v, 1.0))                       # v = m 2^e, m in [0.5, 1)
    t = np.ldexp(m, 8)                                             # bf16 step is 1 in these units
    d = np.abs(t - np.floor(t) - 0.5) / t
    return np.where(v > 0, d, np.inf)


def int4_margins(w_bf16, rotate: bool = True) -> dict:
    """Distance of every int4 decision from its rounding boundary, for tests that compare a kernel
    computing in lower precision: `code` [N][K] = |r/s - nearest half-integer| in units of the step
    (0.5 = far), `scale` [N][K/128] = relative distance of max|r|/7 from a bf16 midpoint. Both from
    the fp64 definition above."""
    out = quantize_int4_g128(w_bf16, rotate)
    r = out["rotated"]
    N, K = r.shape
    s = np.repeat(R.bf16_to_f64(out["scales"]), GROUP, axis=1)
    with np.errstate(divide="ignore", invalid="ignore"):
        z = np.where(s > 0, r / s, 0.0)
    code = np.abs(z - np.floor(z) - 0.5)
    m = np.max(np.abs(r.reshape(N, K // GROUP, GROUP)), axis=-1)
    return {"code": code, "scale": _bf16_midpoint_distance(m / 7.0), "ratio": z}


# ----------------------------------------------------------------------------------------------
# NVFP4
# ----------------------------------------------------------------------------------------------

def e2m1_rne(x) -> np.ndarray:
    """Real x -> E2M1 nibble: nearest of 0, .5, 1, 1.5, 2, 3, 4, 6 (ties to the even code, saturating
    at 6); sign bit 3 from the sign of x (including -0)."""
    x = np.asarray(x, dtype=np.float64)
    a = np.abs(x)
    mids = (E2M1_GRID[1:] + E2M1_GRID[:-1]) / 2
    code = np.zeros(a.shape, dtype=np.int64)
    for i, mid in enumerate(mids):
        # code i + 1 once a passes the midpoint; exactly at the midpoint only if i + 1 is even
        up = (a > mid) | ((a == mid) & ((i + 1) % 2 == 0))
        code = np.where(up, i + 1, code)
    sign = np.signbit(x).astype(np.int64)
    return (code | (sign << 3)).astype(np.uint8)


def e4m3_rne_pos(x) -> np.ndarray:
    """Non-negative real -> E4M3 (fn) byte, round to nearest even, saturating at 448."""
    x = np.asarray(x, dtype=np.float64)
    sat = x >= E4M3_MAX
    sub = x < 2.0 ** -6
    q_sub = np.rint(x * 2.0 ** 9)                   # subnormal step 2^-9; q = 8 is 2^-6, code 0x08
    xs = np.where(sub | sat, 1.0, x)
    m, e = np.frexp(xs)                             # xs = m 2^e, m in [0.5, 1)
    q = np.rint(m * 16.0)                           # 8..16: three mantissa bits, ties to even
    e = np.where(q == 16, e + 1, e)
    q = np.where(q == 16, 8, q)
    normal = ((e.astype(np.int64) - 1 + 7) << 3) | (q.astype(np.int64) - 8)
    normal = np.minimum(normal, 0x7E)
    out = np.where(sub, q_sub.astype(np.int64), normal)
    out = np.where(sat, 0x7E, out)
    return out.astype(np.uint8)


def nvfp4_tscale(w_bf16) -> np.float32:
    """F32 tensor scale of one Linear: amax / (6 * 448) rounded once to fp32, 1 for an all-zero one."""
    w = R.bf16_to_f64(w_bf16)
    amax = float(np.max(np.abs(w))) if w.size else 0.0
    return np.float32(amax / (E2M1_MAX * E4M3_MAX)) if amax > 0 else np.float32(1.0)


def quantize_nvfp4(w_bf16) -> dict:
    """bf16 Linear [N][K] (bit patterns) -> {codes u8 [N][K/2], scales e4m3 [N][K/16], tscale f32}.
    fp64 throughout: ts = F32(amax / 2688) (1 for an all-zero Linear); per 16-block
    sb = E4M3(bm / (6 ts)); d = value(sb) ts; code = E2M1(w / d) (0 where d = 0)."""
    w = R.bf16_to_f64(w_bf16)
    N, K = w.shape
    assert K % BLOCK == 0
    ts = nvfp4_tscale(w_bf16)
    tsd = float(ts)
    blk = w.reshape(N, K // BLOCK, BLOCK)
    bm = np.max(np.abs(blk), axis=-1)
    sb = e4m3_rne_pos(bm / (E2M1_MAX * tsd))
    d = R.e4m3fn_to_f64(sb) * tsd                                   # exact in fp64
    with np.errstate(divide="ignore", invalid="ignore"):
        x = np.where(d[..., None] > 0, blk / d[..., None], 0.0 * blk)
    nib = e2m1_rne(x).reshape(N, K)
    codes = (nib[:, 0::2] | (nib[:, 1::2] << 4)).astype(np.uint8)
    return {"codes": codes, "scales": sb, "tscale": ts}


def nvfp4_margins(w_bf16) -> dict:
    """Relative distance of every NVFP4 decision from its rounding boundary (fp64 definition): `scale`
    [N][K/16] for the block scale's E4M3 rounding, `code` [N][K] for the E2M1 rounding."""
    w = R.bf16_to_f64(w_bf16)
    N, K = w.shape
    out = quantize_nvfp4(w_bf16)
    tsd = float(out["tscale"])
    bm = np.max(np.abs(w.reshape(N, K // BLOCK, BLOCK)), axis=-1)
    v = bm / (E2M1_MAX * tsd)
    # E4M3 boundaries: midpoints between consecutive finite non-negative values
    grid = R.e4m3fn_to_f64(np.arange(0x7F))
    mids = (grid[1:] + grid[:-1]) / 2
    dv = np.min(np.abs(v[..., None] - mids), axis=-1) / np.maximum(v, 2.0 ** -12)
    d = np.repeat(R.e4m3fn_to_f64(out["scales"]) * tsd, BLOCK, axis=1)
    with np.errstate(divide="ignore", invalid="ignore"):
        a = np.where(d > 0, np.abs(w) / d, 0.0)
    emids = (E2M1_GRID[1:] + E2M1_GRID[:-1]) / 2
    dc = np.min(np.abs(a[..., None] - emids), axis=-1) / np.maximum(a, 0.25)
    return {"scale": dv, "code": dc}
