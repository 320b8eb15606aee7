"""fp64 CPU oracle of one Flint mixture-of-experts layer forward.

TEST INFRASTRUCTURE ONLY. Nothing on the product path may import or call this
module; it exists so that tests, the package's smoke check and the benchmark's
CPU-baseline leg can check the CUDA path against a plain, slow, obviously
correct restatement of what the layer computes. It shares no code with the
CUDA library: it decodes every storage format itself, and it applies the
Hadamard rotation as a dense 128x128 matrix product, not as a butterfly.

What the layer computes, and where the pages say so:

* Router: one bf16 row per routed expert, widened exactly and used in FP32 or
  better (WaveCut/Flint-UD-Q4_K_XL-NInfer-v3, "What is inside": router rows;
  kekzle/Flint-NVFP4, "What is in the files": the 47 routers are BF16). The
  score of expert e is the sigmoid of its logit (midagedev/bloomery issue #632,
  description: sigmoid router, 256 experts, 6 per token).
* Selection: the top 6 scores with no correction bias added (issue #632,
  design-round comment: the header shows no router correction bias, an
  unbiased sigmoid256/top6). Ties are broken towards the lower expert index;
  the six slots are then listed by ascending expert id.
* Normalisation: w_k = s_k / max(sum of the selected scores, 2^-14)
  (issue #632, readiness-check and host-policy comments: the SelectedSumFloor
  policy; NInfer README, "What is inside": sigmoid scores renormalised).
* Routed expert: SwiGLU, gate and up rows [2*512][2048] in one bank (gate rows
  first), down [2048][512] (NInfer README, "What is inside", MoE row).
* int4 format: signed 4-bit codes, one bf16 scale per 128 of K, stored against
  a 128-wide Hadamard rotation (Aijuus/flint-w4exp, summary table, weights
  row). The stored matrix is W_q = W * blockdiag(Hn) with Hn = H_128/sqrt(128)
  (Sylvester order), so W x = W_q (Hn x) per 128-segment of K; the same holds
  for the down projection's input, the SwiGLU intermediate.
* NVFP4 format: E2M1 codes two per byte, an E4M3 scale per 16 columns and an
  F32 tensor scale per Linear; value = code x block scale x tensor scale
  (kekzle/Flint-NVFP4, "What is in the files", Layout and lm_head rows).
  Activations stay 16-bit (W4A16, same page, Declaration row).
* Shared expert: an ungated bf16 SwiGLU of width 1024 added with weight 1
  (Aijuus/flint-w4exp, model summary and weights row; NInfer README, shared
  expert row; the three Linears per shared expert are in the quantized-Linear
  count of kekzle/Flint-NVFP4, "What is in the files").
* Combine: y = routed_scale * sum_k w_k * expert_k(x) + shared(x), computed here
  in fp64 without rounding; routed_scale is 1 (no scaling is named anywhere).
* W4A4 (NVFP4 weights only): the routed experts' inputs, x and the SwiGLU
  intermediate h, are themselves quantised to NVFP4 before each projection
  (kekzle/Flint-NVFP4, evaluation table and serving notes: imp quantises the
  activations in prefill, W4A4). Reading: per row (a token's x, a slot's h) an
  F32 scale amax / (6 * 448), an E4M3 scale per 16 values along K and E2M1
  codes, each decision taken in fp32 (quantize_act_nvfp4); the products and
  sums after it stay fp64 here.

Storage conventions (the pages do not fix them; readings listed in the design
notes): int4 codes are two's complement with the low nibble holding the even K
index; E2M1 has its sign in bit 3 and the low nibble holds the even column;
E4M3 is the fn variant (bias 7, no infinities); all matrices are row-major
[out][in]; permuted rows are ordered by (expert ascending, token ascending).
"""

from __future__ import annotations

import math

import numpy as np

NORM_FLOOR = 2.0 ** -14
TOP_K = 6
GROUP = 128          # int4 scale group and Hadamard width along K
NVFP4_BLOCK = 16


# ----------------------------------------------------------------------------------------------
# storage formats
# ----------------------------------------------------------------------------------------------

def bf16_to_f64(bits) -> np.ndarray:
    """bf16 bit patterns (uint16) -> float64, exactly (bf16 is the top half of an IEEE float32)."""
    b = np.asarray(bits, dtype=np.uint16).astype(np.uint32) << 16
    with np.errstate(invalid="ignore"):
        return b.view(np.float32).astype(np.float64)


def e4m3fn_to_f64(bits) -> np.ndarray:
    """E4M3 (fn variant) bytes -> float64 from the format definition: sign bit 7, exponent bits
    6..3 with bias 7, mantissa bits 2..0; exponent field 0 is subnormal (m/8 * 2^-6); the pattern
    with all exponent and mantissa bits set is NaN; there are no infinities."""
    b = np.asarray(bits, dtype=np.int64)
    s = np.where(b & 0x80, -1.0, 1.0)
    e = (b >> 3) & 0xF
    m = (b & 0x7).astype(np.float64)
    normal = (1.0 + m / 8.0) * np.exp2(e.astype(np.float64) - 7.0)
    sub = (m / 8.0) * 2.0 ** -6
    v = s * np.where(e == 0, sub, normal)
    return np.where((b & 0x7F) == 0x7F, np.nan, v)


def e2m1_to_f64(nibbles) -> np.ndarray:
    """E2M1 4-bit codes -> float64: sign bit 3, exponent bits 2..1 (bias 1), mantissa bit 0.
    Exponent 0 is subnormal (m * 0.5); magnitudes are 0, .5, 1, 1.5, 2, 3, 4, 6."""
    n = np.asarray(nibbles, dtype=np.int64)
    s = np.where(n & 0x8, -1.0, 1.0)
    e = (n >> 1) & 0x3
    m = (n & 0x1).astype(np.float64)
    mag = np.where(e == 0, 0.5 * m, (1.0 + 0.5 * m) * np.exp2(e.astype(np.float64) - 1.0))
    return s * mag


def unpack_nibbles(codes_u8) -> np.ndarray:
    """u8 [..., K/2] -> int [..., K] of raw 4-bit fields; the low nibble is the even index."""
    c = np.asarray(codes_u8, dtype=np.uint8)
    out = np.empty(c.shape[:-1] + (2 * c.shape[-1],), dtype=np.int64)
    out[..., 0::2] = c & 0xF
    out[..., 1::2] = c >> 4
    return out


def int4_values(codes_u8) -> np.ndarray:
    """Two's-complement 4-bit codes -> integers in [-8, 7]."""
    n = unpack_nibbles(codes_u8)
    return np.where(n >= 8, n - 16, n)


def dequant_int4(codes_u8, scales_bf16, tscale: float | None = None) -> np.ndarray:
    """int4 g128 matrix [N][K] in fp64: W[n, k] = c[n, k] * s[n, k // 128] (* optional tensor scale)."""
    c = int4_values(codes_u8).astype(np.float64)
    s = bf16_to_f64(scales_bf16)
    W = c * np.repeat(s, GROUP, axis=-1)
    if tscale is not None:
        W = W * float(np.float32(tscale))
    return W


def dequant_nvfp4(codes_u8, scales_e4m3, tscale) -> np.ndarray:
    """NVFP4 matrix [N][K] in fp64: W[n, k] = e2m1(c[n, k]) * e4m3(s[n, k // 16]) * f32(tscale)."""
    v = e2m1_to_f64(unpack_nibbles(codes_u8))
    s = e4m3fn_to_f64(scales_e4m3)
    return v * np.repeat(s, NVFP4_BLOCK, axis=-1) * float(np.float32(tscale))


# ----------------------------------------------------------------------------------------------
# Hadamard rotation
# ----------------------------------------------------------------------------------------------

def hadamard_normalized(n: int = GROUP) -> np.ndarray:
    """Dense Sylvester Hadamard matrix of order n (natural order), scaled by 1/sqrt(n):
    H[i, j] = (-1)^popcount(i & j) / sqrt(n). Symmetric and orthogonal, so Hn @ Hn = I."""
    i = np.arange(n)
    par = np.vectorize(lambda v: bin(int(v)).count("1") & 1)(i[:, None] & i[None, :])
    return np.where(par == 1, -1.0, 1.0) / math.sqrt(n)


_HN = None


def _hn() -> np.ndarray:
    global _HN
    if _HN is None:
        _HN = hadamard_normalized(GROUP)
    return _HN


def rotate_segments(v: np.ndarray) -> np.ndarray:
    """Apply blockdiag(Hn, Hn, ...) along the last axis: every 128-wide segment is multiplied by Hn."""
    v = np.asarray(v, dtype=np.float64)
    n = v.shape[-1]
    assert n % GROUP == 0
    seg = v.reshape(v.shape[:-1] + (n // GROUP, GROUP))
    return (seg @ _hn().T).reshape(v.shape)


# ----------------------------------------------------------------------------------------------
# router
# ----------------------------------------------------------------------------------------------

def sigmoid(z):
    return 1.0 / (1.0 + np.exp(-np.asarray(z, dtype=np.float64)))


def route(logits: np.ndarray, top_k: int = TOP_K, floor: float = NORM_FLOOR) -> dict:
    """Unbiased sigmoid top-k routing with the SelectedSumFloor normalisation.

    logits [T][E] -> ids [T][top_k] (ascending expert id), w [T][top_k] (weights in the same slot
    order), scores [T][E], and gap [T] = (k-th best score) - ((k+1)-th best score)."""
    logits = np.asarray(logits, dtype=np.float64)
    T, E = logits.shape
    s = sigmoid(logits)
    ids = np.empty((T, top_k), dtype=np.int32)
    w = np.empty((T, top_k), dtype=np.float64)
    gap = np.full((T,), np.inf)
    for t in range(T):
        order = sorted(range(E), key=lambda e: (-s[t, e], e))     # score descending, index ascending
        chosen = sorted(order[:top_k])                            # slots by ascending expert id
        ssum = sum(s[t, e] for e in chosen)
        denom = max(ssum, floor)
        ids[t] = chosen
        w[t] = [s[t, e] / denom for e in chosen]
        if top_k < E:
            gap[t] = s[t, order[top_k - 1]] - s[t, order[top_k]]
    return {"ids": ids, "w": w, "scores": s, "gap": gap}


def permutation(ids: np.ndarray, E: int) -> dict:
    """Expert-major order of the (token, slot) pairs: position p holds t*K+k, ordered by
    (expert ascending, token ascending); counts[e], offsets = exclusive prefix (E+1), inv[t, k] = p."""
    ids = np.asarray(ids)
    T, K = ids.shape
    pairs = [(int(ids[t, k]), t, k) for t in range(T) for k in range(K)]
    pairs.sort()
    perm = np.array([t * K + k for (_, t, k) in pairs], dtype=np.int32).reshape(-1)
    inv = np.empty((T, K), dtype=np.int32)
    for p, (_, t, k) in enumerate(pairs):
        inv[t, k] = p
    counts = np.zeros(E, dtype=np.int32)
    for (e, _, _) in pairs:
        counts[e] += 1
    offsets = np.zeros(E + 1, dtype=np.int32)
    for e in range(E):
        offsets[e + 1] = offsets[e] + counts[e]
    return {"counts": counts, "offsets": offsets, "perm": perm, "inv": inv}


# ----------------------------------------------------------------------------------------------
# experts
# ----------------------------------------------------------------------------------------------

def silu(z):
    z = np.asarray(z, dtype=np.float64)
    return z * sigmoid(z)


def swiglu_mlp(xin: np.ndarray, W_gate: np.ndarray, W_up: np.ndarray, W_down: np.ndarray,
               rotated: bool) -> dict:
    """One SwiGLU MLP on rows xin [n][H] with fp64 weights.

    rotated=True applies the stored-against-Hadamard convention: the input and the SwiGLU
    intermediate are each rotated per 128-segment before the matrix that consumes them."""
    xr = rotate_segments(xin) if rotated else np.asarray(xin, dtype=np.float64)
    g = xr @ W_gate.T
    u = xr @ W_up.T
    h = silu(g) * u
    hr = rotate_segments(h) if rotated else h
    out = hr @ W_down.T
    return {"x_in": xr, "g": g, "u": u, "h": h, "h_in": hr, "out": out}


def expert_weights(L: dict, e: int) -> tuple[np.ndarray, np.ndarray, np.ndarray]:
    """fp64 (gate [I][H], up [I][H], down [H][I]) of routed expert e."""
    I = L["I"]
    if L["fmt"] == "int4":
        gts = None if L.get("gu_tscale") is None else L["gu_tscale"][e]
        dts = None if L.get("dn_tscale") is None else L["dn_tscale"][e]
        gu_g = dequant_int4(L["gu_codes"][e, :I], L["gu_scales"][e, :I], None if gts is None else gts[0])
        gu_u = dequant_int4(L["gu_codes"][e, I:], L["gu_scales"][e, I:], None if gts is None else gts[1])
        dn = dequant_int4(L["dn_codes"][e], L["dn_scales"][e], dts)
    elif L["fmt"] == "nvfp4":
        gu_g = dequant_nvfp4(L["gu_codes"][e, :I], L["gu_scales"][e, :I], L["gu_tscale"][e, 0])
        gu_u = dequant_nvfp4(L["gu_codes"][e, I:], L["gu_scales"][e, I:], L["gu_tscale"][e, 1])
        dn = dequant_nvfp4(L["dn_codes"][e], L["dn_scales"][e], L["dn_tscale"][e])
    else:
        raise ValueError(L["fmt"])
    return gu_g, gu_u, dn


def shared_weights(L: dict) -> tuple[np.ndarray, np.ndarray, np.ndarray]:
    Is = L["Is"]
    S = bf16_to_f64(L["sh_gu"])
    return S[:Is], S[Is:], bf16_to_f64(L["sh_dn"])


# ----------------------------------------------------------------------------------------------
# activation quantisation (W4A4)
# ----------------------------------------------------------------------------------------------

_E2M1_MIDS = np.array([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0])


def _e2m1_nearest_even(a):
    """|value| (non-negative) -> E2M1 magnitude code 0..7: nearest of 0, .5, 1, 1.5, 2, 3, 4, 6; at a
    midpoint the even code; above 6 saturates to 6."""
    a = np.asarray(a, dtype=np.float64)
    code = np.zeros(a.shape, dtype=np.int64)
    for i, mid in enumerate(_E2M1_MIDS):
        code = np.where((a > mid) | ((a == mid) & ((i + 1) % 2 == 0)), i + 1, code)
    return code


def _e4m3_nearest_even_pos(x):
    """Non-negative fp32 value -> E4M3 (fn) byte, nearest with ties to even, saturating at 448."""
    x = np.asarray(x, dtype=np.float64)
    grid = e4m3fn_to_f64(np.arange(0x7F))                  # every finite non-negative code, ascending
    idx = np.clip(np.searchsorted(grid, x), 1, 0x7E)
    lo, hi = grid[idx - 1], grid[idx]
    pick_hi = (x - lo > hi - x) | ((x - lo == hi - x) & (idx % 2 == 0))
    code = np.where(pick_hi, idx, idx - 1)
    return np.where(x >= 448.0, 0x7E, code).astype(np.uint8)


def quantize_act_nvfp4(v) -> dict:
    """Rows of activations [R][K] (K a multiple of 16) -> NVFP4 per row, every decision in IEEE fp32 in
    this order: ts = amax / 2688 (1 for an all-zero row); per 16-block sb = E4M3(bm / (6 * ts)) (the
    product and the quotient each rounded to fp32, then nearest-even E4M3, saturating at 448);
    d = sb * ts (rounded to fp32); code = E2M1(v / d) (fp32 quotient, nearest, ties to the even code,
    sign from v; 0 where d = 0). Returns {codes (signed E2M1 values' nibbles) [R][K], scales [R][K/16]
    (E4M3 bytes), ts [R] (f32), values [R][K] (fp64 dequantised: e2m1 x sb x ts)}."""
    v = np.asarray(v, dtype=np.float32)
    R_, K = v.shape
    a = np.abs(v)
    amax = a.max(axis=1)
    ts = np.where(amax > 0, (amax / np.float32(2688.0)).astype(np.float32), np.float32(1.0)).astype(np.float32)
    bm = a.reshape(R_, K // 16, 16).max(axis=2)
    six_ts = (np.float32(6.0) * ts).astype(np.float32)
    q = (bm / six_ts[:, None]).astype(np.float32)
    sb = _e4m3_nearest_even_pos(q)
    sv = e4m3fn_to_f64(sb).astype(np.float32)
    d = (sv * ts[:, None]).astype(np.float32)
    with np.errstate(divide="ignore", invalid="ignore"):
        r = np.where(d[:, :, None] > 0, v.reshape(R_, K // 16, 16) / d[:, :, None], np.float32(0.0)).astype(np.float32)
    mag = _e2m1_nearest_even(np.abs(r))
    sign = np.signbit(v.reshape(R_, K // 16, 16)).astype(np.int64)
    nib = (mag | (sign << 3)).reshape(R_, K)
    vals = e2m1_to_f64(nib) * np.repeat(e4m3fn_to_f64(sb), 16, axis=1) * ts.astype(np.float64)[:, None]
    return {"codes": nib, "scales": sb, "ts": ts, "values": vals}


def moe_forward(L: dict, x_bits: np.ndarray, *, top_k: int = TOP_K, floor: float = NORM_FLOOR,
                routed_scale: float = 1.0, keep: bool = False, expert_override=None, w4a4: bool = False) -> dict:
    """Whole-layer forward in fp64.

    x_bits: bf16 bits [T][H]. Returns y [T][H] (fp64, unrounded), the routing (logits, ids, w,
    gap, counts, offsets, perm, inv) and the shared-expert output ys. With keep=True it also
    returns per-slot intermediates indexed by permuted position p: x_in (the rotated input row),
    h (SwiGLU intermediate before re-rotation), h_in (the down projection's input) and o (the
    expert output before weighting).

    expert_override(e) may return fp64 (gate, up, down) to use instead of the stored codes.
    w4a4 (NVFP4 layers): the routed experts see their inputs quantised per row (quantize_act_nvfp4):
    x before gate|up, and h (rounded to fp32 first, the precision it is formed in) before down."""
    x = bf16_to_f64(x_bits)
    T, H = x.shape
    E = L["E"]
    rotated = L["fmt"] == "int4"
    logits = x @ bf16_to_f64(L["router_w"]).T
    r = route(logits, top_k, floor)
    pm = permutation(r["ids"], E)
    ids, w = r["ids"], r["w"]

    y_routed = np.zeros((T, H))
    slots = {}
    if keep:
        P = T * top_k
        slots = {"x_in": np.zeros((P, H)), "h": np.zeros((P, L["I"])), "h_in": np.zeros((P, L["I"])),
                 "o": np.zeros((P, H))}
    for e in range(E):
        lo, hi = int(pm["offsets"][e]), int(pm["offsets"][e + 1])
        if lo == hi:
            continue
        Wg, Wu, Wd = expert_override(e) if expert_override is not None else expert_weights(L, e)
        flat = pm["perm"][lo:hi]
        toks = flat // top_k
        ks = flat % top_k
        if w4a4:
            if rotated:
                raise ValueError("W4A4 is defined for the NVFP4 format")
            xq = quantize_act_nvfp4(x[toks].astype(np.float32))["values"]
            g, u = xq @ Wg.T, xq @ Wu.T
            h = silu(g) * u
            hq = quantize_act_nvfp4(h.astype(np.float32))["values"]
            res = {"x_in": xq, "g": g, "u": u, "h": h, "h_in": hq, "out": hq @ Wd.T}
        else:
            res = swiglu_mlp(x[toks], Wg, Wu, Wd, rotated)
        for j in range(hi - lo):
            y_routed[toks[j]] += w[toks[j], ks[j]] * res["out"][j]
        if keep:
            slots["x_in"][lo:hi] = res["x_in"]
            slots["h"][lo:hi] = res["h"]
            slots["h_in"][lo:hi] = res["h_in"]
            slots["o"][lo:hi] = res["out"]

    Sg, Su, Sd = shared_weights(L)
    ys = swiglu_mlp(x, Sg, Su, Sd, rotated=False)
    y = routed_scale * y_routed + ys["out"]
    out = {"y": y, "ys": ys["out"], "hs": ys["h"], "logits": logits, **r, **pm}
    if keep:
        out.update(slots)
    return out


def router_gap(L: dict, x_bits: np.ndarray, top_k: int = TOP_K) -> np.ndarray:
    """Per-token gap between the top_k-th and the next sigmoid score, in fp64."""
    x = bf16_to_f64(x_bits)
    s = np.sort(sigmoid(x @ bf16_to_f64(L["router_w"]).T), axis=1)[:, ::-1]
    return s[:, top_k - 1] - s[:, top_k]

# ----------------------------------------------------------------------------------------------
# stack of layers (the model's routed blocks in sequence)
# ----------------------------------------------------------------------------------------------

RMS_EPS = 1e-6


def rmsnorm(x, eps: float = RMS_EPS) -> np.ndarray:
    """Weightless RMSNorm of each row, in fp64: x / sqrt(mean(x^2) + eps).

    The pages name the 47 routed blocks but not the norm between them; this reading takes the
    plain RMSNorm with its weight folded into the next layer (no weight) and eps = 1e-6."""
    x = np.asarray(x, dtype=np.float64)
    return x / np.sqrt(np.mean(x * x, axis=-1, keepdims=True) + eps)


def f64_to_bf16_bits(x) -> np.ndarray:
    """Round fp64 values to bf16 (8 significant bits, round half to even); uint16 bit patterns."""
    x = np.asarray(x, dtype=np.float64)
    m, e = np.frexp(x)                                  # x = m * 2^e, 0.5 <= |m| < 1
    r = np.ldexp(np.rint(np.ldexp(m, 8)), e - 8)        # exact in fp64; a bf16 value, exact in f32
    return (r.astype(np.float32).view(np.uint32) >> 16).astype(np.uint16)


def stack_step(L: dict, x_resid: np.ndarray, *, top_k: int = TOP_K, eps: float = RMS_EPS) -> dict:
    """One layer of a stack on the fp64 residual x: z = bf16(rmsnorm(x)) (the layer's input format),
    y = layer(z), x_next = x + y. Returns z (bf16 bits), y (fp64, unrounded) and x_next."""
    z = f64_to_bf16_bits(rmsnorm(x_resid, eps))
    y = moe_forward(L, z, top_k=top_k)["y"]
    return {"z": z, "y": y, "x_next": np.asarray(x_resid, dtype=np.float64) + y}
