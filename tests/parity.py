"""Shared helpers of the GPU parity tests: run the CUDA layer and the fp64 oracle on the same seeded
inputs and compare them.

Tolerance (bf16 output): |y - y_ref| <= 1e-2 * rms(y_ref) + 1e-3 + half a bf16 ulp of y_ref, per
element. The first two terms are the bound the workload states; the last is the rounding every bf16
output must carry (a perfect fp64 layer rounded once to bf16 already exceeds the first two terms at
a few elements of the full-size workloads). Strict-bound violations are counted and reported.
"""

from __future__ import annotations

import numpy as np

from oracle import flint_moe_ref as R

REL_RMS = 1e-2
ABS = 1e-3


def bf16_half_ulp(v: np.ndarray) -> np.ndarray:
    a = np.abs(np.asarray(v, dtype=np.float64))
    _, ex = np.frexp(a)                      # a = m * 2^ex, m in [0.5, 1)
    return np.where(a > 0, np.ldexp(1.0, ex - 9), 0.0)


def y_tolerance(y_ref: np.ndarray):
    rms = float(np.sqrt(np.mean(y_ref ** 2)))
    strict = REL_RMS * rms + ABS
    return strict, strict + bf16_half_ulp(y_ref)


def compare_y(y_bits: np.ndarray, y_ref: np.ndarray) -> dict:
    y = R.bf16_to_f64(y_bits)
    strict, tol = y_tolerance(y_ref)
    err = np.abs(y - y_ref)
    return {"max_err_over_tol": float(np.max(err / tol)), "violations": int(np.sum(err > tol)),
            "strict_violations": int(np.sum(err > strict)), "max_err_over_strict": float(np.max(err / strict)),
            "finite": bool(np.all(np.isfinite(y)))}


def check_routing(dev_routing: dict, ref: dict, T: int, K: int, gap_min: float = 1e-4):
    """ids, offsets and perm bit-exact where the selection is unique (the oracle's k-th/(k+1)-th
    score gap is at least gap_min for every token), weights to fp32 rounding."""
    ids = dev_routing["ids"].cpu().numpy()
    w = dev_routing["w"].cpu().numpy()
    assert np.all(ref["gap"][:T] >= gap_min), "inputs contain near-tied selections"
    np.testing.assert_array_equal(ids, ref["ids"])
    np.testing.assert_array_equal(dev_routing["offsets"].cpu().numpy(), ref["offsets"])
    np.testing.assert_array_equal(dev_routing["perm"].cpu().numpy(), ref["perm"])
    np.testing.assert_allclose(w, ref["w"], rtol=2e-6, atol=1e-7)


def xq_natural_order(xq: np.ndarray, pair_order: bool) -> np.ndarray:
    """Undo the 0,4,1,5,2,6,3,7 storage order of every 8-block."""
    if not pair_order:
        return xq
    b = xq.reshape(xq.shape[:-1] + (-1, 8))
    out = np.empty_like(b)
    out[..., 0:4] = b[..., 0::2]
    out[..., 4:8] = b[..., 1::2]
    return out.reshape(xq.shape)
