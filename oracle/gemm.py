"""Grouped expert GEMM reference and the error bound it is checked against.

TEST INFRASTRUCTURE ONLY (see oracle/__init__.py).

Source: "Hardware-Native Joint Sparse-Quantization for Trillion-Scale
Mixture-of-Experts" (paperlayer.ai summary): §3.4 (pp.5-6) -- grouped
execution of routing-dependent expert problems in one launch, the sparse
matrix placed as operand A; §D.2 (p.19) -- the dense control differs from the
sparse kernel only in sparsity.

For routed row r of expert e (off[e] <= r < off[e+1]) and output column n:
    y_ref[r, n] = s_x * s_w[e] * sum_k dec(a[r, k]) * dec(w[e, n, k])        (fp64)
    B[r, n]     = s_x * s_w[e] * sum_k |dec(a[r, k]) * dec(w[e, n, k])|
A result y passes when |y - y_ref| <= 2^-10 * B + 1e-6.  The matrix products
use numpy's fp64 matmul as a library primitive.
"""
from __future__ import annotations

import numpy as np

REL_TOL = 2.0 ** -10
ABS_TOL = 1e-6


def expert_of_rows(off: np.ndarray, rows: np.ndarray) -> np.ndarray:
    """Expert index owning each routed row."""
    return np.searchsorted(np.asarray(off, dtype=np.int64), np.asarray(rows), side="right") - 1


def gemm_rows(a_dec: np.ndarray, w_dec: np.ndarray, scale: float):
    """a_dec fp64 [m, K], w_dec fp64 [N, K] -> (y_ref [m, N], bound [m, N]) times the tensor scales."""
    y = (a_dec @ w_dec.T) * scale
    b = (np.abs(a_dec) @ np.abs(w_dec).T) * abs(scale)
    return y, b


def within_tolerance(y: np.ndarray, y_ref: np.ndarray, bound: np.ndarray) -> np.ndarray:
    """Elementwise pass mask for the stated tolerance."""
    return np.abs(np.asarray(y, dtype=np.float64) - y_ref) <= REL_TOL * bound + ABS_TOL


def bf16_half_ulp(v: np.ndarray) -> np.ndarray:
    """Half a bf16 unit in the last place at |v| (the rounding of a bf16 output)."""
    v = np.abs(np.asarray(v, dtype=np.float64))
    e = np.floor(np.log2(np.maximum(v, 2.0 ** -126)))
    return np.where(v == 0, 0.0, 2.0 ** (e - 8))
