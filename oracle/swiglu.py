"""SwiGLU output preparation between the expert up- and down-projections.

TEST INFRASTRUCTURE ONLY (see oracle/__init__.py).

"Hardware-Native Joint Sparse-Quantization for Trillion-Scale Mixture-of-Experts"
(paperlayer.ai summary), §D.1 (p.19): the serving integration fuses SwiGLU output
preparation for the second expert GEMM.  The up-projection's fused weight holds the gate
rows [0, I) and the up rows [I, 2I); with y = the up-projection's output row,
    h[f] = silu(y[f]) * y[I + f],   silu(x) = x * sigmoid(x) = x / (1 + exp(-x)),
computed here in float64.  h then goes through the same NVFP4 block rule as the activations
(oracle/quant.py) with a given tensor scale, to become the down-projection's input.
"""
from __future__ import annotations

import numpy as np

SILU_SLOPE_MAX = 1.1   # sup |silu'(x)| = 1.0998... (at x = 2.3994...)


def silu(x: np.ndarray) -> np.ndarray:
    x = np.asarray(x, dtype=np.float64)
    return x / (1.0 + np.exp(-x))


def swiglu_rows(y: np.ndarray) -> np.ndarray:
    """y float64 [R, 2I] (gate | up) -> h float64 [R, I]."""
    y = np.asarray(y, dtype=np.float64)
    I = y.shape[1] // 2
    return silu(y[:, :I]) * y[:, I:]


def swiglu_error_bound(y: np.ndarray, tau: np.ndarray) -> np.ndarray:
    """Bound on |h(y') - h(y)| for every y' with |y' - y| <= tau elementwise (both [R, 2I]):
    |silu(g') u' - silu(g) u| <= (|silu(g)| + S tau_g) tau_u + S tau_g |u|, S = sup |silu'|."""
    y = np.asarray(y, dtype=np.float64)
    tau = np.asarray(tau, dtype=np.float64)
    I = y.shape[1] // 2
    g, u, tg, tu = y[:, :I], y[:, I:], tau[:, :I], tau[:, I:]
    return (np.abs(silu(g)) + SILU_SLOPE_MAX * tg) * tu + SILU_SLOPE_MAX * tg * np.abs(u)
