"""E2M1 and UE4M3 codecs, written from the number formats' definitions.

TEST INFRASTRUCTURE ONLY (see oracle/__init__.py).

The paper ("Hardware-Native Joint Sparse-Quantization for Trillion-Scale
Mixture-of-Experts", App. A "Blackwell paired 4:8 NVFP4", p.14) stores the
retained weight values on the E2M1 grid and one UE4M3 scale per block; the
formats themselves are the public OCP/NVFP4 ones the paper cites.

E2M1: 4 bits s.e1e0.m, magnitudes {0, .5, 1, 1.5, 2, 3, 4, 6}.
UE4M3: E4M3 without the sign bit: exponent bias 7, subnormals m/8 * 2^-6,
largest finite 448 (code 0x7E); code 0x7F is NaN and is never produced.

Encoders are round-to-nearest onto the grid, ties to the even code, with
saturation at the largest finite magnitude; E2M1 keeps the sign bit of its
input (so -0.1 -> 0x8).  They are written as a plain nearest-point search over
the decoded grid, not as bit tricks.
"""
from __future__ import annotations

import numpy as np

E2M1_MAGNITUDES = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0], dtype=np.float64)


def e2m1_decode(codes) -> np.ndarray:
    """code (low 4 bits) -> value in fp64."""
    c = np.asarray(codes).astype(np.int64) & 0xF
    mag = E2M1_MAGNITUDES[c & 7]
    return np.where(c & 8, -mag, mag)


def ue4m3_decode(codes) -> np.ndarray:
    """code in [0, 127] -> value in fp64 (0x7F decodes to NaN)."""
    c = np.asarray(codes).astype(np.int64) & 0x7F
    e = c >> 3
    m = c & 7
    sub = m.astype(np.float64) / 8.0 * 2.0 ** -6
    nrm = (1.0 + m.astype(np.float64) / 8.0) * np.power(2.0, (e - 7).astype(np.float64))
    v = np.where(e == 0, sub, nrm)
    return np.where(c == 0x7F, np.nan, v)


# The 127 finite UE4M3 values, increasing with the code.
UE4M3_GRID = ue4m3_decode(np.arange(127))


def _nearest_even(x_abs: np.ndarray, grid: np.ndarray) -> np.ndarray:
    """Index of the grid point nearest to each x (grid increasing, x >= 0).

    Values above the last grid point go to the last one (saturation).  On an
    exact tie between two neighbours the even index wins.
    """
    x = np.asarray(x_abs, dtype=np.float64)
    hi = np.searchsorted(grid, x, side="left")          # grid[hi-1] < x <= grid[hi]
    hi = np.clip(hi, 0, len(grid) - 1)
    lo = np.clip(hi - 1, 0, len(grid) - 1)
    d_lo = np.abs(x - grid[lo])
    d_hi = np.abs(grid[hi] - x)
    pick_hi = (d_hi < d_lo) | ((d_hi == d_lo) & (hi % 2 == 0))
    idx = np.where(pick_hi, hi, lo)
    idx = np.where(x >= grid[-1], len(grid) - 1, idx)
    return idx


def e2m1_encode(x) -> np.ndarray:
    """fp32 -> E2M1 code (uint8): RNE onto the grid, ties to even, saturate at 6, sign kept."""
    xf = np.asarray(x, dtype=np.float32)
    mag = _nearest_even(np.abs(xf.astype(np.float64)), E2M1_MAGNITUDES)
    sign = np.signbit(xf).astype(np.int64) << 3
    return (mag | sign).astype(np.uint8)


def ue4m3_encode(x) -> np.ndarray:
    """fp32 >= 0 -> UE4M3 code (uint8): RNE onto the grid, ties to even code, saturate at 448."""
    xf = np.asarray(x, dtype=np.float32).astype(np.float64)
    if np.any(xf < 0) or np.any(~np.isfinite(xf)):
        raise ValueError("ue4m3_encode expects finite non-negative input")
    return _nearest_even(xf, UE4M3_GRID).astype(np.uint8)
