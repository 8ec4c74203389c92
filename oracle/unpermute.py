"""Gate-weighted scatter of expert outputs back to tokens.

TEST INFRASTRUCTURE ONLY (see oracle/__init__.py).

Source: "Hardware-Native Joint Sparse-Quantization for Trillion-Scale
Mixture-of-Experts" (paperlayer.ai summary), §D.1 (p.19): dispatch and scatter
around the expert GEMMs.  The gate weighting is the standard MoE combine.

    out[t, :] = bf16( sum_{j<k} g[t, j] * Y[inv_perm[t*k + j], :] )
with the products and the running sum in fp32, j ascending, acc starting at 0
(one rounding per operation), and a round-to-nearest-even conversion to bf16.
"""
from __future__ import annotations

import numpy as np


def bf16_bits_to_f32(bits: np.ndarray) -> np.ndarray:
    """uint16 bf16 bit patterns -> fp32 values (exact)."""
    return (np.asarray(bits, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """fp32 -> bf16 bit patterns with round-to-nearest-even (finite inputs)."""
    u = np.asarray(x, dtype=np.float32).view(np.uint32).astype(np.uint64)
    lsb = (u >> 16) & 1
    r = (u + 0x7FFF + lsb) >> 16
    return r.astype(np.uint16)


def unpermute_scale(y_bits: np.ndarray, inv_perm: np.ndarray, gates: np.ndarray, top_k: int):
    """y_bits uint16 [R, N] (bf16), inv_perm [T*k], gates fp32 [T, k] -> out bf16 bits [T, N]."""
    y = bf16_bits_to_f32(y_bits)
    g = np.asarray(gates, dtype=np.float32)
    T = g.shape[0]
    inv = np.asarray(inv_perm, dtype=np.int64).reshape(T, top_k)
    acc = np.zeros((T, y.shape[1]), dtype=np.float32)
    for j in range(top_k):
        prod = (g[:, j:j + 1] * y[inv[:, j]]).astype(np.float32)
        acc = (acc + prod).astype(np.float32)
    return f32_to_bf16_bits(acc)
