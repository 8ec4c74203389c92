"""Routing permutation: group routed rows by expert (stable counting sort).

TEST INFRASTRUCTURE ONLY (see oracle/__init__.py).

Source: "Hardware-Native Joint Sparse-Quantization for Trillion-Scale
Mixture-of-Experts" (paperlayer.ai summary): §2 "Execution gap" (p.3) --
grouped GEMM executes routing-dependent expert products with different token
counts together; §D.1 (p.19) -- dispatch and scatter around the expert GEMMs.

Definition: the R = T*k pairs (token t, slot j) are numbered f = t*k + j.
Rows of expert e occupy [off[e], off[e+1]) in ascending f.
perm_src[row] = f and inv_perm[f] = row.
"""
from __future__ import annotations

import numpy as np


def route(ids: np.ndarray, E: int):
    """ids int [T, k] in [0, E) -> (off int32 [E+1], perm_src int32 [R], inv_perm int32 [R])."""
    flat = np.asarray(ids, dtype=np.int64).reshape(-1)
    if np.any(flat < 0) or np.any(flat >= E):
        raise ValueError("expert id out of range")
    R = flat.size
    counts = np.zeros(E, dtype=np.int64)
    for e in flat:                                   # histogram
        counts[e] += 1
    off = np.zeros(E + 1, dtype=np.int64)
    off[1:] = np.cumsum(counts)                      # exclusive scan
    cursor = off[:-1].copy()
    perm_src = np.empty(R, dtype=np.int64)
    inv_perm = np.empty(R, dtype=np.int64)
    for f in range(R):                               # stable scatter in ascending f
        e = flat[f]
        row = cursor[e]
        cursor[e] += 1
        perm_src[row] = f
        inv_perm[f] = row
    return off.astype(np.int32), perm_src.astype(np.int32), inv_perm.astype(np.int32)
