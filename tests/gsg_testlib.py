"""Shared helpers of the GPU parity tests: oracle-side expectations and comparisons.

Both sides are fed the same seeded inputs from grouped_sparse_gemm_b200.inputs; everything
expected is computed by the oracle package alone.
"""
from __future__ import annotations

import numpy as np
import torch

from oracle import gemm as ogemm
from oracle import layout as olayout
from oracle import pack as opack
from oracle import quant as oquant
from oracle import route as oroute


def oracle_pack_sparse(W: np.ndarray):
    """W fp32 [E, N, K] -> (packed bytes in the library's layout, s_w [E], canonical parts per expert)."""
    blocks, sws, canon = [], [], []
    for e in range(W.shape[0]):
        codes, pats, scales, s_w = opack.pack_sparse_expert(W[e])
        blocks.append(olayout.packed_sparse(codes, pats, scales).reshape(-1))
        sws.append(s_w)
        canon.append((codes, pats, scales))
    return np.concatenate(blocks), np.array(sws, dtype=np.float32), canon


def oracle_pack_dense(W: np.ndarray, sf_block: int = 16):
    blocks, sws, canon = [], [], []
    for e in range(W.shape[0]):
        codes, scales, s_w = opack.pack_dense_expert(W[e], sf_block)
        blocks.append(olayout.packed_dense(codes, scales).reshape(-1))
        sws.append(s_w)
        canon.append((codes, scales))
    return np.concatenate(blocks), np.array(sws, dtype=np.float32), canon


def oracle_act(x: np.ndarray, sf_block: int, perm_src, top_k: int, s_x=None):
    """-> (codes bytes [R, K/2], quad scales bytes, s_x, canonical codes [R, K], canonical scales)."""
    q, sc, s = oquant.quantize_routed(x, sf_block, perm_src, top_k, s_x)
    return olayout.pack_act_codes(q), olayout.quad_act_scales(sc).reshape(-1), s, q, sc


def reference_rows(rows, off, a_codes, a_scales, sf_block, w_canon, s_x, s_w, sparse=True, w_sf=32):
    """y_ref and bound for the given routed rows (all N columns), fp64."""
    rows = np.asarray(rows, dtype=np.int64)
    experts = ogemm.expert_of_rows(off, rows)
    first = next(iter(w_canon.values())) if isinstance(w_canon, dict) else w_canon[0]
    N = first[0].shape[0]
    y = np.zeros((rows.size, N))
    b = np.zeros((rows.size, N))
    for e in np.unique(experts):
        sel = np.nonzero(experts == e)[0]
        r = rows[sel]
        ad = oquant.decode_rows(a_codes[r], a_scales[r], sf_block)
        if sparse:
            wd = opack.decode_sparse_expert(*w_canon[e])
        else:
            wd = opack.decode_dense_expert(w_canon[e][0], w_canon[e][1], w_sf)
        ye, be = ogemm.gemm_rows(ad, wd, float(s_x) * float(s_w[e]))
        y[sel] = ye
        b[sel] = be
    return y, b


def assert_gemm_close(y_gpu: torch.Tensor, y_ref: np.ndarray, bound: np.ndarray, what: str = ""):
    """Stated tolerance |y - y_ref| <= 2^-10 B + 1e-6 (fp32 output), plus the bf16 half-ulp when
    the output is bf16 (the result format's own rounding)."""
    y = y_gpu.float().cpu().numpy().astype(np.float64)
    tol = ogemm.REL_TOL * bound + ogemm.ABS_TOL
    if y_gpu.dtype == torch.bfloat16:
        tol = tol + ogemm.bf16_half_ulp(np.abs(y_ref) + tol)
    err = np.abs(y - y_ref)
    bad = err > tol
    if bad.any():
        i = np.argwhere(bad)[:8]
        detail = [(tuple(ix), y[tuple(ix)], y_ref[tuple(ix)], tol[tuple(ix)]) for ix in i]
        raise AssertionError(f"{what}: {bad.sum()} of {bad.size} elements outside tolerance; "
                             f"max err/tol {np.max(err / np.maximum(tol, 1e-30)):.3g}; first {detail}")
    return float(np.max(err / np.maximum(tol, 1e-30))) if err.size else 0.0


def route_np(ids: torch.Tensor, E: int):
    return oroute.route(ids.cpu().numpy(), E)
