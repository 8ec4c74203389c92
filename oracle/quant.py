"""Activation quantization to NVFP4 (W4A4's activation side), canonical form.

TEST INFRASTRUCTURE ONLY (see oracle/__init__.py).

Source: "Hardware-Native Joint Sparse-Quantization for Trillion-Scale
Mixture-of-Experts" (paperlayer.ai summary): §D.1 "Implementation details"
(p.19) -- activation quantization forms 32-element scale blocks and is fused
with dispatch for the first expert GEMM; §3.4 (pp.5-6) -- weights and
quantized activations are packed in corresponding scale blocks.

Reading used here: the tensor scale s_x = amax(|X|) / 2688 over all of X (or a
caller-supplied value), then the same per-block rule as the weights.  Each
token is quantized once and its codes are copied to the token's k routed rows;
this equals permute-then-quantize because blocks never cross rows and the
amax of X equals the amax of any row permutation of it.
"""
from __future__ import annotations

import numpy as np

from .pack import block_quantize, tensor_scale


def act_tensor_scale(x: np.ndarray) -> np.float32:
    """s_x = fl(max|X| / 2688), or 1 when X is all zeros.  X is given as fp32 (exact from bf16)."""
    x = np.asarray(x, dtype=np.float32)
    return tensor_scale(np.max(np.abs(x)) if x.size else np.float32(0))


def quantize_rows(x: np.ndarray, sf_block: int, s_x: np.float32):
    """X fp32 [T, K] -> (codes [T, K] one E2M1 code per byte, scales [T, K/sf_block])."""
    x = np.asarray(x, dtype=np.float32)
    T, K = x.shape
    blocks = x.reshape(T, K // sf_block, sf_block)
    blk_amax = np.max(np.abs(blocks), axis=-1)
    q, sc = block_quantize(blocks, blk_amax, s_x)
    return q.reshape(T, K), sc


def quantize_routed(x: np.ndarray, sf_block: int, perm_src: np.ndarray | None, top_k: int,
                    s_x: np.float32 | None = None):
    """Quantize tokens and lay them out in routed (expert-grouped) row order.

    perm_src[r] = flat index t*k + j of routed row r (None: identity, one row per token).
    Returns (codes [R, K], scales [R, K/sf_block], s_x).
    """
    if s_x is None:
        s_x = act_tensor_scale(x)
    q, sc = quantize_rows(x, sf_block, s_x)
    if perm_src is None:
        return q, sc, np.float32(s_x)
    tok = np.asarray(perm_src, dtype=np.int64) // top_k
    return q[tok], sc[tok], np.float32(s_x)


def decode_rows(codes: np.ndarray, scales: np.ndarray, sf_block: int) -> np.ndarray:
    """Dequantized activations fp64 [R, K] without the tensor scale."""
    from .codecs import e2m1_decode, ue4m3_decode
    R, K = codes.shape
    v = e2m1_decode(codes).reshape(R, K // sf_block, sf_block) * ue4m3_decode(scales)[..., None]
    return v.reshape(R, K)
