"""Weight packing into paired 4:8 NVFP4 and dense NVFP4, in canonical row-major form.

TEST INFRASTRUCTURE ONLY (see oracle/__init__.py).

Source: "Hardware-Native Joint Sparse-Quantization for Trillion-Scale
Mixture-of-Experts" (paperlayer.ai summary):
  * App. A "Blackwell paired 4:8 NVFP4" (p.14, Fig. 3 p.15): every aligned
    group of eight weights keeps two of its four adjacent pairs (six permitted
    patterns); retained values lie on the E2M1 grid; the 16 retained values of
    a 32-weight block share one UE4M3 scale.
  * App. A "Storage layout" (p.15): four retained values plus a pattern index
    per eight-weight group and one UE4M3 scale per 32-weight block.
  * §3.4 "Implementation details" (p.5): E2M1 values, sparse metadata and a
    UE4M3 scale per 32 logical weights are packed together.
The pages learn the support; here it is chosen by pair magnitude (the plain
reading used throughout this repository): the two pairs with the largest
energy w0^2 + w1^2 (computed in fp32, no fused multiply-add) are kept, a tie
going to the lower pair index.  The per-expert FP32 tensor scale is the usual
NVFP4 two-level rule s_w = amax / (6 * 448), or 1 when amax is 0.

Every fp32 operation is done in numpy float32, i.e. IEEE single precision with
one rounding per operation, in the order written below.
"""
from __future__ import annotations

import numpy as np

from .codecs import e2m1_encode, ue4m3_encode, ue4m3_decode

FP4_MAX = np.float32(6.0)
UE4M3_MAX = np.float32(448.0)
TENSOR_SCALE_DEN = np.float32(6.0 * 448.0)   # 2688


def pair_energies(w: np.ndarray) -> np.ndarray:
    """w fp32 [..., K] -> m fp32 [..., K/8, 4]: m_p = fl(fl(w0*w0) + fl(w1*w1))."""
    w = np.asarray(w, dtype=np.float32)
    p = w.reshape(*w.shape[:-1], w.shape[-1] // 8, 4, 2)
    sq0 = p[..., 0] * p[..., 0]
    sq1 = p[..., 1] * p[..., 1]
    return sq0 + sq1


def select_pairs(w: np.ndarray) -> np.ndarray:
    """Kept pair indices int [..., K/8, 2] (i0 < i1): the two largest energies, ties -> lower index."""
    m = pair_energies(w)
    order = np.argsort(-m, axis=-1, kind="stable")       # stable: equal energies keep index order
    keep = np.sort(order[..., :2], axis=-1)
    return keep


def pattern_code(keep: np.ndarray) -> np.ndarray:
    """4-bit metadata per 8-group: i0 in bits 0-1, i1 in bits 2-3."""
    return (keep[..., 0] | (keep[..., 1] << 2)).astype(np.uint8)


def pattern_pairs(code: np.ndarray) -> np.ndarray:
    """Inverse of pattern_code: [..., 2] pair indices."""
    c = np.asarray(code).astype(np.int64)
    return np.stack([c & 3, (c >> 2) & 3], axis=-1)


def prune(w: np.ndarray, keep: np.ndarray) -> np.ndarray:
    """W' = W with the two non-kept pairs of every 8-group set to zero."""
    w = np.asarray(w, dtype=np.float32)
    p = w.reshape(*w.shape[:-1], w.shape[-1] // 8, 4, 2).copy()
    mask = np.zeros(p.shape[:-1], dtype=bool)
    np.put_along_axis(mask, keep, True, axis=-1)
    p[~mask] = 0.0
    return p.reshape(w.shape)


def kept_values(w: np.ndarray, keep: np.ndarray) -> np.ndarray:
    """The four retained values of each 8-group in K order: [..., K/2]."""
    w = np.asarray(w, dtype=np.float32)
    p = w.reshape(*w.shape[:-1], w.shape[-1] // 8, 4, 2)
    kept = np.take_along_axis(p, keep[..., None].repeat(2, axis=-1), axis=-2)   # [..., G, 2, 2]
    return kept.reshape(*w.shape[:-1], w.shape[-1] // 2)


def tensor_scale(amax: np.float32) -> np.float32:
    """s = fl(amax / 2688), or 1 when amax is 0."""
    amax = np.float32(amax)
    if amax == 0:
        return np.float32(1.0)
    return np.float32(amax / TENSOR_SCALE_DEN)


def block_quantize(v: np.ndarray, blk_amax: np.ndarray, s: np.float32):
    """Shared block rule (weights and activations).

    v        fp32 [..., nb, L]  values of each block to encode
    blk_amax fp32 [..., nb]     amax over the block (pruned positions count as 0)
    s        fp32               tensor scale
    Returns (codes uint8 [..., nb, L], scales uint8 [..., nb]).
      sc  = UE4M3(fl(b / fl(6*s)))
      d   = fl(dec(sc) * s);  inv = 0 if d == 0 else fl(1/d)
      q   = E2M1(fl(v * inv))
    """
    s = np.float32(s)
    six_s = np.float32(FP4_MAX * s)
    ratio = (np.asarray(blk_amax, dtype=np.float32) / six_s).astype(np.float32)
    sc = ue4m3_encode(ratio)
    d = (ue4m3_decode(sc).astype(np.float32) * s).astype(np.float32)
    with np.errstate(divide="ignore"):
        inv = np.where(d == 0, np.float32(0.0), (np.float32(1.0) / d)).astype(np.float32)
    q = e2m1_encode((np.asarray(v, dtype=np.float32) * inv[..., None]).astype(np.float32))
    return q, sc


def pack_sparse_expert(w: np.ndarray):
    """One expert W_e fp32 [N, K] -> (codes [N, K/2], patterns [N, K/8], scales [N, K/32], s_w).

    codes: one E2M1 code per byte, the retained values in K order.
    patterns: 4-bit pattern code per 8-group.  scales: UE4M3 per 32 logical weights.
    """
    w = np.asarray(w, dtype=np.float32)
    N, K = w.shape
    assert K % 32 == 0
    keep = select_pairs(w)                                   # [N, K/8, 2]
    wp = prune(w, keep)
    s_w = tensor_scale(np.max(np.abs(wp)) if wp.size else np.float32(0))
    blk_amax = np.max(np.abs(wp).reshape(N, K // 32, 32), axis=-1)
    kv = kept_values(w, keep).reshape(N, K // 32, 16)        # 16 retained values per 32-block
    q, sc = block_quantize(kv, blk_amax, s_w)
    return q.reshape(N, K // 2), pattern_code(keep), sc, s_w


def pack_dense_expert(w: np.ndarray, sf_block: int = 16):
    """Dense NVFP4 control: W_e fp32 [N, K] -> (codes [N, K], scales [N, K/sf_block], s_w)."""
    w = np.asarray(w, dtype=np.float32)
    N, K = w.shape
    assert K % sf_block == 0
    s_w = tensor_scale(np.max(np.abs(w)) if w.size else np.float32(0))
    blocks = w.reshape(N, K // sf_block, sf_block)
    blk_amax = np.max(np.abs(blocks), axis=-1)
    q, sc = block_quantize(blocks, blk_amax, s_w)
    return q.reshape(N, K), sc, s_w


def decode_sparse_expert(codes: np.ndarray, patterns: np.ndarray, scales: np.ndarray) -> np.ndarray:
    """Dequantized logical weights [N, K] in fp64 WITHOUT the tensor scale; pruned slots are 0."""
    from .codecs import e2m1_decode
    N, Kh = codes.shape
    K = 2 * Kh
    vals = e2m1_decode(codes).reshape(N, K // 32, 16) * ue4m3_decode(scales)[..., None]
    vals = vals.reshape(N, K // 8, 2, 2)                     # [N, G, kept pair slot, 2]
    out = np.zeros((N, K // 8, 4, 2), dtype=np.float64)
    pairs = pattern_pairs(patterns)                          # [N, G, 2]
    np.put_along_axis(out, pairs[..., None].repeat(2, axis=-1), vals, axis=-2)
    return out.reshape(N, K)


def decode_dense_expert(codes: np.ndarray, scales: np.ndarray, sf_block: int) -> np.ndarray:
    """Dequantized dense weights [N, K] in fp64 without the tensor scale."""
    from .codecs import e2m1_decode
    N, K = codes.shape
    v = e2m1_decode(codes).reshape(N, K // sf_block, sf_block) * ue4m3_decode(scales)[..., None]
    return v.reshape(N, K)
