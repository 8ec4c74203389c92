"""Storage layouts of the library's packed buffers, written out element by element.

TEST INFRASTRUCTURE ONLY (see oracle/__init__.py).

The pages do not fix a byte layout (App. A "Storage layout", p.15, fixes only
what is stored: four E2M1 values and a pattern index per eight-weight group,
one UE4M3 scale per 32-weight block).  The library stores everything in the
order its grouped GEMM consumes it, and this module restates those index
functions independently of the CUDA code, so packed bytes can be compared
bit for bit.  Constants: weight tiles of 128 output rows ("n-tiles"); an MMA
k-block is 64 stored 4-bit values per row (128 logical K for the paired 4:8
weight, 64 for the dense control); a chunk is 256 logical K.

The packed weight buffer is a sequence of chunk blocks, one per (expert,
n-tile, chunk), each holding the chunk's values, then (sparse) its metadata,
then its scale atoms:
  values  k-block h, row r (0..127), stored value v (0..63): byte c = v // 2
          (low nibble = even v) at h*4096 + (r//8)*256 + (c//16)*128 + (r%8)*16 + c%16
  meta    8192 + r*16 + g//2 for 8-group g (0..31) of the chunk, low nibble = even g
  scales  V + h*512 + 16*(r%32) + 4*(r//32) + j for block j (0..3) of k-block h
Sparse blocks are 11264 bytes (2 k-blocks, V = 10240), dense 18432 (4 k-blocks,
V = 16384).
Activation codes  [R][K/2] row-major, low nibble = even k.
Activation scales [KB][R + 256][4][4] ("quad" entries): entry (kb, r, c, j)
                holds the scale of block 4*kb + j of routed row r + 32*c, or 0
                when r + 32*c >= R.
"""
from __future__ import annotations

import numpy as np

TILE_N = 128
KB_VALUES = 64          # stored 4-bit values per row per MMA k-block
META_CHUNK_K = 256      # logical K per metadata chunk
ACT_SCALE_PAD_ROWS = 256


def tile_values(codes: np.ndarray) -> np.ndarray:
    """codes uint8 [N, V] (one code per byte) -> packed bytes [N//128, V//64, 4096]."""
    codes = np.asarray(codes, dtype=np.uint8)
    N, V = codes.shape
    NT, KB = N // TILE_N, V // KB_VALUES
    out = np.zeros((NT, KB, 4096), dtype=np.uint8)
    for n in range(N):
        nt, r = divmod(n, TILE_N)
        for v in range(V):
            kb, vl = divmod(v, KB_VALUES)
            c, nib = divmod(vl, 2)
            pos = (r // 8) * 256 + (c // 16) * 128 + (r % 8) * 16 + (c % 16)
            out[nt, kb, pos] |= (int(codes[n, v]) & 0xF) << (4 * nib)
    return out


def tile_values_fast(codes: np.ndarray) -> np.ndarray:
    """Vectorised tile_values (same index function; checked equal to it in the tests)."""
    codes = np.asarray(codes, dtype=np.uint8)
    N, V = codes.shape
    NT, KB = N // TILE_N, V // KB_VALUES
    n = np.arange(N)[:, None]
    v = np.arange(V)[None, :]
    nt, r = n // TILE_N, n % TILE_N
    kb, vl = v // KB_VALUES, v % KB_VALUES
    c, nib = vl // 2, vl % 2
    pos = (nt * KB + kb) * 4096 + (r // 8) * 256 + (c // 16) * 128 + (r % 8) * 16 + (c % 16)
    out = np.zeros(NT * KB * 4096, dtype=np.uint16)
    np.add.at(out, pos.ravel(), ((codes & 0xF).astype(np.uint16) << (4 * nib).astype(np.uint16)).ravel())
    return out.astype(np.uint8).reshape(NT, KB, 4096)


def untile_values(packed: np.ndarray, N: int, V: int) -> np.ndarray:
    """Inverse of tile_values."""
    flat = np.asarray(packed, dtype=np.uint8).reshape(-1)
    KB = V // KB_VALUES
    n = np.arange(N)[:, None]
    v = np.arange(V)[None, :]
    nt, r = n // TILE_N, n % TILE_N
    kb, vl = v // KB_VALUES, v % KB_VALUES
    c, nib = vl // 2, vl % 2
    pos = (nt * KB + kb) * 4096 + (r // 8) * 256 + (c // 16) * 128 + (r % 8) * 16 + (c % 16)
    return ((flat[pos] >> (4 * nib)) & 0xF).astype(np.uint8)


def tile_meta(patterns: np.ndarray) -> np.ndarray:
    """patterns uint8 [N, K/8] -> packed bytes [N//128, K//256, 2048]."""
    pat = np.asarray(patterns, dtype=np.uint8)
    N, G = pat.shape
    NT, KC = N // TILE_N, G // 32
    n = np.arange(N)[:, None]
    g = np.arange(G)[None, :]
    nt, r = n // TILE_N, n % TILE_N
    kc, gl = g // 32, g % 32
    pos = (nt * KC + kc) * 2048 + r * 16 + gl // 2
    out = np.zeros(NT * KC * 2048, dtype=np.uint16)
    np.add.at(out, pos.ravel(), ((pat & 0xF).astype(np.uint16) << (4 * (gl % 2)).astype(np.uint16)).ravel())
    return out.astype(np.uint8).reshape(NT, KC, 2048)


def untile_meta(packed: np.ndarray, N: int, G: int) -> np.ndarray:
    flat = np.asarray(packed, dtype=np.uint8).reshape(-1)
    KC = G // 32
    n = np.arange(N)[:, None]
    g = np.arange(G)[None, :]
    nt, r = n // TILE_N, n % TILE_N
    kc, gl = g // 32, g % 32
    pos = (nt * KC + kc) * 2048 + r * 16 + gl // 2
    return ((flat[pos] >> (4 * (gl % 2))) & 0xF).astype(np.uint8)


def tile_scales(scales: np.ndarray) -> np.ndarray:
    """scales uint8 [N, S] (S blocks per row, 4 per k-block) -> packed [N//128, S//4, 512]."""
    sc = np.asarray(scales, dtype=np.uint8)
    N, S = sc.shape
    NT, KB = N // TILE_N, S // 4
    n = np.arange(N)[:, None]
    s = np.arange(S)[None, :]
    nt, r = n // TILE_N, n % TILE_N
    kb, j = s // 4, s % 4
    pos = (nt * KB + kb) * 512 + 16 * (r % 32) + 4 * (r // 32) + j
    out = np.zeros(NT * KB * 512, dtype=np.uint8)
    out[pos.ravel()] = sc.ravel()
    return out.reshape(NT, KB, 512)


def untile_scales(packed: np.ndarray, N: int, S: int) -> np.ndarray:
    flat = np.asarray(packed, dtype=np.uint8).reshape(-1)
    KB = S // 4
    n = np.arange(N)[:, None]
    s = np.arange(S)[None, :]
    nt, r = n // TILE_N, n % TILE_N
    kb, j = s // 4, s % 4
    pos = (nt * KB + kb) * 512 + 16 * (r % 32) + 4 * (r // 32) + j
    return flat[pos]


SPARSE_CHUNK_BYTES = 11264
DENSE_CHUNK_BYTES = 18432


def packed_sparse(codes: np.ndarray, patterns: np.ndarray, scales: np.ndarray) -> np.ndarray:
    """One expert's canonical parts -> its packed chunk blocks [NT, K/256, 11264].

    codes [N, K/2] (retained values), patterns [N, K/8], scales [N, K/32].
    """
    N, Kh = codes.shape
    K = 2 * Kh
    NT, KC = N // TILE_N, K // 256
    out = np.zeros((NT, KC, SPARSE_CHUNK_BYTES), dtype=np.uint8)
    out[:, :, :8192] = tile_values_fast(codes).reshape(NT, KC, 8192)
    out[:, :, 8192:10240] = tile_meta(patterns).reshape(NT, KC, 2048)
    out[:, :, 10240:] = tile_scales(scales).reshape(NT, KC, 1024)
    return out


def packed_dense(codes: np.ndarray, scales: np.ndarray) -> np.ndarray:
    """One expert's dense control parts -> chunk blocks [NT, K/256, 18432] (codes [N, K], scales [N, K/16])."""
    N, K = codes.shape
    NT, KC = N // TILE_N, K // 256
    out = np.zeros((NT, KC, DENSE_CHUNK_BYTES), dtype=np.uint8)
    out[:, :, :16384] = tile_values_fast(codes).reshape(NT, KC, 16384)
    out[:, :, 16384:] = tile_scales(scales).reshape(NT, KC, 2048)
    return out


def pack_act_codes(codes: np.ndarray) -> np.ndarray:
    """codes uint8 [R, K] -> bytes [R, K/2], low nibble = even k."""
    c = np.asarray(codes, dtype=np.uint8)
    return ((c[:, 0::2] & 0xF) | ((c[:, 1::2] & 0xF) << 4)).astype(np.uint8)


def unpack_act_codes(packed: np.ndarray) -> np.ndarray:
    p = np.asarray(packed, dtype=np.uint8)
    out = np.empty((p.shape[0], p.shape[1] * 2), dtype=np.uint8)
    out[:, 0::2] = p & 0xF
    out[:, 1::2] = p >> 4
    return out


def act_scale_rows(R: int) -> int:
    """Row capacity of the activation scale buffer."""
    return R + ACT_SCALE_PAD_ROWS


def quad_act_scales(scales: np.ndarray) -> np.ndarray:
    """scales uint8 [R, S] -> quad entries [S//4, R+256, 4, 4]."""
    sc = np.asarray(scales, dtype=np.uint8)
    R, S = sc.shape
    KB = S // 4
    out = np.zeros((KB, act_scale_rows(R), 4, 4), dtype=np.uint8)
    for c in range(4):
        rows = np.arange(act_scale_rows(R))
        src = rows + 32 * c
        ok = src < R
        for kb in range(KB):
            out[kb, rows[ok], c, :] = sc[src[ok], 4 * kb:4 * kb + 4]
    return out
