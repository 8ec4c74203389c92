"""Pins for the oracle's packer (paired 4:8 support, scales, codes) -- CPU only."""
import itertools
import json
import os

import numpy as np
import pytest

from oracle import codecs, pack, layout

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
ADMISSIBLE = {0x4, 0x8, 0xC, 0x9, 0xD, 0xE}   # the six ways to keep 2 of 4 pairs, i0 < i1


def test_six_admissible_patterns():
    pats = {pack.pattern_code(np.array([a, b])) for a, b in itertools.combinations(range(4), 2)}
    assert {int(p) for p in pats} == ADMISSIBLE


def _bruteforce_keep(w8):
    """Over all six patterns: maximise the kept energy (exact sum of the fp32 pair energies),
    ties -> lexicographically smallest (i0, i1)."""
    m = [np.float32(np.float32(w8[2 * p] * w8[2 * p]) + np.float32(w8[2 * p + 1] * w8[2 * p + 1]))
         for p in range(4)]
    best, best_e = None, None
    for a, b in itertools.combinations(range(4), 2):
        e = float(m[a]) + float(m[b])
        if best_e is None or e > best_e:
            best, best_e = (a, b), e
    return best


def test_support_selection_matches_bruteforce():
    rng = np.random.default_rng(0)
    # coarse values force many exact ties
    w = (rng.integers(-3, 4, size=(64, 8 * 64)) * 0.5).astype(np.float32)
    w2 = rng.normal(size=(64, 8 * 64)).astype(np.float32)
    for mat in (w, w2):
        keep = pack.select_pairs(mat)
        for n in range(mat.shape[0]):
            for g in range(mat.shape[1] // 8):
                assert tuple(keep[n, g]) == _bruteforce_keep(mat[n, 8 * g:8 * g + 8])


def _representable(rng, N, K, s_w):
    """Weights already on the paired 4:8 NVFP4 grid with tensor scale s_w (a power of two).

    Every 32-block keeps a +-6 in one of its kept pairs, so its amax is 6 * dec(sc) * s_w,
    and one block per expert has sc = 448 so that amax(W) = 2688 * s_w.
    """
    G = K // 8
    keep = np.array([list(itertools.combinations(range(4), 2))[i]
                     for i in rng.integers(0, 6, size=N * G)]).reshape(N, G, 2)
    sc = rng.integers(24, 126, size=(N, K // 32)).astype(np.uint8)   # normal scales
    sc[0, 0] = 0x7E
    q = rng.integers(0, 16, size=(N, K // 2)).astype(np.uint8)
    q[:, 0::16] = np.where(rng.random((N, K // 32)) < 0.5, 0x7, 0xF)   # a +-6 in every block
    # a kept value whose pair energy is strictly largest must not be zeroed; make kept pairs
    # dominant by keeping dropped pairs at exactly zero.
    vals = codecs.e2m1_decode(q).reshape(N, K // 32, 16) * codecs.ue4m3_decode(sc)[..., None] * s_w
    vals = vals.reshape(N, G, 2, 2)
    full = np.zeros((N, G, 4, 2))
    np.put_along_axis(full, keep[..., None].repeat(2, axis=-1), vals, axis=-2)
    return full.reshape(N, K).astype(np.float32), keep, q, sc


def test_pack_round_trip_on_representable_weights():
    rng = np.random.default_rng(1)
    N, K, s_w = 16, 256, np.float32(2.0 ** -7)
    w, keep, q, sc = _representable(rng, N, K, s_w)
    codes, pats, scales, s = pack.pack_sparse_expert(w)
    assert s == s_w
    np.testing.assert_array_equal(scales, sc)
    # where both kept pairs carry energy, the support is recovered exactly
    e = pack.pair_energies(w)
    nz_kept = np.take_along_axis(e, keep, axis=-1) > 0
    both = nz_kept.all(axis=-1)
    np.testing.assert_array_equal(pats[both], pack.pattern_code(keep)[both])
    # decoding reproduces W exactly (fp64 of fp32 values)
    dec = pack.decode_sparse_expert(codes, pats, scales) * float(s)
    np.testing.assert_array_equal(dec, w.astype(np.float64))


def test_pack_invariants_random():
    rng = np.random.default_rng(2)
    N, K = 128, 512
    w = (rng.normal(size=(N, K)) * 0.02).astype(np.float32)
    codes, pats, scales, s_w = pack.pack_sparse_expert(w)
    assert set(np.unique(pats).tolist()) <= ADMISSIBLE
    # 2.75 bit per logical weight: values 2 + metadata 0.5 + scale 0.25
    tv, tm, ts = layout.tile_values_fast(codes), layout.tile_meta(pats), layout.tile_scales(scales)
    assert tv.nbytes + tm.nbytes + ts.nbytes == N * K * 2.75 / 8
    dec = pack.decode_sparse_expert(codes, pats, scales)
    pairs = dec.reshape(N, K // 8, 4, 2)
    nz_pairs = np.any(pairs != 0, axis=-1)
    assert np.all(nz_pairs.sum(axis=-1) <= 2)
    kept = np.zeros_like(nz_pairs)
    np.put_along_axis(kept, pack.pattern_pairs(pats), True, axis=-1)
    assert not np.any(nz_pairs & ~kept)                 # pruned positions decode to exactly 0
    # the magnitude rule keeps exactly two distinct pairs for continuous data
    keep = pack.pattern_pairs(pats)
    assert np.all(keep[..., 0] < keep[..., 1])
    # quantization error is bounded by half an E2M1 step at the block scale
    wp = pack.prune(w, keep)
    err = np.abs(dec * float(s_w) - wp)
    step = codecs.ue4m3_decode(scales).repeat(32, axis=1) * float(s_w)
    assert np.all(err <= step * 1.0 + 1e-12)


def test_pack_zero_expert_and_zero_block():
    w = np.zeros((128, 256), dtype=np.float32)
    codes, pats, scales, s_w = pack.pack_sparse_expert(w)
    assert s_w == 1.0 and not scales.any() and not codes.any()
    assert np.all(pats == 0x4)
    w[3, 40] = 1.5
    codes, pats, scales, s_w = pack.pack_sparse_expert(w)
    assert s_w == np.float32(1.5) / np.float32(2688)
    assert scales[3, 1] == 0x7E and scales[0, 0] == 0


def test_golden_row32():
    """Hand-worked example (tests/golden/pack_row32.json)."""
    with open(os.path.join(GOLDEN, "pack_row32.json")) as f:
        g = json.load(f)
    w = np.array([g["w"]], dtype=np.float32)
    codes, pats, scales, s_w = pack.pack_sparse_expert(w)
    assert pats[0].tolist() == g["patterns"]
    assert codes[0].tolist() == g["codes"]
    assert scales[0].tolist() == g["scales"]
    assert s_w == np.float32(np.float32(g["amax"]) / np.float32(2688.0))


def test_dense_pack_matches_sparse_on_already_48_weights():
    """A W that is already paired 4:8 packs to the same values either way (32-blocks)."""
    rng = np.random.default_rng(4)
    N, K = 128, 256
    w, _, _, _ = _representable(rng, N, K, np.float32(2.0 ** -6))
    codes, pats, scales, s = pack.pack_sparse_expert(w)
    dcodes, dscales, ds = pack.pack_dense_expert(w, sf_block=32)
    assert s == ds
    np.testing.assert_array_equal(dscales, scales)
    np.testing.assert_array_equal(pack.decode_dense_expert(dcodes, dscales, 32),
                                  pack.decode_sparse_expert(codes, pats, scales))
