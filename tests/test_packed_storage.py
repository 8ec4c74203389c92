"""save_packed / load_packed: packed weights kept in a file byte for byte (CPU only).

The packed bytes come from the oracle's packer and layout (the format the GEMM reads), so the
round trip is checked on real packed data, and the loader's checks on corrupted files.
"""
import numpy as np
import pytest
import torch

import grouped_sparse_gemm_b200 as gsg
from oracle import layout as olayout
from oracle import pack as opack


def _packed_sparse(E=2, N=128, K=256, seed=5):
    rng = np.random.default_rng(seed)
    blocks, scales = [], []
    for _ in range(E):
        W = rng.normal(0.0, 0.02, size=(N, K)).astype(np.float32)
        codes, pats, sc, s_w = opack.pack_sparse_expert(W)
        blocks.append(olayout.packed_sparse(codes, pats, sc).reshape(-1))
        scales.append(s_w)
    return gsg.PackedSparseWeights(packed=torch.from_numpy(np.concatenate(blocks)),
                                   w_scale=torch.tensor(scales, dtype=torch.float32), E=E, N=N, K=K)


def test_round_trip_is_byte_exact(tmp_path):
    w = _packed_sparse()
    assert w.packed.numel() == gsg.lib().gsg_sparse_packed_bytes(w.E, w.N, w.K)
    p = tmp_path / "w.npz"
    gsg.save_packed(w, str(p))
    r = gsg.load_packed(str(p))
    assert isinstance(r, gsg.PackedSparseWeights) and (r.E, r.N, r.K) == (w.E, w.N, w.K)
    assert torch.equal(r.packed, w.packed) and torch.equal(r.w_scale, w.w_scale)


def test_dense_format_round_trip(tmp_path):
    E, N, K = 1, 128, 256
    w = gsg.PackedDenseWeights(packed=torch.arange(gsg.lib().gsg_dense_packed_bytes(E, N, K)).to(torch.uint8),
                               w_scale=torch.tensor([0.5], dtype=torch.float32), E=E, N=N, K=K)
    p = tmp_path / "d.npz"
    gsg.save_packed(w, str(p))
    r = gsg.load_packed(str(p))
    assert isinstance(r, gsg.PackedDenseWeights) and torch.equal(r.packed, w.packed)


def test_loader_rejects_wrong_sizes_and_versions(tmp_path):
    w = _packed_sparse(E=1)
    good = dict(version=gsg.PACKED_FILE_VERSION, format="sparse", E=1, N=128, K=256,
                packed=w.packed.numpy(), w_scale=w.w_scale.numpy())
    cases = [dict(packed=w.packed.numpy()[:-1]),              # truncated
             dict(K=512),                                     # shape that does not match the bytes
             dict(w_scale=np.zeros(2, dtype=np.float32)),     # one scale per expert
             dict(version=99),
             dict(format="fp8"),
             dict(N=130),                                     # N not whole n-tiles, same byte count
             dict(K=300),                                     # K not whole chunks, same byte count
             dict(E=0, w_scale=np.zeros(0, dtype=np.float32)),
             dict(E=-1),
             dict(N=2 ** 40)]                                 # beyond int range
    for i, bad in enumerate(cases):
        p = tmp_path / f"bad{i}.npz"
        np.savez(p, **{**good, **bad})
        with pytest.raises(ValueError):
            gsg.load_packed(str(p))
