"""Pins for the oracle's routing, activation quantizer, GEMM reference, scatter and layouts (CPU)."""
import json
import os

import numpy as np
import torch

from grouped_sparse_gemm_b200 import inputs
from oracle import codecs, gemm, layout, pack, quant, route, unpermute

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


# ---------------------------------------------------------------- routing
def test_route_invariants_and_library_sort():
    cfg = inputs.CONFIGS["30b_up_prefill"]
    ids = inputs.routing(cfg).numpy()
    off, perm_src, inv_perm = route.route(ids, cfg.E)
    R = ids.size
    assert off[0] == 0 and off[-1] == R and np.all(np.diff(off) >= 0)
    np.testing.assert_array_equal(np.diff(off), np.bincount(ids.reshape(-1), minlength=cfg.E))
    np.testing.assert_array_equal(perm_src[inv_perm], np.arange(R))
    np.testing.assert_array_equal(inv_perm[perm_src], np.arange(R))
    # independent pin: a library stable sort by expert id gives the same row order
    np.testing.assert_array_equal(perm_src, np.argsort(ids.reshape(-1), kind="stable"))


def test_route_edge_cases():
    off, ps, ip = route.route(np.zeros((0, 2), dtype=np.int32), 3)
    assert off.tolist() == [0, 0, 0, 0] and ps.size == 0
    off, ps, ip = route.route(np.array([[2, 2], [0, 2]]), 4)      # duplicate id in one token
    assert off.tolist() == [0, 1, 1, 4, 4]
    assert ps.tolist() == [2, 0, 1, 3]


def test_routing_generator_draws_distinct_experts():
    cfg = inputs.CONFIGS["1t_up_prefill"]
    ids = inputs.routing(cfg)
    assert ids.shape == (cfg.T, cfg.top_k)
    s = torch.sort(ids, dim=1).values
    assert torch.all(s[:, 1:] != s[:, :-1])
    g = inputs.gates(cfg)
    torch.testing.assert_close(g.sum(dim=1), torch.ones(cfg.T), rtol=0, atol=1e-6)


# ---------------------------------------------------------------- activation quantizer
def test_act_scale_and_blocks():
    x = np.zeros((2, 64), dtype=np.float32)
    x[0, 5] = -3.0
    x[1, 40] = 0.75
    s = quant.act_tensor_scale(x)
    assert s == np.float32(np.float32(3.0) / np.float32(2688.0))
    q, sc = quant.quantize_rows(x, 32, s)
    assert sc[0, 0] == 0x7E and sc[0, 1] == 0 and sc[1, 0] == 0
    assert q[0, 5] == 0xF                     # -3 is the block max -> -6 on the grid
    # block with amax 0.75: ratio = 0.75 / (6 s) ~= 112, a UE4M3 value -> 0.75 maps to 6
    assert codecs.ue4m3_decode(sc[1, 1]) == 112.0
    assert q[1, 40] == 0x7
    dec = quant.decode_rows(q, sc, 32) * float(s)
    assert abs(dec[1, 40] - 0.75) <= 0.75 * 2 ** -20


def test_quantize_routed_equals_permute_then_quantize():
    cfg = inputs.CONFIGS["tiny"]
    x = inputs.activations(cfg).float().numpy()
    ids = inputs.routing(cfg).numpy()
    off, perm_src, inv_perm = route.route(ids, cfg.E)
    q, sc, s = quant.quantize_routed(x, 32, perm_src, cfg.top_k)
    xp = x[perm_src // cfg.top_k]
    q2, sc2 = quant.quantize_rows(xp, 32, quant.act_tensor_scale(xp))
    np.testing.assert_array_equal(q, q2)
    np.testing.assert_array_equal(sc, sc2)


# ---------------------------------------------------------------- GEMM reference
def _bruteforce_gemm(a, w):
    m, K = a.shape
    N = w.shape[0]
    y = np.zeros((m, N))
    for i in range(m):
        for n in range(N):
            s = 0.0
            for k in range(K):
                s += a[i, k] * w[n, k]
            y[i, n] = s
    return y


def test_gemm_matches_bruteforce_and_closed_forms():
    rng = np.random.default_rng(5)
    w = (rng.normal(size=(8, 64)) * 0.02).astype(np.float32)
    codes, pats, scales, s_w = pack.pack_sparse_expert(w)
    wd = pack.decode_sparse_expert(codes, pats, scales)
    x = rng.normal(size=(5, 64)).astype(np.float32)
    s_x = quant.act_tensor_scale(x)
    qa, sa = quant.quantize_rows(x, 32, s_x)
    ad = quant.decode_rows(qa, sa, 32)
    y, b = gemm.gemm_rows(ad, wd, float(s_x) * float(s_w))
    yb = _bruteforce_gemm(ad, wd) * float(s_x) * float(s_w)
    np.testing.assert_allclose(y, yb, rtol=1e-13, atol=1e-15)
    assert np.all(b >= np.abs(y) - 1e-15)
    # one-hot activation row returns one column of the decoded weight
    onehot = np.zeros((1, 64))
    onehot[0, 17] = 1.0
    y1, _ = gemm.gemm_rows(onehot, wd, 1.0)
    np.testing.assert_array_equal(y1[0], wd[:, 17])
    # all-equal values: K * v * w
    ones = np.ones((1, 64)) * 0.5
    wconst = np.ones((3, 64)) * 2.0
    y2, b2 = gemm.gemm_rows(ones, wconst, 1.0)
    assert np.all(y2 == 64.0) and np.all(b2 == 64.0)


def test_tolerance_rejects_planted_mistakes():
    """A dropped term, a sign flip or a transposed operand must fail the tolerance."""
    cfg = inputs.CONFIGS["tiny"]
    w = inputs.expert_weight(cfg, 0).numpy()
    codes, pats, scales, s_w = pack.pack_sparse_expert(w)
    wd = pack.decode_sparse_expert(codes, pats, scales)
    x = inputs.activations(cfg).float().numpy()[:16]
    s_x = quant.act_tensor_scale(x)
    qa, sa = quant.quantize_rows(x, 32, s_x)
    ad = quant.decode_rows(qa, sa, 32)
    sc = float(s_x) * float(s_w)
    y, b = gemm.gemm_rows(ad, wd, sc)
    assert gemm.within_tolerance(y, y, b).all()
    wd_drop = wd.copy()
    wd_drop[:, 100] = 0
    y_drop, _ = gemm.gemm_rows(ad, wd_drop, sc)
    assert not gemm.within_tolerance(y_drop, y, b).all()
    assert not gemm.within_tolerance(-y, y, b).all()
    wd_swap = wd.copy()
    wd_swap[:, [0, 1]] = wd_swap[:, [1, 0]]                   # swapped pair elements
    y_swap, _ = gemm.gemm_rows(ad, wd_swap, sc)
    assert not gemm.within_tolerance(y_swap, y, b).all()


# ---------------------------------------------------------------- scatter
def test_unpermute_gather_and_torch_pin():
    rng = np.random.default_rng(6)
    T, k, N = 7, 3, 16
    y_bits = inputs.random_bf16((T * k, N), seed=11).view(torch.uint16).numpy()
    inv = rng.permutation(T * k).astype(np.int32)
    # k = 1, g = 1 is a pure gather
    out = unpermute.unpermute_scale(y_bits[:T], np.arange(T), np.ones((T, 1), np.float32), 1)
    np.testing.assert_array_equal(out, y_bits[:T])
    # torch float32 elementwise ops + bf16 cast as an independent implementation
    g = rng.random((T, k)).astype(np.float32)
    out = unpermute.unpermute_scale(y_bits, inv, g, k)
    yt = torch.from_numpy(y_bits.astype(np.int16)).view(torch.bfloat16).float()
    gt = torch.from_numpy(g)
    acc = torch.zeros(T, N)
    for j in range(k):
        acc = acc + gt[:, j:j + 1] * yt[torch.from_numpy(inv.reshape(T, k)[:, j]).long()]
    ref = acc.to(torch.bfloat16).view(torch.int16).numpy().astype(np.uint16)
    np.testing.assert_array_equal(out, ref)


# ---------------------------------------------------------------- layouts
def test_layout_round_trips_and_handworked_positions():
    rng = np.random.default_rng(7)
    codes = rng.integers(0, 16, size=(256, 128)).astype(np.uint8)
    tv = layout.tile_values(codes)
    np.testing.assert_array_equal(tv, layout.tile_values_fast(codes))
    np.testing.assert_array_equal(layout.untile_values(tv, 256, 128), codes)
    pats = rng.integers(0, 16, size=(128, 64)).astype(np.uint8)
    np.testing.assert_array_equal(layout.untile_meta(layout.tile_meta(pats), 128, 64), pats)
    sc = rng.integers(0, 127, size=(256, 16)).astype(np.uint8)
    np.testing.assert_array_equal(layout.untile_scales(layout.tile_scales(sc), 256, 16), sc)
    # hand-worked positions
    one = np.zeros((128, 64), np.uint8)
    one[9, 35] = 0xA            # row 9, value 35 -> byte c=17, high nibble
    flat = layout.tile_values_fast(one).reshape(-1)
    assert flat[(9 // 8) * 256 + (17 // 16) * 128 + (9 % 8) * 16 + 17 % 16] == 0xA0
    s1 = np.zeros((128, 8), np.uint8)
    s1[33, 6] = 77              # row 33, k-block 1, block 2 -> 512 + 16*1 + 4*1 + 2
    assert layout.tile_scales(s1).reshape(-1)[512 + 22] == 77
    # metadata: n-tile 1, row 2, 8-group 37 = chunk 1, group 5 -> (1*2 + 1)*2048 + 2*16 + 5//2 = 6178,
    # high nibble (odd group)
    m1 = np.zeros((256, 64), np.uint8)
    m1[130, 37] = 0x9
    tm = layout.tile_meta(m1).reshape(-1)
    assert tm[6178] == 0x90 and int(tm.astype(np.int64).sum()) == 0x90
    # a whole sparse chunk block (N=128, K=512: two chunk blocks of 11264 bytes), worked by hand:
    # value 200 of row 5 = chunk 1, k-block 1, stored value 8 -> byte 4096 + 5*16 + 4 = 4180 (low nibble);
    # 8-group 40 of row 5 = chunk 1, group 8 -> 8192 + 5*16 + 4 = 8276 (low nibble);
    # 32-block 9 of row 100 = chunk 1, k-block 0, block 1 -> 10240 + 16*(100%32) + 4*(100//32) + 1 = 10317
    cv = np.zeros((128, 256), np.uint8)
    cv[5, 200] = 0x3
    pt = np.zeros((128, 64), np.uint8)
    pt[5, 40] = 0x6
    scs = np.zeros((128, 16), np.uint8)
    scs[100, 9] = 0x55
    blk = layout.packed_sparse(cv, pt, scs)
    assert blk.shape == (1, 2, 11264)
    assert blk[0, 1, 4180] == 0x03 and blk[0, 1, 8276] == 0x06 and blk[0, 1, 10317] == 0x55
    assert int(blk.astype(np.int64).sum()) == 0x03 + 0x06 + 0x55
    # quad activation scales: entry (kb, r, c, j) = scale of row r + 32c
    R = 70
    asc = rng.integers(1, 127, size=(R, 8)).astype(np.uint8)
    qd = layout.quad_act_scales(asc)
    assert qd.shape == (2, R + 256, 4, 4)
    assert qd[1, 5, 2, 3] == asc[69, 7] and qd[1, 6, 2, 3] == 0 and qd[0, 69, 0, 0] == asc[69, 0]


def test_golden_act_block():
    with open(os.path.join(GOLDEN, "act_block32.json")) as f:
        g = json.load(f)
    x = np.array([g["x"]], dtype=np.float32)
    q, sc = quant.quantize_rows(x, 32, np.float32(g["s_x"]))
    assert sc[0].tolist() == g["scales"]
    assert q[0].tolist() == g["codes"]


def test_swiglu_oracle_pins():
    """silu against its closed forms and an independent float64 implementation (torch), the slope
    bound against a dense grid, and the h error bound against brute-force perturbations."""
    import torch
    from oracle import swiglu as osw
    assert osw.silu(np.array([0.0]))[0] == 0.0
    x = np.linspace(-30, 30, 20001)
    s = osw.silu(x)
    np.testing.assert_allclose(osw.silu(-x), s - x, rtol=0, atol=1e-12)          # silu(-x) = silu(x) - x
    np.testing.assert_allclose(s, torch.nn.functional.silu(torch.from_numpy(x)).numpy(), rtol=1e-15, atol=1e-300)
    assert np.abs(osw.silu(np.array([40.0, -40.0])) - np.array([40.0, 0.0])).max() < 1e-15
    slope = np.abs(np.diff(s) / np.diff(x)).max()
    assert 1.09 < slope <= osw.SILU_SLOPE_MAX
    rng = np.random.default_rng(11)
    y = rng.normal(size=(6, 8)) * 3
    h = osw.swiglu_rows(y)
    np.testing.assert_allclose(h, osw.silu(y[:, :4]) * y[:, 4:], rtol=0, atol=0)
    tau = np.abs(rng.normal(size=y.shape)) * 0.05
    bound = osw.swiglu_error_bound(y, tau)
    for _ in range(200):                                   # no perturbation within tau escapes the bound
        yp = y + tau * rng.uniform(-1, 1, size=y.shape)
        assert np.all(np.abs(osw.swiglu_rows(yp) - h) <= bound + 1e-12)
