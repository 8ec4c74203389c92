"""GPU parity: every kernel of the path against the oracle, through the C ABI.

Packed weights, activation codes/scales, routing and the scatter must match bit for bit;
GEMM outputs must satisfy |y - y_ref| <= 2^-10 * sum|a*w| + 1e-6 (fp32 output; a bf16 output
adds its own half-ulp of rounding).
"""
import numpy as np
import pytest
import torch

from grouped_sparse_gemm_b200 import inputs
from oracle import layout as olayout
from oracle import pack as opack
from oracle import unpermute as ounperm
from tests import gsg_testlib as tl

pytestmark = pytest.mark.gpu
DEV = "cuda:0"


@pytest.fixture(scope="module")
def gsg():
    import grouped_sparse_gemm_b200 as g
    g.load_library()
    assert g.lib().gsg_version() == 1
    return g


def _status_ok(gsg):
    assert gsg.get_device_status() == 0


# ---------------------------------------------------------------- packing
@pytest.mark.parametrize("E,N,K", [(1, 128, 256), (3, 256, 768), (2, 384, 2048)])
def test_pack_sparse_bit_exact(gsg, E, N, K):
    cfg = inputs.custom_config("p", E=E, K=K, N=N, T=1, top_k=1)
    W = inputs.all_weights(cfg)
    W[0, :3] = 0.0                     # a zero row: all-zero blocks
    W[0, 5, :8] = 0.25                 # a group of equal pair energies (ties)
    if E > 1:
        W[1].mul_(1e-3)                # a small-magnitude expert
    pw = gsg.pack_sparse_nvfp4(W.to(DEV))
    packed, sws, _ = tl.oracle_pack_sparse(W.numpy())
    np.testing.assert_array_equal(pw.packed.cpu().numpy(), packed)
    np.testing.assert_array_equal(pw.w_scale.cpu().numpy(), sws)
    _status_ok(gsg)


@pytest.mark.parametrize("E,N,K", [(1, 128, 256), (2, 256, 768)])
def test_pack_dense_bit_exact(gsg, E, N, K):
    cfg = inputs.custom_config("p", E=E, K=K, N=N, T=1, top_k=1)
    W = inputs.all_weights(cfg)
    W[0, 1] = 0.0
    pw = gsg.pack_dense_nvfp4(W.to(DEV))
    packed, sws, _ = tl.oracle_pack_dense(W.numpy(), 16)
    np.testing.assert_array_equal(pw.packed.cpu().numpy(), packed)
    np.testing.assert_array_equal(pw.w_scale.cpu().numpy(), sws)


def test_pack_flags_nonfinite(gsg):
    W = torch.zeros(1, 128, 256)
    W[0, 7, 9] = float("nan")
    gsg.pack_sparse_nvfp4(W.to(DEV))
    assert gsg.get_device_status() == -5
    _status_ok(gsg)


# ---------------------------------------------------------------- routing
@pytest.mark.parametrize("T,k,E,mode", [(32, 2, 4, "uniform"), (512, 8, 128, "zipf"), (64, 8, 128, "uniform"),
                                        (1025, 4, 7, "zipf"), (8192, 8, 384, "zipf"), (3, 1, 1, "uniform"),
                                        (256, 8, 384, "uniform"), (9000, 8, 512, "zipf"),
                                        (1500, 1, 1024, "uniform"), (256, 8, 128, "zipf"),
                                        (2049, 1, 16, "zipf"), (2000, 8, 64, "zipf")])
def test_route_matches_oracle(gsg, T, k, E, mode):
    cfg = inputs.custom_config("r", E=E, K=256, N=128, T=T, top_k=k, routing=mode, zipf_s=1.1)
    ids = inputs.routing(cfg) if k <= E else torch.zeros(T, k, dtype=torch.int32)
    r = gsg.moe_route_permute(ids.to(DEV), E)
    off, ps, ip = tl.route_np(ids, E)
    np.testing.assert_array_equal(r.offsets.cpu().numpy(), off)
    np.testing.assert_array_equal(r.perm_src.cpu().numpy()[:T * k], ps)
    np.testing.assert_array_equal(r.inv_perm.cpu().numpy()[:T * k], ip)
    _status_ok(gsg)


def test_route_duplicates_and_empty(gsg):
    ids = torch.tensor([[2, 2], [0, 2], [2, 0]], dtype=torch.int32)
    r = gsg.moe_route_permute(ids.to(DEV), 4)
    off, ps, ip = tl.route_np(ids, 4)
    np.testing.assert_array_equal(r.offsets.cpu().numpy(), off)
    np.testing.assert_array_equal(r.perm_src.cpu().numpy(), ps)
    r0 = gsg.moe_route_permute(torch.zeros(0, 8, dtype=torch.int32, device=DEV), 5)
    assert r0.offsets.cpu().tolist() == [0] * 6


@pytest.mark.parametrize("T,k,E", [(1, 2, 4), (3000, 8, 64)])   # one routing block; 1024-row chunks
def test_route_flags_bad_ids(gsg, T, k, E):
    """An out-of-range id sets GSG_ERR_BAD_ROUTING, and its pair gets no row: inv_perm = -1, so the
    quantizer and the scatter skip it instead of reading a stale row."""
    ids = torch.randint(0, E, (T, k), generator=torch.Generator().manual_seed(3), dtype=torch.int32)
    ids[0, 1] = E + 5
    ids[T - 1, 0] = -2
    r = gsg.moe_route_permute(ids.to(DEV), E)
    r.inv_perm.fill_(12345)
    r = gsg.moe_route_permute(ids.to(DEV), E, out=r)
    assert gsg.get_device_status() == -4
    _status_ok(gsg)
    ip = r.inv_perm.cpu()
    assert ip[1].item() == -1 and ip[(T - 1) * k].item() == -1
    good = torch.ones(T * k, dtype=torch.bool)
    good[1] = good[(T - 1) * k] = False
    assert (ip[good] >= 0).all() and (ip[good] < T * k).all()


# ---------------------------------------------------------------- activation quantizer
@pytest.mark.parametrize("name,sf", [("tiny", 32), ("30b_down_decode", 32), ("30b_up_prefill", 32), ("tiny", 16),
                                     ("1t_down_decode_b1", 32)])
def test_quantize_matches_oracle(gsg, name, sf):
    cfg = inputs.CONFIGS[name]
    X = inputs.activations(cfg)
    ids = inputs.routing(cfg)
    off, ps, ip = tl.route_np(ids, cfg.E)
    qa = gsg.quantize_act_nvfp4(X.to(DEV), sf_block=sf, inv_perm=torch.from_numpy(ip).to(DEV), top_k=cfg.top_k)
    codes, quad, s, _, _ = tl.oracle_act(X.float().numpy(), sf, ps, cfg.top_k)
    assert qa.x_scale.item() == s
    np.testing.assert_array_equal(qa.codes.cpu().numpy(), codes)
    np.testing.assert_array_equal(qa.scales.cpu().numpy(), quad)
    _status_ok(gsg)


@pytest.mark.parametrize("T,k,E,K,sf", [(5, 40, 64, 512, 32), (9, 33, 48, 256, 16), (3, 3, 3, 768, 32)])
def test_quantize_many_routed_rows(gsg, T, k, E, K, sf):
    # top-k above one warp's 32 lanes, the 16-element block path and a K of three 256-wide slices
    cfg = inputs.custom_config("qk", E=E, K=K, N=128, T=T, top_k=k)
    X = inputs.activations(cfg)
    off, ps, ip = tl.route_np(inputs.routing(cfg), E)
    qa = gsg.quantize_act_nvfp4(X.to(DEV), sf_block=sf, inv_perm=torch.from_numpy(ip).to(DEV), top_k=k)
    codes, quad, s, _, _ = tl.oracle_act(X.float().numpy(), sf, ps, k)
    assert qa.x_scale.item() == s
    np.testing.assert_array_equal(qa.codes.cpu().numpy(), codes)
    np.testing.assert_array_equal(qa.scales.cpu().numpy(), quad)
    _status_ok(gsg)


# ---------------------------------------------------------------- routing + quantizer in one call
@pytest.mark.parametrize("name,T,k,E,K,sf,given_scale", [
    ("tiny", 0, 0, 0, 0, 32, False),
    ("30b_up_prefill", 0, 0, 0, 0, 32, False),        # R = 4096: 1024-row chunks
    ("30b_down_decode", 0, 0, 0, 0, 32, False),       # R = 512: one routing block
    ("1t_down_decode_b1", 0, 0, 0, 0, 32, False),
    ("tiny", 0, 0, 0, 0, 16, False),                  # dense control's 16-element blocks
    ("tiny", 0, 0, 0, 0, 32, True),                   # caller-supplied tensor scale: no amax blocks
    ("custom", 9000, 8, 512, 256, 32, False),         # R = 72000: 8192-row chunks, scan launch
    ("custom", 300, 7, 64, 512, 32, False),           # R = 2100: just past one block
    ("custom", 0, 8, 16, 256, 32, False),             # no tokens
])
def test_dispatch_matches_separate_calls_and_oracle(gsg, name, T, k, E, K, sf, given_scale):
    cfg = inputs.CONFIGS[name] if name != "custom" else inputs.custom_config("dp", E=E, K=K, N=128, T=T, top_k=k)
    X = inputs.activations(cfg).to(DEV)
    ids = inputs.routing(cfg) if cfg.T > 0 else torch.zeros(0, cfg.top_k, dtype=torch.int32)
    ids_d = ids.to(DEV)
    s_in = torch.tensor([0.0625], dtype=torch.float32, device=DEV) if given_scale else None
    r, qa = gsg.moe_dispatch_nvfp4(ids_d, X, cfg.E, sf_block=sf, x_scale_in=s_in)
    r2 = gsg.moe_route_permute(ids_d, cfg.E)
    qa2 = gsg.quantize_act_nvfp4(X, sf, r2.inv_perm, cfg.top_k, x_scale_in=s_in)
    _status_ok(gsg)
    R = cfg.T * cfg.top_k
    for a_, b_ in ((r.offsets, r2.offsets), (r.perm_src[:R], r2.perm_src[:R]), (r.inv_perm[:R], r2.inv_perm[:R]),
                   (qa.codes[:R], qa2.codes[:R]), (qa.scales, qa2.scales), (qa.x_scale, qa2.x_scale)):
        assert torch.equal(a_, b_)
    if given_scale:
        assert qa.x_scale.item() == 0.0625
    if R > 0 and R <= 8192:   # the oracle, on the sizes it finishes in seconds
        off, ps, ip = tl.route_np(ids, cfg.E)
        np.testing.assert_array_equal(r.offsets.cpu().numpy(), off)
        np.testing.assert_array_equal(r.perm_src.cpu().numpy()[:R], ps)
        if not given_scale:
            codes, quad, s, _, _ = tl.oracle_act(X.float().cpu().numpy(), sf, ps, cfg.top_k)
            assert qa.x_scale.item() == s
            np.testing.assert_array_equal(qa.codes.cpu().numpy()[:R], codes)
            np.testing.assert_array_equal(qa.scales.cpu().numpy(), quad)


@pytest.mark.parametrize("T,k,K,given_scale", [(2048, 8, 8192, False), (2304, 8, 7424, True), (1100, 16, 7680, False)])
def test_quantize_two_phase_scales(gsg, T, k, K, given_scale):
    # R*K >= 2^27: scale words staged row-major in the workspace, then rearranged into the quad
    # layout by a second launch (K = 7424: a warp's blocks straddle two tokens; k = 16: rows
    # beyond the eight fetched ahead)
    assert T * k * K >= 1 << 27
    cfg = inputs.custom_config("q2", E=64, K=K, N=128, T=T, top_k=k)
    X = inputs.activations(cfg)
    ids = inputs.routing(cfg)
    off, ps, ip = tl.route_np(ids, cfg.E)
    s_in = torch.tensor([0.03125], dtype=torch.float32, device=DEV) if given_scale else None
    qa = gsg.quantize_act_nvfp4(X.to(DEV), 32, torch.from_numpy(ip).to(DEV), k, x_scale_in=s_in)
    r, qd = gsg.moe_dispatch_nvfp4(ids.to(DEV), X.to(DEV), cfg.E, 32, x_scale_in=s_in)
    _status_ok(gsg)
    codes, quad, s, _, _ = tl.oracle_act(X.float().numpy(), 32, ps, k, 0.03125 if given_scale else None)
    assert qa.x_scale.item() == s
    np.testing.assert_array_equal(qa.codes.cpu().numpy(), codes)
    np.testing.assert_array_equal(qa.scales.cpu().numpy(), quad)
    assert torch.equal(qd.codes, qa.codes) and torch.equal(qd.scales, qa.scales) and torch.equal(qd.x_scale, qa.x_scale)


def _rounding_rows():
    """bf16 rows whose 32-element blocks put values exactly on E2M1 rounding midpoints and block
    maxima exactly on UE4M3 midpoints, subnormals and the saturation limit (with s_x = 1)."""
    mids = [0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0]
    grid = [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]
    blocks = []
    for j in (-6, -2, 0, 3):                      # scale 2^j: block max 6 * 2^j
        v = [6.0] + mids + [-m for m in mids] + grid + [-g for g in grid[1:]] + [0.1, -0.1, -0.0]
        blocks.append([x * 2.0 ** j for x in v[:32]])
    # block maxima / 6 on UE4M3 ties (1.0625 -> 1.0, 1.1875 -> 1.25), a subnormal tie
    # (1.5 * 2^-9 -> 2^-8) and one far above 6 * 448 (saturates)
    for amax in (6.375, 7.125, 9.0 * 2.0 ** -9, 4096.0):
        blocks.append([amax] + [amax * f for f in (0.5, -0.25, 0.125, 0.9, -0.7, 0.33)] + [0.0] * 25)
    rows = [sum(blocks[i:i + 8], []) for i in range(0, len(blocks), 8)]
    return torch.tensor(rows, dtype=torch.float32).to(torch.bfloat16)


@pytest.mark.parametrize("sf", [32, 16])
def test_quantize_rounding_midpoints(gsg, sf):
    X = _rounding_rows()
    assert X.float().abs().max().item() == 4096.0     # 4096 / 6 > 448: the saturating block
    one = torch.tensor([1.0], dtype=torch.float32)
    qa = gsg.quantize_act_nvfp4(X.to(DEV), sf_block=sf, x_scale_in=one.to(DEV))
    codes, quad, s, _, _ = tl.oracle_act(X.float().numpy(), sf, None, 1, np.float32(1.0))
    np.testing.assert_array_equal(qa.codes.cpu().numpy(), codes)
    np.testing.assert_array_equal(qa.scales.cpu().numpy(), quad)
    _status_ok(gsg)


def test_quantize_identity_and_given_scale(gsg):
    cfg = inputs.custom_config("q", E=1, K=512, N=128, T=37, top_k=1, outlier_frac=0.01, outlier_scale=50.0)
    X = inputs.activations(cfg)
    s_in = torch.tensor([0.0123], dtype=torch.float32)
    qa = gsg.quantize_act_nvfp4(X.to(DEV), sf_block=32, x_scale_in=s_in.to(DEV))
    codes, quad, s, _, _ = tl.oracle_act(X.float().numpy(), 32, None, 1, np.float32(0.0123))
    assert qa.x_scale.item() == np.float32(0.0123)
    np.testing.assert_array_equal(qa.codes.cpu().numpy(), codes)
    np.testing.assert_array_equal(qa.scales.cpu().numpy(), quad)
    Z = torch.zeros(5, 256, dtype=torch.bfloat16)
    qz = gsg.quantize_act_nvfp4(Z.to(DEV), sf_block=32)
    assert qz.x_scale.item() == 1.0 and not qz.codes.any().item()


# ---------------------------------------------------------------- scatter
@pytest.mark.parametrize("T,k,N", [(32, 2, 128), (64, 8, 2048), (7, 3, 136)])
def test_unpermute_bit_exact(gsg, T, k, N):
    Y = inputs.random_bf16((T * k, N), seed=21)
    g = inputs.gates(inputs.custom_config("u", E=8, K=256, N=N, T=T, top_k=k))
    ip = torch.randperm(T * k, generator=torch.Generator().manual_seed(5)).to(torch.int32)
    out = gsg.unpermute_scale(Y.to(DEV), ip.to(DEV), g.to(DEV), k)
    ref = ounperm.unpermute_scale(Y.view(torch.uint16).numpy(), ip.numpy(), g.numpy(), k)
    np.testing.assert_array_equal(out.cpu().view(torch.uint16).numpy(), ref)


# ---------------------------------------------------------------- grouped GEMM on oracle-packed inputs
def _gemm_case(counts, N, K, seed=0, sparse=True):
    E = len(counts)
    cfg = inputs.custom_config("g", E=E, K=K, N=N, T=int(sum(counts)), top_k=1, w_sigma=0.02)
    W = inputs.all_weights(cfg).numpy()
    X = inputs.activations(cfg).float().numpy()
    off = np.concatenate([[0], np.cumsum(counts)]).astype(np.int32)
    sf = 32 if sparse else 16
    a_codes, a_quad, s_x, q, sc = tl.oracle_act(X, sf, None, 1)
    if sparse:
        packed, sws, canon = tl.oracle_pack_sparse(W)
    else:
        packed, sws, canon = tl.oracle_pack_dense(W, 16)
    w = dict(packed=packed, w_scale=sws)
    return dict(E=E, N=N, K=K, R=int(off[-1]), off=off, a_codes=a_codes, a_quad=a_quad, s_x=s_x, q=q, sc=sc,
                w=w, canon=canon, sws=sws, sf=sf)


def _run_gemm(gsg, c, sparse, hint, out_dtype, native=False):
    t = lambda a: torch.from_numpy(np.ascontiguousarray(a)).to(DEV)
    act = gsg.QuantizedActivations(codes=t(c["a_codes"]), scales=t(c["a_quad"]),
                                   x_scale=torch.tensor([c["s_x"]], dtype=torch.float32, device=DEV),
                                   R=c["R"], K=c["K"], sf_block=c["sf"])
    off = t(c["off"])
    if sparse:
        w = gsg.PackedSparseWeights(packed=t(c["w"]["packed"]), w_scale=t(c["w"]["w_scale"]), E=c["E"], N=c["N"],
                                    K=c["K"])
        return gsg.grouped_sparse_gemm(act, w, off, max_rows_per_expert=hint, out_dtype=out_dtype)
    w = gsg.PackedDenseWeights(packed=t(c["w"]["packed"]), w_scale=t(c["w"]["w_scale"]), E=c["E"], N=c["N"],
                               K=c["K"])
    if native:
        return gsg.grouped_dense_gemm_native(act, w, off, max_rows_per_expert=hint, out_dtype=out_dtype)
    return gsg.grouped_dense_gemm(act, w, off, max_rows_per_expert=hint, out_dtype=out_dtype)


GEMM_CASES = [
    ([16], 128, 256),                              # one tile
    ([5, 0, 33], 256, 512),                        # ragged, an empty expert, two n-tiles
    ([0, 1, 7, 8, 9, 127, 128, 129], 128, 768),    # the ragged-tail ladder
    ([300, 2, 64], 384, 1024),                     # 128-token tiles, an odd n-tile count: one CTA per tile
    # 128-token tiles run by CTA pairs (256 weight rows per tile, each CTA half of the tokens): tiles
    # whose second CTA gets no rows (8, 1), one row (17), a partial half (100 -> N = 112), exactly
    # half (64, 128) and every ragged edge around them
    ([1, 8, 9, 16, 17, 56, 57, 63, 64, 65, 100, 127, 128, 129, 255, 256, 257, 0, 300], 512, 512),
    # the same pair tiles are 256 tokens in two 128-token halves: second halves of 8 (no rows on the
    # second CTA), 17, 32, 64, 72 and 112 rows, and tiles after a full first tile
    ([136, 145, 160, 192, 200, 240, 512, 520, 3], 256, 768),
]


@pytest.mark.parametrize("counts,N,K", GEMM_CASES)
@pytest.mark.parametrize("hint", [-1, 16, 64])
def test_sparse_gemm_oracle_inputs(gsg, counts, N, K, hint):
    c = _gemm_case(counts, N, K, sparse=True)
    y = _run_gemm(gsg, c, True, hint, torch.float32)
    torch.cuda.synchronize()
    _status_ok(gsg)
    y_ref, bound = tl.reference_rows(np.arange(c["R"]), c["off"], c["q"], c["sc"], 32, c["canon"], c["s_x"], c["sws"])
    tl.assert_gemm_close(y[:c["R"]], y_ref, bound, f"sparse {counts} hint {hint}")


@pytest.mark.parametrize("counts,N,K", GEMM_CASES)
@pytest.mark.parametrize("sparse", [True, False])
def test_gemm_bf16_output(gsg, counts, N, K, sparse):
    """bf16 output of every tile shape (128-token tiles, CTA pairs and wide pair tiles included, whose
    epilogue packs the accumulator into bf16 pairs in registers): within the bound, and exactly the
    fp32 output rounded once to bf16."""
    c = _gemm_case(counts, N, K, sparse=sparse)
    y = _run_gemm(gsg, c, sparse, -1, torch.bfloat16)
    y32 = _run_gemm(gsg, c, sparse, -1, torch.float32)
    torch.cuda.synchronize()
    _status_ok(gsg)
    sf = 32 if sparse else 16
    y_ref, bound = tl.reference_rows(np.arange(c["R"]), c["off"], c["q"], c["sc"], sf, c["canon"], c["s_x"], c["sws"],
                                     sparse=sparse, w_sf=sf)
    tl.assert_gemm_close(y[:c["R"]], y_ref, bound, f"{'sparse' if sparse else 'dense'} bf16 {counts}")
    assert torch.equal(y[:c["R"]], y32[:c["R"]].to(torch.bfloat16))


@pytest.mark.parametrize("counts,N,K", GEMM_CASES)
def test_dense_gemm_oracle_inputs(gsg, counts, N, K):
    c = _gemm_case(counts, N, K, sparse=False)
    y = _run_gemm(gsg, c, False, -1, torch.float32)
    y_ref, bound = tl.reference_rows(np.arange(c["R"]), c["off"], c["q"], c["sc"], 16, c["canon"], c["s_x"],
                                     c["sws"], sparse=False, w_sf=16)
    tl.assert_gemm_close(y[:c["R"]], y_ref, bound, f"dense {counts}")


@pytest.mark.parametrize("counts,N,K", GEMM_CASES)
@pytest.mark.parametrize("out_dtype", [torch.float32, torch.bfloat16])
def test_dense_native_gemm_oracle_inputs(gsg, counts, N, K, out_dtype):
    """The dense control in the activation-stationary orientation (tokens as MMA operand A)."""
    c = _gemm_case(counts, N, K, sparse=False)
    y = _run_gemm(gsg, c, False, -1, out_dtype, native=True)
    torch.cuda.synchronize()
    _status_ok(gsg)
    y_ref, bound = tl.reference_rows(np.arange(c["R"]), c["off"], c["q"], c["sc"], 16, c["canon"], c["s_x"],
                                     c["sws"], sparse=False, w_sf=16)
    tl.assert_gemm_close(y[:c["R"]], y_ref, bound, f"dense native {counts}")


def test_gemm_deterministic(gsg):
    c = _gemm_case([40, 3, 77], 256, 512, sparse=True)
    y1 = _run_gemm(gsg, c, True, 32, torch.float32)
    y2 = _run_gemm(gsg, c, True, 32, torch.float32)
    assert torch.equal(y1, y2)


def test_gemm_flags_corrupt_offsets(gsg):
    """Offsets that decrease or leave [0, R] are clamped in the kernel (a decreasing pair makes
    that expert empty), so nothing is read or written out of bounds, and the call reports
    GSG_ERR_BAD_ROUTING; the rows of the experts whose offsets are intact are still right."""
    c = _gemm_case([16, 8, 24, 8], 128, 256, sparse=True)
    good = c["off"].copy()                       # [0, 16, 24, 48, 56]
    bad = dict(c)
    bad["off"] = np.array([0, 16, 10, 999999, 56], dtype=np.int32)
    y = _run_gemm(gsg, bad, True, -1, torch.float32)
    torch.cuda.synchronize()
    assert gsg.get_device_status() == -4
    _status_ok(gsg)
    # clamped offsets [0, 16, 10, 56, 56]: rows [0, 10) belong to expert 0 alone (rows 10..15 are
    # claimed by expert 2 as well), and they still hold the oracle's values
    y_ref, bound = tl.reference_rows(np.arange(10), good, c["q"], c["sc"], 32, c["canon"], c["s_x"], c["sws"])
    tl.assert_gemm_close(y[:10], y_ref, bound, "expert 0 beside corrupt offsets")


@pytest.mark.parametrize("sparse,counts", [(True, [40, 3, 77, 130, 0, 9]), (False, [40, 3, 77, 130, 0, 9]),
                                           (True, [300, 130, 0, 9]), (False, [300, 130, 0, 9])])
def test_gemm_wait_timeout_aborts_cleanly(gsg, sparse, counts):
    """Failure detection: the test hook makes the MMA warp wait on a barrier that nothing
    arrives on, with a 1 ms limit.  The launch must come back (no hang) with
    GSG_ERR_DEVICE_TIMEOUT in the status word after draining its own copies and tensor-core work
    and freeing its tensor memory; the next normal launch on the same context is correct."""
    import time
    c = _gemm_case(counts, 256, 512, sparse=sparse)   # 64-token tiles; 128-token tiles on CTA pairs
    L = gsg.lib()
    try:
        L.gsg_test_set_gemm_stall_ns(1_000_000)
        t0 = time.time()
        _run_gemm(gsg, c, sparse, -1, torch.float32)
        assert gsg.get_device_status() == -6
        assert time.time() - t0 < 30.0
    finally:
        L.gsg_test_set_gemm_stall_ns(0)
    y = _run_gemm(gsg, c, sparse, -1, torch.float32)
    _status_ok(gsg)
    sf = 32 if sparse else 16
    y_ref, bound = tl.reference_rows(np.arange(c["R"]), c["off"], c["q"], c["sc"], sf, c["canon"], c["s_x"],
                                     c["sws"], sparse=sparse, w_sf=16)
    tl.assert_gemm_close(y[:c["R"]], y_ref, bound, "after a timed-out launch")


@pytest.mark.parametrize("sparse", [True, False])
@pytest.mark.parametrize("counts,N,K", [GEMM_CASES[2], GEMM_CASES[4], GEMM_CASES[5]])
def test_gemm_tiles_decoded_without_table(gsg, sparse, counts, N, K):
    """Tiles past a CTA's tile table are decoded from the expert offsets as the roles reach them
    (the path of launches with more tiles per CTA than the table holds): with the table capped at
    0 and 1 entries the result is bit-identical to the normal launch and within the bound."""
    c = _gemm_case(counts, N, K, sparse=sparse)
    y0 = _run_gemm(gsg, c, sparse, -1, torch.float32)
    L = gsg.lib()
    try:
        for cap in (0, 1):
            L.gsg_test_set_gemm_table_cap(cap)
            y = _run_gemm(gsg, c, sparse, -1, torch.float32)
            torch.cuda.synchronize()
            _status_ok(gsg)
            assert torch.equal(y[:c["R"]], y0[:c["R"]]), f"table cap {cap}"
    finally:
        L.gsg_test_set_gemm_table_cap(-1)
    sf = 32 if sparse else 16
    y_ref, bound = tl.reference_rows(np.arange(c["R"]), c["off"], c["q"], c["sc"], sf, c["canon"], c["s_x"],
                                     c["sws"], sparse=sparse, w_sf=sf)
    tl.assert_gemm_close(y0[:c["R"]], y_ref, bound, "with the full tile table")


def test_dense_and_sparse_agree_on_48_weights(gsg):
    """The control differs from the sparse kernel only in sparsity: a W that is already paired
    4:8 gives results within tolerance of one reference on both (32-blocks copied into 16-blocks)."""
    counts, N, K = [20, 9], 128, 512
    c = _gemm_case(counts, N, K, sparse=True)
    # dense weights: scatter the retained codes with +0 at pruned slots; duplicate each 32-block scale
    dblocks = []
    for (codes, pats, scales) in c["canon"]:
        full = np.zeros((N, K // 8, 4, 2), dtype=np.uint8)
        np.put_along_axis(full, opack.pattern_pairs(pats)[..., None].repeat(2, axis=-1),
                          codes.reshape(N, K // 8, 2, 2), axis=-2)
        dblocks.append(olayout.packed_dense(full.reshape(N, K), np.repeat(scales, 2, axis=1)).reshape(-1))
    # activations with 16-blocks carrying the same scale as their 32-block
    q, sc = c["q"], c["sc"]
    d = dict(c)
    d["w"] = dict(packed=np.concatenate(dblocks), w_scale=c["sws"])
    d["a_quad"] = olayout.quad_act_scales(np.repeat(sc, 2, axis=1)).reshape(-1)
    d["sf"] = 16
    y_sparse = _run_gemm(gsg, c, True, -1, torch.float32)
    y_dense = _run_gemm(gsg, d, False, -1, torch.float32)
    y_ref, bound = tl.reference_rows(np.arange(c["R"]), c["off"], q, sc, 32, c["canon"], c["s_x"], c["sws"])
    tl.assert_gemm_close(y_sparse[:c["R"]], y_ref, bound, "sparse")
    tl.assert_gemm_close(y_dense[:c["R"]], y_ref, bound, "dense control")


# ---------------------------------------------------------------- the whole path
@pytest.mark.parametrize("name", ["tiny", "30b_down_decode", "1t_down_decode_b1"])
def test_pipeline_matches_oracle(gsg, name):
    cfg = inputs.CONFIGS[name]
    E, N, K = cfg.E, cfg.N, cfg.K
    W = torch.stack([inputs.expert_weight(cfg, e, DEV) for e in range(E)])
    X = inputs.activations(cfg)
    ids = inputs.routing(cfg)
    gates = inputs.gates(cfg)
    pw = gsg.pack_sparse_nvfp4(W)
    r = gsg.moe_route_permute(ids.to(DEV), E)
    qa = gsg.quantize_act_nvfp4(X.to(DEV), 32, r.inv_perm, cfg.top_k)
    counts = torch.bincount(ids.reshape(-1).long(), minlength=E)
    Y = gsg.grouped_sparse_gemm(qa, pw, r.offsets, int(counts.max()), out_dtype=torch.float32)
    out = gsg.unpermute_scale(Y.to(torch.bfloat16), r.inv_perm, gates.to(DEV), cfg.top_k)
    torch.cuda.synchronize()
    _status_ok(gsg)
    # oracle, from the same inputs only
    off, ps, ip = tl.route_np(ids, E)
    _, _, s_x, q, sc = tl.oracle_act(X.float().numpy(), 32, ps, cfg.top_k)
    touched = np.unique(ids.numpy())
    rows = np.arange(cfg.R)
    canon = {}
    sws = np.zeros(E, dtype=np.float32)
    for e in touched:
        codes, pats, scales, s_w = opack.pack_sparse_expert(W[int(e)].cpu().numpy())
        canon[int(e)] = (codes, pats, scales)
        sws[e] = s_w
    y_ref, bound = tl.reference_rows(rows, off, q, sc, 32, canon, s_x, sws)
    tl.assert_gemm_close(Y[:cfg.R], y_ref, bound, f"pipeline GEMM {name}")
    # scatter: tolerance form against y_ref (sum_j |g_j| (tol_j) + bf16 rounding of the sum)
    g = gates.numpy().astype(np.float64)
    yr = y_ref[ip.reshape(cfg.T, cfg.top_k)]
    br = bound[ip.reshape(cfg.T, cfg.top_k)]
    ref = np.einsum("tj,tjn->tn", g, yr)
    tol = np.einsum("tj,tjn->tn", np.abs(g), 2.0 ** -10 * br + 1e-6 + tl.ogemm.bf16_half_ulp(np.abs(yr) + 1e-6))
    tol = tol + 2.0 ** -8 * np.abs(ref) + 1e-6
    err = np.abs(out.float().cpu().numpy() - ref)
    assert np.all(err <= tol), float(np.max(err / tol))


# ---------------------------------------------------------------- up-projection with the SwiGLU epilogue
def _unquad(quad: np.ndarray, R: int, K: int) -> np.ndarray:
    """Quad activation-scale bytes -> scales [R, K/32] (entry (kb, r, 0, j) is row r, block 4 kb + j)."""
    q = np.asarray(quad, dtype=np.uint8).reshape(K // 128, R + olayout.ACT_SCALE_PAD_ROWS, 4, 4)
    return q[:, :R, 0, :].transpose(1, 0, 2).reshape(R, K // 32)


SWIGLU_CASES = [
    ([16], 128, 256),                        # one tile, I = 128
    ([40, 0, 77], 256, 512),                 # ragged with an empty expert
    ([0, 1, 7, 9, 33, 64], 128, 768),        # the small-tile ladder
    ([300, 5], 384, 256),                    # tiles above 64 rows (64-token tiles), I = 384
]


@pytest.mark.parametrize("counts,I,K", SWIGLU_CASES)
def test_swiglu_gemm_matches_oracle(gsg, counts, I, K):
    from oracle import codecs as ocodecs
    from oracle import quant as oquant
    from oracle import swiglu as oswiglu
    c = _gemm_case(counts, 2 * I, K, sparse=True)
    R = c["R"]
    y_ref, b = tl.reference_rows(np.arange(R), c["off"], c["q"], c["sc"], 32, c["canon"], c["s_x"], c["sws"])
    h_ref = oswiglu.swiglu_rows(y_ref)
    s_h = np.float32(np.abs(h_ref).max() / 2688.0)
    t = lambda a: torch.from_numpy(np.ascontiguousarray(a)).to(DEV)
    act = gsg.QuantizedActivations(codes=t(c["a_codes"]), scales=t(c["a_quad"]),
                                   x_scale=torch.tensor([c["s_x"]], dtype=torch.float32, device=DEV), R=R, K=K,
                                   sf_block=32)
    w = gsg.PackedSparseWeights(packed=t(c["w"]["packed"]), w_scale=t(c["w"]["w_scale"]), E=c["E"], N=2 * I, K=K)
    hq = gsg.grouped_sparse_gemm_swiglu(act, w, t(c["off"]), torch.tensor([s_h], device=DEV),
                                        max_rows_per_expert=max(counts))
    _status_ok(gsg)
    codes = olayout.unpack_act_codes(hq.codes.cpu().numpy()[:R])
    quad = hq.scales.cpu().numpy()
    scales = _unquad(quad, R, I)
    hd = oquant.decode_rows(codes, scales, 32) * float(s_h)
    # one quantization step of the block (|v - dec(q(v))| <= d for the E2M1 grid, saturation
    # included) + the exact propagation of the GEMM tolerance through silu(g) * u + the fp32
    # evaluation of silu (fast exponential and division: a few ulp, 2^-16 relative is ample)
    d_blk = np.repeat(ocodecs.ue4m3_decode(scales).astype(np.float64) * float(s_h), 32, axis=1)
    tau = 2.0 ** -10 * b + 1e-6
    bound = d_blk + oswiglu.swiglu_error_bound(y_ref, tau) + 2.0 ** -16 * np.abs(h_ref)
    err = np.abs(hd - h_ref)
    assert np.all(err <= bound), (np.max(err - bound), np.argmax(err - bound))
    # almost every code equals the oracle's quantization of the exact h
    qr, scr = oquant.quantize_rows(h_ref.astype(np.float32), 32, s_h)
    assert np.mean(codes == qr) > 0.95 and np.mean(scales == scr) > 0.95
    # scale entries that refer to rows >= R are zero
    q5 = quad.reshape(I // 128, R + olayout.ACT_SCALE_PAD_ROWS, 4, 4)
    for cc in range(4):
        rr = np.arange(R + olayout.ACT_SCALE_PAD_ROWS)
        assert not q5[:, rr + 32 * cc >= R, cc, :].any()


# ---------------------------------------------------------------- a whole MoE layer
@pytest.mark.parametrize("name", ["tiny_layer"])
def test_moe_layer_pipeline(gsg, name):
    """route -> quantize -> up-projection with the SwiGLU epilogue -> down-projection -> unpermute,
    every stage checked against the oracle on the inputs it actually received: routing and X
    quantization bit-exact, h within one quantization step plus the propagated GEMM tolerance,
    the down-projection within the GEMM tolerance on the GPU's own h, the scatter bit-exact."""
    from oracle import codecs as ocodecs
    from oracle import quant as oquant
    from oracle import swiglu as oswiglu
    L = inputs.LAYERS[name]
    up, dn = L.up(), L.down()
    X, ids, g = inputs.activations(up), inputs.routing(up), inputs.gates(up)
    Wu = inputs.all_weights(up).numpy()
    Wd = torch.stack([inputs.down_weight(L, e) for e in range(L.E)]).numpy()
    pu, swu, cu = tl.oracle_pack_sparse(Wu)
    pdn, swd, cd = tl.oracle_pack_sparse(Wd)
    off, ps, ip = tl.route_np(ids, L.E)
    codes, quad, s_x, q, sc = tl.oracle_act(X.float().numpy(), 32, ps, L.top_k)
    R = L.R
    y_up, b_up = tl.reference_rows(np.arange(R), off, q, sc, 32, cu, s_x, swu)
    h_ref = oswiglu.swiglu_rows(y_up)
    s_h = np.float32(np.abs(h_ref).max() / 2688.0)
    t = lambda a: torch.from_numpy(np.ascontiguousarray(a)).to(DEV)
    # --- the GPU path, every step through the library
    r = gsg.moe_route_permute(ids.to(DEV), L.E)
    qa = gsg.quantize_act_nvfp4(X.to(DEV), 32, r.inv_perm, L.top_k)
    wu = gsg.PackedSparseWeights(packed=t(pu), w_scale=t(swu), E=L.E, N=2 * L.I, K=L.H)
    wd = gsg.PackedSparseWeights(packed=t(pdn), w_scale=t(swd), E=L.E, N=L.H, K=L.I)
    hq = gsg.grouped_sparse_gemm_swiglu(qa, wu, r.offsets, torch.tensor([s_h], device=DEV))
    Y2 = gsg.grouped_sparse_gemm(hq, wd, r.offsets)
    out = gsg.unpermute_scale(Y2, r.inv_perm, g.to(DEV), L.top_k)
    _status_ok(gsg)
    np.testing.assert_array_equal(r.offsets.cpu().numpy(), off)
    np.testing.assert_array_equal(qa.codes.cpu().numpy(), codes)
    # h
    hc = olayout.unpack_act_codes(hq.codes.cpu().numpy()[:R])
    hs = _unquad(hq.scales.cpu().numpy(), R, L.I)
    hd = oquant.decode_rows(hc, hs, 32) * float(s_h)
    bound_h = (np.repeat(ocodecs.ue4m3_decode(hs).astype(np.float64) * float(s_h), 32, axis=1) +
               oswiglu.swiglu_error_bound(y_up, 2.0 ** -10 * b_up + 1e-6) + 2.0 ** -16 * np.abs(h_ref))
    assert np.all(np.abs(hd - h_ref) <= bound_h)
    # down-projection on the GPU's h
    y_dn, b_dn = tl.reference_rows(np.arange(R), off, hc, hs, 32, cd, s_h, swd)
    tl.assert_gemm_close(Y2[:R], y_dn, b_dn, "layer down-projection")
    # scatter
    ref = ounperm.unpermute_scale(Y2.cpu().view(torch.uint16).numpy(), ip, g.numpy(), L.top_k)
    np.testing.assert_array_equal(out.cpu().view(torch.uint16).numpy(), ref)


# ---------------------------------------------------------------- down-projection with the combine epilogue
@pytest.mark.parametrize("name", ["tiny", "30b_down_decode", "1t_down_decode_b1", "dup"])
def test_combine_gemm_equals_gemm_then_unpermute(gsg, name):
    """The fused combine is the unfused GEMM (bf16 Y) + scatter bit for bit, on every token, and
    it leaves its counters at zero so the workspace can be reused."""
    if name == "dup":     # a token that picks the same expert twice, and uneven expert loads
        cfg = inputs.custom_config("dup", E=5, K=512, N=256, T=40, top_k=3, routing="zipf", zipf_s=1.5)
        ids = inputs.routing(cfg)
        ids[3] = torch.tensor([2, 2, 4], dtype=torch.int32)
    else:
        cfg = inputs.CONFIGS[name]
        ids = inputs.routing(cfg)
    X, g = inputs.activations(cfg).to(DEV), inputs.gates(cfg).to(DEV)
    L = gsg.lib()
    w = gsg.PackedSparseWeights(packed=torch.empty(L.gsg_sparse_packed_bytes(cfg.E, cfg.N, cfg.K), dtype=torch.uint8,
                                                   device=DEV),
                                w_scale=torch.empty(cfg.E, dtype=torch.float32, device=DEV), E=cfg.E, N=cfg.N, K=cfg.K)
    for e in range(cfg.E):    # one expert at a time (the 1T weights are 22 GB in fp32)
        gsg.pack_sparse_nvfp4(inputs.expert_weight(cfg, e, DEV)[None], out=w.expert(e))
    r = gsg.moe_route_permute(ids.to(DEV), cfg.E)
    qa = gsg.quantize_act_nvfp4(X, 32, r.inv_perm, cfg.top_k)
    Y = gsg.grouped_sparse_gemm(qa, w, r.offsets)
    ref = gsg.unpermute_scale(Y, r.inv_perm, g, cfg.top_k)
    ws = gsg.combine_workspace(cfg.E, cfg.N, cfg.K, cfg.T, cfg.top_k, DEV)
    for _ in range(2):
        out = gsg.grouped_sparse_gemm_combine(qa, w, r, g, ws)
        _status_ok(gsg)
        np.testing.assert_array_equal(out.cpu().view(torch.uint16).numpy(), ref.cpu().view(torch.uint16).numpy())
        slots = cfg.T * cfg.top_k * cfg.N * 2
        assert not ws[(slots + 255) // 256 * 256:].any()          # counters back at zero
    # and against the oracle scatter of the GPU's own Y
    oref = ounperm.unpermute_scale(Y.cpu().view(torch.uint16).numpy(), r.inv_perm.cpu().numpy(), g.cpu().numpy(),
                                   cfg.top_k)
    np.testing.assert_array_equal(out.cpu().view(torch.uint16).numpy(), oref)


def test_combine_wait_timeout_then_clean_call(gsg):
    """The combine's abort path: with the timeout hook the launch returns GSG_ERR_DEVICE_TIMEOUT (its
    CTAs still pass the grid barrier and reset its counters); the next normal call on the same
    workspace is the scatter's result bit for bit and leaves the counters at zero."""
    cfg = inputs.custom_config("ct", E=6, K=512, N=256, T=48, top_k=4, routing="zipf", zipf_s=1.2)
    ids = inputs.routing(cfg)
    X, g = inputs.activations(cfg).to(DEV), inputs.gates(cfg).to(DEV)
    w = gsg.pack_sparse_nvfp4(inputs.all_weights(cfg).to(DEV))
    r = gsg.moe_route_permute(ids.to(DEV), cfg.E)
    qa = gsg.quantize_act_nvfp4(X, 32, r.inv_perm, cfg.top_k)
    ref = gsg.unpermute_scale(gsg.grouped_sparse_gemm(qa, w, r.offsets), r.inv_perm, g, cfg.top_k)
    ws = gsg.combine_workspace(cfg.E, cfg.N, cfg.K, cfg.T, cfg.top_k, DEV)
    L = gsg.lib()
    try:
        L.gsg_test_set_gemm_stall_ns(1_000_000)
        gsg.grouped_sparse_gemm_combine(qa, w, r, g, ws)
        assert gsg.get_device_status() == -6
    finally:
        L.gsg_test_set_gemm_stall_ns(0)
    slots = cfg.T * cfg.top_k * cfg.N * 2
    assert not ws[(slots + 255) // 256 * 256:].any()          # the barrier's counters back at zero
    out = gsg.grouped_sparse_gemm_combine(qa, w, r, g, ws)
    _status_ok(gsg)
    assert torch.equal(out, ref)
    assert not ws[(slots + 255) // 256 * 256:].any()


def test_combine_skips_corrupt_slot_indices(gsg):
    """perm_src entries outside [0, T*k) are skipped by the combine epilogue (nothing stored)
    and reported as GSG_ERR_BAD_ROUTING; every token none of whose rows was corrupted still gets
    the scatter's result bit for bit."""
    cfg = inputs.custom_config("cc", E=6, K=512, N=256, T=48, top_k=4, routing="zipf", zipf_s=1.2)
    ids = inputs.routing(cfg)
    X, g = inputs.activations(cfg).to(DEV), inputs.gates(cfg).to(DEV)
    w = gsg.pack_sparse_nvfp4(inputs.all_weights(cfg).to(DEV))
    r = gsg.moe_route_permute(ids.to(DEV), cfg.E)
    qa = gsg.quantize_act_nvfp4(X, 32, r.inv_perm, cfg.top_k)
    Y = gsg.grouped_sparse_gemm(qa, w, r.offsets)
    ref = gsg.unpermute_scale(Y, r.inv_perm, g, cfg.top_k)
    R = cfg.R
    bad_rows = [5, R - 1]
    lost = {int(r.perm_src[i].item()) // cfg.top_k for i in bad_rows}
    ps_bad = r.perm_src.clone()
    ps_bad[bad_rows[0]] = R + 7
    ps_bad[bad_rows[1]] = -3
    rb = gsg.Routing(offsets=r.offsets, perm_src=ps_bad, inv_perm=r.inv_perm, T=cfg.T, k=cfg.top_k, E=cfg.E)
    ws = gsg.combine_workspace(cfg.E, cfg.N, cfg.K, cfg.T, cfg.top_k, DEV)
    out = torch.zeros(cfg.T, cfg.N, dtype=torch.bfloat16, device=DEV)
    gsg.grouped_sparse_gemm_combine(qa, w, rb, g, ws, out=out)
    assert gsg.get_device_status() == -4
    _status_ok(gsg)
    keep = torch.tensor([t not in lost for t in range(cfg.T)])
    assert keep.sum().item() == cfg.T - len(lost)
    assert torch.equal(out.cpu()[keep], ref.cpu()[keep])
