"""GPU parity at the full sizes of the workloads, through the C ABI.

Every expert-projection configuration at its real size (30B-A3B up-projection prefill, the 1T
up-projection prefill of 8192 tokens top-8 on 384 experts, the 1T down-projection decode batches)
and the whole MoE layer at the 30B-A3B and 1T shapes.  The oracle cannot redo a whole launch at
these sizes in seconds, so:
  * every expert is packed on the GPU; the packed bytes and tensor scale of sampled experts (the
    largest, the smallest non-empty, the first, the last and two seeded others) are compared bit
    for bit with the oracle's packer and layout;
  * routing and the quantized activations of the whole batch are compared bit for bit (at the
    1T prefill shape this is the two-phase scale path at exactly the bench's size);
  * GEMM outputs are checked on sampled rows of the sampled experts -- first, last, middle, the
    rows around 64 and 128 (the split of a token tile between two SMs and the token-tile edge)
    and the first row of the last partial token tile -- at the stated bound, all N columns.
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
    return g


def _sample_experts(counts: np.ndarray, n_seeded: int = 2, seed: int = 11):
    nz = np.flatnonzero(counts)
    chosen = {int(np.argmax(counts)), int(nz[np.argmin(counts[nz])]), int(nz[0]), int(nz[-1])}
    rest = np.array([e for e in nz if e not in chosen])
    if rest.size:
        rng = np.random.default_rng(seed)
        chosen |= {int(e) for e in rng.choice(rest, size=min(n_seeded, rest.size), replace=False)}
    return sorted(chosen)


def _sample_rows(off: np.ndarray, experts):
    rows = []
    for e in experts:
        lo, hi = int(off[e]), int(off[e + 1])
        n = hi - lo
        cand = {0, n - 1, n // 2, 31, 32, 63, 64, 65, 127, 128, 129,
                ((n - 1) // 64) * 64, ((n - 1) // 128) * 128}
        rows += sorted(lo + c for c in cand if 0 <= c < n)
    return np.array(rows, dtype=np.int64)


def _pack_all(gsg, cfg, weight_fn, sample_e):
    """Pack every expert on the GPU one at a time (the fp32 weights of the 1T shapes do not fit
    at once); oracle-pack the sampled ones and compare bytes and tensor scale bit for bit."""
    E, N, K = cfg.E, cfg.N, cfg.K
    pw = gsg.PackedSparseWeights(
        packed=torch.empty(gsg.lib().gsg_sparse_packed_bytes(E, N, K), dtype=torch.uint8, device=DEV),
        w_scale=torch.empty(E, dtype=torch.float32, device=DEV), E=E, N=N, K=K)
    canon, sws = {}, np.zeros(E, dtype=np.float32)
    for e in range(E):
        We = weight_fn(e)
        sub = pw.expert(e)
        gsg.pack_sparse_nvfp4(We[None], out=sub)
        if e in sample_e:
            codes, pats, scales, s_w = opack.pack_sparse_expert(We.cpu().numpy())
            canon[e] = (codes, pats, scales)
            sws[e] = s_w
            np.testing.assert_array_equal(sub.packed.cpu().numpy(),
                                          olayout.packed_sparse(codes, pats, scales).reshape(-1), err_msg=f"e={e}")
            assert sub.w_scale.item() == s_w
        del We
    return pw, canon, sws


def _check_dispatch(gsg, cfg, ids, X, r, qa):
    """Routing and the whole batch's quantized activations bit for bit against the oracle."""
    off, ps, ip = tl.route_np(ids, cfg.E)
    R = cfg.R
    np.testing.assert_array_equal(r.offsets.cpu().numpy(), off)
    np.testing.assert_array_equal(r.perm_src.cpu().numpy()[:R], ps)
    np.testing.assert_array_equal(r.inv_perm.cpu().numpy()[:R], ip)
    codes, quad, s_x, q, sc = tl.oracle_act(X.float().numpy(), 32, ps, cfg.top_k)
    assert qa.x_scale.item() == s_x
    np.testing.assert_array_equal(qa.codes.cpu().numpy()[:R], codes)
    np.testing.assert_array_equal(qa.scales.cpu().numpy(), quad)
    return off, ps, ip, s_x, q, sc


FULL_SIZE = ["30b_up_prefill", "30b_down_decode", "1t_up_prefill", "1t_down_decode_b1", "1t_down_decode_b32",
             "1t_down_decode_b128", "1t_down_decode_b256"]


@pytest.mark.parametrize("name", FULL_SIZE)
def test_gemm_full_size_sampled(gsg, name):
    """The bench's own calls (combined routing + quantization, then the GEMM with the routing's
    row-count hint) at the configuration's full size."""
    cfg = inputs.CONFIGS[name]
    ids = inputs.routing(cfg)
    off_np, _, _ = tl.route_np(ids, cfg.E)
    counts = np.diff(off_np)
    sample_e = _sample_experts(counts)
    pw, canon, sws = _pack_all(gsg, cfg, lambda e: inputs.expert_weight(cfg, e, DEV), sample_e)
    X = inputs.activations(cfg)
    r, qa = gsg.moe_dispatch_nvfp4(ids.to(DEV), X.to(DEV), cfg.E, 32)
    Y = gsg.grouped_sparse_gemm(qa, pw, r.offsets, int(counts.max()), out_dtype=torch.bfloat16)
    Y32 = gsg.grouped_sparse_gemm(qa, pw, r.offsets, int(counts.max()), out_dtype=torch.float32)
    assert gsg.get_device_status() == 0
    off, ps, ip, s_x, q, sc = _check_dispatch(gsg, cfg, ids, X, r, qa)
    rows = _sample_rows(off, sample_e)
    y_ref, bound = tl.reference_rows(rows, off, q, sc, 32, canon, s_x, sws)
    sel = torch.from_numpy(rows).to(DEV)
    tl.assert_gemm_close(Y32[sel], y_ref, bound, f"{name} sampled rows, fp32 output")
    tl.assert_gemm_close(Y[sel], y_ref, bound, f"{name} sampled rows, bf16 output")
    # the bf16 output is the fp32 result rounded once
    assert torch.equal(Y[sel], Y32[sel].to(torch.bfloat16))


def test_gemm_65k_tokens_sampled(gsg):
    """The 1T up-projection at 65,536 tokens top-8 (R = 524,288 routed rows, past the tensor roof's
    ridge point): routing bit for bit over the whole batch, the activation tensor scale, the
    quantized codes and scales of the sampled rows bit for bit, and the GEMM on the sampled rows
    of the sampled experts at the stated bound (bf16 and fp32 outputs).  Output offsets reach
    2^32 bytes here, so 32-bit address arithmetic anywhere on the path would show."""
    from oracle import gemm as ogemm
    from oracle import quant as oquant
    cfg = inputs.CONFIGS["1t_up_prefill_65k"]
    R, K = cfg.R, cfg.K
    ids = inputs.routing(cfg)
    off, ps, ip = tl.route_np(ids, cfg.E)
    counts = np.diff(off)
    sample_e = _sample_experts(counts)
    pw, canon, sws = _pack_all(gsg, cfg, lambda e: inputs.expert_weight(cfg, e, DEV), sample_e)
    X = inputs.activations(cfg)
    r, qa = gsg.moe_dispatch_nvfp4(ids.to(DEV), X.to(DEV), cfg.E, 32)
    Y = gsg.grouped_sparse_gemm(qa, pw, r.offsets, int(counts.max()), out_dtype=torch.bfloat16)
    Y32 = gsg.grouped_sparse_gemm(qa, pw, r.offsets, int(counts.max()), out_dtype=torch.float32)
    assert gsg.get_device_status() == 0
    np.testing.assert_array_equal(r.offsets.cpu().numpy(), off)
    np.testing.assert_array_equal(r.perm_src.cpu().numpy()[:R], ps)
    np.testing.assert_array_equal(r.inv_perm.cpu().numpy()[:R], ip)
    s_x = oquant.act_tensor_scale(X.float().numpy())
    assert qa.x_scale.item() == s_x
    rows = _sample_rows(off, sample_e)
    sel = torch.from_numpy(rows).to(DEV)
    q, sc = oquant.quantize_rows(X[torch.from_numpy(ps[rows] // cfg.top_k)].float().numpy(), 32, s_x)
    np.testing.assert_array_equal(olayout.unpack_act_codes(qa.codes[sel].cpu().numpy()), q)
    q5 = qa.scales.view(K // 128, -1, 4, 4)
    np.testing.assert_array_equal(q5[:, sel, 0, :].cpu().numpy().transpose(1, 0, 2).reshape(rows.size, K // 32), sc)
    # reference rows, expert by expert
    experts = ogemm.expert_of_rows(off, rows)
    y_ref, bound = np.zeros((rows.size, cfg.N)), np.zeros((rows.size, cfg.N))
    for e in np.unique(experts):
        i = np.nonzero(experts == e)[0]
        y_ref[i], bound[i] = ogemm.gemm_rows(oquant.decode_rows(q[i], sc[i], 32),
                                             opack.decode_sparse_expert(*canon[e]), float(s_x) * float(sws[e]))
    tl.assert_gemm_close(Y32[sel], y_ref, bound, "65k tokens sampled rows, fp32 output")
    tl.assert_gemm_close(Y[sel], y_ref, bound, "65k tokens sampled rows, bf16 output")
    assert torch.equal(Y[sel], Y32[sel].to(torch.bfloat16))


@pytest.mark.parametrize("name", ["30b_layer", "1t_layer"])
def test_moe_layer_full_size_sampled(gsg, name):
    """route + quantize -> up-projection with the SwiGLU epilogue -> down-projection -> unpermute
    at the layer's real shapes.  The tensor scale of h is calibrated on the oracle's h of the
    sampled rows.  Checked: routing and X's quantization bit for bit (whole batch); on sampled
    rows, h within one quantization step plus the propagated GEMM bound, and the
    down-projection within the GEMM bound on the GPU's own h; the scatter bit for bit (all
    tokens) on the GPU's own down-projection output."""
    from oracle import codecs as ocodecs
    from oracle import quant as oquant
    from oracle import swiglu as oswiglu
    L = inputs.LAYERS[name]
    up, dn = L.up(), L.down()
    X, ids, g = inputs.activations(up), inputs.routing(up), inputs.gates(up)
    off_np, _, _ = tl.route_np(ids, L.E)
    counts = np.diff(off_np)
    sample_e = _sample_experts(counts)
    wu, cu, swu = _pack_all(gsg, up, lambda e: inputs.expert_weight(up, e, DEV), sample_e)
    wd, cd, swd = _pack_all(gsg, dn, lambda e: inputs.down_weight(L, e, DEV), sample_e)
    R = L.R
    # the oracle's up-projection and h on the sampled rows, and the calibrated tensor scale of h
    codes_o, quad_o, s_x, q, sc = tl.oracle_act(X.float().numpy(), 32, tl.route_np(ids, L.E)[1], L.top_k)
    rows = _sample_rows(off_np, sample_e)
    y_up, b_up = tl.reference_rows(rows, off_np, q, sc, 32, cu, s_x, swu)
    h_ref = oswiglu.swiglu_rows(y_up)
    s_h = np.float32(np.abs(h_ref).max() / 2688.0)
    # the GPU layer
    r, qa = gsg.moe_dispatch_nvfp4(ids.to(DEV), X.to(DEV), L.E, 32)
    hq = gsg.grouped_sparse_gemm_swiglu(qa, wu, r.offsets, torch.tensor([s_h], device=DEV), int(counts.max()))
    Y2 = gsg.grouped_sparse_gemm(hq, wd, r.offsets, int(counts.max()))
    out = gsg.unpermute_scale(Y2, r.inv_perm, g.to(DEV), L.top_k)
    assert gsg.get_device_status() == 0
    off, ps, ip, s_x2, _, _ = _check_dispatch(gsg, up, ids, X, r, qa)
    assert s_x2 == s_x
    # h on the sampled rows
    hc = olayout.unpack_act_codes(hq.codes.cpu().numpy()[:R])
    q5 = hq.scales.cpu().numpy().reshape(L.I // 128, R + olayout.ACT_SCALE_PAD_ROWS, 4, 4)
    hs = q5[:, :R, 0, :].transpose(1, 0, 2).reshape(R, L.I // 32)
    hd = oquant.decode_rows(hc[rows], hs[rows], 32) * float(s_h)
    bound_h = (np.repeat(ocodecs.ue4m3_decode(hs[rows]).astype(np.float64) * float(s_h), 32, axis=1) +
               oswiglu.swiglu_error_bound(y_up, 2.0 ** -10 * b_up + 1e-6) + 2.0 ** -16 * np.abs(h_ref))
    err = np.abs(hd - h_ref)
    assert np.all(err <= bound_h), float(np.max(err / bound_h))
    # the down-projection on the GPU's h, sampled rows
    y_dn, b_dn = tl.reference_rows(rows, off, hc, hs, 32, cd, s_h, swd)
    tl.assert_gemm_close(Y2[torch.from_numpy(rows).to(DEV)], y_dn, b_dn, f"{name} down-projection")
    # the scatter of the GPU's down-projection output, every token
    ref = ounperm.unpermute_scale(Y2.cpu().view(torch.uint16).numpy(), ip, g.numpy(), L.top_k)
    np.testing.assert_array_equal(out.cpu().view(torch.uint16).numpy(), ref)
