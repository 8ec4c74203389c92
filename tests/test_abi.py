"""The C ABI library loads, exports every declared symbol and rejects bad arguments on the host
(no GPU needed: every check here returns before any CUDA call)."""
import ctypes
import os
import re

import pytest

import grouped_sparse_gemm_b200 as gsg

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def L():
    from grouped_sparse_gemm_b200 import _build
    _build.build()
    return gsg.load_library()


def declared_symbols():
    with open(os.path.join(ROOT, "include", "gsg.h")) as f:
        text = f.read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(gsg_[a-z0-9_]+)\s*\(", text)))


def test_every_declared_symbol_is_exported(L):
    decl = declared_symbols()
    assert len(decl) >= 15
    for name in decl:
        assert hasattr(L, name), name
    assert sorted(decl) == sorted(gsg.EXPORTED_SYMBOLS)


def test_sizes(L):
    E, N, K = 3, 256, 512
    assert L.gsg_sparse_packed_bytes(E, N, K) * 8 == 2.75 * E * N * K     # 2.75 bit per weight
    assert L.gsg_dense_packed_bytes(E, N, K) * 8 == 4.5 * E * N * K
    assert L.gsg_act_codes_bytes(10, 256) == 1280
    assert L.gsg_act_scales_bytes(10, 256, 32) == 2 * (10 + 256) * 16
    assert L.gsg_workspace_size(gsg.OP_ROUTE, 384, 0, 0, 64, 8) == 0          # single-launch routing
    assert L.gsg_workspace_size(gsg.OP_ROUTE, 384, 0, 0, 8192, 8) == 2 * 8 * 384 * 4   # 8192-row chunks
    assert L.gsg_workspace_size(gsg.OP_ROUTE, 128, 0, 0, 256, 8) == 0             # one block up to 2048 rows
    assert L.gsg_workspace_size(gsg.OP_ROUTE, 128, 0, 0, 512, 8) == 2 * 4 * 128 * 4    # 1024-row chunks
    assert L.gsg_workspace_size(gsg.OP_ROUTE, 128, 0, 0, 2000, 8) == 2 * 16 * 128 * 4  # 1024-row chunks
    assert L.gsg_workspace_size(gsg.OP_GEMM, 384, 4096, 7168, 8192, 8) == 0
    # routing workspace (4 chunks x 128 experts x 2 int32) + one float per amax block, each 256-byte rounded
    assert L.gsg_workspace_size(gsg.OP_DISPATCH, 128, 0, 2048, 512, 8) == 4096 + 256
    assert L.gsg_workspace_size(gsg.OP_DISPATCH, 128, 0, 768, 64, 8) == 256        # one routing block
    # from R*K = 2^27 the quantizer stages its scale words row-major: R * K/128 words after the partials
    raw = 65536 * (7168 // 128) * 4
    assert L.gsg_workspace_size(gsg.OP_QUANTIZE, 0, 0, 7168, 8192, 8) == 512 * 4 + raw
    assert L.gsg_workspace_size(gsg.OP_DISPATCH, 384, 0, 7168, 8192, 8) == 2 * 8 * 384 * 4 + 1024 + raw
    assert L.gsg_workspace_size(gsg.OP_QUANTIZE, 0, 0, 2048, 512, 8) == 128 * 4     # partials only


def test_status_strings(L):
    for s in (0, -1, -2, -3, -4, -5, -6, -7, 42):
        assert L.gsg_status_string(s)


P = ctypes.c_void_p(16)   # a non-NULL, 16-byte aligned placeholder never dereferenced by the checks below


def test_host_argument_checks(L):
    # bad shapes (K % 256, N % 128) -> unsupported shape, no launch
    assert L.gsg_pack_sparse_nvfp4(P, 1, 128, 100, P, P, P, 1 << 20, None) == -2
    assert L.gsg_pack_sparse_nvfp4(P, 1, 100, 256, P, P, P, 1 << 20, None) == -2
    assert L.gsg_pack_sparse_nvfp4(None, 1, 128, 256, P, P, P, 1 << 20, None) == -1
    assert L.gsg_pack_sparse_nvfp4(P, 1, 128, 256, P, P, None, 0, None) == -7
    assert L.gsg_grouped_sparse_gemm(P, P, P, P, P, P, 4, 128, 300, 8, -1, P, 0, None) == -2
    assert L.gsg_grouped_sparse_gemm(P, P, P, P, P, P, 4, 128, 256, 8, -1, P, 7, None) == -1
    assert L.gsg_grouped_sparse_gemm(P, P, P, P, P, P, 2000, 128, 256, 8, -1, P, 0, None) == -2
    assert L.gsg_grouped_sparse_gemm(P, P, P, None, P, P, 4, 128, 256, 8, -1, P, 0, None) == -1
    assert L.gsg_grouped_sparse_gemm(P, P, P, P, P, P, 4, 128, 256, 0, -1, P, 0, None) == 0  # R = 0
    assert L.gsg_moe_route_permute(P, 4, 2, 0, P, P, P, None, 0, None) == -2
    assert L.gsg_moe_route_permute(P, 4, 2, 5000, P, P, P, None, 0, None) == -2
    assert L.gsg_moe_route_permute(P, 8192, 8, 16, P, P, P, None, 0, None) == -7
    assert L.gsg_quantize_act_nvfp4(P, 4, 256, 24, P, 2, None, P, P, P, P, 1 << 20, None) == -1
    assert L.gsg_quantize_act_nvfp4(P, 4, 256, 32, None, 2, None, P, P, P, P, 1 << 20, None) == -1
    assert L.gsg_quantize_act_nvfp4(P, 4, 200, 32, P, 2, None, P, P, P, P, 1 << 20, None) == -2
    assert L.gsg_quantize_act_nvfp4(P, 4, 256, 32, P, 2, None, P, P, P, None, 0, None) == -7
    assert L.gsg_unpermute_scale(P, P, P, 4, 2, 12, P, None) == -1
    assert L.gsg_unpermute_scale(P, P, P, 0, 2, 128, P, None) == 0
    # the GEMM with the combine: bad k, bad N, too many token sums for a 32-bit index, NULL gates
    assert L.gsg_grouped_sparse_gemm_combine(P, P, P, P, P, P, 4, 256, 256, 8, 0, -1, P, P, P, 1 << 20, P, None) == -1
    assert L.gsg_grouped_sparse_gemm_combine(P, P, P, P, P, P, 4, 200, 256, 8, 2, -1, P, P, P, 1 << 20, P, None) == -2
    assert L.gsg_grouped_sparse_gemm_combine(P, P, P, P, P, P, 4, 32768, 256, 1 << 20, 1, -1, P, P, P, 1 << 20, P,
                                             None) == -2
    assert L.gsg_grouped_sparse_gemm_combine(P, P, P, P, P, P, 4, 256, 256, 8, 2, -1, P, None, P, 1 << 20, P, None) == -1
    # two-phase scale path (R*K >= 2^27): its workspace is needed even with a caller-supplied s_x
    assert L.gsg_quantize_act_nvfp4(P, 2048, 8192, 32, P, 8, P, P, P, P, None, 0, None) == -7
    # the combined routing + quantize call: the checks of both calls, and its own workspace
    ws_need = L.gsg_workspace_size(gsg.OP_DISPATCH, 16, 0, 256, 4, 2)
    assert L.gsg_moe_dispatch_nvfp4(P, P, 4, 2, 16, 256, 24, None, P, P, P, P, P, P, P, 1 << 20, None) == -1
    assert L.gsg_moe_dispatch_nvfp4(P, P, 4, 2, 0, 256, 32, None, P, P, P, P, P, P, P, 1 << 20, None) == -2
    assert L.gsg_moe_dispatch_nvfp4(P, P, 4, 2, 16, 200, 32, None, P, P, P, P, P, P, P, 1 << 20, None) == -2
    assert L.gsg_moe_dispatch_nvfp4(P, None, 4, 2, 16, 256, 32, None, P, P, P, P, P, P, P, 1 << 20, None) == -1
    assert L.gsg_moe_dispatch_nvfp4(P, P, 4, 2, 16, 256, 32, None, P, P, P, P, P, P, None, 0, None) == -7
    assert L.gsg_moe_dispatch_nvfp4(P, P, 4, 2, 16, 256, 32, None, P, P, P, P, P, P, P, ws_need - 1, None) == -7
    assert L.gsg_moe_dispatch_nvfp4(P, P, 4, 2, 16, 256, 32, None, P, P, P, P, P, P, ctypes.c_void_p(20), 1 << 20, None) == -7


def test_binding_refuses_cpu_tensors():
    import torch
    with pytest.raises(ValueError):
        gsg.quantize_act_nvfp4(torch.zeros(4, 256, dtype=torch.bfloat16))
