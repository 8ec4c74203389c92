"""gsg_moe_route_permute_noalloc (routing with the library's fixed scratch, for callers that may
not allocate device memory) against gsg_moe_route_permute (caller-supplied workspace).

Both calls go through the C ABI.  The GPU test routes two different problems in a row that both
need the scratch (more than one routing chunk), so the second call runs on the first one's
leftover scratch contents; routing is integer work, so outputs must match bit for bit.  This file
is collected last so that it runs both after the other tests and, alone, in a fresh process
where its first call does the per-device set-up.
"""
import ctypes

import pytest
import torch

import grouped_sparse_gemm_b200 as gsg

P = ctypes.c_void_p(16)   # non-NULL placeholder, never dereferenced by the host-side checks


def _p(t):
    return ctypes.c_void_p(t.data_ptr())


def test_noalloc_rejects_sizes_beyond_the_scratch():
    from grouped_sparse_gemm_b200 import _build
    _build.build()
    L = gsg.load_library()
    # R = 2^20 rows over E = 384 experts: 128 chunks * 384 > 32768 -> unsupported, nothing launched
    assert L.gsg_moe_route_permute_noalloc(P, 1 << 17, 8, 384, P, P, P, None) == -2
    assert L.gsg_moe_route_permute_noalloc(P, -1, 8, 384, P, P, P, None) == -1
    assert L.gsg_moe_route_permute_noalloc(P, 4, 2, 5000, P, P, P, None) == -2


def _route_with_workspace(L, ids, E, stream):
    T, k = ids.shape
    R = T * k
    off = torch.empty(E + 1, dtype=torch.int32, device="cuda")
    ps = torch.empty(R, dtype=torch.int32, device="cuda")
    ip = torch.empty(R, dtype=torch.int32, device="cuda")
    need = L.gsg_workspace_size(gsg.OP_ROUTE, E, 0, 0, T, k)
    assert need > 0
    ws = torch.empty(need, dtype=torch.uint8, device="cuda")
    assert L.gsg_moe_route_permute(_p(ids), T, k, E, _p(off), _p(ps), _p(ip), _p(ws), need, stream) == 0
    return off, ps, ip


def _route_noalloc(L, ids, E, stream):
    T, k = ids.shape
    R = T * k
    off = torch.full((E + 1,), -7, dtype=torch.int32, device="cuda")
    ps = torch.full((R,), -7, dtype=torch.int32, device="cuda")
    ip = torch.full((R,), -7, dtype=torch.int32, device="cuda")
    assert L.gsg_moe_route_permute_noalloc(_p(ids), T, k, E, _p(off), _p(ps), _p(ip), stream) == 0
    return off, ps, ip


@pytest.mark.gpu
def test_noalloc_matches_workspace_routing_twice_in_a_row():
    L = gsg.load_library()
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    g = torch.Generator().manual_seed(77)
    cases = [(8192, 8, 384), (3000, 7, 128)]     # R = 65536 (8 chunks of 8192), R = 21000 (21 of 1024)
    inputs = [torch.randint(0, E, (T, k), generator=g, dtype=torch.int32).cuda() for T, k, E in cases]
    got = [_route_noalloc(L, ids, E, stream) for ids, (_, _, E) in zip(inputs, cases)]
    want = [_route_with_workspace(L, ids, E, stream) for ids, (_, _, E) in zip(inputs, cases)]
    torch.cuda.synchronize()
    assert L.gsg_get_device_status(stream) == 0
    for (T, k, E), a, b in zip(cases, got, want):
        for x, y in zip(a, b):
            assert torch.equal(x, y), (T, k, E)
        assert int(a[0][E]) == T * k
