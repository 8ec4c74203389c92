"""grouped_sparse_gemm_b200 -- grouped paired-4:8 NVFP4 expert GEMM for routed MoE on B200.

Thin Python binding over the C ABI of ``libgsg.so`` (declared in ``include/gsg.h``).  The
functions keep the ABI's names without the ``gsg_`` prefix and only marshal arguments: torch
provides device memory and the current stream, every step runs in the library's CUDA kernels.
There is no CPU fallback: if the library is missing or no GPU is present the calls raise.

The path (after "Hardware-Native Joint Sparse-Quantization for Trillion-Scale Mixture-of-Experts",
paperlayer.ai summary, §3.4 and §D.1): pack_sparse_nvfp4 (offline weights) ->
moe_route_permute -> quantize_act_nvfp4 -> grouped_sparse_gemm -> unpermute_scale
(moe_dispatch_nvfp4 = the routing and quantizer calls in one).  save_packed / load_packed keep
packed weights in a file: the packed format is the storage format.
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass
from typing import Optional

import torch

from . import _build

__all__ = [
    "GsgError", "lib", "load_library", "library_path",
    "PackedSparseWeights", "PackedDenseWeights", "Routing", "QuantizedActivations",
    "pack_sparse_nvfp4", "pack_dense_nvfp4", "moe_route_permute", "moe_route_permute_noalloc",
    "quantize_act_nvfp4", "moe_dispatch_nvfp4",
    "grouped_sparse_gemm", "grouped_sparse_gemm_swiglu", "grouped_sparse_gemm_combine", "combine_workspace",
    "grouped_dense_gemm", "grouped_dense_gemm_native", "unpermute_scale", "OP_COMBINE", "OP_DISPATCH",
    "get_device_status",
    "save_packed", "load_packed",
    "act_scales_bytes", "workspace_size", "OP_PACK_SPARSE", "OP_PACK_DENSE", "OP_ROUTE",
    "OP_QUANTIZE", "OP_GEMM", "EXPORTED_SYMBOLS",
]

OP_PACK_SPARSE, OP_PACK_DENSE, OP_ROUTE, OP_QUANTIZE, OP_GEMM, OP_COMBINE, OP_DISPATCH = 1, 2, 3, 4, 5, 6, 7
OUT_BF16, OUT_F32 = 0, 1
ACT_SCALE_PAD_ROWS = 256

EXPORTED_SYMBOLS = [
    "gsg_sparse_packed_bytes", "gsg_dense_packed_bytes", "gsg_act_codes_bytes", "gsg_act_scales_bytes",
    "gsg_workspace_size",
    "gsg_pack_sparse_nvfp4", "gsg_pack_dense_nvfp4", "gsg_moe_route_permute",
    "gsg_quantize_act_nvfp4", "gsg_grouped_sparse_gemm", "gsg_grouped_dense_gemm",
    "gsg_unpermute_scale", "gsg_get_device_status", "gsg_status_string", "gsg_version",
    "gsg_moe_route_permute_noalloc", "gsg_grouped_sparse_gemm_swiglu", "gsg_grouped_sparse_gemm_combine",
    "gsg_moe_dispatch_nvfp4", "gsg_test_set_gemm_stall_ns", "gsg_grouped_dense_gemm_native",
    "gsg_test_set_gemm_table_cap",
]

_STATUS = {0: "ok", -1: "invalid argument", -2: "unsupported shape", -3: "CUDA error",
           -4: "bad routing", -5: "non-finite input", -6: "device timeout", -7: "workspace"}


class GsgError(RuntimeError):
    def __init__(self, fn: str, status: int):
        super().__init__(f"{fn} failed: {_STATUS.get(status, status)} ({status})")
        self.status = status


_lib: Optional[ctypes.CDLL] = None


def library_path() -> str:
    return _build.LIB


def load_library(build_if_missing: bool = False) -> ctypes.CDLL:
    """Load libgsg.so (optionally compiling it first).  Raises when it is not there."""
    global _lib
    if _lib is not None:
        return _lib
    path = library_path()
    if not os.path.exists(path):
        if not build_if_missing:
            raise RuntimeError(f"libgsg.so is not built ({path}); run grouped_sparse_gemm_b200._build.build()")
        _build.build()
    L = ctypes.CDLL(path)
    vp, i, sz, fp = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t, ctypes.c_void_p
    sig = {
        "gsg_sparse_packed_bytes": (sz, [i, i, i]),
        "gsg_dense_packed_bytes": (sz, [i, i, i]),
        "gsg_act_codes_bytes": (sz, [i, i]),
        "gsg_act_scales_bytes": (sz, [i, i, i]),
        "gsg_workspace_size": (sz, [i, i, i, i, i, i]),
        "gsg_pack_sparse_nvfp4": (i, [vp, i, i, i, vp, fp, vp, sz, vp]),
        "gsg_pack_dense_nvfp4": (i, [vp, i, i, i, vp, fp, vp, sz, vp]),
        "gsg_moe_route_permute": (i, [vp, i, i, i, vp, vp, vp, vp, sz, vp]),
        "gsg_quantize_act_nvfp4": (i, [vp, i, i, i, vp, i, vp, vp, vp, vp, vp, sz, vp]),
        "gsg_moe_dispatch_nvfp4": (i, [vp, vp, i, i, i, i, i, vp, vp, vp, vp, vp, vp, vp, vp, sz, vp]),
        "gsg_grouped_sparse_gemm": (i, [vp, vp, vp, vp, vp, vp, i, i, i, i, i, vp, i, vp]),
        "gsg_grouped_dense_gemm": (i, [vp, vp, vp, vp, vp, vp, i, i, i, i, i, vp, i, vp]),
        "gsg_grouped_dense_gemm_native": (i, [vp, vp, vp, vp, vp, vp, i, i, i, i, i, vp, i, vp]),
        "gsg_unpermute_scale": (i, [vp, vp, vp, i, i, i, vp, vp]),
        "gsg_get_device_status": (i, [vp]),
        "gsg_status_string": (ctypes.c_char_p, [i]),
        "gsg_version": (i, []),
        "gsg_moe_route_permute_noalloc": (i, [vp, i, i, i, vp, vp, vp, vp]),
        "gsg_grouped_sparse_gemm_swiglu": (i, [vp, vp, vp, vp, vp, vp, i, i, i, i, i, vp, vp, vp, vp]),
        "gsg_grouped_sparse_gemm_combine": (i, [vp, vp, vp, vp, vp, vp, i, i, i, i, i, i, vp, vp, vp, sz, vp, vp]),
        "gsg_test_set_gemm_stall_ns": (None, [ctypes.c_ulonglong]),
        "gsg_test_set_gemm_table_cap": (None, [ctypes.c_int]),
    }
    for name, (res, args) in sig.items():
        f = getattr(L, name)
        f.restype = res
        f.argtypes = args
    _lib = L
    return L


def lib() -> ctypes.CDLL:
    return load_library()


# ------------------------------------------------------------------ helpers
def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream: Optional[torch.cuda.Stream] = None):
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def _check(fn: str, st: int):
    if st != 0:
        raise GsgError(fn, st)


def _need_cuda(*ts: Optional[torch.Tensor]):
    for t in ts:
        if t is None:
            continue
        if not t.is_cuda:
            raise ValueError("grouped_sparse_gemm_b200 works on CUDA tensors only (no CPU fallback)")
        if not t.is_contiguous():
            raise ValueError("tensors must be contiguous")


def workspace_size(op: int, E: int = 0, N: int = 0, K: int = 0, T: int = 0, k: int = 1) -> int:
    return int(lib().gsg_workspace_size(op, E, N, K, T, k))


def act_scales_bytes(R: int, K: int, sf_block: int) -> int:
    return int(lib().gsg_act_scales_bytes(R, K, sf_block))


def _workspace(nbytes: int, device) -> torch.Tensor:
    return torch.empty(max(int(nbytes), 16), dtype=torch.uint8, device=device)


# ------------------------------------------------------------------ packed containers
SPARSE_CHUNK_BYTES = 11264     # one (expert, n-tile, 256-wide K chunk) block: values | metadata | scales
DENSE_CHUNK_BYTES = 18432


@dataclass
class PackedSparseWeights:
    packed: torch.Tensor   # uint8 [E*N*K*11/32], chunk blocks (see include/gsg.h)
    w_scale: torch.Tensor  # fp32 [E]
    E: int
    N: int
    K: int

    def nbytes(self) -> int:
        return self.packed.numel()

    def expert(self, e: int) -> "PackedSparseWeights":
        """View of expert e alone (E = 1)."""
        n = self.packed.numel() // self.E
        return PackedSparseWeights(self.packed[e * n:(e + 1) * n], self.w_scale[e:e + 1], 1, self.N, self.K)


@dataclass
class PackedDenseWeights:
    packed: torch.Tensor   # uint8 [E*N*K*9/16]
    w_scale: torch.Tensor  # fp32 [E]
    E: int
    N: int
    K: int

    def nbytes(self) -> int:
        return self.packed.numel()

    def expert(self, e: int) -> "PackedDenseWeights":
        n = self.packed.numel() // self.E
        return PackedDenseWeights(self.packed[e * n:(e + 1) * n], self.w_scale[e:e + 1], 1, self.N, self.K)


@dataclass
class Routing:
    offsets: torch.Tensor   # int32 [E+1]
    perm_src: torch.Tensor  # int32 [R]
    inv_perm: torch.Tensor  # int32 [R]
    T: int
    k: int
    E: int


@dataclass
class QuantizedActivations:
    codes: torch.Tensor     # uint8 [R, K/2]
    scales: torch.Tensor    # uint8, quad layout
    x_scale: torch.Tensor   # fp32 [1]
    R: int
    K: int
    sf_block: int


# ------------------------------------------------------------------ storage
PACKED_FILE_VERSION = 1


def save_packed(w, path: str) -> None:
    """Packed weights (PackedSparseWeights or PackedDenseWeights, any device) to an .npz file: the
    packed bytes exactly as the GEMM reads them, the per-expert FP32 tensor scales, E, N, K and
    the format.  No re-encoding: load_packed gives back the same bytes."""
    import numpy as np
    fmt = "sparse" if isinstance(w, PackedSparseWeights) else "dense"
    np.savez(path, version=PACKED_FILE_VERSION, format=fmt, E=w.E, N=w.N, K=w.K,
             packed=w.packed.detach().cpu().numpy(), w_scale=w.w_scale.detach().cpu().numpy())


def load_packed(path: str, device=None):
    """Packed weights from a save_packed file, on `device` (default: CPU).  Checks the version,
    the format and that the byte count is the library's size for (E, N, K); raises ValueError
    otherwise."""
    import numpy as np
    with np.load(path, allow_pickle=False) as d:
        if int(d["version"]) != PACKED_FILE_VERSION:
            raise ValueError(f"{path}: packed-weights file version {int(d['version'])}, expected "
                             f"{PACKED_FILE_VERSION}")
        fmt = str(d["format"])
        E, N, K = int(d["E"]), int(d["N"]), int(d["K"])
        packed, w_scale = d["packed"], d["w_scale"]
    if fmt not in ("sparse", "dense"):
        raise ValueError(f"{path}: unknown packed format {fmt!r}")
    # the shape rule of the packers (whole 128-row n-tiles, whole 256-wide K chunks, int range),
    # checked before the byte count so that a wrong N or K of the right size is still rejected
    int_max = 2 ** 31 - 1
    if not (1 <= E <= int_max and 128 <= N <= int_max and 256 <= K <= int_max and N % 128 == 0
            and K % 256 == 0):
        raise ValueError(f"{path}: E={E} N={N} K={K} is not a packed shape (E >= 1, N a multiple of 128, "
                         f"K a multiple of 256)")
    L = lib()
    need = L.gsg_sparse_packed_bytes(E, N, K) if fmt == "sparse" else L.gsg_dense_packed_bytes(E, N, K)
    if packed.dtype != np.uint8 or packed.ndim != 1 or packed.size != need:
        raise ValueError(f"{path}: {packed.size} packed bytes, expected {need} for {fmt} E={E} N={N} K={K}")
    if w_scale.dtype != np.float32 or w_scale.shape != (E,):
        raise ValueError(f"{path}: tensor scales of shape {w_scale.shape} / {w_scale.dtype}, expected ({E},) float32")
    pk = torch.from_numpy(packed.copy()).to(device or "cpu")
    ws = torch.from_numpy(w_scale.copy()).to(device or "cpu")
    cls = PackedSparseWeights if fmt == "sparse" else PackedDenseWeights
    return cls(packed=pk, w_scale=ws, E=E, N=N, K=K)


# ------------------------------------------------------------------ entry points
def pack_sparse_nvfp4(W: torch.Tensor, out: Optional[PackedSparseWeights] = None,
                      workspace: Optional[torch.Tensor] = None, stream=None) -> PackedSparseWeights:
    """W fp32 [E, N, K] -> paired 4:8 NVFP4 packed weights (gsg_pack_sparse_nvfp4)."""
    _need_cuda(W)
    assert W.dtype == torch.float32 and W.dim() == 3
    E, N, K = W.shape
    L = lib()
    dev = W.device
    if out is None:
        out = PackedSparseWeights(
            packed=torch.empty(L.gsg_sparse_packed_bytes(E, N, K), dtype=torch.uint8, device=dev),
            w_scale=torch.empty(E, dtype=torch.float32, device=dev), E=E, N=N, K=K)
    need = workspace_size(OP_PACK_SPARSE, E, N, K)
    ws = workspace if workspace is not None else _workspace(need, dev)
    _check("gsg_pack_sparse_nvfp4", L.gsg_pack_sparse_nvfp4(
        _ptr(W), E, N, K, _ptr(out.packed), _ptr(out.w_scale), _ptr(ws), ws.numel(), _stream(stream)))
    return out


def pack_dense_nvfp4(W: torch.Tensor, out: Optional[PackedDenseWeights] = None,
                     workspace: Optional[torch.Tensor] = None, stream=None) -> PackedDenseWeights:
    """W fp32 [E, N, K] -> dense NVFP4 (16-element blocks) for the control GEMM."""
    _need_cuda(W)
    assert W.dtype == torch.float32 and W.dim() == 3
    E, N, K = W.shape
    L = lib()
    dev = W.device
    if out is None:
        out = PackedDenseWeights(
            packed=torch.empty(L.gsg_dense_packed_bytes(E, N, K), dtype=torch.uint8, device=dev),
            w_scale=torch.empty(E, dtype=torch.float32, device=dev), E=E, N=N, K=K)
    need = workspace_size(OP_PACK_DENSE, E, N, K)
    ws = workspace if workspace is not None else _workspace(need, dev)
    _check("gsg_pack_dense_nvfp4", L.gsg_pack_dense_nvfp4(
        _ptr(W), E, N, K, _ptr(out.packed), _ptr(out.w_scale), _ptr(ws), ws.numel(), _stream(stream)))
    return out


def moe_route_permute(topk_ids: torch.Tensor, E: int, out: Optional[Routing] = None,
                      workspace: Optional[torch.Tensor] = None, stream=None) -> Routing:
    """topk ids int32 [T, k] -> expert offsets, perm_src, inv_perm (gsg_moe_route_permute)."""
    _need_cuda(topk_ids)
    assert topk_ids.dtype == torch.int32 and topk_ids.dim() == 2
    T, k = topk_ids.shape
    dev = topk_ids.device
    if out is None:
        out = Routing(offsets=torch.empty(E + 1, dtype=torch.int32, device=dev),
                      perm_src=torch.empty(max(T * k, 1), dtype=torch.int32, device=dev),
                      inv_perm=torch.empty(max(T * k, 1), dtype=torch.int32, device=dev), T=T, k=k, E=E)
    ws = workspace
    if ws is None:   # the size query only when the call has to allocate
        need = workspace_size(OP_ROUTE, E, 0, 0, T, k)
        ws = _workspace(need, dev) if need else None
    _check("gsg_moe_route_permute", lib().gsg_moe_route_permute(
        _ptr(topk_ids), T, k, E, _ptr(out.offsets), _ptr(out.perm_src), _ptr(out.inv_perm),
        _ptr(ws), 0 if ws is None else ws.numel(), _stream(stream)))
    return out


def moe_route_permute_noalloc(topk_ids: torch.Tensor, E: int, out: Routing, stream=None) -> Routing:
    """gsg_moe_route_permute_noalloc: the same routing with the library's fixed scratch instead of
    a workspace, for callers that may not allocate device memory at this point (outputs in `out`
    are caller-allocated; nothing is allocated here)."""
    _need_cuda(topk_ids, out.offsets, out.perm_src, out.inv_perm)
    assert topk_ids.dtype == torch.int32 and topk_ids.dim() == 2
    T, k = topk_ids.shape
    _check("gsg_moe_route_permute_noalloc", lib().gsg_moe_route_permute_noalloc(
        _ptr(topk_ids), T, k, E, _ptr(out.offsets), _ptr(out.perm_src), _ptr(out.inv_perm), _stream(stream)))
    return out


def quantize_act_nvfp4(X: torch.Tensor, sf_block: int = 32, inv_perm: Optional[torch.Tensor] = None,
                       top_k: int = 1, x_scale_in: Optional[torch.Tensor] = None,
                       out: Optional[QuantizedActivations] = None,
                       workspace: Optional[torch.Tensor] = None, stream=None) -> QuantizedActivations:
    """X bf16 [T, K] -> NVFP4 codes/scales in routed row order (gsg_quantize_act_nvfp4)."""
    _need_cuda(X, inv_perm, x_scale_in)
    assert X.dtype == torch.bfloat16 and X.dim() == 2
    T, K = X.shape
    R = T * top_k
    dev = X.device
    if out is None:
        out = QuantizedActivations(
            codes=torch.empty(max(R, 1), K // 2, dtype=torch.uint8, device=dev),
            scales=torch.empty(act_scales_bytes(R, K, sf_block), dtype=torch.uint8, device=dev),
            x_scale=torch.empty(1, dtype=torch.float32, device=dev), R=R, K=K, sf_block=sf_block)
    ws = workspace if workspace is not None else _workspace(workspace_size(OP_QUANTIZE, 0, 0, K, T, top_k), dev)
    _check("gsg_quantize_act_nvfp4", lib().gsg_quantize_act_nvfp4(
        _ptr(X), T, K, sf_block, _ptr(inv_perm), top_k, _ptr(x_scale_in), _ptr(out.codes),
        _ptr(out.scales), _ptr(out.x_scale), _ptr(ws), ws.numel(), _stream(stream)))
    return out


def moe_dispatch_nvfp4(topk_ids: torch.Tensor, X: torch.Tensor, E: int, sf_block: int = 32,
                       x_scale_in: Optional[torch.Tensor] = None, out_route: Optional[Routing] = None,
                       out_act: Optional[QuantizedActivations] = None, workspace: Optional[torch.Tensor] = None,
                       stream=None):
    """moe_route_permute + quantize_act_nvfp4 in one call (gsg_moe_dispatch_nvfp4): the same
    outputs bit for bit, one launch fewer.  Returns (Routing, QuantizedActivations)."""
    _need_cuda(topk_ids, X, x_scale_in)
    assert topk_ids.dtype == torch.int32 and topk_ids.dim() == 2
    assert X.dtype == torch.bfloat16 and X.dim() == 2 and X.shape[0] == topk_ids.shape[0]
    T, k = topk_ids.shape
    K = X.shape[1]
    R = T * k
    dev = X.device
    if out_route is None:
        out_route = Routing(offsets=torch.empty(E + 1, dtype=torch.int32, device=dev),
                            perm_src=torch.empty(max(R, 1), dtype=torch.int32, device=dev),
                            inv_perm=torch.empty(max(R, 1), dtype=torch.int32, device=dev), T=T, k=k, E=E)
    if out_act is None:
        out_act = QuantizedActivations(
            codes=torch.empty(max(R, 1), K // 2, dtype=torch.uint8, device=dev),
            scales=torch.empty(act_scales_bytes(R, K, sf_block), dtype=torch.uint8, device=dev),
            x_scale=torch.empty(1, dtype=torch.float32, device=dev), R=R, K=K, sf_block=sf_block)
    ws = workspace if workspace is not None else _workspace(workspace_size(OP_DISPATCH, E, 0, K, T, k), dev)
    _check("gsg_moe_dispatch_nvfp4", lib().gsg_moe_dispatch_nvfp4(
        _ptr(topk_ids), _ptr(X), T, k, E, K, sf_block, _ptr(x_scale_in), _ptr(out_route.offsets),
        _ptr(out_route.perm_src), _ptr(out_route.inv_perm), _ptr(out_act.codes), _ptr(out_act.scales),
        _ptr(out_act.x_scale), _ptr(ws), ws.numel(), _stream(stream)))
    return out_route, out_act


def grouped_sparse_gemm(act: QuantizedActivations, w: PackedSparseWeights, offsets: torch.Tensor,
                        max_rows_per_expert: int = -1, out: Optional[torch.Tensor] = None,
                        out_dtype: torch.dtype = torch.bfloat16, stream=None) -> torch.Tensor:
    """Y [R, N] = per-expert X_e . W_e^T on paired 4:8 NVFP4 weights (gsg_grouped_sparse_gemm)."""
    assert act.sf_block == 32 and act.K == w.K
    _need_cuda(act.codes, act.scales, offsets)
    if out is None:
        out = torch.empty(max(act.R, 1), w.N, dtype=out_dtype, device=act.codes.device)
    ydt = OUT_F32 if out.dtype == torch.float32 else OUT_BF16
    _check("gsg_grouped_sparse_gemm", lib().gsg_grouped_sparse_gemm(
        _ptr(act.codes), _ptr(act.scales), _ptr(act.x_scale), _ptr(w.packed), _ptr(w.w_scale),
        _ptr(offsets), w.E, w.N, w.K, act.R, max_rows_per_expert, _ptr(out), ydt, _stream(stream)))
    return out


def grouped_sparse_gemm_swiglu(act: QuantizedActivations, w: PackedSparseWeights, offsets: torch.Tensor,
                               h_scale: torch.Tensor, max_rows_per_expert: int = -1,
                               out: Optional[QuantizedActivations] = None, stream=None) -> QuantizedActivations:
    """Up-projection (fused gate|up weights [2I, K]) with SwiGLU and NVFP4 quantization of
    h = silu(gate) * up in the epilogue (gsg_grouped_sparse_gemm_swiglu): returns h's codes and
    scales, ready as the down-projection's activations (tensor scale h_scale, fp32 [1])."""
    assert act.sf_block == 32 and act.K == w.K and w.N % 256 == 0
    _need_cuda(act.codes, act.scales, offsets, h_scale)
    I = w.N // 2
    dev = act.codes.device
    if out is None:
        out = QuantizedActivations(codes=torch.empty(max(act.R, 1), I // 2, dtype=torch.uint8, device=dev),
                                   scales=torch.empty(act_scales_bytes(act.R, I, 32), dtype=torch.uint8, device=dev),
                                   x_scale=h_scale, R=act.R, K=I, sf_block=32)
    _check("gsg_grouped_sparse_gemm_swiglu", lib().gsg_grouped_sparse_gemm_swiglu(
        _ptr(act.codes), _ptr(act.scales), _ptr(act.x_scale), _ptr(w.packed), _ptr(w.w_scale),
        _ptr(offsets), w.E, w.N, w.K, act.R, max_rows_per_expert, _ptr(h_scale), _ptr(out.codes),
        _ptr(out.scales), _stream(stream)))
    return out


def combine_workspace(E: int, N: int, K: int, T: int, k: int, device) -> torch.Tensor:
    """A zeroed workspace for grouped_sparse_gemm_combine (reusable call after call)."""
    return torch.zeros(max(workspace_size(OP_COMBINE, E, N, K, T, k), 16), dtype=torch.uint8, device=device)


def grouped_sparse_gemm_combine(act: QuantizedActivations, w: PackedSparseWeights, routing: "Routing",
                                gates: torch.Tensor, workspace: torch.Tensor, max_rows_per_expert: int = -1,
                                out: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """Down-projection with the gate-weighted combine fused into the epilogue
    (gsg_grouped_sparse_gemm_combine): out [T, N] bf16, bit for bit grouped_sparse_gemm followed by
    unpermute_scale.  workspace from combine_workspace (zero before the first call, left zero)."""
    assert act.sf_block == 32 and act.K == w.K and act.R == routing.T * routing.k
    _need_cuda(act.codes, act.scales, routing.offsets, routing.perm_src, gates, workspace)
    T, k = routing.T, routing.k
    if out is None:
        out = torch.empty(max(T, 1), w.N, dtype=torch.bfloat16, device=act.codes.device)
    _check("gsg_grouped_sparse_gemm_combine", lib().gsg_grouped_sparse_gemm_combine(
        _ptr(act.codes), _ptr(act.scales), _ptr(act.x_scale), _ptr(w.packed), _ptr(w.w_scale),
        _ptr(routing.offsets), w.E, w.N, w.K, T, k, max_rows_per_expert, _ptr(routing.perm_src), _ptr(gates),
        _ptr(workspace), workspace.numel(), _ptr(out), _stream(stream)))
    return out


def grouped_dense_gemm(act: QuantizedActivations, w: PackedDenseWeights, offsets: torch.Tensor,
                       max_rows_per_expert: int = -1, out: Optional[torch.Tensor] = None,
                       out_dtype: torch.dtype = torch.bfloat16, stream=None) -> torch.Tensor:
    """Dense-NVFP4 control on the same skeleton (gsg_grouped_dense_gemm)."""
    assert act.sf_block == 16 and act.K == w.K
    _need_cuda(act.codes, act.scales, offsets)
    if out is None:
        out = torch.empty(max(act.R, 1), w.N, dtype=out_dtype, device=act.codes.device)
    ydt = OUT_F32 if out.dtype == torch.float32 else OUT_BF16
    _check("gsg_grouped_dense_gemm", lib().gsg_grouped_dense_gemm(
        _ptr(act.codes), _ptr(act.scales), _ptr(act.x_scale), _ptr(w.packed), _ptr(w.w_scale),
        _ptr(offsets), w.E, w.N, w.K, act.R, max_rows_per_expert, _ptr(out), ydt, _stream(stream)))
    return out


def grouped_dense_gemm_native(act: QuantizedActivations, w: PackedDenseWeights, offsets: torch.Tensor,
                              max_rows_per_expert: int = -1, out: Optional[torch.Tensor] = None,
                              out_dtype: torch.dtype = torch.bfloat16, stream=None) -> torch.Tensor:
    """The dense-NVFP4 control with the token rows as MMA operand A (the activation-stationary
    orientation, gsg_grouped_dense_gemm_native); the same result as grouped_dense_gemm."""
    assert act.sf_block == 16 and act.K == w.K
    _need_cuda(act.codes, act.scales, offsets)
    if out is None:
        out = torch.empty(max(act.R, 1), w.N, dtype=out_dtype, device=act.codes.device)
    ydt = OUT_F32 if out.dtype == torch.float32 else OUT_BF16
    _check("gsg_grouped_dense_gemm_native", lib().gsg_grouped_dense_gemm_native(
        _ptr(act.codes), _ptr(act.scales), _ptr(act.x_scale), _ptr(w.packed), _ptr(w.w_scale),
        _ptr(offsets), w.E, w.N, w.K, act.R, max_rows_per_expert, _ptr(out), ydt, _stream(stream)))
    return out


def unpermute_scale(Y: torch.Tensor, inv_perm: torch.Tensor, gates: torch.Tensor, top_k: int,
                    out: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """out[t] = bf16(sum_j gates[t, j] * Y[inv_perm[t*k + j]]) (gsg_unpermute_scale)."""
    _need_cuda(Y, inv_perm, gates)
    assert Y.dtype == torch.bfloat16 and gates.dtype == torch.float32
    T = gates.shape[0]
    N = Y.shape[1]
    if out is None:
        out = torch.empty(T, N, dtype=torch.bfloat16, device=Y.device)
    _check("gsg_unpermute_scale", lib().gsg_unpermute_scale(
        _ptr(Y), _ptr(inv_perm), _ptr(gates), T, top_k, N, _ptr(out), _stream(stream)))
    return out


def get_device_status(stream=None) -> int:
    """Synchronise the stream; return and clear the device status word (0 = ok)."""
    return int(lib().gsg_get_device_status(_stream(stream)))
