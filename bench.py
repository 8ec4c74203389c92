#!/usr/bin/env python3
"""Benchmark of the grouped sparse-NVFP4 expert GEMM path on B200.

One step = one pass of the hot path over one batch of routed tokens, inputs resident in HBM:
moe_dispatch_nvfp4 (routing + activation quantization into routed order) -> grouped_sparse_gemm
-> unpermute_scale, replayed as one CUDA graph (the weights are packed once, offline, as in
serving).  The L2 cache is flushed before every timed step (a 256 MB write, then a 256 MB read
of another buffer, so that L2 holds neither the step's inputs nor dirty lines whose write-back
would land in the step); each step is timed with CUDA events on the launching stream and the
flush is left outside the events.

Reported (rank 0, one JSON line):
  value     dense-equivalent TFLOP/s of the whole step (2*R*N*K per step, the unit the sparse
            NVFP4 tensor peak is quoted in), summed over ranks / max time over ranks
  e2e       the same metric through the Python API with host (pinned) inputs and outputs,
            host<->device copies inside the timed region: a double-buffered serving loop
            (uploads, compute and downloads of neighbouring steps overlap on three streams);
            e2e.serial is the same calls one step at a time
  roofline  the grouped GEMM kernel alone against its binding roof: algorithmic bytes per launch
            / its event time against the measured HBM copy bandwidth, or (past the ridge point,
            e.g. --config 1t_up_prefill_65k) dense-equivalent TFLOP/s against the measured bf16
            tensor peak x 8 (the sparse NVFP4 / dense bf16 nominal ratio)
  cpu_baseline  the CPU oracle timed on a bounded sample of the same workload (N=1, rank 0)
  control   the dense-NVFP4 grouped GEMM on the same routed activations

--impl reference runs the CPU oracle as the reference arm (the pages ship no implementation).
Multi-GPU (torchrun): every rank runs an independent replica (weak scaling); the path has no
data exchange on one GPU's workload.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import grouped_sparse_gemm_b200 as gsg  # noqa: E402
from grouped_sparse_gemm_b200 import inputs  # noqa: E402

DEFAULT_CONFIG = "1t_up_prefill"          # the largest configuration: the headline
SECONDARY_CONFIG = "30b_up_prefill"       # reported beside it (GEMM and step times only)
METRIC = "grouped sparse-NVFP4 GEMM TFLOP/s + weight GB/s, as % of B200 roofline"
SPARSE_NVFP4_PEAK_TFLOPS_NOMINAL = 18000.0     # the pages' sparse NVFP4 figure (dense-equivalent)
HBM_NOMINAL_GBS = 8000.0
L2_FLUSH_BYTES = 256 << 20


class L2Flush:
    """Flush of the 126 MB L2 before a timed step: a 256 MB write, then a 256 MB read of a
    second buffer (the read writes back the dirty lines the write left, outside the timing, and
    leaves L2 full of clean lines that no step touches), then a random 0-4 µs spin.  The spin
    spreads the step's start over the event timer's tick (about 2 µs on B200), so that the mean
    of many event intervals is not biased by the tick."""

    def __init__(self, dev):
        self.w = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
        self.r = torch.ones(L2_FLUSH_BYTES // 8, dtype=torch.int64, device=dev)
        self.reseed()

    def reseed(self):
        self.rng = np.random.default_rng(1234)

    def fill_(self, v: int):
        self.w.fill_(v)
        self.r.sum()
        torch.cuda._sleep(int(self.rng.integers(0, 8192)))


# ------------------------------------------------------------------ distributed plumbing
def dist_setup(backend: str = "nccl"):
    """One process per GPU (torchrun env).  The process group carries only the barrier and the
    max-over-ranks of the timings: the ranks are independent replicas.  ``backend="gloo"`` runs the
    same host logic on CPU."""
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        if backend == "nccl":
            torch.cuda.set_device(local)
            torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                                 device_id=torch.device(f"cuda:{local}"))
        else:
            torch.distributed.init_process_group(backend, timeout=datetime.timedelta(seconds=60))
    return world, rank, local


def job_value(flops_per_rank: float, world: int, max_ms: float) -> float:
    """Whole-job TFLOP/s: the work of all ranks over the slowest rank's time."""
    return world * flops_per_rank / (max_ms * 1e-3) / 1e12


def barrier(world):
    if world > 1:
        torch.distributed.barrier()


def max_over_ranks(x: float, world: int, dev) -> float:
    if world == 1:
        return x
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


# ------------------------------------------------------------------ peaks and clocks
def measured_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}, "fallback"


def gpu_uuid(dev) -> str | None:
    """The UUID ("GPU-...") of the device torch uses as `dev`.  nvidia-smi and NVML number GPUs
    physically, while under CUDA_VISIBLE_DEVICES torch's device 0 can be any of them: the UUID
    names the same GPU on both sides."""
    try:
        u = str(torch.cuda.get_device_properties(dev).uuid)
    except Exception:
        return None
    return u if u.startswith("GPU-") else "GPU-" + u


class ClockSampler:
    """nvidia-smi clocks and throttle reasons sampled during the timed region, on the GPU with
    the given UUID (the one the process runs on)."""
    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, uuid: str | None):
        self.f = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)
        self.uuid = uuid
        try:
            if uuid is None:
                raise RuntimeError("no device UUID")
            self.p = subprocess.Popen(["nvidia-smi", f"--query-gpu={self.Q}", "--format=csv,noheader,nounits",
                                       "-i", uuid, "-lms", "50"], stdout=self.f, stderr=subprocess.DEVNULL)
        except Exception:
            self.p = None
        # the first query initialises NVML and can stall the device briefly: wait for it to land
        # before the timed region starts
        t0 = time.time()
        while self.p is not None and time.time() - t0 < 10.0 and os.path.getsize(self.f.name) == 0:
            time.sleep(0.05)
        time.sleep(0.2)

    def stop(self):
        if self.p is None:
            return None
        self.p.terminate()
        try:
            self.p.wait(timeout=5)
        except Exception:
            self.p.kill()
        self.f.flush()
        self.f.seek(0)
        rows = [r.split(",") for r in self.f.read().strip().splitlines() if r.strip()]
        os.unlink(self.f.name)
        sm, reasons, smax = [], set(), None
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for r in rows:
            try:
                sm.append(float(r[1]))
                smax = float(r[2])
                for n, v in zip(names, r[5:9]):
                    if v.strip().lower() == "active":
                        reasons.add(n)
            except (ValueError, IndexError):
                continue
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": smax, "reasons": sorted(reasons), "samples": 0,
                    "gpu_uuid": self.uuid}
        busy = [s for s in sm if s > 0.5 * max(sm)]
        return {"sm_mhz": statistics.median(busy), "sm_max_mhz": smax, "reasons": sorted(reasons),
                "samples": len(sm), "gpu_uuid": self.uuid}


# ------------------------------------------------------------------ workload
class Workload:
    """Packed weights, routed inputs and every output buffer of one step, resident on the GPU."""

    def __init__(self, cfg: inputs.MoEConfig, dev: torch.device, with_dense: bool = True):
        self.cfg, self.dev = cfg, dev
        E, N, K, T, k = cfg.E, cfg.N, cfg.K, cfg.T, cfg.top_k
        u8 = dict(dtype=torch.uint8, device=dev)
        L = gsg.lib()
        self.pw = gsg.PackedSparseWeights(packed=torch.empty(L.gsg_sparse_packed_bytes(E, N, K), **u8),
                                          w_scale=torch.empty(E, dtype=torch.float32, device=dev), E=E, N=N, K=K)
        self.pd = None
        if with_dense:
            self.pd = gsg.PackedDenseWeights(packed=torch.empty(L.gsg_dense_packed_bytes(E, N, K), **u8),
                                             w_scale=torch.empty(E, dtype=torch.float32, device=dev), E=E, N=N, K=K)
        ws_pack = torch.empty(max(gsg.workspace_size(gsg.OP_PACK_SPARSE, 1, N, K), 16), **u8)
        for e in range(E):          # generate and pack one expert at a time (offline step)
            We = inputs.expert_weight(cfg, e, str(dev))[None]
            gsg.pack_sparse_nvfp4(We, out=self.pw.expert(e), workspace=ws_pack)
            if with_dense:
                gsg.pack_dense_nvfp4(We, out=self.pd.expert(e), workspace=ws_pack)
            del We
        torch.cuda.synchronize()
        self.X_h = inputs.activations(cfg)
        self.ids_h = inputs.routing(cfg)
        self.gates_h = inputs.gates(cfg)
        self.X = self.X_h.to(dev)
        self.ids = self.ids_h.to(dev)
        self.gates = self.gates_h.to(dev)
        counts = torch.bincount(self.ids_h.reshape(-1).long(), minlength=E)
        self.counts = counts
        self.max_rows = int(counts.max())
        self.touched = int((counts > 0).sum())
        R = cfg.R
        self.route = gsg.Routing(offsets=torch.empty(E + 1, dtype=torch.int32, device=dev),
                                 perm_src=torch.empty(R, dtype=torch.int32, device=dev),
                                 inv_perm=torch.empty(R, dtype=torch.int32, device=dev), T=T, k=k, E=E)
        self.ws_disp = torch.empty(max(gsg.workspace_size(gsg.OP_DISPATCH, E, 0, K, T, k), 16), **u8)
        self.qa = gsg.QuantizedActivations(codes=torch.empty(R, K // 2, **u8),
                                           scales=torch.empty(gsg.act_scales_bytes(R, K, 32), **u8),
                                           x_scale=torch.empty(1, dtype=torch.float32, device=dev), R=R, K=K,
                                           sf_block=32)
        self.Y = torch.empty(R, N, dtype=torch.bfloat16, device=dev)
        self.out = torch.empty(T, N, dtype=torch.bfloat16, device=dev)
        self.qa16 = None
        self.Yd = None
        if with_dense:
            self.Yd = torch.empty(R, N, dtype=torch.bfloat16, device=dev)

    # one step of the hot path
    def step(self):
        c = self.cfg
        gsg.moe_dispatch_nvfp4(self.ids, self.X, c.E, 32, out_route=self.route, out_act=self.qa,
                               workspace=self.ws_disp)
        gsg.grouped_sparse_gemm(self.qa, self.pw, self.route.offsets, self.max_rows, out=self.Y)
        gsg.unpermute_scale(self.Y, self.route.inv_perm, self.gates, c.top_k, out=self.out)

    def step_fused(self):
        """The same step with the scatter fused into the GEMM's epilogue (bit-identical out)."""
        c = self.cfg
        if getattr(self, "ws_comb", None) is None:
            self.ws_comb = gsg.combine_workspace(c.E, c.N, c.K, c.T, c.top_k, self.dev)
        gsg.moe_dispatch_nvfp4(self.ids, self.X, c.E, 32, out_route=self.route, out_act=self.qa,
                               workspace=self.ws_disp)
        gsg.grouped_sparse_gemm_combine(self.qa, self.pw, self.route, self.gates, self.ws_comb, self.max_rows,
                                        out=self.out)

    def launches_per_step(self) -> int:
        """Library kernels one step launches (the library's rules: routing in one launch up to 2048
        rows, histogram + scatter while ceil(R/1024)*E <= 16384, else histogram + scan + scatter;
        the quantizer in one launch, two from R*K = 2^27 when the scale words are staged)."""
        R, E, K = self.cfg.R, self.cfg.E, self.cfg.K
        route = 1 if R <= 2048 else (2 if -(-R // 1024) * E <= 16384 else 3)
        quant = 2 if R * K >= (1 << 27) else 1
        return route + quant + 1 + 1    # routing (the amax pass in its first launch), quantize, GEMM, scatter

    def gemm(self):
        gsg.grouped_sparse_gemm(self.qa, self.pw, self.route.offsets, self.max_rows, out=self.Y)

    def prepare_dense(self):
        self.qa16 = gsg.quantize_act_nvfp4(self.X, 16, self.route.inv_perm, self.cfg.top_k)

    def dense_gemm(self):
        gsg.grouped_dense_gemm(self.qa16, self.pd, self.route.offsets, self.max_rows, out=self.Yd)

    def dense_gemm_native(self):
        gsg.grouped_dense_gemm_native(self.qa16, self.pd, self.route.offsets, self.max_rows, out=self.Yd)

    # algorithmic bytes of one grouped GEMM launch
    def gemm_bytes(self):
        c = self.cfg
        w = self.touched * c.N * c.K * 11 // 32          # 2.75 bit per weight of every touched expert
        a = c.R * c.K // 2 + c.R * c.K // 32            # activation codes + one scale per 32
        y = c.R * c.N * 2
        return w, a, y

    def dense_gemm_bytes(self):
        c = self.cfg
        return self.touched * c.N * c.K * 9 // 16 + c.R * c.K // 2 + c.R * c.K // 16 + c.R * c.N * 2


def capture(fn, warm=2):
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        for _ in range(warm):
            fn()
    torch.cuda.current_stream().wait_stream(s)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        fn()
    torch.cuda.synchronize()
    return g


def capture_timed(fn):
    """CUDA graph of fn between two timing events recorded inside the graph (event-record nodes),
    so that the measured interval holds the kernels and the gaps between them but not the graph's
    launch latency.  Returns (graph, (start, end)); None when events cannot be captured."""
    try:
        ev = (torch.cuda.Event(enable_timing=True, external=True), torch.cuda.Event(enable_timing=True, external=True))

        def body():
            ev[0].record()
            fn()
            ev[1].record()
        return capture(body), ev
    except Exception:
        torch.cuda.synchronize()
        return None


def timed_graph_ms(gt, steps: int, flush_buf: "L2Flush", world: int):
    """Mean of the in-graph event interval over `steps` replays, L2 flushed before each."""
    g, (e0, e1) = gt
    barrier(world)
    torch.cuda.synchronize()
    ts = []
    for i in range(steps):
        flush_buf.fill_(i & 0xFF)
        g.replay()
        e1.synchronize()
        ts.append(e0.elapsed_time(e1))
    torch.cuda.synchronize()
    barrier(world)
    return sum(ts) / steps, ts


def batched_ms(replay, flush: "L2Flush", reps: int, world: int) -> float:
    """Per-step device time at a resolution finer than the event timer's tick: `reps` x (flush +
    replay) back to back between two events, minus `reps` x (flush alone) timed the same way,
    divided by reps.  Each run starts behind a 5 ms spin so that the host has queued it before
    the GPU gets there; both runs draw the same dither spins.  Costs a step pushes into the next
    flush (write-back of the lines it dirtied) count against the step."""
    total = []
    for with_step in (True, False):
        flush.reseed()
        barrier(world)
        torch.cuda.synchronize()
        torch.cuda._sleep(10_000_000)
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        for i in range(reps):
            flush.fill_(i & 0xFF)
            if with_step:
                replay()
        b.record()
        torch.cuda.synchronize()
        total.append(a.elapsed_time(b))
    barrier(world)
    return (total[0] - total[1]) / reps


def timed_ms(fn, steps: int, flush_buf: "L2Flush", world: int):
    """Mean device time of fn over `steps` runs, L2 flushed before each (outside the events)."""
    starts = [torch.cuda.Event(enable_timing=True) for _ in range(steps)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(steps)]
    barrier(world)
    torch.cuda.synchronize()
    for i in range(steps):
        flush_buf.fill_(i & 0xFF)
        starts[i].record()
        fn()
        ends[i].record()
    torch.cuda.synchronize()
    barrier(world)
    ts = [a.elapsed_time(b) for a, b in zip(starts, ends)]
    return sum(ts) / steps, ts


class E2EPipeline:
    """End to end through the public API as a serving loop runs it: every step copies its inputs
    (X, top-k ids, gates) from pinned host memory to the device on an upload stream, runs route ->
    quantize -> GEMM -> scatter on the compute stream, and copies its result to pinned host memory
    on a download stream.  Inputs and results are double-buffered, so step i's upload and step
    i-1's download overlap step i-1's and step i's compute.  The packed weights rotate over three
    replicas (3 x 138 MB at the 30B prefill shape, against a 126 MB L2): a step never finds the
    weights of the step before it in L2, so no flush is needed between steps.  Timed: K steps
    between an event on the upload stream before the first upload and one on the download
    stream after the last download."""

    NW = 3

    def __init__(self, wl: "Workload"):
        self.wl, c = wl, wl.cfg
        self.X_p, self.ids_p, self.g_p = wl.X_h.pin_memory(), wl.ids_h.pin_memory(), wl.gates_h.pin_memory()
        self.out_p = [torch.empty(c.T, c.N, dtype=torch.bfloat16).pin_memory() for _ in range(2)]
        self.X = [wl.X, torch.empty_like(wl.X)]
        self.ids = [wl.ids, torch.empty_like(wl.ids)]
        self.gates = [wl.gates, torch.empty_like(wl.gates)]
        self.out = [wl.out, torch.empty_like(wl.out)]
        self.pw = [wl.pw] + [gsg.PackedSparseWeights(packed=wl.pw.packed.clone(), w_scale=wl.pw.w_scale.clone(),
                                                     E=c.E, N=c.N, K=c.K) for _ in range(self.NW - 1)]
        self.up, self.comp, self.down = torch.cuda.Stream(), torch.cuda.Stream(), torch.cuda.Stream()
        self.uploaded = [torch.cuda.Event() for _ in range(2)]
        self.computed = [torch.cuda.Event() for _ in range(2)]
        self.downloaded = [torch.cuda.Event() for _ in range(2)]

    def h2d_bytes(self) -> int:
        return self.X_p.numel() * 2 + self.ids_p.numel() * 4 + self.g_p.numel() * 4

    def d2h_bytes(self) -> int:
        return self.out_p[0].numel() * 2

    def step(self, i: int, first: bool):
        wl, c, b = self.wl, self.wl.cfg, i & 1
        with torch.cuda.stream(self.up):
            if not first:
                self.up.wait_event(self.computed[b])          # step i-2 is done reading set b
            self.X[b].copy_(self.X_p, non_blocking=True)
            self.ids[b].copy_(self.ids_p, non_blocking=True)
            self.gates[b].copy_(self.g_p, non_blocking=True)
            self.uploaded[b].record(self.up)
        s = self.comp
        s.wait_event(self.uploaded[b])
        if not first:
            s.wait_event(self.downloaded[b])                  # step i-2's result has left out[b]
        gsg.moe_dispatch_nvfp4(self.ids[b], self.X[b], c.E, 32, out_route=wl.route, out_act=wl.qa,
                               workspace=wl.ws_disp, stream=s)
        gsg.grouped_sparse_gemm(wl.qa, self.pw[i % self.NW], wl.route.offsets, wl.max_rows, out=wl.Y, stream=s)
        gsg.unpermute_scale(wl.Y, wl.route.inv_perm, self.gates[b], c.top_k, out=self.out[b], stream=s)
        self.computed[b].record(s)
        with torch.cuda.stream(self.down):
            self.down.wait_event(self.computed[b])
            self.out_p[b].copy_(self.out[b], non_blocking=True)
            self.downloaded[b].record(self.down)

    def run(self, steps: int) -> float:
        """Mean ms per step over `steps` pipelined steps (after a synchronised start)."""
        torch.cuda.synchronize()
        t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        t0.record(self.up)
        self.comp.wait_stream(self.up)
        self.down.wait_stream(self.up)
        h0 = time.perf_counter()
        for i in range(steps):
            self.step(i, first=i < 2)
        self.host_ms = (time.perf_counter() - h0) * 1e3 / steps     # host time to issue one step
        self.down.wait_stream(self.comp)
        self.down.wait_stream(self.up)
        t1.record(self.down)
        torch.cuda.synchronize()
        return t0.elapsed_time(t1) / steps

    def copy_ms(self, reps: int = 20):
        """Device time of one step's uploads alone and of its download alone."""
        res = []
        for fn in (lambda: (self.X[0].copy_(self.X_p, non_blocking=True),
                            self.ids[0].copy_(self.ids_p, non_blocking=True),
                            self.gates[0].copy_(self.g_p, non_blocking=True)),
                   lambda: self.out_p[0].copy_(self.out[0], non_blocking=True)):
            torch.cuda.synchronize()
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record()
            for _ in range(reps):
                fn()
            b.record()
            torch.cuda.synchronize()
            res.append(a.elapsed_time(b) / reps)
        return res

    def copies_together_ms(self, reps: int = 20) -> float:
        """Device time per step of the uploads and the download issued together on their two
        streams (what the pipelined loop overlaps): the host link's two directions at once."""
        torch.cuda.synchronize()
        cur = torch.cuda.current_stream()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(cur)
        self.up.wait_stream(cur)
        self.down.wait_stream(cur)
        for _ in range(reps):
            with torch.cuda.stream(self.up):
                self.X[0].copy_(self.X_p, non_blocking=True)
                self.ids[0].copy_(self.ids_p, non_blocking=True)
                self.gates[0].copy_(self.g_p, non_blocking=True)
            with torch.cuda.stream(self.down):
                self.out_p[1].copy_(self.out[1], non_blocking=True)
        cur.wait_stream(self.up)
        cur.wait_stream(self.down)
        b.record(cur)
        torch.cuda.synchronize()
        return a.elapsed_time(b) / reps


# ------------------------------------------------------------------ CPU oracle (baseline / reference arm)
class OracleSample:
    """The CPU oracle on a bounded sample of the workload.

    Prerequisites (untimed): oracle routing and activation quantization of the whole batch, and
    oracle packing of the sampled experts' weights (packing is the offline step).  Timed unit:
    the oracle's grouped GEMM for one (expert, 128-row weight tile) -- decode of the packed
    weights and of the expert's activation rows, fp64 matmul, tensor scales.
    """

    def __init__(self, cfg, X_h, ids_h, n_experts: int, seed: int = 0):
        from oracle import pack as opack
        from oracle import quant as oquant
        from oracle import route as oroute
        self.cfg = cfg
        ids = ids_h.numpy()
        counts = np.bincount(ids.reshape(-1), minlength=cfg.E)
        order = [int(e) for e in np.argsort(-counts, kind="stable") if counts[e] > 0]
        big = order[: max(1, n_experts // 2)]
        rng = np.random.default_rng(seed)
        rest = [int(e) for e in rng.permutation(order[len(big):])][: max(0, n_experts - len(big))]
        self.experts = big + rest
        self.off, perm_src, _ = oroute.route(ids, cfg.E)
        self.q, self.sc, self.s_x = oquant.quantize_routed(X_h.float().numpy(), 32, perm_src, cfg.top_k)
        self.packed = {e: opack.pack_sparse_expert(inputs.expert_weight(cfg, e).numpy()) for e in self.experts}
        self.units = [(e, nt) for e in self.experts for nt in range(cfg.N // 128)]

    def run(self, units):
        from oracle import gemm as ogemm
        from oracle import pack as opack
        from oracle import quant as oquant
        rows = 0
        t0 = time.perf_counter()
        for e, nt in units:
            lo, hi = int(self.off[e]), int(self.off[e + 1])
            codes, pats, scales, s_w = self.packed[e]
            sl = slice(nt * 128, (nt + 1) * 128)
            wd = opack.decode_sparse_expert(codes[sl], pats[sl], scales[sl])
            ad = oquant.decode_rows(self.q[lo:hi], self.sc[lo:hi], 32)
            ogemm.gemm_rows(ad, wd, float(self.s_x) * float(s_w))
            rows += hi - lo
        dt = time.perf_counter() - t0
        return dt, 2.0 * rows * 128 * self.cfg.K


def blas_threads() -> int:
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 0) for i in threadpool_info() if i.get("user_api") == "blas"]
        if n:
            return int(max(n))
    except Exception:
        pass
    return os.cpu_count() or 1


def workload_config(cfg, l2="flushed before every timed step (256 MB write + 256 MB read of another buffer, "
                              "outside the events)"):
    return {"workload": f"{cfg.name}: E={cfg.E} K={cfg.K} N={cfg.N}, {cfg.T} tokens top-{cfg.top_k} "
                        f"(R={cfg.R}), routing {cfg.routing}"
                        + (f" s={cfg.zipf_s}" if cfg.routing == "zipf" else ""),
            "E": cfg.E, "K": cfg.K, "N": cfg.N, "tokens": cfg.T, "top_k": cfg.top_k, "routed_rows": cfg.R,
            "weights": "paired 4:8 NVFP4 (2.75 bit/weight)", "l2": l2}


def run_reference(args, world, rank):
    """Reference arm: the CPU oracle, a bounded sample per step (about 90 s in all), rank 0 only."""
    if rank != 0:
        return
    cfg = inputs.CONFIGS[args.config]
    smp = OracleSample(cfg, inputs.activations(cfg), inputs.routing(cfg), n_experts=2)
    t_unit, _ = smp.run(smp.units[:2])
    t_unit /= 2
    per_step = int(max(1, min(len(smp.units), 90.0 / max(1, args.steps + args.warmup) / max(t_unit, 1e-6))))
    units = smp.units[:per_step]
    for _ in range(args.warmup):
        smp.run(units)
    ts, fl = [], 0.0
    for _ in range(args.steps):
        dt, fl = smp.run(units)
        ts.append(dt)
    mean = sum(ts) / len(ts)
    value = fl / mean / 1e12
    sample = (f"per step: the oracle grouped GEMM (packed-weight and activation decode + fp64 matmul) of "
              f"{per_step} (expert, 128-row weight tile) units of experts {smp.experts}; routing, activation "
              f"quantization and weight packing done once beforehand")
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": mean * 1e3, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": workload_config(cfg, l2="n/a (CPU)"),
            "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": blas_threads(), "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def tensor_roof_binds(flops: float, nbytes: float, tensor_tflops: float, hbm_gbs: float) -> bool:
    """The binding roof of a launch: the tensor pipe when its flops at the tensor peak take longer
    than its bytes at the HBM peak (past the ridge point), else HBM."""
    return flops / (tensor_tflops * 1e12) > nbytes / (hbm_gbs * 1e9)


def traffic_from_profiles(config_name: str, algorithmic_bytes: int):
    """DRAM bytes per GEMM launch from the committed ncu summary, if the kernel is unchanged.
    An entry captured on a smaller case of the same instantiation ("scaled_from") is scaled to
    this launch by its algorithmic bytes (the kernel's DRAM traffic grows in proportion to them).
    Returns (bytes or None, how)."""
    p = os.path.join(ROOT, "profiles", "gemm_traffic.json")
    if not os.path.exists(p):
        return None, "no capture"
    with open(p) as f:
        d = json.load(f)
    src = os.path.join(ROOT, "grouped_sparse_gemm_b200", "csrc", "gsg_gemm.cu")
    with open(src, "rb") as f:
        sha = hashlib.sha256(f.read()).hexdigest()[:16]
    ent = d.get(config_name)
    if not ent:
        return None, "no capture of this workload"
    if ent.get("gemm_src_sha") != sha:
        return None, "kernel changed since the capture"
    if ent.get("scaled_from"):
        ratio = algorithmic_bytes / float(ent["algorithmic_bytes_captured"])
        return int(ent["dram_bytes_per_launch_captured"] * ratio), (
            f"ncu capture of {ent['scaled_from']} scaled by algorithmic bytes ({ratio:.3f}x)")
    return ent.get("dram_bytes_per_launch"), "ncu capture of this launch"


def run_ours(args, world, rank, local):
    dev = torch.device(f"cuda:{local}")
    torch.cuda.set_device(dev)
    gsg.load_library()
    cfg = inputs.CONFIGS[args.config]
    wl = Workload(cfg, dev, with_dense=not args.quick)
    flush = L2Flush(dev)
    wl.step()
    torch.cuda.synchronize()
    st = gsg.get_device_status()
    if st != 0:
        raise RuntimeError(f"device status {st} after the first step")
    g_step = capture(wl.step)
    g_gemm = capture(wl.gemm)
    gt_step, gt_gemm = capture_timed(wl.step), capture_timed(wl.gemm)
    in_graph = gt_step is not None and gt_gemm is not None
    for _ in range(args.warmup):
        flush.fill_(1)
        (gt_step[0] if in_graph else g_step).replay()
    torch.cuda.synchronize()

    clocks = ClockSampler(gpu_uuid(dev))
    if in_graph:
        step_ms, _ = timed_graph_ms(gt_step, args.steps, flush, world)
        gemm_ms, _ = timed_graph_ms(gt_gemm, args.steps, flush, world)
    else:
        step_ms, _ = timed_ms(g_step.replay, args.steps, flush, world)
        gemm_ms, _ = timed_ms(g_gemm.replay, args.steps, flush, world)
    # the same, from long back-to-back runs (finer than the timer tick); the larger of the two
    # figures is the one reported
    step_b_ms = batched_ms(g_step.replay, flush, 200, world)
    gemm_b_ms = batched_ms(g_gemm.replay, flush, 200, world)
    clk = clocks.stop()
    step_event_ms, gemm_event_ms = step_ms, gemm_ms
    step_ms, gemm_ms = max(step_ms, step_b_ms), max(gemm_ms, gemm_b_ms)
    # the same steps timed from outside the graph (adds the graph launch latency), for reference
    step_outer_ms, _ = timed_ms(g_step.replay, max(10, args.steps // 10), flush, world)
    step_ms = max_over_ranks(step_ms, world, dev)
    gemm_ms_max = max_over_ranks(gemm_ms, world, dev)
    step_outer_ms = max_over_ranks(step_outer_ms, world, dev)
    st = gsg.get_device_status()
    if st != 0:
        raise RuntimeError(f"device status {st} after timing")

    flops = 2.0 * cfg.R * cfg.N * cfg.K
    w_b, a_b, y_b = wl.gemm_bytes()
    touched, max_rows = wl.touched, wl.max_rows
    X_h, ids_h = wl.X_h, wl.ids_h
    launches = wl.launches_per_step()
    value = job_value(flops, world, step_ms)
    peaks, peak_kind = measured_peaks()
    hbm_peak = float(peaks["hbm_gbs"])
    tensor_peak = float(peaks["bf16_tflops"]) * 8.0     # sparse NVFP4 / dense bf16 nominal ratio 18 / 2.25
    gemm_bytes = w_b + a_b + y_b
    achieved_gbs = gemm_bytes / (gemm_ms * 1e-3) / 1e9
    gemm_tflops = flops / (gemm_ms * 1e-3) / 1e12
    # the binding roof: the larger of the two lower bounds on the launch's time (the tensor roof
    # binds only past the ridge point, e.g. the 65,536-token 1T prefill)
    tensor_bound = tensor_roof_binds(flops, gemm_bytes, tensor_peak, hbm_peak)

    # the same number of bytes read by a plain library reduction (torch int64 sum) on the same
    # harness (flush, in-graph events): what a bare read of the GEMM's traffic achieves at this size
    rbuf = torch.empty(((w_b + a_b + y_b) + 7) // 8, dtype=torch.int64, device=dev)
    rout = torch.empty((), dtype=torch.int64, device=dev)
    read = lambda: torch.sum(rbuf, dim=0, out=rout)
    gt_read = capture_timed(read)
    read_ms = timed_graph_ms(gt_read, max(10, args.steps // 10), flush, world)[0] if gt_read is not None else None
    if read_ms is not None:   # the same two timings as the GEMM's, the larger kept
        read_ms = max(read_ms, batched_ms(capture(read).replay, flush, 200, world))
    del rbuf, gt_read

    # end to end through the Python API: pinned host inputs -> device, step, result -> pinned host
    e2e = None
    if not args.quick:
        pipe = E2EPipeline(wl)
        pipe.run(max(3, args.warmup))
        barrier(world)
        e2e_ms = max_over_ranks(pipe.run(max(10, args.steps // 10)), world, dev)
        host_ms = pipe.host_ms
        h2d_ms, d2h_ms = pipe.copy_ms()
        both_ms = pipe.copies_together_ms()

        # the same calls one step at a time (copies, step, copy back), L2 flushed before each
        def e2e_step():
            cur = torch.cuda.current_stream()
            for st in (pipe.up, pipe.comp, pipe.down):
                st.wait_stream(cur)
            pipe.step(0, first=True)
            cur.wait_stream(pipe.down)
        serial_ms = max_over_ranks(timed_ms(e2e_step, max(10, args.steps // 10), flush, world)[0], world, dev)
        e2e = {"value": job_value(flops, world, e2e_ms), "unit": "TFLOP/s", "ms_per_step": e2e_ms,
               "h2d_bytes_per_step": int(pipe.h2d_bytes()), "d2h_bytes_per_step": int(pipe.d2h_bytes()),
               "path": "per step: pinned host -> device copies (upload stream), 3 library calls via the Python "
                       "binding (compute stream), result -> pinned host (download stream); double-buffered so "
                       "uploads and downloads overlap neighbouring steps' compute; weights rotate over 3 "
                       "replicas, no L2 flush",
               "parts_us": {"host_issue_per_step": host_ms * 1e3, "h2d_alone": h2d_ms * 1e3,
                            "d2h_alone": d2h_ms * 1e3, "h2d_and_d2h_together": both_ms * 1e3},
               "serial": {"value": job_value(flops, world, serial_ms), "ms_per_step": serial_ms,
                          "how": "one step at a time, every stream joined before the end event, L2 flushed "
                                 "before each step"}}
        del pipe

    control = None
    if not args.quick:
        wl.prepare_dense()
        gt_dense = capture_timed(wl.dense_gemm) if in_graph else None
        if gt_dense is not None:
            dense_ms, _ = timed_graph_ms(gt_dense, max(10, args.steps // 2), flush, world)
        else:
            dense_ms, _ = timed_ms(capture(wl.dense_gemm).replay, max(10, args.steps // 2), flush, world)
        gt_native = capture_timed(wl.dense_gemm_native) if in_graph else None
        if gt_native is not None:
            native_ms, _ = timed_graph_ms(gt_native, max(10, args.steps // 2), flush, world)
        else:
            native_ms, _ = timed_ms(capture(wl.dense_gemm_native).replay, max(10, args.steps // 2), flush, world)
        control = {"kernel": "dense-NVFP4 grouped GEMM (16-element UE4M3 blocks, 4.5 bit/weight), same skeleton; "
                             "weights as MMA operand A (transposed, as the sparse kernel) and tokens as operand A "
                             "(native, activation-stationary)",
                   "gemm_ms": dense_ms, "tflops": flops / (dense_ms * 1e-3) / 1e12,
                   "hbm_gbs": wl.dense_gemm_bytes() / (dense_ms * 1e-3) / 1e9,
                   "sparse_speedup": dense_ms / gemm_ms,
                   "native_gemm_ms": native_ms, "sparse_speedup_vs_native": native_ms / gemm_ms}

    traffic = traffic_from_profiles(cfg.name, int(gemm_bytes))
    secondary = None
    if not args.quick and SECONDARY_CONFIG != cfg.name:
        secondary = secondary_figures(SECONDARY_CONFIG, dev, args, world)

    cpu = None
    if world == 1 and rank == 0 and not args.no_cpu_baseline:
        smp = OracleSample(cfg, X_h, ids_h, cpu_sample_experts(cfg, args.cpu_experts))
        # (expert, weight tile) units in a seeded order, one at a time, until about 12 s of CPU work
        order = np.random.default_rng(5).permutation(len(smp.units))
        dt, fl, done, rows = 0.0, 0.0, 0, 0
        while dt < 12.0:
            e, nt = smp.units[order[done % len(order)]]
            d2, f2 = smp.run([(e, nt)])
            dt, fl, done = dt + d2, fl + f2, done + 1
            rows += int(smp.off[e + 1] - smp.off[e])
        cpu = {"value": fl / dt / 1e12, "unit": "TFLOP/s", "cores": blas_threads(), "kind": "oracle",
               "sample": (f"the oracle grouped GEMM (packed-weight and activation decode + fp64 matmul) of {done} "
                          f"(expert, 128-row weight tile) units drawn in a seeded order from the "
                          f"{len(smp.units)} units of {len(smp.experts)} experts (the largest half and seeded random "
                          f"others), {rows} routed rows x 128 outputs x K={cfg.K} in all, {dt:.1f} s; routing, "
                          f"quantization and packing untimed")}

    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": step_ms, "higher_is_better": True, "scaling": "weak",
            "timing": ("the larger of two device timings: the mean of CUDA events recorded inside the replayed "
                       "graph around each step (and around the GEMM alone for the roofline), L2 flushed before "
                       "every replay; and 200 back-to-back (flush + replay) minus 200 flushes alone, over 200"
                       if in_graph else
                       "CUDA events around each graph replay; L2 flushed before every replay"),
            "timings_ms": {"step_in_graph_events": step_event_ms, "step_back_to_back": step_b_ms,
                           "gemm_in_graph_events": gemm_event_ms, "gemm_back_to_back": gemm_b_ms,
                           "event_timer_tick_us": 2.048},
            "ms_per_step_incl_graph_launch": step_outer_ms,
            "vs_baseline": None, "dtype": "nvfp4", "data": "synthetic (seeded; random weights, no checkpoint)",
            "config": workload_config(cfg),
            "weight_gbs": world * w_b / (step_ms * 1e-3) / 1e9,
            "roofline_pct": {
                "tensor_sparse_nvfp4_nominal_18pf": 100.0 * value / world / SPARSE_NVFP4_PEAK_TFLOPS_NOMINAL,
                "hbm_nominal_8tbs": 100.0 * (gemm_bytes / (step_ms * 1e-3) / 1e9) / HBM_NOMINAL_GBS},
            "gemm": {"ms": gemm_ms_max, "tflops": gemm_tflops, "weight_gbs": w_b / (gemm_ms * 1e-3) / 1e9,
                     "total_gbs": achieved_gbs, "token_tile": gsg_token_tile(max_rows, cfg.R, cfg.E),
                     "touched_experts": touched, "max_rows_per_expert": max_rows,
                     "tensor_frac_of_measured": gemm_tflops / tensor_peak},
            "roofline": ({"bound": "tensor", "achieved": gemm_tflops, "peak": tensor_peak, "unit": "TFLOP/s",
                          "frac": gemm_tflops / tensor_peak, "traffic": traffic[0], "traffic_source": traffic[1],
                          "kernel": "grouped_gemm_kernel<sparse>",
                          "algorithmic_flops_per_launch": flops,
                          "algorithmic_bytes_per_launch": int(gemm_bytes), "hbm_frac": achieved_gbs / hbm_peak,
                          "peak_source": f"{peak_kind} bf16_tflops (burst) x 8, the sparse NVFP4 / dense bf16 "
                                         f"nominal ratio (18 / 2.25 PFLOP/s)"}
                         if tensor_bound else
                         {"bound": "hbm", "achieved": achieved_gbs, "peak": hbm_peak, "unit": "GB/s",
                          "frac": achieved_gbs / hbm_peak, "traffic": traffic[0], "traffic_source": traffic[1],
                          "kernel": "grouped_gemm_kernel<sparse>",
                          "algorithmic_bytes_per_launch": int(gemm_bytes),
                          "peak_source": f"{peak_kind} hbm_gbs (burst copy)"}),
            "read_ceiling": None if read_ms is None else {
                "gbs": (w_b + a_b + y_b) / (read_ms * 1e-3) / 1e9, "us": read_ms * 1e3,
                "gemm_frac_of_it": achieved_gbs / ((w_b + a_b + y_b) / (read_ms * 1e-3) / 1e9),
                "how": "torch int64 sum over the GEMM's algorithmic byte count, same flush and timings"},
            "e2e": e2e,
            "cpu_baseline": cpu,
            "control": control,
            "gpu_launches": launches * args.steps,
            "secondary": secondary,
            "clocks": clk,
        }
        print(json.dumps(line), flush=True)


def cpu_sample_experts(cfg, requested):
    """Experts in the CPU oracle's sample: as requested, else about 1.2e8 weights' worth (24 at the
    30B shapes, 4 at the 1T shapes) so that the sample's untimed preparation stays near 15 s."""
    if requested:
        return requested
    return int(min(24, max(2, 1.2e8 // (cfg.N * cfg.K))))


def secondary_figures(name: str, dev, args, world):
    """A second configuration's GEMM and step times (same flush and two timings as the headline,
    no control, no end-to-end, no CPU sample)."""
    cfg = inputs.CONFIGS[name]
    wl = Workload(cfg, dev, with_dense=False)
    flush = L2Flush(dev)
    wl.step()
    torch.cuda.synchronize()
    res = {"workload": workload_config(cfg)["workload"]}
    for tag, fn in (("step", wl.step), ("gemm", wl.gemm)):
        gt = capture_timed(fn)
        for _ in range(args.warmup):
            flush.fill_(1)
            gt[0].replay()
        ev, _ = timed_graph_ms(gt, args.steps, flush, world)
        bb = batched_ms(capture(fn).replay, flush, 200, world)
        res[tag + "_ms"] = max_over_ranks(max(ev, bb), world, dev)
        del gt
    st = gsg.get_device_status()
    if st != 0:
        raise RuntimeError(f"device status {st} on {name}")
    flops = 2.0 * cfg.R * cfg.N * cfg.K
    w_b, a_b, y_b = wl.gemm_bytes()
    peaks, _ = measured_peaks()
    res.update({"step_tflops": job_value(flops, world, res["step_ms"]),
                "gemm_tflops": flops / (res["gemm_ms"] * 1e-3) / 1e12,
                "gemm_hbm_gbs": (w_b + a_b + y_b) / (res["gemm_ms"] * 1e-3) / 1e9,
                "gemm_hbm_frac": (w_b + a_b + y_b) / (res["gemm_ms"] * 1e-3) / 1e9 / float(peaks["hbm_gbs"])})
    del wl, flush
    torch.cuda.empty_cache()
    return res


def gsg_token_tile(max_rows: int, R: int, E: int) -> int:
    """The GEMM's token tile for this routing (the library's rule, restated for the report)."""
    for bn in (16, 32, 64):
        if 0 < max_rows <= bn:
            return bn
    return 128 if R >= 64 * E else 64


# ------------------------------------------------------------------ every configuration
def run_all_configs(args, local):
    """Per configuration (the tiny case, the 30B and 1T prefill and decode shapes, the 1T decode
    batch sweep): the GEMM alone and the whole step, in-graph after an L2 flush, the dense-NVFP4
    control on the same routed rows, algorithmic GB/s and the fraction of the measured HBM copy
    bandwidth.  One JSON line per configuration."""
    dev = torch.device(f"cuda:{local}")
    torch.cuda.set_device(dev)
    gsg.load_library()
    flush = L2Flush(dev)
    peaks, kind = measured_peaks()
    hbm = float(peaks["hbm_gbs"])
    tensor = float(peaks["bf16_tflops"]) * 8.0   # sparse NVFP4 / dense bf16 nominal ratio
    names = args.configs.split(",") if args.configs else list(inputs.CONFIGS)
    reps = max(10, min(args.steps, 500))
    for name in names:
        cfg = inputs.CONFIGS[name]
        wl = Workload(cfg, dev, with_dense=True)
        wl.step()
        wl.prepare_dense()
        torch.cuda.synchronize()
        res = {"config": name, "E": cfg.E, "K": cfg.K, "N": cfg.N, "tokens": cfg.T, "top_k": cfg.top_k,
               "routed_rows": cfg.R, "touched_experts": wl.touched, "max_rows_per_expert": wl.max_rows}
        wl.step_fused()   # allocates the combine workspace outside the capture
        torch.cuda.synchronize()
        for tag, fn in (("gemm", wl.gemm), ("step", wl.step), ("step_fused", wl.step_fused),
                        ("dense_gemm", wl.dense_gemm), ("dense_native_gemm", wl.dense_gemm_native)):
            gt = capture_timed(fn)
            for _ in range(3):
                flush.fill_(1)
                gt[0].replay()
            ms, _ = timed_graph_ms(gt, reps, flush, 1)
            b_ms = batched_ms(capture(fn).replay, flush, min(reps, 100), 1)
            res[tag + "_us_events"], res[tag + "_us_back_to_back"] = ms * 1e3, b_ms * 1e3
            res[tag + "_us"] = max(ms, b_ms) * 1e3
            del gt
        st = gsg.get_device_status()
        if st != 0:
            raise RuntimeError(f"device status {st} on {name}")
        w, a, y = wl.gemm_bytes()
        # a plain read of the same number of bytes on the same harness (what a bare read achieves)
        rbuf = torch.empty((w + a + y + 7) // 8, dtype=torch.int64, device=dev)
        rout = torch.empty((), dtype=torch.int64, device=dev)
        read = lambda: torch.sum(rbuf, dim=0, out=rout)
        gt = capture_timed(read)
        for _ in range(3):
            flush.fill_(1)
            gt[0].replay()
        res["read_same_bytes_us"] = max(timed_graph_ms(gt, reps, flush, 1)[0],
                                        batched_ms(capture(read).replay, flush, min(reps, 100), 1)) * 1e3
        del gt, rbuf
        flops = 2.0 * cfg.R * cfg.N * cfg.K
        g_s = res["gemm_us"] * 1e-6
        res.update({"gemm_tflops": flops / g_s / 1e12, "gemm_weight_gbs": w / g_s / 1e9,
                    "gemm_total_gbs": (w + a + y) / g_s / 1e9, "gemm_hbm_frac": (w + a + y) / g_s / 1e9 / hbm,
                    "gemm_tensor_frac": flops / g_s / 1e12 / tensor,
                    "binding_roof": "tensor" if tensor_roof_binds(flops, w + a + y, tensor, hbm) else "hbm",
                    "dense_gemm_gbs": wl.dense_gemm_bytes() / (res["dense_gemm_us"] * 1e-6) / 1e9,
                    "sparse_speedup": res["dense_gemm_us"] / res["gemm_us"],
                    "sparse_speedup_vs_native": res["dense_native_gemm_us"] / res["gemm_us"],
                    "gemm_frac_of_read": res["read_same_bytes_us"] / res["gemm_us"],
                    "hbm_peak_gbs": hbm, "peak_source": kind, "reps": reps,
                    "timing": "the larger of: in-graph CUDA events around each replay, L2 flushed (256 MB write + "
                              "256 MB read of another buffer) before every replay; and back-to-back (flush + replay) "
                              "runs minus flush-only runs, per replay"})
        print(json.dumps(res), flush=True)
        del wl
        torch.cuda.empty_cache()


# ------------------------------------------------------------------ a whole MoE layer
class LayerWorkload:
    """route -> quantize -> up-projection with the SwiGLU epilogue -> down-projection -> unpermute,
    all buffers resident.  The tensor scale of h (the down-projection's input) is calibrated once
    beforehand, like the packing: the amax of h from an unfused fp32 pass over the same batch."""

    def __init__(self, L: inputs.MoELayer, dev: torch.device):
        self.L, self.dev = L, dev
        up, dn = L.up(), L.down()
        E, H, I, T, k, R = L.E, L.H, L.I, L.T, L.top_k, L.R
        u8 = dict(dtype=torch.uint8, device=dev)
        lib = gsg.lib()
        self.wu = gsg.PackedSparseWeights(packed=torch.empty(lib.gsg_sparse_packed_bytes(E, 2 * I, H), **u8),
                                          w_scale=torch.empty(E, dtype=torch.float32, device=dev), E=E, N=2 * I, K=H)
        self.wd = gsg.PackedSparseWeights(packed=torch.empty(lib.gsg_sparse_packed_bytes(E, H, I), **u8),
                                          w_scale=torch.empty(E, dtype=torch.float32, device=dev), E=E, N=H, K=I)
        ws = torch.empty(max(gsg.workspace_size(gsg.OP_PACK_SPARSE, 1, 2 * I, H),
                             gsg.workspace_size(gsg.OP_PACK_SPARSE, 1, H, I), 16), **u8)
        for e in range(E):
            gsg.pack_sparse_nvfp4(inputs.expert_weight(up, e, str(dev))[None], out=self.wu.expert(e), workspace=ws)
            gsg.pack_sparse_nvfp4(inputs.down_weight(L, e, str(dev))[None], out=self.wd.expert(e), workspace=ws)
        self.X = inputs.activations(up).to(dev)
        ids_h = inputs.routing(up)
        self.ids = ids_h.to(dev)
        self.gates = inputs.gates(up).to(dev)
        counts = torch.bincount(ids_h.reshape(-1).long(), minlength=E)
        self.max_rows = int(counts.max())
        self.touched = int((counts > 0).sum())
        self.route = gsg.Routing(offsets=torch.empty(E + 1, dtype=torch.int32, device=dev),
                                 perm_src=torch.empty(R, dtype=torch.int32, device=dev),
                                 inv_perm=torch.empty(R, dtype=torch.int32, device=dev), T=T, k=k, E=E)
        self.ws_route = torch.empty(max(gsg.workspace_size(gsg.OP_ROUTE, E, 0, 0, T, k), 16), **u8)
        self.ws_quant = torch.empty(max(gsg.workspace_size(gsg.OP_QUANTIZE, 0, 0, H, T, k), 16), **u8)
        self.ws_disp = torch.empty(max(gsg.workspace_size(gsg.OP_DISPATCH, E, 0, H, T, k), 16), **u8)
        self.qa = gsg.QuantizedActivations(codes=torch.empty(R, H // 2, **u8),
                                           scales=torch.empty(gsg.act_scales_bytes(R, H, 32), **u8),
                                           x_scale=torch.empty(1, dtype=torch.float32, device=dev), R=R, K=H,
                                           sf_block=32)
        self.h_scale = torch.ones(1, dtype=torch.float32, device=dev)
        self.hq = gsg.QuantizedActivations(codes=torch.empty(R, I // 2, **u8),
                                           scales=torch.empty(gsg.act_scales_bytes(R, I, 32), **u8),
                                           x_scale=self.h_scale, R=R, K=I, sf_block=32)
        self.Y2 = torch.empty(R, H, dtype=torch.bfloat16, device=dev)
        self.out = torch.empty(T, H, dtype=torch.bfloat16, device=dev)
        # calibration of h's tensor scale (offline, like the packing)
        gsg.moe_route_permute(self.ids, E, out=self.route, workspace=self.ws_route)
        gsg.quantize_act_nvfp4(self.X, 32, self.route.inv_perm, k, out=self.qa, workspace=self.ws_quant)
        y = gsg.grouped_sparse_gemm(self.qa, self.wu, self.route.offsets, self.max_rows, out_dtype=torch.float32)
        h = torch.nn.functional.silu(y[:R, :I]) * y[:R, I:]
        amax = float(h.abs().max())
        self.h_scale.fill_(amax / 2688.0 if amax > 0 else 1.0)
        del y, h
        torch.cuda.synchronize()

    def step(self):
        L = self.L
        gsg.moe_dispatch_nvfp4(self.ids, self.X, L.E, 32, out_route=self.route, out_act=self.qa,
                               workspace=self.ws_disp)
        gsg.grouped_sparse_gemm_swiglu(self.qa, self.wu, self.route.offsets, self.h_scale, self.max_rows,
                                       out=self.hq)
        gsg.grouped_sparse_gemm(self.hq, self.wd, self.route.offsets, self.max_rows, out=self.Y2)
        gsg.unpermute_scale(self.Y2, self.route.inv_perm, self.gates, L.top_k, out=self.out)

    def flops(self) -> float:
        L = self.L
        return 2.0 * L.R * (2 * L.I * L.H + L.H * L.I)

    def weight_bytes(self) -> int:
        L = self.L
        return self.touched * (2 * L.I * L.H + L.H * L.I) * 11 // 32


def run_layer(args, local):
    """One MoE layer per step (see LayerWorkload), timed in-graph after an L2 flush: latency per
    token batch, tokens/s, dense-equivalent TFLOP/s of the two GEMMs, weight GB/s."""
    dev = torch.device(f"cuda:{local}")
    torch.cuda.set_device(dev)
    gsg.load_library()
    L = inputs.LAYERS[args.layer]
    wl = LayerWorkload(L, dev)
    flush = L2Flush(dev)
    wl.step()
    torch.cuda.synchronize()
    st = gsg.get_device_status()
    if st != 0:
        raise RuntimeError(f"device status {st} after the first layer step")
    gt = capture_timed(wl.step)
    for _ in range(args.warmup):
        flush.fill_(1)
        gt[0].replay()
    ms_ev, _ = timed_graph_ms(gt, args.steps, flush, 1)
    ms_b = batched_ms(capture(wl.step).replay, flush, min(args.steps, 200), 1)
    ms = max(ms_ev, ms_b)
    st = gsg.get_device_status()
    if st != 0:
        raise RuntimeError(f"device status {st} after timing")
    print(json.dumps({
        "layer": L.name, "us_in_graph_events": ms_ev * 1e3, "us_back_to_back": ms_b * 1e3, "E": L.E, "hidden": L.H, "expert_ffn": L.I, "tokens": L.T, "top_k": L.top_k,
        "routed_rows": L.R, "routing": L.routing, "steps": args.steps, "warmup": args.warmup,
        "us_per_layer": ms * 1e3, "tokens_per_s": L.T / (ms * 1e-3),
        "tflops_dense_equivalent": wl.flops() / (ms * 1e-3) / 1e12,
        "weight_gbs": wl.weight_bytes() / (ms * 1e-3) / 1e9, "h_tensor_scale": float(wl.h_scale.item()),
        "kernels": "routing with the amax pass, quantize, up-projection + SwiGLU + NVFP4 of h, down-projection, unpermute",
        "timing": "the larger of: in-graph CUDA events around the layer, L2 flushed (256 MB write + 256 MB "
                  "read of another buffer) before every replay; and back-to-back (flush + layer) runs minus "
                  "flush-only runs, per layer"}),
          flush=True)


# ------------------------------------------------------------------ G x N sweep
SWEEP_SHAPES = {            # expert projection shapes: (K, N)
    "30b_up": (2048, 1536), "30b_down": (768, 2048), "1t_up": (7168, 4096), "1t_down": (2048, 7168)}


class Energy:
    """Board energy counter through NVML (read only); None when NVML is not available."""

    def __init__(self, uuid: str | None):
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nv, self.h = pynvml, pynvml.nvmlDeviceGetHandleByUUID(uuid)
            self.nv.nvmlDeviceGetTotalEnergyConsumption(self.h)
        except Exception:
            self.nv = None

    def mj(self):
        return None if self.nv is None else float(self.nv.nvmlDeviceGetTotalEnergyConsumption(self.h))


def run_sweep(args, local):
    """Sparse GEMM vs the dense-NVFP4 control over expert-group count G x tokens per expert, for
    the 30B-A3B and 1T expert shapes (weights N(0, 0.02), activations N(0, 1), every expert with
    the same token count).  Per point: in-graph time after an L2 flush, and energy per call from
    the board's energy counter over ~0.2 s of back-to-back replays.  One JSON line per point."""
    dev = torch.device(f"cuda:{local}")
    torch.cuda.set_device(dev)
    gsg.load_library()
    L = gsg.lib()
    u8 = dict(dtype=torch.uint8, device=dev)
    flush = L2Flush(dev)
    energy = Energy(gpu_uuid(dev))
    Gs = [int(x) for x in args.sweep_g.split(",")]
    Ns = [int(x) for x in args.sweep_n.split(",")]
    shapes = args.sweep_shapes.split(",")
    reps = max(10, min(args.steps, 200))
    for shape in shapes:
        K, N = SWEEP_SHAPES[shape]
        Gmax = max(Gs)
        pw = gsg.PackedSparseWeights(packed=torch.empty(L.gsg_sparse_packed_bytes(Gmax, N, K), **u8),
                                     w_scale=torch.empty(Gmax, dtype=torch.float32, device=dev), E=Gmax, N=N, K=K)
        pd = gsg.PackedDenseWeights(packed=torch.empty(L.gsg_dense_packed_bytes(Gmax, N, K), **u8),
                                    w_scale=torch.empty(Gmax, dtype=torch.float32, device=dev), E=Gmax, N=N, K=K)
        ws = torch.empty(max(gsg.workspace_size(gsg.OP_PACK_SPARSE, 1, N, K), 16), **u8)
        cfg_w = inputs.custom_config("sweep", E=Gmax, K=K, N=N, T=1, top_k=1, w_sigma=0.02)
        for e in range(Gmax):
            We = inputs.expert_weight(cfg_w, e, str(dev))[None]
            gsg.pack_sparse_nvfp4(We, out=pw.expert(e), workspace=ws)
            gsg.pack_dense_nvfp4(We, out=pd.expert(e), workspace=ws)
            del We
        sp_per, dn_per = pw.packed.numel() // Gmax, pd.packed.numel() // Gmax
        for G in Gs:
            pwG = gsg.PackedSparseWeights(pw.packed[:G * sp_per], pw.w_scale[:G], G, N, K)
            pdG = gsg.PackedDenseWeights(pd.packed[:G * dn_per], pd.w_scale[:G], G, N, K)
            for nt in Ns:
                R = G * nt
                X = inputs.random_bf16((R, K), seed=7, device=str(dev))
                off = torch.arange(0, R + 1, nt, dtype=torch.int32, device=dev)
                qa32 = gsg.quantize_act_nvfp4(X, 32)
                qa16 = gsg.quantize_act_nvfp4(X, 16)
                Ys = torch.empty(R, N, dtype=torch.bfloat16, device=dev)
                Yd = torch.empty(R, N, dtype=torch.bfloat16, device=dev)
                run_s = lambda: gsg.grouped_sparse_gemm(qa32, pwG, off, nt, out=Ys)
                run_d = lambda: gsg.grouped_dense_gemm(qa16, pdG, off, nt, out=Yd)
                run_n = lambda: gsg.grouped_dense_gemm_native(qa16, pdG, off, nt, out=Yd)
                line = {"sweep": shape, "K": K, "N": N, "G": G, "tokens_per_expert": nt, "R": R}
                for tag, fn, wbytes in (("sparse", run_s, G * sp_per), ("dense", run_d, G * dn_per),
                                        ("dense_native", run_n, G * dn_per)):
                    gt = capture_timed(fn)
                    for _ in range(3):
                        flush.fill_(1)
                        gt[0].replay()
                    ms = max(timed_graph_ms(gt, reps, flush, 1)[0], batched_ms(capture(fn).replay, flush, reps, 1))
                    e_call = None
                    e0 = energy.mj()
                    if e0 is not None:
                        n = max(20, int(0.2 / max(ms * 1e-3, 1e-6)))
                        torch.cuda.synchronize()
                        e0 = energy.mj()
                        for _ in range(n):
                            gt[0].replay()
                        torch.cuda.synchronize()
                        e_call = (energy.mj() - e0) / n
                    act = R * K // 2 + R * K // (32 if tag == "sparse" else 16)
                    line[tag] = {"us": ms * 1e3, "tflops": 2.0 * R * N * K / (ms * 1e-3) / 1e12,
                                 "hbm_gbs": (wbytes + act + R * N * 2) / (ms * 1e-3) / 1e9,
                                 "mj_per_call": e_call}
                    del gt
                line["sparse_speedup"] = line["dense"]["us"] / line["sparse"]["us"]
                line["sparse_speedup_vs_native"] = line["dense_native"]["us"] / line["sparse"]["us"]
                st = gsg.get_device_status()
                if st != 0:
                    raise RuntimeError(f"device status {st} in the sweep")
                print(json.dumps(line), flush=True)
                del X, qa32, qa16, Ys, Yd
        del pw, pd
        torch.cuda.empty_cache()


def run_profile_steps(args, local):
    """The step graph replayed warmup + steps times and nothing else, so that a profiler's launch
    list holds only the step's kernels in step order."""
    dev = torch.device(f"cuda:{local}")
    torch.cuda.set_device(dev)
    gsg.load_library()
    cfg = inputs.CONFIGS[args.config]
    wl = Workload(cfg, dev, with_dense=False)
    wl.step()
    torch.cuda.synchronize()
    g = capture(wl.step, warm=0)
    for _ in range(args.warmup + args.steps):
        g.replay()
    torch.cuda.synchronize()
    st = gsg.get_device_status()
    print(json.dumps({"profile_steps": args.warmup + args.steps, "config": cfg.name,
                      "kernels_per_step": wl.launches_per_step(), "status": st}), flush=True)
    if st != 0:
        raise RuntimeError(f"device status {st}")


def run_profile_quantize(args, local):
    """Routing + activation quantization (gsg_moe_dispatch_nvfp4) at a configuration's activation
    shape, warmup + steps times, with nothing else on the device (no weights): a small process
    for profiler captures of the quantizer's kernels."""
    dev = torch.device(f"cuda:{local}")
    torch.cuda.set_device(dev)
    gsg.load_library()
    cfg = inputs.CONFIGS[args.config]
    X = inputs.activations(cfg).to(dev)
    ids = inputs.routing(cfg).to(dev)
    ws = torch.empty(max(gsg.workspace_size(gsg.OP_DISPATCH, cfg.E, 0, cfg.K, cfg.T, cfg.top_k), 16),
                     dtype=torch.uint8, device=dev)
    r, qa = gsg.moe_dispatch_nvfp4(ids, X, cfg.E, 32, workspace=ws)
    for _ in range(args.warmup + args.steps):
        gsg.moe_dispatch_nvfp4(ids, X, cfg.E, 32, out_route=r, out_act=qa, workspace=ws)
    torch.cuda.synchronize()
    st = gsg.get_device_status()
    print(json.dumps({"profile_quantize": 1 + args.warmup + args.steps, "config": cfg.name, "status": st}),
          flush=True)
    if st != 0:
        raise RuntimeError(f"device status {st}")


def main():
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--config", default=DEFAULT_CONFIG, choices=sorted(inputs.CONFIGS))
    ap.add_argument("--quick", action="store_true", help="skip e2e, dense control and CPU baseline")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-experts", type=int, default=None,
                    help="experts in the CPU oracle's sample (default: by expert size, 24 at 30B, 4 at 1T)")
    ap.add_argument("--all-configs", action="store_true",
                    help="GEMM, step and dense control for every configuration (one JSON line each)")
    ap.add_argument("--configs", default=None, help="comma-separated subset for --all-configs")
    ap.add_argument("--layer", default=None, choices=sorted(inputs.LAYERS),
                    help="time a whole MoE layer (up + SwiGLU + down) instead of the headline step")
    ap.add_argument("--sweep", action="store_true",
                    help="G x N sweep of the sparse GEMM against the dense control (one JSON line per point)")
    ap.add_argument("--sweep-shapes", default="30b_up,30b_down,1t_up,1t_down")
    ap.add_argument("--sweep-g", default="1,8,32,128")
    ap.add_argument("--sweep-n", default="1,8,32,128,512")
    ap.add_argument("--profile-steps", action="store_true",
                    help="for profiler launch lists: only replay the step graph (warmup + steps), print no bench line")
    ap.add_argument("--profile-quantize", action="store_true",
                    help="for profiler captures: only routing + quantization at --config's activation shape")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    world, rank, local = dist_setup()
    try:
        if args.impl == "reference":
            run_reference(args, world, rank)
        elif args.profile_steps:
            run_profile_steps(args, local)
        elif args.profile_quantize:
            run_profile_quantize(args, local)
        elif args.sweep:
            run_sweep(args, local)
        elif args.layer:
            run_layer(args, local)
        elif args.all_configs:
            run_all_configs(args, local)
        else:
            run_ours(args, world, rank, local)
    finally:
        if world > 1:
            torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
