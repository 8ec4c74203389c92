"""bench.py's multi-rank host logic on CPU: two gloo ranks (torch.distributed over 127.0.0.1)
take the same collective steps as the NCCL ranks of a GPU run -- barrier, max over ranks of a
timing, the whole-job value over the slowest rank -- and the reference arm returns at once on
every rank but 0."""
import os
import socket

import pytest
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    import sys
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    import bench
    w, r, local = bench.dist_setup(backend="gloo")
    try:
        bench.barrier(w)
        ms = 1.0 + rank                       # rank r "took" 1 + r ms
        mx = bench.max_over_ranks(ms, w, "cpu")
        val = bench.job_value(1e9, w, mx)     # 1 GFLOP per rank
        class A:                              # the reference arm on a rank other than 0 does no work
            steps, warmup, config = 1, 3, "tiny"
        ref = bench.run_reference(A, w, r) if r != 0 else None
        bench.barrier(w)
        out[rank] = (mx, val, ref)
    finally:
        torch.distributed.destroy_process_group()


def test_two_gloo_ranks_take_max_and_aggregate():
    world = 2
    port = _free_port()
    ctx = mp.get_context("spawn")
    manager = ctx.Manager()
    out = manager.dict()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, out)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
    for p in procs:
        if p.is_alive():
            p.kill()
        assert p.exitcode == 0
    for r in range(world):
        mx, val, ref = out[r]
        assert mx == 2.0                                    # the slowest rank's time
        assert val == pytest.approx(2 * 1e9 / 2e-3 / 1e12)  # all ranks' work over that time
        assert ref is None
