"""Multi-rank plumbing of bench.py on CPU: two gloo ranks exercise the same
initialisation, barrier and max-over-ranks reduction that the GPU run uses
over NCCL (every rank an independent replica; no data-path collective)."""
import os
import socket

import pytest
import torch
import torch.multiprocessing as mp


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    os.environ.update({"RANK": str(rank), "WORLD_SIZE": str(world), "LOCAL_RANK": str(rank),
                       "MASTER_ADDR": "127.0.0.1", "MASTER_PORT": str(port)})
    import bench
    import torch.distributed as dist
    r, w, local = bench.dist_init("gloo")
    try:
        bench.barrier(w)
        # each rank's "step time": the job's time is the slowest rank's
        m = bench.max_over_ranks(1.0 + 2.5 * r, w, torch.device("cpu"))
        v = bench.job_throughput(16 * 1024, w, m)
        bench.barrier(w)
        out.put((r, w, local, m, v))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_max_over_ranks_and_job_throughput():
    world = 2
    ctx = mp.get_context("spawn")
    out = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, out)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
    codes = [p.exitcode for p in procs]
    for p in procs:
        if p.is_alive():
            p.kill()
    assert codes == [0, 0], codes
    got = sorted(out.get(timeout=5) for _ in range(world))
    slow = 1.0 + 2.5 * (world - 1)
    for r, (rank, w, local, m, v) in enumerate(got):
        assert (rank, w, local) == (r, world, r)
        assert m == pytest.approx(slow)
        assert v == pytest.approx(16 * 1024 * world / (slow * 1e-3))


def test_reference_arm_runs_on_rank_zero_only(capsys, monkeypatch):
    import argparse
    import bench
    monkeypatch.setenv("RANK", "1")
    args = argparse.Namespace(gpus=2, steps=1, warmup=3, impl="reference")
    bench.run_reference(args)  # returns without work or output on rank != 0
    assert capsys.readouterr().out == ""
