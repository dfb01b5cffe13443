"""The multi-GPU path of the benchmark: independent replicas, one process per GPU.

The method shards by token rows with no data-path collective, so `bench.py --gpus N`
runs N replicas; the process group only carries the barrier and the max over ranks of
the device-timed region. These tests run that plumbing as two `gloo` ranks on CPU.
"""
import os
import socket

import pytest
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    import sys
    sys.path.insert(0, ROOT)
    import bench
    r, w, local = bench.dist_setup(world, backend="gloo")
    try:
        # each rank reports a different device time; every rank must see the slowest
        ms = 10.0 + 7.5 * r
        got = bench.max_over_ranks(ms, w)
        bench.barrier(w)
        value = bench.aggregate_tokens_per_s(2048, 50, w, got)
        out[r] = (r, w, local, got, value, bench.replica_seed(r))
    finally:
        torch.distributed.destroy_process_group()


def test_two_gloo_replicas():
    world = 2
    port = _free_port()
    ctx = mp.get_context("spawn")
    with ctx.Manager() as mgr:
        out = mgr.dict()
        procs = [ctx.Process(target=_rank_main, args=(r, world, port, out)) for r in range(world)]
        for p in procs:
            p.start()
        for p in procs:
            p.join(timeout=120)
        codes = [p.exitcode for p in procs]
        res = dict(out)
    assert codes == [0, 0], codes
    assert sorted(res) == [0, 1]
    slowest = 10.0 + 7.5 * (world - 1)
    for r in range(world):
        rank, w, local, got, value, seed = res[r]
        assert (rank, w, local) == (r, world, r)
        assert got == slowest  # max over ranks, identical on every rank
        # whole-job tokens over the slowest rank's time
        assert value == pytest.approx(2048 * 50 * world / (slowest / 1e3))
    # replicas draw different synthetic batches (weak scaling)
    assert res[0][5] != res[1][5]


def test_single_process_needs_no_group():
    import sys
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(3.25, 1) == 3.25
    bench.barrier(1)
    assert bench.aggregate_tokens_per_s(100, 10, 1, 1000.0) == pytest.approx(1000.0)
