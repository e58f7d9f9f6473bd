"""Multi-process logic of bench.py on CPU with the gloo backend (world size 2).

Replicas only: every rank processes its own batch (distinct seeds), there is
no collective on the data path, and the reported time is the max over ranks.
"""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench
from rotated_bit_quantized_block_b200 import workloads as wl


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        elapsed = 10.0 + 5.0 * rank  # rank 1 is the slow one
        m = bench.max_over_ranks(elapsed, world, torch.device("cpu"))
        ids = bench.replica_ids(rank)
        w = wl.WORKLOADS["tiny_w8a8"]
        X, _, _ = wl.linear_inputs(w, 0, replica=ids[0])
        value = bench.whole_job_tokens_per_s(w.M, world, 3, m)
        out[rank] = (m, tuple(ids), float(np.abs(X.astype(np.float32)).sum()), value)
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_two_rank_replicas_max_timing_and_throughput():
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
            assert p.exitcode == 0
        res = dict(out)
    assert res[0][0] == res[1][0] == 15.0              # max over ranks
    assert set(res[0][1]).isdisjoint(res[1][1])         # no shared batches
    assert res[0][2] != res[1][2]                       # different synthetic inputs
    w = wl.WORKLOADS["tiny_w8a8"]
    assert res[0][3] == pytest.approx(w.M * world * 3 / 0.015)


def test_single_rank_reduction_is_identity():
    assert bench.max_over_ranks(3.5, 1, torch.device("cpu")) == 3.5
    assert bench.replica_ids(0) == [0, 1] and bench.replica_ids(3) == [6, 7]
