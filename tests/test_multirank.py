"""The multi-GPU bench path (independent replicas) on CPU: two gloo ranks.

Ranks score independent seeded streams (no data-path collective); the only
exchange is the max-over-ranks reduction of the timed region, done here with
gloo exactly as bench.py does it with NCCL."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import synth


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=__import__("datetime").timedelta(seconds=60))
    try:
        import bench
        w = synth.WORKLOADS["bert-base-len2-100"]
        st = synth.make_stream(bench.replica_workload(w, rank), 50)
        mine = [10.0 + rank, 3.0 * (2 - rank)]
        red = bench.reduce_times(mine, dist, "cpu")
        q.put((rank, st.lengths.tolist(), red.tolist()))
    finally:
        dist.destroy_process_group()


def test_two_replicas_have_distinct_streams_and_max_reduced_times():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    out = {}
    for _ in range(2):
        r, lens, red = q.get(timeout=120)
        out[r] = (lens, red)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert out[0][0] != out[1][0]                      # each replica its own requests
    assert out[0][1] == out[1][1] == [11.0, 6.0]       # max over ranks, elementwise


def test_single_process_reduction_and_rate():
    import bench
    assert bench.reduce_times([1.5, 2.5], None, "cpu").tolist() == [1.5, 2.5]
    # 2 ranks x 10,000 requests x 5 steps in 1 s of the slowest rank
    assert bench.whole_job_rate(2, 10000, 5, 1000.0) == 100000.0
    w = synth.WORKLOADS["bert-base-len2-100"]
    assert bench.replica_workload(w, 0) == w
