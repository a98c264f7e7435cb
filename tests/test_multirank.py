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


def _ensemble_worker(rank, world, port, q):
    """Each rank is one expert: its scores of the same inputs are gathered in
    rank order and every rank reaches the same vote."""
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=__import__("datetime").timedelta(seconds=60))
    try:
        from classifier_scoring_b200.ensemble import gather_scores
        from oracle import ensemble as E
        rng = np.random.default_rng(7 + rank)
        local = torch.from_numpy(rng.normal(size=40).astype(np.float32))
        allv = gather_scores(local)
        d, v = E.majority_vote(allv.numpy())
        q.put((rank, local.numpy().tolist(), allv.numpy().tolist(), d.tolist(), v.tolist()))
    finally:
        dist.destroy_process_group()


def test_ensemble_scores_gather_in_rank_order_and_vote_alike():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    world = 3
    procs = [ctx.Process(target=_ensemble_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    out = {}
    for _ in range(world):
        r, local, allv, d, v = q.get(timeout=120)
        out[r] = (local, allv, d, v)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for r in range(world):
        assert out[r][1] == [out[k][0] for k in range(world)]     # row k = rank k's expert
        assert out[r][2:] == out[0][2:]                            # the same decisions everywhere


def test_code_hash_ignores_comments_and_metric_names(tmp_path):
    import bench
    a = tmp_path / "a.cu"
    b = tmp_path / "b.cu"
    a.write_text("int f() {  // one\n  return 1;\n}\n")
    b.write_text("// header\nint f() {\n\n  return 1;   // two\n}\n")
    assert bench.code_sha(str(a)) == bench.code_sha(str(b))
    b.write_text("int f() {\n  return 2;\n}\n")
    assert bench.code_sha(str(a)) != bench.code_sha(str(b))
    assert bench.metric_for("bert-base-len2-100") == bench.METRIC
    assert "len 5" in bench.metric_for("bert-base-len5-500")
