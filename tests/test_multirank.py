"""The multi-rank bench logic (one process per GPU, replicas of the workload, no data
collective) on CPU: two gloo ranks agree on the slowest rank's time and the whole-job
throughput, exactly as bench.py computes them under torchrun."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        r, w, local = bench.dist_env()
        assert (r, w, local) == (rank, world, rank)
        my_time = 0.5 + 0.25 * rank            # rank 1 is the slowest
        slowest = bench.max_over_ranks(my_time, w)
        value = bench.aggregate(2048, 100, w, slowest)
        out.put((rank, slowest, value))
    finally:
        dist.destroy_process_group()


def test_two_rank_max_and_aggregate():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    res = sorted(q.get(timeout=10) for _ in range(2))
    for rank, slowest, value in res:
        assert slowest == pytest.approx(0.75)
        assert value == pytest.approx(2048 * 100 * 2 / 0.75)


def test_single_rank_is_identity():
    assert bench.max_over_ranks(1.25, 1) == 1.25
    assert bench.aggregate(10, 4, 1, 2.0) == 20.0


def test_byte_counts_match_the_layouts():
    from linear_attention_tree_b200 import workloads as W
    w = W.config(3)
    vb = bench.verify_bytes(w)
    # S_root fp32 + q,k,v bf16 + log_a,b fp32 + parent + offsets + o fp32 + U fp32
    expect = (32 * 32 * 128 * 128 * 4 + 2048 * 32 * 384 * 2 + 2048 * 32 * 8 + 4 * 2048 + 4 * 33
              + 2048 * 32 * 128 * 4 * 2)
    assert vb == expect
    cb = bench.commit_bytes(w)
    assert cb > 2 * 32 * 32 * 128 * 128 * 4
