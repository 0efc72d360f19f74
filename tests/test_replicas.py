"""The multi-GPU form of the path is replicas (one process per GPU, each on its
own seeded copy of the workload, no data exchange): what bench.py does across
ranks -- the per-rank seeds, the max-over-ranks time and the whole-job
throughput -- run here as two gloo ranks on the CPU."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench
from hierarchical_block_sparse_b200.workloads import WORKLOADS, make_inputs


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank, world, port, out):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        ms = 10.0 + 5.0 * rank  # rank 1 is the slow one
        job_ms = bench.max_over_ranks(ms, dist, torch.device("cpu"))
        w = WORKLOADS["tiny_f32_n1k"]
        Q, _, _, _ = make_inputs(w, seed=bench.replica_seed(w.seed, rank))
        out[rank] = (job_ms, float(Q.double().sum()))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_replicas_take_the_slowest_rank_and_distinct_seeds():
    world = 2
    with mp.Manager() as m:
        out = m.dict()
        mp.spawn(_rank, args=(world, _free_port(), out), nprocs=world, join=True)
        res = dict(out)
    assert res[0][0] == res[1][0] == 15.0        # every rank reports the max-over-ranks time
    assert res[0][1] != res[1][1]                # each replica has its own inputs
    assert bench.job_tokens_per_s(1024, world, 15.0) == pytest.approx(2 * 1024 / 0.015)


def test_single_process_needs_no_collective():
    assert bench.max_over_ranks(7.5, None, torch.device("cpu")) == 7.5
    assert bench.replica_seed(42, 0) == 42
