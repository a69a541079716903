"""Data-parallel host logic of bench.py on two CPU ranks (gloo): max-over-ranks timing, whole-job
throughput, and per-rank token shards with replicated weights.  No GPU is involved."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench
from activation_quantized_gemm_b200 import synth


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        local_ms = [3.0, 5.5][rank]                      # rank 1 is the slow one
        t = bench.max_over_ranks(local_ms, "cpu")
        x = synth.activation_bf16(4, 256, seed=bench.shard_seed(1, rank))
        w = synth.weight_bf16(8, 256, seed=1)
        xs = [None] * world
        ws = [None] * world
        dist.all_gather_object(xs, x.tobytes())
        dist.all_gather_object(ws, w.tobytes())
        out[rank] = (t, xs[0] != xs[1], ws[0] == ws[1])
    finally:
        dist.destroy_process_group()


def test_two_ranks_max_time_and_shards():
    world = 2
    with mp.get_context("spawn").Manager() as m:   # no fork of a multi-threaded test process
        out = m.dict()
        mp.spawn(_worker, args=(world, _free_port(), out), nprocs=world, join=True)
        res = dict(out)
    for rank in range(world):
        t, x_distinct, w_same = res[rank]
        assert t == 5.5, "every rank reports the slowest rank's time"
        assert x_distinct, "each rank quantizes its own tokens"
        assert w_same, "weights are replicated"


def test_job_throughput_counts_every_rank():
    # 2 ranks x 10 steps x 1e12 ops in 4 ms (max over ranks) = 5e15 ops/s
    assert bench.job_throughput(1e12, 10, 2, 4.0) == pytest.approx(5e15)
    assert bench.job_throughput(1e12, 10, 1, 4.0) == pytest.approx(2.5e15)


def test_single_process_max_is_identity():
    assert bench.max_over_ranks(7.25, "cpu") == 7.25


def test_shard_seeds_are_distinct():
    seeds = {bench.shard_seed(2, r) for r in range(8)}
    assert len(seeds) == 8
    a = synth.activation_bf16(2, 128, seed=bench.shard_seed(2, 0))
    b = synth.activation_bf16(2, 128, seed=bench.shard_seed(2, 1))
    assert not np.array_equal(a, b)
