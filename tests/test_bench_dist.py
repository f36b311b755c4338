"""The multi-GPU bench path on CPU: two gloo ranks run bench.py's rank
bookkeeping (per-rank layer seed, max-over-ranks step time, whole-job
throughput).  The path has no data-path collective; only the timing is
reduced."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench
from quip_synth import CONFIGS


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        cfg = CONFIGS["attn7b"]
        rc = bench.rank_config(cfg, rank)
        ms = 3.0 + rank                                  # rank 1 is the slow one
        slowest = bench.max_over_ranks(ms, world, "cpu")
        value = bench.job_throughput(cfg, world, slowest)
        out[rank] = (rc.seed, slowest, value)
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_reduce_the_step_time_and_count_every_layer():
    world, port = 2, _free_port()
    mgr = mp.Manager()
    out = mgr.dict()
    mp.spawn(_rank_main, args=(world, port, out), nprocs=world, join=True)
    cfg = CONFIGS["attn7b"]
    assert out[0][0] == cfg.seed and out[1][0] == cfg.seed + 1      # own layer per rank
    for r in range(world):
        assert out[r][1] == pytest.approx(4.0)                      # max over ranks
        assert out[r][2] == pytest.approx(world * cfg.m * cfg.n / 4.0e-3)


def test_single_rank_needs_no_process_group():
    cfg = CONFIGS["tiny"]
    assert bench.max_over_ranks(2.5, 1, "cpu") == 2.5
    assert bench.job_throughput(cfg, 1, 2.5) == pytest.approx(cfg.m * cfg.n / 2.5e-3)
    assert bench.rank_config(cfg, 0) == cfg
