"""The N > 1 path of bench.py on CPU: world-size-2 gloo ranks run the host
logic of the replica job (one independent sequence per rank, job time = the
slowest rank's, throughput over all ranks).  No GPU and no data-path
collective: the ranks only agree on the time."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench
import synth


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        cfg = synth.get_config("tiny")
        toks = bench.rank_tokens(cfg, 512, rank)
        digests = [None] * world
        dist.all_gather_object(digests, hash(toks.tobytes()))
        ms = 100.0 + 25.0 * rank  # this rank's device time
        job_ms = bench.max_over_ranks(ms, dist, world, "cpu")
        out[rank] = (digests, job_ms, bench.aggregate_tokens_per_s(world, 3, 512, job_ms))
    finally:
        dist.destroy_process_group()


def test_two_replicas_gloo():
    world = 2
    manager = mp.Manager()
    out = manager.dict()
    mp.spawn(_rank_main, args=(world, _free_port(), out), nprocs=world, join=True)
    assert set(out.keys()) == {0, 1}
    d0, ms0, v0 = out[0]
    d1, ms1, v1 = out[1]
    assert d0 == d1 and d0[0] != d0[1]          # each replica has its own sequence
    assert ms0 == ms1 == 125.0                   # job time = slowest rank
    assert v0 == v1 == pytest.approx(2 * 3 * 512 / 0.125)


def test_single_rank_needs_no_process_group():
    assert bench.max_over_ranks(42.0, None, 1, "cpu") == 42.0
    cfg = synth.get_config("tiny")
    assert np.array_equal(bench.rank_tokens(cfg, 256, 0), bench.rank_tokens(cfg, 256, 0))
