"""The multi-rank benchmark plumbing on CPU: two gloo ranks on 127.0.0.1.

The hot path shards over independent batches (heads and sequences share
nothing), so N GPUs run N independent problems with no collective on the data
path; the only cross-rank steps are the barriers around the timed region and
the max-over-ranks reduction of the elapsed time.  These tests run exactly
those steps, plus the per-rank input seeding, with the gloo backend.
"""
import os
import socket
import sys

import pytest
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    import torch.distributed as dist

    import bench
    from deltanet_sequence_mixing_b200 import inputs as gen

    w, r, _ = bench.dist_setup(None)
    assert (w, r) == (world, rank) and dist.get_backend() == "gloo"
    bench.barrier(w)
    # every rank times its own region; the job takes the slowest rank's time
    ms = bench.max_over_ranks(10.0 + 5.0 * rank, w)
    # independent batches: the per-rank seeds never collide
    seeds = bench.input_seeds(rank)
    x = gen.make_inputs(1, 1, 8, 4, 4, torch.float32, seed=seeds[0])
    gathered = [None] * w
    dist.all_gather_object(gathered, (seeds, x["q"].sum().item()))
    rate = bench.whole_job_rate(w, 100, 4, ms)
    out.put((rank, ms, gathered, rate))
    bench.barrier(w)
    dist.destroy_process_group()


@pytest.mark.parametrize("world", [2])
def test_weak_scaling_plumbing_gloo(world):
    ctx = mp.get_context("spawn")
    out = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, out)) for r in range(world)]
    for p in procs:
        p.start()
    res = [out.get(timeout=120) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    res.sort()
    slowest = 10.0 + 5.0 * (world - 1)
    for rank, ms, gathered, rate in res:
        assert ms == slowest                       # max over ranks, same on every rank
        assert rate == pytest.approx(world * 100 * 4 / (slowest * 1e-3))
        seeds = [g[0] for g in gathered]
        flat = [sd for ss in seeds for sd in ss]
        assert len(set(flat)) == len(flat)         # no shared input sets
        sums = [g[1] for g in gathered]
        assert len(set(sums)) == world             # and the draws differ


def test_reference_arm_other_ranks_exit_without_work(monkeypatch):
    sys.path.insert(0, ROOT)
    import argparse

    import bench

    monkeypatch.setenv("RANK", "1")
    monkeypatch.setenv("WORLD_SIZE", "2")
    args = argparse.Namespace(steps=1, warmup=3)
    assert bench.run_reference(args) == 0
