"""Host logic of bench.py's multi-GPU mode on CPU, with two gloo ranks.

The path has no exchange step, so the multi-GPU mode runs independent replicas, one per rank.  These tests check
three things:
- every rank gets the slowest rank's time;
- the whole-job figure is the per-rank work times the number of ranks, over that time;
- one GPU needs no process group.
"""
import datetime
import json
import os
import socket

import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, outdir):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        bench._barrier(world)
        # rank r "took" 1 + r ms per call
        ms = bench._max_over_ranks(1.0 + rank, torch.device("cpu"), world)
        res = {"step_bytes": 10 ** 9, "ms_per_call": ms, "ms_per_step": 1000 * ms, "calls_per_step": 1000,
               "per_call_spread": {}, "steps": 10, "path": 1, "copies": 2}
        entry = bench._decode_entry(res, 1000.0, "measured", world)
        with open(os.path.join(outdir, f"{rank}.json"), "w") as f:
            json.dump({"ms": ms, "value": entry["value"], "achieved": entry["roofline"]["achieved"],
                       "frac": entry["roofline"]["frac"]}, f)
        bench._barrier(world)
    finally:
        dist.destroy_process_group()


def test_two_ranks_take_the_slowest_time(tmp_path):
    world = 2
    mp.spawn(_worker, args=(world, _free_port(), str(tmp_path)), nprocs=world, join=True)
    got = [json.load(open(tmp_path / f"{r}.json")) for r in range(world)]
    for g in got:
        assert g["ms"] == 2.0  # the slower rank's time, on every rank
        # 1 GB per call in 2 ms = 500 GB/s per GPU; the job moves twice that
        assert g["achieved"] == 500.0
        assert g["value"] == 1000.0
        assert g["frac"] == 0.5


def test_one_gpu_needs_no_process_group():
    assert not dist.is_initialized()
    bench._barrier(1)
    assert bench._max_over_ranks(3.25, torch.device("cpu"), 1) == 3.25
