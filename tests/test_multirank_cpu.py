"""The N > 1 bench path on CPU ranks (gloo, world size 2): the path shards by
batch with no exchange, so the only collective is the max of the per-rank
step times, and the whole-job rate counts every rank's work."""
import os
import socket
import subprocess
import sys

import numpy as np
import pytest
import torch.multiprocessing as mp

ROOT = os.path.join(os.path.dirname(__file__), "..")
sys.path.insert(0, ROOT)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    import torch
    import torch.distributed as dist
    import bench
    from vision_transformer_shifted_window_b200 import synthetic as syn
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        ms = [0.7, 1.3][rank]
        got = bench.max_over_ranks(ms, world, device=None)
        w = syn.WORKLOADS[3]
        inp = syn.make_inputs(w, B=1, H=8, W=8, seed=1000 + w.index + 7919 * rank)
        out[rank] = (got, float(inp["q"].sum()))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_take_the_slowest_time_and_independent_inputs():
    port = _free_port()
    manager = mp.get_context("spawn").Manager()
    out = manager.dict()
    mp.spawn(_rank_main, args=(2, port, out), nprocs=2, join=True)
    assert out[0][0] == pytest.approx(1.3) and out[1][0] == pytest.approx(1.3)
    assert out[0][1] != out[1][1]  # each rank draws its own shard of the batch


def test_reference_arm_prints_only_on_rank_zero():
    env = dict(os.environ, WORLD_SIZE="2", RANK="1", LOCAL_RANK="1")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--steps", "1"],
                       env=env, capture_output=True, text=True, timeout=120)
    assert r.returncode == 0 and r.stdout.strip() == ""
