"""Host logic of bench.py's N > 1 path, on CPU with the gloo backend.

The path does not shard (replicas only): each rank runs its own cell, and the only
cross-rank steps are the reductions of the timing line (max of the step and
end-to-end times, sum of the edges) and the barriers around the timed region."""
import os
import socket
import subprocess
import sys

import numpy as np
import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    import datetime

    import torch
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    import bench

    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        dev = torch.device("cpu")
        step_ms = [12.5, 20.0][rank]
        edges = [1000.0, 1500.0][rank]
        e2e_s = [0.7, 0.4][rank]
        dist.barrier()
        got = (bench.reduce_ranks(dist, dev, step_ms, "max"), bench.reduce_ranks(dist, dev, edges, "sum"),
               bench.reduce_ranks(dist, dev, e2e_s, "max"))
        out.put((rank, got))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_timing_reductions_over_two_gloo_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.SimpleQueue()
    port = _free_port()
    mp.start_processes(_rank_main, args=(2, port, q), nprocs=2, join=True, start_method="spawn")
    res = dict(q.get() for _ in range(2))
    for r in (0, 1):
        assert res[r] == (20.0, 2500.0, 0.7)


def test_replicas_draw_different_cells():
    import synth
    w = synth.WORKLOADS["tiny"]
    a, _, box_a = synth.make_cell(w, 0)
    b, _, box_b = synth.make_cell(w, 1)
    assert a.shape == b.shape and np.array_equal(box_a, box_b)
    assert not np.array_equal(a, b)


@pytest.mark.parametrize("rank", ["1"])
def test_reference_arm_other_ranks_exit_without_work(rank):
    env = dict(os.environ, RANK=rank, WORLD_SIZE="2", LOCAL_RANK=rank)
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--gpus", "2",
                        "--steps", "1", "--warmup", "0"], env=env, capture_output=True, text=True, timeout=120)
    assert r.returncode == 0, r.stderr
    assert r.stdout.strip() == ""
