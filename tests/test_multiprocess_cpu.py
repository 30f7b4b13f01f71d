"""Multi-rank host logic of bench.py on CPU: world_size 2 over gloo.

The bench runs one independent replica per GPU; its only cross-rank steps are
the barrier and the max-over-ranks of the measured time.  Both are exercised
here without a GPU, plus the reference arm's rule that ranks other than 0 exit
without work."""
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


def _worker(rank, world, port, out):
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    torch.distributed.init_process_group("gloo", rank=rank, world_size=world)
    import bench
    slowest = bench.max_over_ranks(10.0 + 5.0 * rank, world, device="cpu")
    torch.distributed.barrier()
    out[rank] = slowest
    torch.distributed.destroy_process_group()


def test_max_over_ranks_world2_gloo():
    port = _free_port()
    with mp.Manager() as m:
        out = m.dict()
        mp.spawn(_worker, args=(2, port, out), nprocs=2, join=True)
        assert dict(out) == {0: 15.0, 1: 15.0}


def test_reference_arm_non_zero_rank_exits_without_work(monkeypatch):
    sys.path.insert(0, ROOT)
    import bench
    monkeypatch.setenv("RANK", "1")
    monkeypatch.setenv("WORLD_SIZE", "2")
    args = type("A", (), {"steps": 1, "warmup": 0})()
    # rank 1 must return before touching CUDA (this container has none)
    assert bench.run_reference(args) is None
