"""Multi-rank host logic on CPU: world_size 2 over gloo.

The prefill runs one independent replica per GPU; the decode step splits its
batch of sequences over the ranks and gathers the next-token ids on the host.
The cross-rank steps (barrier, max-over-ranks of the measured time, the batch
split and the id gather) are exercised here without a GPU, plus the
reference arm's rule that ranks other than 0 exit without work.
Not measured on hardware: every GPU run available here has one GPU."""
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


def _shard_worker(rank, world, port, batch, out):
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    torch.distributed.init_process_group("gloo", rank=rank, world_size=world)
    from llama_decoder_only_rmsnorm_b200.sharding import gather_ids, shard
    first, count = shard(batch, world, rank)
    # stand-in for this rank's decode step: the "next id" of sequence s is 1000 + 7 s
    local = torch.tensor([1000 + 7 * s for s in range(first, first + count)], dtype=torch.int32)
    got = gather_ids(local, batch, world, rank)
    out[rank] = (first, count, None if got is None else got.tolist())
    torch.distributed.destroy_process_group()


@pytest.mark.parametrize("batch", [32, 7])
def test_decode_batch_split_and_host_gather_world2_gloo(batch):
    port = _free_port()
    with mp.Manager() as m:
        out = m.dict()
        mp.spawn(_shard_worker, args=(2, port, batch, out), nprocs=2, join=True)
        res = dict(out)
    (f0, c0, ids0), (f1, c1, ids1) = res[0], res[1]
    assert (f0, f1) == (0, c0) and c0 + c1 == batch and c0 - c1 in (0, 1)
    assert ids1 is None                                  # only rank 0 receives the ids
    assert ids0 == [1000 + 7 * s for s in range(batch)]  # in sequence order


def test_shard_covers_the_batch_once():
    sys.path.insert(0, ROOT)
    from llama_decoder_only_rmsnorm_b200.sharding import shard
    for batch in (1, 5, 8, 32, 33, 100):
        for world in range(1, 9):
            seen = []
            for r in range(world):
                first, count = shard(batch, world, r)
                assert count in (batch // world, batch // world + 1)
                seen.extend(range(first, first + count))
            assert seen == list(range(batch)), (batch, world)
    assert shard(32, 8, 3) == (12, 4)
    with pytest.raises(ValueError):
        shard(4, 2, 2)


def test_reference_arm_non_zero_rank_exits_without_work(monkeypatch):
    sys.path.insert(0, ROOT)
    import bench
    monkeypatch.setenv("RANK", "1")
    monkeypatch.setenv("WORLD_SIZE", "2")
    args = type("A", (), {"steps": 1, "warmup": 0})()
    # rank 1 must return before touching CUDA (this container has none)
    assert bench.run_reference(args) is None
