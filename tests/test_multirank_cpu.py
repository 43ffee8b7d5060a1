"""Multi-rank host logic on the CPU (gloo, world size 2).

The decode step shards over sequences with no exchange step: each rank runs
its own batch, and the only cross-rank traffic is the timing reduction
(max of the per-rank step times, sum of the per-rank bytes).  These tests
run that host logic as two gloo ranks: the per-rank batch seeds, the
inputs they produce, and bench.py's reduction helper.
"""
from __future__ import annotations

import hashlib
import os
import socket
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _digest(w) -> str:
    h = hashlib.sha256()
    for t in (w.q, w.kv, w.indices):
        h.update(t.contiguous().view(torch.uint8).numpy().tobytes())
    return h.hexdigest()


def _rank_main(rank: int, world: int, port: int, out_dir: str) -> None:
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        import bench
        from sparse_mla_decode_05_b200 import inputs
        w = inputs.make_config("c1", seed=inputs.shard_seed("c1", rank))
        dig = _digest(w)
        digs = [None] * world
        dist.all_gather_object(digs, dig)
        mx = bench.reduce_over_ranks(10.0 + rank, "max", "cpu")
        sm = bench.reduce_over_ranks(inputs.algorithmic_bytes(w), "sum", "cpu")
        res = {"digs": digs, "max": mx, "sum": sm, "own_bytes": inputs.algorithmic_bytes(w)}
        torch.save(res, os.path.join(out_dir, f"rank{rank}.pt"))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_two_rank_shards_and_reductions(tmp_path):
    world = 2
    mp.start_processes(_rank_main, args=(world, _free_port(), str(tmp_path)), nprocs=world,
                       start_method="spawn", join=True)
    r0 = torch.load(tmp_path / "rank0.pt")
    r1 = torch.load(tmp_path / "rank1.pt")
    # both ranks saw the same gathered digests; the shards differ
    assert r0["digs"] == r1["digs"]
    assert r0["digs"][0] != r0["digs"][1]
    # rank 0's shard is the workload itself (the single-GPU inputs)
    from sparse_mla_decode_05_b200 import inputs
    assert r0["digs"][0] == _digest(inputs.make_config("c1"))
    # max of the step times and sum of the bytes, identical on every rank
    assert r0["max"] == r1["max"] == 11.0
    assert r0["sum"] == r1["sum"] == r0["own_bytes"] + r1["own_bytes"]


def test_shard_seed_rules():
    from sparse_mla_decode_05_b200 import inputs
    assert inputs.shard_seed("c2", 0) is None
    seeds = {inputs.shard_seed("c2", r) for r in range(1, 8)}
    assert len(seeds) == 7 and 1002 not in seeds
    with pytest.raises(ValueError):
        inputs.shard_seed("c2", -1)


def test_reduce_without_process_group_is_identity():
    import bench
    assert bench.reduce_over_ranks(3.5, "max", "cpu") == 3.5
    assert bench.reduce_over_ranks(7, "sum", "cpu") == 7.0
