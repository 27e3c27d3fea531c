"""The N > 1 host path of bench.py on CPU: two gloo ranks.

Requests are independent, so every rank runs its own seeded batch (weak
scaling) and the only collective is the max over ranks of the device times.
This checks, without a GPU, that the ranks draw disjoint inputs and that the
timing reduction gives every rank the slowest rank's value.
"""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out_dir):
    import sys
    sys.path.insert(0, ROOT)
    import bench
    import workloads
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank,
                            world_size=world)
    try:
        ms = [3.25, 7.5][rank]
        got = bench.max_over_ranks(ms, dist, torch.device("cpu"))
        w = workloads.WORKLOADS["tiny"]
        d = workloads.drafter_inputs(w, seed=w.seed + bench.rank_seed_offset(rank))
        torch.save({"max": got, "L": d["L"], "anchor": d["anchor"]},
                   os.path.join(out_dir, f"rank{rank}.pt"))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_two_ranks_disjoint_inputs_and_max_time(tmp_path):
    port = _free_port()
    mp.start_processes(_rank_main, args=(2, port, str(tmp_path)), nprocs=2, join=True,
                       start_method="spawn")
    r0 = torch.load(tmp_path / "rank0.pt")
    r1 = torch.load(tmp_path / "rank1.pt")
    assert r0["max"] == r1["max"] == 7.5
    assert not torch.equal(r0["L"], r1["L"])           # each rank its own batch


def test_single_rank_is_identity():
    import sys
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(4.0) == 4.0
    assert bench.rank_seed_offset(0) == 0
    assert len({bench.rank_seed_offset(r) for r in range(8)}) == 8
