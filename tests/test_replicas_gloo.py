"""Replica mode of bench.py on CPU: two gloo ranks, each with its own prompt, agree on the
slowest rank's timings (the max over ranks), and their inputs differ while their shapes and
codec agree.  No GPU and no data-path collective are involved."""
import os
import socket
import sys

import numpy as np
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
    sys.path.insert(0, ROOT)
    import bench

    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        mine = [10.0 + rank, 5.0 - rank, 3.0 * (rank + 1)]
        got = bench.max_over_ranks(mine, dist, "cpu")
        _, cod, x, tok, offs = bench.make_inputs("c1", rank, "cpu")
        np.save(os.path.join(out_dir, f"r{rank}.npy"),
                np.array(got + [float(x.float().sum()), float(x.shape[0]), float(cod.step_scale)]))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_replica_timing_is_max_over_ranks(tmp_path):
    world = 2
    mp.start_processes(_rank_main, args=(world, _free_port(), str(tmp_path)), nprocs=world, start_method="spawn")
    r0, r1 = (np.load(tmp_path / f"r{r}.npy") for r in range(world))
    assert np.array_equal(r0[:3], [11.0, 5.0, 6.0])  # element-wise max of both ranks' values
    assert np.array_equal(r0[:3], r1[:3])            # every rank holds the same result
    assert r0[4] == r1[4] and r0[5] == r1[5]         # same shapes and codec on every rank
    assert r0[3] != r1[3]                            # but each rank codes its own prompt


def test_single_process_needs_no_collective():
    sys.path.insert(0, ROOT)
    import bench

    assert bench.max_over_ranks([1.5, 2]) == [1.5, 2.0]
