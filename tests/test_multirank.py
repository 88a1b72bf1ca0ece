"""The multi-rank (torchrun) path of bench.py on CPU: two gloo ranks.

Users are independent, so ranks shard users with no data exchange; the only
collective is the max over ranks of the timings.  Checked here: the shards are
disjoint and cover the global batch, a rank's batch regenerates exactly the
rows of those users in a single-process batch, and the max-reduction returns the
slowest rank's numbers on every rank.
"""

import os
import socket
import sys

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import bench  # noqa: E402
from gen import CONFIGS, make_batch  # noqa: E402


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, B, out):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        users = bench.rank_users(B, rank)
        times = [10.0 + rank, 3.0 - rank]  # rank 0 slower on the second entry
        red = bench.max_over_ranks(times, world, torch.device("cpu"))
        b = make_batch(CONFIGS["c0"], users=users)
        out[rank] = (users, red, b.seq_offsets.tolist(), b.item_ids.tolist(), b.ts.tolist())
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_shard_users_and_take_the_max():
    world, B = 2, 3
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    mp.start_processes(_worker, args=(world, _free_port(), B, out), nprocs=world,
                       start_method="spawn", join=True)
    u0, r0, off0, it0, ts0 = out[0]
    u1, r1, off1, it1, ts1 = out[1]
    assert sorted(u0 + u1) == list(range(world * B)) and not set(u0) & set(u1)
    assert r0 == r1 == [11.0, 3.0]
    # each rank's users regenerate exactly their rows of the single-process batch
    full = make_batch(CONFIGS["c0"], users=list(range(world * B)))
    for users, off, items, ts in ((u0, off0, it0, ts0), (u1, off1, it1, ts1)):
        for k, u in enumerate(users):
            a, e = full.seq_offsets[u], full.seq_offsets[u + 1]
            a2, e2 = off[k], off[k + 1]
            assert e - a == e2 - a2
            assert np.array_equal(full.item_ids[a:e], np.asarray(items[a2:e2]))
            assert np.array_equal(full.ts[a:e], np.asarray(ts[a2:e2]))


def test_single_rank_max_is_identity():
    assert bench.max_over_ranks([1.5, 2.5], 1, None) == [1.5, 2.5]
    assert bench.rank_users(4, 0) == [0, 1, 2, 3]
    assert bench.rank_users(4, 2) == [8, 9, 10, 11]
