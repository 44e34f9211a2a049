"""Host-side logic of the multi-GPU replicas (bench.py --gpus N) on CPU: example
ranges per rank and the max-over-ranks timing, with two gloo ranks."""
import os
import socket

import pytest
import torch.multiprocessing as mp

from recsys_feature_interaction_b200 import replicas


def test_example_ranges_cover_without_overlap():
    per = 4096
    ranges = [replicas.example_range(r, 8, per) for r in range(8)]
    assert ranges[0] == (0, per) and ranges[-1] == (7 * per, 8 * per)
    assert all(a[1] == b[0] for a, b in zip(ranges, ranges[1:]))
    split = [replicas.split_range(r, 3, 10) for r in range(3)]
    assert split == [(0, 4), (4, 7), (7, 10)]
    with pytest.raises(ValueError):
        replicas.example_range(3, 2, 10)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, results):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    r, w = replicas.init("gloo", timeout_s=60)
    assert (r, w) == (rank, world)
    replicas.barrier()
    mx = replicas.max_over_ranks(1.5 + rank)  # the slowest rank's time
    results[rank] = (mx, replicas.example_range(r, w, 100))
    replicas.finish()


def test_two_gloo_ranks_agree_on_the_max_time():
    world = 2
    with mp.get_context("spawn").Manager() as m:
        results = m.dict()
        mp.spawn(_worker, args=(world, _free_port(), results), nprocs=world, join=True)
        res = dict(results)
    assert res[0][0] == res[1][0] == 2.5
    assert res[0][1] == (0, 100) and res[1][1] == (100, 200)
