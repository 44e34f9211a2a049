"""Host-side logic of the multi-GPU replicas (bench.py --gpus N) on CPU: example
ranges per rank, the max-over-ranks timing, and the data-parallel training step's one
exchange (the average of each layer's flat gradient buffer over the ranks), with two gloo
ranks."""
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


_DIMS = dict(n=6, d=8, k=3, n_l=2, dims=[18, 10, 7, 32], layers=2)


def test_gradient_buckets_lay_out_aligned_views():
    gb = replicas.GradBuckets(device="cpu", **_DIMS)
    assert len(gb.flats) == len(gb.grads) == 2
    g = gb.grads[1]
    assert g["Y"].shape == (6, 3) and g["W_L"].shape == (2, 6) and g["out_gamma"].shape == (8,)
    assert [w.shape for w in g["W"]] == [(10, 18), (7, 10), (32, 7)] and [b.shape for b in g["b"]] == [(10,), (7,), (32,)]
    views = [g["Y"], *g["W"], *g["b"], g["fmb_gamma"], g["fmb_beta"], g["W_L"], g["out_gamma"], g["out_beta"]]
    base = gb.flats[1].data_ptr()
    starts = sorted((v.data_ptr() - base) // 4 for v in views)
    assert all(o % replicas.GradBuckets.ALIGN == 0 for o in starts)
    # disjoint, in bounds, and every view writes through to its layer's flat buffer
    ends = sorted(((v.data_ptr() - base) // 4, (v.data_ptr() - base) // 4 + v.numel()) for v in views)
    assert all(a[1] <= b[0] for a, b in zip(ends, ends[1:])) and ends[-1][1] <= gb.numel
    g["W"][2].fill_(3.0)
    assert float(gb.flats[1].sum()) == 3.0 * 32 * 7 and float(gb.flats[0].sum()) == 0.0
    replicas.average_gradients(gb.flats)  # one rank: nothing to exchange
    assert float(gb.flats[1].sum()) == 3.0 * 32 * 7


def _grad_worker(rank, world, port, results):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    replicas.init("gloo", timeout_s=60)
    gb = replicas.GradBuckets(device="cpu", **_DIMS)
    for l, g in enumerate(gb.grads):  # rank- and layer-dependent gradients
        for j, w in enumerate(g["W"]):
            w.fill_(float(rank + 1) * (l + 1) * (j + 1))
        g["Y"].fill_(-2.0 * rank)
        g["out_beta"].fill_(10.0 + rank)
    replicas.average_gradients(gb.flats)
    results[rank] = [gb.flats[l].clone().numpy() for l in range(2)]
    replicas.finish()


def test_two_gloo_ranks_average_their_gradients():
    world = 2
    with mp.get_context("spawn").Manager() as m:
        results = m.dict()
        mp.spawn(_grad_worker, args=(world, _free_port(), results), nprocs=world, join=True)
        res = dict(results)
    import numpy as np

    gb = replicas.GradBuckets(device="cpu", **_DIMS)
    for l, g in enumerate(gb.grads):  # the mean over ranks 0 and 1, written by hand
        for j, w in enumerate(g["W"]):
            w.fill_(1.5 * (l + 1) * (j + 1))
        g["Y"].fill_(-1.0)
        g["out_beta"].fill_(10.5)
    for l in range(2):
        assert np.array_equal(res[0][l], res[1][l])
        assert np.array_equal(res[0][l], gb.flats[l].numpy())
