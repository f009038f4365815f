"""The N > 1 path on CPU: two gloo ranks (world_size 2) shard a packed batch by image.

Checks that both ranks derive the same partition without communication, that the shards cover
every image exactly once with balanced cost, that encoding each rank's shard separately (CPU
oracle, fp64) and reassembling by image gives the full-batch result, and that the step-time
reduction takes the maximum over ranks.
"""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from resolution_vit_vision_b200 import dist as vd
from resolution_vit_vision_b200 import synthetic as syn

GRIDS = [(1, 4, 6), (2, 2, 4), (1, 6, 2), (1, 8, 4), (1, 2, 2)]


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, out_q, window=0):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        from oracle import vit_oracle as vo
        idx, grids, rows = vd.shard(GRIDS, rank, world, depth=1, window=window)
        wts = syn.make_weights(1, 64, 3)
        patches = syn.make_patches(GRIDS, 4)
        mine = {}
        for i, g, (a, b) in zip(idx, grids, rows):
            mine[i] = vo.vit_encode(patches[a:b], [g], wts, window=window)
        parts = [None] * world
        dist.all_gather_object(parts, (idx, mine))
        t = vd.max_over_ranks(1.5 + rank)
        if rank == 0:
            out_q.put((parts, t))
    finally:
        dist.barrier()
        dist.destroy_process_group()


@pytest.mark.parametrize("window", [0, 4])
def test_two_gloo_ranks_shard_and_reassemble(window):
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q, window)) for r in range(world)]
    for p in procs:
        p.start()
    parts, tmax = q.get(timeout=240)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert tmax == 2.5                                       # max over ranks
    seen = sorted(i for idx, _ in parts for i in idx)
    assert seen == list(range(len(GRIDS)))                  # every image exactly once
    assert [idx for idx, _ in parts] == vd.lpt_partition(GRIDS, world, depth=1, window=window)
    # reassembled per-image tokens equal the full-batch encode
    from oracle import vit_oracle as vo
    wts = syn.make_weights(1, 64, 3)
    full = vo.vit_encode(syn.make_patches(GRIDS, 4), GRIDS, wts, window=window)
    per_image = {}
    for _, mine in parts:
        per_image.update(mine)
    got = np.concatenate([per_image[i] for i in range(len(GRIDS))])
    np.testing.assert_allclose(got, full, rtol=1e-10, atol=1e-12)


def test_lpt_partition_properties():
    wl = syn.WORKLOADS["mixed8"]
    for world in (1, 2, 3, 4, 8):
        parts = vd.lpt_partition(wl.grids, world)
        assert sorted(i for p in parts for i in p) == list(range(len(wl.grids)))
        loads = [sum(vd.image_cost(wl.grids[i]) for i in p) for p in parts]
        biggest = max(vd.image_cost(g) for g in wl.grids)
        assert max(loads) - min(loads) <= biggest + 1e-6     # LPT bound
    assert vd.lpt_partition(wl.grids, 2) == vd.lpt_partition(list(wl.grids), 2)   # deterministic
    assert vd.max_over_ranks(3.25) == 3.25                  # no process group: identity


def test_windowed_cost_model_matches_the_oracle_windows():
    # the attention part of the windowed cost is 4 * 1280 * sum of squared window sizes, with the
    # windows the oracle builds; full-attention blocks count the whole frame
    from oracle import vit_oracle as vo
    wl = syn.WORKLOADS["mixed8"]
    for g in list(wl.grids) + [(3, 10, 14), (1, 2, 2)]:
        lin = vd.image_cost(g, depth=0)
        win = sum(len(x) ** 2 for x in vo.window_groups([g], 0, 8))
        t, h, w = g
        assert vd.image_cost(g, 1, window=8) - lin == pytest.approx(
            2.0 * t * h * w * (1280 * 3840 + 1280 * 1280 + 2 * 1280 * 5120) + 4.0 * 1280 * win)
        full = vd.image_cost(g, 4, window=8, full_blocks=(1, 3)) - vd.image_cost(g, 4, window=8, full_blocks=())
        assert full == pytest.approx(2 * 4.0 * 1280 * (t * (h * w) ** 2 - win))
    parts = vd.lpt_partition(wl.grids, 4, window=8, full_blocks=(7, 15, 23, 31))
    assert sorted(i for p in parts for i in p) == list(range(len(wl.grids)))
    loads = [sum(vd.image_cost(wl.grids[i], 32, 8, (7, 15, 23, 31)) for i in p) for p in parts]
    assert max(loads) - min(loads) <= max(vd.image_cost(g, 32, 8, (7, 15, 23, 31)) for g in wl.grids) + 1e-6


def test_bench_work_model_windows_match_the_oracle():
    import importlib.util
    from oracle import vit_oracle as vo
    spec = importlib.util.spec_from_file_location("bench_mod", os.path.join(os.path.dirname(__file__), "..", "bench.py"))
    bench = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(bench)
    grids = list(syn.WORKLOADS["mixed8"].grids) + [(2, 6, 10)]
    assert sorted(bench.windows_of(grids, 8)) == sorted(len(x) for x in vo.window_groups(grids, 0, 8))
    P, _, per, _, total = bench.work_model(grids, 32, 3584, 8, (7, 15, 23, 31))
    _, _, per0, _, total0 = bench.work_model(grids, 32, 3584)
    assert total0 - total == pytest.approx(28 * (per0["attention"] - per["attention_window"]))
