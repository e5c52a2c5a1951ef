"""The multi-GPU host logic on CPU with two gloo ranks: each rank draws its own inputs (weak
scaling, no data exchange), the step time is the max over ranks and the throughput counts
every rank's images."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench
import synthetic as S


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        wl = S.WORKLOADS["vits16_336_b1"]
        seeds = bench.rank_image_seeds(wl, rank)
        img = S.make_images(wl.spec, 1, seeds[0])
        ms_local = 10.0 + 5.0 * rank
        ms_max = bench.allreduce_max(ms_local, dist, "cpu")
        # every rank's first image, gathered only to check that the ranks' inputs differ
        sig = torch.tensor([float(img.sum())])
        allsig = [torch.zeros(1) for _ in range(world)]
        dist.all_gather(allsig, sig)
        q.put((rank, seeds, ms_max, bench.images_per_s(world, 8, 10, ms_max), [float(x) for x in allsig]))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_max_time_and_weak_scaling():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = [q.get(timeout=120) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    res.sort()
    (_, s0, m0, v0, sig0), (_, s1, m1, v1, sig1) = res
    assert m0 == m1 == 15.0                      # the slowest rank's time, on every rank
    assert v0 == v1 == pytest.approx(2 * 8 * 10 / 0.015)
    assert set(s0).isdisjoint(s1)                # distinct inputs per rank
    assert sig0 == sig1 and sig0[0] != sig0[1]
