"""Multi-rank logic of the data-parallel layer on CPU (gloo, world size 2).

Each rank routes its own, differently seeded batch; the popularity statistic
is made global by summing the per-expert counts over ranks (the all_reduce the
benchmark issues before the popularity update), and step time is the maximum
over ranks.  Summed counts must equal the counts of routing the union of the
batches, so the window mean after the all_reduce is the window mean of the
union."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import oracle
from routing_dispatch_expert_fp32_b200 import workloads as wl

W_ = wl.tiny("dist", T=300, d=8, E=16, k=2, F=8, zipf_s=1.2, capacity_factor=None, W=3, P=4)


def _logits(rank, step):
    return wl.rng_for(W_, step, wl.TENSOR_LOGITS, rank).standard_normal((W_.T, W_.E),
                                                                        dtype=np.float32)


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        hist = np.zeros((W_.W, W_.E), np.int32)
        results = []
        for step in range(4):
            r = oracle.route(_logits(rank, step), wl.zipf_bias(W_), W_.k)
            counts = torch.from_numpy(r["counts"].astype(np.int64))
            dist.all_reduce(counts)                      # global popularity
            mean, hot = oracle.popularity_update(counts.numpy().astype(np.int32), hist, step,
                                                 W_.P)
            t = torch.tensor([float(rank + 1) * 1.5])    # this rank's elapsed time
            dist.all_reduce(t, op=dist.ReduceOp.MAX)     # the step takes the slowest rank
            results.append((counts.numpy().tolist(), mean.tolist(), hot.tolist(), t.item()))
        out[rank] = results
    finally:
        dist.destroy_process_group()


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def test_two_ranks_share_popularity_and_take_the_slowest_time():
    world = 2
    with mp.Manager() as m:
        out = m.dict()
        mp.start_processes(_worker, args=(world, _free_port(), out), nprocs=world,
                           start_method="spawn", join=True)
        res = dict(out)
    assert res[0] == res[1]  # every rank holds the same global statistic
    hist = np.zeros((W_.W, W_.E), np.int32)
    for step, (counts, mean, hot, t) in enumerate(res[0]):
        union = np.concatenate([_logits(r, step) for r in range(world)])
        ref = oracle.route(union, wl.zipf_bias(W_), W_.k)
        assert counts == ref["counts"].tolist()
        mean_ref, hot_ref = oracle.popularity_update(ref["counts"], hist, step, W_.P)
        assert mean == mean_ref.tolist() and hot == hot_ref.tolist()
        assert t == 3.0
