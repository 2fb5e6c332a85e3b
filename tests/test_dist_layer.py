"""Multi-rank host logic of the layer step on CPU (gloo, world size 2).

``MoELayer.forward`` on each rank must issue the step's calls in this order:
gate, route, the counts hook (here a gloo all_reduce, as bench.py's NCCL one),
popularity update, dispatch, expert FFN, combine -- so that the popularity
update sees the counts summed over ranks -- and ``forward_route`` +
``forward_rest`` (the two CUDA graphs of a multi-rank step) must issue the
same sequence.  The library calls are replaced by recorders on CPU tensors
(no GPU here); the routing counts come from the oracle.  bench.py's
max_over_ranks gives every rank the slowest rank's time."""
import os
import socket
import sys

import numpy as np
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import oracle
from conftest import ROOT
from routing_dispatch_expert_fp32_b200 import workloads as wl

W_ = wl.tiny("dist_layer", T=200, d=16, E=8, k=2, F=32, zipf_s=1.1, capacity_factor=None,
             W=3, P=2)


def _logits(rank):
    return wl.rng_for(W_, 0, wl.TENSOR_LOGITS, rank).standard_normal((W_.T, W_.E),
                                                                     dtype=np.float32)


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    sys.path.insert(0, ROOT)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import bench
        from routing_dispatch_expert_fp32_b200 import moe
        calls = []
        r = oracle.route(_logits(rank), None, W_.k)

        def rec(name, fn=None):
            def f(*a, **kw):
                calls.append(name)
                if fn is not None:
                    fn(*a, **kw)
            return f

        def route(logits, bias, k, cap, ids, w, counts, *rest, **kw):
            counts.copy_(torch.from_numpy(r["counts"]))

        seen = []

        def popularity(counts, *a, **kw):
            seen.append(counts.clone().tolist())

        for name in ["moe_gate", "moe_dispatch", "moe_expert_ffn", "moe_combine"]:
            setattr(moe, name, rec(name))
        moe.moe_route = rec("moe_route", route)
        moe.moe_popularity_update_dev = rec("moe_popularity_update_dev", popularity)
        layer = moe.MoELayer(W_.T, W_.d, W_.E, W_.k, W_.F, torch.float32, W=W_.W, P=W_.P,
                             device="cpu")
        x = torch.zeros(W_.T, W_.d)

        def hook(c):
            calls.append("all_reduce")
            dist.all_reduce(c)

        layer.forward(x, "Wg", "W1", "W2", None, counts_hook=hook)
        first = list(calls)
        calls.clear()
        layer.forward_route(x, "Wg", None)
        hook(layer.counts)
        layer.forward_rest(x, "W1", "W2")
        second = list(calls)
        t = bench.max_over_ranks(dist, 1.5 * (rank + 1), "cpu")
        out[rank] = (first, second, seen, t)
    finally:
        dist.destroy_process_group()


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def test_layer_step_orders_the_counts_exchange_before_popularity(libmoe_path):
    world = 2
    with mp.Manager() as m:
        out = m.dict()
        mp.start_processes(_worker, args=(world, _free_port(), out), nprocs=world,
                           start_method="spawn", join=True)
        res = dict(out)
    order = ["moe_gate", "moe_route", "all_reduce", "moe_popularity_update_dev",
             "moe_dispatch", "moe_expert_ffn", "moe_combine"]
    union = oracle.route(np.concatenate([_logits(r) for r in range(world)]), None, W_.k)
    for rank in range(world):
        first, second, seen, t = res[rank]
        assert first == order and second == order
        # the popularity update saw the counts summed over both ranks, twice
        assert seen == [union["counts"].tolist()] * 2
        assert t == 3.0
