"""Cross-layer correlation counts and the popularity forecast on the GPU
against the oracle: counts bit for bit, the forecast bit for bit (both sides
evaluate the same IEEE double operations in the same order), hot experts
exactly."""
import json
import os

import numpy as np
import pytest
import torch

import oracle
from conftest import GOLDEN
from parity import dev, host
from routing_dispatch_expert_fp32_b200 import workloads as wl

pytestmark = pytest.mark.gpu


def _ids(rng, T, E, k):
    return np.argsort(rng.random((T, E)), axis=1)[:, :k].astype(np.int32)


def gpu_corr(moe, a, b, E, init=None):
    C = dev(np.zeros((E, E), np.int32) if init is None else init)
    moe.moe_correlation_update(dev(a), dev(b), C)
    torch.cuda.synchronize()
    return host(C)


def gpu_forecast(moe, pop, C, k_prev, k_next, P):
    E = C.shape[0]
    pred = torch.empty(E, device="cuda")
    hot = torch.empty(max(P, 1), dtype=torch.int32, device="cuda")
    moe.moe_popularity_forecast(dev(pop), dev(C), k_prev, k_next, pred, P, hot)
    torch.cuda.synchronize()
    return host(pred), host(hot)[:P]


def test_forecast_golden(moe):
    g = json.load(open(os.path.join(GOLDEN, "correlation_example.json")))
    C = gpu_corr(moe, np.array(g["ids_prev"], np.int32), np.array(g["ids_next"], np.int32),
                 g["E"])
    assert C.tolist() == g["C"]
    pred, hot = gpu_forecast(moe, np.array(g["pop_prev"], np.float32), C, 1, 2, 2)
    assert pred.tolist() == g["pred"] and hot.tolist() == g["hot_P2"]


@pytest.mark.parametrize("T,E,k_prev,k_next", [
    (16384, 64, 2, 2), (32768, 256, 8, 8), (4096, 16, 2, 2), (777, 128, 4, 1), (100, 1024, 3, 5),
    (1, 3, 1, 3), (5000, 200, 2, 6), (333, 129, 1, 1),
])
def test_correlation_and_forecast_match_oracle(moe, T, E, k_prev, k_next):
    rng = np.random.default_rng(T + E)
    a, b = _ids(rng, T, E, k_prev), _ids(rng, T, E, k_next)
    init = rng.integers(0, 5, (E, E)).astype(np.int32)
    C_ref = init.copy()
    oracle.correlation_update(a, b, C_ref)
    C = gpu_corr(moe, a, b, E, init)
    assert np.array_equal(C, C_ref)
    pop = (rng.random(E) * 1000).astype(np.float32)
    pop[rng.integers(0, E, 3)] = pop.max()  # ties in the hot ranking
    P = min(E, 8)
    pr, hr = oracle.popularity_forecast(pop, C_ref, k_prev, k_next, P)
    pg, hg = gpu_forecast(moe, pop, C, k_prev, k_next, P)
    assert np.array_equal(pg, pr) and np.array_equal(hg, hr)
    assert moe.moe_device_error() == 0


def test_forecast_of_routed_layers_reproduces_next_layer_counts(moe):
    # Two consecutive layers routed by moe_route: with the previous layer's own
    # counts the forecast is exactly the next layer's counts.
    T, E, k = 4096, 32, 2
    rng = np.random.default_rng(1)
    ids = []
    for _ in range(2):
        logits = dev(rng.standard_normal((T, E), dtype=np.float32))
        layer = moe.MoELayer(T, 8, E, k, 8, torch.bfloat16, identity_experts=True)
        moe.moe_route(logits, None, k, 0, layer.ids, layer.w, layer.counts, layer.kept,
                      layer.offsets, layer.slot_row, layer.row_slot, layer.n_dropped,
                      layer.workspace)
        ids.append((layer.ids.clone(), layer.counts.clone()))
    C = torch.zeros(E, E, dtype=torch.int32, device="cuda")
    moe.moe_correlation_update(ids[0][0], ids[1][0], C)
    pred = torch.empty(E, device="cuda")
    hot = torch.empty(4, dtype=torch.int32, device="cuda")
    moe.moe_popularity_forecast(ids[0][1].float(), C, k, k, pred, 4, hot)
    torch.cuda.synchronize()
    assert torch.equal(pred, ids[1][1].float())


def test_out_of_range_ids_are_skipped_and_flagged(moe):
    moe.moe_device_error()
    a = np.array([[0], [5], [1]], np.int32)
    b = np.array([[1], [1], [-2]], np.int32)
    C = gpu_corr(moe, a, b, 4)
    assert C.sum() == 1 and C[0, 1] == 1
    assert moe.moe_device_error() & moe.MOE_DEVERR_EXPERT_INDEX
