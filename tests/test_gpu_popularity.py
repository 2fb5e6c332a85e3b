"""moe_popularity_update on the GPU against the oracle: hist, mean and hot
bit-exact, including the hand-worked example and resume from copied state."""
import json
import os

import numpy as np
import pytest
import torch

import oracle
from conftest import GOLDEN
from parity import dev, host

pytestmark = pytest.mark.gpu


def gpu_step(moe, counts, hist_d, step, P):
    E = counts.shape[0]
    mean = torch.empty(E, device="cuda")
    hot = torch.empty(max(P, 1), dtype=torch.int32, device="cuda")
    moe.moe_popularity_update(dev(counts), hist_d, step, mean, P, hot)
    torch.cuda.synchronize()
    return host(mean), host(hot)[:P]


def test_popularity_golden(moe):
    g = json.load(open(os.path.join(GOLDEN, "popularity_example.json")))
    hist = torch.full((g["W"], g["E"]), 12345, dtype=torch.int32, device="cuda")  # stale rows
    for step, (c, exp) in enumerate(zip(g["counts"], g["after_step"])):
        mean, hot = gpu_step(moe, np.array(c, np.int32), hist, step, g["P"])
        assert mean.tolist() == exp["mean"] and hot.tolist() == exp["hot"]


@pytest.mark.parametrize("E,W,P,steps", [(64, 4, 8, 8), (16, 10, 16, 25), (1024, 3, 100, 7),
                                         (5, 1, 0, 3), (256, 4, 8, 9)])
def test_popularity_matches_oracle(moe, E, W, P, steps):
    rng = np.random.default_rng(E + W)
    hist_ref = np.zeros((W, E), np.int32)
    hist = torch.zeros(W, E, dtype=torch.int32, device="cuda")
    for s in range(steps):
        counts = rng.integers(0, 3000, E).astype(np.int32)
        counts[rng.integers(0, E, 3)] = counts.max()  # ties
        mr, hr = oracle.popularity_update(counts, hist_ref, s, P)
        mg, hg = gpu_step(moe, counts, hist, s, P)
        assert np.array_equal(mg, mr) and np.array_equal(hg, hr), s
        assert np.array_equal(host(hist), hist_ref)


def test_popularity_resume(moe):
    rng = np.random.default_rng(9)
    E, W, P = 64, 4, 8
    counts = rng.integers(0, 1000, (10, E)).astype(np.int32)
    hist = torch.zeros(W, E, dtype=torch.int32, device="cuda")
    ref = [gpu_step(moe, counts[s], hist, s, P) for s in range(10)]
    hist2 = torch.zeros(W, E, dtype=torch.int32, device="cuda")
    for s in range(6):
        gpu_step(moe, counts[s], hist2, s, P)
    saved = host(hist2)
    resumed = dev(saved)
    for s in range(6, 10):
        m, h = gpu_step(moe, counts[s], resumed, s, P)
        assert np.array_equal(m, ref[s][0]) and np.array_equal(h, ref[s][1])
