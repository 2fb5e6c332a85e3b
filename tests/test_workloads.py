"""Seeded input generator: shapes, seeds and the capacity arithmetic (CPU only)."""
import math

import numpy as np

from routing_dispatch_expert_fp32_b200 import workloads as wl


def test_capacity_is_ceil_of_factor_times_load():
    # ceil(1.25 * T * k / E): 640 for both workloads that set a capacity
    assert wl.WORKLOADS["skewed_drops"].capacity == 640
    assert wl.WORKLOADS["multistep_window"].capacity == 640
    assert wl.WORKLOADS["fine_grained"].capacity == 0
    w = wl.tiny("c", T=7, d=8, E=3, k=2, F=8)
    assert w.capacity == math.ceil(1.25 * 7 * 2 / 3) == 6


def test_generation_is_seeded_and_rank_distinct():
    w = wl.tiny("c", T=64, d=16, E=8, k=2, F=32)
    a, b = wl.make_step(w, 0), wl.make_step(w, 0)
    assert np.array_equal(a["x"], b["x"]) and np.array_equal(a["bias"], b["bias"])
    assert not np.array_equal(wl.make_step(w, 1)["x"], a["x"])
    assert not np.array_equal(wl.make_step(w, 0, rank=1)["x"], a["x"])
    ww = wl.make_weights(w)
    assert ww["W1"].shape == (8, 32, 16) and ww["W2"].shape == (8, 16, 32)
    assert ww["Wg"].shape == (8, 16) and ww["W1"].dtype == np.uint16


def test_zipf_bias_is_a_permuted_zipf_law():
    w = wl.WORKLOADS["skewed_drops"]
    b = wl.zipf_bias(w).astype(np.float64)
    ranks = np.argsort(-b)
    # consecutive ranks r, r+1 differ by 0.8 * s * ln((r+1)/r)
    diffs = b[ranks[:-1]] - b[ranks[1:]]
    r = np.arange(1, w.E)
    np.testing.assert_allclose(diffs, 0.8 * 1.2 * np.log((r + 1) / r), rtol=1e-5)
    H = np.sum(np.arange(1, w.E + 1) ** -1.2)
    np.testing.assert_allclose(b.max(), 0.8 * np.log(1 / H), rtol=1e-6)


def test_bias_random_walk_steps():
    w = wl.WORKLOADS["multistep_window"].with_(T=16, d=8, F=8)
    b0, b1 = wl.bias_at_step(w, 0), wl.bias_at_step(w, 1)
    step = (b1.astype(np.float64) - b0)
    assert 0.01 < np.std(step) < 0.1


def test_bf16_conversion_round_trip():
    v = np.array([1.0, -2.5, 3.140625, 1e-30], np.float32)
    assert np.array_equal(wl.bf16_bits_to_f32(wl.to_bf16_bits(v))[:3], v[:3])
    assert wl.to_bf16_bits(np.array([1 + 2 ** -8], np.float32))[0] == 0x3F80


def test_backward_generators_are_seeded_and_shaped():
    w = wl.WORKLOADS["skewed_drops"].with_(T=64, F=32, d=16)
    a, b = wl.make_grad(w, 1), wl.make_grad(w, 1)
    assert a.dtype == np.uint16 and a.shape == (64, 16) and np.array_equal(a, b)
    assert not np.array_equal(a, wl.make_grad(w, 2))
    inp = wl.ffn_backward_inputs(w, 100)
    assert inp["Xp"].shape == (100, 16) and inp["dYp"].shape == (100, 16)
    assert inp["H"].shape == (100, 32)
    h = wl.bf16_bits_to_f32(inp["H"])
    assert (h >= 0).all() and 0.3 < (h == 0).mean() < 0.7  # about half zeros, as after a ReLU
    again = wl.ffn_backward_inputs(w, 100)
    assert all(np.array_equal(inp[k], again[k]) for k in inp)
    lg = wl.router_logits(w)
    assert lg.dtype == np.float32 and lg.shape == (64, w.E)
    assert np.array_equal(lg, wl.router_logits(w))


def test_expert_weights_come_from_per_expert_streams():
    # expert e's slice is drawn from PCG64(SeedSequence(seed, spawn_key=(e,))),
    # whatever thread draws it
    w = wl.tiny("c", T=8, d=16, E=5, k=2, F=24)
    W = wl.make_weights(w)
    seed = wl.seed_for(w, 0, wl.TENSOR_W1)
    for e in range(w.E):
        rng = np.random.Generator(np.random.PCG64(np.random.SeedSequence(seed, spawn_key=(e,))))
        ref = wl.to_bf16_bits(rng.standard_normal((24, 16), dtype=np.float32)
                              * np.float32(1 / math.sqrt(16)))
        assert np.array_equal(W["W1"][e], ref), e
    assert not np.array_equal(W["W1"][0], W["W1"][1])
