"""moe_route on the GPU against the oracle: bit-exact ids, counts, kept,
offsets, slot_row, row_slot, n_dropped; weights within fp32 rounding."""
import numpy as np
import pytest
import torch

import oracle
from parity import dev, host
from routing_dispatch_expert_fp32_b200 import workloads as wl

pytestmark = pytest.mark.gpu


def run_route(moe, logits, bias, k, capacity):
    T, E = logits.shape
    i32 = torch.int32
    L = dev(logits)
    B = None if bias is None else dev(bias)
    out = dict(ids=torch.full((T, k), -7, dtype=i32, device="cuda"),
               w=torch.full((T, k), -7.0, device="cuda"),
               counts=torch.full((E,), -7, dtype=i32, device="cuda"),
               kept=torch.full((E,), -7, dtype=i32, device="cuda"),
               offsets=torch.full((E + 1,), -7, dtype=i32, device="cuda"),
               slot_row=torch.full((T, k), -7, dtype=i32, device="cuda"),
               row_slot=torch.full((max(T * k, 1),), -7, dtype=i32, device="cuda"),
               n_dropped=torch.full((1,), -7, dtype=i32, device="cuda"))
    ws = torch.empty(moe.moe_route_workspace_size(T, E, k), dtype=torch.uint8, device="cuda")
    moe.moe_route(L, B, k, capacity, out["ids"], out["w"], out["counts"], out["kept"],
                  out["offsets"], out["slot_row"], out["row_slot"], out["n_dropped"], ws)
    torch.cuda.synchronize()
    return {n: host(t) for n, t in out.items()}


def check_route(moe, logits, bias, k, capacity):
    g = run_route(moe, logits, bias, k, capacity)
    r = oracle.route(logits, bias, k, capacity)
    R = int(r["offsets"][-1])
    for name in ["ids", "counts", "kept", "offsets", "slot_row"]:
        assert np.array_equal(g[name], r[name]), name
    assert np.array_equal(g["row_slot"][:R], r["row_slot"]), "row_slot"
    assert int(g["n_dropped"][0]) == r["n_dropped"]
    np.testing.assert_allclose(g["w"], r["w"], rtol=4e-6, atol=1e-8)
    if logits.shape[0]:
        np.testing.assert_allclose(g["w"].astype(np.float64).sum(1), 1.0, atol=2e-6)
    assert moe.moe_device_error() == 0
    return g, r


WORKLOAD_SHAPES = [  # (T, E, k, capacity, zipf_s) of the five layer workloads
    (512, 8, 2, 0, None), (4096, 16, 2, 640, 1.2), (16384, 64, 2, 640, 1.1),
    (32768, 256, 8, 0, 1.0), (65536, 128, 4, 0, None), (65536, 128, 4, 0, 1.5),
]


@pytest.mark.parametrize("T,E,k,cap,s", WORKLOAD_SHAPES)
def test_route_workload_shapes(moe, T, E, k, cap, s):
    w = wl.tiny("r", T=T, d=8, E=E, k=k, F=8, zipf_s=s, capacity_factor=None, index=50 + E)
    rng = wl.rng_for(w, 0, wl.TENSOR_LOGITS)
    logits = rng.standard_normal((T, E), dtype=np.float32)
    check_route(moe, logits, wl.zipf_bias(w), k, cap)


@pytest.mark.parametrize("T,E,k,cap", [
    (1, 4, 2, 0), (1, 1, 1, 0), (7, 3, 3, 0), (129, 5, 5, 2), (200, 12, 3, 7), (257, 100, 7, 3),
    (300, 33, 4, 0), (1000, 1024, 32, 0), (513, 1000, 8, 1), (130, 17, 16, 0), (4097, 9, 1, 100),
])
def test_route_edge_shapes(moe, T, E, k, cap):
    rng = np.random.default_rng(T * 7 + E)
    logits = rng.standard_normal((T, E), dtype=np.float32)
    bias = rng.standard_normal(E).astype(np.float32)
    check_route(moe, logits, bias, k, cap)


def test_route_ties_break_to_lower_index(moe):
    rng = np.random.default_rng(3)
    logits = rng.integers(-2, 3, (777, 24)).astype(np.float32)  # many exact ties
    logits[5] = 0.0
    logits[6, ::2] = -0.0
    check_route(moe, logits, None, 5, 40)


def test_route_all_tokens_to_one_expert(moe):
    T, E = 1000, 16
    logits = np.tile(np.linspace(-1, 1, E, dtype=np.float32)[::-1], (T, 1))
    g, r = check_route(moe, logits, None, 2, 100)
    assert g["counts"][0] == T and g["kept"][0] == 100 and g["n_dropped"][0] == 2 * T - 200


def test_route_capacity_zero_means_unlimited_and_capacity_one(moe):
    rng = np.random.default_rng(4)
    logits = rng.standard_normal((640, 16), dtype=np.float32)
    check_route(moe, logits, None, 2, 0)
    g, _ = check_route(moe, logits, None, 2, 1)
    assert g["kept"].max() == 1


def test_route_golden_example(moe):
    import json, os
    from conftest import GOLDEN
    gd = json.load(open(os.path.join(GOLDEN, "route_example_a.json")))
    g, _ = check_route(moe, np.array(gd["logits"], np.float32), None, gd["k"], gd["capacity"])
    assert g["slot_row"].tolist() == gd["slot_row"]
    assert g["row_slot"][:7].tolist() == gd["row_slot"]


def test_route_empty_batch(moe):
    g = run_route(moe, np.zeros((0, 8), np.float32), None, 2, 0)
    assert g["counts"].tolist() == [0] * 8 and g["offsets"].tolist() == [0] * 9
    assert g["n_dropped"][0] == 0


def test_route_is_deterministic(moe):
    rng = np.random.default_rng(5)
    logits = rng.standard_normal((20000, 64), dtype=np.float32)
    runs = [run_route(moe, logits, None, 4, 900) for _ in range(3)]
    for other in runs[1:]:
        for name in runs[0]:
            assert np.array_equal(runs[0][name], other[name]), name


def _with_nans(rng, T, E, frac):
    """Logits N(0,1) with a fraction of entries replaced by NaNs of several bit
    patterns (quiet, negative, all-ones) and infinities; some rows all NaN and
    some with fewer than k numbers."""
    lg = rng.standard_normal((T, E)).astype(np.float32)
    bits = np.array([0x7FC00000, 0xFFC00000, 0xFFFFFFFF, 0x7F800001], np.uint32).view(np.float32)
    special = np.concatenate([bits, np.array([np.inf, -np.inf], np.float32)])
    mask = rng.random((T, E)) < frac
    lg[mask] = special[rng.integers(0, len(special), int(mask.sum()))]
    lg[0] = np.nan
    lg[1, 1:] = np.nan
    lg[2, : E - 1] = -np.inf
    return lg


@pytest.mark.parametrize("T,E,k,cap", [(600, 8, 2, 0), (600, 16, 3, 90), (513, 24, 4, 0),
                                       (777, 64, 2, 30), (1100, 128, 4, 0), (300, 256, 8, 0)])
def test_route_nan_logits_rank_first_and_stay_in_range(moe, T, E, k, cap):
    """NaN scores rank above every number, NaNs among themselves by index (the
    oracle's reading); every id stays in [0, E) and routing is bit-exact."""
    rng = np.random.default_rng(T + E)
    logits = _with_nans(rng, T, E, 0.1)
    g = run_route(moe, logits, None, k, cap)
    r = oracle.route(logits, None, k, cap)
    R = int(r["offsets"][-1])
    for name in ["ids", "counts", "kept", "offsets", "slot_row"]:
        assert np.array_equal(g[name], r[name]), name
    assert np.array_equal(g["row_slot"][:R], r["row_slot"])
    assert int(g["n_dropped"][0]) == r["n_dropped"]
    assert g["ids"].min() >= 0 and g["ids"].max() < E
    np.testing.assert_allclose(g["w"], r["w"], rtol=4e-6, atol=1e-8, equal_nan=True)
    assert np.array_equal(np.isnan(g["w"]), np.isnan(r["w"]))
    assert moe.moe_device_error() == 0


@pytest.mark.parametrize("E", [8, 20, 40, 128])
def test_route_unaligned_logits_take_the_scalar_loads(moe, E):
    """A logits pointer that is not 16-byte aligned (an offset view) routes the
    same as an aligned copy."""
    rng = np.random.default_rng(E)
    T, k = 300, 2
    logits = rng.standard_normal((T, E)).astype(np.float32)
    flat = torch.empty(T * E + 1, device="cuda")
    view = flat[1:].view(T, E)
    view.copy_(dev(logits))
    i32 = torch.int32
    out = dict(ids=torch.empty((T, k), dtype=i32, device="cuda"),
               w=torch.empty((T, k), device="cuda"),
               counts=torch.empty((E,), dtype=i32, device="cuda"),
               kept=torch.empty((E,), dtype=i32, device="cuda"),
               offsets=torch.empty((E + 1,), dtype=i32, device="cuda"),
               slot_row=torch.empty((T, k), dtype=i32, device="cuda"),
               row_slot=torch.empty((T * k,), dtype=i32, device="cuda"),
               n_dropped=torch.empty((1,), dtype=i32, device="cuda"))
    ws = torch.empty(moe.moe_route_workspace_size(T, E, k), dtype=torch.uint8, device="cuda")
    moe.moe_route(view, None, k, 0, out["ids"], out["w"], out["counts"], out["kept"],
                  out["offsets"], out["slot_row"], out["row_slot"], out["n_dropped"], ws)
    torch.cuda.synchronize()
    r = oracle.route(logits, None, k, 0)
    for name in ["ids", "counts", "offsets", "slot_row"]:
        assert np.array_equal(host(out[name]), r[name]), name
    np.testing.assert_allclose(host(out["w"]), r["w"], rtol=4e-6, atol=1e-8)


@pytest.mark.parametrize("T,E,k,cap", [
    (1000, 36, 3, 0), (999, 68, 1, 40), (4100, 100, 8, 0), (333, 132, 5, 9), (2049, 252, 6, 0),
    (40000, 64, 2, 700), (20000, 200, 7, 0), (1, 64, 8, 0), (31, 128, 4, 1),
])
def test_route_tiled_shapes(moe, T, E, k, cap):
    """Shapes of the TMA-tiled kernel (32 < E <= 256, E % 4 == 0, k <= 8): partial
    last slabs, skipped slabs, every chunk size (32, 64, 128 tokens) and
    ragged last chunks."""
    rng = np.random.default_rng(T + 3 * E + k)
    logits = rng.standard_normal((T, E), dtype=np.float32)
    bias = (0.5 * rng.standard_normal(E)).astype(np.float32)
    check_route(moe, logits, bias, k, cap)


@pytest.mark.parametrize("E,k", [(64, 2), (96, 5), (128, 4), (256, 8)])
def test_route_near_and_exact_ties_for_many_experts(moe, E, k):
    """Scores a few units in the last place apart, and exact integer ties, so
    that the selection's truncated keys collide and tokens are ranked again
    exactly; -0.0 logits and a -0.0 bias tie with +0.0."""
    rng = np.random.default_rng(E + k)
    T = 700
    base = rng.standard_normal((T, 1)).astype(np.float32)
    steps = rng.integers(-3, 4, (T, E)).astype(np.float32)
    near = (base + steps * np.float32(1.2e-7) * np.abs(base)).astype(np.float32)
    check_route(moe, near, None, k, 0)
    ints = rng.integers(-2, 3, (T, E)).astype(np.float32)
    ints[3] = 0.0
    ints[4, ::2] = -0.0
    bias = np.zeros(E, np.float32)
    bias[::3] = -0.0
    check_route(moe, ints, bias, k, 25)
