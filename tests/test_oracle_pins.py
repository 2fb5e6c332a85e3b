"""Pins of the CPU oracle against things other than itself (CPU only).

Each test ties one oracle function to what the pages and the mathematics fix:
hand-worked examples (tests/golden), brute force on tiny inputs, closed forms,
invariants and special cases that reduce to a library routine.
"""
import itertools
import json
import math
import os

import numpy as np
import pytest

import oracle
from routing_dispatch_expert_fp32_b200 import workloads as wl
from conftest import GOLDEN


def _golden(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return json.load(f)


def _expr(s: str) -> float:
    """Evaluate the golden files' tiny arithmetic ("1 + 2^-8") exactly in double."""
    return float(eval(s.replace("^", "**"), {"__builtins__": {}}, {}))


# ------------------------------------------------------------- bf16 storage --
def test_bf16_rounding_golden():
    g = _golden("bf16_rounding.json")
    for case in g["cases"]:
        assert oracle.round_bf16(_expr(case["value"])) == int(case["bits"], 16), case


def test_bf16_rounding_agrees_with_float32_path_on_float32_values():
    # For values exactly representable in fp32, one rounding from double equals
    # the integer-trick rounding of the fp32 bits (an independent implementation).
    rng = np.random.default_rng(1)
    v = (rng.standard_normal(20000) * np.exp(rng.uniform(-30, 30, 20000))).astype(np.float32)
    ref = wl.to_bf16_bits(v)
    got = np.array([oracle.round_bf16(float(a)) for a in v], np.uint16)
    assert np.array_equal(got, ref)


# -------------------------------------------------------------------- route --
def _check_route_against(g, r, slot_row, row_slot):
    assert r["ids"].tolist() == g["ids"]
    np.testing.assert_allclose(r["w"], np.array(g["w"]), rtol=0, atol=2e-7)
    assert r["counts"].tolist() == g["counts"]
    assert r["kept"].tolist() == g["kept"]
    assert r["offsets"].tolist() == g["offsets"]
    assert r["n_dropped"] == g["n_dropped"]
    assert r["slot_row"].tolist() == slot_row
    assert r["row_slot"].tolist() == row_slot


def test_route_example_a():
    g = _golden("route_example_a.json")
    r = oracle.route(np.array(g["logits"], np.float32), None, g["k"], g["capacity"])
    _check_route_against(g, r, g["slot_row"], g["row_slot"])


def test_route_example_a_bias_shifts_identically():
    # A per-expert bias equal to a constant moves every z by the same amount:
    # nothing changes (softmax is shift invariant).
    g = _golden("route_example_a.json")
    r = oracle.route(np.array(g["logits"], np.float32), np.full(g["E"], 0.5, np.float32),
                     g["k"], g["capacity"])
    _check_route_against(g, r, g["slot_row"], g["row_slot"])


def test_route_example_b_token_major_and_rank_major():
    g = _golden("route_example_b.json")
    lg = np.array(g["logits"], np.float32)
    r = oracle.route(lg, None, g["k"], g["capacity"])
    _check_route_against(g, r, g["token_major"]["slot_row"], g["token_major"]["row_slot"])
    r = oracle.route(lg, None, g["k"], g["capacity"], rank_major=True)
    _check_route_against(g, r, g["rank_major"]["slot_row"], g["rank_major"]["row_slot"])


def test_route_signed_zero_ties_to_lower_index():
    lg = np.array([[-0.0, 0.0, -1.0], [0.0, -0.0, -1.0]], np.float32)
    r = oracle.route(lg, None, 1)
    assert r["ids"][:, 0].tolist() == [0, 0]


@pytest.mark.parametrize("seed", range(6))
def test_route_topk_brute_force(seed):
    rng = np.random.default_rng(100 + seed)
    T, E, k = 48, int(rng.integers(2, 9)), None
    k = int(rng.integers(1, E + 1))
    # small integers: many exact ties, so the tie rule is exercised
    lg = rng.integers(-2, 3, (T, E)).astype(np.float32)
    bias = rng.integers(-1, 2, E).astype(np.float32) * np.float32(0.5)
    r = oracle.route(lg, bias, k)
    z = lg + bias  # fp32 + fp32, IEEE nearest
    for t in range(T):
        # (1) stable order of (-z, index)
        order = sorted(range(E), key=lambda e: (-float(z[t, e]), e))[:k]
        assert r["ids"][t].tolist() == order
        # (2) the chosen set maximises sum z; among maximisers it is the
        #     lexicographically smallest index set
        best = max(itertools.combinations(range(E), k),
                   key=lambda s: (sum(float(z[t, e]) for e in s), [-e for e in s]))
        assert sorted(order) == list(best)


def _nan_bits(bits):
    return np.array([bits], np.uint32).view(np.float32)[0]


def test_route_nan_ranks_above_every_number_hand_worked():
    # Reading for non-finite scores (the pages assume finite ones): a NaN key
    # ranks above every number, NaNs among themselves by index; the weights of
    # a row whose first choice is NaN are NaN.
    nan, inf = np.float32(np.nan), np.float32(np.inf)
    neg_nan, ones_nan = _nan_bits(0xFFC00000), _nan_bits(0xFFFFFFFF)
    lg = np.array([[1.0, nan, 2.0, nan, -inf],        # -> 1, 3, 2
                   [nan, nan, nan, nan, nan],          # -> 0, 1, 2
                   [inf, 0.0, neg_nan, -1.0, 3.0],     # -> 2, 0, 4
                   [-inf, ones_nan, -inf, 5.0, -inf],  # -> 1, 3, 0
                   [0.5, -0.5, 2.0, 1.0, -inf]],       # -> 2, 3, 0 (no NaN)
                  np.float32)
    r = oracle.route(lg, None, 3)
    assert r["ids"].tolist() == [[1, 3, 2], [0, 1, 2], [2, 0, 4], [1, 3, 0], [2, 3, 0]]
    assert np.isnan(r["w"][:4]).all()
    assert np.isfinite(r["w"][4]).all()
    assert r["counts"].tolist() == [4, 3, 4, 3, 1]


@pytest.mark.parametrize("seed", range(3))
def test_route_nan_and_infinities_brute_force(seed):
    rng = np.random.default_rng(900 + seed)
    T, E = 64, int(rng.integers(3, 12))
    k = int(rng.integers(1, E + 1))
    pool = np.array([np.nan, _nan_bits(0xFFC00001), np.inf, -np.inf, 0.0, -0.0, 1.0, -2.0, 2.0],
                    np.float32)
    lg = pool[rng.integers(0, len(pool), (T, E))]
    r = oracle.route(lg, None, k)
    for t in range(T):
        z = lg[t]
        order = sorted(range(E), key=lambda e: (0, 0.0, e) if np.isnan(z[e])
                       else (1, -float(z[e]), e))[:k]
        assert r["ids"][t].tolist() == order


@pytest.mark.parametrize("seed", range(4))
def test_route_weights_are_renormalised_full_softmax(seed):
    rng = np.random.default_rng(200 + seed)
    T, E, k = 64, 12, 3
    lg = (rng.standard_normal((T, E)) * 3).astype(np.float32)
    bias = rng.standard_normal(E).astype(np.float32)
    r = oracle.route(lg, bias, k)
    z = (lg + bias).astype(np.float64)
    p = np.exp(z - z.max(1, keepdims=True))
    p /= p.sum(1, keepdims=True)  # full softmax over all E experts
    sel = np.take_along_axis(p, r["ids"].astype(np.int64), 1)
    ref = sel / sel.sum(1, keepdims=True)
    np.testing.assert_allclose(r["w"], ref, rtol=2e-7, atol=1e-12)
    np.testing.assert_allclose(r["w"].astype(np.float64).sum(1), 1.0, atol=1e-6)


@pytest.mark.parametrize("capacity", [0, 1, 7, 40])
def test_route_capacity_invariants(capacity):
    rng = np.random.default_rng(300 + capacity)
    T, E, k = 200, 9, 3
    lg = rng.standard_normal((T, E)).astype(np.float32)
    bias = np.linspace(1.5, -1.5, E).astype(np.float32)  # skewed demand
    r = oracle.route(lg, bias, k, capacity)
    ids, sr, rs, off = r["ids"], r["slot_row"], r["row_slot"], r["offsets"]
    # counts by brute force
    assert r["counts"].tolist() == [int((ids == e).sum()) for e in range(E)]
    kept = np.minimum(r["counts"], capacity) if capacity > 0 else r["counts"]
    assert r["kept"].tolist() == kept.tolist()
    assert off.tolist() == [0] + np.cumsum(kept).tolist()
    assert r["n_dropped"] == T * k - int(kept.sum())
    R = int(off[-1])
    # row_slot is a bijection onto the kept slots, inverse of slot_row
    flat = sr.reshape(-1)
    kept_slots = np.nonzero(flat >= 0)[0]
    assert len(kept_slots) == R == len(rs)
    assert sorted(rs.tolist()) == kept_slots.tolist()
    assert all(flat[rs[row]] == row for row in range(R))
    # each group holds one expert's slots, token order strictly increasing,
    # and exactly its first `capacity` slots in token order are kept
    for e in range(E):
        group = rs[off[e]:off[e + 1]]
        assert all(ids.reshape(-1)[s] == e for s in group)
        toks = (group // k).tolist()
        assert toks == sorted(toks) and len(set(toks)) == len(toks)
        visitors = [t * k + j for t in range(T) for j in range(k) if ids[t, j] == e]
        limit = len(visitors) if capacity <= 0 else capacity
        assert group.tolist() == visitors[:limit]


def test_route_every_token_to_one_expert_and_k_equals_e():
    T, E = 33, 4
    lg = np.tile(np.array([0.0, 5.0, 1.0, 2.0], np.float32), (T, 1))
    r = oracle.route(lg, None, 1, capacity=10)
    assert r["counts"].tolist() == [0, T, 0, 0] and r["kept"].tolist() == [0, 10, 0, 0]
    assert r["n_dropped"] == T - 10 and r["slot_row"][:10, 0].tolist() == list(range(10))
    r = oracle.route(lg, None, E)
    assert r["ids"][0].tolist() == [1, 3, 2, 0] and r["counts"].tolist() == [T] * E


# ---------------------------------------------------------- dispatch/combine --
def _bf16(a):
    return wl.to_bf16_bits(np.asarray(a, np.float32))


def test_dispatch_combine_identity_experts_reproduce_x_exactly():
    rng = np.random.default_rng(5)
    T, d, E, k = 96, 40, 6, 3
    x = _bf16(rng.standard_normal((T, d)))
    r = oracle.route(rng.standard_normal((T, E)).astype(np.float32), None, k)
    Xp = oracle.dispatch(x, k, r["row_slot"])
    y = oracle.combine(Xp, T, k, r["slot_row"], r["w"])  # identity experts: Yp = Xp
    # sum_j w_j = 1 within 1e-7, far inside half a bf16 ulp: y rounds back to x
    assert np.array_equal(y, x)


def test_combine_with_drops_scales_by_kept_weight():
    g = _golden("route_example_a.json")
    r = oracle.route(np.array(g["logits"], np.float32), None, g["k"], g["capacity"])
    x = _bf16(np.arange(-12, 12).reshape(4, 6))  # small integers: 0.75 x is exact
    Xp = oracle.dispatch(x, g["k"], r["row_slot"])
    y = wl.bf16_bits_to_f32(oracle.combine(Xp, 4, g["k"], r["slot_row"], r["w"]))
    ref = wl.bf16_bits_to_f32(x) * np.array(g["identity_expert_output_scale"],
                                            np.float32)[:, None]
    assert np.array_equal(y, ref)


def test_dispatch_groups_rows_by_expert_in_token_order():
    g = _golden("route_example_a.json")
    r = oracle.route(np.array(g["logits"], np.float32), None, g["k"], g["capacity"])
    x = np.arange(4 * 3, dtype=np.float32).reshape(4, 3)
    Xp = oracle.dispatch(x, g["k"], r["row_slot"])
    # rows: e0 <- t1; e1 <- t0, t2; e2 <- t0, t1; e3 <- t2, t3
    assert (Xp[:, 0] / 3).astype(int).tolist() == [1, 0, 2, 0, 1, 2, 3]


def test_combine_fp32_weighted_sum_closed_form():
    rng = np.random.default_rng(6)
    T, d, k, R = 20, 7, 2, 40
    Yp = rng.standard_normal((R, d)).astype(np.float32)
    sr = rng.permutation(R).astype(np.int32).reshape(T, k)
    sr[3, 1] = -1
    w = rng.uniform(0, 1, (T, k)).astype(np.float32)
    y = oracle.combine(Yp, T, k, sr, w)
    ref = np.zeros((T, d))
    for t in range(T):
        for j in range(k):
            if sr[t, j] >= 0:
                ref[t] += float(w[t, j]) * Yp[sr[t, j]].astype(np.float64)
    np.testing.assert_allclose(y, ref.astype(np.float32), rtol=1e-6, atol=1e-7)


# ----------------------------------------------------------------- expert FFN --
def _groups(E, sizes):
    return np.array([0] + np.cumsum(sizes).tolist(), np.int32)


def test_ffn_negative_first_layer_gives_zero():
    rng = np.random.default_rng(7)
    E, d, F = 2, 16, 24
    Xp = _bf16(np.abs(rng.standard_normal((10, d))) + 0.1)
    W1 = _bf16(-np.abs(rng.standard_normal((E, F, d))) - 0.01)
    W2 = _bf16(rng.standard_normal((E, d, F)))
    Yp, H = oracle.expert_ffn(Xp, W1, W2, _groups(E, [4, 6]), want_h=True)
    assert not wl.bf16_bits_to_f32(H).any() and not wl.bf16_bits_to_f32(Yp).any()


def test_ffn_identity_weights_reproduce_input():
    rng = np.random.default_rng(8)
    E, d = 3, 32
    Xp = _bf16(np.abs(rng.standard_normal((12, d))))
    I = _bf16(np.broadcast_to(np.eye(d, dtype=np.float32), (E, d, d)))
    Yp = oracle.expert_ffn(Xp, I, I, _groups(E, [5, 0, 7]))
    assert np.array_equal(Yp, Xp)


def test_ffn_matches_matmul_when_relu_is_inactive_fp32():
    # Non-negative inputs and weights: ReLU is the identity and the expert is
    # two library matmuls.  d != F and distinct experts catch a transposed
    # weight or a wrong expert index.
    rng = np.random.default_rng(9)
    E, d, F = 3, 24, 40
    sizes = [5, 9, 4]
    Xp = rng.uniform(0, 1, (sum(sizes), d)).astype(np.float32)
    W1 = rng.uniform(0, 1, (E, F, d)).astype(np.float32)
    W2 = rng.uniform(0, 1, (E, d, F)).astype(np.float32)
    off = _groups(E, sizes)
    Yp, H = oracle.expert_ffn(Xp, W1, W2, off, want_h=True)
    for e in range(E):
        xe = Xp[off[e]:off[e + 1]].astype(np.float64)
        he = (xe @ W1[e].astype(np.float64).T).astype(np.float32)  # stored fp32 h
        ye = he.astype(np.float64) @ W2[e].astype(np.float64).T
        np.testing.assert_allclose(H[off[e]:off[e + 1]], he, rtol=1e-6)
        np.testing.assert_allclose(Yp[off[e]:off[e + 1]], ye, rtol=1e-6)


def test_ffn_relu_matches_matmul_with_clamp_fp32():
    rng = np.random.default_rng(10)
    E, d, F = 2, 20, 36
    sizes = [6, 5]
    Xp = rng.standard_normal((11, d)).astype(np.float32)
    W1 = rng.standard_normal((E, F, d)).astype(np.float32)
    W2 = rng.standard_normal((E, d, F)).astype(np.float32)
    off = _groups(E, sizes)
    Yp = oracle.expert_ffn(Xp, W1, W2, off)
    for e in range(E):
        xe = Xp[off[e]:off[e + 1]].astype(np.float64)
        he = np.maximum(xe @ W1[e].astype(np.float64).T, 0).astype(np.float32)
        ye = he.astype(np.float64) @ W2[e].astype(np.float64).T
        np.testing.assert_allclose(Yp[off[e]:off[e + 1]], ye, rtol=1e-5, atol=1e-6)


def test_ffn_bf16_positive_homogeneity_is_exact():
    # ReLU(2v) = 2 ReLU(v) and bf16 rounding commutes with scaling by 2.
    rng = np.random.default_rng(11)
    E, d, F = 2, 32, 48
    x = rng.standard_normal((8, d)).astype(np.float32)
    W1 = _bf16(rng.standard_normal((E, F, d)) / 6)
    W2 = _bf16(rng.standard_normal((E, d, F)) / 7)
    off = _groups(E, [3, 5])
    y1 = wl.bf16_bits_to_f32(oracle.expert_ffn(_bf16(x), W1, W2, off))
    y2 = wl.bf16_bits_to_f32(oracle.expert_ffn(_bf16(2 * x), W1, W2, off))
    assert np.array_equal(2 * y1, y2)


def test_ffn_rows_equals_grouped():
    rng = np.random.default_rng(12)
    E, d, F = 3, 16, 24
    Xp = _bf16(rng.standard_normal((9, d)))
    W1 = _bf16(rng.standard_normal((E, F, d)) / 4)
    W2 = _bf16(rng.standard_normal((E, d, F)) / 5)
    off = _groups(E, [2, 3, 4])
    Yp, H = oracle.expert_ffn(Xp, W1, W2, off, want_h=True)
    experts = np.repeat(np.arange(E), [2, 3, 4])
    Y2, H2 = oracle.expert_ffn_rows(Xp, experts, W1, W2, want_h=True)
    assert np.array_equal(Yp, Y2) and np.array_equal(H, H2)


# ---------------------------------------------------------------------- gate --
@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_gate_matches_matmul(dtype):
    rng = np.random.default_rng(13)
    T, d, E = 17, 45, 6
    x = rng.standard_normal((T, d)).astype(np.float32)
    Wg = rng.standard_normal((E, d)).astype(np.float32)
    if dtype == "bf16":
        x, Wg = _bf16(x), _bf16(Wg)
        xf, wf = wl.bf16_bits_to_f32(x), wl.bf16_bits_to_f32(Wg)
    else:
        xf, wf = x, Wg
    got = oracle.gate(x, Wg)
    ref = (xf.astype(np.float64) @ wf.astype(np.float64).T)
    ulp = np.spacing(np.abs(ref).astype(np.float32))
    assert np.all(np.abs(got - ref) <= ulp)


# ---------------------------------------------------------------- popularity --
def test_popularity_golden():
    g = _golden("popularity_example.json")
    hist = np.zeros((g["W"], g["E"]), np.int32)
    for step, (c, exp) in enumerate(zip(g["counts"], g["after_step"])):
        mean, hot = oracle.popularity_update(np.array(c, np.int32), hist, step, g["P"])
        assert mean.tolist() == exp["mean"], step
        assert hot.tolist() == exp["hot"], step
        n = min(step + 1, g["W"])
        assert (mean * n).tolist() == exp["sum"]


def test_popularity_resume_from_copied_state_is_identical():
    rng = np.random.default_rng(14)
    E, W, P = 10, 4, 3
    counts = rng.integers(0, 50, (9, E)).astype(np.int32)
    hist = np.zeros((W, E), np.int32)
    outs = [oracle.popularity_update(counts[s], hist, s, P) for s in range(9)]
    hist2 = np.zeros((W, E), np.int32)
    for s in range(5):
        oracle.popularity_update(counts[s], hist2, s, P)
    saved = hist2.copy()
    resumed = np.zeros((W, E), np.int32)
    resumed[:] = saved
    for s in range(5, 9):
        mean, hot = oracle.popularity_update(counts[s], resumed, s, P)
        assert np.array_equal(mean, outs[s][0]) and np.array_equal(hot, outs[s][1])


def test_popularity_mean_is_window_average_closed_form():
    rng = np.random.default_rng(15)
    E, W, P = 7, 3, 7
    counts = rng.integers(0, 1000, (6, E)).astype(np.int32)
    hist = np.zeros((W, E), np.int32)
    for s in range(6):
        mean, hot = oracle.popularity_update(counts[s], hist, s, P)
        lo = max(0, s + 1 - W)
        sums = counts[lo:s + 1].astype(np.int64).sum(0)
        n = s + 1 - lo
        assert np.array_equal(mean, (sums.astype(np.float32) / np.float32(n)))
        assert hot.tolist() == sorted(range(E), key=lambda e: (-sums[e], e))


@pytest.mark.parametrize("dtype,eps,y_bits_if_unrounded", [
    ("bf16", 2.0 ** -8, 0x4041),   # 3 + 3*2^-8 rounds up to 3 + 2^-6
    ("f32", 2.0 ** -24, None),
])
def test_ffn_hidden_activation_is_stored_at_storage_precision(dtype, eps, y_bits_if_unrounded):
    # Hand-worked: x = [1, 1]; every hidden unit is 1 + eps, a tie that rounds
    # to 1.0 at the storage precision; three such units summed by W2 = [1,1,1]
    # give exactly 3.0.  Without the storage rounding of H the sum is
    # 3 + 3 eps, which rounds to the next value above 3.
    d, F = 2, 3
    x = np.array([[1.0, 1.0]], np.float32)
    W1 = np.array([[[1.0, eps]] * F], np.float32)
    W2 = np.ones((1, d, F), np.float32)
    off = np.array([0, 1], np.int32)
    if dtype == "bf16":
        x, W1, W2 = _bf16(x), _bf16(W1), _bf16(W2)
        Yp, H = oracle.expert_ffn(x, W1, W2, off, want_h=True)
        assert H.tolist() == [[0x3F80] * F]
        assert Yp.tolist() == [[0x4040] * d]
        assert y_bits_if_unrounded != 0x4040
    else:
        Yp, H = oracle.expert_ffn(x, W1, W2, off, want_h=True)
        assert H.tolist() == [[1.0] * F]
        assert Yp.tolist() == [[3.0] * d]
        assert float(np.float32(3.0 + 3.0 * eps)) != 3.0


# ------------------------------------------- cross-layer correlation forecast --
def test_correlation_golden():
    g = _golden("correlation_example.json")
    C = np.zeros((g["E"], g["E"]), np.int32)
    oracle.correlation_update(np.array(g["ids_prev"]), np.array(g["ids_next"]), C)
    assert C.tolist() == g["C"]
    pred, hot = oracle.popularity_forecast(np.array(g["pop_prev"]), C, g["k_prev"],
                                           g["k_next"], 2)
    assert pred.tolist() == g["pred"] and hot.tolist() == g["hot_P2"]
    pred, _ = oracle.popularity_forecast(np.array(g["same_batch_pop"]), C, g["k_prev"],
                                         g["k_next"], 0)
    assert pred.tolist() == g["same_batch_pred"]


def _layer_ids(rng, T, E, k):
    return np.argsort(rng.random((T, E)), axis=1)[:, :k].astype(np.int32)


@pytest.mark.parametrize("E,k_prev,k_next", [(8, 2, 2), (16, 1, 3), (5, 5, 1), (32, 4, 8)])
def test_correlation_counts_brute_force_and_accumulate(E, k_prev, k_next):
    rng = np.random.default_rng(E * 10 + k_prev)
    T = 157
    a, b = _layer_ids(rng, T, E, k_prev), _layer_ids(rng, T, E, k_next)
    C = np.full((E, E), 3, np.int32)  # accumulates into what is there
    oracle.correlation_update(a, b, C)
    ref = np.full((E, E), 3, np.int64)
    for t in range(T):
        for i in a[t]:
            for h in b[t]:
                ref[i, h] += 1
    assert np.array_equal(C, ref)


@pytest.mark.parametrize("E,k_prev,k_next", [(8, 2, 2), (16, 1, 3), (12, 3, 1), (64, 2, 4)])
def test_forecast_from_same_batch_reproduces_next_layer_counts(E, k_prev, k_next):
    # With pop_prev the same batch's previous-layer counts, the forecast is
    # exactly the next layer's counts: sum_i C[i][h] = k_prev * counts_next[h].
    rng = np.random.default_rng(E + 7 * k_next)
    T = 400
    a, b = _layer_ids(rng, T, E, k_prev), _layer_ids(rng, T, E, k_next)
    C = np.zeros((E, E), np.int32)
    oracle.correlation_update(a, b, C)
    counts_prev = np.bincount(a.ravel(), minlength=E).astype(np.float32)
    counts_next = np.bincount(b.ravel(), minlength=E)
    pred, _ = oracle.popularity_forecast(counts_prev, C, k_prev, k_next, 0)
    np.testing.assert_allclose(pred, counts_next, rtol=2e-7)


def test_forecast_is_linear_and_ignores_unseen_rows():
    rng = np.random.default_rng(3)
    E, T = 10, 200
    a = _layer_ids(rng, T, E - 2, 2)  # experts 8 and 9 never chosen at layer j
    b = _layer_ids(rng, T, E, 2)
    C = np.zeros((E, E), np.int32)
    oracle.correlation_update(a, b, C)
    p1 = rng.uniform(0, 5, E).astype(np.float32)
    p2 = rng.uniform(0, 5, E).astype(np.float32)
    f1, _ = oracle.popularity_forecast(p1, C, 2, 2, 0)
    f2, _ = oracle.popularity_forecast(p2, C, 2, 2, 0)
    f12, _ = oracle.popularity_forecast(p1 + p2, C, 2, 2, 0)
    np.testing.assert_allclose(f12, f1 + f2, rtol=1e-5)
    bump = p1.copy()
    bump[8:] += 100.0  # popularity on rows with no observed pairs adds nothing
    fb, _ = oracle.popularity_forecast(bump, C, 2, 2, 0)
    assert np.array_equal(fb, f1)
    np.testing.assert_allclose(f1.sum(), p1[:8].sum(), rtol=1e-5)  # k_next / k_prev = 1


# ------------------------------------------------------ load-balancing loss --
def test_aux_loss_golden():
    g = _golden("aux_loss_example.json")
    lg = np.array(g["logits"], np.float32)
    r = oracle.route(lg, None, g["k"])
    assert r["counts"].tolist() == g["counts"]
    loss, P = oracle.aux_loss(lg, None, g["k"], r["counts"])
    np.testing.assert_allclose(P, g["prob_mean"], rtol=1e-7)
    np.testing.assert_allclose(loss, g["loss"], rtol=1e-7)


@pytest.mark.parametrize("E,k", [(8, 2), (16, 1), (5, 5)])
def test_aux_loss_uniform_router_is_one(E, k):
    T = 96
    lg = np.full((T, E), 0.37, np.float32)  # every probability 1/E, any routing
    r = oracle.route(lg, None, k)
    loss, P = oracle.aux_loss(lg, None, k, r["counts"])
    np.testing.assert_allclose(P, 1.0 / E, rtol=1e-7)
    np.testing.assert_allclose(loss, 1.0, rtol=1e-6)


def test_aux_loss_is_invariant_to_relabelling_experts():
    rng = np.random.default_rng(4)
    T, E, k = 300, 12, 3
    lg = rng.standard_normal((T, E)).astype(np.float32)
    b = rng.standard_normal(E).astype(np.float32)
    perm = rng.permutation(E)
    r = oracle.route(lg, b, k)
    r2 = oracle.route(lg[:, perm], b[perm], k)
    l1, P1 = oracle.aux_loss(lg, b, k, r["counts"])
    l2, P2 = oracle.aux_loss(lg[:, perm], b[perm], k, r2["counts"])
    np.testing.assert_allclose(l1, l2, rtol=1e-6)
    np.testing.assert_allclose(P1[perm], P2, rtol=1e-6)


def test_aux_loss_collapsed_router_approaches_e():
    T, E = 64, 8
    lg = np.zeros((T, E), np.float32)
    lg[:, 3] = 40.0  # softmax ~ one-hot on expert 3, every token routed there
    r = oracle.route(lg, None, 1)
    loss, P = oracle.aux_loss(lg, None, 1, r["counts"])
    np.testing.assert_allclose(loss, E, rtol=1e-6)
    np.testing.assert_allclose(P.sum(), 1.0, rtol=1e-6)


def test_aux_loss_probabilities_include_the_routing_bias():
    # zero logits, bias (ln 3, 0): every token has p = (3/4, 1/4) and is routed
    # to expert 0, so loss = 2 * (1 * 3/4 + 0 * 1/4) = 1.5
    lg = np.zeros((10, 2), np.float32)
    b = np.array([np.log(3.0), 0.0], np.float32)
    r = oracle.route(lg, b, 1)
    loss, P = oracle.aux_loss(lg, b, 1, r["counts"])
    np.testing.assert_allclose(P, [0.75, 0.25], rtol=1e-7)
    np.testing.assert_allclose(loss, 1.5, rtol=1e-7)
