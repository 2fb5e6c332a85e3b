"""The whole layer on the GPU (gate, route, popularity, dispatch, expert FFN,
combine) against the oracle, on the five workloads at full size.

Routing is checked bit for bit against the oracle routing the GPU's own fp32
logits (the gate itself is checked against the oracle's logits separately).
Expert outputs and the layer output are checked on sampled rows / tokens the
oracle computes one by one; properties that hold at any size (counts sum, the
permutation, identity experts) are checked on every element."""
import numpy as np
import pytest
import torch

import oracle
from parity import assert_close, dev, host
from routing_dispatch_expert_fp32_b200 import workloads as wl

pytestmark = pytest.mark.gpu


def sample_rows(offsets, counts_rank, rng, per_group=3, groups=8):
    """Rows of the hottest and coldest non-empty groups: first, last, random."""
    E = len(offsets) - 1
    sizes = np.diff(offsets)
    order = [e for e in np.argsort(-sizes, kind="stable") if sizes[e] > 0]
    pick = order[: groups // 2] + order[-(groups // 2):]
    rows = []
    for e in dict.fromkeys(pick):
        a, b = int(offsets[e]), int(offsets[e + 1])
        rows += [a, b - 1] + rng.integers(a, b, per_group).tolist()
    return np.unique(np.array(rows, np.int64))


def check_layer(moe, w: wl.Workload, step_inputs, weights, layer, rng, n_tokens=48):
    x, bias = step_inputs["x"], step_inputs["bias"]
    xd = dev(x)
    dW = {k: dev(v) for k, v in weights.items()}
    logits_in = dev(step_inputs["logits"]) if w.logits_direct else None
    layer.forward(xd, dW.get("Wg"), dW.get("W1"), dW.get("W2"),
                  None if bias is None else dev(bias), logits=logits_in)
    torch.cuda.synchronize()
    assert moe.moe_device_error() == 0
    logits = step_inputs["logits"] if w.logits_direct else host(layer.logits)
    if not w.logits_direct:  # gate vs oracle on sampled tokens
        toks = rng.choice(w.T, min(w.T, 64), replace=False)
        ref = oracle.gate(x[toks], weights["Wg"])
        assert np.abs(logits[toks] - ref).max() <= 1e-5 * np.abs(ref).max() + 1e-6
    r = oracle.route(logits, bias, w.k, w.capacity)
    R = int(r["offsets"][-1])
    for name in ["ids", "counts", "kept", "offsets", "slot_row"]:
        assert np.array_equal(host(getattr(layer, name)), r[name]), name
    assert np.array_equal(host(layer.row_slot)[:R], r["row_slot"])
    assert int(host(layer.n_dropped)[0]) == r["n_dropped"]
    np.testing.assert_allclose(host(layer.w), r["w"], rtol=4e-6, atol=1e-8)
    # dispatch: every row is its token's input (a byte copy), checked in blocks
    blk = 1 << 14
    for a in range(0, R, blk):
        b = min(R, a + blk)
        assert np.array_equal(host(layer.Xp[a:b]), x[r["row_slot"][a:b] // w.k]), (a, b)
    y = host(layer.y)
    if w.identity_experts:
        toks = rng.choice(w.T, 256, replace=False)
        Yt = x[np.repeat(toks, w.k)]  # identity experts: slot (t, j) outputs x[t]
        sr = np.where(r["slot_row"][toks] >= 0,
                      np.arange(len(toks) * w.k, dtype=np.int32).reshape(-1, w.k), -1)
        ref_y = oracle.combine(Yt, len(toks), w.k, sr.astype(np.int32), r["w"][toks])
        assert_close(y[toks], ref_y, "y")
        if r["n_dropped"] == 0:
            # value-equal; a -0.0 input comes back as +0.0 (the weighted sum
            # starts from +0.0), exactly as in the oracle
            assert np.array_equal(wl.bf16_bits_to_f32(y), wl.bf16_bits_to_f32(x))
        return r
    # expert outputs on sampled rows
    rows = sample_rows(r["offsets"], None, rng)
    expert_of_row = np.searchsorted(r["offsets"], rows, side="right") - 1
    rows_d = torch.from_numpy(rows).cuda()
    # the rows' inputs are their tokens' x (the dispatch check above)
    Yr, Hr = oracle.expert_ffn_rows(x[r["row_slot"][rows] // w.k], expert_of_row, weights["W1"],
                                    weights["W2"], want_h=True)
    assert_close(host(layer.H[rows_d]), Hr, "H rows")
    assert_close(host(layer.Yp[rows_d]), Yr, "Yp rows")
    # layer output on sampled tokens, recomputed from x by the oracle
    toks = np.unique(np.concatenate([rng.choice(w.T, n_tokens, replace=False), [0, w.T - 1]]))
    ys = []
    for t in toks:
        rows_t = [s for s in r["slot_row"][t] if s >= 0]
        acc = np.zeros((1, w.d), np.float64)
        if rows_t:
            es = np.searchsorted(r["offsets"], rows_t, side="right") - 1
            Yt = oracle.expert_ffn_rows(np.repeat(x[t:t + 1], len(rows_t), 0), es,
                                        weights["W1"], weights["W2"])
            # oracle combine of this token's expert outputs
            sr = np.full((1, w.k), -1, np.int32)
            sr[0, [j for j in range(w.k) if r["slot_row"][t, j] >= 0]] = np.arange(len(rows_t))
            ys.append(oracle.combine(Yt, 1, w.k, sr, r["w"][t:t + 1])[0])
        else:
            ys.append(np.zeros(w.d, x.dtype))
    assert_close(y[toks], np.stack(ys), "y tokens")
    return r


def make_layer(moe, w):
    tdt = torch.bfloat16 if w.dtype == "bf16" else torch.float32
    return moe.MoELayer(w.T, w.d, w.E, w.k, w.F, tdt, capacity=w.capacity, W=w.W, P=w.P,
                        identity_experts=w.identity_experts)


@pytest.mark.parametrize("name", ["tiny_fp32", "skewed_drops", "fine_grained"])
def test_layer_single_step(moe, name):
    w = wl.WORKLOADS[name]
    weights = wl.make_weights(w)
    layer = make_layer(moe, w)
    r = check_layer(moe, w, wl.make_step(w, 0), weights, layer, np.random.default_rng(1))
    if name == "skewed_drops":
        assert r["n_dropped"] > 0  # the Zipf bias overloads the hot experts


def test_layer_tiny_fp32_every_element(moe):
    w = wl.WORKLOADS["tiny_fp32"]
    weights, inp = wl.make_weights(w), wl.make_step(w, 0)
    layer = make_layer(moe, w)
    layer.forward(dev(inp["x"]), dev(weights["Wg"]), dev(weights["W1"]), dev(weights["W2"]))
    torch.cuda.synchronize()
    ref = oracle.layer(inp["x"], weights["Wg"], weights["W1"], weights["W2"], None, w.k, 0,
                       logits=host(layer.logits))
    assert_close(host(layer.y), ref["y"], "y", max_abs_frac=1e-5, mean_rel=1e-6)


def test_layer_multistep_window(moe):
    w = wl.WORKLOADS["multistep_window"]
    weights = wl.make_weights(w)
    layer = make_layer(moe, w)
    hist_ref = np.zeros((w.W, w.E), np.int32)
    rng = np.random.default_rng(2)
    prev_hot = None
    for s in range(w.steps):
        r = check_layer(moe, w, wl.make_step(w, s), weights, layer, rng, n_tokens=16)
        mean_ref, hot_ref = oracle.popularity_update(r["counts"], hist_ref, s, w.P)
        assert np.array_equal(host(layer.mean), mean_ref), s
        assert np.array_equal(host(layer.hot)[: w.P], hot_ref), s
        assert np.array_equal(host(layer.hist), hist_ref), s
        prev_hot = hot_ref
    assert prev_hot is not None


@pytest.mark.parametrize("T", wl.BW_SWEEP_TOKENS)
@pytest.mark.parametrize("s", [None, 1.5])
def test_layer_bw_sweep_identity_experts(moe, T, s):
    w = wl.WORKLOADS["bw_sweep"].with_(T=T, zipf_s=s)
    layer = make_layer(moe, w)
    check_layer(moe, w, wl.make_step(w, 0), {}, layer, np.random.default_rng(3))


def test_graph_replay_matches_eager_and_advances_the_window(moe):
    w = wl.tiny("graph", T=700, d=256, E=12, k=2, F=384, zipf_s=1.1, W=3, P=4)
    weights = {k: dev(v) for k, v in wl.make_weights(w).items()}
    steps = [wl.make_step(w, s) for s in range(5)]
    x = dev(steps[0]["x"]).clone()
    bias = dev(steps[0]["bias"]).clone()
    graphed, eager = make_layer(moe, w), make_layer(moe, w)
    g = graphed.capture(x, weights["Wg"], weights["W1"], weights["W2"], bias)
    graphed.hist.zero_()
    graphed.step_dev.zero_()  # the capture's warm-up forward advanced the window
    hist_ref = np.zeros((w.W, w.E), np.int32)
    for s, inp in enumerate(steps):
        x.copy_(dev(inp["x"]))
        g.replay()
        y_e = eager.forward(dev(inp["x"]), weights["Wg"], weights["W1"], weights["W2"], bias)
        torch.cuda.synchronize()
        assert torch.equal(graphed.y, y_e), s
        r = oracle.route(host(graphed.logits), host(bias), w.k, w.capacity)
        mean_ref, hot_ref = oracle.popularity_update(r["counts"], hist_ref, s, w.P)
        assert np.array_equal(host(graphed.mean), mean_ref), s
        assert np.array_equal(host(graphed.hot)[: w.P], hot_ref), s
    assert int(graphed.step_dev.item()) == len(steps)
    assert moe.moe_device_error() == 0


def test_concurrent_batches_match_sequential_and_keep_one_window(moe):
    """capture_concurrent: three batches of one layer on three streams in one
    graph give each batch the same output as running it alone, and their
    popularity updates enter the shared window in list order."""
    w = wl.tiny("conc", T=600, d=256, E=12, k=2, F=384, zipf_s=1.1, W=8, P=4)
    weights = {k: dev(v) for k, v in wl.make_weights(w).items()}
    steps = [wl.make_step(w, s) for s in range(3)]
    xs = [dev(s["x"]) for s in steps]
    bias = dev(steps[0]["bias"])
    layers = [make_layer(moe, w) for _ in range(3)]
    for L in layers[1:]:
        L.share_popularity(layers[0])
    calls = [dict(x=x, Wg=weights["Wg"], W1=weights["W1"], W2=weights["W2"], bias=bias)
             for x in xs]
    g = moe.capture_concurrent(layers, calls)
    layers[0].hist.zero_()
    layers[0].step_dev.zero_()  # the capture's warm-up advanced the window
    for _ in range(2):
        g.replay()
    torch.cuda.synchronize()
    alone = make_layer(moe, w)
    hist_ref = np.zeros((w.W, w.E), np.int32)
    s = 0
    for rep in range(2):
        for i, x in enumerate(xs):
            y = alone.forward(x, weights["Wg"], weights["W1"], weights["W2"], bias)
            torch.cuda.synchronize()
            if rep == 1:
                assert torch.equal(layers[i].y, y), i
            r = oracle.route(host(alone.logits), host(bias), w.k, w.capacity)
            mean_ref, hot_ref = oracle.popularity_update(r["counts"], hist_ref, s, w.P)
            s += 1
    assert int(layers[0].step_dev.item()) == 6
    assert np.array_equal(host(layers[0].hist), hist_ref)
    assert np.array_equal(host(layers[0].mean), mean_ref)
    assert np.array_equal(host(layers[0].hot)[: w.P], hot_ref)
    assert moe.moe_device_error() == 0


def _expert_subset(offsets, rng, n_hot=4, n_cold=4, n_rand=8):
    """The n_hot largest and n_cold smallest non-empty groups and n_rand others."""
    sizes = np.diff(offsets)
    nonempty = [int(e) for e in np.argsort(-sizes, kind="stable") if sizes[e] > 0]
    pick = nonempty[:n_hot] + nonempty[-n_cold:]
    rest = [e for e in nonempty if e not in pick]
    pick += rng.choice(rest, min(n_rand, len(rest)), replace=False).tolist()
    return sorted(set(pick))


@pytest.mark.parametrize("name", ["multistep_window", "fine_grained"])
def test_every_row_of_sixteen_experts_at_full_size(moe, name):
    """Every expert-output row (H and Yp) of 16 experts -- the 4 hottest, the 4
    coldest and 8 seeded others -- at the workload's full size, in the launch
    configuration bench.py times, against the oracle (its OpenMP build on all
    host cores), each expert on its own scale."""
    w = wl.WORKLOADS[name]
    weights = wl.make_weights(w)
    inp = wl.make_step(w, 0)
    layer = make_layer(moe, w)
    dW = {k: dev(v) for k, v in weights.items()}
    layer.forward(dev(inp["x"]), dW["Wg"], dW["W1"], dW["W2"], dev(inp["bias"]))
    torch.cuda.synchronize()
    assert moe.moe_device_error() == 0
    offsets = host(layer.offsets)
    row_slot = host(layer.row_slot)
    # the routing itself is checked bit for bit by the single-step tests; here
    # the grouped rows are taken as the GPU laid them out
    experts = _expert_subset(offsets, np.random.default_rng(11))
    assert len(experts) >= 16
    rows = np.concatenate([np.arange(offsets[e], offsets[e + 1]) for e in experts])
    expert_of_row = np.repeat(experts, [offsets[e + 1] - offsets[e] for e in experts])
    rows_d = torch.from_numpy(rows).cuda()
    H, Y = host(layer.H[rows_d]), host(layer.Yp[rows_d])
    xr = inp["x"][row_slot[rows] // w.k]
    try:
        oracle.use_parallel(True)
        Yr, Hr = oracle.expert_ffn_rows(xr, expert_of_row, weights["W1"], weights["W2"],
                                        want_h=True)
    finally:
        oracle.use_parallel(False)
    start = 0
    for e in experts:
        n = int(offsets[e + 1] - offsets[e])
        sl = slice(start, start + n)
        assert_close(H[sl], Hr[sl], f"H expert {e} ({n} rows)")
        assert_close(Y[sl], Yr[sl], f"Yp expert {e} ({n} rows)")
        start += n
