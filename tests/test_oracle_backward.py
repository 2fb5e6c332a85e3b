"""Pins of the oracle's backward pass (CPU only): adjoint identities, library
matmul special cases, closed forms of the renormalised softmax, and central
finite differences of the oracle's own forward pass on a tiny fp32 layer."""
import numpy as np
import pytest

import oracle
from routing_dispatch_expert_fp32_b200 import workloads as wl


def _route(rng, T, E, k, cap=0):
    return oracle.route(rng.standard_normal((T, E)).astype(np.float32), None, k, cap)


def test_dispatch_backward_is_the_adjoint_of_dispatch():
    rng = np.random.default_rng(1)
    T, d, E, k = 50, 12, 6, 2
    r = _route(rng, T, E, k, cap=12)  # with drops
    x = rng.standard_normal((T, d)).astype(np.float32)
    G = rng.standard_normal((len(r["row_slot"]), d)).astype(np.float32)
    lhs = float(np.sum(oracle.dispatch(x, k, r["row_slot"]).astype(np.float64) * G))
    rhs = float(np.sum(x.astype(np.float64) * oracle.dispatch_backward(G, T, k, r["slot_row"])))
    np.testing.assert_allclose(lhs, rhs, rtol=1e-5)


def test_combine_backward_rows_are_the_adjoint_of_combine_and_dw_is_a_dot():
    rng = np.random.default_rng(2)
    T, d, E, k = 40, 9, 5, 3
    r = _route(rng, T, E, k, cap=20)
    R = len(r["row_slot"])
    Yp = rng.standard_normal((R, d)).astype(np.float32)
    g = rng.standard_normal((T, d)).astype(np.float32)
    y = oracle.combine(Yp, T, k, r["slot_row"], r["w"])
    dw, dYp = oracle.combine_backward(g, Yp, k, r["slot_row"], r["w"])
    lhs = float(np.sum(y.astype(np.float64) * g))
    rhs = float(np.sum(Yp.astype(np.float64) * dYp))
    np.testing.assert_allclose(lhs, rhs, rtol=1e-5)
    # d/dw of sum(g * y) is the dot of g with the slot's row; dropped slots: 0
    for t in range(T):
        for j in range(k):
            row = r["slot_row"][t, j]
            ref = 0.0 if row < 0 else float(np.dot(g[t].astype(np.float64), Yp[row]))
            np.testing.assert_allclose(dw[t, j], ref, rtol=1e-6, atol=1e-6)


def test_expert_ffn_backward_matches_matmuls_fp32():
    rng = np.random.default_rng(3)
    E, d, F = 3, 10, 14
    sizes = [4, 0, 7]
    off = np.array([0] + np.cumsum(sizes).tolist(), np.int32)
    R = off[-1]
    Xp = rng.standard_normal((R, d)).astype(np.float32)
    W1 = rng.standard_normal((E, F, d)).astype(np.float32)
    W2 = rng.standard_normal((E, d, F)).astype(np.float32)
    Yp, H = oracle.expert_ffn(Xp, W1, W2, off, want_h=True)
    dYp = rng.standard_normal((R, d)).astype(np.float32)
    dH, dXp, dW1, dW2 = oracle.expert_ffn_backward(Xp, H, dYp, W1, W2, off)
    for e in range(E):
        a, b = off[e], off[e + 1]
        h = H[a:b].astype(np.float64)
        g = dYp[a:b].astype(np.float64)
        dh = (g @ W2[e].astype(np.float64)) * (h > 0)
        np.testing.assert_allclose(dH[a:b], dh, rtol=1e-5, atol=1e-6)
        np.testing.assert_allclose(dXp[a:b], dh @ W1[e].astype(np.float64), rtol=1e-5, atol=1e-5)
        np.testing.assert_allclose(dW2[e], g.T @ h, rtol=1e-5, atol=1e-5)
        np.testing.assert_allclose(dW1[e], dh.T @ Xp[a:b].astype(np.float64), rtol=1e-5,
                                   atol=1e-5)
    assert not dW1[1].any() and not dW2[1].any()  # empty group


def test_route_backward_closed_forms():
    rng = np.random.default_rng(4)
    T, E, k = 30, 7, 3
    r = _route(rng, T, E, k)
    dw = rng.standard_normal((T, k)).astype(np.float32)
    dl, db = oracle.route_backward(r["ids"], r["w"], dw, E)
    np.testing.assert_allclose(dl.sum(1), 0.0, atol=1e-6)        # softmax shift invariance
    np.testing.assert_allclose(db, dl.sum(0), rtol=1e-5, atol=1e-6)
    for t in range(T):                                             # unselected experts: 0
        mask = np.ones(E, bool)
        mask[r["ids"][t]] = False
        assert not dl[t, mask].any()
    dl2, _ = oracle.route_backward(r["ids"], r["w"], np.full((T, k), 2.5, np.float32), E)
    assert np.abs(dl2).max() < 1e-6                                # equal upstream: no change
    # k = 2, two experts: dz_0 = w0 w1 (dw0 - dw1)
    r2 = oracle.route(np.array([[0.3, -0.4]], np.float32), None, 2)
    dl3, _ = oracle.route_backward(r2["ids"], r2["w"], np.array([[1.0, -2.0]], np.float32), 2)
    w0, w1 = r2["w"][0]
    np.testing.assert_allclose(dl3[0, r2["ids"][0, 0]], w0 * w1 * 3.0, rtol=1e-6)


def _tiny_layer(seed):
    """fp32 layer whose routing gap and ReLU pre-activations stay clear of the
    finite-difference step (the first seed from `seed` that qualifies)."""
    for s in range(seed, seed + 500):
        rng = np.random.default_rng(s)
        T, d, E, k, F = 6, 5, 4, 2, 7
        x = rng.standard_normal((T, d)).astype(np.float32)
        Wg = (rng.standard_normal((E, d)) * 0.7).astype(np.float32)
        W1 = rng.standard_normal((E, F, d)).astype(np.float32)
        W2 = rng.standard_normal((E, d, F)).astype(np.float32)
        bias = np.array([0.3, -0.2, 0.1, 0.0], np.float32)
        fwd = oracle.layer(x, Wg, W1, W2, bias, k)
        z = np.sort(fwd["logits"] + bias, 1)[:, ::-1]
        e_of_row = np.searchsorted(fwd["offsets"], np.arange(len(fwd["Xp"])), "right") - 1
        pre = np.einsum("rc,rfc->rf", fwd["Xp"].astype(np.float64), W1[e_of_row])
        if (z[:, k - 1] - z[:, k]).min() > 0.05 and np.abs(pre).min() > 0.02:
            return x, Wg, W1, W2, bias, k
    raise AssertionError("no qualifying seed")


def _loss(x, Wg, W1, W2, bias, k, g):
    y = oracle.layer(x, Wg, W1, W2, bias, k)["y"]
    return float(np.sum(y.astype(np.float64) * g))


@pytest.mark.parametrize("seed", [5, 1000])
def test_layer_backward_matches_central_finite_differences(seed):
    x, Wg, W1, W2, bias, k = _tiny_layer(seed)
    fwd = oracle.layer(x, Wg, W1, W2, bias, k)
    g = np.random.default_rng(seed + 100).standard_normal(fwd["y"].shape).astype(np.float32)
    grads = oracle.layer_backward(x, Wg, W1, W2, bias, k, fwd, g)
    eps = 1e-3
    rng = np.random.default_rng(seed + 200)
    for name, arr in [("dx", x), ("dWg", Wg), ("dW1", W1), ("dW2", W2)]:
        for _ in range(6):
            idx = tuple(rng.integers(0, n) for n in arr.shape)
            plus, minus = arr.copy(), arr.copy()
            plus[idx] += eps
            minus[idx] -= eps
            args = dict(x=x, Wg=Wg, W1=W1, W2=W2)
            key = {"dx": "x", "dWg": "Wg", "dW1": "W1", "dW2": "W2"}[name]
            args_p, args_m = dict(args), dict(args)
            args_p[key], args_m[key] = plus, minus
            fd = (_loss(args_p["x"], args_p["Wg"], args_p["W1"], args_p["W2"], bias, k, g) -
                  _loss(args_m["x"], args_m["Wg"], args_m["W1"], args_m["W2"], bias, k, g)) / (2 * eps)
            an = float(grads[name][idx])
            assert abs(fd - an) <= 2e-3 * max(1.0, abs(an)), (name, idx, fd, an)
    # bias gradient
    for e in range(len(bias)):
        bp, bm = bias.copy(), bias.copy()
        bp[e] += eps
        bm[e] -= eps
        fd = (_loss(x, Wg, W1, W2, bp, k, g) - _loss(x, Wg, W1, W2, bm, k, g)) / (2 * eps)
        assert abs(fd - grads["dbias"][e]) <= 2e-3 * max(1.0, abs(grads["dbias"][e]))
