"""Backward pass on the GPU against the oracle's backward.

Small shapes (several 128-row, 256-column and 64-deep tiles, ragged tails,
empty groups, spare rows filled with NaN that must not leak into any sum) are
compared element by element; the full-size workloads are compared on sampled
rows and sampled hidden units, each computed by the oracle from the same
seeded inputs.  Index and exactly-rounded outputs (dlogits, dYp) are compared
bit for bit; fp32-accumulated ones within the bounds stated at each check."""
import numpy as np
import pytest
import torch

import oracle
from parity import as_f64, assert_close, dev, host
from routing_dispatch_expert_fp32_b200 import workloads as wl

pytestmark = pytest.mark.gpu

NAN_BF16 = np.uint16(0x7FC0)


def rand(shape, scale, dtype, seed):
    a = np.random.default_rng(seed).standard_normal(shape, dtype=np.float32) * np.float32(scale)
    return wl.to_bf16_bits(a) if dtype == "bf16" else a


def relu_rand(shape, dtype, seed):
    a = np.maximum(np.random.default_rng(seed).standard_normal(shape, dtype=np.float32), 0)
    return wl.to_bf16_bits(a) if dtype == "bf16" else a


def padded(a, rows, fill_nan=True):
    """a's rows followed by spare rows (NaN, or zero) up to `rows`, on the device."""
    out = np.empty((rows,) + a.shape[1:], a.dtype)
    out[: a.shape[0]] = a
    out[a.shape[0]:] = NAN_BF16 if a.dtype == np.uint16 else np.float32(np.nan)
    if not fill_nan:
        out[a.shape[0]:] = 0
    return dev(out)


def tdt(dtype):
    return torch.bfloat16 if dtype == "bf16" else torch.float32


# ------------------------------------------------------------ expert FFN ----
def run_ffn_bwd(moe, Xp, H, dYp, W1, W2, offsets, Rmax, dtype, weight_grads=True):
    E, F, d = W1.shape
    R = Xp.shape[0]
    dH = torch.zeros(Rmax, F, dtype=tdt(dtype), device="cuda")
    dXp = torch.zeros(Rmax, d, dtype=tdt(dtype), device="cuda")
    dW1 = torch.full((E, F, d), 7.0, device="cuda") if weight_grads else None
    dW2 = torch.full((E, d, F), 7.0, device="cuda") if weight_grads else None
    moe.moe_expert_ffn_backward(padded(Xp, Rmax), padded(H, Rmax), padded(dYp, Rmax), dev(W1),
                                dev(W2), dev(offsets), dH, dXp, dW1, dW2)
    torch.cuda.synchronize()
    assert moe.moe_device_error() == 0
    out = dict(dH=host(dH), dXp=host(dXp))
    if weight_grads:
        out.update(dW1=host(dW1), dW2=host(dW2))
    assert R <= Rmax
    return out


@pytest.mark.parametrize("sizes,d,F,dtype,rmax", [
    ([0, 1, 127, 128, 129, 300], 200, 328, "bf16", 0),
    ([5, 0, 260], 64, 256, "bf16", 0),
    ([513], 1024, 512, "bf16", 0),
    ([3, 77, 131, 0, 0, 256, 1], 136, 520, "bf16", 0),
    ([0, 0, 0], 64, 64, "bf16", 0),
    ([64, 65, 63], 8, 16, "bf16", 0),
    ([40, 90, 1], 64, 128, "f32", 0),
    ([0, 65, 200], 72, 100, "f32", 0),
    # row capacity >= 1024 per group: the input gradients take the 2-CTA pair
    # tiles (weights read N-major), with ragged groups, an empty one, N and K
    # not multiples of the tile
    ([1000, 1300], 200, 328, "bf16", 2048),
    ([0, 700, 1900, 3], 136, 520, "bf16", 4096),
    ([2048], 64, 256, "bf16", 2048),
    # 460 groups of 0-4 rows: more than three waves of 128-row tiles, so both
    # input gradients take the 1-CTA kernel
    ([int(v) for v in np.random.default_rng(7).integers(0, 5, 460)], 256, 256, "bf16", 0),
])
def test_ffn_backward_small_shapes_elementwise(moe, sizes, d, F, dtype, rmax):
    E, R = len(sizes), sum(sizes)
    offsets = np.array([0] + np.cumsum(sizes).tolist(), np.int32)
    Xp = rand((R, d), 1.0, dtype, 11)
    H = relu_rand((R, F), dtype, 12)
    dYp = rand((R, d), 1.0, dtype, 13)
    W1 = rand((E, F, d), d ** -0.5, dtype, 14)
    W2 = rand((E, d, F), F ** -0.5, dtype, 15)
    Rmax = max(R + 37, rmax)
    g = run_ffn_bwd(moe, Xp, H, dYp, W1, W2, offsets, Rmax, dtype)
    tol = dict(max_abs_frac=1e-4, mean_rel=1e-5) if dtype == "f32" else {}
    if R:
        dHr, dXr, dW1r, dW2r = oracle.expert_ffn_backward(Xp, H, dYp, W1, W2, offsets)
        assert_close(g["dH"][:R], dHr, "dH", **tol)
        # the ReLU's gradient: exactly zero wherever the stored activation is not positive
        assert not as_f64(g["dH"][:R])[as_f64(H) <= 0].any()
        assert_close(g["dXp"][:R], dXr, "dXp", **tol)
        for e in range(E):
            if sizes[e]:
                assert_close(g["dW1"][e], dW1r[e], f"dW1[{e}]", **tol)
                assert_close(g["dW2"][e], dW2r[e], f"dW2[{e}]", **tol)
    for e in range(E):  # an expert without rows gets zero weight gradients
        if not sizes[e]:
            assert not g["dW1"][e].any() and not g["dW2"][e].any()
    assert not g["dH"][R:].any() and not g["dXp"][R:].any()  # spare rows untouched


def test_ffn_backward_input_grads_only(moe):
    sizes, d, F = [100, 0, 300], 128, 256
    E, R = len(sizes), sum(sizes)
    offsets = np.array([0] + np.cumsum(sizes).tolist(), np.int32)
    Xp, H, dYp = rand((R, d), 1, "bf16", 1), relu_rand((R, F), "bf16", 2), rand((R, d), 1, "bf16", 3)
    W1, W2 = rand((E, F, d), 0.1, "bf16", 4), rand((E, d, F), 0.1, "bf16", 5)
    g = run_ffn_bwd(moe, Xp, H, dYp, W1, W2, offsets, R, "bf16", weight_grads=False)
    dHr, dXr, _, _ = oracle.expert_ffn_backward(Xp, H, dYp, W1, W2, offsets)
    assert_close(g["dH"], dHr, "dH")
    assert_close(g["dXp"], dXr, "dXp")


def test_ffn_backward_identity_weights(moe):
    """W1 = W2 = I and H > 0: dH = dYp and dXp = dYp exactly; dW2 = dYp^T H."""
    E, d = 2, 128
    sizes = [70, 190]
    R = sum(sizes)
    offsets = np.array([0, 70, 260], np.int32)
    I = wl.to_bf16_bits(np.broadcast_to(np.eye(d, dtype=np.float32), (E, d, d)).copy())
    H = wl.to_bf16_bits(np.abs(np.random.default_rng(0).standard_normal((R, d))) + 0.5)
    dYp = rand((R, d), 1.0, "bf16", 1)
    Xp = rand((R, d), 1.0, "bf16", 2)
    g = run_ffn_bwd(moe, Xp, H, dYp, I, I, offsets, R, "bf16")
    assert np.array_equal(g["dH"], dYp) and np.array_equal(g["dXp"], dYp)


# --------------------------------------------------- combine / dispatch ----
def small_route(T, E, k, capacity, seed):
    logits = np.random.default_rng(seed).standard_normal((T, E), dtype=np.float32)
    return oracle.route(logits, None, k, capacity)


@pytest.mark.parametrize("T,E,k,cap,d,dtype", [
    (300, 8, 2, 60, 200, "bf16"),
    (257, 16, 4, 0, 64, "bf16"),
    (100, 4, 1, 10, 1032, "bf16"),
    (300, 8, 2, 60, 68, "f32"),
    (64, 40, 32, 30, 16, "bf16"),
])
def test_combine_backward(moe, T, E, k, cap, d, dtype):
    r = small_route(T, E, k, cap, 5)
    R = int(r["offsets"][-1])
    Yp = rand((R, d), 1.0, dtype, 6)
    dy = rand((T, d), 1.0, dtype, 7)
    dw_r, dYp_r = oracle.combine_backward(dy, Yp, k, r["slot_row"], r["w"])
    Rmax = R + 9
    dYp = torch.zeros(Rmax, d, dtype=tdt(dtype), device="cuda")
    dw = torch.full((T, k), 5.0, device="cuda")
    moe.moe_combine_backward(dev(dy), padded(Yp, Rmax), k, dev(r["slot_row"]), dev(r["w"]), dw, dYp)
    torch.cuda.synchronize()
    assert moe.moe_device_error() == 0
    # dYp = w * dy rounded once: bit for bit
    assert np.array_equal(host(dYp)[:R], dYp_r)
    assert not host(dYp)[R:].any()
    # dw = <dy, Yp[row]>: fp32 lanes over d / 32 terms each, then a 5-level tree
    g = host(dw)
    kept = r["slot_row"] >= 0
    assert not g[~kept].any()
    t_idx, j_idx = np.nonzero(kept)
    rows = r["slot_row"][t_idx, j_idx]
    mag = np.abs(as_f64(dy)[t_idx] * as_f64(Yp)[rows]).sum(axis=1)
    bound = (d / 32 + 6) * 2.0 ** -24 * mag + 1e-30
    assert np.all(np.abs(g[kept].astype(np.float64) - dw_r[kept]) <= bound)


@pytest.mark.parametrize("T,E,k,cap,d,dtype", [
    (300, 8, 2, 60, 200, "bf16"), (257, 16, 4, 0, 64, "f32"), (64, 40, 32, 30, 16, "bf16")])
def test_dispatch_backward(moe, T, E, k, cap, d, dtype):
    r = small_route(T, E, k, cap, 8)
    R = int(r["offsets"][-1])
    dXp = rand((R, d), 1.0, dtype, 9)
    ref = oracle.dispatch_backward(dXp, T, k, r["slot_row"])
    dx = torch.full((T, d), 3.0, dtype=tdt(dtype), device="cuda")
    moe.moe_dispatch_backward(padded(dXp, R + 4), k, dev(r["slot_row"]), dx)
    torch.cuda.synchronize()
    g = as_f64(host(dx))
    # fp32 running sum of at most k terms, rounded once to dtype
    ulp = 2.0 ** -7 if dtype == "bf16" else 2.0 ** -23
    mag = np.zeros((T, d))
    for j in range(k):
        rows = r["slot_row"][:, j]
        mag[rows >= 0] += np.abs(as_f64(dXp)[rows[rows >= 0]])
    assert np.all(np.abs(g - as_f64(ref)) <= ulp * np.abs(as_f64(ref)) + k * 2.0 ** -24 * mag
                  + 1e-30)
    dropped_all = (r["slot_row"] < 0).all(axis=1)
    assert not g[dropped_all].any()


# ------------------------------------------------------------- routing -----
@pytest.mark.parametrize("T,E,k,cap", [(1000, 64, 4, 70), (300, 8, 2, 0), (77, 1000, 32, 3),
                                       (513, 256, 8, 20), (1, 2, 1, 0)])
def test_route_backward(moe, T, E, k, cap):
    r = small_route(T, E, k, cap, 21)
    dw = np.random.default_rng(22).standard_normal((T, k), dtype=np.float32)
    dw[r["slot_row"] < 0] = 0  # as the combine backward leaves dropped slots
    dl_r, db_r = oracle.route_backward(r["ids"], r["w"], dw, E)
    dl = torch.full((T, E), 9.0, device="cuda")
    db = torch.full((E,), 9.0, device="cuda")
    ws = torch.empty(moe.moe_route_workspace_size(T, E, k), dtype=torch.uint8, device="cuda")
    moe.moe_route_backward(dev(r["ids"]), dev(r["w"]), dev(dw), E, dl, db, ws)
    torch.cuda.synchronize()
    assert moe.moe_device_error() == 0
    assert np.array_equal(host(dl).view(np.uint32), dl_r.view(np.uint32))  # bit for bit
    # dbias: the fp32 dlogits summed in double (chunks of 256 tokens, then chunks)
    bound = 2.0 ** -23 * np.abs(dl_r.astype(np.float64)).sum(axis=0) + 2.0 ** -24 * np.abs(db_r)
    assert np.all(np.abs(host(db).astype(np.float64) - db_r) <= bound + 1e-37)
    # without dbias no workspace is needed
    dl2 = torch.zeros(T, E, device="cuda")
    moe.moe_route_backward(dev(r["ids"]), dev(r["w"]), dev(dw), E, dl2, None, None)
    torch.cuda.synchronize()
    assert torch.equal(dl, dl2)


# ---------------------------------------------------------------- gate -----
@pytest.mark.parametrize("T,d,E,dtype", [(300, 200, 8, "bf16"), (513, 64, 256, "bf16"),
                                         (100, 136, 16, "f32"), (5, 8, 3, "f32"),
                                         (4097, 1024, 16, "bf16"), (2000, 72, 1000, "f32"),
                                         (300, 64, 12, "bf16"), (70, 2056, 64, "bf16")])
def test_gate_backward(moe, T, d, E, dtype):
    x = rand((T, d), 1.0, dtype, 31)
    Wg = rand((E, d), d ** -0.5, dtype, 32)
    dl = np.random.default_rng(33).standard_normal((T, E), dtype=np.float32)
    dl[np.random.default_rng(34).random((T, E)) < 0.7] = 0  # sparse, as routing leaves it
    dx0 = rand((T, d), 1.0, dtype, 35)
    dx_r, dWg_r = oracle.gate_backward(x, Wg, dl, dx0)
    dx = dev(dx0)
    dWg = torch.full((E, d), 4.0, device="cuda")
    ws = torch.empty(max(moe.moe_gate_backward_workspace_size(T, d, E, tdt(dtype)), 1),
                     dtype=torch.uint8, device="cuda")
    moe.moe_gate_backward(dev(x), dev(Wg), dev(dl), dx, dWg, ws)
    torch.cuda.synchronize()
    tol = dict(max_abs_frac=1e-5, mean_rel=1e-6) if dtype == "f32" else {}
    assert_close(host(dx), dx_r, "dx", **tol)
    assert_close(host(dWg), dWg_r, "dWg", max_abs_frac=1e-4, mean_rel=1e-5)


# ---------------------------------------------------------- whole layer ----
@pytest.mark.parametrize("T,d,E,k,F,cap,dtype", [
    (512, 128, 8, 2, 256, 160, "bf16"),
    (300, 64, 16, 4, 200, 0, "bf16"),
    (512, 64, 8, 2, 128, 0, "f32"),
])
def test_layer_backward_every_element(moe, T, d, E, k, F, cap, dtype):
    rng = np.random.default_rng(41)
    x = rand((T, d), 1.0, dtype, 42)
    Wg = rand((E, d), d ** -0.5, dtype, 43)
    W1 = rand((E, F, d), d ** -0.5, dtype, 44)
    W2 = rand((E, d, F), F ** -0.5, dtype, 45)
    bias = (0.5 * rng.standard_normal(E)).astype(np.float32)
    dy = rand((T, d), 1.0, dtype, 46)
    logits = oracle.gate(x, Wg)  # both sides route the same scores
    fwd = oracle.layer(x, Wg, W1, W2, bias, k, cap, logits=logits)
    ref = oracle.layer_backward(x, Wg, W1, W2, bias, k, fwd, dy)
    layer = moe.MoELayer(T, d, E, k, F, tdt(dtype), capacity=cap)
    xd, Wgd, W1d, W2d = dev(x), dev(Wg), dev(W1), dev(W2)
    layer.forward(xd, Wgd, W1d, W2d, dev(bias), logits=dev(logits))
    g = layer.backward(dev(dy), xd, Wgd, W1d, W2d)
    torch.cuda.synchronize()
    assert moe.moe_device_error() == 0
    R = int(fwd["offsets"][-1])
    assert np.array_equal(host(layer.slot_row), fwd["slot_row"])
    tol = dict(max_abs_frac=1e-4, mean_rel=1e-5) if dtype == "f32" else {}
    assert_close(host(layer.dw), ref["dw"], "dw", **tol)
    assert_close(host(layer.dH)[:R], ref["dH"], "dH", **tol)
    for name in ["dlogits", "dbias", "dx", "dW1", "dW2", "dWg"]:
        assert_close(host(g[name]), ref[name], name, **tol)


# ------------------------------------------------- full-size, sampled ------
def groups_to_check(offsets, rng):
    sizes = np.diff(offsets)
    nz = [e for e in np.argsort(sizes, kind="stable") if sizes[e] > 0]
    return list(dict.fromkeys([nz[0], nz[len(nz) // 2], nz[-1], int(rng.choice(nz))]))


@pytest.mark.parametrize("name", ["skewed_drops", "multistep_window", "fine_grained"])
def test_ffn_backward_full_size_sampled(moe, name):
    w = wl.WORKLOADS[name]
    rng = np.random.default_rng(51)
    r = oracle.route(wl.router_logits(w), wl.zipf_bias(w), w.k, w.capacity)
    offsets = r["offsets"]
    Rmax = w.T * w.k
    inp = wl.ffn_backward_inputs(w, Rmax)
    weights = wl.make_weights(w)
    W1, W2 = weights["W1"], weights["W2"]
    E, F, d = W1.shape
    dH = torch.zeros(Rmax, F, dtype=torch.bfloat16, device="cuda")
    dXp = torch.zeros(Rmax, d, dtype=torch.bfloat16, device="cuda")
    dW1 = torch.empty(E, F, d, device="cuda")
    dW2 = torch.empty(E, d, F, device="cuda")
    moe.moe_expert_ffn_backward(dev(inp["Xp"]), dev(inp["H"]), dev(inp["dYp"]), dev(W1), dev(W2),
                                dev(offsets), dH, dXp, dW1, dW2)
    torch.cuda.synchronize()
    assert moe.moe_device_error() == 0
    for e in groups_to_check(offsets, rng):
        a, b = int(offsets[e]), int(offsets[e + 1])
        # rows: first, last and random rows of the group, all hidden units
        rows = np.unique(np.concatenate([[a, b - 1], rng.integers(a, b, 4)]))
        rd = torch.from_numpy(rows).cuda()
        one = np.array([0, len(rows)], np.int32)
        dHr, dXr, _, _ = oracle.expert_ffn_backward(
            inp["Xp"][rows], inp["H"][rows], inp["dYp"][rows], W1[e:e + 1], W2[e:e + 1], one)
        assert_close(host(dH[rd]), dHr, f"dH rows e={e}")
        assert_close(host(dXp[rd]), dXr, f"dXp rows e={e}")
        # weight gradients: every row of the group, sampled hidden units fs
        fs = np.unique(np.concatenate([[0, F - 1], rng.choice(F, 2, replace=False)]))
        grp = np.array([0, b - a], np.int32)
        _, _, dW1r, dW2r = oracle.expert_ffn_backward(
            inp["Xp"][a:b], inp["H"][a:b][:, fs], inp["dYp"][a:b], W1[e][fs][None],
            np.ascontiguousarray(W2[e][:, fs])[None], grp)
        assert_close(host(dW1[e][torch.from_numpy(fs).cuda()]), dW1r[0], f"dW1 e={e}")
        assert_close(host(dW2[e][:, torch.from_numpy(fs).cuda()]), dW2r[0], f"dW2 e={e}")
    # experts without rows: zero weight gradients
    for e in np.nonzero(np.diff(offsets) == 0)[0]:
        assert not dW1[e].any() and not dW2[e].any()


# ------------------------------------------------------------ edge cases ---
def test_backward_edge_cases(moe):
    E, d, F, k = 3, 64, 128, 2
    W1 = dev(rand((E, F, d), 0.1, "bf16", 61))
    W2 = dev(rand((E, d, F), 0.1, "bf16", 62))
    z = lambda *s: torch.zeros(*s, dtype=torch.bfloat16, device="cuda")
    # no rows at all: zero weight gradients
    dW1 = torch.full((E, F, d), 3.0, device="cuda")
    dW2 = torch.full((E, d, F), 3.0, device="cuda")
    offsets = dev(np.zeros(E + 1, np.int32))
    moe.moe_expert_ffn_backward(z(0, d), z(0, F), z(0, d), W1, W2, offsets, z(0, F), z(0, d),
                                dW1, dW2)
    torch.cuda.synchronize()
    assert not dW1.any() and not dW2.any()
    # no tokens: route backward gives dbias = 0, gate backward dWg = 0
    ws = torch.empty(max(moe.moe_route_workspace_size(0, E, k), 1), dtype=torch.uint8,
                     device="cuda")
    db = torch.full((E,), 2.0, device="cuda")
    e_ids = torch.zeros(0, k, dtype=torch.int32, device="cuda")
    e_f = torch.zeros(0, k, device="cuda")
    moe.moe_route_backward(e_ids, e_f, e_f, E, torch.zeros(0, E, device="cuda"), db, ws)
    dWg = torch.full((E, d), 2.0, device="cuda")
    moe.moe_gate_backward(z(0, d), z(E, d), torch.zeros(0, E, device="cuda"), z(0, d), dWg)
    torch.cuda.synchronize()
    assert not db.any() and not dWg.any()
    # one token, k = E: every expert chosen once, weights sum to one
    T1 = 1
    r = oracle.route(np.array([[0.3, -1.0, 2.0]], np.float32), None, E, 0)
    dw = np.array([[0.5, -2.0, 1.0]], np.float32)
    dl_r, db_r = oracle.route_backward(r["ids"], r["w"], dw, E)
    dl = torch.empty(T1, E, device="cuda")
    db = torch.empty(E, device="cuda")
    ws = torch.empty(moe.moe_route_workspace_size(T1, E, E), dtype=torch.uint8, device="cuda")
    moe.moe_route_backward(dev(r["ids"]), dev(r["w"]), dev(dw), E, dl, db, ws)
    torch.cuda.synchronize()
    assert np.array_equal(host(dl).view(np.uint32), dl_r.view(np.uint32))
    assert abs(float(host(dl).astype(np.float64).sum())) < 1e-6  # softmax gradient sums to zero
    assert moe.moe_device_error() == 0
