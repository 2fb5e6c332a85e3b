"""The fused expert path (moe_expert_ffn_gather + unweighted combine) on the GPU
against the oracle.

The first GEMM gathers its rows from x by row_slot (no Xp), the second applies
each row's gate weight, and output decode sums the rows.  Small shapes with
ragged groups, drops and empty experts are compared element by element; the
full-size bf16 workloads through MoELayer(fused=True) on routing (bit for bit),
sampled hidden rows and sampled layer outputs, as in the unfused layer test."""
import numpy as np
import pytest
import torch

import oracle
from parity import assert_close, dev, host
from routing_dispatch_expert_fp32_b200 import workloads as wl
from test_gpu_layer import sample_rows

pytestmark = pytest.mark.gpu


def rand(shape, scale, seed):
    a = np.random.default_rng(seed).standard_normal(shape, dtype=np.float32) * np.float32(scale)
    return wl.to_bf16_bits(a)


@pytest.mark.parametrize("T,d,E,k,F,cap", [
    (300, 200, 8, 2, 328, 60),     # drops, ragged tiles in every dimension
    (513, 1024, 16, 2, 512, 0),
    (64, 136, 40, 4, 520, 3),      # most experts empty or tiny, heavy drops
    (1000, 64, 4, 1, 256, 0),
])
def test_fused_ffn_and_combine_match_oracle(moe, T, d, E, k, F, cap):
    x = rand((T, d), 1.0, 1)
    W1 = rand((E, F, d), d ** -0.5, 2)
    W2 = rand((E, d, F), F ** -0.5, 3)
    logits = np.random.default_rng(4).standard_normal((T, E), dtype=np.float32)
    r = oracle.route(logits, None, k, cap)
    R = int(r["offsets"][-1])
    Rmax = T * k
    row_slot = np.full(Rmax, -7, np.int32)  # rows past R are never read
    row_slot[:R] = r["row_slot"]
    Xp = oracle.dispatch(x, k, r["row_slot"])
    Y_ref, H_ref = oracle.expert_ffn(Xp, W1, W2, r["offsets"], want_h=True)
    y_ref = oracle.combine(Y_ref, T, k, r["slot_row"], r["w"])
    xd, W1d, W2d = dev(x), dev(W1), dev(W2)
    offd, rsd, wd = dev(r["offsets"]), dev(row_slot), dev(r["w"])
    H = torch.zeros(Rmax, F, dtype=torch.bfloat16, device="cuda")
    Yp = torch.zeros(Rmax, d, dtype=torch.bfloat16, device="cuda")
    # unweighted: the same H and Yp as the unfused expert FFN
    moe.moe_expert_ffn_gather(xd, k, rsd, None, W1d, W2d, offd, H, Yp)
    torch.cuda.synchronize()
    assert moe.moe_device_error() == 0
    if R:
        assert_close(host(H)[:R], H_ref, "H")
        assert_close(host(Yp)[:R], Y_ref, "Yp")
    assert not host(H)[R:].any() and not host(Yp)[R:].any()
    # weighted rows, then output decode as a plain sum
    moe.moe_expert_ffn_gather(xd, k, rsd, wd, W1d, W2d, offd, H, Yp)
    y = torch.empty(T, d, dtype=torch.bfloat16, device="cuda")
    moe.moe_combine(Yp, k, dev(r["slot_row"]), None, y)
    torch.cuda.synchronize()
    assert moe.moe_device_error() == 0
    assert_close(host(y), y_ref, "y")
    dropped_all = (r["slot_row"] < 0).all(axis=1)
    assert not host(y)[dropped_all].any()


def test_fused_identity_experts_reproduce_rows(moe):
    """W1 = W2 = I, x >= 0: H and the unweighted Yp are the gathered rows, bit for bit."""
    T, d, E, k = 200, 128, 3, 2
    x = wl.to_bf16_bits(np.abs(np.random.default_rng(0).standard_normal((T, d))))
    I = wl.to_bf16_bits(np.broadcast_to(np.eye(d, dtype=np.float32), (E, d, d)).copy())
    r = oracle.route(np.random.default_rng(1).standard_normal((T, E), dtype=np.float32), None, k, 0)
    R = int(r["offsets"][-1])
    H = torch.zeros(R, d, dtype=torch.bfloat16, device="cuda")
    Yp = torch.zeros(R, d, dtype=torch.bfloat16, device="cuda")
    moe.moe_expert_ffn_gather(dev(x), k, dev(r["row_slot"]), None, dev(I), dev(I),
                              dev(r["offsets"]), H, Yp)
    torch.cuda.synchronize()
    rows = x[r["row_slot"] // k]
    assert np.array_equal(host(H), rows) and np.array_equal(host(Yp), rows)


def test_fused_bad_row_slot_is_flagged_not_followed(moe):
    T, d, E, k, F = 64, 64, 2, 1, 64
    x = rand((T, d), 1.0, 5)
    W1, W2 = rand((E, F, d), 0.1, 6), rand((E, d, F), 0.1, 7)
    row_slot = np.arange(T, dtype=np.int32)
    row_slot[5] = T * k + 100  # out of range: read as a zero row, flagged
    offsets = np.array([0, 32, 64], np.int32)
    H = torch.zeros(T, F, dtype=torch.bfloat16, device="cuda")
    Yp = torch.zeros(T, d, dtype=torch.bfloat16, device="cuda")
    moe.moe_device_error()
    moe.moe_expert_ffn_gather(dev(x), k, dev(row_slot), None, dev(W1), dev(W2), dev(offsets), H,
                              Yp)
    torch.cuda.synchronize()
    assert moe.moe_device_error() & moe.MOE_DEVERR_ROW_INDEX
    assert not host(H)[5].any()


@pytest.mark.parametrize("name", ["skewed_drops", "multistep_window", "fine_grained"])
def test_fused_layer_full_size_sampled(moe, name):
    w = wl.WORKLOADS[name]
    weights = wl.make_weights(w)
    inp = wl.make_step(w, 0)
    x, bias = inp["x"], inp["bias"]
    layer = moe.MoELayer(w.T, w.d, w.E, w.k, w.F, torch.bfloat16, capacity=w.capacity, W=w.W,
                         P=w.P, fused=True)
    layer.forward(dev(x), dev(weights["Wg"]), dev(weights["W1"]), dev(weights["W2"]),
                  None if bias is None else dev(bias))
    torch.cuda.synchronize()
    assert moe.moe_device_error() == 0
    # routing of the layer's own fp32 logits (the gate is checked in the unfused test)
    r = oracle.route(host(layer.logits), bias, w.k, w.capacity)
    for n in ["ids", "counts", "offsets", "slot_row"]:
        assert np.array_equal(host(getattr(layer, n)), r[n]), n
    rng = np.random.default_rng(2)
    rows = sample_rows(r["offsets"], None, rng)
    er = np.searchsorted(r["offsets"], rows, side="right") - 1
    _, Hr = oracle.expert_ffn_rows(x[r["row_slot"][rows] // w.k], er, weights["W1"],
                                   weights["W2"], want_h=True)
    assert_close(host(layer.H[torch.from_numpy(rows).cuda()]), Hr, "H rows")
    toks = np.unique(np.concatenate([rng.choice(w.T, 48, replace=False), [0, w.T - 1]]))
    ys = []
    for t in toks:
        kept = [j for j in range(w.k) if r["slot_row"][t, j] >= 0]
        if not kept:
            ys.append(np.zeros(w.d, x.dtype))
            continue
        es = np.searchsorted(r["offsets"], r["slot_row"][t, kept], side="right") - 1
        Yt = oracle.expert_ffn_rows(np.repeat(x[t:t + 1], len(kept), 0), es, weights["W1"],
                                    weights["W2"])
        sr = np.full((1, w.k), -1, np.int32)
        sr[0, kept] = np.arange(len(kept))
        ys.append(oracle.combine(Yt, 1, w.k, sr, r["w"][t:t + 1])[0])
    assert_close(host(layer.y)[toks], np.stack(ys), "y tokens")
