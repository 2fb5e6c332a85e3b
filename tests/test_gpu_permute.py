"""moe_dispatch / moe_combine on the GPU against the oracle: dispatch is a
byte copy (bit-exact); combine within the output tolerance; identity experts
reproduce x exactly when nothing is dropped."""
import numpy as np
import pytest
import torch

import oracle
from parity import assert_close, dev, host
from routing_dispatch_expert_fp32_b200 import workloads as wl

pytestmark = pytest.mark.gpu


def routed(T, E, k, cap, seed, bias_s=None):
    rng = np.random.default_rng(seed)
    logits = rng.standard_normal((T, E), dtype=np.float32)
    bias = None
    if bias_s is not None:
        bias = wl.zipf_bias(wl.tiny("p", T=T, d=8, E=E, k=k, F=8, zipf_s=bias_s, index=seed))
    return oracle.route(logits, bias, k, cap)


def make_x(T, d, dtype, seed):
    x = np.random.default_rng(seed).standard_normal((T, d), dtype=np.float32)
    return wl.to_bf16_bits(x) if dtype == "bf16" else x


@pytest.mark.parametrize("T,d,E,k,cap,dtype", [
    (512, 64, 8, 2, 0, "f32"), (4096, 1024, 16, 2, 640, "bf16"), (1, 8, 4, 2, 0, "bf16"),
    (333, 264, 12, 3, 50, "bf16"), (100, 4, 6, 2, 10, "f32"), (2048, 7168, 128, 4, 0, "bf16"),
    (5000, 520, 32, 8, 0, "bf16"),
])
def test_dispatch_and_combine_match_oracle(moe, T, d, E, k, cap, dtype):
    r = routed(T, E, k, cap, seed=T + d)
    x = make_x(T, d, dtype, seed=d)
    R = int(r["offsets"][-1])
    Rmax = T * k
    tdt = torch.bfloat16 if dtype == "bf16" else torch.float32
    sr, w = dev(r["slot_row"]), dev(r["w"])
    Xp = torch.zeros(Rmax, d, dtype=tdt, device="cuda")
    moe.moe_dispatch(dev(x), k, sr, Xp)
    Xp_ref = oracle.dispatch(x, k, r["row_slot"])
    got = host(Xp)
    assert np.array_equal(got[:R], Xp_ref)
    assert not got[R:].any(), "rows past R were written"
    # combine with arbitrary expert outputs
    Yp = (np.random.default_rng(1).standard_normal((Rmax, d), dtype=np.float32))
    Yp = wl.to_bf16_bits(Yp) if dtype == "bf16" else Yp
    y = torch.empty(T, d, dtype=tdt, device="cuda")
    moe.moe_combine(dev(Yp), k, sr, w, y)
    y_ref = oracle.combine(Yp, T, k, r["slot_row"], r["w"])
    assert_close(host(y), y_ref, "combine", max_abs_frac=1e-5 if dtype == "f32" else 1e-2,
                 mean_rel=1e-6 if dtype == "f32" else 5e-3)
    if dtype == "bf16":
        # Per element: fp32 accumulation of k terms errs by at most k * 2^-24 * S
        # (S = sum_j |w_j Yp_j|), and the two bf16 roundings differ by at most
        # one bf16 ulp, i.e. 2^-7 of the value.
        g, ref = wl.bf16_bits_to_f32(host(y)), wl.bf16_bits_to_f32(y_ref)
        Yf = wl.bf16_bits_to_f32(Yp).astype(np.float64)
        S = np.zeros((T, d))
        for j in range(k):
            rows = r["slot_row"][:, j]
            keep = rows >= 0
            S[keep] += np.abs(r["w"][keep, j, None] * Yf[rows[keep]])
        bound = 2.0 ** -7 * np.maximum(np.abs(ref), np.abs(g)) + k * 2.0 ** -23 * S
        assert np.all(np.abs(g - ref) <= bound)
    assert moe.moe_device_error() == 0


@pytest.mark.parametrize("T,bias_s", [(8192, None), (8192, 1.5), (16384, 1.5)])
def test_identity_experts_reproduce_x(moe, T, bias_s):
    d, E, k = 7168, 128, 4
    r = routed(T, E, k, 0, seed=T, bias_s=bias_s)
    x = make_x(T, d, "bf16", seed=3)
    Xp = torch.empty(T * k, d, dtype=torch.bfloat16, device="cuda")
    y = torch.empty(T, d, dtype=torch.bfloat16, device="cuda")
    xd = dev(x)
    moe.moe_dispatch(xd, k, dev(r["slot_row"]), Xp)
    moe.moe_combine(Xp, k, dev(r["slot_row"]), dev(r["w"]), y)
    assert torch.equal(y, xd)


def test_combine_dropped_tokens_get_zero_and_partial_weight(moe):
    import json, os
    from conftest import GOLDEN
    g = json.load(open(os.path.join(GOLDEN, "route_example_a.json")))
    r = oracle.route(np.array(g["logits"], np.float32), None, g["k"], g["capacity"])
    x = wl.to_bf16_bits(np.arange(-16, 16, dtype=np.float32).reshape(4, 8))
    Xp = torch.zeros(8, 8, dtype=torch.bfloat16, device="cuda")
    y = torch.empty(4, 8, dtype=torch.bfloat16, device="cuda")
    moe.moe_dispatch(dev(x), 2, dev(r["slot_row"]), Xp)
    moe.moe_combine(Xp, 2, dev(r["slot_row"]), dev(r["w"]), y)
    scale = np.array(g["identity_expert_output_scale"], np.float32)[:, None]
    ref = wl.bf16_bits_to_f32(x) * scale
    assert np.array_equal(wl.bf16_bits_to_f32(host(y)), ref)
    sr = r["slot_row"].copy()
    sr[2] = -1  # token 2 fully dropped
    moe.moe_combine(Xp, 2, dev(sr), dev(r["w"]), y)
    assert not wl.bf16_bits_to_f32(host(y))[2].any()


def test_out_of_range_rows_are_skipped_and_flagged(moe):
    moe.moe_device_error()  # clear
    T, d, k = 64, 64, 2
    x = dev(make_x(T, d, "bf16", 1))
    sr = np.arange(T * k, dtype=np.int32).reshape(T, k)
    sr[10, 1] = T * k + 5  # beyond R_max: must not be written
    sr[11, 0] = -9
    Xp = torch.zeros(T * k, d, dtype=torch.bfloat16, device="cuda")
    moe.moe_dispatch(x, k, dev(sr), Xp)
    bits = moe.moe_device_error()
    assert bits & moe.MOE_DEVERR_ROW_INDEX
    got = host(Xp)
    assert np.array_equal(got[0], host(x)[0])


def test_rejects_rows_not_multiple_of_16_bytes(moe):
    x = torch.zeros(4, 12, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(moe.MoeError):
        moe.moe_dispatch(x, 1, torch.zeros(4, 1, dtype=torch.int32, device="cuda"),
                         torch.zeros(4, 12, dtype=torch.bfloat16, device="cuda"))
