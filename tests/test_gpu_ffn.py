"""moe_expert_ffn and moe_gate on the GPU against the oracle.

Small shapes span several 128-row, 256-column and 64-deep tiles with ragged
tails and empty groups and are compared element by element; the full-size
workloads are compared on sampled rows (first, last and random rows of the
hottest and coldest groups)."""
import numpy as np
import pytest
import torch

import oracle
from parity import assert_close, dev, host
from routing_dispatch_expert_fp32_b200 import workloads as wl

pytestmark = pytest.mark.gpu


def rand(shape, scale, dtype, seed):
    a = np.random.default_rng(seed).standard_normal(shape, dtype=np.float32) * np.float32(scale)
    return wl.to_bf16_bits(a) if dtype == "bf16" else a


def run_ffn(moe, Xp, W1, W2, offsets, Rmax):
    E, F, d = W1.shape
    tdt = torch.bfloat16 if Xp.dtype == np.uint16 else torch.float32
    Xd = torch.zeros(Rmax, d, dtype=tdt, device="cuda")
    Xd[: Xp.shape[0]] = dev(Xp)
    H = torch.zeros(Rmax, F, dtype=tdt, device="cuda")
    Yp = torch.zeros(Rmax, d, dtype=tdt, device="cuda")
    moe.moe_expert_ffn(Xd, dev(W1), dev(W2), dev(offsets), H, Yp)
    torch.cuda.synchronize()
    return host(H), host(Yp)


@pytest.mark.parametrize("sizes,d,F,dtype", [
    ([0, 1, 127, 128, 129, 300], 200, 328, "bf16"),
    ([5, 0, 260], 64, 256, "bf16"),
    ([513], 1024, 512, "bf16"),
    ([3, 77, 131, 0, 0, 256, 1], 136, 520, "bf16"),
    ([0, 0, 0], 64, 64, "bf16"),
    ([40, 90, 1], 64, 128, "f32"),
    ([0, 65, 200], 72, 100, "f32"),
    # enough 128-row tiles (>= 3 waves) that the first GEMM stays on 1-CTA tiles
    ([1000, 1, 0, 1999, 1000], 64, 4096, "bf16"),
    # groups just under and over 16-, 64-, 128- and 256-row boundaries, K not a
    # multiple of 64, odd and even numbers of k-blocks
    ([1, 15, 16, 17, 63, 64, 65, 0, 255, 256, 257, 511, 513], 136, 384, "bf16"),
    ([1, 15, 16, 17, 63, 64, 65, 0, 255, 256, 257, 511, 513], 256, 640, "bf16"),
    ([3, 40, 0, 129, 300, 2], 192, 256, "bf16"),
    ([70, 5, 1, 33], 384, 128, "bf16"),
])
def test_ffn_small_shapes_elementwise(moe, sizes, d, F, dtype):
    E = len(sizes)
    R = sum(sizes)
    offsets = np.array([0] + np.cumsum(sizes).tolist(), np.int32)
    Xp = rand((R, d), 1.0, dtype, 1)
    W1 = rand((E, F, d), d ** -0.5, dtype, 2)
    W2 = rand((E, d, F), F ** -0.5, dtype, 3)
    Rmax = R + 37  # spare rows must stay untouched
    H, Yp = run_ffn(moe, Xp, W1, W2, offsets, Rmax)
    if R:
        Yr, Hr = oracle.expert_ffn(Xp, W1, W2, offsets, want_h=True)
        tol = dict(max_abs_frac=1e-5, mean_rel=1e-6) if dtype == "f32" else {}
        assert_close(H[:R], Hr, "H", **tol)
        assert_close(Yp[:R], Yr, "Yp", **tol)
    assert not H[R:].any() and not Yp[R:].any()
    assert moe.moe_device_error() == 0


@pytest.mark.parametrize("sizes,d,F", [
    ([0, 1, 17, 255, 256, 257, 600, 16], 256, 512),
    ([3, 700, 1, 0, 129], 200, 768),                  # K tail in the first GEMM
])
def test_ffn_dense_groups_elementwise(moe, sizes, d, F):
    """R_max >= 1024 rows per expert selects the 2-CTA kernels."""
    E = len(sizes)
    R = sum(sizes)
    offsets = np.array([0] + np.cumsum(sizes).tolist(), np.int32)
    Xp = rand((R, d), 1.0, "bf16", 11)
    W1 = rand((E, F, d), d ** -0.5, "bf16", 12)
    W2 = rand((E, d, F), F ** -0.5, "bf16", 13)
    Rmax = 1024 * E + 5
    H, Yp = run_ffn(moe, Xp, W1, W2, offsets, Rmax)
    Yr, Hr = oracle.expert_ffn(Xp, W1, W2, offsets, want_h=True)
    assert_close(H[:R], Hr, "H")
    assert_close(Yp[:R], Yr, "Yp")
    assert not H[R:].any() and not Yp[R:].any()
    assert moe.moe_device_error() == 0


@pytest.mark.parametrize("sizes,d,F", [
    ([1, 15, 16, 17, 63, 64, 65, 0, 127, 128, 129, 255, 256, 257, 3], 128, 256),
    ([40, 0, 129, 7, 300, 2, 16], 200, 512),          # K tail in the first GEMM
    ([5, 130, 61, 1, 0, 250], 512, 768),
])
def test_ffn_sparse_groups_with_many_tiles_elementwise(moe, sizes, d, F):
    """A row capacity of three or more waves of 128-row tiles (the sparse
    regime of the large workloads): 1-CTA tiles, many per CTA."""
    E = len(sizes)
    R = sum(sizes)
    offsets = np.array([0] + np.cumsum(sizes).tolist(), np.int32)
    Xp = rand((R, d), 1.0, "bf16", 21)
    W1 = rand((E, F, d), d ** -0.5, "bf16", 22)
    W2 = rand((E, d, F), F ** -0.5, "bf16", 23)
    Rmax = 60000
    H, Yp = run_ffn(moe, Xp, W1, W2, offsets, Rmax)
    Yr, Hr = oracle.expert_ffn(Xp, W1, W2, offsets, want_h=True)
    assert_close(H[:R], Hr, "H")
    assert_close(Yp[:R], Yr, "Yp")
    assert not H[R:].any() and not Yp[R:].any()
    assert moe.moe_device_error() == 0


def test_ffn_relu_kills_negative_first_layer(moe):
    E, d, F = 2, 128, 256
    Xp = wl.to_bf16_bits(np.abs(np.random.default_rng(0).standard_normal((300, d))) + 0.1)
    W1 = wl.to_bf16_bits(-np.abs(np.random.default_rng(1).standard_normal((E, F, d))) - 0.01)
    W2 = rand((E, d, F), 0.1, "bf16", 2)
    H, Yp = run_ffn(moe, Xp, W1, W2, np.array([0, 170, 300], np.int32), 300)
    assert not wl.bf16_bits_to_f32(H).any() and not wl.bf16_bits_to_f32(Yp).any()


def test_ffn_identity_weights_reproduce_input(moe):
    E, d = 3, 256
    Xp = wl.to_bf16_bits(np.abs(np.random.default_rng(0).standard_normal((400, d))))
    I = wl.to_bf16_bits(np.broadcast_to(np.eye(d, dtype=np.float32), (E, d, d)).copy())
    H, Yp = run_ffn(moe, Xp, I, I, np.array([0, 130, 131, 400], np.int32), 400)
    assert np.array_equal(Yp, Xp) and np.array_equal(H, Xp)


def test_ffn_bad_offsets_are_flagged_not_followed(moe):
    moe.moe_device_error()
    E, d, F = 3, 64, 64
    Xp = rand((100, d), 1.0, "bf16", 0)
    W1, W2 = rand((E, F, d), 0.1, "bf16", 1), rand((E, d, F), 0.1, "bf16", 2)
    run_ffn(moe, Xp, W1, W2, np.array([0, 60, 20, 100], np.int32), 100)  # decreasing
    assert moe.moe_device_error() & moe.MOE_DEVERR_OFFSETS
    run_ffn(moe, Xp, W1, W2, np.array([0, 60, 80, 500], np.int32), 100)  # beyond R_max
    assert moe.moe_device_error() & moe.MOE_DEVERR_OFFSETS


@pytest.mark.parametrize("T,d,E,dtype", [
    (512, 64, 8, "f32"), (4096, 1024, 16, "bf16"),        # CUDA-core gate (E <= 32)
    (333, 200, 6, "bf16"), (130, 64, 20, "f32"), (1001, 1024, 32, "bf16"), (7, 512, 1, "bf16"),
    (1000, 136, 300, "bf16"), (16384, 2048, 64, "bf16"),  # tensor-core gate
    (200, 4096, 32, "bf16"),                              # E <= 32 but Wg too big to stage
])
def test_gate_matches_oracle(moe, T, d, E, dtype):
    x = rand((T, d), 1.0, dtype, 5)
    Wg = rand((E, d), d ** -0.5, dtype, 6)
    logits = torch.empty(T, E, device="cuda")
    moe.moe_gate(dev(x), dev(Wg), logits)
    got = host(logits)
    rows = np.arange(T) if T <= 4096 else np.random.default_rng(0).choice(T, 512, replace=False)
    ref = oracle.gate(x[rows], Wg)
    err = np.abs(got[rows].astype(np.float64) - ref)
    assert err.max() <= 1e-5 * np.abs(ref).max() + 1e-6
