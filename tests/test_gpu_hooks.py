"""The tcgen05 GEMMs under the test-only hooks (a separate build of the
library; the shipped libmoe.so has no hooks).

1. Bounded waits.  With the producers told to issue no loads, every MMA and
   epilogue wait of the forward (1-CTA and pair) and backward GEMMs runs out
   (20 ms in the test build) with nothing in flight: the call returns, the
   device error word reports MOE_DEVERR_TIMEOUT, and the next calls (hooked
   build and shipped library) are correct -- the kernels freed their tensor
   memory and left the context usable.
2. Many tiles per CTA.  With the grid capped to one CTA (one pair), a single
   CTA walks every tile, so each accumulator hand-off between the MMA warp and
   the epilogue is exercised; the result is compared element by element with
   the oracle and bit for bit with the shipped library.
"""
import ctypes

import numpy as np
import pytest
import torch

import oracle
from parity import assert_close, dev, host
from routing_dispatch_expert_fp32_b200 import workloads as wl

pytestmark = pytest.mark.gpu

P = ctypes.c_void_p


def _p(t):
    return None if t is None else P(t.data_ptr())


def _stream():
    return P(torch.cuda.current_stream().cuda_stream)


def _device_error(lib):
    bits = ctypes.c_int32(0)
    assert lib.moe_device_error(ctypes.byref(bits), 1) == 0
    return bits.value


def _rand(shape, scale, seed):
    a = np.random.default_rng(seed).standard_normal(shape, dtype=np.float32) * np.float32(scale)
    return wl.to_bf16_bits(a)


# (sizes, d, F, R_max) reaching each forward kernel:
#   pair, pair_wide  R_max >= 1024 rows per expert: 2-CTA 256 x 256 tiles for
#                    whole 256-row blocks, 1-CTA 128 x 256 tiles for the tails;
#   one_cta, ragged  sparse groups with at least three waves of 128-row tiles:
#                    1-CTA 128 x 256 tiles (ragged adds groups of several tiles)
_SMALL = [int(v) for v in np.random.default_rng(7).integers(0, 41, 64)]
SHAPES = {
    "pair": ([700, 0, 1300], 136, 384, 3100),
    "pair_wide": ([700, 0, 1300, 5, 250], 256, 768, 5200),
    "one_cta": (_SMALL, 136, 264, 60000),
    "ragged": (_SMALL + [300, 517], 128, 256, 60000),
}


def _case(name):
    sizes, d, F, Rmax = SHAPES[name]
    E, R = len(sizes), sum(sizes)
    offsets = np.array([0] + np.cumsum(sizes).tolist(), np.int32)
    Xp = _rand((R, d), 1.0, 1)
    W1, W2 = _rand((E, F, d), d ** -0.5, 2), _rand((E, d, F), F ** -0.5, 3)
    Xd = torch.zeros(Rmax, d, dtype=torch.bfloat16, device="cuda")
    Xd[:R] = dev(Xp)
    return dict(E=E, R=R, d=d, F=F, Rmax=Rmax, offsets=offsets, Xp=Xp, W1=W1, W2=W2, Xd=Xd,
                W1d=dev(W1), W2d=dev(W2), offd=dev(offsets))


def _ffn(lib, c):
    H = torch.zeros(c["Rmax"], c["F"], dtype=torch.bfloat16, device="cuda")
    Y = torch.zeros(c["Rmax"], c["d"], dtype=torch.bfloat16, device="cuda")
    rc = lib.moe_expert_ffn(_p(c["Xd"]), _p(c["W1d"]), _p(c["W2d"]), 1, c["E"], c["d"], c["F"],
                            _p(c["offd"]), c["Rmax"], _p(H), _p(Y), _stream())
    assert rc == 0
    torch.cuda.synchronize()
    return H, Y


def _ffn_bwd(lib, c, H, weights=True):
    g = torch.from_numpy(_rand((c["Rmax"], c["d"]), 1.0, 4).view(np.int16)).view(
        torch.bfloat16).cuda()
    dH = torch.zeros_like(H)
    dX = torch.zeros_like(c["Xd"])
    dW1 = torch.zeros(c["E"], c["F"], c["d"], device="cuda") if weights else None
    dW2 = torch.zeros(c["E"], c["d"], c["F"], device="cuda") if weights else None
    rc = lib.moe_expert_ffn_backward(_p(c["Xd"]), _p(H), _p(g), _p(c["W1d"]), _p(c["W2d"]), 1,
                                     c["E"], c["d"], c["F"], _p(c["offd"]), c["Rmax"], _p(dH),
                                     _p(dX), _p(dW1), _p(dW2), _stream())
    assert rc == 0
    torch.cuda.synchronize()
    return [t for t in (dH, dX, dW1, dW2) if t is not None]


@pytest.mark.parametrize("name", sorted(SHAPES))
def test_stalled_producer_waits_run_out_and_the_context_stays_usable(hooked, moe, name):
    c = _case(name)
    H_ref, Y_ref = _ffn(moe.lib, c)
    bwd_ref = _ffn_bwd(moe.lib, c, H_ref)
    _device_error(hooked)
    try:
        assert hooked.moe_test_hooks(1, 0) == 0
        _ffn(hooked, c)  # returns, the device does not hang or fault
        assert _device_error(hooked) & moe.MOE_DEVERR_TIMEOUT
        _ffn_bwd(hooked, c, H_ref)  # input- and weight-gradient GEMMs
        assert _device_error(hooked) & moe.MOE_DEVERR_TIMEOUT
    finally:
        assert hooked.moe_test_hooks(0, 0) == 0
    # the same build, unstalled, and the shipped library both compute correctly
    H, Y = _ffn(hooked, c)
    assert torch.equal(H, H_ref) and torch.equal(Y, Y_ref)
    for a, b in zip(_ffn_bwd(hooked, c, H_ref), bwd_ref):
        assert torch.equal(a, b)
    assert _device_error(hooked) == 0
    H2, Y2 = _ffn(moe.lib, c)
    assert torch.equal(H2, H_ref) and torch.equal(Y2, Y_ref)
    assert moe.moe_device_error() == 0


@pytest.mark.parametrize("name", sorted(SHAPES))
@pytest.mark.parametrize("max_ctas", [1, 2])
def test_one_cta_walks_every_tile(hooked, moe, name, max_ctas):
    c = _case(name)
    H_ref, Y_ref = _ffn(moe.lib, c)
    bwd_ref = _ffn_bwd(moe.lib, c, H_ref)
    try:
        assert hooked.moe_test_hooks(0, max_ctas) == 0
        H, Y = _ffn(hooked, c)
        bwd = _ffn_bwd(hooked, c, H_ref)
    finally:
        assert hooked.moe_test_hooks(0, 0) == 0
    assert _device_error(hooked) == 0
    # every tile computed by the one CTA (pair) matches the full grid bit for bit
    assert torch.equal(H, H_ref) and torch.equal(Y, Y_ref)
    for a, b in zip(bwd, bwd_ref):
        assert torch.equal(a, b)
    # and the oracle element by element; rows past R stay untouched
    R = c["R"]
    Yr, Hr = oracle.expert_ffn(c["Xp"], c["W1"], c["W2"], c["offsets"], want_h=True)
    assert_close(host(H[:R]), Hr, "H")
    assert_close(host(Y[:R]), Yr, "Yp")
    assert not host(Y[R:]).any() and not host(H[R:]).any()
