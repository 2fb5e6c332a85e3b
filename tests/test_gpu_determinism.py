"""Repeat-run determinism of the whole layer on the GPU.

The same inputs are pushed through the layer's forward and backward three
times; every output the layer produces (routing tables, weights, grouped rows,
hidden activations, expert outputs, the layer output, the popularity window,
and every gradient) must hash the same each time.  No kernel of the library
uses floating-point atomics or any reduction whose order depends on
scheduling, so the results are bit-identical run to run.  Shapes cover the
2-CTA pair tiles with 1-CTA tails (dense groups), the 1-CTA kernel with
capacity drops, and the warp-per-token router."""
import hashlib

import numpy as np
import pytest
import torch

from parity import dev
from routing_dispatch_expert_fp32_b200 import workloads as wl

pytestmark = pytest.mark.gpu


def digest(t) -> str:
    if t is None:
        return "-"
    a = t.detach().contiguous().view(torch.uint8).cpu().numpy()
    return hashlib.sha256(a.tobytes()).hexdigest()


FORWARD = ["logits", "ids", "w", "counts", "kept", "offsets", "slot_row", "row_slot",
           "n_dropped", "Xp", "H", "Yp", "y", "hist", "mean", "hot"]
ROWS = {"row_slot", "Xp", "H", "Yp"}


@pytest.mark.parametrize("T,d,E,k,F,cf", [
    (4096, 512, 8, 2, 512, None),        # dense: pair blocks + 1-CTA tails
    (3000, 256, 48, 4, 768, (5, 4)),     # capacity drops, warp router, 1-CTA tiles
])
def test_layer_forward_backward_bit_identical_across_runs(moe, T, d, E, k, F, cf):
    from fractions import Fraction
    w = wl.tiny("det", T=T, d=d, E=E, k=k, F=F, zipf_s=1.1,
                capacity_factor=None if cf is None else Fraction(*cf), index=70 + E)
    weights = {n: dev(a) for n, a in wl.make_weights(w).items()}
    step = wl.make_step(w, 0)
    x, bias = dev(step["x"]), dev(step["bias"])
    dy = dev(wl.make_grad(w, 0))
    runs = []
    for _ in range(3):
        layer = moe.MoELayer(T, d, E, k, F, torch.bfloat16, capacity=w.capacity, W=4, P=4)
        layer.forward(x, weights["Wg"], weights["W1"], weights["W2"], bias)
        R = int(layer.offsets[-1].item())
        # grouped buffers: only their first R rows are written
        fwd = {n: digest(getattr(layer, n)[:R] if n in ROWS else getattr(layer, n))
               for n in FORWARD}
        g = layer.backward(dy, x, weights["Wg"], weights["W1"], weights["W2"])
        torch.cuda.synchronize()
        assert moe.moe_device_error() == 0
        bwd = {n: digest(v) for n, v in g.items()}
        runs.append((fwd, bwd))
    for fwd, bwd in runs[1:]:
        assert fwd == runs[0][0]
        assert bwd == runs[0][1]
