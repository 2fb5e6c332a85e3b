"""GShard load-balancing loss on the GPU against the oracle (fp32 softmax on
the GPU vs double in the oracle: relative 1e-5), plus its closed forms and
run-to-run determinism."""
import json
import os

import numpy as np
import pytest
import torch

import oracle
from conftest import GOLDEN
from parity import dev, host
from routing_dispatch_expert_fp32_b200 import workloads as wl

pytestmark = pytest.mark.gpu


def gpu_aux(moe, logits, bias, k, counts):
    T, E = logits.shape
    loss = torch.empty(1, device="cuda")
    P = torch.empty(E, device="cuda")
    ws = torch.empty(moe.moe_route_workspace_size(T, E, k), dtype=torch.uint8, device="cuda")
    moe.moe_aux_loss(dev(logits), None if bias is None else dev(bias), k, dev(counts), loss, P,
                     ws)
    torch.cuda.synchronize()
    return float(host(loss)[0]), host(P)


@pytest.mark.parametrize("T,E,k,s", [(512, 8, 2, None), (4096, 16, 2, 1.2), (16384, 64, 2, 1.1),
                                     (32768, 256, 8, 1.0), (65536, 128, 4, 1.5), (1, 3, 2, None),
                                     (1000, 1024, 8, 1.0), (300, 20, 3, 1.3), (257, 600, 2, 1.0)])
def test_aux_loss_matches_oracle(moe, T, E, k, s):
    w = wl.tiny("aux", T=T, d=8, E=E, k=k, F=8, zipf_s=s, capacity_factor=None, index=70 + E)
    logits = wl.rng_for(w, 0, wl.TENSOR_LOGITS).standard_normal((T, E), dtype=np.float32)
    bias = wl.zipf_bias(w)
    r = oracle.route(logits, bias, k)
    l_ref, P_ref = oracle.aux_loss(logits, bias, k, r["counts"])
    l, P = gpu_aux(moe, logits, bias, k, r["counts"])
    np.testing.assert_allclose(P, P_ref, rtol=1e-5, atol=1e-9)
    np.testing.assert_allclose(l, l_ref, rtol=1e-5)
    l2, P2 = gpu_aux(moe, logits, bias, k, r["counts"])
    assert l2 == l and np.array_equal(P2, P)  # fixed summation order


def test_aux_loss_golden_and_closed_forms(moe):
    g = json.load(open(os.path.join(GOLDEN, "aux_loss_example.json")))
    l, P = gpu_aux(moe, np.array(g["logits"], np.float32), None, g["k"],
                   np.array(g["counts"], np.int32))
    np.testing.assert_allclose(P, g["prob_mean"], rtol=1e-6)
    np.testing.assert_allclose(l, g["loss"], rtol=1e-6)
    lg = np.full((777, 12), -1.5, np.float32)  # uniform router
    r = oracle.route(lg, None, 3)
    l, P = gpu_aux(moe, lg, None, 3, r["counts"])
    np.testing.assert_allclose(l, 1.0, rtol=1e-6)
