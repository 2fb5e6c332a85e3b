"""moe_route_noalloc: the router variant for callers that cannot allocate.

Callers such as serving loops with a fixed memory plan, or plugins whose host
framework owns every device allocation, cannot hand moe_route a workspace.
moe_route_noalloc keeps that scratch in a device array built into the library.
This test calls it through the C ABI twice in a row (different batches, so the
second call runs on the scratch the first one left behind) and checks each
result against moe_route with a caller-provided workspace: integer outputs bit
for bit, weights within the routing tests' tolerance.  It lives in its own file
that pytest collects last, and it also passes when run alone.
"""
import ctypes

import numpy as np
import pytest
import torch

pytestmark = pytest.mark.gpu


def _outputs(T, E, k):
    i32 = torch.int32
    return dict(ids=torch.full((T, k), -7, dtype=i32, device="cuda"),
                w=torch.full((T, k), -7.0, device="cuda"),
                counts=torch.full((E,), -7, dtype=i32, device="cuda"),
                kept=torch.full((E,), -7, dtype=i32, device="cuda"),
                offsets=torch.full((E + 1,), -7, dtype=i32, device="cuda"),
                slot_row=torch.full((T, k), -7, dtype=i32, device="cuda"),
                row_slot=torch.full((T * k,), -7, dtype=i32, device="cuda"),
                n_dropped=torch.full((1,), -7, dtype=i32, device="cuda"))


def _p(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _noalloc(moe, logits, bias, k, capacity, out):
    f = moe.lib.moe_route_noalloc
    P, I = ctypes.c_void_p, ctypes.c_int
    f.argtypes = [P, P, I, I, I, I, P, P, P, P, P, P, P, P, P]
    f.restype = I
    T, E = logits.shape
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    return f(_p(logits), _p(bias), T, E, k, capacity, _p(out["ids"]), _p(out["w"]),
             _p(out["counts"]), _p(out["kept"]), _p(out["offsets"]), _p(out["slot_row"]),
             _p(out["row_slot"]), _p(out["n_dropped"]), stream)


@pytest.mark.parametrize("T,E,k,capacity", [(4096, 16, 2, 640), (20000, 128, 4, 0)])
def test_noalloc_route_matches_workspace_route_twice(moe, T, E, k, capacity):
    rng = np.random.default_rng(T + E)
    for call in range(2):
        logits = torch.from_numpy(rng.standard_normal((T, E), dtype=np.float32)).cuda()
        bias = torch.from_numpy(rng.standard_normal(E).astype(np.float32)).cuda()
        got = _outputs(T, E, k)
        assert _noalloc(moe, logits, bias, k, capacity, got) == 0
        ref = _outputs(T, E, k)
        ws = torch.empty(moe.moe_route_workspace_size(T, E, k), dtype=torch.uint8,
                         device="cuda")
        moe.moe_route(logits, bias, k, capacity, ref["ids"], ref["w"], ref["counts"],
                      ref["kept"], ref["offsets"], ref["slot_row"], ref["row_slot"],
                      ref["n_dropped"], ws)
        torch.cuda.synchronize()
        R = int(ref["offsets"][-1].item())
        for name in ["ids", "counts", "kept", "offsets", "slot_row", "n_dropped"]:
            assert torch.equal(got[name], ref[name]), (call, name)
        assert torch.equal(got["row_slot"][:R], ref["row_slot"][:R]), call
        np.testing.assert_allclose(got["w"].cpu().numpy(), ref["w"].cpu().numpy(),
                                   rtol=4e-6, atol=1e-8)


def test_noalloc_route_rejects_problems_beyond_its_scratch(moe):
    # 2 x 4096 chunks x 1024 experts x 4 B = 32 MiB > 4 MiB of built-in scratch
    T, E, k = 4096 * 128, 1024, 1
    dummy = torch.empty(16, device="cuda")
    out = {n: dummy for n in ["ids", "w", "counts", "kept", "offsets", "slot_row", "row_slot",
                              "n_dropped"]}
    logits = torch.empty(1, device="cuda")
    f = moe.lib.moe_route_noalloc
    f.argtypes = [ctypes.c_void_p] * 2 + [ctypes.c_int] * 4 + [ctypes.c_void_p] * 9
    rc = f(_p(logits), None, T, E, k, 0, *[_p(out[n]) for n in
           ["ids", "w", "counts", "kept", "offsets", "slot_row", "row_slot", "n_dropped"]], None)
    assert rc == -3  # MOE_ERR_WORKSPACE: nothing launched
