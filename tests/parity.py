"""Helpers for the GPU parity tests: host<->device conversion and the
output tolerances.

Tolerances for floating-point outputs (expert FFN, combine): the maximum
absolute error is at most 1e-2 of the largest reference magnitude, and the
summed absolute error is at most 5e-3 of the summed reference magnitude,
against the oracle fed the same bf16-rounded inputs.  Routing outputs,
permutations and popularity are compared bit for bit.
"""
import numpy as np
import torch

MAX_ABS_FRAC = 1e-2
MEAN_REL = 5e-3


def dev(a: np.ndarray, device="cuda") -> torch.Tensor:
    """numpy -> device tensor; uint16 arrays are bf16 bit patterns."""
    a = np.ascontiguousarray(a)
    if a.dtype == np.uint16:
        return torch.from_numpy(a.view(np.int16)).to(device).view(torch.bfloat16)
    return torch.from_numpy(a).to(device)


def host(t: torch.Tensor) -> np.ndarray:
    """device tensor -> numpy; bf16 comes back as uint16 bit patterns."""
    t = t.detach().contiguous().cpu()
    if t.dtype == torch.bfloat16:
        return t.view(torch.int16).numpy().view(np.uint16)
    return t.numpy()


def as_f64(a: np.ndarray) -> np.ndarray:
    if a.dtype == np.uint16:
        return (a.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    return a.astype(np.float64)


def assert_close(got: np.ndarray, ref: np.ndarray, what: str = "",
                 max_abs_frac=MAX_ABS_FRAC, mean_rel=MEAN_REL):
    g, r = as_f64(got), as_f64(ref)
    assert g.shape == r.shape, (what, g.shape, r.shape)
    assert np.all(np.isfinite(g)), f"{what}: non-finite output"
    err = np.abs(g - r)
    scale = np.abs(r).max() if r.size else 0.0
    max_err = err.max() if err.size else 0.0
    assert max_err <= max_abs_frac * scale + 1e-30, \
        f"{what}: max abs err {max_err:.3e} > {max_abs_frac} * {scale:.3e}"
    denom = np.abs(r).sum()
    if denom > 0:
        rel = err.sum() / denom
        assert rel <= mean_rel, f"{what}: mean relative err {rel:.3e} > {mean_rel}"
