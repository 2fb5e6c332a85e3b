"""Seeded synthetic inputs for the MoE layer (shared by tests, smoke and bench).

This module draws random tensors and fixes the shapes of the five workloads;
it holds none of the layer's arithmetic (no routing, no FFN, no combine).
Both the CUDA library and the CPU oracle receive the arrays built here.

Generator: numpy PCG64, seed = 1000 * workload + 10 * step + tensor_id
(+ 100000 * rank for independent per-rank batches).  The expert weight stacks
W1 and W2 draw expert e's slice from its own stream, PCG64 seeded with
SeedSequence(seed, spawn_key=(e,)), so the experts are drawn in parallel
threads.  Floats are drawn in fp32; bf16 tensors are rounded to bf16 once here
(nearest even) and travel as uint16 bit patterns, so both sides read the same
bits.

Workloads (sizes from the pages' MoE settings; expert FFN is FC-ReLU-FC as in
PopFetcher, section 5.1; top-k gating with GShard capacity as in "A Survey on
Mixture of Experts", section 5):
  tiny_fp32        T=512,   d=64,   E=8,   k=2, F=128,  fp32, no bias, no capacity
  skewed_drops     T=4096,  d=1024, E=16,  k=2, F=4096, bf16, Zipf(1.2) bias, capacity 1.25
  multistep_window 8 steps of T=16384, d=2048, E=64, k=2, F=8192, bf16, Zipf(1.1) bias
                   random-walking (sigma 0.05) between steps, capacity 1.25, window W=4, top-8
  fine_grained     T=32768, d=4096, E=256, k=8, F=1024, bf16, Zipf(1.0) bias, no capacity
  bw_sweep         T in {8192,16384,32768,65536}, d=7168, E=128, k=4, bf16, identity experts,
                   logits ~ N(0,1) drawn directly, with or without a Zipf(1.5) bias
"""
from __future__ import annotations

import concurrent.futures
import dataclasses
import math
import os
from fractions import Fraction

import numpy as np

TENSOR_X, TENSOR_WG, TENSOR_W1, TENSOR_W2, TENSOR_BIAS, TENSOR_LOGITS, TENSOR_PERM = range(7)
TENSOR_DY, TENSOR_XP, TENSOR_H, TENSOR_DYP = range(7, 11)


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    index: int                 # seed base: 1000 * index
    T: int
    d: int
    E: int
    k: int
    F: int                     # expert hidden width (0: identity experts)
    dtype: str                 # "f32" or "bf16"
    zipf_s: float | None       # None: no bias
    capacity_factor: Fraction | None
    steps: int = 1
    walk_sigma: float = 0.0
    W: int = 4                 # popularity window
    P: int = 8                 # hot experts reported
    logits_direct: bool = False
    bias_scale: float = 0.8

    @property
    def capacity(self) -> int:
        """ceil(cf * T * k / E) in exact arithmetic; 0 means unlimited."""
        if self.capacity_factor is None:
            return 0
        return math.ceil(self.capacity_factor * self.T * self.k / self.E)

    @property
    def identity_experts(self) -> bool:
        return self.F == 0

    def with_(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)


WORKLOADS = {
    "tiny_fp32": Workload("tiny_fp32", 1, 512, 64, 8, 2, 128, "f32", None, None, P=4),
    "skewed_drops": Workload("skewed_drops", 2, 4096, 1024, 16, 2, 4096, "bf16", 1.2,
                             Fraction(5, 4)),
    "multistep_window": Workload("multistep_window", 3, 16384, 2048, 64, 2, 8192, "bf16", 1.1,
                                 Fraction(5, 4), steps=8, walk_sigma=0.05, W=4, P=8),
    "fine_grained": Workload("fine_grained", 4, 32768, 4096, 256, 8, 1024, "bf16", 1.0, None),
    "bw_sweep": Workload("bw_sweep", 5, 65536, 7168, 128, 4, 0, "bf16", 1.5, None,
                         logits_direct=True),
}
BW_SWEEP_TOKENS = (8192, 16384, 32768, 65536)


def seed_for(w: Workload, step: int, tensor_id: int, rank: int = 0) -> int:
    return 1000 * w.index + 10 * step + tensor_id + 100000 * rank


def rng_for(w: Workload, step: int, tensor_id: int, rank: int = 0) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(seed_for(w, step, tensor_id, rank)))


# ------------------------------------------------------------ bf16 storage --
def to_bf16_bits(a: np.ndarray) -> np.ndarray:
    """fp32 -> bf16 bit patterns, nearest even (finite inputs)."""
    u = np.ascontiguousarray(a, dtype=np.float32).view(np.uint32)
    lsb = (u >> 16) & 1
    return ((u + np.uint32(0x7FFF) + lsb) >> 16).astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    return (np.ascontiguousarray(b, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


def _normal(rng, shape, scale, dtype):
    a = rng.standard_normal(shape, dtype=np.float32)
    if scale != 1.0:
        a *= np.float32(scale)
    return to_bf16_bits(a) if dtype == "bf16" else a


def _normal_experts(seed, E, rows, cols, scale, dtype):
    """[E, rows, cols]: expert e from PCG64(SeedSequence(seed, spawn_key=(e,))),
    the experts drawn in parallel threads (numpy releases the GIL while it
    fills large arrays)."""
    out = np.empty((E, rows, cols), np.uint16 if dtype == "bf16" else np.float32)

    def one(e):
        rng = np.random.Generator(np.random.PCG64(np.random.SeedSequence(seed, spawn_key=(e,))))
        out[e] = _normal(rng, (rows, cols), scale, dtype)

    workers = max(1, min(E, os.cpu_count() or 1))
    with concurrent.futures.ThreadPoolExecutor(max_workers=workers) as ex:
        list(ex.map(one, range(E)))
    return out


# ------------------------------------------------------------------ bias ----
def zipf_bias(w: Workload, rank: int = 0) -> np.ndarray | None:
    """b_e = scale * ln(r_e^-s / H_{E,s}), r_e = 1 + perm[e] (a seeded permutation),
    so the hot experts are not tied to the index order."""
    if w.zipf_s is None:
        return None
    perm = rng_for(w, 0, TENSOR_PERM, rank).permutation(w.E)
    r = 1.0 + perm.astype(np.float64)
    H = np.sum(np.arange(1, w.E + 1, dtype=np.float64) ** (-w.zipf_s))
    return (w.bias_scale * np.log(r ** (-w.zipf_s) / H)).astype(np.float32)


def bias_at_step(w: Workload, step: int, rank: int = 0) -> np.ndarray | None:
    """Step 0: the Zipf bias; each later step adds walk_sigma * N(0,1) per expert."""
    b = zipf_bias(w, rank)
    if b is None:
        return None
    b = b.astype(np.float64)
    for s in range(1, step + 1):
        b = b + w.walk_sigma * rng_for(w, s, TENSOR_BIAS, rank).standard_normal(w.E)
    return b.astype(np.float32)


# --------------------------------------------------------------- tensors ----
def make_weights(w: Workload, rank: int = 0) -> dict:
    """Gate and expert weights ~ N(0, 1/fan_in); fixed across steps."""
    out = {}
    if not w.logits_direct:
        out["Wg"] = _normal(rng_for(w, 0, TENSOR_WG, rank), (w.E, w.d), 1.0 / math.sqrt(w.d),
                            w.dtype)
    if not w.identity_experts:
        out["W1"] = _normal_experts(seed_for(w, 0, TENSOR_W1, rank), w.E, w.F, w.d,
                                    1.0 / math.sqrt(w.d), w.dtype)
        out["W2"] = _normal_experts(seed_for(w, 0, TENSOR_W2, rank), w.E, w.d, w.F,
                                    1.0 / math.sqrt(w.F), w.dtype)
    return out


def make_step(w: Workload, step: int = 0, rank: int = 0) -> dict:
    """Per-step inputs: tokens x ~ N(0,1) (and logits ~ N(0,1) when drawn directly)."""
    out = {"x": _normal(rng_for(w, step, TENSOR_X, rank), (w.T, w.d), 1.0, w.dtype),
           "bias": bias_at_step(w, step, rank)}
    if w.logits_direct:
        out["logits"] = rng_for(w, step, TENSOR_LOGITS, rank).standard_normal(
            (w.T, w.E), dtype=np.float32)
    return out


def make_grad(w: Workload, step: int = 0, rank: int = 0) -> np.ndarray:
    """Upstream gradient of the layer output, dy ~ N(0, 1) [T, d] in the layer's dtype."""
    return _normal(rng_for(w, step, TENSOR_DY, rank), (w.T, w.d), 1.0, w.dtype)


def router_logits(w: Workload, step: int = 0, rank: int = 0) -> np.ndarray:
    """Router scores ~ N(0, 1) [T, E] fp32 (the workload's bias adds its skew)."""
    return rng_for(w, step, TENSOR_LOGITS, rank).standard_normal((w.T, w.E), dtype=np.float32)


def ffn_backward_inputs(w: Workload, R_max: int, step: int = 0, rank: int = 0) -> dict:
    """Grouped rows for the expert backward alone: Xp, dYp ~ N(0, 1) [R_max, d] and
    H = max(0, N(0, 1)) [R_max, F] (about half exact zeros, as after a ReLU)."""
    H = rng_for(w, step, TENSOR_H, rank).standard_normal((R_max, w.F), dtype=np.float32)
    np.maximum(H, 0.0, out=H)
    return {"Xp": _normal(rng_for(w, step, TENSOR_XP, rank), (R_max, w.d), 1.0, w.dtype),
            "H": to_bf16_bits(H) if w.dtype == "bf16" else H,
            "dYp": _normal(rng_for(w, step, TENSOR_DYP, rank), (R_max, w.d), 1.0, w.dtype)}


def tiny(name: str, T: int, d: int, E: int, k: int, F: int, dtype: str = "bf16",
         zipf_s: float | None = 1.2, capacity_factor: Fraction | None = Fraction(5, 4),
         index: int = 9, **kw) -> Workload:
    """A small workload of the same structure, for parity cases the oracle finishes fast."""
    return Workload(name, index, T, d, E, k, F, dtype, zipf_s, capacity_factor, **kw)
