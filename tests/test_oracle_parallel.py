"""The OpenMP build of the oracle (CPU only).

The same moe_oracle.c compiled with -fopenmp runs its independent token and
row loops on several host cores.  Every value is computed by the same
operations in the same order, so it must agree bit for bit with the
single-threaded build, and it must pass the same pins.
"""
import os
import subprocess
import sys

import numpy as np

import oracle
from conftest import ROOT
from routing_dispatch_expert_fp32_b200 import workloads as wl


def _layer_outputs():
    w = wl.tiny("omp", T=300, d=64, E=7, k=3, F=96, zipf_s=1.1)
    W, inp = wl.make_weights(w), wl.make_step(w, 0)
    r = oracle.layer(inp["x"], W["Wg"], W["W1"], W["W2"], inp["bias"], w.k, w.capacity)
    rows = r["Xp"][::5]
    experts = (np.searchsorted(r["offsets"], np.arange(0, len(r["Xp"]), 5), side="right") - 1)
    Ys, Hs = oracle.expert_ffn_rows(rows, experts, W["W1"], W["W2"], want_h=True)
    return dict(r, Ys=Ys, Hs=Hs)


def test_parallel_build_matches_serial_bit_for_bit():
    try:
        serial = _layer_outputs()
        assert oracle.use_parallel(True, threads=4) == 4
        par = _layer_outputs()
    finally:
        oracle.use_parallel(False)
    for name in ["logits", "ids", "w", "offsets", "slot_row", "Xp", "H", "Yp", "y", "Ys", "Hs"]:
        assert np.array_equal(np.asarray(serial[name]), np.asarray(par[name])), name


def test_serial_build_reports_one_thread():
    oracle.use_parallel(False)
    assert oracle.use_parallel(False) == 1


def test_pins_pass_on_the_parallel_build():
    lib = oracle.build(parallel=True)
    env = dict(os.environ, MOE_ORACLE_LIB=lib, OMP_NUM_THREADS="4")
    res = subprocess.run([sys.executable, "-m", "pytest", "-x", "-q", "-p", "no:cacheprovider",
                          os.path.join(ROOT, "tests", "test_oracle_pins.py"),
                          os.path.join(ROOT, "tests", "test_oracle_backward.py")],
                         cwd=ROOT, env=env, capture_output=True, text=True, timeout=600)
    assert res.returncode == 0, res.stdout[-3000:]
