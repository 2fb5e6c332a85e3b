"""The C ABI: the library loads without a GPU, exports every function that
include/moe.h declares, and rejects bad arguments on the host before any CUDA
call (CPU only; no compute entry point runs here)."""
import ctypes
import os
import re
import subprocess

import pytest

from conftest import ROOT

HEADER = os.path.join(ROOT, "include", "moe.h")


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(moe_\w+)\s*\(", text)))


def test_header_declares_the_layer_calls():
    names = declared_functions()
    for n in ["moe_gate", "moe_route", "moe_route_workspace_size", "moe_dispatch",
              "moe_expert_ffn", "moe_combine", "moe_popularity_update", "moe_device_error",
              "moe_status_string", "moe_version"]:
        assert n in names


def test_library_exports_every_declared_symbol(libmoe_path):
    out = subprocess.check_output(["nm", "-D", "--defined-only", libmoe_path], text=True)
    exported = {line.split()[-1] for line in out.splitlines() if line.strip()}
    missing = [n for n in declared_functions() if n not in exported]
    assert not missing, missing


def test_library_does_not_link_libcuda(libmoe_path):
    out = subprocess.check_output(["ldd", libmoe_path], text=True)
    assert "libcuda.so" not in out and "libcudart.so" not in out


@pytest.fixture(scope="module")
def lib(libmoe_path):
    return ctypes.CDLL(libmoe_path)


def test_status_strings_and_version(lib):
    lib.moe_status_string.restype = ctypes.c_char_p
    assert lib.moe_status_string(0) == b"ok"
    assert lib.moe_status_string(-3) == b"workspace missing or too small"
    assert lib.moe_version() == 100


def test_route_workspace_size(lib):
    lib.moe_route_workspace_size.restype = ctypes.c_size_t
    f = lib.moe_route_workspace_size
    assert f(0, 8, 2) >= 256
    assert f(4096, 16, 2) >= 2 * 16 * 16 * 4  # two int32 [chunk][expert] tables
    assert f(8192, 16, 2) > f(4096, 16, 2) and f(4096, 64, 2) > f(4096, 16, 2)
    assert f(-1, 8, 2) == 0


P = ctypes.c_void_p
FAKE = P(0x1000)  # never dereferenced: every call below fails validation first


def _route(lib, T=64, E=8, k=2, ws=FAKE, ws_bytes=1 << 20, logits=FAKE, counts=FAKE):
    return lib.moe_route(logits, None, T, E, k, 0, FAKE, FAKE, counts, FAKE, FAKE, FAKE, FAKE,
                         FAKE, ws, ctypes.c_size_t(ws_bytes), None)


@pytest.mark.parametrize("kw,code", [
    (dict(E=0), -1), (dict(E=1025), -1), (dict(k=0), -1), (dict(k=9), -1), (dict(T=-1), -1),
    (dict(E=64, k=33), -1), (dict(counts=None), -1), (dict(logits=None), -1),
    (dict(ws=None), -3), (dict(ws_bytes=16), -3),
])
def test_route_rejects_bad_arguments(lib, kw, code):
    assert _route(lib, **kw) == code


def test_dispatch_combine_reject_bad_arguments(lib):
    d = lib.moe_dispatch
    assert d(FAKE, 7, 4, 64, 2, FAKE, FAKE, 8, None) == -2          # dtype
    assert d(FAKE, 1, 4, 60, 2, FAKE, FAKE, 8, None) == -2          # 120-byte rows
    assert d(P(0x1008), 1, 4, 64, 2, FAKE, FAKE, 8, None) == -2     # misaligned x
    assert d(None, 1, 4, 64, 2, FAKE, FAKE, 8, None) == -1
    assert d(FAKE, 1, 4, 64, 33, FAKE, FAKE, 8, None) == -1         # k > 32
    assert d(FAKE, 1, 0, 64, 2, FAKE, FAKE, 0, None) == 0            # T = 0 is a no-op
    c = lib.moe_combine
    assert c(FAKE, 1, 4, 64, 2, None, FAKE, FAKE, 8, None) == -1    # slot_row missing
    assert c(FAKE, 0, 4, 6, 2, FAKE, FAKE, FAKE, 8, None) == -2     # 24-byte fp32 rows


def test_ffn_gate_popularity_reject_bad_arguments(lib):
    f = lib.moe_expert_ffn
    assert f(FAKE, FAKE, FAKE, 1, 4, 100, 64, FAKE, 8, FAKE, FAKE, None) == -2  # d % 8
    assert f(FAKE, FAKE, FAKE, 1, 0, 64, 64, FAKE, 8, FAKE, FAKE, None) == -1
    assert f(FAKE, FAKE, FAKE, 1, 4, 64, 64, None, 8, FAKE, FAKE, None) == -1
    assert f(FAKE, FAKE, FAKE, 1, 4, 64, 64, FAKE, 0, FAKE, FAKE, None) == 0    # nothing to do
    fg = lib.moe_expert_ffn_gather
    fg.argtypes = [P, ctypes.c_int, ctypes.c_int, P, P, P, P] + [ctypes.c_int] * 4 + \
        [P, ctypes.c_int, P, P, P]
    assert fg(FAKE, 16, 2, FAKE, FAKE, FAKE, FAKE, 0, 4, 64, 64, FAKE, 32, FAKE, FAKE, None) == -2
    assert fg(FAKE, 16, 0, FAKE, FAKE, FAKE, FAKE, 1, 4, 64, 64, FAKE, 32, FAKE, FAKE, None) == -1
    assert fg(FAKE, 16, 2, None, FAKE, FAKE, FAKE, 1, 4, 64, 64, FAKE, 32, FAKE, FAKE, None) == -1
    assert fg(FAKE, 16, 2, FAKE, None, FAKE, FAKE, 1, 4, 60, 64, FAKE, 32, FAKE, FAKE, None) == -2
    assert fg(FAKE, 0, 2, FAKE, None, FAKE, FAKE, 1, 4, 64, 64, FAKE, 32, FAKE, FAKE, None) == 0
    g = lib.moe_gate
    assert g(FAKE, FAKE, 1, 8, 12, 4, FAKE, None) == -2                          # 24-byte rows
    assert g(FAKE, FAKE, 1, 0, 64, 4, FAKE, None) == 0
    pu = lib.moe_popularity_update
    pu.argtypes = [P, ctypes.c_int, P, ctypes.c_int, ctypes.c_int64, P, ctypes.c_int, P, P]
    assert pu(FAKE, 8, FAKE, 4, 0, FAKE, 9, FAKE, None) == -1                   # P > E
    assert pu(FAKE, 8, FAKE, 0, 0, FAKE, 2, FAKE, None) == -1                   # W = 0
    assert pu(FAKE, 8, FAKE, 4, -1, FAKE, 2, FAKE, None) == -1                  # step < 0


def test_backward_entry_points_reject_bad_arguments(lib):
    i, z = ctypes.c_int, ctypes.c_size_t
    cb = lib.moe_combine_backward
    cb.argtypes = [P, P, i, i, i, i, P, P, P, P, i, P]
    assert cb(FAKE, FAKE, 1, 4, 64, 33, FAKE, FAKE, FAKE, FAKE, 8, None) == -1   # k > 32
    assert cb(FAKE, FAKE, 0, 4, 6, 2, FAKE, FAKE, FAKE, FAKE, 8, None) == -2     # 24-byte rows
    assert cb(None, None, 1, 0, 64, 2, None, None, None, None, 0, None) == 0     # T = 0
    fb = lib.moe_expert_ffn_backward
    fb.argtypes = [P] * 5 + [i] * 4 + [P, i, P, P, P, P, P]
    assert fb(FAKE, FAKE, FAKE, FAKE, FAKE, 1, 0, 64, 64, FAKE, 8, FAKE, FAKE, None, None,
              None) == -1                                                         # E = 0
    assert fb(FAKE, FAKE, FAKE, FAKE, FAKE, 1, 2, 60, 64, FAKE, 8, FAKE, FAKE, None, None,
              None) == -2                                                         # d % 8
    assert fb(None, None, None, FAKE, FAKE, 1, 2, 64, 64, FAKE, 0, None, None, None, None,
              None) == 0                                                          # no rows
    db = lib.moe_dispatch_backward
    db.argtypes = [P, i, i, i, i, P, P, i, P]
    assert db(FAKE, 1, 4, 64, 40, FAKE, FAKE, 8, None) == -1                     # k > 32
    rb = lib.moe_route_backward
    rb.argtypes = [P, P, P, i, i, i, P, P, P, z, P]
    assert rb(FAKE, FAKE, FAKE, 4, 2, 3, FAKE, None, None, 0, None) == -1        # k > E
    assert rb(FAKE, FAKE, FAKE, 4, 8, 2, FAKE, FAKE, None, 0, None) == -3        # dbias, no ws
    assert rb(None, None, None, 0, 8, 2, None, None, None, 0, None) == 0         # T = 0
    gb = lib.moe_gate_backward
    gb.argtypes = [P, P, i, i, i, i, P, P, P, P, z, P]
    assert gb(FAKE, FAKE, 1, 4, 64, 2000, FAKE, FAKE, FAKE, None, 0, None) == -1  # E > 1024
    assert gb(FAKE, FAKE, 1, 4, 64, 16, FAKE, FAKE, FAKE, None, 0, None) == -3    # dWg, no ws
    assert gb(None, FAKE, 1, 0, 64, 16, None, None, None, None, 0, None) == 0     # T = 0
    ws = lib.moe_gate_backward_workspace_size
    ws.argtypes, ws.restype = [i, i, i, i], z
    assert ws(4096, 1024, 16, 1) >= 3 * 4096 * 16 * 2  # the three bf16 planes
    assert ws(0, 1024, 16, 1) == 0
