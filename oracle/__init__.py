"""CPU oracle of the MoE layer hot path (test infrastructure only).

Only the test suite, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  The product library never loads it and
shares no code with it: the arithmetic lives in ``moe_oracle.c`` (plain C,
loops that follow the definitions, double accumulation), and this module only
compiles that file with gcc and marshals numpy arrays through ctypes.

bf16 tensors travel as ``np.uint16`` arrays holding the bf16 bit patterns;
fp32 tensors as ``np.float32``.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "moe_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
# the same source built with -fopenmp: its independent token / row loops run on
# all host cores (every value computed by the same operations in the same order)
_LIB_OMP = os.path.join(_HERE, "liboracle_omp.so")

F32 = 0
BF16 = 1

_lib = None
# The mutation tests point a fresh process at a deliberately broken build.
_lib_path = os.environ.get("MOE_ORACLE_LIB") or _LIB


def build(force: bool = False, parallel: bool = False) -> str:
    """Compile moe_oracle.c into liboracle.so (no fused multiply-add, no fast
    math), or with ``parallel`` into liboracle_omp.so (the same flags plus
    -fopenmp)."""
    out = _LIB_OMP if parallel else _LIB
    if force or not os.path.exists(out) or os.path.getmtime(out) < os.path.getmtime(_SRC):
        tmp = out + f".tmp{os.getpid()}"
        subprocess.check_call(
            ["gcc", "-O2", "-std=c11", "-ffp-contract=off", "-fno-fast-math", "-fPIC",
             *(["-fopenmp"] if parallel else []), "-shared", "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, out)
    return out


def use_parallel(parallel: bool = True, threads: int = 0) -> int:
    """Switch the wrappers to the OpenMP build (or back); returns the thread
    count the marked loops use (``threads`` > 0 caps it)."""
    use_library(build(parallel=True) if parallel else None)
    lib = _load()
    if threads > 0:
        lib.oracle_set_threads(int(threads))
    return int(lib.oracle_threads())


def use_library(path: str | None) -> None:
    """Point the wrappers at another build of the oracle (None: the default one).

    The mutation tests compile deliberately broken copies of moe_oracle.c and
    check that the pins reject them."""
    global _lib, _lib_path
    _lib, _lib_path = None, (path or _LIB)


def _load():
    global _lib
    if _lib is None:
        if _lib_path == _LIB:
            build()
        elif _lib_path == _LIB_OMP:
            build(parallel=True)
        lib = ctypes.CDLL(_lib_path)
        p, i32, i64 = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64
        lib.oracle_gate.argtypes = [p, p, i32, i32, i32, i32, p]
        lib.oracle_gate.restype = None
        lib.oracle_route.argtypes = [p, p, i32, i32, i32, i32, i32, p, p, p, p, p, p, p, p]
        lib.oracle_route.restype = i32
        lib.oracle_dispatch.argtypes = [p, i32, i32, i32, i32, p, i32, p]
        lib.oracle_dispatch.restype = None
        lib.oracle_expert_ffn_row.argtypes = [p, p, p, i32, i32, i32, i32, p, p]
        lib.oracle_expert_ffn_row.restype = None
        lib.oracle_expert_ffn.argtypes = [p, p, p, i32, i32, i32, i32, p, p, p]
        lib.oracle_expert_ffn.restype = None
        lib.oracle_combine.argtypes = [p, i32, i32, i32, i32, p, p, p]
        lib.oracle_combine.restype = None
        lib.oracle_popularity_update.argtypes = [p, i32, p, i32, i64, p, i32, p]
        lib.oracle_popularity_update.restype = i32
        lib.oracle_correlation_update.argtypes = [p, i32, p, i32, i32, i32, p]
        lib.oracle_correlation_update.restype = None
        lib.oracle_popularity_forecast.argtypes = [p, p, i32, i32, i32, p, i32, p]
        lib.oracle_popularity_forecast.restype = None
        lib.oracle_aux_loss.argtypes = [p, p, i32, i32, i32, p, p]
        lib.oracle_aux_loss.restype = ctypes.c_float
        lib.oracle_combine_backward.argtypes = [p, p, i32, i32, i32, i32, p, p, p, p]
        lib.oracle_combine_backward.restype = None
        lib.oracle_expert_ffn_backward.argtypes = [p, p, p, p, p, i32, i32, i32, i32, p, p, p, p,
                                                   p]
        lib.oracle_expert_ffn_backward.restype = None
        lib.oracle_dispatch_backward.argtypes = [p, i32, i32, i32, i32, p, p]
        lib.oracle_dispatch_backward.restype = None
        lib.oracle_route_backward.argtypes = [p, p, p, i32, i32, i32, p, p]
        lib.oracle_route_backward.restype = None
        lib.oracle_gate_backward.argtypes = [p, p, i32, i32, i32, i32, p, p, p]
        lib.oracle_gate_backward.restype = None
        lib.oracle_expert_ffn_rows.argtypes = [p, p, i32, p, p, i32, i32, i32, p, p]
        lib.oracle_expert_ffn_rows.restype = None
        lib.oracle_threads.argtypes = []
        lib.oracle_threads.restype = i32
        lib.oracle_set_threads.argtypes = [i32]
        lib.oracle_set_threads.restype = None
        lib.oracle_round_bf16.argtypes = [ctypes.c_double]
        lib.oracle_round_bf16.restype = ctypes.c_uint16
        _lib = lib
    return _lib


def _ptr(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _dtype_code(a: np.ndarray) -> int:
    if a.dtype == np.uint16:
        return BF16
    if a.dtype == np.float32:
        return F32
    raise TypeError(f"oracle tensors are float32 or bf16 bits (uint16), got {a.dtype}")


def _c(a, dtype=None):
    a = np.ascontiguousarray(a if dtype is None else a.astype(dtype, copy=False))
    return a


def round_bf16(v: float) -> int:
    """bf16 bits of the double ``v`` rounded once, to nearest even."""
    return int(_load().oracle_round_bf16(float(v)))


def gate(x: np.ndarray, Wg: np.ndarray) -> np.ndarray:
    """logits[T,E] = x[T,d] . Wg[E,d]^T, double accumulation, fp32 result."""
    x, Wg = _c(x), _c(Wg)
    dt = _dtype_code(x)
    assert _dtype_code(Wg) == dt and x.shape[1] == Wg.shape[1]
    T, d = x.shape
    E = Wg.shape[0]
    out = np.empty((T, E), np.float32)
    _load().oracle_gate(_ptr(x), _ptr(Wg), dt, T, d, E, _ptr(out))
    return out


def route(logits: np.ndarray, bias, k: int, capacity: int = 0, rank_major: bool = False):
    """Top-k routing with capacity; returns a dict of the route outputs.

    ``row_slot`` is returned trimmed to R = offsets[E] rows.
    """
    logits = _c(logits, np.float32)
    T, E = logits.shape
    b = None if bias is None else _c(bias, np.float32)
    ids = np.empty((T, k), np.int32)
    w = np.empty((T, k), np.float32)
    counts = np.empty(E, np.int32)
    kept = np.empty(E, np.int32)
    offsets = np.empty(E + 1, np.int32)
    slot_row = np.empty((T, k), np.int32)
    row_slot = np.full(max(T * k, 1), -1, np.int32)
    nd = np.zeros(1, np.int32)
    rc = _load().oracle_route(_ptr(logits), _ptr(b), T, E, k, int(capacity), int(rank_major),
                              _ptr(ids), _ptr(w), _ptr(counts), _ptr(kept), _ptr(offsets),
                              _ptr(slot_row), _ptr(row_slot), _ptr(nd))
    if rc != 0:
        raise ValueError("oracle_route: invalid sizes")
    R = int(offsets[E])
    return dict(ids=ids, w=w, counts=counts, kept=kept, offsets=offsets, slot_row=slot_row,
                row_slot=row_slot[:R].copy(), n_dropped=int(nd[0]))


def dispatch(x: np.ndarray, k: int, row_slot: np.ndarray) -> np.ndarray:
    """Xp[row] = x[row_slot[row] // k]."""
    x = _c(x)
    dt = _dtype_code(x)
    T, d = x.shape
    rs = _c(row_slot, np.int32)
    R = rs.shape[0]
    Xp = np.empty((R, d), x.dtype)
    _load().oracle_dispatch(_ptr(x), dt, T, d, k, _ptr(rs), R, _ptr(Xp))
    return Xp


def expert_ffn(Xp: np.ndarray, W1: np.ndarray, W2: np.ndarray, offsets: np.ndarray,
               want_h: bool = False):
    """Yp (and optionally H) for every grouped row; W1 [E,F,d], W2 [E,d,F]."""
    Xp, W1, W2 = _c(Xp), _c(W1), _c(W2)
    dt = _dtype_code(Xp)
    E, F, d = W1.shape
    assert W2.shape == (E, d, F) and Xp.shape[1] == d
    off = _c(offsets, np.int32)
    R = int(off[E])
    Yp = np.zeros((Xp.shape[0], d), Xp.dtype)
    H = np.zeros((Xp.shape[0], F), Xp.dtype) if want_h else None
    _load().oracle_expert_ffn(_ptr(Xp), _ptr(W1), _ptr(W2), dt, E, d, F, _ptr(off), _ptr(H),
                              _ptr(Yp))
    Yp = Yp[:R]
    return (Yp, H[:R]) if want_h else Yp


def expert_ffn_rows(rows: np.ndarray, experts, W1: np.ndarray, W2: np.ndarray,
                    want_h: bool = False):
    """FFN of selected rows: rows[n,d] each through experts[n]."""
    rows, W1, W2 = _c(rows), _c(W1), _c(W2)
    dt = _dtype_code(rows)
    E, F, d = W1.shape
    n = rows.shape[0]
    ex = _c(np.asarray(experts), np.int32)
    assert ex.shape == (n,) and (n == 0 or (ex.min() >= 0 and ex.max() < E))
    Y = np.empty((n, d), rows.dtype)
    H = np.empty((n, F), rows.dtype) if want_h else None
    _load().oracle_expert_ffn_rows(_ptr(rows), _ptr(ex), n, _ptr(W1), _ptr(W2), dt, d, F,
                                   _ptr(H), _ptr(Y))
    return (Y, H) if want_h else Y


def combine(Yp: np.ndarray, T: int, k: int, slot_row: np.ndarray, w: np.ndarray) -> np.ndarray:
    """y[t] = sum_j w[t,j] Yp[slot_row[t,j]] over kept slots."""
    Yp = _c(Yp)
    dt = _dtype_code(Yp)
    d = Yp.shape[1]
    sr, ww = _c(slot_row, np.int32), _c(w, np.float32)
    y = np.empty((T, d), Yp.dtype)
    _load().oracle_combine(_ptr(Yp), dt, T, d, k, _ptr(sr), _ptr(ww), _ptr(y))
    return y


def popularity_update(counts: np.ndarray, hist: np.ndarray, step: int, P: int):
    """Updates ``hist`` [W,E] in place; returns (mean[E] fp32, hot[P] int32)."""
    counts = _c(counts, np.int32)
    assert hist.dtype == np.int32 and hist.flags.c_contiguous
    W, E = hist.shape
    mean = np.empty(E, np.float32)
    hot = np.empty(max(P, 1), np.int32)
    rc = _load().oracle_popularity_update(_ptr(counts), E, _ptr(hist), W, int(step), _ptr(mean),
                                          P, _ptr(hot))
    if rc != 0:
        raise ValueError("oracle_popularity_update: invalid sizes")
    return mean, hot[:P].copy()


def correlation_update(ids_prev: np.ndarray, ids_next: np.ndarray, C: np.ndarray) -> None:
    """Adds the consecutive-layer co-selection counts of one batch into C [E,E] (in place)."""
    a, b = _c(ids_prev, np.int32), _c(ids_next, np.int32)
    assert C.dtype == np.int32 and C.flags.c_contiguous and a.shape[0] == b.shape[0]
    T = a.shape[0]
    _load().oracle_correlation_update(_ptr(a), a.shape[1], _ptr(b), b.shape[1], T, C.shape[0],
                                      _ptr(C))


def popularity_forecast(pop_prev: np.ndarray, C: np.ndarray, k_prev: int, k_next: int, P: int):
    """Next-layer popularity forecast (fp32 [E]) and its top-P experts."""
    pop = _c(pop_prev, np.float32)
    Cc = _c(C, np.int32)
    E = Cc.shape[0]
    pred = np.empty(E, np.float32)
    hot = np.empty(max(P, 1), np.int32)
    _load().oracle_popularity_forecast(_ptr(pop), _ptr(Cc), E, k_prev, k_next, _ptr(pred), P,
                                       _ptr(hot))
    return pred, hot[:P].copy()


def aux_loss(logits: np.ndarray, bias, k: int, counts: np.ndarray):
    """GShard balancing loss E * sum_e f_e P_e; returns (loss fp32, P_e [E] fp32)."""
    lg = _c(logits, np.float32)
    T, E = lg.shape
    b = None if bias is None else _c(bias, np.float32)
    cnt = _c(counts, np.int32)
    P = np.empty(E, np.float32)
    loss = _load().oracle_aux_loss(_ptr(lg), _ptr(b), T, E, k, _ptr(cnt), _ptr(P))
    return np.float32(loss), P


def combine_backward(dy, Yp, k, slot_row, w):
    """(dw [T,k] fp32, dYp [rows(Yp), d] dtype; rows no slot names stay zero)."""
    dy, Yp = _c(dy), _c(Yp)
    dt = _dtype_code(dy)
    T, d = dy.shape
    sr, ww = _c(slot_row, np.int32), _c(w, np.float32)
    dw = np.empty((T, k), np.float32)
    dYp = np.zeros_like(Yp)
    _load().oracle_combine_backward(_ptr(dy), _ptr(Yp), dt, T, d, k, _ptr(sr), _ptr(ww), _ptr(dw),
                                    _ptr(dYp))
    return dw, dYp


def expert_ffn_backward(Xp, H, dYp, W1, W2, offsets):
    """(dH, dXp, dW1 fp32 [E,F,d], dW2 fp32 [E,d,F]) over the grouped rows."""
    Xp, H, dYp, W1, W2 = _c(Xp), _c(H), _c(dYp), _c(W1), _c(W2)
    dt = _dtype_code(Xp)
    E, F, d = W1.shape
    off = _c(offsets, np.int32)
    dH = np.zeros_like(H)
    dXp = np.zeros_like(Xp)
    dW1 = np.zeros((E, F, d), np.float32)
    dW2 = np.zeros((E, d, F), np.float32)
    _load().oracle_expert_ffn_backward(_ptr(Xp), _ptr(H), _ptr(dYp), _ptr(W1), _ptr(W2), dt, E, d,
                                       F, _ptr(off), _ptr(dH), _ptr(dXp), _ptr(dW1), _ptr(dW2))
    return dH, dXp, dW1, dW2


def dispatch_backward(dXp, T, k, slot_row):
    dXp = _c(dXp)
    dt = _dtype_code(dXp)
    d = dXp.shape[1]
    dx = np.empty((T, d), dXp.dtype)
    _load().oracle_dispatch_backward(_ptr(dXp), dt, T, d, k, _ptr(_c(slot_row, np.int32)),
                                     _ptr(dx))
    return dx


def route_backward(ids, w, dw, E):
    """(dlogits [T,E] fp32, dbias [E] fp32)."""
    ids, w, dw = _c(ids, np.int32), _c(w, np.float32), _c(dw, np.float32)
    T, k = ids.shape
    dl = np.empty((T, E), np.float32)
    db = np.empty(E, np.float32)
    _load().oracle_route_backward(_ptr(ids), _ptr(w), _ptr(dw), T, E, k, _ptr(dl), _ptr(db))
    return dl, db


def gate_backward(x, Wg, dlogits, dx):
    """Adds the gate's input gradient into a copy of dx; returns (dx, dWg fp32)."""
    x, Wg = _c(x), _c(Wg)
    dt = _dtype_code(x)
    T, d = x.shape
    E = Wg.shape[0]
    dx = np.array(dx, copy=True)
    dWg = np.empty((E, d), np.float32)
    _load().oracle_gate_backward(_ptr(x), _ptr(Wg), dt, T, d, E, _ptr(_c(dlogits, np.float32)),
                                 _ptr(dx), _ptr(dWg))
    return dx, dWg


def layer_backward(x, Wg, W1, W2, bias, k, fwd, dy):
    """Whole-layer backward from the forward record `fwd` (layer(..., want_h) output)."""
    dw, dYp = combine_backward(dy, fwd["Yp"], k, fwd["slot_row"], fwd["w"])
    dH, dXp, dW1, dW2 = expert_ffn_backward(fwd["Xp"], fwd["H"], dYp, W1, W2, fwd["offsets"])
    dx = dispatch_backward(dXp, x.shape[0], k, fwd["slot_row"])
    dlogits, dbias = route_backward(fwd["ids"], fwd["w"], dw, Wg.shape[0])
    dx, dWg = gate_backward(x, Wg, dlogits, dx)
    return dict(dw=dw, dYp=dYp, dH=dH, dXp=dXp, dW1=dW1, dW2=dW2, dlogits=dlogits,
                dbias=dbias, dx=dx, dWg=dWg)


def layer(x, Wg, W1, W2, bias, k, capacity=0, logits=None):
    """Whole layer: gate (unless logits are given), route, dispatch, FFN, combine."""
    if logits is None:
        logits = gate(x, Wg)
    r = route(logits, bias, k, capacity)
    Xp = dispatch(x, k, r["row_slot"])
    Yp, H = expert_ffn(Xp, W1, W2, r["offsets"], want_h=True)
    y = combine(Yp, x.shape[0], k, r["slot_row"], r["w"])
    return dict(logits=logits, Xp=Xp, H=H, Yp=Yp, y=y, **r)
