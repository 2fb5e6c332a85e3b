"""ctypes binding of libmoe.so (include/moe.h): argument marshalling only.

Every function has the C name, takes torch tensors that live on the current
CUDA device, passes their data pointers and the current stream, and raises
MoeError on a non-zero status.  Every step of the computation runs in the
library's CUDA kernels; there is no other implementation behind these names.
If libmoe.so is missing this module fails to import.
"""
from __future__ import annotations

import ctypes
import os

import torch

_LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libmoe.so")
if not os.path.exists(_LIB_PATH):
    raise ImportError(f"{_LIB_PATH} is missing: build it with "
                      "`python -m routing_dispatch_expert_fp32_b200.build` (needs nvcc)")
lib = ctypes.CDLL(_LIB_PATH)

MOE_OK = 0
MOE_DTYPE_F32 = 0
MOE_DTYPE_BF16 = 1
MOE_DEVERR_ROW_INDEX = 1
MOE_DEVERR_OFFSETS = 2
MOE_DEVERR_TIMEOUT = 4
MOE_DEVERR_EXPERT_INDEX = 8

_p, _i, _i64, _sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_size_t
_SIGS = {
    "moe_status_string": ([_i], ctypes.c_char_p),
    "moe_version": ([], _i),
    "moe_device_error": ([_p, _i], _i),
    "moe_gate": ([_p, _p, _i, _i, _i, _i, _p, _p], _i),
    "moe_route_workspace_size": ([_i, _i, _i], _sz),
    "moe_route": ([_p, _p, _i, _i, _i, _i, _p, _p, _p, _p, _p, _p, _p, _p, _p, _sz, _p], _i),
    "moe_dispatch": ([_p, _i, _i, _i, _i, _p, _p, _i, _p], _i),
    "moe_expert_ffn": ([_p, _p, _p, _i, _i, _i, _i, _p, _i, _p, _p, _p], _i),
    "moe_combine": ([_p, _i, _i, _i, _i, _p, _p, _p, _i, _p], _i),
    "moe_expert_ffn_gather": ([_p, _i, _i, _p, _p, _p, _p, _i, _i, _i, _i, _p, _i, _p, _p, _p],
                              _i),
    "moe_popularity_update": ([_p, _i, _p, _i, _i64, _p, _i, _p, _p], _i),
    "moe_popularity_update_dev": ([_p, _i, _p, _i, _p, _p, _i, _p, _p], _i),
    "moe_route_noalloc": ([_p, _p, _i, _i, _i, _i, _p, _p, _p, _p, _p, _p, _p, _p, _p], _i),
    "moe_correlation_update": ([_p, _i, _p, _i, _i, _i, _p, _p], _i),
    "moe_popularity_forecast": ([_p, _p, _i, _i, _i, _p, _i, _p, _p], _i),
    "moe_aux_loss": ([_p, _p, _i, _i, _i, _p, _p, _p, _p, _sz, _p], _i),
    "moe_combine_backward": ([_p, _p, _i, _i, _i, _i, _p, _p, _p, _p, _i, _p], _i),
    "moe_expert_ffn_backward": ([_p, _p, _p, _p, _p, _i, _i, _i, _i, _p, _i, _p, _p, _p, _p, _p],
                                _i),
    "moe_dispatch_backward": ([_p, _i, _i, _i, _i, _p, _p, _i, _p], _i),
    "moe_route_backward": ([_p, _p, _p, _i, _i, _i, _p, _p, _p, _sz, _p], _i),
    "moe_gate_backward_workspace_size": ([_i, _i, _i, _i], _sz),
    "moe_gate_backward": ([_p, _p, _i, _i, _i, _i, _p, _p, _p, _p, _sz, _p], _i),
}
for _name, (_args, _res) in _SIGS.items():
    _f = getattr(lib, _name)
    _f.argtypes, _f.restype = _args, _res


class MoeError(RuntimeError):
    def __init__(self, fn: str, status: int):
        msg = lib.moe_status_string(status).decode()
        super().__init__(f"{fn} failed: {msg} ({status})")
        self.status = status


def _check(fn: str, status: int) -> None:
    if status != MOE_OK:
        raise MoeError(fn, status)


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream=None):
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.bfloat16:
        return MOE_DTYPE_BF16
    if t.dtype == torch.float32:
        return MOE_DTYPE_F32
    raise TypeError(f"unsupported dtype {t.dtype}")


def moe_version() -> int:
    return lib.moe_version()


def moe_device_error(clear: bool = True) -> int:
    bits = ctypes.c_int32(0)
    _check("moe_device_error", lib.moe_device_error(ctypes.byref(bits), int(clear)))
    return bits.value


def moe_gate(x, Wg, logits, stream=None):
    T, d = x.shape
    E = Wg.shape[0]
    _check("moe_gate", lib.moe_gate(_ptr(x), _ptr(Wg), dtype_code(x), T, d, E, _ptr(logits),
                                     _stream(stream)))


def moe_route_workspace_size(T: int, E: int, k: int) -> int:
    return int(lib.moe_route_workspace_size(T, E, k))


def moe_route(logits, bias, k, capacity, ids, w, counts, kept, offsets, slot_row, row_slot,
              n_dropped, workspace, stream=None):
    T, E = logits.shape
    _check("moe_route", lib.moe_route(
        _ptr(logits), _ptr(bias), T, E, k, int(capacity), _ptr(ids), _ptr(w), _ptr(counts),
        _ptr(kept), _ptr(offsets), _ptr(slot_row), _ptr(row_slot), _ptr(n_dropped),
        _ptr(workspace), workspace.numel() * workspace.element_size(), _stream(stream)))


def moe_dispatch(x, k, slot_row, Xp, stream=None):
    T, d = x.shape
    _check("moe_dispatch", lib.moe_dispatch(_ptr(x), dtype_code(x), T, d, k, _ptr(slot_row),
                                            _ptr(Xp), Xp.shape[0], _stream(stream)))


def moe_expert_ffn(Xp, W1, W2, offsets, H, Yp, stream=None):
    E, F, d = W1.shape
    _check("moe_expert_ffn", lib.moe_expert_ffn(
        _ptr(Xp), _ptr(W1), _ptr(W2), dtype_code(Xp), E, d, F, _ptr(offsets), Xp.shape[0],
        _ptr(H), _ptr(Yp), _stream(stream)))


def moe_expert_ffn_gather(x, k, row_slot, w, W1, W2, offsets, H, Yp, stream=None):
    """Expert FFN on rows gathered from x by row_slot; w (or None) scales each row."""
    T, d = x.shape
    E, F, _ = W1.shape
    _check("moe_expert_ffn_gather", lib.moe_expert_ffn_gather(
        _ptr(x), T, k, _ptr(row_slot), _ptr(w), _ptr(W1), _ptr(W2), dtype_code(x), E, d, F,
        _ptr(offsets), H.shape[0], _ptr(H), _ptr(Yp), _stream(stream)))


def moe_combine(Yp, k, slot_row, w, y, stream=None):
    T, d = y.shape
    _check("moe_combine", lib.moe_combine(_ptr(Yp), dtype_code(Yp), T, d, k, _ptr(slot_row),
                                          _ptr(w), _ptr(y), Yp.shape[0], _stream(stream)))


def moe_popularity_update(counts, hist, step, mean, P, hot, stream=None):
    W, E = hist.shape
    _check("moe_popularity_update", lib.moe_popularity_update(
        _ptr(counts), E, _ptr(hist), W, int(step), _ptr(mean), P, _ptr(hot), _stream(stream)))


def moe_popularity_update_dev(counts, hist, step_dev, mean, P, hot, stream=None):
    """step_dev: int64 device tensor of one element, advanced by the call."""
    W, E = hist.shape
    _check("moe_popularity_update_dev", lib.moe_popularity_update_dev(
        _ptr(counts), E, _ptr(hist), W, _ptr(step_dev), _ptr(mean), P, _ptr(hot),
        _stream(stream)))


def moe_route_noalloc(logits, bias, k, capacity, ids, w, counts, kept, offsets, slot_row,
                      row_slot, n_dropped, stream=None):
    T, E = logits.shape
    _check("moe_route_noalloc", lib.moe_route_noalloc(
        _ptr(logits), _ptr(bias), T, E, k, int(capacity), _ptr(ids), _ptr(w), _ptr(counts),
        _ptr(kept), _ptr(offsets), _ptr(slot_row), _ptr(row_slot), _ptr(n_dropped),
        _stream(stream)))


def moe_correlation_update(ids_prev, ids_next, C, stream=None):
    T, k_prev = ids_prev.shape
    _check("moe_correlation_update", lib.moe_correlation_update(
        _ptr(ids_prev), k_prev, _ptr(ids_next), ids_next.shape[1], T, C.shape[0], _ptr(C),
        _stream(stream)))


def moe_popularity_forecast(pop_prev, C, k_prev, k_next, pred, P, hot, stream=None):
    _check("moe_popularity_forecast", lib.moe_popularity_forecast(
        _ptr(pop_prev), _ptr(C), C.shape[0], k_prev, k_next, _ptr(pred), P, _ptr(hot),
        _stream(stream)))


def moe_aux_loss(logits, bias, k, counts, loss, prob_mean, workspace, stream=None):
    T, E = logits.shape
    _check("moe_aux_loss", lib.moe_aux_loss(
        _ptr(logits), _ptr(bias), T, E, k, _ptr(counts), _ptr(loss), _ptr(prob_mean),
        _ptr(workspace), workspace.numel() * workspace.element_size(), _stream(stream)))


def moe_combine_backward(dy, Yp, k, slot_row, w, dw, dYp, stream=None):
    T, d = dy.shape
    _check("moe_combine_backward", lib.moe_combine_backward(
        _ptr(dy), _ptr(Yp), dtype_code(dy), T, d, k, _ptr(slot_row), _ptr(w), _ptr(dw),
        _ptr(dYp), Yp.shape[0], _stream(stream)))


def moe_expert_ffn_backward(Xp, H, dYp, W1, W2, offsets, dH, dXp, dW1, dW2, stream=None):
    E, F, d = W1.shape
    _check("moe_expert_ffn_backward", lib.moe_expert_ffn_backward(
        _ptr(Xp), _ptr(H), _ptr(dYp), _ptr(W1), _ptr(W2), dtype_code(Xp), E, d, F,
        _ptr(offsets), Xp.shape[0], _ptr(dH), _ptr(dXp), _ptr(dW1), _ptr(dW2), _stream(stream)))


def moe_dispatch_backward(dXp, k, slot_row, dx, stream=None):
    T, d = dx.shape
    _check("moe_dispatch_backward", lib.moe_dispatch_backward(
        _ptr(dXp), dtype_code(dXp), T, d, k, _ptr(slot_row), _ptr(dx), dXp.shape[0],
        _stream(stream)))


def moe_route_backward(ids, w, dw, E, dlogits, dbias, workspace, stream=None):
    T, k = ids.shape
    nbytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check("moe_route_backward", lib.moe_route_backward(
        _ptr(ids), _ptr(w), _ptr(dw), T, E, k, _ptr(dlogits), _ptr(dbias), _ptr(workspace),
        nbytes, _stream(stream)))


def moe_gate_backward_workspace_size(T: int, d: int, E: int, dtype=torch.bfloat16) -> int:
    code = MOE_DTYPE_BF16 if dtype == torch.bfloat16 else MOE_DTYPE_F32
    return int(lib.moe_gate_backward_workspace_size(T, d, E, code))


def moe_gate_backward(x, Wg, dlogits, dx, dWg, workspace=None, stream=None):
    T, d = x.shape
    E = Wg.shape[0]
    nbytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check("moe_gate_backward", lib.moe_gate_backward(
        _ptr(x), _ptr(Wg), dtype_code(x), T, d, E, _ptr(dlogits), _ptr(dx), _ptr(dWg),
        _ptr(workspace), nbytes, _stream(stream)))


class MoELayer:
    """One MoE layer's device buffers plus the call sequence of the hot path.

    Weights stay resident; ``forward`` runs gate (unless logits are given),
    route, popularity, dispatch, expert FFN and combine on the current stream,
    all through the C ABI.  ``identity_experts`` skips the FFN (Yp = Xp).
    The popularity step counter lives in device memory (``step_dev``), so a
    forward captured by ``capture`` keeps advancing the window on replay.
    """

    def __init__(self, T, d, E, k, F, dtype, capacity=0, W=4, P=8, device="cuda",
                 identity_experts=False, fused=False):
        self.T, self.d, self.E, self.k, self.F = T, d, E, k, F
        self.dtype, self.capacity, self.W, self.P = dtype, capacity, W, P
        self.identity_experts = identity_experts
        # fused: the first expert GEMM gathers its rows from x and the second
        # applies the gate weights (no dispatch pass, combine is a plain sum);
        # bf16 layers with experts only, forward only
        self.fused = bool(fused) and not identity_experts and dtype == torch.bfloat16
        dev, i32 = device, torch.int32
        Rmax = max(T * k, 1)
        self.logits = torch.empty(T, E, dtype=torch.float32, device=dev)
        self.ids = torch.empty(T, k, dtype=i32, device=dev)
        self.w = torch.empty(T, k, dtype=torch.float32, device=dev)
        self.counts = torch.empty(E, dtype=i32, device=dev)
        self.kept = torch.empty(E, dtype=i32, device=dev)
        self.offsets = torch.empty(E + 1, dtype=i32, device=dev)
        self.slot_row = torch.empty(T, k, dtype=i32, device=dev)
        self.row_slot = torch.empty(Rmax, dtype=i32, device=dev)
        self.n_dropped = torch.empty(1, dtype=i32, device=dev)
        self.workspace = torch.empty(moe_route_workspace_size(T, E, k), dtype=torch.uint8,
                                     device=dev)
        self.Xp = torch.empty(Rmax, d, dtype=dtype, device=dev)
        self.H = None if identity_experts else torch.empty(Rmax, F, dtype=dtype, device=dev)
        self.Yp = self.Xp if identity_experts else torch.empty(Rmax, d, dtype=dtype, device=dev)
        self.y = torch.empty(T, d, dtype=dtype, device=dev)
        self.hist = torch.zeros(W, E, dtype=i32, device=dev)
        self.mean = torch.empty(E, dtype=torch.float32, device=dev)
        self.hot = torch.empty(max(P, 1), dtype=i32, device=dev)
        self.step_dev = torch.zeros(1, dtype=torch.int64, device=dev)

    def share_popularity(self, other: "MoELayer"):
        """Use other's popularity window (ring, step counter, mean, hot): two
        instances that run batches of the same layer concurrently keep one
        window, provided their updates are ordered (see capture_concurrent)."""
        self.hist, self.mean, self.hot, self.step_dev = (other.hist, other.mean, other.hot,
                                                         other.step_dev)

    def forward(self, x, Wg=None, W1=None, W2=None, bias=None, logits=None, stream=None,
                popularity=True, counts_hook=None, popularity_done=None):
        """One layer step: ``forward_route``, then (when ``popularity``) the
        counts hook -- e.g. an all_reduce of the per-expert counts across
        data-parallel ranks -- and ``forward_rest``."""
        self.forward_route(x, Wg, bias, logits, stream)
        if popularity and counts_hook is not None:
            counts_hook(self.counts)
        return self.forward_rest(x, W1, W2, stream, popularity, popularity_done)

    def forward_route(self, x, Wg=None, bias=None, logits=None, stream=None):
        """Gate (unless logits are given) and route: the part of a step before
        the per-expert counts may be exchanged."""
        if logits is None:
            moe_gate(x, Wg, self.logits, stream)
            logits = self.logits
        moe_route(logits, bias, self.k, self.capacity, self.ids, self.w, self.counts, self.kept,
                  self.offsets, self.slot_row, self.row_slot, self.n_dropped, self.workspace,
                  stream)

    def forward_rest(self, x, W1=None, W2=None, stream=None, popularity=True,
                     popularity_done=None):
        """Popularity update, dispatch, expert FFN and combine (after
        ``forward_route`` and any exchange of the counts); returns y."""
        if popularity:
            moe_popularity_update_dev(self.counts, self.hist, self.step_dev, self.mean, self.P,
                                      self.hot, stream)
            if popularity_done is not None:
                popularity_done()
        if self.fused:
            moe_expert_ffn_gather(x, self.k, self.row_slot, self.w, W1, W2, self.offsets, self.H,
                                  self.Yp, stream)
            moe_combine(self.Yp, self.k, self.slot_row, None, self.y, stream)
            return self.y
        moe_dispatch(x, self.k, self.slot_row, self.Xp, stream)
        if not self.identity_experts:
            moe_expert_ffn(self.Xp, W1, W2, self.offsets, self.H, self.Yp, stream)
        moe_combine(self.Yp, self.k, self.slot_row, self.w, self.y, stream)
        return self.y

    def backward(self, dy, x, Wg=None, W1=None, W2=None, stream=None, weight_grads=True):
        """Gradients of the last ``forward`` given dy = dLoss/dy.

        Runs combine, expert-FFN, dispatch, route and gate backward through the
        C ABI on the forward's stored tensors and returns a dict with dx,
        dlogits, dbias and (when ``weight_grads``) dW1, dW2, dWg; dWg and the
        gate's share of dx only when Wg is given (the forward ran the gate).
        """
        if self.fused:
            raise RuntimeError("backward needs the unfused forward (Xp and unweighted Yp)")
        T, d, E, k, F = self.T, self.d, self.E, self.k, self.F
        dev = self.y.device
        if not hasattr(self, "dYp"):
            Rmax = self.Xp.shape[0]
            self.dw = torch.empty(T, k, dtype=torch.float32, device=dev)
            self.dYp = torch.empty(Rmax, d, dtype=self.dtype, device=dev)
            self.dH = None if self.identity_experts else torch.empty(Rmax, F, dtype=self.dtype,
                                                                     device=dev)
            self.dXp = self.dYp if self.identity_experts else torch.empty(
                Rmax, d, dtype=self.dtype, device=dev)
            self.dx = torch.empty(T, d, dtype=self.dtype, device=dev)
            self.dlogits = torch.empty(T, E, dtype=torch.float32, device=dev)
            self.dbias = torch.empty(E, dtype=torch.float32, device=dev)
            self.dW1 = None if self.identity_experts else torch.empty(E, F, d, dtype=torch.float32,
                                                                      device=dev)
            self.dW2 = None if self.identity_experts else torch.empty(E, d, F, dtype=torch.float32,
                                                                      device=dev)
            self.dWg = torch.empty(E, d, dtype=torch.float32, device=dev)
            self.gate_ws = torch.empty(
                max(moe_gate_backward_workspace_size(T, d, E, self.dtype), 1), dtype=torch.uint8,
                device=dev)
        moe_combine_backward(dy, self.Yp, k, self.slot_row, self.w, self.dw, self.dYp, stream)
        if not self.identity_experts:
            moe_expert_ffn_backward(self.Xp, self.H, self.dYp, W1, W2, self.offsets, self.dH,
                                    self.dXp, self.dW1 if weight_grads else None,
                                    self.dW2 if weight_grads else None, stream)
        moe_dispatch_backward(self.dXp, k, self.slot_row, self.dx, stream)
        moe_route_backward(self.ids, self.w, self.dw, E, self.dlogits, self.dbias,
                           self.workspace, stream)
        out = dict(dx=self.dx, dlogits=self.dlogits, dbias=self.dbias)
        if Wg is not None:
            moe_gate_backward(x, Wg, self.dlogits, self.dx,
                              self.dWg if weight_grads else None, self.gate_ws, stream)
            if weight_grads:
                out["dWg"] = self.dWg
        if weight_grads and not self.identity_experts:
            out.update(dW1=self.dW1, dW2=self.dW2)
        return out

    def launches_per_backward(self, gate=True, weight_grads=True) -> int:
        """Kernel launches one backward makes."""
        n = 1 + 1 + 2  # combine, dispatch, route (dlogits + dbias)
        if not self.identity_experts:
            n += 4 if weight_grads else 2
        if gate:
            tc = self.dtype == torch.bfloat16 and self.d % 8 == 0 and self.E % 8 == 0
            if tc:  # plane split, dx GEMM, dWg GEMM (+ slice reduction)
                n += 2
                if weight_grads:
                    # the workspace holds slice partials beyond the 3 bf16 planes
                    # (6 T E bytes, rounded up to 256, + 256) only when sliced
                    planes = (6 * self.T * self.E + 255) // 256 * 256 + 256
                    n += 2 if lib.moe_gate_backward_workspace_size(
                        self.T, self.d, self.E, MOE_DTYPE_BF16) > planes else 1
            else:
                n += 1
                if weight_grads:
                    n += 2 if moe_gate_backward_workspace_size(self.T, self.d, self.E,
                                                               self.dtype) else 1
        return n

    def capture(self, x, Wg=None, W1=None, W2=None, bias=None, logits=None, popularity=True):
        """Records one ``forward`` on these tensors into a CUDA graph and returns it.

        ``graph.replay()`` then reruns the whole layer on whatever the captured
        tensors hold (copy new tokens into ``x`` first).  Capturing runs the
        layer once (torch's warm-up), which advances the popularity window.
        """
        side = torch.cuda.Stream()
        side.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(side):
            self.forward(x, Wg, W1, W2, bias, logits=logits, popularity=popularity)
        torch.cuda.current_stream().wait_stream(side)
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph):
            self.forward(x, Wg, W1, W2, bias, logits=logits, popularity=popularity)
        return graph

    def capture_split(self, x, Wg=None, W1=None, W2=None, bias=None, logits=None,
                      counts_hook=None):
        """Records one step as two CUDA graphs, (route, rest): gate + route, and
        popularity + dispatch + expert FFN + combine.  A multi-rank step
        replays the first, runs the counts exchange (``counts_hook``, e.g. an
        NCCL all_reduce, outside any graph) and replays the second.  Capturing
        runs one step (with the hook), which advances the popularity window."""
        side = torch.cuda.Stream()
        side.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(side):
            self.forward(x, Wg, W1, W2, bias, logits=logits, counts_hook=counts_hook)
        torch.cuda.current_stream().wait_stream(side)
        g_route, g_rest = torch.cuda.CUDAGraph(), torch.cuda.CUDAGraph()
        with torch.cuda.graph(g_route):
            self.forward_route(x, Wg, bias, logits)
        with torch.cuda.graph(g_rest):
            self.forward_rest(x, W1, W2)
        return g_route, g_rest

    def launches_per_forward(self, gate=True, popularity=True) -> int:
        """Kernel launches one forward makes (route is three kernels)."""
        n = 3 + 1  # route, combine
        n += 0 if self.fused else 1  # dispatch
        n += 1 if gate else 0
        n += 1 if popularity else 0
        n += 0 if self.identity_experts else 2
        return n


def capture_concurrent(layers, calls):
    """One CUDA graph that runs ``layers[i].forward(**calls[i])`` for every i,
    each on a stream of its own, so independent batches overlap on the GPU
    (small kernels of one batch fill SMs the other batch's GEMM waves leave
    idle).  Layers that share a popularity window (``share_popularity``) get
    their updates ordered in list order.  Capturing runs every forward once
    (torch's warm-up), which advances the window."""
    main = torch.cuda.current_stream()
    side = torch.cuda.Stream()
    side.wait_stream(main)
    with torch.cuda.stream(side):
        for layer, call in zip(layers, calls):
            layer.forward(**call)
    main.wait_stream(side)
    streams = [torch.cuda.Stream() for _ in layers]
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        cap = torch.cuda.current_stream()
        prev = None
        for layer, call, st in zip(layers, calls, streams):
            st.wait_stream(cap)
            done = torch.cuda.Event()
            with torch.cuda.stream(st):
                def before(counts, wait_for=prev):
                    if wait_for is not None:
                        torch.cuda.current_stream().wait_event(wait_for)

                def after(ev=done):
                    ev.record(torch.cuda.current_stream())

                layer.forward(**call, counts_hook=before, popularity_done=after)
            prev = done
        for st in streams:
            cap.wait_stream(st)
    return graph
