"""Benchmark of the MoE layer hot path: tokens/s on B200, roofline fractions.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]

One step = gate projection, top-k routing with capacity, popularity window
update, dispatch (input encode), expert FC-ReLU-FC and combine (output decode)
over one batch of T tokens, every stage a kernel of libmoe.so behind the C ABI.
Inputs are seeded synthetic tensors of the workload's shapes (workloads.py);
weights are random-init and resident in HBM.  The timed region is bracketed by
a barrier and a device synchronize on both sides and timed with CUDA events on
the launching stream; with N ranks (torchrun, one GPU each, independent
per-rank batches: weak scaling) the time is the max over ranks and the only
collective in a step is the all_reduce of the per-expert counts that keeps the
popularity statistic global.

The headline line is the largest single-GPU workload (fine_grained: T=32768,
d=4096, E=256, k=8, F=1024).  With one rank the line also carries, under
extras.workloads, the same measurement of multistep_window (all 8 steps, the
popularity window and top-8 on) and of the bandwidth sweep at T=65536 with and
without its Zipf bias.

Prints ONE JSON line (rank 0).  ``--impl reference`` times the CPU oracle on a
bounded sample of the same workload instead (rank 0 only).
"""
from __future__ import annotations

import argparse
import datetime
import gc
import json
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from routing_dispatch_expert_fp32_b200 import workloads as wl  # noqa: E402

DEFAULT_WORKLOAD = "fine_grained"
# Peaks used when MEASURED_PEAKS.json is absent (an earlier measurement on this
# kind of B200: STREAM-style copy, cuBLAS bf16 burst and power-capped loop).
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
# A timed region this long, or one that saw the power cap, is judged against
# the sustained tensor peak; a shorter one at full clocks against the burst peak.
SUSTAINED_REGION_MS = 1000.0


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=0, help="timed steps (0: workload default)")
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD, choices=sorted(wl.WORKLOADS))
    ap.add_argument("--tokens", type=int, default=0, help="override T (bw_sweep sizes)")
    ap.add_argument("--no-bias", action="store_true", help="bw_sweep without the Zipf bias")
    ap.add_argument("--experts", type=int, default=0,
                    help="override E (smaller profiling cases of the same shapes)")
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--concurrent", type=int, default=0,
                    help="independent batches in flight on one GPU (one stream each, one CUDA "
                         "graph, popularity updates in order); 1 = one batch at a time; "
                         "0 = by size: 3 when the expert GEMMs of a step are under 0.2 TFLOP "
                         "(their waves leave SMs idle that another batch's kernels fill), 2 for "
                         "identity experts, else 1 (measured slower there)")
    ap.add_argument("--path", default="unfused", choices=["unfused", "fused"],
                    help="fused: gather the first GEMM's rows from x and weight the second "
                         "GEMM's rows (no dispatch pass); bf16 expert layers only")
    ap.add_argument("--no-graph", action="store_true",
                    help="issue the step kernel by kernel instead of replaying a CUDA graph")
    ap.add_argument("--no-extras", action="store_true",
                    help="skip the other workloads, the backward and the f2/f4 timings")
    ap.add_argument("--cpu-seconds", type=float, default=12.0,
                    help="target CPU time of each oracle sample (0: skip the CPU legs)")
    return ap.parse_args()


def workload_of(args) -> wl.Workload:
    w = wl.WORKLOADS[args.workload]
    if args.tokens:
        w = w.with_(T=args.tokens)
    if args.no_bias:
        w = w.with_(zipf_s=None)
    if args.experts:
        w = w.with_(E=args.experts)
    return w


def default_steps(w: wl.Workload) -> int:
    # about 2-4 s of timed work on one B200
    return {"tiny_fp32": 20000, "skewed_drops": 4000, "multistep_window": 400,
            "fine_grained": 300, "bw_sweep": 1000}[w.name]


# the other workloads of the one-rank line: (label, workload, timed steps)
EXTRA_WORKLOADS = [
    ("multistep_window", wl.WORKLOADS["multistep_window"], 96),
    ("bw_sweep_T65536_zipf1.5", wl.WORKLOADS["bw_sweep"], 100),
    ("bw_sweep_T65536_no_bias", wl.WORKLOADS["bw_sweep"].with_(zipf_s=None), 100),
]


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            p = json.load(f)
        out = dict(FALLBACK_PEAKS)
        out.update({k: float(p[k]) for k in FALLBACK_PEAKS if k in p})
        return out, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


GEMM_SOURCES = ["gemm_tc.cu", "tc_ptx.cuh", "grouped.cuh", "common.cuh"]


def gemm_traffic(workload: str, kernel: str):
    """Measured DRAM bytes per launch of the grouped GEMM from profiles/traffic.md,
    or None when missing or taken on different kernel sources."""
    import hashlib
    h = hashlib.sha256()
    for f in GEMM_SOURCES:
        with open(os.path.join(ROOT, "routing_dispatch_expert_fp32_b200", "csrc", f), "rb") as fh:
            h.update(fh.read())
    sha = h.hexdigest()[:16]
    path = os.path.join(ROOT, "profiles", "traffic.md")
    if not os.path.exists(path):
        return None
    for line in open(path):
        cells = [c.strip() for c in line.strip().strip("|").split("|")]
        if len(cells) == 4 and cells[0] == workload and cells[1] == kernel and cells[3] == sha:
            try:
                return int(cells[2])
            except ValueError:
                return None
    return None


def config_of(w: wl.Workload, n: int, fused: bool = False):
    c = {"workload": w.name, "T": w.T, "d": w.d, "E": w.E, "k": w.k, "F": w.F,
         "capacity": w.capacity, "zipf_s": w.zipf_s, "global_batch_tokens": w.T * n,
         "parallelism": f"dp{n}" if n > 1 else "single",
         "l2": "inputs larger than L2: expert weights read every step exceed 126 MB"
               if not w.identity_experts else
               "inputs larger than L2: x and the grouped rows exceed 126 MB"}
    if w.identity_experts:
        c["experts"] = "identity"
    if w.steps > 1:
        c["popularity_window"] = w.W
        c["batches"] = w.steps
    c["path"] = "fused" if fused else "unfused"
    return c


# --------------------------------------------------------------- clocks ---
REASON_BITS = {"sw_power_cap": 0x4, "hw_slowdown": 0x8, "sw_thermal_slowdown": 0x20,
               "hw_thermal_slowdown": 0x40, "hw_power_brake_slowdown": 0x80}
REJECTING = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown")


class ClockSampler:
    """SM clock, throttle reasons and power read (query only) during a timed
    region: NVML from a side thread at about 1-2 kHz, else nvidia-smi every
    200 ms."""

    def __init__(self, cuda_index: int):
        self.cuda_index = cuda_index
        self.nvml = None
        self.samples = []
        try:
            import pynvml
            import torch
            pynvml.nvmlInit()
            uuid = str(torch.cuda.get_device_properties(cuda_index).uuid)
            try:
                h = pynvml.nvmlDeviceGetHandleByUUID(uuid if uuid.startswith("GPU-")
                                                     else "GPU-" + uuid)
            except Exception:
                h = pynvml.nvmlDeviceGetHandleByIndex(cuda_index)
            self.nvml, self.handle = pynvml, h
            self.max_mhz = float(pynvml.nvmlDeviceGetMaxClockInfo(h, pynvml.NVML_CLOCK_SM))
        except Exception:
            self.nvml = None

    # -- NVML thread
    def _loop(self):
        nv, h = self.nvml, self.handle
        reasons_fn = getattr(nv, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
            nv.nvmlDeviceGetCurrentClocksThrottleReasons
        while not self.stop_flag.is_set():
            try:
                sm = nv.nvmlDeviceGetClockInfo(h, nv.NVML_CLOCK_SM)
                rs = reasons_fn(h)
                pw = nv.nvmlDeviceGetPowerUsage(h) / 1000.0
                self.samples.append((time.perf_counter(), float(sm), int(rs), pw))
            except Exception:
                pass
            time.sleep(0.0003)

    def start(self):
        self.samples = []
        self.t0 = time.perf_counter()
        if self.nvml is not None:
            self.old_switch = sys.getswitchinterval()
            sys.setswitchinterval(1e-4)
            self.stop_flag = threading.Event()
            self.thread = threading.Thread(target=self._loop, daemon=True)
            self.thread.start()
            return
        self.proc = None
        try:
            q = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.hw_slowdown,"
                 "clocks_event_reasons.hw_thermal_slowdown,"
                 "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={q}", "--format=csv,noheader,nounits",
                 "-i", str(self.cuda_index), "-lms", "200"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.lines = []
            self.thread = threading.Thread(
                target=lambda: [self.lines.append(x.strip()) for x in self.proc.stdout],
                daemon=True)
            self.thread.start()
        except (OSError, ValueError):
            self.proc = None

    def stop(self):
        dt = time.perf_counter() - self.t0
        if self.nvml is not None:
            self.stop_flag.set()
            self.thread.join(timeout=2)
            sys.setswitchinterval(self.old_switch)
            sm = [s[1] for s in self.samples]
            bits = 0
            for s in self.samples:
                bits |= s[2]
            reasons = sorted(n for n, b in REASON_BITS.items() if bits & b)
            return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": self.max_mhz,
                    "sm_min_mhz": min(sm) if sm else None, "reasons": reasons,
                    "samples": len(sm), "rate_hz": round(len(sm) / dt, 1) if dt > 0 else None,
                    "power_w_max": max(s[3] for s in self.samples) if sm else None,
                    "source": "nvml"}
        if getattr(self, "proc", None) is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"],
                    "samples": 0}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.thread.join(timeout=2)
        sm, mx, reasons, power = [], None, set(), []
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in self.lines:
            f = [x.strip() for x in line.split(",")]
            if len(f) < 7:
                continue
            try:
                sm.append(float(f[0]))
                mx = float(f[1])
                power.append(float(f[2]))
            except ValueError:
                continue
            for name, v in zip(names, f[3:7]):
                if v.lower() == "active":
                    reasons.add(name)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": mx,
                "reasons": sorted(reasons), "samples": len(sm),
                "power_w_max": max(power) if power else None, "source": "nvidia-smi"}


def tensor_peak(peaks, src, clocks, region_ms):
    """The bf16 peak a tensor-bound kernel is judged against: the sustained one
    for a region of a second or more or one that saw the power cap, else the
    burst one."""
    capped = clocks is not None and "sw_power_cap" in clocks.get("reasons", [])
    key = "bf16_tflops_sustained" if (capped or region_ms >= SUSTAINED_REGION_MS) \
        else "bf16_tflops"
    why = ("power cap seen in the region" if capped else
           f"region {region_ms:.0f} ms >= {SUSTAINED_REGION_MS:.0f} ms"
           if region_ms >= SUSTAINED_REGION_MS else
           f"region {region_ms:.0f} ms at full clocks")
    return peaks[key], f"of {src} {key} ({why})"


# ----------------------------------------------------------- reference ---
def cpu_oracle_run(w: wl.Workload, target_s: float, parallel: bool = False):
    """The oracle as it stands on a bounded token sample of the workload:
    gate, route (capacity rescaled to the sample), dispatch, FFN, combine.
    ``parallel`` uses the OpenMP build on every host core."""
    import oracle

    cores = oracle.use_parallel(parallel)
    weights = wl.make_weights(w)
    inp = wl.make_step(w, 0)

    def run(n):
        x = inp["x"][:n]
        cap = 0
        if w.capacity_factor is not None:
            cap = int(np.ceil(float(w.capacity_factor) * n * w.k / w.E))
        t0 = time.perf_counter()
        if w.identity_experts:
            r = oracle.route(inp["logits"][:n], inp["bias"], w.k, cap)
            Xp = oracle.dispatch(x, w.k, r["row_slot"])
            oracle.combine(Xp, n, w.k, r["slot_row"], r["w"])
        else:
            oracle.layer(x, weights.get("Wg"), weights["W1"], weights["W2"], inp["bias"], w.k,
                         cap)
        return time.perf_counter() - t0

    n = min(w.T, 8)
    dt = run(n)
    while dt < target_s / 8 and n < w.T:
        n = min(w.T, n * 4)
        dt = run(n)
    if dt < target_s and n < w.T:
        n = min(w.T, max(n + 1, int(n * target_s / max(dt, 1e-6))))
        dt = run(n)
    oracle.use_parallel(False)
    return n / dt, n, dt, cores


def reference_arm(args, w):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    steps = args.steps or 3
    times = []
    n, cores = 0, 1
    per = args.cpu_seconds / max(1, steps)
    for _ in range(steps):
        _, n, dt, cores = cpu_oracle_run(w, per, parallel=True)
        times.append(dt)
    value = n * len(times) / sum(times)
    line = {"impl": "reference", "metric": "MoE layer tokens/s", "value": value,
            "unit": "tokens/s", "n_gpus": args.gpus, "steps": steps, "warmup": args.warmup,
            "ms_per_step": 1e3 * sum(times) / len(times), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64 (oracle)",
            "data": "synthetic", "config": config_of(w, args.gpus),
            "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": cores, "kind": "oracle",
                             "sample": f"first {n} tokens of the batch per step, whole layer, "
                                       f"OpenMP build on {cores} host threads"},
            "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


# ------------------------------------------------------------------ ours ---
def backward_extras(moe, w, layer, b, weights, stream, torch, reps=20):
    """Times the layer's backward (after a forward of batch b) stage by stage:
    combine, expert FFN (input gradients alone, then with weight gradients),
    dispatch, route and gate backward, each with events around it."""
    dy_np = wl.make_grad(w, 1)
    dy = (torch.from_numpy(dy_np.view(np.int16)).view(torch.bfloat16)
          if dy_np.dtype == np.uint16 else torch.from_numpy(dy_np)).cuda()
    Wg, W1, W2 = weights.get("Wg"), weights.get("W1"), weights.get("W2")
    layer.forward(b["x"], Wg, W1, W2, b["bias"], logits=b.get("logits"), popularity=False)
    layer.backward(dy, b["x"], Wg, W1, W2)  # allocates the gradient buffers
    R = int(layer.offsets[-1].item())
    names = ["combine_bwd", "ffn_bwd_input", "ffn_bwd_weights", "dispatch_bwd", "route_bwd",
             "gate_bwd"]
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(len(names) + 1)]
          for _ in range(reps)]
    for i in range(reps + 3):
        e = ev[i - 3] if i >= 3 else None
        rec = (lambda j: e[j].record(stream)) if e else (lambda j: None)
        rec(0)
        moe.moe_combine_backward(dy, layer.Yp, w.k, layer.slot_row, layer.w, layer.dw, layer.dYp)
        rec(1)
        if not w.identity_experts:
            moe.moe_expert_ffn_backward(layer.Xp, layer.H, layer.dYp, W1, W2, layer.offsets,
                                        layer.dH, layer.dXp, None, None)
        rec(2)
        if not w.identity_experts:
            moe.moe_expert_ffn_backward(layer.Xp, layer.H, layer.dYp, W1, W2, layer.offsets,
                                        layer.dH, layer.dXp, layer.dW1, layer.dW2)
        rec(3)
        moe.moe_dispatch_backward(layer.dXp, w.k, layer.slot_row, layer.dx)
        rec(4)
        moe.moe_route_backward(layer.ids, layer.w, layer.dw, w.E, layer.dlogits, layer.dbias,
                               layer.workspace)
        rec(5)
        if Wg is not None:
            moe.moe_gate_backward(b["x"], Wg, layer.dlogits, layer.dx, layer.dWg, layer.gate_ws)
        rec(6)
    torch.cuda.synchronize()
    ms = np.zeros(len(names))
    for e in ev:
        ms += np.array([e[j].elapsed_time(e[j + 1]) for j in range(len(names))])
    ms /= reps
    es = 2 if w.dtype == "bf16" else 4
    out = {n: {"ms": float(m)} for n, m in zip(names, ms)}
    if not w.identity_experts:
        # the second call redoes the two input-gradient GEMMs, then the two
        # weight-gradient GEMMs: its excess over the first is theirs
        wgt_ms = float(ms[2] - ms[1])
        out["ffn_bwd_weights"] = {"ms_all_four": float(ms[2]), "ms_weight_gemms": wgt_ms}
        out["ffn_bwd_input"]["tflops"] = 4.0 * R * w.d * w.F / (ms[1] * 1e-3) / 1e12
        if wgt_ms > 0:
            out["ffn_bwd_weights"]["tflops"] = 4.0 * R * w.d * w.F / (wgt_ms * 1e-3) / 1e12
    out["combine_bwd"]["gbs"] = (R * w.d * es * 2 + w.T * w.d * es) / (ms[0] * 1e-3) / 1e9
    out["dispatch_bwd"]["gbs"] = (R * w.d * es + w.T * w.d * es) / (ms[3] * 1e-3) / 1e9
    out["route_bwd"]["gbs"] = w.T * w.E * 4 / (ms[4] * 1e-3) / 1e9
    if Wg is not None:
        out["gate_bwd"]["tflops"] = 4.0 * w.T * w.d * w.E / (ms[5] * 1e-3) / 1e12
    out["step_ms"] = float(ms[0] + ms[2:].sum())
    out["R"] = R
    out["note"] = (f"{reps} backward passes after one forward, events around each call; "
                   "step_ms = combine + FFN (all four GEMMs) + dispatch + route + gate")
    return out


def max_over_ranks(dist, ms: float, device) -> float:
    """The slowest rank's time (every rank gets it)."""
    import torch
    t = torch.tensor([ms], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


class Ctx:
    """The process's torch, binding and rank layout."""

    def __init__(self, torch, dist, moe, world, rank, local, args, peaks, peak_src):
        self.torch, self.dist, self.moe = torch, dist, moe
        self.world, self.rank, self.local = world, rank, local
        self.args, self.peaks, self.peak_src = args, peaks, peak_src
        self.hook = (lambda c: dist.all_reduce(c)) if world > 1 else None

    def barrier(self):
        if self.world > 1:
            self.dist.barrier()

    def max_over_ranks(self, ms: float) -> float:
        return ms if self.world == 1 else max_over_ranks(self.dist, ms, "cuda")


def measure(ctx: Ctx, w: wl.Workload, steps: int, warmup: int, full: bool):
    """Times `steps` layer steps of workload w (graph replay on one rank) and a
    stage-by-stage pass; with `full` also the end-to-end path, the backward and
    the f2/f4 kernels.  Returns the fields of the JSON line."""
    torch, moe, args = ctx.torch, ctx.moe, ctx.args
    world, rank = ctx.world, ctx.rank
    peaks = ctx.peaks
    tdt = torch.bfloat16 if w.dtype == "bf16" else torch.float32
    to_dev = lambda a: (torch.from_numpy(a.view(np.int16)).view(torch.bfloat16)  # noqa: E731
                        if a.dtype == np.uint16 else torch.from_numpy(a)).cuda()
    # one layer replicated on every rank (data parallel): the same weights everywhere,
    # a differently seeded batch per rank
    weights = {k: to_dev(v) for k, v in wl.make_weights(w).items()}
    nb = w.steps if w.steps > 1 else 2
    batches = []
    for s in range(nb):
        inp = wl.make_step(w, s, rank)
        batches.append({k: (None if v is None else to_dev(v)) for k, v in inp.items()})
    fused = args.path == "fused"
    layer = moe.MoELayer(w.T, w.d, w.E, w.k, w.F, tdt, capacity=w.capacity, W=w.W, P=w.P,
                         identity_experts=w.identity_experts, fused=fused)
    stream = torch.cuda.current_stream()
    hook = ctx.hook

    def step(i, ev=None, collective=True):
        b = batches[i % nb]
        if ev is None:
            layer.forward(b["x"], weights.get("Wg"), weights.get("W1"), weights.get("W2"),
                          b["bias"], logits=b.get("logits"),
                          counts_hook=hook if collective else None)
            return
        # same calls as MoELayer.forward, with an event after each stage
        ev[0].record(stream)
        logits = b.get("logits")
        if logits is None:
            moe.moe_gate(b["x"], weights["Wg"], layer.logits)
            logits = layer.logits
        ev[1].record(stream)
        moe.moe_route(logits, b["bias"], w.k, w.capacity, layer.ids, layer.w, layer.counts,
                      layer.kept, layer.offsets, layer.slot_row, layer.row_slot,
                      layer.n_dropped, layer.workspace)
        if hook is not None:
            hook(layer.counts)
        moe.moe_popularity_update_dev(layer.counts, layer.hist, layer.step_dev, layer.mean,
                                      layer.P, layer.hot)
        ev[2].record(stream)
        if not layer.fused:
            moe.moe_dispatch(b["x"], w.k, layer.slot_row, layer.Xp)
        ev[3].record(stream)
        if layer.fused:
            moe.moe_expert_ffn_gather(b["x"], w.k, layer.row_slot, layer.w, weights["W1"],
                                      weights["W2"], layer.offsets, layer.H, layer.Yp)
        elif not w.identity_experts:
            moe.moe_expert_ffn(layer.Xp, weights["W1"], weights["W2"], layer.offsets, layer.H,
                               layer.Yp)
        ev[4].record(stream)
        moe.moe_combine(layer.Yp, w.k, layer.slot_row, None if layer.fused else layer.w, layer.y)
        ev[5].record(stream)

    # R per batch (untimed): algorithmic work of each step
    # and U, the tokens with at least one kept slot (input encode reads their rows)
    R_of, U_of = [], []
    for i in range(nb):
        step(i)
        R_of.append(int(layer.offsets[-1].item()))
        U_of.append(int((layer.slot_row >= 0).any(dim=1).sum().item()))
    # CUDA graphs per input batch: one graph of the whole step on one rank; with
    # several ranks two graphs (gate + route, the rest) around the NCCL
    # all_reduce of the counts.
    use_graph = not args.no_graph
    graphs = []
    if use_graph:
        for b in batches:
            call = dict(x=b["x"], Wg=weights.get("Wg"), W1=weights.get("W1"),
                        W2=weights.get("W2"), bias=b["bias"], logits=b.get("logits"))
            graphs.append(layer.capture(**call) if world == 1 else
                          layer.capture_split(**call, counts_hook=hook))

    def run_step(i):
        if not use_graph:
            step(i)
        elif world == 1:
            graphs[i % nb].replay()
        else:
            g_route, g_rest = graphs[i % nb]
            g_route.replay()
            hook(layer.counts)
            g_rest.replay()

    # Concurrent batches (single rank, graphs): `conc` layer instances with
    # their own buffers and one shared popularity window; group g runs
    # batches g*conc .. g*conc+conc-1 (mod nb), one per stream, in one graph.
    conc = args.concurrent
    if conc <= 0:
        if w.identity_experts:
            conc = 2
        else:
            conc = 3 if 4.0 * w.T * w.k * w.d * w.F < 2e11 else 1
    conc = conc if use_graph and world == 1 else 1
    layers = [layer]
    groups = []
    if conc > 1:
        for _ in range(conc - 1):
            extra = moe.MoELayer(w.T, w.d, w.E, w.k, w.F, tdt, capacity=w.capacity, W=w.W,
                                 P=w.P, identity_experts=w.identity_experts, fused=fused)
            extra.share_popularity(layer)
            layers.append(extra)
        for g in range(max(1, nb // conc)):
            idx = [(g * conc + i) % nb for i in range(conc)]
            calls = [dict(x=batches[j]["x"], Wg=weights.get("Wg"), W1=weights.get("W1"),
                          W2=weights.get("W2"), bias=batches[j]["bias"],
                          logits=batches[j].get("logits")) for j in idx]
            groups.append(moe.capture_concurrent(layers, calls))

    def run_group(g):
        groups[g % len(groups)].replay()

    for i in range(warmup):
        if conc > 1:
            run_group(i)
        else:
            run_step(i)
    torch.cuda.synchronize()

    # ---- timed region: the step as shipped (graph replay), events on the stream ----
    sampler = ClockSampler(ctx.local) if rank == 0 else None
    ctx.barrier()
    torch.cuda.synchronize()
    if sampler:
        sampler.start()
    t_start = torch.cuda.Event(enable_timing=True)
    t_end = torch.cuda.Event(enable_timing=True)
    t_start.record(stream)
    if conc > 1:  # exactly `steps` steps: whole groups, then single batches
        for g in range(steps // conc):
            run_group(g)
        for i in range(steps % conc):
            run_step(i)
    else:
        for i in range(steps):
            run_step(i)
    t_end.record(stream)
    torch.cuda.synchronize()
    clocks = sampler.stop() if sampler else None
    ctx.barrier()
    elapsed_ms = ctx.max_over_ranks(t_start.elapsed_time(t_end))
    # one batch at a time (the single-stream graphs), for comparison
    seq = None
    if conc > 1:
        seq_steps = min(steps, 1000)
        s0, s1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        torch.cuda.synchronize()
        s0.record(stream)
        for i in range(seq_steps):
            run_step(i)
        s1.record(stream)
        torch.cuda.synchronize()
        seq_ms = s0.elapsed_time(s1)
        seq = {"value": w.T * seq_steps / (seq_ms * 1e-3), "ms_per_step": seq_ms / seq_steps,
               "steps": seq_steps, "note": "the same graphs replayed one batch at a time"}

    # ---- timed region 2: the same calls issued one by one with an event after
    # each stage: per-stage device times and the kernels' roofline numbers ----
    stage_steps = min(steps, 500)
    nev = 6
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(nev)] for _ in range(stage_steps)]
    ctx.barrier()
    torch.cuda.synchronize()
    if sampler:
        sampler.start()
    for i in range(stage_steps):
        step(i, evs[i])
    torch.cuda.synchronize()
    stage_clocks = sampler.stop() if sampler else None
    ctx.barrier()
    stage_ms = np.zeros(nev - 1)
    for e in evs:
        stage_ms += np.array([e[j].elapsed_time(e[j + 1]) for j in range(nev - 1)])
    stage_total_ms = float(stage_ms.sum())
    stage_ms /= stage_steps
    # input encode and output decode alone (the layer holds the stage pass's last batch)
    kernel_times = {}
    if rank == 0 and w.dtype == "bf16":
        kernel_times = permute_kernel_times(ctx, w, layer,
                                            batches[(stage_steps - 1) % nb]["x"], peaks)

    out = {"elapsed_ms": elapsed_ms, "steps": steps,
           "value": w.T * steps * world / (elapsed_ms * 1e-3),
           "ms_per_step": elapsed_ms / steps, "clocks": clocks,
           "gpu_launches": layer.launches_per_forward(gate=not w.logits_direct) * steps,
           "timing": {"value": (f"CUDA-graph replay, {conc} independent batches in flight "
                                "(one stream each, popularity updates in order)")
                      if conc > 1 else "CUDA-graph replay of the whole step"
                      if use_graph and world == 1 else
                      "CUDA-graph replays of gate + route and of the rest of the step around "
                      "the NCCL all_reduce of the counts" if use_graph else
                      "kernels issued one by one (programmatic dependent launch)",
                      "batches_in_flight": conc, "one_batch_at_a_time": seq,
                      "stages_and_roofline": f"{stage_steps} steps issued stage by stage, "
                                             "events between stages",
                      "stage_clocks": stage_clocks}}

    # ---- end to end: pinned host x -> device, layer, y -> pinned host ----
    if full:
        out.update(e2e_measure(ctx, w, steps, nb, batches, weights, layer, layers, conc,
                               use_graph, tdt))

    # ---- next-row kernels: cross-layer correlation + popularity forecast ----
    # Batches 0 and 1 stand for two consecutive layers of the same tokens.
    extras = {}
    if full and rank == 0 and not args.no_extras:
        extras = f2_f4_backward_extras(ctx, w, step, nb, batches, weights, layer, stream)
    out["extras"] = extras
    out["device_error_bits"] = moe.moe_device_error()

    # ---- per-stage numbers and the dominant kernel's roofline ----
    R_mean = float(np.mean([R_of[i % nb] for i in range(stage_steps)]))
    U_mean = float(np.mean([U_of[i % nb] for i in range(stage_steps)]))
    names = ["gate", "route+popularity", "dispatch", "expert_ffn", "combine"]
    es = 2 if w.dtype == "bf16" else 4
    per = {}
    alg = {
        "gate": (2.0 * w.T * w.d * w.E, "flop") if not w.logits_direct else (0, "flop"),
        "route+popularity": (w.T * w.E * 4 + w.T * w.k * 4 * 4 + R_mean * 4, "byte"),
        "dispatch": ((0 if layer.fused else U_mean * w.d * es + R_mean * w.d * es
                      + w.T * w.k * 4), "byte"),
        "expert_ffn": (4.0 * R_mean * w.d * w.F, "flop"),
        "combine": (R_mean * w.d * es + w.T * w.d * es + w.T * w.k * 8, "byte"),
    }
    tc_peak, tc_src = tensor_peak(peaks, ctx.peak_src, stage_clocks, stage_total_ms)
    for j, n in enumerate(names):
        amount, kind = alg[n]
        ms = float(stage_ms[j])
        ent = {"ms": ms}
        if ms > 0 and amount:
            if kind == "flop":
                ent["tflops"] = amount / (ms * 1e-3) / 1e12
                ent["frac_bf16"] = ent["tflops"] / tc_peak
            else:
                ent["gbs"] = amount / (ms * 1e-3) / 1e9
                ent["frac_hbm"] = ent["gbs"] / peaks["hbm_gbs"]
        per[n] = ent
    for name, v in kernel_times.items():
        per[name]["kernel"] = v
    out["stages"] = per
    out["R_mean"] = R_mean
    out["U_mean"] = U_mean
    if w.identity_experts:
        dom = "dispatch" if per["dispatch"]["ms"] >= per["combine"]["ms"] else "combine"
        amount = alg[dom][0]
        roof = {"bound": "hbm", "kernel": f"{dom}_kernel",
                "achieved": amount / (per[dom]["ms"] * 1e-3) / 1e9,
                "peak": peaks["hbm_gbs"], "unit": "GB/s",
                "peak_source": f"of {ctx.peak_src} hbm_gbs",
                "bytes_per_launch": amount}
    else:
        # the grouped GEMM: two launches per step, 2*R*d*F flops each
        launch_ms = per["expert_ffn"]["ms"] / 2
        # the library's rule: R_max / E >= 1024 (dense): 2-CTA pair tiles for
        # the whole 256-row blocks of every group, then 1-CTA tiles for the
        # tails; else pair tiles when 128-row tiles would fill fewer than three
        # waves of SMs, else 1-CTA tiles
        nsm = torch.cuda.get_device_properties(ctx.local).multi_processor_count

        def kernel_for(N):
            if w.dtype != "bf16" or layer.fused:
                return "gemm_tc_kernel"
            if w.T * w.k >= 1024 * w.E:
                return "gemm_tc2_kernel+gemm_tc_kernel"
            tiles = (w.T * w.k // 128 + w.E) * ((N + 255) // 256)
            return "gemm_tc2_kernel" if tiles < 3 * nsm else "gemm_tc_kernel"
        kinds = [kernel_for(N) for N in (w.F, w.d)]
        achieved = 2.0 * R_mean * w.d * w.F / (launch_ms * 1e-3) / 1e12
        roof = {"bound": "tensor", "kernel": kinds[0] if kinds[0] == kinds[1]
                else " | ".join(kinds), "achieved": achieved, "peak": tc_peak,
                "unit": "TFLOP/s", "peak_source": tc_src,
                "frac_burst": achieved / peaks["bf16_tflops"],
                "frac_sustained": achieved / peaks["bf16_tflops_sustained"],
                "flops_per_launch": 2.0 * R_mean * w.d * w.F}
        # mixed bound of the grouped GEMM: every expert's weights are read once
        # per launch (E*d*F*s bytes) besides the rows; experts with few rows
        # are bound by that stream, not by the tensor cores
        weight_bytes = w.E * w.d * w.F * es
        act_bytes = R_mean * (w.d + w.F) * es
        t_hbm = (weight_bytes + act_bytes) / (peaks["hbm_gbs"] * 1e9) * 1e3
        t_tc = 2.0 * R_mean * w.d * w.F / (tc_peak * 1e12) * 1e3
        roof["mixed_bound"] = {
            "hbm_ms_per_launch": t_hbm, "tensor_ms_per_launch": t_tc,
            "binding": "hbm" if t_hbm > t_tc else "tensor",
            "frac_of_binding": max(t_hbm, t_tc) / launch_ms,
            "note": "weights E*d*F*s + rows R*(d+F)*s bytes per launch at the HBM peak vs "
                    "2*R*d*F flops at the tensor peak"}
        if w.dtype == "f32":
            # fp32 FMA peak: 148 SMs x 128 lanes x 2 flop x the max SM clock
            roof["bound"] = "alu"
            roof["kernel"] = "gemm_simt_f32_kernel"
            roof["peak"] = 148 * 128 * 2 * peaks.get("sm_max_mhz", 1965.0) * 1e6 / 1e12
            roof["peak_source"] = "derived fp32 FMA peak: 148 x 128 x 2 x sm_max_mhz"
            roof.pop("frac_burst", None)
            roof.pop("frac_sustained", None)
            roof.pop("mixed_bound", None)
    roof["frac"] = roof["achieved"] / roof["peak"]
    roof["traffic"] = (gemm_traffic(w.name + ("/fused" if layer.fused else ""), roof["kernel"])
                       if roof["kernel"].startswith("gemm_tc") and args.tokens == 0
                       and args.experts == 0 else None)
    out["roofline"] = roof

    # release this workload's device memory before the next one
    del graphs, groups, layers, layer, batches, weights
    gc.collect()
    torch.cuda.synchronize()
    torch.cuda.empty_cache()
    return out


def e2e_measure(ctx, w, steps, nb, batches, weights, layer, layers, conc, use_graph, tdt):
    """The same steps through the public API with every batch's x (and logits)
    copied in from pinned host memory and y copied back, inside the timed region."""
    torch, moe, hook = ctx.torch, ctx.moe, ctx.hook
    stream = torch.cuda.current_stream()
    e2e_steps = max(10, steps // 4)
    host_x = [batches[i]["x"].cpu().pin_memory() for i in range(nb)]
    host_logits = [None if batches[i].get("logits") is None else
                   batches[i]["logits"].cpu().pin_memory() for i in range(nb)]
    host_y = torch.empty(w.T, w.d, dtype=tdt).pin_memory()
    dx = torch.empty_like(batches[0]["x"])
    dlog = None if host_logits[0] is None else torch.empty_like(batches[0]["logits"])
    h2d = host_x[0].numel() * host_x[0].element_size() + (
        0 if dlog is None else host_logits[0].numel() * 4)
    d2h = host_y.numel() * host_y.element_size()

    def e2e_step(i):
        b = batches[i % nb]
        dx.copy_(host_x[i % nb], non_blocking=True)
        if dlog is not None:
            dlog.copy_(host_logits[i % nb], non_blocking=True)
        layer.forward(dx, weights.get("Wg"), weights.get("W1"), weights.get("W2"), b["bias"],
                      logits=dlog, counts_hook=hook)
        host_y.copy_(layer.y, non_blocking=True)

    if use_graph and ctx.world == 1:
        # Two units, each a graph over `conc` batches with its own layer
        # instances and device input buffers; copies run on their own streams
        # so unit u's inputs arrive and unit u-1's outputs leave while the
        # other unit computes (every step still copies its x in and its y out).
        def make_unit(unit_layers, first):
            idx = [(first + i) % nb for i in range(len(unit_layers))]
            xs = [batches[j]["x"].clone() for j in idx]
            lg = [None if batches[j].get("logits") is None else batches[j]["logits"].clone()
                  for j in idx]
            calls = [dict(x=xs[i], Wg=weights.get("Wg"), W1=weights.get("W1"),
                          W2=weights.get("W2"), bias=batches[j]["bias"], logits=lg[i])
                     for i, j in enumerate(idx)]
            if len(unit_layers) > 1:
                g = moe.capture_concurrent(unit_layers, calls)
            else:
                g = unit_layers[0].capture(**calls[0])
            hy = [torch.empty(w.T, w.d, dtype=tdt).pin_memory() for _ in unit_layers]
            return dict(graph=g, idx=idx, xs=xs, lg=lg, layers=unit_layers, hy=hy,
                        comp=None, out=None)

        second = []
        for _ in range(conc):
            extra = moe.MoELayer(w.T, w.d, w.E, w.k, w.F, tdt, capacity=w.capacity, W=w.W,
                                 P=w.P, identity_experts=w.identity_experts, fused=layer.fused)
            extra.share_popularity(layer)
            second.append(extra)
        units = [make_unit(layers, 0), make_unit(second, conc % nb)]
        s_in, s_out = torch.cuda.Stream(), torch.cuda.Stream()

        def e2e_unit(it):
            u = units[it % 2]
            if u["comp"] is not None:
                s_in.wait_event(u["comp"])  # the unit's previous replay has read its inputs
            with torch.cuda.stream(s_in):
                for i, j in enumerate(u["idx"]):
                    u["xs"][i].copy_(host_x[j], non_blocking=True)
                    if u["lg"][i] is not None:
                        u["lg"][i].copy_(host_logits[j], non_blocking=True)
                ev_in = torch.cuda.Event()
                ev_in.record(s_in)
            stream.wait_event(ev_in)
            if u["out"] is not None:
                stream.wait_event(u["out"])  # its previous outputs have left
            u["graph"].replay()
            u["comp"] = torch.cuda.Event()
            u["comp"].record(stream)
            s_out.wait_event(u["comp"])
            with torch.cuda.stream(s_out):
                for L, hy in zip(u["layers"], u["hy"]):
                    hy.copy_(L.y, non_blocking=True)
                u["out"] = torch.cuda.Event()
                u["out"].record(s_out)

        e2e_steps = (e2e_steps + conc - 1) // conc * conc
        for it in range(4):
            e2e_unit(it)
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(s_in)
        for it in range(e2e_steps // conc):
            e2e_unit(it)
        e1.record(s_out)
        torch.cuda.synchronize()
        note = ("pinned host x in and y out every step, on copy streams that overlap the other "
                "of two alternating graph units")
        del units, second
    else:
        for i in range(3):
            e2e_step(i)
        ctx.barrier()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for i in range(e2e_steps):
            e2e_step(i)
        e1.record(stream)
        torch.cuda.synchronize()
        ctx.barrier()
        note = "pinned host x in and y out every step, in stream order"
    e2e_ms = ctx.max_over_ranks(e0.elapsed_time(e1))
    return {"e2e": {"value": w.T * e2e_steps * ctx.world / (e2e_ms * 1e-3), "unit": "tokens/s",
                    "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "note": note}}


def permute_kernel_times(ctx, w, layer, x, peaks, reps=8, n_rep=5):
    """Input encode and output decode alone: back-to-back launches inside one CUDA
    graph (programmatic launch, as in the step's graph), rotating over enough
    copies of their buffers that a round moves more than twice the L2, so each
    launch streams HBM.  The layer holds the routing of its last batch; the bytes
    are that batch's (U tokens with a kept slot, R kept rows)."""
    torch, moe = ctx.torch, ctx.moe
    es = x.element_size()
    R = int(layer.offsets[-1].item())
    U = int((layer.slot_row >= 0).any(dim=1).sum().item())
    l2 = getattr(torch.cuda.get_device_properties(ctx.local), "L2_cache_size", 126 << 20)
    jobs = {}
    if not layer.fused:
        jobs["dispatch"] = U * w.d * es + R * w.d * es + w.T * w.k * 4
    jobs["combine"] = R * w.d * es + w.T * w.d * es + w.T * w.k * 8
    out = {}
    wts = None if layer.fused else layer.w
    for name, nbytes in jobs.items():
        if nbytes <= 0:
            continue
        n_sets = int(min(16, max(2, -(-2 * l2 // nbytes))))
        if name == "dispatch":
            sets = [(x, layer.Xp)] + [(x.clone(), torch.empty_like(layer.Xp))
                                      for _ in range(n_sets - 1)]
            call = lambda a, b: moe.moe_dispatch(a, w.k, layer.slot_row, b)  # noqa: E731
        else:
            sets = [(layer.Yp, layer.y)] + [(layer.Yp.clone(), torch.empty_like(layer.y))
                                            for _ in range(n_sets - 1)]
            call = lambda a, b: moe.moe_combine(a, w.k, layer.slot_row, wts, b)  # noqa: E731
        for a, b in sets:  # warm: loads the kernels, sets attributes outside the capture
            call(a, b)
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            for _ in range(reps):
                for a, b in sets:
                    call(a, b)
        g.replay()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for _ in range(n_rep):
            g.replay()
        e1.record()
        torch.cuda.synchronize()
        ms = e0.elapsed_time(e1) / (n_rep * reps * n_sets)
        gbs = nbytes / (ms * 1e-3) / 1e9
        out[name] = {"ms": ms, "gbs": gbs, "frac_hbm": gbs / peaks["hbm_gbs"],
                     "bytes_per_launch": nbytes, "launches": n_rep * reps * n_sets,
                     "buffer_sets": n_sets}
        del g, sets
        torch.cuda.empty_cache()
    return out


def f2_f4_backward_extras(ctx, w, step, nb, batches, weights, layer, stream):
    torch, moe = ctx.torch, ctx.moe
    ids_a = torch.empty_like(layer.ids)
    step(0, collective=False)  # rank 0 only: no collective here
    ids_a.copy_(layer.ids)
    step(1 % nb, collective=False)
    C = torch.zeros(w.E, w.E, dtype=torch.int32, device="cuda")
    pred = torch.empty(w.E, device="cuda")
    hot_f = torch.empty(max(w.P, 1), dtype=torch.int32, device="cuda")
    reps = 200
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(3)]
    for _ in range(3):
        moe.moe_correlation_update(ids_a, layer.ids, C)
        moe.moe_popularity_forecast(layer.mean, C, w.k, w.k, pred, w.P, hot_f)
    torch.cuda.synchronize()
    ev[0].record(stream)
    for _ in range(reps):
        moe.moe_correlation_update(ids_a, layer.ids, C)
    ev[1].record(stream)
    for _ in range(reps):
        moe.moe_popularity_forecast(layer.mean, C, w.k, w.k, pred, w.P, hot_f)
    ev[2].record(stream)
    torch.cuda.synchronize()
    corr_ms = ev[0].elapsed_time(ev[1]) / reps
    fc_ms = ev[1].elapsed_time(ev[2]) / reps
    # GShard balancing loss of the last routing call (re-reads the logits)
    logits_last = batches[1 % nb].get("logits")
    if logits_last is None:
        logits_last = layer.logits
    aux_loss = torch.empty(1, device="cuda")
    aux_P = torch.empty(w.E, device="cuda")
    bias_last = batches[1 % nb]["bias"]
    for _ in range(3):
        moe.moe_aux_loss(logits_last, bias_last, w.k, layer.counts, aux_loss, aux_P,
                         layer.workspace)
    ev[0].record(stream)
    for _ in range(reps):
        moe.moe_aux_loss(logits_last, bias_last, w.k, layer.counts, aux_loss, aux_P,
                         layer.workspace)
    ev[1].record(stream)
    torch.cuda.synchronize()
    aux_ms = ev[0].elapsed_time(ev[1]) / reps
    corr_bytes = 2 * w.T * w.k * 4 + 2 * w.E * w.E * 4
    bwd = (None if layer.fused else
           backward_extras(moe, w, layer, batches[1 % nb], weights, stream, torch))
    return {
        "backward": bwd,
        "correlation_update": {"ms": corr_ms, "pairs": w.T * w.k * w.k,
                               "gbs": corr_bytes / (corr_ms * 1e-3) / 1e9},
        "popularity_forecast": {"ms": fc_ms, "E": w.E},
        "aux_loss": {"ms": aux_ms, "value": float(aux_loss.item()),
                     "gbs": w.T * w.E * 4 / (aux_ms * 1e-3) / 1e9},
        "note": "timed separately (200 back-to-back launches each), outside the step",
    }


def workload_summary(w, m):
    """The compact entry of one extra workload in the line."""
    return {"config": config_of(w, 1), "value": m["value"], "unit": "tokens/s",
            "ms_per_step": m["ms_per_step"], "steps": m["steps"], "R_mean": m["R_mean"],
            "roofline": m["roofline"], "stages": m["stages"], "clocks": m["clocks"],
            "stage_clocks": m["timing"]["stage_clocks"],
            "batches_in_flight": m["timing"]["batches_in_flight"],
            "one_batch_at_a_time": m["timing"]["one_batch_at_a_time"],
            "device_error_bits": m["device_error_bits"]}


def main():
    args = parse()
    w = workload_of(args)
    if args.impl == "reference":
        reference_arm(args, w)
        return

    import torch
    import torch.distributed as dist

    from routing_dispatch_expert_fp32_b200 import moe

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    if world > 1:
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    peaks, peak_src = load_peaks()
    ctx = Ctx(torch, dist, moe, world, rank, local, args, peaks, peak_src)
    steps = args.steps or default_steps(w)
    warmup = max(3, args.warmup)

    head = measure(ctx, w, steps, warmup, full=True)
    extras = head.pop("extras")
    headline_default = (args.workload == DEFAULT_WORKLOAD and not args.tokens
                        and not args.no_bias and not args.experts and args.path == "unfused")
    if world == 1 and headline_default and not args.no_extras:
        extras["workloads"] = {}
        for label, w2, st in EXTRA_WORKLOADS:
            extras["workloads"][label] = workload_summary(w2, measure(ctx, w2, st, warmup,
                                                                      full=False))

    if rank == 0:
        cpu = None
        if world == 1 and args.cpu_seconds > 0:
            rate_all, n_all, dt_all, cores = cpu_oracle_run(w, args.cpu_seconds, parallel=True)
            rate_1, n_1, dt_1, _ = cpu_oracle_run(w, args.cpu_seconds, parallel=False)
            cpu = {"value": rate_all, "unit": "tokens/s", "cores": cores, "kind": "oracle",
                   "sample": f"first {n_all} tokens of one batch through the whole layer "
                             f"({dt_all:.1f} s, capacity rescaled to the sample), OpenMP build "
                             f"on {cores} host threads",
                   "one_core": {"value": rate_1, "unit": "tokens/s", "cores": 1,
                                "sample": f"first {n_1} tokens ({dt_1:.1f} s), "
                                          "single-threaded build"}}
        line = {"metric": "MoE layer tokens/s", "value": head["value"], "unit": "tokens/s",
                "n_gpus": world, "steps": steps, "warmup": warmup,
                "ms_per_step": head["ms_per_step"], "higher_is_better": True,
                "scaling": "weak", "vs_baseline": None, "dtype": w.dtype, "data": "synthetic",
                "config": config_of(w, world, args.path == "fused"),
                "e2e": head["e2e"], "gpu_launches": head["gpu_launches"],
                "roofline": head["roofline"], "stages": head["stages"],
                "clocks": head["clocks"], "cpu_baseline": cpu, "timing": head["timing"],
                "extras": extras, "device_error_bits": head["device_error_bits"]}
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
