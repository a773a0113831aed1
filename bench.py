#!/usr/bin/env python
"""Benchmark of the W4A16 MoE layer (one JSON line on stdout).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--path PATH]
                    [--impl ours|reference]

Default workload (the one the tokens/s metric is quoted on): OLMoE-shaped decode, 16 layers of
H=2048, I=1024, E=64 experts all resident, top-8, one token per step, fresh router logits
every step. A step is one token through all 16 layers: for every layer the router, grouping,
gate/up with SiLU*up, down projection and combine (the packer runs offline, before timing).
Weights are drawn on the device (seeded), packed once by the library's packer and stay
resident; per-step activations and logits are pre-generated and resident. The 3.3 GB packed
bank and the per-step routing keep every layer's experts out of L2 between reuses ("inputs
larger than L2").

value: tokens/s over all ranks (each rank runs its own replica: the layer does not shard
across GPUs here), timed with CUDA events around exactly K steps, max over ranks.
e2e: the same steps through the same C ABI with the per-step inputs copied from pinned host
memory and every layer's output copied back, the copies on two copy streams over two buffer
pairs so that they overlap the neighbouring steps' layers; the host waits for every step's
result, one step behind (step i + 1 is queued before the host waits for step i), as a serving
loop would. The timed region runs from before the first input copy to after the last output copy.
roofline: the dominant kernel's algorithmic bytes (distinct routed experts' packed weights and
scales) per launch over its CUDA-event duration, against the measured HBM copy bandwidth.
cpu_baseline: the oracle (plain C++) on the host cores over a bounded sample of the workload.
--impl reference times that oracle as the reference arm.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import moe_inputs as mi  # noqa: E402

METRIC = "W4A16 MoE-layer tokens/s; % of HBM roofline (decode) / tensor peak (prefill)"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
# B200 datasheet figures (HGX HBM3e bandwidth; dense bf16 tensor), reported beside the measured
# peaks, which stay the primary denominators
DATASHEET = {"hbm_gbs": 7700.0, "bf16_tflops": 2250.0}


def expert_bytes(H: int, I: int) -> int:
    codes = 2 * I * H // 2 + H * I // 2
    scales = 2 * (2 * I * (H // 128) + H * (I // 128))
    return codes + scales


PROFILE = os.path.join(ROOT, "profiles", "moe_decode_rows_kernel_olmoe_decode.json")
PROFILE_SOURCES = ["quantized_mixture_experts_grouped_b200/csrc/ffn_decode_rows.cu",
                   "quantized_mixture_experts_grouped_b200/csrc/decode_common.cuh",
                   "quantized_mixture_experts_grouped_b200/csrc/common.cuh",
                   "quantized_mixture_experts_grouped_b200/csrc/tc.cuh"]


def code_of(text: str) -> str:
    """C++/CUDA source without its comments and blank space: what the compiler sees of it (a
    comment-only edit does not change the kernel the profile was taken of). String literals that
    contain comment markers are not special-cased; the profiled sources have none."""
    import re
    text = re.sub(r"/\*.*?\*/", " ", text, flags=re.S)
    text = re.sub(r"//[^\n]*", "", text)
    return "\n".join(" ".join(line.split()) for line in text.splitlines() if line.strip())


def source_hash(files=None) -> str:
    """First 16 hex digits of the SHA-256 of the profiled kernel's source files, in order, with
    comments and blank space removed (code_of)."""
    import hashlib
    files = PROFILE_SOURCES if files is None else files
    code = "\n".join(code_of(open(os.path.join(ROOT, f), encoding="utf-8").read()) for f in files)
    return hashlib.sha256(code.encode()).hexdigest()[:16]


def profiled_traffic():
    """DRAM bytes (read + write) per launch of the decode kernel from the committed ncu record
    (profiles/*.json: "source_hash", "traffic_bytes_per_launch"), or None when the record is
    missing or the kernel's sources changed since the capture."""
    try:
        rec = json.load(open(PROFILE))
        digest = source_hash()
    except (OSError, ValueError):
        return None
    if rec.get("source_hash") != digest or not isinstance(rec.get("traffic_bytes_per_launch"), int):
        return None
    return rec["traffic_bytes_per_launch"]


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


# ----------------------------------------------------------------------------- clocks

class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.path = None

    def start(self):
        fd, self.path = tempfile.mkstemp(prefix="clocks_", suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.FIELDS}",
                                          "--format=csv,noheader,nounits", "-lms", "200"],
                                         stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except (OSError, FileNotFoundError):
            self.proc = None

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"], "samples": 0}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        rows = []
        for line in open(self.path):
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                rows.append(parts)
            except ValueError:
                pass
        os.unlink(self.path)
        sm = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        mx = [float(r[2]) for r in rows if r[2].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[5 + i].lower() == "active"})
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": reasons, "samples": len(rows)}


# ----------------------------------------------------------------------------- distributed

def dist_setup(args):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        backend = "nccl" if (args.impl == "ours" and torch.cuda.is_available()) else "gloo"
        if backend == "nccl":
            torch.cuda.set_device(local)
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=600))
    elif torch.cuda.is_available():
        torch.cuda.set_device(local)
    return rank, world, local


def all_max(x: float, world: int) -> float:
    if world == 1:
        return x
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier(world: int):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


# ----------------------------------------------------------------------------- CPU oracle

class OracleLayer:
    """One layer of the workload packed by the oracle on the host (CPU baseline / reference)."""

    def __init__(self, wl: mi.Workload, layer: int, experts):
        import oracle
        self.oracle = oracle
        self.wl = wl
        self.w13 = np.zeros((wl.E, oracle.packed_bytes(2 * wl.I, wl.H)), np.uint8)
        self.s13 = np.zeros((wl.E, oracle.scale_count(2 * wl.I, wl.H)), np.uint16)
        self.w2 = np.zeros((wl.E, oracle.packed_bytes(wl.H, wl.I)), np.uint8)
        self.s2 = np.zeros((wl.E, oracle.scale_count(wl.H, wl.I)), np.uint16)
        for e in experts:
            a, b = mi.expert_weights(wl, layer, e)
            self.w13[e], self.s13[e] = oracle.pack(*oracle.quantize(a))
            self.w2[e], self.s2[e] = oracle.pack(*oracle.quantize(b))

    def forward(self, x, logits, threads: int):
        idx, wts = self.oracle.route(logits, self.wl.k)
        return self.oracle.moe_ffn(x, idx, wts, self.w13, self.s13, self.w2, self.s2, self.wl.H, self.wl.I,
                                   n_threads=threads)


def oracle_threads(wl: mi.Workload) -> int:
    return max(1, min(os.cpu_count() or 1, wl.T * wl.k))


def cpu_baseline(wl: mi.Workload, budget_s: float = 12.0):
    """Oracle tokens/s over a bounded sample: one layer (the routed experts of one logits draw,
    packed by the oracle), forwards repeated for about budget_s, scaled by the layer count."""
    logits = mi.router_logits(wl, 0, 0)
    import oracle
    idx, _ = oracle.route(logits, wl.k)
    layer = OracleLayer(wl, 0, sorted(set(idx.ravel().tolist())))
    x = mi.activations(wl, 0, 0)
    threads = oracle_threads(wl)
    layer.forward(x, logits, threads)
    reps, t0 = 0, time.perf_counter()
    while True:
        layer.forward(x, logits, threads)
        reps += 1
        el = time.perf_counter() - t0
        if el >= budget_s or reps >= 1000:
            break
    per_layer = el / reps
    value = wl.T / (per_layer * wl.layers)
    return {"value": value, "unit": "tokens/s", "cores": threads, "kind": "oracle",
            "sample": f"{reps} forwards of one {wl.name} layer (T={wl.T}, routed experts packed by the oracle), "
                      f"{per_layer * 1e3:.1f} ms each, scaled to {wl.layers} layers per token"}


def run_reference(args, wl: mi.Workload, rank: int, world: int):
    if rank != 0:
        return
    if wl.layers == 1:
        run_reference_tokens(args, wl, world)
        return
    import oracle
    threads = oracle_threads(wl)
    steps_total = args.warmup + args.steps
    logits_all = [[mi.router_logits(wl, l, s) for l in range(wl.layers)] for s in range(steps_total)]
    needed = set()
    for s in range(steps_total):
        for l in range(wl.layers):
            needed |= set(oracle.route(logits_all[s][l], wl.k)[0].ravel().tolist())
    layer = OracleLayer(wl, 0, sorted(needed))
    x = mi.activations(wl, 0, 0)
    # size each step so that the whole run stays near two minutes: a step runs `per_step` of
    # the workload's layers and counts as per_step / layers of a token
    t0 = time.perf_counter()
    layer.forward(x, logits_all[0][0], threads)
    t_layer = time.perf_counter() - t0
    per_step = int(max(1, min(wl.layers, round(120.0 / steps_total / max(t_layer, 1e-6)))))
    for s in range(args.warmup):
        for l in range(per_step):
            layer.forward(x, logits_all[s][l], threads)
    t0 = time.perf_counter()
    for s in range(args.warmup, steps_total):
        for l in range(per_step):
            layer.forward(x, logits_all[s][l], threads)
    el = time.perf_counter() - t0
    value = wl.T * args.steps * per_step / wl.layers / el
    line = {"metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": el / args.steps * 1e3, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic", "impl": "reference",
            "config": config_of(wl, args, "oracle"),
            "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": threads, "kind": "oracle",
                             "sample": f"every step = {per_step} of the {wl.layers} layer forwards of a token "
                                       f"(one {wl.name} layer's packed bank, T={wl.T}, fresh logits per layer "
                                       f"and step) on the host cores"},
            "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def run_reference_tokens(args, wl: mi.Workload, world: int):
    """Reference arm of a one-layer, large-batch workload: the routing of all T tokens is taken
    once and the experts it selects are packed by the oracle; each step then runs the oracle on
    the next `per_step` consecutive tokens of the layer, sized so that the whole run stays near
    two minutes."""
    import oracle
    logits = mi.router_logits(wl, 0, 0)
    idx, wts = oracle.route(logits, wl.k)
    layer = OracleLayer(wl, 0, sorted(set(idx.ravel().tolist())))
    x = mi.activations(wl, 0, 0)
    threads = max(1, os.cpu_count() or 1)
    steps_total = args.warmup + args.steps
    pos = [0]

    def step(n):
        start = pos[0] if pos[0] + n <= wl.T else 0
        toks = np.arange(start, start + n, dtype=np.int32)
        oracle.moe_ffn(x, idx, wts, layer.w13, layer.s13, layer.w2, layer.s2, wl.H, wl.I, tokens=toks,
                       n_threads=threads)
        pos[0] = start + n

    probe = min(8, wl.T)
    t0 = time.perf_counter()
    step(probe)
    t_tok = (time.perf_counter() - t0) / probe
    per_step = int(max(1, min(wl.T, round(120.0 / steps_total / max(t_tok, 1e-9)))))
    for _ in range(args.warmup):
        step(per_step)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        step(per_step)
    el = time.perf_counter() - t0
    value = per_step * args.steps / el
    line = {"metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": el / args.steps * 1e3, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic", "impl": "reference",
            "config": config_of(wl, args, "oracle"),
            "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": threads, "kind": "oracle",
                             "sample": f"every step = {per_step} consecutive tokens of one {wl.name} layer "
                                       f"(T={wl.T}, the routing of all its tokens, experts packed by the "
                                       f"oracle) on the host cores"},
            "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def config_of(wl: mi.Workload, args, path: str):
    return {"workload": wl.name, "weights": getattr(args, "weights", "w4a16"), "layers": wl.layers, "hidden": wl.H, "intermediate": wl.I, "experts": wl.E,
            "top_k": wl.k, "tokens_per_step": wl.T, "slots": wl.slots or wl.E, "routing": wl.routing,
            "path": path, "l2": "inputs larger than L2 (packed bank of all layers, fresh routing per step)"}


# ----------------------------------------------------------------------------- GPU arm

class DecodeBench:
    """All layers resident; per-step inputs resident; one CUDA graph per distinct step."""

    RING = 32   # distinct step inputs (fresh routing each); replayed cyclically

    def __init__(self, wl: mi.Workload, path: str, device, weights: str = "w4a16"):
        import quantized_mixture_experts_grouped_b200 as q
        self.q, self.wl, self.dev = q, wl, device
        self.flags = q.PATHS[path]
        self.bf16 = weights == "bf16"
        H, I, E, k, T, Ls = wl.H, wl.I, wl.E, wl.k, wl.T, wl.layers
        self.banks = []
        for l in range(Ls):
            w13b, w2b = mi.device_bank_weights(wl, l, device)
            if self.bf16:        # the BF16 comparison: unquantised experts
                self.banks.append((w13b, None, w2b, None))
                continue
            w13, s13 = q.alloc_bank(E, 2 * I, H, device)
            w2, s2 = q.alloc_bank(E, H, I, device)
            q.moe_quantize_pack(w13b, w13, s13)
            q.moe_quantize_pack(w2b, w2, s2)
            del w13b, w2b
            self.banks.append((w13, s13, w2, s2))
        torch.cuda.synchronize()
        R = self.RING
        # per ring slot, per layer: x [T][H] and logits [T][E], one contiguous block per slot
        self.in_elems = Ls * (T * H + T * E)
        host = np.empty((R, self.in_elems), np.uint16)
        for r in range(R):
            parts = []
            for l in range(Ls):
                parts.append(mi.activations(wl, l, r).ravel())
                parts.append(mi.router_logits(wl, l, r).ravel())
            host[r] = np.concatenate(parts)
        self.inputs_host = torch.from_numpy(host.view(np.int16)).view(torch.bfloat16).pin_memory()
        self.inputs = self.inputs_host.to(device)
        # two staging / output buffer pairs (end to end): step i uses pair i % 2
        self.staging = [torch.empty(self.in_elems, dtype=torch.bfloat16, device=device) for _ in range(2)]
        self.out = torch.empty((R, Ls, T, H), dtype=torch.bfloat16, device=device)
        self.out_e2e = [torch.empty((Ls, T, H), dtype=torch.bfloat16, device=device) for _ in range(2)]
        # two pinned result buffers: the host reads step i's result while step i + 1 runs
        self.out_host = torch.empty((2, Ls, T, H), dtype=torch.bfloat16).pin_memory()
        self.done = [torch.cuda.Event(), torch.cuda.Event()]
        self.pending = None
        self.idx = torch.empty((Ls, T, k), dtype=torch.int32, device=device)
        self.wts = torch.empty((Ls, T, k), dtype=torch.float32, device=device)
        self.ws = q.alloc_workspace(T, H, I, E, k, device)
        self.stream = torch.cuda.Stream(device)

    def _views(self, buf, l):
        wl = self.wl
        off = l * (wl.T * wl.H + wl.T * wl.E)
        x = buf[off: off + wl.T * wl.H].view(wl.T, wl.H)
        lg = buf[off + wl.T * wl.H: off + wl.T * wl.H + wl.T * wl.E].view(wl.T, wl.E)
        return x, lg

    def _layers(self, buf, out, events=None):
        q, wl = self.q, self.wl
        for l in range(wl.layers):
            x, lg = self._views(buf, l)
            w13, s13, w2, s2 = self.banks[l]
            if events is not None:
                events[2 * l].record(self.stream)
            if self.bf16:
                q.moe_bf16_layer(x, lg, wl.k, w13, w2, wl.H, wl.I, self.idx[l], self.wts[l], self.ws, out[l],
                                 flags=self.flags, stream=self.stream)
            else:
                q.moe_w4a16_layer(x, lg, wl.k, w13, s13, w2, s2, wl.H, wl.I, self.idx[l], self.wts[l], self.ws,
                                  out[l], flags=self.flags, stream=self.stream)
            if events is not None:
                events[2 * l + 1].record(self.stream)

    def capture(self):
        q = self.q
        self.graphs = []
        torch.cuda.synchronize()
        with torch.cuda.stream(self.stream):
            self._layers(self.inputs[0], self.out[0])          # warm: lazy init outside capture
        self.stream.synchronize()
        n0 = q.moe_launch_count()
        for r in range(self.RING):
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=self.stream):
                self._layers(self.inputs[r], self.out[r])
            self.graphs.append(g)
        self.launches_per_step = (q.moe_launch_count() - n0) // self.RING
        # the same steps with an event pair around every layer (kernel timing pass)
        self.ev = []
        self.ev_graphs = []
        for r in range(self.RING):
            evs = [torch.cuda.Event(enable_timing=True, external=True) for _ in range(2 * self.wl.layers)]
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=self.stream):
                self._layers(self.inputs[r], self.out[r], evs)
            self.ev.append(evs)
            self.ev_graphs.append(g)
        # end-to-end: the layers read the step's inputs from a staging buffer that each step
        # fills from pinned host memory; every layer's output goes back to pinned host memory
        self.e2e_graphs = []
        for b in range(2):
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=self.stream):
                self._layers(self.staging[b], self.out_e2e[b])
            self.e2e_graphs.append(g)
        self.h2d_stream = torch.cuda.Stream(self.stream.device)
        self.d2h_stream = torch.cuda.Stream(self.stream.device)
        self.in_ready = [torch.cuda.Event(), torch.cuda.Event()]
        self.computed = [torch.cuda.Event(), torch.cuda.Event()]
        torch.cuda.synchronize()

    def e2e_step(self, r):
        """One step end to end: its inputs from pinned host memory (copy stream), the layers
        (compute stream), its outputs back to pinned host memory (second copy stream). Buffer
        pair r % 2 is reused once step r - 2 has been computed and copied out, so the copies of
        neighbouring steps overlap the layers. The host then waits for the previous step's
        result: it reads every step's result, one step behind."""
        b = r % 2
        with torch.cuda.stream(self.h2d_stream):
            self.h2d_stream.wait_event(self.done[b])          # step r - 2 copied out of pair b
            self.staging[b].copy_(self.inputs_host[r % self.RING], non_blocking=True)
            self.in_ready[b].record(self.h2d_stream)
        self.stream.wait_event(self.in_ready[b])
        self.e2e_graphs[b].replay()
        self.computed[b].record(self.stream)
        with torch.cuda.stream(self.d2h_stream):
            self.d2h_stream.wait_event(self.computed[b])
            self.out_host[b].copy_(self.out_e2e[b], non_blocking=True)
            self.done[b].record(self.d2h_stream)
        self.e2e_drain()
        self.pending = b

    def e2e_drain(self):
        """Waits until the host can read the last queued step's result."""
        if self.pending is not None:
            self.done[self.pending].synchronize()
            self.pending = None

    def distinct_experts_mean(self) -> float:
        """Mean number of distinct experts the ring's logits select per layer (top-k by bf16 logit
        descending, id ascending): the experts whose packed bytes one layer launch must read."""
        wl, tot = self.wl, 0
        for r in range(self.RING):
            for l in range(wl.layers):
                lg = mi.bf16_bits_to_f32(mi.router_logits(wl, l, r))
                order = np.lexsort((np.broadcast_to(np.arange(wl.E), lg.shape), -lg), axis=-1)[:, :wl.k]
                tot += len(np.unique(order))
        return tot / (self.RING * wl.layers)

    def run(self, graphs, n, start=0):
        for i in range(n):
            graphs[(start + i) % self.RING].replay()

    def h2d_bytes(self):
        return self.in_elems * 2

    def d2h_bytes(self):
        return self.out_e2e[0].numel() * 2


def run_ours(args, wl: mi.Workload, rank: int, world: int, local: int):
    device = torch.device("cuda", local)
    bench = DecodeBench(wl, args.path, device, args.weights)
    bench.capture()
    s = bench.stream
    peaks, peaks_kind = load_peaks()
    sampler = ClockSampler(local)
    with torch.cuda.stream(s):
        bench.run(bench.graphs, args.warmup)
        s.synchronize()
        sampler.start()
        # keep the GPU busy ~1.5 s so the clock sampler sees the regime the timed steps run in
        t0 = time.perf_counter()
        i = 0
        while time.perf_counter() - t0 < 1.5:
            bench.run(bench.graphs, 64, i)
            s.synchronize()
            i += 64
        barrier(world)
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(s)
        bench.run(bench.graphs, args.steps, args.warmup)
        e1.record(s)
        e1.synchronize()
        torch.cuda.synchronize()
        barrier(world)
        clocks = sampler.stop()
        ms_total = all_max(e0.elapsed_time(e1), world)

        # kernel timing pass: per-layer event pairs (one launch of the fused kernel per layer)
        bench.run(bench.ev_graphs, max(3, args.warmup))
        s.synchronize()
        nk = max(args.steps, bench.RING)
        durs = []
        for i in range(nk):
            r = i % bench.RING
            bench.ev_graphs[r].replay()
            s.synchronize()
            evs = bench.ev[r]
            durs.extend(evs[2 * l].elapsed_time(evs[2 * l + 1]) for l in range(wl.layers))
        layer_ms = statistics.fmean(durs)

        # end to end through host buffers
        for i in range(max(3, args.warmup)):
            bench.e2e_step(i)
        bench.e2e_drain()
        barrier(world)
        f0, f1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        f0.record(s)
        bench.h2d_stream.wait_event(f0)      # the first timed input copy starts after f0
        for i in range(args.steps):
            bench.e2e_step(args.warmup + i)
        f1.record(bench.d2h_stream)          # after the last step's outputs are in host memory
        f1.synchronize()
        bench.e2e_drain()
        e2e_ms = all_max(f0.elapsed_time(f1), world)
    status = bench.q.moe_workspace_status(bench.ws, s)
    distinct_mean = bench.distinct_experts_mean()
    h2d_bytes, d2h_bytes = bench.h2d_bytes(), bench.d2h_bytes()

    launches_per_layer = bench.launches_per_step / wl.layers
    del bench
    torch.cuda.empty_cache()
    # the prefill layer measured in the same process (a figure for the tensor-bound side)
    secondary = None
    if not args.no_secondary and wl.name == "olmoe_decode" and wl.T == 1 and args.weights == "w4a16":
        pw = mi.WORKLOADS["olmoe_prefill"]
        r = measure_single_layer(pw, "auto", 20, 3, world, local)
        secondary = {"workload": pw.name, "us_per_layer": r["ms"] * 1e3, "tokens_per_s": pw.T * world / (r["ms"] / 1e3),
                     "e2e_tokens_per_s": pw.T * world / (r["e2e_ms"] / 1e3),
                     "achieved_tflops": r["achieved"], "peak_tflops": r["peak"], "frac": r["achieved"] / r["peak"],
                     "frac_datasheet": r["achieved"] / DATASHEET["bf16_tflops"],
                     "peak_kind": f"{r['peaks_kind']} bf16 dense (burst)", "steps": 20, "warmup": 3,
                     "clocks": r["clocks"], "device_status": r["status"]}
    if rank != 0:
        return
    tokens = wl.T * args.steps * world
    value = tokens / (ms_total / 1e3)
    per_expert = (2 * (3 * wl.H * wl.I)) if args.weights == "bf16" else expert_bytes(wl.H, wl.I)
    bytes_per_layer = distinct_mean * per_expert
    # duration of the one launch of a layer: the timed step over its layers (the launches of a
    # step run back to back, so this includes the gap between two launches)
    us_layer = ms_total / args.steps / wl.layers * 1e3
    achieved = bytes_per_layer / (us_layer / 1e6) / 1e9
    hbm_peak = float(peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"]))
    line = {
        "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_total / args.steps, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": dict(config_of(wl, args, args.path), us_per_layer=ms_total / args.steps / wl.layers * 1e3),
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": hbm_peak, "unit": "GB/s",
                     "frac": achieved / hbm_peak, "frac_datasheet": achieved / DATASHEET["hbm_gbs"],
                     "traffic": profiled_traffic() if (wl.T == 1 and args.path in ("auto", "decode")) else None,
                     "kernel": ("moe_decode_rows_kernel" if wl.T == 1 else "moe_decode_mma_kernel")
                               + " (the one launch per layer; duration = timed step / layers)"
                               if args.path in ("auto", "decode") and args.weights == "w4a16"
                               else "all launches of the layer (timed step / layers)",
                     "algorithmic_bytes_per_launch": bytes_per_layer, "us_per_launch": us_layer,
                     "launches_per_layer": launches_per_layer,
                     "us_per_launch_event_pair": layer_ms * 1e3,
                     "peak_kind": f"{peaks_kind} HBM copy"},
        "e2e": {"value": tokens / (e2e_ms / 1e3), "unit": "tokens/s", "h2d_bytes_per_step": h2d_bytes,
                "d2h_bytes_per_step": d2h_bytes},
        "gpu_launches": int(launches_per_layer * wl.layers) * args.steps,
        "clocks": clocks,
        "device_status": status,
    }
    if secondary is not None:
        line["secondary"] = secondary
    if world == 1 and not args.no_cpu_baseline and args.weights == "w4a16":
        line["cpu_baseline"] = cpu_baseline(wl)
    print(json.dumps(line), flush=True)


# ----------------------------------------------------------------------------- one-layer workloads

def cpu_baseline_tokens(wl: mi.Workload, budget_s: float = 12.0):
    """Oracle tokens/s for a one-layer workload over a bounded sample of its tokens (the layer's
    experts packed by the oracle; tokens taken in order until about budget_s of work)."""
    import oracle
    logits = mi.router_logits(wl, 0, 0)
    idx, wts = oracle.route(logits, wl.k)
    layer = OracleLayer(wl, 0, sorted(set(idx.ravel().tolist())))
    x = mi.activations(wl, 0, 0)
    threads = max(1, os.cpu_count() or 1)
    done, t_used, n = 0, 0.0, 1
    while t_used < budget_s and done < wl.T:
        toks = np.arange(done, min(wl.T, done + n), dtype=np.int32)
        t0 = time.perf_counter()
        oracle.moe_ffn(x, idx, wts, layer.w13, layer.s13, layer.w2, layer.s2, wl.H, wl.I, tokens=toks,
                       n_threads=threads)
        t_used += time.perf_counter() - t0
        done += len(toks)
        n = min(2 * n, 64)
    return {"value": done / t_used, "unit": "tokens/s", "cores": threads, "kind": "oracle",
            "sample": f"the first {done} of the {wl.T} tokens of one {wl.name} layer ({t_used:.1f} s of oracle "
                      f"work, experts packed by the oracle)"}


def measure_single_layer(wl: mi.Workload, path: str, steps: int, warmup: int, world: int, local: int,
                         weights: str = "w4a16") -> dict:
    """Large-batch workloads (prefill, large expert): one layer of T tokens per step through
    moe_w4a16_layer (route, permute, gather, two grouped GEMMs, combine), timed with CUDA events
    (max over ranks) with inputs resident, then end to end with host copies every step."""
    import quantized_mixture_experts_grouped_b200 as q
    device = torch.device("cuda", local)
    H, I, E, k, T = wl.H, wl.I, wl.E, wl.k, wl.T
    w13b, w2b = mi.device_bank_weights(wl, 0, device)
    bf16 = weights == "bf16"
    if bf16:               # the BF16 comparison: unquantised experts
        w13, s13, w2, s2 = w13b, None, w2b, None
    else:
        w13, s13 = q.alloc_bank(E, 2 * I, H, device)
        w2, s2 = q.alloc_bank(E, H, I, device)
        q.moe_quantize_pack(w13b, w13, s13)
        q.moe_quantize_pack(w2b, w2, s2)
    del w13b, w2b
    x_host = torch.from_numpy(mi.activations(wl, 0, 0).view(np.int16)).view(torch.bfloat16).pin_memory()
    lg_host = torch.from_numpy(mi.router_logits(wl, 0, 0).view(np.int16)).view(torch.bfloat16).pin_memory()
    x, lg = x_host.to(device), lg_host.to(device)
    idx = torch.empty((T, k), dtype=torch.int32, device=device)
    wts = torch.empty((T, k), dtype=torch.float32, device=device)
    out = torch.empty((T, H), dtype=torch.bfloat16, device=device)
    ws = q.alloc_workspace(T, H, I, E, k, device)
    # end to end: two buffer sets (inputs on the device, outputs on the device and in pinned host
    # memory), step i uses set i % 2; copies on two copy streams overlap the neighbouring steps
    xs2 = [torch.empty_like(x) for _ in range(2)]
    lgs2 = [torch.empty_like(lg) for _ in range(2)]
    outs2 = [torch.empty_like(out) for _ in range(2)]
    out_host = [torch.empty((T, H), dtype=torch.bfloat16).pin_memory() for _ in range(2)]
    flags = q.PATHS[path]
    s = torch.cuda.Stream(device)
    peaks, peaks_kind = load_peaks()
    sampler = ClockSampler(local)

    def call(xx, ll, oo=out):
        if bf16:
            q.moe_bf16_layer(xx, ll, k, w13, w2, H, I, idx, wts, ws, oo, flags=flags, stream=s)
        else:
            q.moe_w4a16_layer(xx, ll, k, w13, s13, w2, s2, H, I, idx, wts, ws, oo, flags=flags, stream=s)

    h2d, d2h = torch.cuda.Stream(device), torch.cuda.Stream(device)
    in_ready = [torch.cuda.Event(), torch.cuda.Event()]
    computed = [torch.cuda.Event(), torch.cuda.Event()]
    done = [torch.cuda.Event(), torch.cuda.Event()]
    pending = [None]

    def e2e_step(i):
        """Inputs up (copy stream), the layer, the output back (second copy stream); the host
        waits for the previous step's output, one step behind."""
        b = i % 2
        with torch.cuda.stream(h2d):
            h2d.wait_event(done[b])            # step i - 2 is computed and copied out of set b
            xs2[b].copy_(x_host, non_blocking=True)
            lgs2[b].copy_(lg_host, non_blocking=True)
            in_ready[b].record(h2d)
        s.wait_event(in_ready[b])
        call(xs2[b], lgs2[b], outs2[b])
        computed[b].record(s)
        with torch.cuda.stream(d2h):
            d2h.wait_event(computed[b])
            out_host[b].copy_(outs2[b], non_blocking=True)
            done[b].record(d2h)
        if pending[0] is not None:
            done[pending[0]].synchronize()
        pending[0] = b

    with torch.cuda.stream(s):
        n0 = q.moe_launch_count()
        call(x, lg)
        launches = q.moe_launch_count() - n0
        for _ in range(warmup):
            call(x, lg)
        s.synchronize()
        sampler.start()
        t0 = time.perf_counter()
        while time.perf_counter() - t0 < 1.0:
            call(x, lg)
            s.synchronize()
        barrier(world)
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(s)
        for _ in range(steps):
            call(x, lg)
        e1.record(s)
        e1.synchronize()
        barrier(world)
        clocks = sampler.stop()
        ms = all_max(e0.elapsed_time(e1), world) / steps
        # end to end: inputs from pinned host memory, output back to the host, every step
        for i in range(warmup):
            e2e_step(i)
        done[pending[0]].synchronize()
        pending[0] = None
        s.synchronize()
        barrier(world)
        f0, f1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        f0.record(s)
        h2d.wait_event(f0)                     # the first timed input copy starts after f0
        for i in range(steps):
            e2e_step(warmup + i)
        f1.record(d2h)                         # after the last step's output is in host memory
        f1.synchronize()
        e2e_ms = all_max(f0.elapsed_time(f1), world) / steps
    status = q.moe_workspace_status(ws, s)
    flops = 6.0 * H * I * T * k
    achieved = flops / (ms / 1e3) / 1e12
    peak = float(peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"]))
    res = dict(ms=ms, e2e_ms=e2e_ms, clocks=clocks, status=status, launches=launches, achieved=achieved,
               peak=peak, peaks_kind=peaks_kind, h2d=(x.numel() + lg.numel()) * 2, d2h=out.numel() * 2)
    del w13, s13, w2, s2, ws, xs2, lgs2, outs2
    torch.cuda.empty_cache()
    return res


def run_single_layer(args, wl: mi.Workload, rank: int, world: int, local: int):
    r = measure_single_layer(wl, args.path, args.steps, args.warmup, world, local, args.weights)
    if rank != 0:
        return
    T, ms, e2e_ms, achieved, peak = wl.T, r["ms"], r["e2e_ms"], r["achieved"], r["peak"]
    line = {
        "metric": METRIC, "value": T * world / (ms / 1e3), "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": dict(config_of(wl, args, args.path), us_per_layer=ms * 1e3,
                       l2="inputs larger than L2 (packed bank of the layer)"),
        "roofline": {"bound": "tensor", "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
                     "frac": achieved / peak, "frac_datasheet": achieved / DATASHEET["bf16_tflops"], "traffic": None,
                     "kernel": "whole layer (route, permute, gather, gate/up and down grouped GEMMs, combine): "
                               "6*H*I*T*k flop over the layer's event-timed duration",
                     "peak_kind": f"{r['peaks_kind']} bf16 dense (burst)"},
        "e2e": {"value": T * world / (e2e_ms / 1e3), "unit": "tokens/s",
                "h2d_bytes_per_step": r["h2d"], "d2h_bytes_per_step": r["d2h"]},
        "gpu_launches": r["launches"] * args.steps,
        "clocks": r["clocks"],
        "device_status": r["status"],
    }
    if world == 1 and not args.no_cpu_baseline and args.weights == "w4a16":
        line["cpu_baseline"] = cpu_baseline_tokens(wl)
    print(json.dumps(line), flush=True)


def run_slots(args, wl: mi.Workload, rank: int, world: int, local: int):
    """Batched decode through the GPU slot cache: every layer keeps S of its E experts on the
    device, the rest in a pinned host bank; each layer call routes, reads the routed set back to
    the host, refills misses by cudaMemcpyAsync on a copy stream and runs the FFN in waves."""
    import quantized_mixture_experts_grouped_b200 as q
    device = torch.device("cuda", local)
    H, I, E, k, T, S, Ls = wl.H, wl.I, wl.E, wl.k, wl.T, wl.slots, wl.layers
    caches = []
    for l in range(Ls):
        w13b, w2b = mi.device_bank_weights(wl, l, device)
        d13, ds13 = q.alloc_bank(E, 2 * I, H, device)
        d2, ds2 = q.alloc_bank(E, H, I, device)
        q.moe_quantize_pack(w13b, d13, ds13)
        q.moe_quantize_pack(w2b, d2, ds2)
        del w13b, w2b
        bank = q.alloc_bank(E, 2 * I, H, pinned=True) + q.alloc_bank(E, H, I, pinned=True)
        for hst, dev in zip(bank, (d13, ds13, d2, ds2)):
            hst.copy_(dev)
        del d13, ds13, d2, ds2
        pool = q.alloc_bank(S, 2 * I, H, device) + q.alloc_bank(S, H, I, device)
        caches.append(q.SlotCache(E, S, H, I, bank, pool))
        if l == 0:
            bank0 = bank
    torch.cuda.synchronize()
    R = 8    # distinct step inputs, replayed cyclically
    xs = torch.stack([torch.stack([torch.from_numpy(mi.activations(wl, l, r).view(np.int16)) for l in range(Ls)])
                      for r in range(R)]).view(torch.bfloat16).to(device)
    lgs = torch.stack([torch.stack([torch.from_numpy(mi.router_logits(wl, l, r).view(np.int16)) for l in range(Ls)])
                       for r in range(R)]).view(torch.bfloat16).to(device)
    steps_total = args.warmup + args.steps
    idx_all = torch.empty((steps_total, Ls, T, k), dtype=torch.int32, device=device)
    wts = torch.empty((T, k), dtype=torch.float32, device=device)
    out = torch.empty((Ls, T, H), dtype=torch.bfloat16, device=device)
    wave_tables = torch.empty(E * ((E + S - 1) // S + 1), dtype=torch.int32, device=device)
    ws = q.alloc_workspace(T, H, I, E, k, device)
    s, cs = torch.cuda.Stream(device), torch.cuda.Stream(device)
    flags = q.PATHS[args.path]
    loads = [0]
    waves = [0]

    def step(i):
        r = i % R
        for l in range(Ls):
            nw, nl = caches[l].layer(xs[r, l], lgs[r, l], k, idx_all[i, l], wts, wave_tables, ws, out[l], flags,
                                     stream=s, copy_stream=cs)
            loads[0] += nl
            waves[0] += nw

    # the refills' own copy rate on this machine (their bound): the pattern of moe_slot_cache_layer,
    # four copies per expert (W13 codes and scales, W2 codes and scales) from the pinned bank,
    # here 2 S experts into a scratch pool of S slots, timed on the copy stream
    scratch = q.alloc_bank(S, 2 * I, H, device) + q.alloc_bank(S, H, I, device)

    def refill_pattern():
        for e in range(2 * S):
            for hst, dev in zip(bank0, scratch):
                dev[e % S].copy_(hst[e % E], non_blocking=True)

    with torch.cuda.stream(cs):
        refill_pattern()
        c0, c1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        c0.record(cs)
        for _ in range(4):
            refill_pattern()
        c1.record(cs)
        c1.synchronize()
    h2d_peak = 4 * 2 * S * expert_bytes(H, I) / (c0.elapsed_time(c1) / 1e3) / 1e9
    del scratch
    sampler = ClockSampler(local)
    with torch.cuda.stream(s):
        for i in range(args.warmup):
            step(i)
        s.synchronize()
        loads[0] = waves[0] = 0
        n0 = q.moe_launch_count()
        sampler.start()
        barrier(world)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(s)
        for i in range(args.warmup, steps_total):
            step(i)
        e1.record(s)
        e1.synchronize()
        clocks = sampler.stop()
        ms = all_max(e0.elapsed_time(e1), world) / args.steps
        launches = (q.moe_launch_count() - n0) // args.steps
        status = q.moe_workspace_status(ws, s)
        loads_t, waves_t = loads[0], waves[0]
        # the same steps with the refill copies left out (dry run: waves planned and committed
        # as before, FFNs on whatever the pool holds): the time of everything but the copies,
        # for the fraction of the copy time that the overlap hides
        for c in caches:
            c.dry_run(True)
        barrier(world)
        e0.record(s)
        for i in range(args.warmup, steps_total):
            step(i)
        e1.record(s)
        e1.synchronize()
        ms_nocopy = all_max(e0.elapsed_time(e1), world) / args.steps
        for c in caches:
            c.dry_run(False)
    if rank != 0:
        return
    idx_h = idx_all[args.warmup:].cpu().numpy()
    needed = sum(len(np.unique(idx_h[i, l])) for i in range(args.steps) for l in range(Ls))
    h2d_bytes = loads_t * expert_bytes(H, I)
    h2d_gbs = h2d_bytes / (args.steps * ms / 1e3) / 1e9
    copy_ms = h2d_bytes / args.steps / (h2d_peak * 1e9) * 1e3
    hidden = max(0.0, min(1.0, (copy_ms + ms_nocopy - ms) / max(1e-9, min(copy_ms, ms_nocopy))))
    line = {
        "metric": METRIC, "value": T * world / (ms / 1e3), "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": dict(config_of(wl, args, args.path), us_per_layer=ms / Ls * 1e3,
                       l2="pinned host bank of all layers, 16 device slots per layer"),
        "memory": {"slot_pool_bytes": Ls * S * expert_bytes(H, I), "pinned_bank_bytes": Ls * E * expert_bytes(H, I),
                   "resident_fraction": S / E, "device_peak_reserved_bytes": torch.cuda.max_memory_reserved(device)},
        "slot_cache": {"hit_rate": 1.0 - loads_t / max(1, needed), "misses_per_layer_step": loads_t / (args.steps * Ls),
                       "distinct_per_layer_step": needed / (args.steps * Ls), "waves_per_layer_step": waves_t / (args.steps * Ls),
                       "h2d_gbs": h2d_gbs, "h2d_peak_gbs": h2d_peak,
                       # copies alone (at the refill pattern's measured rate), everything else alone (dry run),
                       # and the share of the shorter of the two hidden under the other
                       "overlap": {"copy_ms": copy_ms, "other_ms": ms_nocopy, "step_ms": ms,
                                   "hidden_fraction": hidden},
                       # the compute part alone: the distinct experts' bytes over the dry-run step
                       # (routing, host read-back and every wave's FFN, no copies)
                       "compute_hbm_gbs": needed * expert_bytes(H, I) / args.steps / (ms_nocopy / 1e3) / 1e9,
                       "compute_hbm_frac": needed * expert_bytes(H, I) / args.steps / (ms_nocopy / 1e3) / 1e9
                                           / float(load_peaks()[0].get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"]))},
        "roofline": {"bound": "h2d", "achieved": h2d_gbs, "peak": h2d_peak, "unit": "GB/s",
                     "frac": h2d_gbs / h2d_peak, "traffic": None,
                     "kernel": "refill copies (cudaMemcpyAsync, pinned host -> slot pool) over the step time",
                     "peak_kind": "the refill copy pattern (4 copies per expert, pinned bank -> device) measured in this run"},
        "e2e": {"value": T * world / (ms / 1e3), "unit": "tokens/s", "h2d_bytes_per_step": h2d_bytes // args.steps,
                "d2h_bytes_per_step": Ls * 8 * ((E + 63) // 64)},
        "gpu_launches": launches * args.steps,
        "clocks": clocks,
        "device_status": status,
    }
    if world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(wl)
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="olmoe_decode",
                    choices=["olmoe_decode", "olmoe_slots", "olmoe_prefill", "large_expert"])
    ap.add_argument("--path", default="auto", choices=["auto", "simple", "decode", "grouped", "sequential"])
    ap.add_argument("--weights", default="w4a16", choices=["w4a16", "bf16"],
                    help="bf16: the same layer on unquantised experts (the BF16 comparison)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-secondary", action="store_true",
                    help="skip the prefill layer measured after the default decode workload")
    ap.add_argument("--layers", type=int, default=None,
                    help="fewer layers than the workload's (profiling runs only; the metric uses 16)")
    ap.add_argument("--routing", default=None, choices=["normal", "zipf"],
                    help="router logits: N(0,1) or Zipf(1.1) popularity + Gumbel (default: the workload's)")
    ap.add_argument("--tokens", type=int, default=None,
                    help="tokens per step other than the workload's (ablations; the metric uses the default)")
    args = ap.parse_args()
    args.warmup = max(3, args.warmup)
    wl = mi.WORKLOADS[args.workload]
    if args.layers is not None:
        import dataclasses
        wl = dataclasses.replace(wl, layers=max(1, args.layers))
    if args.tokens is not None:
        import dataclasses
        wl = dataclasses.replace(wl, T=max(1, args.tokens))
    if args.routing is not None:
        import dataclasses
        wl = dataclasses.replace(wl, routing=args.routing)
    rank, world, local = dist_setup(args)
    try:
        if args.impl == "reference":
            run_reference(args, wl, rank, world)
        elif wl.T > 16:
            run_single_layer(args, wl, rank, world, local)
        elif wl.slots:
            run_slots(args, wl, rank, world, local)
        else:
            run_ours(args, wl, rank, world, local)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
