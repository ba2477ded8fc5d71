#!/usr/bin/env python
"""Benchmark of the mixed W4/W8 x A8 linear layers on B200.

One step = one pass of the hot path over a whole synthetic model: for every
decoder layer, the per-token INT8 quantization of the four distinct projection
inputs (attention input shared by q/k/v, attention output, MLP input shared
by gate/up, MLP hidden) and the seven linear projections, all launched through
the C ABI and replayed as one CUDA graph.  Weights are random, packed once,
and resident in HBM; the per-step weight stream (1.8 GB for the default
workload) is far larger than the 126 MB L2, so no explicit L2 flush is done.

Default workload (N = 1): Llama-3.2-3B-shaped decode (hidden 3072, 24 q / 8 kv
heads x 128, MLP 8192, 28 layers), 128 x 128 tiles, 25% INT8 tiles, M = 1
token; M = 8 and 32 are reported alongside.  The headline value is decode HBM
throughput on packed-weight bytes (GB/s).  A Qwen3-4B-shaped prefill (M = 2048,
40% INT8 tiles, 1% outlier channels) is measured as well and reported in INT8
TOPS.

Multi-GPU (torchrun): the path has no data-path exchange, so every rank runs
an independent replica of the workload (weak scaling); the job value is the
bytes all ranks streamed over the max-over-ranks time.
"""
from __future__ import annotations

import argparse
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

METRIC = "mixed W4/W8A8 linear: decode HBM GB/s, prefill INT8 TOPS (% of roofline)"

WORKLOADS = {
    "decode-llama-3.2-3b": dict(model="llama-3.2-3b", phase="decode", bN=128, frac8=0.25, M=1, extra_M=(8, 32),
                                outlier=0.0),
    "prefill-qwen3-4b": dict(model="qwen3-4b", phase="prefill", bN=128, frac8=0.40, M=2048, extra_M=(),
                             outlier=0.01),
    "decode-single-2048": dict(model="single-2048", phase="decode", bN=128, frac8=0.5, M=1, extra_M=(16,),
                               outlier=0.0),
    "decode-dense-8b": dict(model="dense-8b", phase="decode", bN=128, frac8=0.5, M=1, extra_M=(16, 64),
                            outlier=0.0),
    "prefill-dense-8b": dict(model="dense-8b", phase="prefill", bN=128, frac8=0.5, M=4096, extra_M=(),
                             outlier=0.0),
    "decode-qwen3-14b": dict(model="qwen3-14b", phase="decode", bN=128, frac8=0.30, M=1, extra_M=(16, 64),
                             outlier=0.0),
    "prefill-qwen3-14b": dict(model="qwen3-14b", phase="prefill", bN=128, frac8=0.30, M=8192, extra_M=(),
                              outlier=0.01),
}
# DRAM traffic per launch (dram__bytes_read.sum + dram__bytes_write.sum) of the dominant kernels,
# from an ncu capture of the named workload, valid only while the kernel source is unchanged
# (sha256 prefix of the source file and the shared header).
MEASURED_TRAFFIC = {
    # one Llama-3.2-3B layer's four decode launches at 1 token read 64,740,608 B and wrote
    # 23,808 B -> 16,191,104 B per launch (algorithmic: 16,128,638 B per launch)
    "decode": {"src": ("w8_a8_quantized_b200/csrc/decode_rows.cu", "w8_a8_quantized_b200/csrc/aq_internal.cuh"),
               "sha": "9ff17c3bbdb451a8", "bytes_per_launch": 16191104},
    "prefill": {"src": ("w8_a8_quantized_b200/csrc/tc_linear.cu", "w8_a8_quantized_b200/csrc/aq_internal.cuh"),
                "sha": None, "bytes_per_launch": None},
}


def measured_traffic(phase: str):
    import hashlib
    rec = MEASURED_TRAFFIC[phase]
    if rec["sha"] is None:
        return None
    h = hashlib.sha256()
    for f in rec["src"]:
        with open(os.path.join(ROOT, f), "rb") as fh:
            h.update(fh.read())
    return rec["bytes_per_launch"] if h.hexdigest()[:16] == rec["sha"] else None


CFG_ID = {"llama-3.2-3b": 2, "qwen3-4b": 3, "dense-8b": 4, "qwen3-14b": 5, "single-2048": 1}
INPUT_OF = {"q": "attn_in", "k": "attn_in", "v": "attn_in", "o": "attn_out", "gate": "mlp_in", "up": "mlp_in",
            "down": "mlp_hidden"}


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)  # ~0.25 s timed at 1 token: several clock samples
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="aq", choices=["aq", "reference"])
    ap.add_argument("--workload", default="decode-llama-3.2-3b", choices=sorted(WORKLOADS))
    ap.add_argument("--no-prefill", action="store_true", help="skip the secondary prefill measurement")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--tokens", type=int, default=None, help="measure only this token count")
    ap.add_argument("--no-e2e", action="store_true", help="skip the host-buffer end-to-end measurement")
    ap.add_argument("--layers", type=int, default=None,
                    help="build only the first N layers (small cases for profiling; the line records the count)")
    return ap.parse_args()


# ----------------------------------------------------------------------------- peaks
def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            p = json.load(f)
        return dict(hbm=p["hbm_gbs"], bf16=p["bf16_tflops"], bf16_sust=p["bf16_tflops_sustained"], src="measured")
    return dict(hbm=6650.0, bf16=1590.0, bf16_sust=1400.0, src="fallback")


# ----------------------------------------------------------------------------- clocks
class ClockSampler:
    """nvidia-smi sampling (every 50 ms) of SM clock and throttle reasons while running."""
    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.lines = []

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.Q}",
                                          "--format=csv,noheader,nounits", "-lms", "50"],
                                         stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.t = threading.Thread(target=self._read, daemon=True)
            self.t.start()
        except OSError:
            self.proc = None
        return self

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def __exit__(self, *exc):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self):
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            f = [x.strip() for x in ln.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                mx = float(f[2])
            except ValueError:
                continue
            for n, v in zip(names, f[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm)}


# ----------------------------------------------------------------------------- model
class Model:
    """Packed random weights and synthetic activations of one workload on one GPU."""

    def __init__(self, wl: dict, M: int, device, rank: int, layers=None):
        import torch
        from w8_a8_quantized_b200 import aq, synth
        self.torch, self.aq = torch, aq
        self.wl, self.M, self.dev = wl, M, device
        model = wl["model"]
        cfg = CFG_ID[model]
        self.layers = synth.MODELS[model]["layers"] if layers is None else min(layers, synth.MODELS[model]["layers"])
        self.projs = synth.projections(model)
        self.weights = []
        self.weight_bytes = 0
        self.macs = 0
        for l in range(self.layers):
            layer = {}
            for pid, (name, N, K) in enumerate(self.projs):
                p = synth.projection_inputs(N, K, wl["bN"], 128, wl["frac8"], (cfg, l, pid))
                w = aq.aq_pack(torch.from_numpy(p.codes).to(device), torch.from_numpy(p.scales).to(device),
                               torch.from_numpy(p.pmap).to(device), wl["bN"], 128)
                layer[name] = w
                self.weight_bytes += w.nbytes
                self.macs += N * K
            self.weights.append(layer)
        self.in_dims = {}
        for name, N, K in self.projs:
            self.in_dims[INPUT_OF[name]] = K
        self.out_dims = {name: N for name, N, K in self.projs}
        self.set_tokens(M)

    def set_tokens(self, M: int):
        torch, aq = self.torch, self.aq
        from w8_a8_quantized_b200 import synth
        self.M = M
        cfg = CFG_ID[self.wl["model"]]
        self.x = []  # per layer: input kind -> bf16 [M, K] on device
        self.x_host = []
        # decode: distinct activations for every layer; prefill: a pool of 4 distinct
        # activation sets cycled over the layers (each set is far larger than a tile)
        n_sets = self.layers if self.wl["phase"] == "decode" else min(4, self.layers)
        for l in range(n_sets):
            d, h = {}, {}
            for kind, K in self.in_dims.items():
                bits = synth.activations(M, K, (cfg, l, 100 + sorted(self.in_dims).index(kind), M),
                                         outlier_frac=self.wl["outlier"])
                h[kind] = torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).pin_memory()
                d[kind] = h[kind].to(self.dev)
            self.x.append(d)
            self.x_host.append(h)
        self.x = [self.x[l % n_sets] for l in range(self.layers)]
        self.x_host_sets = self.x_host
        self.xq = {k: torch.empty((M, K), dtype=torch.int8, device=self.dev) for k, K in self.in_dims.items()}
        self.sx = {k: torch.empty((M,), dtype=torch.float32, device=self.dev) for k in self.in_dims}
        self.y = {n: torch.empty((M, N), dtype=torch.float32, device=self.dev) for n, N in self.out_dims.items()}
        self.phase = aq.AQ_PHASE_DECODE if self.wl["phase"] == "decode" else aq.AQ_PHASE_PREFILL
        self.members = {}
        for name, _, _ in self.projs:
            self.members.setdefault(INPUT_OF[name], []).append(name)
        self.groups = [{kind: aq.Group([self.weights[l][n] for n in names], self.phase, M)
                        for kind, names in self.members.items()} for l in range(self.layers)]
        need = max([g.ws.numel() for layer in self.groups for g in layer.values()] +
                   [aq.aq_workspace_bytes(self.phase, M, w) for layer in self.weights for w in layer.values()])
        for layer in self.groups:
            for g in layer.values():
                g.ws = None  # one shared workspace (the step runs in stream order)
        self.ws = torch.zeros(need, dtype=torch.uint8, device=self.dev)
        self.run = aq.aq_linear_decode if self.phase == aq.AQ_PHASE_DECODE else aq.aq_linear_prefill
        # long-prefill variant: one temporary all-INT8 copy buffer, reused by every projection
        self.tmp = None
        if self.phase == aq.AQ_PHASE_PREFILL:
            need = max(aq.aq_expanded_bytes(w) for layer in self.weights for w in layer.values())
            self.tmp = torch.empty(need + 256, dtype=torch.uint8, device=self.dev)
        # groups run as one fused launch (activation preparation inside) up to 2 tokens; from
        # 3 tokens on as one preparation launch plus one grouped CUDA-core launch (up to 4 tokens,
        # or up to 8 for groups of three or more) or one tensor-core launch per member
        self.fused = self.phase == aq.AQ_PHASE_DECODE and M <= 2

    def step(self, mode="group"):
        """Enqueue one pass; returns the number of kernel launches.

        mode "group": the hot path, one aq_linear_group call per shared input
        (query/key/value, attention output, gate/up, MLP hidden) per layer.
        mode "linear": only the linear kernels on already-quantized inputs.
        mode "expanded": as "linear", through the long-prefill variant (each projection
        expanded to a temporary INT8 copy, then the pure INT8 GEMM)."""
        aq = self.aq
        n = 0
        for l, kind in [(l, kind) for l in range(self.layers) for kind in self.members]:
            names = self.members[kind]
            if mode == "group":
                self.groups[l][kind](self.x[l][kind], [self.y[nm] for nm in names], ws=self.ws)
                rows = self.phase == aq.AQ_PHASE_DECODE and (self.M <= 4 or (len(names) >= 3 and self.M <= 8))
                n += 1 if self.fused else 1 + (1 if rows else len(names))  # fused, or quantize + members
            elif mode == "expanded":
                for nm in names:
                    aq.aq_linear_prefill_expanded(self.weights[l][nm], self.xq[kind], self.sx[kind],
                                                  out=self.y[nm], ws=self.ws, tmp=self.tmp)
                    n += 2
            else:
                for nm in names:
                    self.run(self.weights[l][nm], self.xq[kind], self.sx[kind], out=self.y[nm], ws=self.ws)
                    n += 1
        return n

    def quantize_inputs(self):
        """Fill the pre-quantized inputs used by mode "linear" (from layer 0's activations)."""
        for kind in self.members:
            self.aq.aq_quant_act(self.x[0][kind], self.xq[kind], self.sx[kind])

    def graph(self, **kw):
        torch = self.torch
        s = torch.cuda.Stream(self.dev)
        s.wait_stream(torch.cuda.current_stream(self.dev))
        with torch.cuda.stream(s):
            self.step(**kw)
        torch.cuda.current_stream(self.dev).wait_stream(s)
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            launches = self.step(**kw)
        return g, launches


def max_over_ranks(torch, value: float, device) -> float:
    """The largest of every rank's value; every rank calls it at the same point."""
    t = torch.tensor([value], dtype=torch.float64, device=device)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def job_rate(world: int, units_per_rank: float, ms: float, scale: float) -> float:
    """Whole-job throughput: the units all ranks processed (each rank the same
    amount: independent replicas) over the slowest rank's time, in units of `scale`."""
    return world * units_per_rank / (ms * 1e-3) / scale


def time_graph(torch, g, steps, warmup, dist_on, dev):
    for _ in range(warmup):
        g.replay()
    torch.cuda.synchronize(dev)
    if dist_on:
        torch.distributed.barrier()
    torch.cuda.synchronize(dev)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.nvtx.range_push("aq_timed")
    e0.record()
    for _ in range(steps):
        g.replay()
    e1.record()
    torch.cuda.nvtx.range_pop()
    torch.cuda.synchronize(dev)
    if dist_on:
        torch.distributed.barrier()
    ms = e0.elapsed_time(e1) / steps
    if dist_on:
        ms = max_over_ranks(torch, ms, dev)
    return ms


def time_e2e(torch, model, g, steps, warmup, dev):
    """Same metric through the public API with host buffers: every step copies its
    activations host->device from pinned memory, replays the step and reads the
    last layer's outputs back to pinned host memory."""
    h2d = sum(t.numel() * 2 for layer in model.x_host_sets for t in layer.values())
    outs = [model.y[n] for n in model.out_dims]
    host_out = [torch.empty(o.shape, dtype=o.dtype, pin_memory=True) for o in outs]
    d2h = sum(o.numel() * o.element_size() for o in outs)

    def one():
        for l, layer in enumerate(model.x_host_sets):
            for kind, t in layer.items():
                model.x[l][kind].copy_(t, non_blocking=True)
        g.replay()
        for o, h in zip(outs, host_out):
            h.copy_(o, non_blocking=True)

    for _ in range(warmup):
        one()
    torch.cuda.synchronize(dev)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(steps):
        one()
    e1.record()
    torch.cuda.synchronize(dev)
    return e0.elapsed_time(e1) / steps, h2d, d2h


# ----------------------------------------------------------------------------- CPU oracle
def oracle_run(wl, budget_s, M):
    """Time the CPU oracle on a bounded sample of the workload: whole projections
    of the first layers (unpack of the packed form, activation quantization,
    integer tile products, fp64 rescale), until `budget_s` seconds are used.
    Returns (units done, seconds, description)."""
    import oracle
    from w8_a8_quantized_b200 import synth
    cfg = CFG_ID[wl["model"]]
    projs = synth.projections(wl["model"])
    layers = synth.MODELS[wl["model"]]["layers"]
    done_bytes = done_macs = 0
    n_proj = 0
    rows = M if wl["phase"] == "decode" else min(M, 64)
    t_used = 0.0
    for l in range(layers):
        for pid, (name, N, K) in enumerate(projs):
            p = synth.projection_inputs(N, K, wl["bN"], 128, wl["frac8"], (cfg, l, pid))
            pk = oracle.pack(p.codes, p.scales, p.pmap, wl["bN"], 128)
            x = synth.activations(rows, K, (cfg, l, 999, rows), outlier_frac=wl["outlier"])
            t0 = time.perf_counter()
            xq, sx = oracle.quant_act(x)
            oracle.linear_packed(pk, xq, sx)
            t_used += time.perf_counter() - t0
            done_bytes += oracle.packed_bytes(pk)
            done_macs += N * K * rows
            n_proj += 1
            if t_used >= budget_s:
                break
        if t_used >= budget_s:
            break
    desc = (f"{n_proj} whole projections of the first layer(s) of the workload, {rows} token(s) each, "
            f"unpack + quantize + tile products + fp64 rescale")
    return done_bytes, done_macs, t_used, desc


def cpu_threads():
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 1) for i in threadpool_info() if i.get("user_api") == "blas"]
        return max(n) if n else 1
    except Exception:
        return os.cpu_count() or 1


# ----------------------------------------------------------------------------- main
def main():
    args = parse()
    wl = WORKLOADS[args.workload]
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    peaks = load_peaks()

    if args.impl == "reference":
        if rank != 0:
            return 0
        return run_reference(args, wl, peaks)

    import torch
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    dist_on = world > 1
    if dist_on:
        import datetime
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                             device_id=dev)
    from w8_a8_quantized_b200 import aq
    aq.lib()

    Ms = [wl["M"], *wl["extra_M"]] if args.tokens is None else [args.tokens]
    t_setup = time.time()
    model = Model(wl, Ms[0], dev, rank, args.layers)
    setup_s = time.time() - t_setup

    results = {}
    clocks = None
    for M in Ms:
        if M != model.M:
            model.set_tokens(M)
        g, launches = model.graph()
        if M == Ms[0]:
            with ClockSampler(local) as cs:
                ms = time_graph(torch, g, args.steps, args.warmup, dist_on, dev)
            clocks = cs.summary()
        else:
            ms = time_graph(torch, g, args.steps, args.warmup, dist_on, dev)
        if model.fused:  # the step holds nothing but the dominant (fused decode) kernel
            g_lin, lin_launches, ms_lin = None, launches, ms
        else:
            model.quantize_inputs()
            g_lin, lin_launches = model.graph(mode="linear")
            ms_lin = time_graph(torch, g_lin, args.steps, args.warmup, dist_on, dev)
        res = dict(ms=ms, launches=launches, ms_linear_only=ms_lin, linear_launches=lin_launches)
        if M == Ms[0]:
            if args.no_e2e:
                res.update(ms_e2e=float("nan"), h2d=0, d2h=0)
            else:
                ms_e2e, h2d, d2h = time_e2e(torch, model, g, args.steps, args.warmup, dev)
                if dist_on:  # every rank times it, the slowest one counts
                    ms_e2e = max_over_ranks(torch, ms_e2e, dev)
                res.update(ms_e2e=ms_e2e, h2d=h2d, d2h=d2h)
        results[M] = res
        aq.check_all_workspaces()
        rc, info = aq.aq_workspace_status(model.ws)
        if rc != 0:
            raise RuntimeError(f"kernel reported error {rc} ({info})")
        del g, g_lin

    r0 = results[Ms[0]]
    decode = wl["phase"] == "decode"
    wbytes = model.weight_bytes
    if decode:
        unit = "GB/s"
        value = job_rate(world, wbytes, r0["ms"], 1e9)
        achieved = wbytes / (r0["ms_linear_only"] * 1e-3) / 1e9
        roof = {"bound": "hbm", "achieved": achieved, "peak": peaks["hbm"], "unit": "GB/s",
                "frac": achieved / peaks["hbm"], "traffic": measured_traffic("decode"),
                "algorithmic_bytes_per_launch": wbytes / r0["linear_launches"],
                "kernel": "decode linear (all projections, activation quantization excluded)",
                "peak_source": peaks["src"]}
        e2e_val = job_rate(world, wbytes, r0["ms_e2e"], 1e9)
    else:
        unit = "TOPS"
        ops = 2.0 * model.M * model.macs
        value = job_rate(world, ops, r0["ms"], 1e12)
        achieved = ops / (r0["ms_linear_only"] * 1e-3) / 1e12
        int8_peak = 2.0 * peaks["bf16"]  # dense INT8 = 2x dense BF16 (nominal ratio 4.5 / 2.25)
        roof = {"bound": "tensor", "achieved": achieved, "peak": int8_peak, "unit": "TFLOP/s",
                "frac": achieved / int8_peak, "traffic": measured_traffic("prefill"),
                "kernel": "prefill linear (all projections, activation quantization excluded)",
                "peak_source": f"{peaks['src']} bf16 x 2"}
        e2e_val = job_rate(world, ops, r0["ms_e2e"], 1e12)

    line = {
        "metric": METRIC, "value": value, "unit": unit, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": r0["ms"], "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "int8", "data": "synthetic (seeded random codes, scales, maps, activations)",
        "config": {"workload": args.workload, "model_shape": wl["model"], "phase": wl["phase"], "tokens": Ms[0],
                   "tile": [wl["bN"], 128], "int8_tile_fraction": wl["frac8"], "layers": model.layers,
                   "projections_per_layer": 7, "packed_weight_bytes": wbytes, "parallelism": f"replicas x{world}",
                   "l2": ("not flushed: weights streamed per step exceed the 126 MB L2" if wbytes > 126e6 else
                          "not flushed: weights of a reduced --layers case may stay in L2 (profiling only)"),
                   "graph": "one CUDA graph per step"},
        "e2e": {"value": e2e_val, "unit": unit, "h2d_bytes_per_step": r0["h2d"], "d2h_bytes_per_step": r0["d2h"]},
        "gpu_launches": r0["launches"] * args.steps,
        "roofline": roof,
        "clocks": clocks,
        "by_tokens": {},
        "setup_s": setup_s,
    }
    for M, r in results.items():
        if decode:
            line["by_tokens"][str(M)] = {"ms_per_step": r["ms"], "GB/s": wbytes / (r["ms"] * 1e-3) / 1e9,
                                         "linear_only_GB/s": wbytes / (r["ms_linear_only"] * 1e-3) / 1e9}
        else:
            line["by_tokens"][str(M)] = {"ms_per_step": r["ms"],
                                         "TOPS": 2.0 * M * model.macs / (r["ms"] * 1e-3) / 1e12}
    del model
    torch.cuda.empty_cache()

    if decode and not args.no_prefill and args.workload == "decode-llama-3.2-3b":
        pwl = WORKLOADS["prefill-qwen3-4b"]
        pm = Model(pwl, pwl["M"], dev, rank, args.layers)
        g, launches = pm.graph()
        ms = time_graph(torch, g, max(3, args.steps // 2), max(3, args.warmup), dist_on, dev)
        pm.quantize_inputs()
        g_lin, _ = pm.graph(mode="linear")
        ms_lin = time_graph(torch, g_lin, max(3, args.steps // 2), max(3, args.warmup), dist_on, dev)
        g_exp, _ = pm.graph(mode="expanded")
        ms_exp = time_graph(torch, g_exp, max(3, args.steps // 2), max(3, args.warmup), dist_on, dev)
        ops = 2.0 * pm.M * pm.macs
        int8_peak = 2.0 * peaks["bf16"]
        line["prefill"] = {"workload": "prefill-qwen3-4b", "tokens": pm.M, "ms_per_step": ms,
                           "TOPS": ops / (ms * 1e-3) / 1e12, "linear_only_TOPS": ops / (ms_lin * 1e-3) / 1e12,
                           "frac_of_int8_peak": ops / (ms_lin * 1e-3) / 1e12 / int8_peak,
                           "int8_peak_TOPS": int8_peak, "peak_source": f"{peaks['src']} bf16 x 2",
                           "long_prefill_expanded_TOPS": ops / (ms_exp * 1e-3) / 1e12}
        aq.check_all_workspaces()
        del g, g_lin, g_exp, pm
        torch.cuda.empty_cache()

    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        b, macs, t, desc = oracle_run(wl, 10.0, wl["M"])
        v = b / t / 1e9 if decode else 2.0 * macs / t / 1e12
        line["cpu_baseline"] = {"value": v, "unit": unit, "cores": cpu_threads(), "kind": "oracle", "sample": desc}

    if dist_on:
        torch.distributed.barrier()
        torch.distributed.destroy_process_group()
    if rank == 0:
        print(json.dumps(line), flush=True)
    return 0


def run_reference(args, wl, peaks):
    """The CPU oracle as the reference arm: each step is a bounded sample of the
    workload (one whole projection in turn), timed on the host cores."""
    import oracle
    from w8_a8_quantized_b200 import synth
    cfg = CFG_ID[wl["model"]]
    projs = synth.projections(wl["model"])
    rows = wl["M"] if wl["phase"] == "decode" else min(wl["M"], 16)
    prepared = []
    for pid, (name, N, K) in enumerate(projs):
        p = synth.projection_inputs(N, K, wl["bN"], 128, wl["frac8"], (cfg, 0, pid))
        prepared.append((oracle.pack(p.codes, p.scales, p.pmap, wl["bN"], 128),
                         synth.activations(rows, K, (cfg, 0, 999, rows), outlier_frac=wl["outlier"]), N * K))
    tot_b = tot_macs = 0
    tot_t = 0.0
    for i in range(args.warmup + args.steps):
        pk, x, nk = prepared[i % len(prepared)]
        t0 = time.perf_counter()
        xq, sx = oracle.quant_act(x)
        oracle.linear_packed(pk, xq, sx)
        dt = time.perf_counter() - t0
        if i >= args.warmup:
            tot_t += dt
            tot_b += oracle.packed_bytes(pk)
            tot_macs += nk * rows
    decode = wl["phase"] == "decode"
    unit = "GB/s" if decode else "TOPS"
    value = tot_b / tot_t / 1e9 if decode else 2.0 * tot_macs / tot_t / 1e12
    desc = (f"one whole projection of layer 0 per step (cycling q,k,v,o,gate,up,down), {rows} token(s): "
            "unpack + quantize + tile products + fp64 rescale")
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": unit, "n_gpus": 1, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": tot_t / max(args.steps, 1) * 1e3, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": args.workload, "model_shape": wl["model"], "phase": wl["phase"],
                       "tokens": rows},
            "cpu_baseline": {"value": value, "unit": unit, "cores": cpu_threads(), "kind": "oracle", "sample": desc},
            "e2e": {"value": value, "unit": unit, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


if __name__ == "__main__":
    sys.exit(main())
