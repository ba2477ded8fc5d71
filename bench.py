#!/usr/bin/env python
"""Benchmark of the mixed W4/W8 x A8 linear layers on B200.

One step = one pass of the hot path over a whole synthetic model: for every
decoder layer, the per-token INT8 quantization of the four distinct projection
inputs (attention input shared by q/k/v, attention output, MLP input shared
by gate/up, MLP hidden) and the seven linear projections, all launched through
the C ABI and replayed as one CUDA graph.  Weights are random, packed once,
and resident in HBM; every decode workload's per-step weight stream is far
larger than the 126 MB L2 (the single 2048 x 2048 layer is replicated into 128
distinct copies for that reason), so no explicit L2 flush is done.

Headline (the JSON line's value): Llama-3.2-3B-shaped decode (hidden 3072,
24 q / 8 kv heads x 128, MLP 8192, 28 layers), 128 x 128 tiles, 25% INT8
tiles, 1 token, in packed-weight GB/s; 8, 32 and 64 tokens are reported in
`by_tokens`.  `by_workload` carries the other configurations: the single
2048 x 2048 layer (1 and 16 tokens), the Qwen3-4B-shaped prefill (2048 tokens,
1% outlier channels), the 8B-class model (decode at 1, 16 and 64 tokens for
64- and 128-row tiles and 0/25/50/100% INT8 tiles; prefill of 4096 tokens) and
the Qwen3-14B-shaped model (decode at 1, 16 and 64 tokens; prefill of a
65,536-token context as 8 chunks of 8192 tokens through all 40 layers).
Prefill is reported in INT8 TOPS against the dense INT8 rate measured on the
same GPU by a tcgen05 loop (aq_measure_i8_peak).

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

# gen "host": weights and activations drawn with numpy (synth.projection_inputs, the
# values the GPU parity tests regenerate for the oracle); gen "device": the same
# recipe drawn on the GPU (models too large to draw on the host in seconds).
WORKLOADS = {
    "decode-llama-3.2-3b": dict(model="llama-3.2-3b", phase="decode", bN=128, frac8=0.25, M=1, extra_M=(8, 32, 64),
                                outlier=0.0, gen="host"),
    "prefill-qwen3-4b": dict(model="qwen3-4b", phase="prefill", bN=128, frac8=0.40, M=2048, extra_M=(),
                             outlier=0.01, gen="host"),
    "decode-single-2048": dict(model="single-2048", phase="decode", bN=128, frac8=0.5, M=1, extra_M=(16,),
                               outlier=0.0, gen="host", layers=128),
    "decode-dense-8b": dict(model="dense-8b", phase="decode", bN=128, frac8=0.5, M=1, extra_M=(16, 64),
                            outlier=0.0, gen="device"),
    "prefill-dense-8b": dict(model="dense-8b", phase="prefill", bN=128, frac8=0.5, M=4096, extra_M=(),
                             outlier=0.0, gen="device"),
    "decode-qwen3-14b": dict(model="qwen3-14b", phase="decode", bN=128, frac8=0.30, M=1, extra_M=(16, 64),
                             outlier=0.0, gen="device"),
    "prefill-qwen3-14b": dict(model="qwen3-14b", phase="prefill", bN=128, frac8=0.30, M=8192, extra_M=(),
                              outlier=0.01, gen="device", chunks=8),
}
# DRAM traffic per launch (dram__bytes_read.sum + dram__bytes_write.sum) of the dominant kernels,
# from an ncu capture of the named workload, valid only while the kernel source is unchanged
# (sha256 prefix of the source files).
MEASURED_TRAFFIC = {
    # four Llama-3.2-3B layers at 1 token (16 launches of the streaming kernel) read 259,310,848 B
    # and wrote 0 B -> 16,206,928 B per launch (algorithmic: 16,128,638 B per launch)
    "decode": {"src": ("w8_a8_quantized_b200/csrc/decode_stream.cu", "w8_a8_quantized_b200/csrc/aq_internal.cuh"),
               "sha": "93bb17d4f34e1fc8", "bytes_per_launch": 16206928},
    # the Qwen3-4B-shaped prefill's gate projection (N 9728, K 2560, 2048 tokens): 23,168,512 B read,
    # 26,489,344 B written (the rest of the 79.7 MB fp32 output still in L2 at the end of the launch)
    "prefill": {"src": ("w8_a8_quantized_b200/csrc/tc_linear.cu", "w8_a8_quantized_b200/csrc/aq_internal.cuh"),
                "sha": "ed409c05043d3c62", "bytes_per_launch": 49657856},
}


def source_sha(files) -> str:
    import hashlib
    h = hashlib.sha256()
    for f in files:
        with open(os.path.join(ROOT, f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def measured_traffic(phase: str):
    rec = MEASURED_TRAFFIC[phase]
    if rec["sha"] is None:
        return None
    return rec["bytes_per_launch"] if source_sha(rec["src"]) == rec["sha"] else None


CFG_ID = {"llama-3.2-3b": 2, "qwen3-4b": 3, "dense-8b": 4, "qwen3-14b": 5, "single-2048": 1}
INPUT_OF = {"q": "attn_in", "k": "attn_in", "v": "attn_in", "o": "attn_out", "gate": "mlp_in", "up": "mlp_in",
            "down": "mlp_hidden"}


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)  # ~0.2 s timed at 1 token
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="aq", choices=["aq", "reference"])
    ap.add_argument("--workload", default="decode-llama-3.2-3b", choices=sorted(WORKLOADS))
    ap.add_argument("--no-by-workload", action="store_true", help="measure only the headline workload")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--tokens", type=int, default=None, help="measure only this token count")
    ap.add_argument("--no-e2e", action="store_true", help="skip the host-buffer end-to-end measurement")
    ap.add_argument("--layers", type=int, default=None,
                    help="build only the first N layers (small cases for profiling; the line records the count)")
    ap.add_argument("--bn", type=int, default=None, help="tile rows (64 or 128) instead of the workload's")
    ap.add_argument("--frac8", type=float, default=None, help="INT8 tile fraction instead of the workload's")
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
    """SM clock and clock-event reasons, sampled through NVML every millisecond
    while the `with` block runs (nvidia-smi every 50 ms where NVML is missing)."""
    REASONS = {0x4: "sw_power_cap", 0x8: "hw_slowdown", 0x20: "sw_thermal_slowdown", 0x40: "hw_thermal_slowdown"}
    SMI = ("clocks.sm,clocks.max.sm,clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
           "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.sm, self.max_mhz, self.reasons = [], None, set()
        self.stop = threading.Event()
        self.mode, self.t, self.proc = None, None, None

    def _nvml(self):
        import pynvml
        pynvml.nvmlInit()
        vis = os.environ.get("CUDA_VISIBLE_DEVICES")
        h = None
        if vis:
            ids = [v.strip() for v in vis.split(",")]
            if self.gpu < len(ids):
                tok = ids[self.gpu]
                h = (pynvml.nvmlDeviceGetHandleByUUID(tok) if tok.startswith(("GPU-", "MIG-"))
                     else pynvml.nvmlDeviceGetHandleByIndex(int(tok)))
        if h is None:
            h = pynvml.nvmlDeviceGetHandleByIndex(self.gpu)
        return pynvml, h

    def _poll_nvml(self, nv, h):
        reasons = getattr(nv, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
            nv.nvmlDeviceGetCurrentClocksThrottleReasons
        while True:
            self.sm.append(float(nv.nvmlDeviceGetClockInfo(h, nv.NVML_CLOCK_SM)))
            r = int(reasons(h))
            for bit, name in self.REASONS.items():
                if r & bit:
                    self.reasons.add(name)
            if self.stop.wait(0.001):
                return

    def _poll_smi(self):
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in self.proc.stdout:
            f = [x.strip() for x in line.split(",")]
            try:
                self.sm.append(float(f[0]))
                self.max_mhz = float(f[1])
            except (ValueError, IndexError):
                continue
            for n, v in zip(names, f[2:6]):
                if v.lower().startswith("active"):
                    self.reasons.add(n)

    def __enter__(self):
        try:
            nv, h = self._nvml()
            self.max_mhz = float(nv.nvmlDeviceGetMaxClockInfo(h, nv.NVML_CLOCK_SM))
            self.mode = "nvml 1 ms"
            self.t = threading.Thread(target=self._poll_nvml, args=(nv, h), daemon=True)
        except Exception:
            try:
                self.proc = subprocess.Popen(["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.SMI}",
                                              "--format=csv,noheader,nounits", "-lms", "50"],
                                             stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            except OSError:
                return self
            self.mode = "nvidia-smi 50 ms"
            self.t = threading.Thread(target=self._poll_smi, daemon=True)
        self.t.start()
        time.sleep(0.01)  # first samples before the timed region
        return self

    def __exit__(self, *exc):
        self.stop.set()
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
        if self.t is not None:
            self.t.join(timeout=5)

    def summary(self):
        return {"sm_mhz": statistics.median(self.sm) if self.sm else None, "sm_max_mhz": self.max_mhz,
                "reasons": sorted(self.reasons), "samples": len(self.sm), "sampler": self.mode}


# ----------------------------------------------------------------------------- model
class Model:
    """Packed random weights and synthetic activations of one workload on one GPU."""

    def __init__(self, wl: dict, M: int, device, rank: int, layers=None, keep_host=True):
        import torch
        from w8_a8_quantized_b200 import aq, synth
        self.torch, self.aq = torch, aq
        self.wl, self.M, self.dev = wl, M, device
        self.keep_host = keep_host
        self.device_gen = wl.get("gen", "host") == "device"
        model = wl["model"]
        cfg = CFG_ID[model]
        n_layers = wl.get("layers", synth.MODELS[model]["layers"])
        self.layers = n_layers if layers is None else min(layers, n_layers)
        self.projs = synth.projections(model)
        self.weights = []
        self.weight_bytes = 0
        self.macs = 0
        for l in range(self.layers):
            layer = {}
            for pid, (name, N, K) in enumerate(self.projs):
                if self.device_gen:
                    codes, scales, pmap = synth.device_projection_inputs(N, K, wl["bN"], 128, wl["frac8"],
                                                                         (cfg, l, pid), device)
                else:
                    p = synth.projection_inputs(N, K, wl["bN"], 128, wl["frac8"], (cfg, l, pid))
                    codes, scales, pmap = (torch.from_numpy(p.codes).to(device), torch.from_numpy(p.scales).to(device),
                                           torch.from_numpy(p.pmap).to(device))
                w = aq.aq_pack(codes, scales, pmap, wl["bN"], 128)
                del codes, scales, pmap
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
        self.x = self.x_host_sets = self.groups = None
        cfg = CFG_ID[self.wl["model"]]
        xs, hs = [], []  # per activation set: input kind -> bf16 [M, K] on device / pinned host
        # decode: distinct activations for every layer; prefill: a pool of 4 distinct
        # activation sets cycled over the layers (each set is far larger than a tile)
        n_sets = self.layers if self.wl["phase"] == "decode" else min(4, self.layers)
        for l in range(n_sets):
            d, h = {}, {}
            for kind, K in self.in_dims.items():
                seed = (cfg, l, 100 + sorted(self.in_dims).index(kind), M)
                if self.device_gen:
                    d[kind] = synth.device_activations(M, K, seed, self.dev, outlier_frac=self.wl["outlier"])
                    if self.keep_host:
                        h[kind] = d[kind].cpu().pin_memory()
                else:
                    bits = synth.activations(M, K, seed, outlier_frac=self.wl["outlier"])
                    h[kind] = torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).pin_memory()
                    d[kind] = h[kind].to(self.dev)
            xs.append(d)
            hs.append(h)
        self.x = [xs[l % n_sets] for l in range(self.layers)]
        self.x_host_sets = hs
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
        # 3 tokens on as one preparation launch plus one linear launch over all members (CUDA
        # cores up to 3 tokens; tensor cores in decode when every member's rows are whole
        # 128-row blocks; CUDA cores up to 8 tokens for groups of three or more otherwise), else
        # one linear launch per member (prefill)
        self.fused = self.phase == aq.AQ_PHASE_DECODE and M <= 2
        decode = self.phase == aq.AQ_PHASE_DECODE
        self.one_launch = {kind: len(names) == 1 or (decode and (
            M <= 3 or all(self.out_dims[nm] % 128 == 0 for nm in names) or (len(names) >= 3 and M <= 8)))
            for kind, names in self.members.items()}

    def step(self, mode="group", chunks=1):
        """Enqueue one pass over every layer (`chunks` passes for a chunked
        prefill); returns the number of kernel launches.

        mode "group": the hot path, one aq_linear_group call per shared input
        (query/key/value, attention output, gate/up, MLP hidden) per layer.
        mode "linear": only the linear kernels on already-quantized inputs.
        mode "expanded": as "linear", through the long-prefill variant (each projection
        expanded to a temporary INT8 copy, then the pure INT8 GEMM)."""
        aq = self.aq
        n = 0
        for _ in range(chunks):
            for l, kind in [(l, kind) for l in range(self.layers) for kind in self.members]:
                names = self.members[kind]
                if mode == "group":
                    self.groups[l][kind](self.x[l][kind], [self.y[nm] for nm in names], ws=self.ws)
                    n += 1 if self.fused else 1 + (1 if self.one_launch[kind] else len(names))  # quantize + linear
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
        """Fill the pre-quantized inputs used by modes "linear" and "expanded"."""
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

    def free(self):
        self.weights = self.groups = self.x = self.x_host_sets = None
        self.xq = self.sx = self.y = self.ws = self.tmp = None


def max_over_ranks(torch, value: float, device) -> float:
    """The largest of every rank's value; every rank calls it at the same point."""
    t = torch.tensor([value], dtype=torch.float64, device=device)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def job_rate(world: int, units_per_rank: float, ms: float, scale: float) -> float:
    """Whole-job throughput: the units all ranks processed (each rank the same
    amount: independent replicas) over the slowest rank's time, in units of `scale`."""
    return world * units_per_rank / (ms * 1e-3) / scale


def time_graph(torch, g, steps, warmup, dist_on, dev, sampler=None):
    """Mean device time of one replay of `g` (CUDA events on the replay stream,
    barrier + synchronize on both sides, max over ranks); the clock sampler, if
    given, runs across the timed replays."""
    for _ in range(warmup):
        g.replay()
    torch.cuda.synchronize(dev)
    if dist_on:
        torch.distributed.barrier()
    torch.cuda.synchronize(dev)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if sampler is not None:
        sampler.__enter__()
    torch.cuda.nvtx.range_push("aq_timed")
    e0.record()
    for _ in range(steps):
        g.replay()
    e1.record()
    torch.cuda.nvtx.range_pop()
    torch.cuda.synchronize(dev)
    if sampler is not None:
        sampler.__exit__(None, None, None)
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


def measure(torch, label, wl, Ms, steps, warmup, dist_on, dev, peaks, i8_peak, layers=None, sampler_gpu=None,
            e2e=False, linear_only=True, expanded=False):
    """Build the model of `wl`, time its step at every token count in Ms and
    return (summary dict, clocks of the first count or None, (e2e ms, h2d, d2h)
    or None, the model)."""
    from w8_a8_quantized_b200 import aq
    t0 = time.time()
    model = Model(wl, Ms[0], dev, 0, layers, keep_host=e2e)
    chunks = wl.get("chunks", 1)
    decode = wl["phase"] == "decode"
    res = {"model_shape": wl["model"], "phase": wl["phase"], "tile": [wl["bN"], 128],
           "int8_tile_fraction": wl["frac8"], "layers": model.layers, "packed_weight_bytes": model.weight_bytes,
           "weights": "device-drawn" if model.device_gen else "host-drawn", "steps": steps, "warmup": warmup,
           "by_tokens": {}}
    if chunks > 1:
        res["chunks"] = chunks
        res["context_tokens"] = chunks * Ms[0]
    clocks = e2e_res = None
    for M in Ms:
        if M != model.M:
            model.set_tokens(M)
        g, launches = model.graph(chunks=chunks)
        sampler = ClockSampler(sampler_gpu) if (sampler_gpu is not None and M == Ms[0]) else None
        ms = time_graph(torch, g, steps, warmup, dist_on, dev, sampler)
        if sampler is not None:
            clocks = sampler.summary()
        ops = 2.0 * M * model.macs * chunks
        ent = {"ms_per_step": ms, "launches_per_step": launches}
        if decode:
            ent["GB/s"] = model.weight_bytes / (ms * 1e-3) / 1e9
            ent["frac_of_hbm"] = ent["GB/s"] / peaks["hbm"]
        else:
            ent["TOPS"] = ops / (ms * 1e-3) / 1e12
        if decode and model.fused:  # the step holds nothing but the fused decode kernel
            ent["linear_only_ms_per_step"], ent["linear_launches_per_step"] = ms, launches
        elif linear_only:
            model.quantize_inputs()
            g_lin, ent["linear_launches_per_step"] = model.graph(mode="linear", chunks=chunks)
            ent["linear_only_ms_per_step"] = time_graph(torch, g_lin, steps, warmup, dist_on, dev)
            del g_lin
        if "linear_only_ms_per_step" in ent:
            t_lin = ent["linear_only_ms_per_step"] * 1e-3
            if decode:
                ent["linear_only_GB/s"] = model.weight_bytes / t_lin / 1e9
                ent["linear_only_frac_of_hbm"] = ent["linear_only_GB/s"] / peaks["hbm"]
            else:
                ent["linear_only_TOPS"] = ops / t_lin / 1e12
                ent["linear_only_frac_of_int8_peak"] = ent["linear_only_TOPS"] / i8_peak
        if expanded and not decode:
            model.quantize_inputs()
            g_exp, _ = model.graph(mode="expanded", chunks=chunks)
            ent["long_prefill_expanded_TOPS"] = ops / (time_graph(torch, g_exp, steps, warmup, dist_on, dev)
                                                       * 1e-3) / 1e12
            del g_exp
        if e2e and M == Ms[0]:
            ms_e2e, h2d, d2h = time_e2e(torch, model, g, steps, warmup, dev)
            if dist_on:  # every rank times it, the slowest one counts
                ms_e2e = max_over_ranks(torch, ms_e2e, dev)
            e2e_res = (ms_e2e, h2d, d2h)
        res["by_tokens"][str(M)] = ent
        del g
        aq.check_all_workspaces()
        rc, info = aq.aq_workspace_status(model.ws)
        if rc != 0:
            raise RuntimeError(f"{label}: kernel reported error {rc} ({info})")
    res["wall_s"] = time.time() - t0
    return res, clocks, e2e_res, model


def by_workload_plan(steps, warmup):
    """(label, workload, overrides, token counts, steps, warmup) of every secondary measurement."""
    few = max(3, steps // 4)
    plan = [("decode-single-2048", "decode-single-2048", {}, [1, 16], steps, warmup),
            ("prefill-qwen3-4b", "prefill-qwen3-4b", {}, [2048], max(3, steps // 2), max(3, warmup)),
            ("decode-qwen3-14b", "decode-qwen3-14b", {}, [1, 16, 64], steps, warmup),
            ("prefill-qwen3-14b-64k-context", "prefill-qwen3-14b", {}, [8192], 3, 3)]
    for bN in (128, 64):
        plan.append((f"prefill-dense-8b-bN{bN}", "prefill-dense-8b", {"bN": bN}, [4096], few, 3))
    for bN in (128, 64):
        for f8 in (0.0, 0.25, 0.5, 1.0):
            plan.append((f"decode-dense-8b-bN{bN}-int8-{int(f8 * 100)}pct", "decode-dense-8b",
                         {"bN": bN, "frac8": f8}, [1, 16, 64], steps, warmup))
    return plan


# ----------------------------------------------------------------------------- CPU oracle
def oracle_run(wl, budget_s, M):
    """Time the CPU oracle on a bounded sample of the workload: whole projections
    of the first layers (unpack of the packed form, activation quantization,
    integer tile products, fp64 rescale), until `budget_s` seconds are used.
    Returns (packed bytes done, MACs done, seconds, process CPU seconds, description)."""
    import oracle
    from w8_a8_quantized_b200 import synth
    cfg = CFG_ID[wl["model"]]
    projs = synth.projections(wl["model"])
    layers = synth.MODELS[wl["model"]]["layers"]
    done_bytes = done_macs = 0
    n_proj = 0
    rows = M if wl["phase"] == "decode" else min(M, 64)
    t_used = cpu_used = 0.0
    for l in range(layers):
        for pid, (name, N, K) in enumerate(projs):
            p = synth.projection_inputs(N, K, wl["bN"], 128, wl["frac8"], (cfg, l, pid))
            pk = oracle.pack(p.codes, p.scales, p.pmap, wl["bN"], 128)
            x = synth.activations(rows, K, (cfg, l, 999, rows), outlier_frac=wl["outlier"])
            t0, c0 = time.perf_counter(), time.process_time()
            xq, sx = oracle.quant_act(x)
            oracle.linear_packed(pk, xq, sx)
            t_used += time.perf_counter() - t0
            cpu_used += time.process_time() - c0
            done_bytes += oracle.packed_bytes(pk)
            done_macs += N * K * rows
            n_proj += 1
            if t_used >= budget_s:
                break
        if t_used >= budget_s:
            break
    desc = (f"{n_proj} whole projections of the first layer(s) of the workload, {rows} token(s) each, "
            f"unpack + quantize + tile products + fp64 rescale")
    return done_bytes, done_macs, t_used, cpu_used, desc


def cpu_model() -> str:
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return "unknown"


def blas_threads():
    """Threads of the BLAS pool the oracle's matrix products may use."""
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 1) for i in threadpool_info() if i.get("user_api") == "blas"]
        return max(n) if n else 1
    except Exception:
        return os.cpu_count() or 1


def threads_used(cpu_s, wall_s):
    """Cores the timed region actually kept busy: process CPU time (all threads)
    over wall time, at least 1."""
    return max(1.0, round(cpu_s / wall_s, 1)) if wall_s > 0 else 1.0


def cpu_baseline(wl, budget_s, decode, legs=("single_thread", "all_cores")):
    """The oracle on the host cores, once with one BLAS thread and once with the
    default BLAS pool (all cores offered); `value` and `cores` are the second
    run's, `cores` being the cores it kept busy (CPU time over wall time)."""
    from threadpoolctl import threadpool_limits
    unit = "GB/s" if decode else "TOPS"
    out = {"kind": "oracle", "unit": unit, "cpu": cpu_model(), "nproc": os.cpu_count()}
    for label in legs:
        if label == "single_thread":
            with threadpool_limits(limits=1, user_api="blas"):
                b, macs, t, c, desc = oracle_run(wl, budget_s, wl["M"])
            pool = 1
        else:
            b, macs, t, c, desc = oracle_run(wl, budget_s, wl["M"])
            pool = blas_threads()
        out[label] = {"value": b / t / 1e9 if decode else 2.0 * macs / t / 1e12, "blas_threads": pool,
                      "threads": threads_used(c, t), "sample": desc}
    out["value"] = out["all_cores"]["value"]
    out["cores"] = out["all_cores"]["threads"]
    out["sample"] = out["all_cores"]["sample"]
    return out


# ----------------------------------------------------------------------------- main
def main():
    args = parse()
    wl = dict(WORKLOADS[args.workload])
    if args.bn is not None:
        wl["bN"] = args.bn
    if args.frac8 is not None:
        wl["frac8"] = args.frac8
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
    i8_peak = aq.aq_measure_i8_peak(20000, device=dev)  # dense INT8 TOPS of this GPU (tcgen05 loop)

    decode = wl["phase"] == "decode"
    Ms = [wl["M"], *wl["extra_M"]] if args.tokens is None else [args.tokens]
    res, clocks, e2e_res, model = measure(torch, args.workload, wl, Ms, args.steps, args.warmup, dist_on, dev,
                                          peaks, i8_peak, layers=args.layers, sampler_gpu=local,
                                          e2e=not args.no_e2e, expanded=not decode)
    head = res["by_tokens"][str(Ms[0])]
    wbytes, layers_built, n_proj = model.weight_bytes, model.layers, len(model.projs)
    ops = 2.0 * Ms[0] * model.macs * wl.get("chunks", 1)
    model.free()
    del model
    torch.cuda.empty_cache()
    if decode:
        unit, units, scale = "GB/s", wbytes, 1e9
        achieved = wbytes / (head["linear_only_ms_per_step"] * 1e-3) / 1e9
        roof = {"bound": "hbm", "achieved": achieved, "peak": peaks["hbm"], "unit": "GB/s",
                "frac": achieved / peaks["hbm"], "traffic": measured_traffic("decode"),
                "algorithmic_bytes_per_launch": wbytes / head["linear_launches_per_step"],
                "kernel": ("decode linear, all projections (1 token: one fused launch per shared input, "
                           "activation quantization inside)" if Ms[0] <= 2 else
                           "decode linear, all projections, activation quantization excluded"),
                "peak_source": f"{peaks['src']} copy bandwidth (of {peaks['src']})"}
    else:
        unit, units, scale = "TOPS", ops, 1e12
        achieved = head["linear_only_TOPS"]
        roof = {"bound": "tensor", "achieved": achieved, "peak": i8_peak, "unit": "TFLOP/s",
                "frac": achieved / i8_peak, "traffic": measured_traffic("prefill"),
                "kernel": "prefill linear, all projections, activation quantization excluded",
                "peak_source": "measured: dense INT8 tcgen05 loop on this GPU, this run",
                "frac_of_bf16_peak_x2": achieved / (2.0 * peaks["bf16"])}
    value = job_rate(world, units, head["ms_per_step"], scale)

    line = {
        "metric": METRIC, "value": value, "unit": unit, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": head["ms_per_step"], "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "int8", "data": "synthetic (seeded random codes, scales, maps, activations)",
        "config": {"workload": args.workload, "model_shape": wl["model"], "phase": wl["phase"], "tokens": Ms[0],
                   "tile": [wl["bN"], 128], "int8_tile_fraction": wl["frac8"], "layers": layers_built,
                   "projections_per_layer": n_proj,
                   "packed_weight_bytes": wbytes, "parallelism": f"replicas x{world}",
                   "l2": ("not flushed: weights streamed per step exceed the 126 MB L2" if wbytes > 126e6 else
                          "not flushed: weights of a reduced --layers case may stay in L2 (profiling only)"),
                   "graph": "one CUDA graph per step"},
        "e2e": ({"value": job_rate(world, units, e2e_res[0], scale), "unit": unit, "h2d_bytes_per_step": e2e_res[1],
                 "d2h_bytes_per_step": e2e_res[2]} if e2e_res else None),
        "gpu_launches": head["launches_per_step"] * args.steps,
        "roofline": roof,
        "clocks": clocks,
        "by_tokens": res["by_tokens"],
        "int8_peak_measured_TOPS": i8_peak,
        "setup_s": res["wall_s"],
    }

    if not args.no_by_workload and args.tokens is None and args.layers is None and args.bn is None \
            and args.frac8 is None:
        by = {}
        for label, wname, over, ms_list, st, wu in by_workload_plan(args.steps, args.warmup):
            if wname == args.workload and not over:
                continue
            wl2 = dict(WORKLOADS[wname], **over)
            r, _, _, m = measure(torch, label, wl2, ms_list, st, wu, dist_on, dev, peaks, i8_peak,
                                 linear_only=wl2["phase"] == "prefill" and wl2.get("chunks", 1) == 1,
                                 expanded=label == "prefill-qwen3-4b")
            m.free()
            del m
            torch.cuda.empty_cache()
            by[label] = r
        line["by_workload"] = by

    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(wl, 6.0, decode)
        for label, wname, over, *_ in by_workload_plan(args.steps, args.warmup):
            if label in line.get("by_workload", {}):  # a shorter sample, all cores only
                wl2 = dict(WORKLOADS[wname], **over)
                line["by_workload"][label]["cpu_baseline"] = cpu_baseline(wl2, 1.0, wl2["phase"] == "decode",
                                                                          legs=("all_cores",))

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
    tot_t = tot_c = 0.0
    for i in range(args.warmup + args.steps):
        pk, x, nk = prepared[i % len(prepared)]
        t0, c0 = time.perf_counter(), time.process_time()
        xq, sx = oracle.quant_act(x)
        oracle.linear_packed(pk, xq, sx)
        dt, dc = time.perf_counter() - t0, time.process_time() - c0
        if i >= args.warmup:
            tot_t += dt
            tot_c += dc
            tot_b += oracle.packed_bytes(pk)
            tot_macs += nk * rows
    decode = wl["phase"] == "decode"
    unit = "GB/s" if decode else "TOPS"
    value = tot_b / tot_t / 1e9 if decode else 2.0 * tot_macs / tot_t / 1e12
    world = int(os.environ.get("WORLD_SIZE", "1"))
    desc = (f"one whole projection of layer 0 per step (cycling through the layer's projections), "
            f"{rows} token(s): unpack + quantize + tile products + fp64 rescale"
            + (f"; rank 0 of {world} alone" if world > 1 else ""))
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": unit, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": tot_t / max(args.steps, 1) * 1e3, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": args.workload, "model_shape": wl["model"], "phase": wl["phase"],
                       "tokens": rows},
            "cpu_baseline": {"value": value, "unit": unit, "cores": threads_used(tot_c, tot_t),
                             "blas_threads": blas_threads(), "nproc": os.cpu_count(),
                             "cpu": cpu_model(), "kind": "oracle", "sample": desc},
            "e2e": {"value": value, "unit": unit, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


if __name__ == "__main__":
    sys.exit(main())
