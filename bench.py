#!/usr/bin/env python
"""Benchmark of the LRB (low-rank binary) matmul path on B200.

Headline: batch-1 decode of the Llama-2-7B attention projection (d_out = d_in = 4096,
r = 2048, 1.0 bit/weight).  One step is one pass of a chain of distinct layer instances
(y of one layer is x of the next), enough of them that the weights (>= 3x the L2 size)
stream from HBM on every step; the chain is captured once as a CUDA graph of the public
API calls and replayed.  Reported: microseconds per layer (whole job), achieved HBM GB/s
of the layer forward against the measured copy bandwidth, the CPU oracle on the host cores,
and an end-to-end figure with host<->device copies inside the timed region.

Launch: ``python bench.py [--gpus N --steps K --warmup W]``; for N > 1 one process per GPU
(torchrun), each an independent replica (the path has no cross-GPU exchange).
``--impl reference`` times the CPU oracle instead (rank 0 only).
"""
from __future__ import annotations

import argparse
import glob
import json
import os
import statistics
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from rank_binary_factorized_b200 import synth  # noqa: E402

HEADLINE = "attn7b"
METRIC = "binary low-rank matmul µs/layer + achieved HBM GB/s (% roofline), batch 1"
L2_BYTES = 126 * 1024 * 1024
FALLBACK_HBM_GBS = 6650.0
FALLBACK_BF16_TFLOPS = 1590.0


def parse_args():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["nq", "reference"], default="nq")
    ap.add_argument("--batch", type=int, default=1)
    ap.add_argument("--headline-only", action="store_true", help="skip the other workloads")
    ap.add_argument("--layer70b-only", action="store_true",
                    help="run only the 70B decoder-layer section (for profiling: its first launches are the "
                         "first layer's kernels); prints its figures alone")
    ap.add_argument("--only", default=None,
                    help="run just these extra sections (comma list of attn7b_b8, mlp7b, prefill, pack, "
                         "calib, signgrad, model70b) "
                         "after the headline; implies no CPU baseline")
    ap.add_argument("--cpu-seconds", type=float, default=12.0, help="CPU oracle sample budget")
    return ap.parse_args()


# --------------------------------------------------------------------------- plumbing
def dist_env():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return rank, world, local


def measured_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), float(d["bf16_tflops"]), float(d.get("bf16_tflops_sustained", d["bf16_tflops"])), "measured"
    return FALLBACK_HBM_GBS, FALLBACK_BF16_TFLOPS, 1400.0, "fallback"


HOST_SIDE_MARKER = "// ------------------------------------------------------------------------------ host side"


def device_source_sha(path: str, text: str = None) -> str:
    """Hash of a kernel file's device part (everything before its host-side marker) with
    comments and whitespace removed, so that host-only or comment edits keep a capture valid and
    any code edit of a kernel invalidates it."""
    import hashlib
    import re
    if text is None:
        text = open(path).read()
    code = text.split(HOST_SIDE_MARKER)[0]
    code = re.sub(r"/\*.*?\*/", "", code, flags=re.S)
    code = re.sub(r"//[^\n]*", "", code)
    code = re.sub(r"\s+", "", code)
    return hashlib.sha256(code.encode()).hexdigest()[:16]


def profile_traffic(kernel_key: str):
    """DRAM bytes per launch recorded from an ncu capture in profiles/ (None if absent or
    if the kernel source changed since: the summary records the device-code hash)."""
    for path in glob.glob(os.path.join(ROOT, "profiles", "*.md")):
        text = open(path).read()
        tag = "traffic[%s]:" % kernel_key
        if tag not in text:
            continue
        line = [ln for ln in text.splitlines() if ln.startswith(tag)][0]
        fields = dict(kv.split("=") for kv in line[len(tag):].split())
        src = os.path.join(ROOT, fields["source"])
        if not os.path.exists(src) or device_source_sha(src) != fields["device_sha"]:
            return None
        return float(fields["bytes"])
    return None


def nvml_index(local: int) -> int:
    """NVML index of this rank's GPU.  CUDA_VISIBLE_DEVICES maps the local ordinal to the
    physical one; a UUID entry is looked up through NVML, and anything unreadable falls back to
    the local ordinal (the clock record then names that GPU)."""
    vis = os.environ.get("CUDA_VISIBLE_DEVICES", "").strip()
    if not vis:
        return local
    entries = [e.strip() for e in vis.split(",") if e.strip()]
    if local >= len(entries):
        return local
    try:
        return int(entries[local])
    except ValueError:
        pass
    try:
        import pynvml
        pynvml.nvmlInit()
        return int(pynvml.nvmlDeviceGetIndex(pynvml.nvmlDeviceGetHandleByUUID(entries[local])))
    except Exception:
        return local


class ClockSampler:
    """Samples SM clock and throttle reasons through NVML while the timed region runs."""

    REASONS = {
        0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap", 0x8: "hw_slowdown",
        0x10: "sync_boost", 0x20: "sw_thermal_slowdown", 0x40: "hw_thermal_slowdown",
        0x80: "hw_power_brake_slowdown", 0x100: "display_clock_setting",
    }

    def __init__(self, index: int, period_s: float = 0.01):
        self.index, self.period = index, period_s
        self.samples, self.reasons, self.max_mhz = [], set(), None
        self._stop = threading.Event()
        self._thread = None
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nv = pynvml
            self.h = pynvml.nvmlDeviceGetHandleByIndex(index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
        except Exception:
            self.nv = None

    def _run(self):
        while not self._stop.is_set():
            try:
                self.samples.append(self.nv.nvmlDeviceGetClockInfo(self.h, self.nv.NVML_CLOCK_SM))
                bits = self.nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
                for b, name in self.REASONS.items():
                    if bits & b and name != "gpu_idle":
                        self.reasons.add(name)
            except Exception:
                pass
            time.sleep(self.period)

    def __enter__(self):
        if self.nv is not None:
            self._thread = threading.Thread(target=self._run, daemon=True)
            self._thread.start()
        return self

    def __exit__(self, *exc):
        self._stop.set()
        if self._thread:
            self._thread.join()

    def summary(self):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": ["unsampled"]}
        return {"sm_mhz": float(statistics.median(self.samples)), "sm_max_mhz": self.max_mhz,
                "reasons": sorted(self.reasons), "samples": len(self.samples)}


# --------------------------------------------------------------------------- GPU arm
class Chain:
    """n distinct instances of one projection shape on the device, chained y -> x."""

    def __init__(self, torch, nq, d_out, d_in, r, M, n, seed, ws=None):
        self.M, self.n = M, n
        self.layers = []
        for i in range(n):
            p = synth.make_projection("chain", d_out, d_in, r, seed=seed, key=i)
            self.layers.append(nq.Layer.from_host(p.U, p.V, p.s1, p.s2, r))
        need = max(L.workspace_bytes(M) for L in self.layers)
        self.ws = ws if ws is not None and ws.numel() >= need else torch.zeros(need, dtype=torch.uint8, device="cuda")
        xb = synth.acts_bf16(synth.rng_for(seed, 999), (M, d_in))
        self.x0 = torch.from_numpy(xb.view(np.int16)).cuda().view(torch.bfloat16)
        self.bufs = [torch.empty((M, d_out), dtype=torch.bfloat16, device="cuda") for _ in range(2)]
        self.chained = d_in == d_out

    def run(self, nq, stream):
        x = self.x0
        for i, L in enumerate(self.layers):
            y = self.bufs[i % 2]
            nq.layer_forward(L, x, y, ws=self.ws, stream=stream)
            x = y if self.chained else self.x0
        return x

    @property
    def weight_bytes(self):
        return sum(L.storage_bytes for L in self.layers)


def graph_of(torch, fn, stream):
    g = torch.cuda.CUDAGraph()
    with torch.cuda.stream(stream):
        fn()  # warm (attribute setup, lazy loads) outside the capture
        torch.cuda.synchronize()
        with torch.cuda.graph(g, stream=stream):
            fn()
    torch.cuda.synchronize()
    return g


def timed_replays(torch, g, stream, steps, warmup, dist=None, sampler=None):
    """Device time of `steps` replays (ms), bracketed by barrier + sync, max over ranks."""
    with torch.cuda.stream(stream):
        for _ in range(warmup):
            g.replay()
    torch.cuda.synchronize()
    if dist is not None:
        dist.barrier()
    torch.cuda.synchronize()
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    ctx = sampler if sampler is not None else _null()
    with ctx:
        start.record(stream)
        with torch.cuda.stream(stream):
            for _ in range(steps):
                g.replay()
        end.record(stream)
        torch.cuda.synchronize()
    if dist is not None:
        dist.barrier()
    torch.cuda.synchronize()
    return max_over_ranks(torch, start.elapsed_time(end), dist, "cuda")


def max_over_ranks(torch, ms, dist, device):
    """The slowest rank's time: every rank gets the maximum of the ranks' values."""
    if dist is None:
        return ms
    t = torch.tensor([ms], device=device, dtype=torch.float64)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_us_per_layer(ms, steps, layers_per_step, world):
    """Whole-job time per layer: every rank runs `layers_per_step` layers per step, so the job
    processes steps x layers_per_step x world layers in the slowest rank's time."""
    return ms * 1e3 / (steps * layers_per_step * world)


class _null:
    def __enter__(self):
        return self

    def __exit__(self, *a):
        return False


def decode_bytes(d_out, d_in, r, M):
    """Algorithmic bytes of one projection: packed signs + fp16 scales + bf16 in/out."""
    return r * (d_in + d_out) // 8 + 2 * (d_in + d_out) + 2 * M * (d_in + d_out)


def n_instances(layer_bytes):
    return max(8, int(np.ceil(3 * L2_BYTES / layer_bytes)))


def gpu_arm(args, rank, world, local):
    import torch
    from rank_binary_factorized_b200 import nq

    torch.cuda.set_device(local)
    dist = None
    if world > 1:
        import datetime
        import torch.distributed as tdist
        tdist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=torch.device("cuda", local))
        dist = tdist
    hbm_gbs, bf16_tf, bf16_tf_sus, peak_src = measured_peaks()
    stream = torch.cuda.Stream()

    if args.layer70b_only:
        return {"metric": METRIC, "value": None, "unit": "us/layer", "n_gpus": world,
                "note": "70B decoder-layer section alone (profiling run); no headline",
                "headline_layer70b": headline_layer70b(torch, nq, stream, args, hbm_gbs, peak_src, local)}

    # ---- headline: 7B attention projection, batch M, chain of distinct instances
    (_, d_out, d_in, r), = synth.WORKLOADS[HEADLINE]
    M = args.batch
    lbytes = decode_bytes(d_out, d_in, r, M)
    n = n_instances(lbytes)
    chain = Chain(torch, nq, d_out, d_in, r, M, n, seed=synth.workload_seed(HEADLINE))
    g = graph_of(torch, lambda: chain.run(nq, stream), stream)
    sampler = ClockSampler(nvml_index(local))
    ms = timed_replays(torch, g, stream, args.steps, args.warmup, dist, sampler)
    nq.sync_status(stream)
    us_per_layer_job = job_us_per_layer(ms, args.steps, n, world)  # all ranks' layers in the max time
    us_per_layer_gpu = ms * 1e3 / (args.steps * n)  # one GPU's layer forward
    achieved = lbytes / (us_per_layer_gpu * 1e-6) / 1e9
    del g

    result = {
        "metric": METRIC,
        "value": round(us_per_layer_job, 4),
        "unit": "us/layer",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(ms / args.steps, 4),
        "higher_is_better": False,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "int32",
        "data": "synthetic (seeded iid +-1 signs, fp16 0.02|N(0,1)| scales, bf16 N(0,1) activations)",
        "config": {
            "workload": "Llama-2-7B attention projection d_out=d_in=4096 r=2048 (1.0 bit/weight), decode batch %d" % M,
            "batch": M,
            "operands": "1-bit packed U, V (uint32 words); fp16 s1, s2; bf16 x, y",
            "arithmetic": "s2 x in fp32, fixed-point per batch row (23-bit integers); sign products on u8 x s8 "
                          "MMAs with exact int32 accumulation; fp64 sums across row slices; fp32 scale by s1, bf16 out",
            "layers_per_step": n,
            "chain": "y of each layer is x of the next (distinct weights per layer)",
            "l2": "no flush: %d distinct layers = %.0f MB of weights per step > 3x L2" % (n, chain.weight_bytes / 1e6),
            "parallelism": "replicas" if world > 1 else "single GPU",
        },
        "roofline": {
            "bound": "hbm",
            "kernel": "decode layer forward (stage-1 + stage-2 kernels, PDL-chained)",
            "achieved": round(achieved, 1),
            "peak": hbm_gbs,
            "peak_source": peak_src + " (MEASURED_PEAKS.json hbm_gbs)" if peak_src == "measured" else peak_src,
            "unit": "GB/s",
            "frac": round(achieved / hbm_gbs, 4),
            "traffic": profile_traffic("decode_attn7b_b%d" % M),
            "algorithmic_bytes_per_launch": lbytes,
        },
        "clocks": sampler.summary(),
        "gpu_launches": 2 * n * args.steps,
    }

    # ---- end to end through the public API: H2D of the step's input from pinned memory,
    # the chain of layer_forward calls (captured once as a graph), D2H of the result
    result["e2e"] = e2e_measure(torch, nq, chain, stream, args, dist, world)

    # ---- one public-API call on a cold L2: what the first layer of a decode step sees
    result["latency_single_call"] = single_call_latency(torch, nq, chain, stream)
    del chain

    # ---- second headline: a Llama-2-70B decoder layer's projections at batch 1
    result["headline_layer70b"] = headline_layer70b(torch, nq, stream, args, hbm_gbs, peak_src, local)

    if not args.headline_only or args.only is not None:
        result["extra"] = extras(torch, nq, stream, args, hbm_gbs, bf16_tf, bf16_tf_sus, peak_src)

    if args.only is not None:
        pass
    elif rank == 0 and world == 1:
        result["cpu_baseline"] = cpu_baseline(args.cpu_seconds)
        result["parity_margins"] = parity_margins(torch, nq)
    elif rank == 0:
        result["cpu_baseline"] = None

    if dist is not None:
        dist.barrier()
        dist.destroy_process_group()
    return result


def single_call_latency(torch, nq, chain, stream, calls=50):
    """One nq_layer_forward call of the headline layer through the Python binding, after a read
    of 256 MB that leaves nothing of the layer in L2: host time from just before the call to
    the end of a stream synchronise (argument checks, ctypes, launch, kernels, sync), and the
    device time between CUDA events recorded around the call on its stream."""
    flush = torch.empty(256 << 20, dtype=torch.uint8, device="cuda").view(torch.int64)
    flush.fill_(1)
    y = torch.empty((chain.M, chain.layers[0].d_out), dtype=torch.bfloat16, device="cuda")
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    host, dev = [], []
    for i in range(calls + 3):
        L = chain.layers[i % chain.n]
        with torch.cuda.stream(stream):
            torch.max(flush)  # reads 256 MB: L2 holds the flush buffer's clean lines afterwards
        stream.synchronize()
        t0 = time.perf_counter()
        e0.record(stream)
        nq.layer_forward(L, chain.x0, y, ws=chain.ws, stream=stream)
        e1.record(stream)
        stream.synchronize()
        t1 = time.perf_counter()
        if i >= 3:
            host.append((t1 - t0) * 1e6)
            dev.append(e0.elapsed_time(e1) * 1e3)
    del flush
    return {"host_us": round(statistics.median(host), 2), "device_us": round(statistics.median(dev), 2),
            "calls": calls, "l2": "flushed before every call (a 256 MB read on the same stream)",
            "note": "median of one nq_layer_forward call (7B attention projection, batch 1) through the Python "
                    "binding: host time includes argument checks, the ctypes call, both launches and the "
                    "synchronise"}


def headline_layer70b(torch, nq, stream, args, hbm_gbs, peak_src, local):
    """Batch-1 decode of a Llama-2-70B decoder layer's LRB projections (q, k, v grouped; o;
    gate and up fused with SiLU.mul; down) over distinct layer instances (> 3x L2 per step)."""
    sampler = ClockSampler(nvml_index(local))
    r = _extra_block(torch, nq, stream, max(10, args.steps // 2), max(3, args.warmup), hbm_gbs, "layer70b", sampler)
    alg = r["block_bytes"]
    return {"workload": "Llama-2-70B decoder layer: q,o 8192x8192 r=2240; k,v 1024x8192 r=512; gate,up "
                        "28672x8192 and down 8192x28672 r=3520; decode batch 1",
            "value": r["us_per_block"], "unit": "us/layer", "steps": r["steps"], "layers_per_step": r["blocks_per_step"],
            "grouped": r["grouped"],
            "roofline": {"bound": "hbm", "kernel": "decode layer (8 stage kernels, PDL-chained)",
                         "achieved": r["GB_s"], "peak": hbm_gbs,
                         "peak_source": peak_src + " (MEASURED_PEAKS.json hbm_gbs)" if peak_src == "measured" else peak_src,
                         "unit": "GB/s", "frac": r["frac_hbm"], "traffic": profile_traffic("decode_layer70b_b1"),
                         "algorithmic_bytes_per_launch": alg},
            "clocks": sampler.summary(),
            "l2": "no flush: %d distinct layers per step, %.0f MB > 3x L2" % (r["blocks_per_step"],
                                                                            r["blocks_per_step"] * alg / 1e6)}


def e2e_measure(torch, nq, chain, stream, args, dist, world):
    M = chain.M
    d_in = chain.layers[0].d_in
    d_out = chain.layers[0].d_out
    host_x = torch.from_numpy(synth.acts_bf16(synth.rng_for(77), (M, d_in)).view(np.int16)).pin_memory()
    host_y = torch.empty((M, d_out), dtype=torch.int16).pin_memory()
    x_dev = chain.x0

    def step():
        x_dev.view(torch.int16).copy_(host_x, non_blocking=True)
        y = chain.run(nq, stream)
        host_y.copy_(y.view(torch.int16), non_blocking=True)

    g = graph_of(torch, step, stream)
    ms = timed_replays(torch, g, stream, args.steps, args.warmup, dist)
    del g
    return {"value": round(ms * 1e3 / (args.steps * chain.n * world), 4), "unit": "us/layer",
            "h2d_bytes_per_step": int(host_x.numel() * 2), "d2h_bytes_per_step": int(host_y.numel() * 2),
            "note": "graph of public-API layer_forward calls with a pinned-host H2D of x and D2H of y per step"}


def extras(torch, nq, stream, args, hbm_gbs, bf16_tf, bf16_tf_sus, peak_src):
    out = {}
    steps = max(5, args.steps // 5)
    warm = max(3, args.warmup)
    want = None if args.only is None else set(args.only.split(","))

    def on(name):
        return want is None or name in want

    # decode batch 8 of the headline shape
    (_, d_out, d_in, r), = synth.WORKLOADS[HEADLINE]
    if on("attn7b_b8"):
        out.update(_extra_b8(torch, nq, stream, steps, warm, hbm_gbs, d_out, d_in, r))
    if on("mlp7b"):
        out["mlp7b"] = _extra_block(torch, nq, stream, steps, warm, hbm_gbs, "mlp7b")
    if on("prefill"):
        out["prefill70b_gate"] = _extra_prefill(torch, nq, stream, steps, bf16_tf)
    if on("pack"):
        out["pack_70b_gate_U"] = _extra_pack(torch, nq, stream, steps, warm, hbm_gbs)
    if on("calib"):
        out.update(_extra_calib(torch, nq, stream, steps, warm, hbm_gbs, bf16_tf))
    if on("signgrad"):
        out.update(_extra_sign_grads(torch, nq, stream, steps, warm, hbm_gbs, bf16_tf))
    if on("model70b"):
        out["model70b_decode_b1"] = _extra_model70b(torch, nq, stream, hbm_gbs)
    nq.sync_status(stream)
    return out


def _extra_b8(torch, nq, stream, steps, warm, hbm_gbs, d_out, d_in, r):
    lb = decode_bytes(d_out, d_in, r, 8)
    ch = Chain(torch, nq, d_out, d_in, r, 8, n_instances(lb), seed=synth.workload_seed(HEADLINE) + 50)
    g = graph_of(torch, lambda: ch.run(nq, stream), stream)
    ms = timed_replays(torch, g, stream, steps, warm)
    us = ms * 1e3 / (steps * ch.n)
    del g, ch
    return {"attn7b_b8": {"us_per_layer": round(us, 3), "GB_s": round(lb / us / 1e3, 1),
                          "frac_hbm": round(lb / us / 1e3 / hbm_gbs, 4)}}


def _extra_block(torch, nq, stream, steps, warm, hbm_gbs, wl, sampler=None):
    """A 7B MLP block or a 70B decoder layer's projections (+ SiLU.mul), decode batch 1."""
    shapes = synth.WORKLOADS[wl]
    block_bytes = sum(decode_bytes(do, di, r, 1) for (_, do, di, r) in shapes)
    reps = max(2, int(np.ceil(3 * L2_BYTES / block_bytes)))
    blocks = []
    for b in range(reps):
        projs = {}
        for idx, (name, do, di, rr) in enumerate(shapes):
            p = synth.make_projection(name, do, di, rr, seed=synth.workload_seed(wl), key=1000 * b + idx)
            projs[name] = nq.Layer.from_host(p.U, p.V, p.s1, p.s2, rr)
        blocks.append(projs)
    need = max(L.workspace_bytes(1) for bl in blocks for L in bl.values())
    for bl in blocks:
        if all(n in bl for n in ("q", "k", "v")):
            need = max(need, nq.group_workspace_bytes([bl[n] for n in ("q", "k", "v")], 1))
        need = max(need, nq.mlp_gate_up_workspace_bytes(bl["gate"], bl["up"], 1))
    ws = torch.zeros(need, dtype=torch.uint8, device="cuda")
    dmodel = shapes[0][2]
    x = torch.zeros((1, dmodel), dtype=torch.bfloat16, device="cuda").normal_()
    bufs = {name: torch.empty((1, do), dtype=torch.bfloat16, device="cuda") for (name, do, di, rr) in shapes}
    h = torch.empty((1, blocks[0]["gate"].d_out), dtype=torch.bfloat16, device="cuda")
    attn_in = torch.zeros((1, shapes[0][1]), dtype=torch.bfloat16, device="cuda").normal_()

    def run_blocks():
        xx = x
        for bl in blocks:
            if "q" in bl:  # q, k, v share their input: one grouped call
                nq.layer_forward_group([bl["q"], bl["k"], bl["v"]], xx, [bufs["q"], bufs["k"], bufs["v"]], ws=ws,
                                       stream=stream)
                nq.layer_forward(bl["o"], attn_in, bufs["o"], ws=ws, stream=stream)
                xin = bufs["o"]
            else:
                xin = xx
            nq.mlp_gate_up(bl["gate"], bl["up"], xin, h, ws=ws, stream=stream)
            nq.layer_forward(bl["down"], h, bufs["down"], ws=ws, stream=stream)
            xx = bufs["down"]

    g = graph_of(torch, run_blocks, stream)
    ms = timed_replays(torch, g, stream, steps, warm, sampler=sampler)
    us = ms * 1e3 / (steps * reps)
    del g, blocks
    return {"us_per_block": round(us, 3), "block_bytes": block_bytes, "GB_s": round(block_bytes / us / 1e3, 1),
            "frac_hbm": round(block_bytes / us / 1e3 / hbm_gbs, 4), "blocks_per_step": reps, "steps": steps,
            "block": "+".join(n for (n, *_r) in shapes) + " + silu_mul",
            "grouped": ("q,k,v one nq_layer_forward_group call (shared input); " if shapes[0][0] == "q" else "")
                       + "gate,up and SiLU.mul one nq_mlp_gate_up call"}


def _extra_prefill(torch, nq, stream, steps, bf16_tf):
    """The 70B gate projection (28672 x 8192, r = 3520) on the tensor-core path."""
    (_, do, di, r), = synth.WORKLOADS["prefill70b"]
    p = synth.make_projection("gate", do, di, r, seed=synth.workload_seed("prefill70b"))
    L = nq.Layer.from_host(p.U, p.V, p.s1, p.s2, r)
    pre = {}
    for M in (64, 512, 2048):
        x = torch.zeros((M, di), dtype=torch.bfloat16, device="cuda").normal_()
        y = torch.empty((M, do), dtype=torch.bfloat16, device="cuda")
        ws = L.workspace(M)
        g = graph_of(torch, lambda: nq.lrb_matmul(L, x, y, ws=ws, stream=stream), stream)
        psteps = max(20, steps)
        ms = timed_replays(torch, g, stream, psteps, 3)
        us = ms * 1e3 / psteps
        flops = 2.0 * M * r * (di + do)
        pre["M%d" % M] = {"us": round(us, 2), "TFLOP_s": round(flops / us / 1e6, 2),
                          "frac_bf16": round(flops / us / 1e6 / bf16_tf, 4)}
        del g
    return pre


def _extra_calib(torch, nq, stream, steps, warm, hbm_gbs, bf16_tf):
    """Scale-only calibration products: the layer transpose at decode batch 1 and the two
    scale gradients at batch 8 (7B attention shape, distinct instances > 3x L2), and the
    scale gradients of the 70B gate at M = 2048 on the tensor cores."""
    out = {}
    (_, do, di, r), = synth.WORKLOADS[HEADLINE]
    for (key, M) in (("transposed_attn7b_b1", 1), ("scale_grads_attn7b_b8", 8)):
        lb = decode_bytes(do, di, r, M)
        ch = Chain(torch, nq, do, di, r, M, n_instances(lb), seed=synth.workload_seed(HEADLINE) + 70 + M)
        ybar = torch.zeros((M, do), dtype=torch.bfloat16, device="cuda").normal_()
        xbar = torch.empty((M, di), dtype=torch.bfloat16, device="cuda")
        if M == 1:
            def run():
                for L in ch.layers:
                    nq.lrb_transposed(L, ybar, xbar, ws=ch.ws, stream=stream)
        else:
            def run():
                for L in ch.layers:
                    nq.lrb_scale_grads(L, ch.x0, ybar, ws=ch.ws, stream=stream)
        g = graph_of(torch, run, stream)
        ms = timed_replays(torch, g, stream, steps, warm)
        us = ms * 1e3 / (steps * ch.n)
        moved = lb if M == 1 else 2 * lb  # the gradients read every weight twice (two passes)
        out[key] = {"us_per_layer": round(us, 3), "GB_s": round(moved / us / 1e3, 1),
                    "frac_hbm": round(moved / us / 1e3 / hbm_gbs, 4),
                    "l2": "no flush: %d distinct layers > 3x L2" % ch.n}
        del g, ch
    (_, do, di, r), = synth.WORKLOADS["prefill70b"]
    p = synth.make_projection("gate", do, di, r, seed=synth.workload_seed("prefill70b"))
    L = nq.Layer.from_host(p.U, p.V, p.s1, p.s2, r)
    M = 2048
    x = torch.zeros((M, di), dtype=torch.bfloat16, device="cuda").normal_()
    ybar = torch.zeros((M, do), dtype=torch.bfloat16, device="cuda").normal_()
    ws = L.workspace(M)
    g = graph_of(torch, lambda: nq.lrb_scale_grads(L, x, ybar, ws=ws, stream=stream), stream)
    ms = timed_replays(torch, g, stream, 3, 2)
    us = ms * 1e3 / 3
    flops = 2 * 2.0 * M * r * (di + do)  # two passes of the two products
    out["scale_grads_prefill70b_gate_M2048"] = {"us": round(us, 2), "TFLOP_s": round(flops / us / 1e6, 2),
                                                "frac_bf16": round(flops / us / 1e6 / bf16_tf, 4)}
    del g
    # latent factors -> packed layer (balancing, scales, signs) for the 70B gate projection
    Uh = torch.randn((do, r), dtype=torch.float32, device="cuda")
    Vh = torch.randn((di, r), dtype=torch.float32, device="cuda")
    g = graph_of(torch, lambda: nq.lrb_from_latent(Uh, Vh, stream=stream), stream)
    ms = timed_replays(torch, g, stream, steps, warm)
    us = ms * 1e3 / steps
    moved = 4 * (do + di) * r + (do + di) * r // 8 + 2 * (do + di)  # fp32 in, bits and fp16 scales out
    out["from_latent_70b_gate"] = {"us": round(us, 2), "GB_s": round(moved / us / 1e3, 1),
                                   "frac_hbm": round(moved / us / 1e3 / hbm_gbs, 4)}
    del g
    return out


def _extra_sign_grads(torch, nq, stream, steps, warm, hbm_gbs, bf16_tf):
    """Gradients with respect to the sign factors (the refinement step's straight-through
    backward): the 7B attention shape at batch 1 (distinct layer instances, one fp32 gradient
    pair of 2 x 4096 x 2048 written per call) and the 70B gate at M = 64 and 2048."""
    out = {}
    (_, do, di, r), = synth.WORKLOADS[HEADLINE]
    ch = Chain(torch, nq, do, di, r, 1, 16, seed=synth.workload_seed(HEADLINE) + 90)
    ybar = torch.zeros((1, do), dtype=torch.bfloat16, device="cuda").normal_()
    gU = torch.empty((do, r), dtype=torch.float32, device="cuda")
    gV = torch.empty((di, r), dtype=torch.float32, device="cuda")
    ws = torch.empty(nq.sign_grads_workspace_bytes(ch.layers[0], 1), dtype=torch.uint8, device="cuda")

    def run():
        for Lc in ch.layers:
            nq.lrb_sign_grads(Lc, ch.x0, ybar, gU=gU, gV=gV, ws=ws, stream=stream)
    g = graph_of(torch, run, stream)
    ms = timed_replays(torch, g, stream, steps, warm)
    us = ms * 1e3 / (steps * ch.n)
    moved = r * (do + di) // 8 + 4 * r * (do + di) + 2 * (do + di) + 4 * (do + di)  # bits, fp32 out, scales, acts
    out["sign_grads_attn7b_b1"] = {"us_per_layer": round(us, 3), "GB_s": round(moved / us / 1e3, 1),
                                   "frac_hbm": round(moved / us / 1e3 / hbm_gbs, 4),
                                   "note": "16 distinct layers; output 2 x 32 MB fp32 per call"}
    del g, ch
    (_, do, di, r), = synth.WORKLOADS["prefill70b"]
    p70 = synth.make_projection("gate", do, di, r, seed=synth.workload_seed("prefill70b"))
    L70 = nq.Layer.from_host(p70.U, p70.V, p70.s1, p70.s2, r)
    gU = torch.empty((do, r), dtype=torch.float32, device="cuda")
    gV = torch.empty((di, r), dtype=torch.float32, device="cuda")
    for M in (64, 2048):
        x = torch.zeros((M, di), dtype=torch.bfloat16, device="cuda").normal_()
        ybar = torch.zeros((M, do), dtype=torch.bfloat16, device="cuda").normal_()
        ws = torch.empty(nq.sign_grads_workspace_bytes(L70, M), dtype=torch.uint8, device="cuda")
        g = graph_of(torch, lambda: nq.lrb_sign_grads(L70, x, ybar, gU=gU, gV=gV, ws=ws, stream=stream), stream)
        ms = timed_replays(torch, g, stream, 20, 3)
        us = ms * 1e3 / 20
        flops = 4.0 * M * r * (di + do)  # two GEMM 1 passes and the two outer products
        wbytes = 4 * r * (do + di)
        out["sign_grads_prefill70b_gate_M%d" % M] = {
            "us": round(us, 2), "TFLOP_s": round(flops / us / 1e6, 2), "frac_bf16": round(flops / us / 1e6 / bf16_tf, 4),
            "out_GB_s": round(wbytes / us / 1e3, 1), "out_frac_hbm": round(wbytes / us / 1e3 / hbm_gbs, 4),
            "traffic": profile_traffic("sign_grads_umma_gate70b_m%d" % M)}
        del g
    return out


def _extra_model70b(torch, nq, stream, hbm_gbs, n_layers=80):
    """One token (batch 1) through the LRB projections of 80 Llama-2-70B decoder layers
    (q, k, v, o, gate, up, down + SiLU.mul each; attention core and norms are not LRB
    matmuls).  Random packed signs and scales generated on the device: every layer distinct."""
    shapes = synth.WORKLOADS["layer70b"]
    gen = torch.Generator(device="cuda")
    gen.manual_seed(synth.workload_seed("layer70b") + 80)

    def words(rows, r):
        ld = -(-(r // 32) // 4) * 4
        return torch.randint(-2 ** 31, 2 ** 31 - 1, (rows, ld), dtype=torch.int32, device="cuda", generator=gen)

    def scales(n):
        return (0.02 * torch.randn(n, device="cuda", generator=gen).abs()).half()

    layers = []
    for _ in range(n_layers):
        layers.append({name: nq.Layer(words(do, r), words(di, r), scales(do), scales(di), r)
                       for (name, do, di, r) in shapes})
    need = max(L.workspace_bytes(1) for bl in layers for L in bl.values())
    need = max(need, nq.group_workspace_bytes([layers[0]["q"], layers[0]["k"], layers[0]["v"]], 1),
               nq.mlp_gate_up_workspace_bytes(layers[0]["gate"], layers[0]["up"], 1))
    ws = torch.zeros(need, dtype=torch.uint8, device="cuda")
    dmodel = shapes[0][2]
    x = torch.zeros((1, dmodel), dtype=torch.bfloat16, device="cuda").normal_()
    bufs = {name: torch.empty((1, do), dtype=torch.bfloat16, device="cuda") for (name, do, di, r) in shapes}
    h = torch.empty((1, layers[0]["gate"].d_out), dtype=torch.bfloat16, device="cuda")

    def token():
        xx = x
        for bl in layers:
            nq.layer_forward_group([bl["q"], bl["k"], bl["v"]], xx, [bufs["q"], bufs["k"], bufs["v"]], ws=ws,
                                   stream=stream)
            nq.layer_forward(bl["o"], bufs["q"], bufs["o"], ws=ws, stream=stream)  # stands in for attention
            nq.mlp_gate_up(bl["gate"], bl["up"], bufs["o"], h, ws=ws, stream=stream)
            nq.layer_forward(bl["down"], h, bufs["down"], ws=ws, stream=stream)
            xx = bufs["down"]

    g = graph_of(torch, token, stream)
    ms = timed_replays(torch, g, stream, 10, 3)
    us = ms * 1e3 / 10
    wbytes = sum(L.U.numel() * 4 + L.V.numel() * 4 + 2 * (L.d_out + L.d_in) for bl in layers for L in bl.values())
    alg = n_layers * sum(decode_bytes(do, di, r, 1) for (_, do, di, r) in shapes)
    del g, layers
    return {"layers": n_layers, "weights_GB": round(wbytes / 1e9, 3), "us_per_token": round(us, 1),
            "tokens_per_s": round(1e6 / us, 1), "GB_s": round(alg / us / 1e3, 1),
            "frac_hbm": round(alg / us / 1e3 / hbm_gbs, 4),
            "note": "LRB projections + SiLU.mul only; o takes q's output in place of attention; q,k,v "
                    "grouped; gate,up and SiLU.mul one fused call"}


def _extra_pack(torch, nq, stream, steps, warm, hbm_gbs):
    """Pack of the 70B gate U: 28672 x 3520 fp32 latent -> packed words."""
    rows, rr = 28672, 3520
    lat = torch.randn((rows, rr), dtype=torch.float32, device="cuda")
    pk = torch.empty((rows, rr // 32), dtype=torch.int32, device="cuda")
    g = graph_of(torch, lambda: nq.pack_signs(lat, r=rr, out=pk, stream=stream), stream)
    ms = timed_replays(torch, g, stream, steps, warm)
    us = ms * 1e3 / steps
    pbytes = 4 * rows * rr + rows * rr // 8
    del g
    return {"us": round(us, 2), "GB_s": round(pbytes / us / 1e3, 1), "frac_hbm": round(pbytes / us / 1e3 / hbm_gbs, 4),
            "traffic": profile_traffic("pack_gate70b_u")}


# --------------------------------------------------------------------------- CPU oracle
def cpu_baseline(budget_s: float):
    """The oracle (plain single-threaded C, fp64, factored order) on the headline layer."""
    import oracle
    (_, d_out, d_in, r), = synth.WORKLOADS[HEADLINE]
    p = synth.make_projection("cpu", d_out, d_in, r, seed=synth.workload_seed(HEADLINE))
    xb = synth.acts_bf16(synth.rng_for(5), (1, d_in))
    times = []
    t_end = time.perf_counter() + budget_s
    while time.perf_counter() < t_end or len(times) < 3:
        t0 = time.perf_counter()
        oracle.factored_packed(p.U, p.V, p.s1, p.s2, r, xb)
        times.append(time.perf_counter() - t0)
    us = statistics.median(times) * 1e6
    return {"value": round(us, 1), "unit": "us/layer", "cores": 1, "kind": "oracle",
            "sample": "%d forwards of the factored fp64 oracle (s1 (.) U (V^T (s2 (.) x))) on one 4096x4096 r=2048 "
                      "layer at batch 1, single thread, median" % len(times)}


def parity_margins(torch, nq, nrows=64):
    """Parity headroom per configuration on sampled rows (the first, the last and a spread): the
    CPU oracle's exact forward against the GPU's bf16 output, as the largest |err| / bound for
    the stated bound 2e-3 S + 1e-5 (S = sum of |terms|) and for that bound plus half a bf16 unit
    of y (the rounding of the output itself).  Runs in the CPU-baseline leg (rank 0, N = 1)."""
    import oracle
    cases = [("attn7b", 0, 1), ("attn7b", 0, 8), ("mlp7b", 0, 1), ("layer70b", 4, 1), ("layer70b", 6, 1),
             ("prefill70b", 0, 64)]
    out = {}
    for wl, idx, M in cases:
        p = synth.make_workload(wl)[idx]
        xb = synth.make_input(wl, p.d_in, M, key=4242)
        L = nq.Layer.from_host(p.U, p.V, p.s1, p.s2, p.r)
        x = torch.from_numpy(np.ascontiguousarray(xb).view(np.int16)).cuda().view(torch.bfloat16)
        y = nq.layer_forward(L, x)
        nq.sync_status()
        yb = y.view(torch.int16).cpu().numpy().view(np.uint16)
        rows = np.unique(np.concatenate([[0, p.d_out - 1], np.linspace(0, p.d_out - 1, nrows).astype(np.int64)]))
        y_ref, S = oracle.dense_packed(p.U, p.V, p.s1, p.s2, p.r, xb, rows=rows)
        got = (yb[:, rows].astype(np.uint32) << 16).view(np.float32).astype(np.float64)
        err = np.abs(got - y_ref)
        bound = 2e-3 * S + 1e-5
        _, e = np.frexp(np.abs(y_ref))
        half_ulp = np.ldexp(0.5, np.maximum(np.where(y_ref == 0, -125, e), -125) - 8)
        out["%s/%s M=%d" % (wl, p.name, M)] = {"strict": round(float((err / bound).max()), 4),
                                                "with_bf16_rounding": round(float((err / (bound + half_ulp)).max()), 4),
                                                "rows": int(rows.size)}
        del L, x, y
    return out


def reference_arm(args):
    rank, world, local = dist_env()
    if rank != 0:
        return None
    base = cpu_baseline(max(1.0, min(args.cpu_seconds, 60.0)))
    steps_us = []
    import oracle
    (_, d_out, d_in, r), = synth.WORKLOADS[HEADLINE]
    p = synth.make_projection("cpu", d_out, d_in, r, seed=synth.workload_seed(HEADLINE))
    xb = synth.acts_bf16(synth.rng_for(6), (args.batch, d_in))
    for _ in range(args.warmup):
        oracle.factored_packed(p.U, p.V, p.s1, p.s2, r, xb)
    for _ in range(args.steps):
        t0 = time.perf_counter()
        oracle.factored_packed(p.U, p.V, p.s1, p.s2, r, xb)
        steps_us.append((time.perf_counter() - t0) * 1e6)
    v = statistics.median(steps_us)
    return {"impl": "reference", "metric": METRIC, "value": round(v, 1), "unit": "us/layer", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(v / 1e3, 3), "higher_is_better": False,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": "Llama-2-7B attention projection d_out=d_in=4096 r=2048 (1.0 bit/weight), decode batch %d"
                                   % args.batch,
                       "batch": args.batch, "layers_per_step": 1},
            "cpu_baseline": {**base, "value": round(v, 1)},
            "e2e": {"value": round(v, 1), "unit": "us/layer", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}


def main():
    args = parse_args()
    rank, world, local = dist_env()
    if args.impl == "reference":
        res = reference_arm(args)
        if res is not None:
            print(json.dumps(res), flush=True)
        return 0
    res = gpu_arm(args, rank, world, local)
    if rank == 0:
        print(json.dumps(res), flush=True)
    return 0


if __name__ == "__main__":
    sys.exit(main())
