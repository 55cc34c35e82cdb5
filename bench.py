#!/usr/bin/env python
"""Benchmark of the expert-routed MoE FFN layer on B200.

A step is one full layer call (route -> plan -> grouped gate/up + SwiGLU -> grouped
down -> combine) over one batch of synthetic hidden states, on weights resident in
HBM. The default run measures the five workloads of the metric (MoE-layer tokens/s at
T = 1, 16, 32, 512, 4096) in one process and prints ONE JSON line on rank 0: the 1-token
decode workload (d=2560, E=512, top-10 + 1 shared, f=1024, int4 g128) is the headline
``value``; every workload has its entry in ``workloads``.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload all|NAME]
    python bench.py --impl reference ...   # the fp64 CPU oracle on host cores

Timing: the K steps of a workload are captured into CUDA graphs; the K-step region is
replayed until at least ``--min-seconds`` have passed, each replay timed with CUDA events
on the launch stream, and the median per-step time over the replays is reported.
L2: each step reads a different copy of the layer's weights (``replicas`` copies, cycled)
and a different hidden batch (a pool of 64), so no step finds its weights in the 126 MB L2
(the inputs of the cycle are far larger than L2).
Multi-GPU: every rank runs its own replica of the layer (weak scaling, no data-path
collective); the time is the max over ranks.
"""
from __future__ import annotations

import argparse
import json
import os
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from expert_routed_ffn_route_b200 import synth  # noqa: E402

HBM_FALLBACK_GBS = 6650.0
TC_FALLBACK_TFLOPS = 1590.0
HBM_NOMINAL_GBS = 8000.0      # the HBM3e figure the decode target is stated against
TC_NOMINAL_TFLOPS = 2250.0    # dense bf16/fp16 tensor-core peak of one B200
L2_BYTES = 126 * 2 ** 20
POOL = 64
ALL_WORKLOADS = ("decode", "verify16", "verify32", "prefill", "long", "prefill_nvfp4",
                 "long_nvfp4")
FP4_OVER_BF16 = 4.0           # nominal dense FP4 / BF16 tensor-core ratio of a B200 (9 / 2.25)
HEADLINE = "decode"


def parse(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=64)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default="all", choices=["all", *synth.CONFIGS])
    ap.add_argument("--replicas", type=int, default=0, help="weight copies cycled (0: auto)")
    ap.add_argument("--min-seconds", type=float, default=1.0,
                    help="replay the K-step region until this much time has passed")
    ap.add_argument("--cpu-seconds", type=float, default=8.0)
    ap.add_argument("--no-cpu", action="store_true", help="skip the CPU oracle baseline")
    return ap.parse_args(argv)


def measured_peaks():
    """(hbm GB/s, tensor TFLOP/s burst, tensor TFLOP/s sustained, kind)."""
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as fh:
            d = json.load(fh)
        return (float(d["hbm_gbs"]), float(d["bf16_tflops"]),
                float(d.get("bf16_tflops_sustained", d["bf16_tflops"])), "measured")
    return HBM_FALLBACK_GBS, TC_FALLBACK_TFLOPS, TC_FALLBACK_TFLOPS, "fallback"


def bank_bytes_per_expert(cfg, fmt=None):
    """(weight bytes, scale bytes) of one expert (gate, up, down) in ``fmt`` (default: the
    routed bank's format). NVFP4: 4-bit codes, one E4M3 byte per 16 values, three fp32
    tensor scales."""
    fmt = cfg.fmt if fmt is None else fmt
    bits = synth.FMT_BITS[fmt]
    w = 3 * cfg.d * cfg.f * bits // 8
    if fmt == "bf16":
        s = 0
    elif fmt == "nvfp4":
        s = 3 * cfg.d * cfg.f // 16 + 3 * 4
    else:
        s = 3 * cfg.d * cfg.f // cfg.group * 2
    return w, s


def layer_flops(cfg):
    """Algorithmic FLOPs of one layer call: 2 * 3 * d * f per (token, expert) pair, over
    the T * k routed pairs and the T shared-expert rows (the router's 2 * T * E * d is
    included too)."""
    return (2 * 3 * cfg.d * cfg.f * (cfg.T * cfg.k + cfg.T * cfg.n_shared)
            + 2 * cfg.T * cfg.E * cfg.d)


def pool_size(cfg):
    """Hidden batches cycled: 64 for the small calls (each touches few experts, so the
    batches must differ), fewer for large T (every batch touches nearly every expert)."""
    return int(min(POOL, max(4, 4096 // cfg.T)))


def replicas_for(cfg, requested=0):
    """Weight copies cycled: enough that a cycle of steps touches more than 4x L2."""
    if requested > 0:
        return requested
    w_b, s_b = bank_bytes_per_expert(cfg)
    touched = min(cfg.E, cfg.T * cfg.k) + 1
    step_bytes = touched * (w_b + s_b) + cfg.E * cfg.d * 2
    return int(min(16, max(1, np.ceil(4 * L2_BYTES / step_bytes))))


def workload_config(cfg, world, replicas=0):
    """The ``config`` object of a bench line (identical for both arms)."""
    R = replicas_for(cfg, replicas)
    weights = (f"{cfg.fmt} g{cfg.group}" if cfg.fmt != "nvfp4" else
               "nvfp4 routed (E2M1, E4M3 per 16, fp32 per matrix; activations NVFP4 per row), "
               f"{cfg.shared_fmt or cfg.fmt} shared")
    return {"workload": cfg.name, "T": cfg.T, "d": cfg.d, "E": cfg.E, "k": cfg.k,
            "f": cfg.f, "n_shared": cfg.n_shared, "weights": weights,
            "router": "bf16, fp32 logits" + (", Zipf(1.1) bias" if cfg.zipf_s else ""),
            "parallelism": f"replicas x{world}",
            "l2": (f"inputs larger than L2: {R} weight copies x {pool_size(cfg)} hidden "
                   "batches cycled"),
            "cuda_graph": True}


def max_over_ranks(values, device="cpu"):
    """Element-wise max of per-rank values over the process group (the job is as fast as its
    slowest rank); identity without a process group."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return [float(v) for v in values]
    t = torch.tensor([float(v) for v in values], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(v) for v in t.tolist()]


KERNEL_SOURCES = {
    "decode_fused": ("decode_fused.cu", "gemv_frag.cuh", "pipeline.cuh", "common.cuh"),
    "gemv_tma": ("gemv_tma.cu", "gemv_frag.cuh", "pipeline.cuh", "common.cuh"),
    "tc_grouped": ("tc_grouped.cu", "tc_common.cuh", "pipeline.cuh", "common.cuh"),
    "nv_grouped": ("nvfp4_grouped.cu", "tc_common.cuh", "pipeline.cuh", "common.cuh"),
}


def source_tokens(text):
    """C/C++/CUDA source with comments removed and whitespace collapsed: what the compiler
    sees, so that edits to comments alone keep a digest."""
    import re
    out, i, n = [], 0, len(text)
    while i < n:
        c = text[i]
        if c == '"' or c == "'":  # string or character literal, kept whole
            j = i + 1
            while j < n and text[j] != c:
                j += 2 if text[j] == "\\" else 1
            out.append(text[i:j + 1])
            i = j + 1
        elif text.startswith("//", i):
            j = text.find("\n", i)
            i = n if j < 0 else j
        elif text.startswith("/*", i):
            j = text.find("*/", i + 2)
            i = n if j < 0 else j + 2
            out.append(" ")
        else:
            out.append(c)
            i += 1
    return re.sub(r"\s+", " ", "".join(out)).strip()


def kernel_source_digest(kernel="gemv_tma", read=None):
    """Digest of the sources of one kernel, comments and whitespace aside (ties committed ncu
    counters to the code they were taken from). ``read`` maps a file name under csrc/ to its
    text (default: the working tree)."""
    import hashlib
    if read is None:
        def read(name):
            with open(os.path.join(ROOT, "expert_routed_ffn_route_b200", "csrc", name)) as fh:
                return fh.read()
    h = hashlib.sha256()
    for f in KERNEL_SOURCES[kernel]:
        h.update(source_tokens(read(f)).encode())
    return h.hexdigest()[:16]


def profiled_traffic(workload, kernel):
    """DRAM bytes per launch of the dominant kernel from the committed ncu summary
    ``profiles/<kernel>_gate_up_<workload>.md`` (``profiles/<kernel>_<workload>.md`` for the
    single-kernel layer), if it was captured from the current kernel sources (else None)."""
    import re
    name = f"{kernel}_{workload}.md" if kernel == "decode_fused" else f"{kernel}_gate_up_{workload}.md"
    path = os.path.join(ROOT, "profiles", name)
    if not os.path.exists(path):
        return None
    text = open(path).read()
    m = re.search(r"traffic_bytes_per_launch:\s*([0-9.]+)", text)
    d = re.search(r"source_digest:\s*([0-9a-f]+)", text)
    if not m or not d or d.group(1) != kernel_source_digest(kernel):
        return None
    return float(m.group(1))


# ----------------------------------------------------------------------------- CPU oracle

def _oracle_bank(b):
    if b is None:
        return None
    d = b.arrays()
    d.update(fmt=b.fmt, group=b.group)
    return d


def _blas_threads():
    try:
        from threadpoolctl import threadpool_info
        return max([i.get("num_threads", 1) for i in threadpool_info()] or [1])
    except Exception:
        return os.cpu_count()


# Tokens of the batched oracle call timed per workload: the whole batch where that ends in
# seconds, else the first tokens of it (the oracle dequantises each touched expert once per
# call, about 0.1 s an expert, so its cost grows with the experts a slice touches).
CPU_SLICE = {"tiny": 64, "decode": 1, "verify16": 8, "verify32": 8, "prefill": 16, "long": 64,
             "prefill_nvfp4": 8, "long_nvfp4": 32}


def cpu_oracle_rate(cfg, L, seconds, n_tokens=None):
    """Tokens/s of the fp64 oracle on this host, on a bounded sample of the workload: batched
    layer calls on the first ``n_tokens`` tokens of the batch (every touched expert
    dequantised once per call, as the workload's own call does), repeated until ``seconds``
    pass (at least one call)."""
    from oracle import moe_oracle as O
    from oracle import nvfp4 as NV
    routed, shared = _oracle_bank(L.routed), _oracle_bank(L.shared)
    forward = NV.layer_forward_nvfp4 if cfg.fmt == "nvfp4" else O.layer_forward
    n = L.x.shape[0] if n_tokens is None else min(n_tokens, L.x.shape[0])
    x = L.x[:n]
    t0 = time.perf_counter()
    done = calls = 0
    while True:
        forward(x, L.router_w, L.router_bias, routed, shared, cfg.k)
        done += n
        calls += 1
        if time.perf_counter() - t0 >= seconds:
            break
    el = time.perf_counter() - t0
    sample = (f"{calls} batched layer call(s) on the first {n} of the {cfg.T} tokens of "
              f"'{cfg.name}' (each touched expert dequantised once a call) in {el:.1f} s")
    return done / el, _blas_threads(), sample


def cpu_baseline(cfg, L, seconds, one_thread=True):
    """The oracle's tokens/s with the host's BLAS threads (``value``) and, for the headline,
    with one thread (``value_1thread``)."""
    n = CPU_SLICE.get(cfg.name)
    rate, cores, sample = cpu_oracle_rate(cfg, L, seconds, n)
    out = {"value": rate, "unit": "tokens/s", "cores": cores, "kind": "oracle", "sample": sample}
    if not one_thread:
        return out
    try:
        from threadpoolctl import threadpool_limits
    except Exception:
        return out
    with threadpool_limits(limits=1):
        r1, _, s1 = cpu_oracle_rate(cfg, L, seconds / 3, n)
    out.update(value_1thread=r1, sample_1thread=s1)
    return out


def oracle_inputs(cfg, n_tokens=None):
    """Inputs of a workload for the oracle with only the experts its tokens touch drawn
    (the others are never read); ``n_tokens`` restricts the call to its first tokens."""
    from oracle import moe_oracle as O
    L = synth.make_layer(cfg, routed=synth.make_bank(cfg, "routed", experts=[]),
                         shared=synth.make_bank(cfg, "shared") if cfg.n_shared else None)
    n_tokens = CPU_SLICE.get(cfg.name) if n_tokens is None else n_tokens
    if n_tokens is not None:
        L.x = L.x[:n_tokens]
    need = np.unique(O.select_topk(O.router_logits(L.x, L.router_w, L.router_bias), cfg.k)[0])
    L.routed = synth.make_bank(cfg, "routed", experts=need)
    return L


# ----------------------------------------------------------------------------- clocks

class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.gpu = gpu_index
        self.proc = None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None
        return self

    def __exit__(self, *a):
        self.lines = []
        if self.proc is not None:
            self.proc.terminate()
            try:
                out, _ = self.proc.communicate(timeout=5)
            except Exception:
                self.proc.kill()
                out = ""
            self.lines = [l for l in out.splitlines() if l.strip()]

    def summary(self):
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for l in getattr(self, "lines", []):
            parts = [p.strip() for p in l.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                mx = float(parts[2])
            except ValueError:
                continue
            for n, v in zip(names, parts[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        return {"sm_mhz": float(np.median(sm)) if sm else None, "sm_max_mhz": mx,
                "reasons": sorted(reasons), "samples": len(sm)}


# ----------------------------------------------------------------------------- GPU arm

class BankCache:
    """Host-side weight banks, drawn once per (format, seed, shape) and reused by the
    workloads that share them (decode, verify and prefill use one int4 bank)."""

    def __init__(self):
        self.banks = {}

    def get(self, cfg, which):
        key = (which, cfg.fmt if which == "routed" else (cfg.shared_fmt or cfg.fmt), cfg.seed,
               cfg.d, cfg.f, cfg.E if which == "routed" else cfg.n_shared)
        if key not in self.banks:
            self.banks[key] = synth.make_bank(cfg, which)
        return self.banks[key]


def run_workload(name, args, world, local_rank, cache):
    """Times one workload; returns its bench entry (and the host inputs)."""
    import torch
    from expert_routed_ffn_route_b200 import binding as B
    dev = torch.device("cuda", local_rank)
    cfg = synth.CONFIGS[name]

    # ---- inputs
    routed = cache.get(cfg, "routed")
    shared = cache.get(cfg, "shared") if cfg.n_shared else None
    L = synth.make_layer(cfg, routed=routed, shared=shared)
    n_pool = pool_size(cfg)
    pool = [L.x] + [synth.make_hidden(cfg, L.router_w, L.router_bias, stream=f"pool{i}")
                    for i in range(1, n_pool)]
    base = B.DeviceLayer(L, device=dev)
    x_dev = [torch.from_numpy(x.view(np.int16)).to(dev).view(torch.bfloat16) for x in pool]

    w_b, s_b = bank_bytes_per_expert(cfg)
    per_exp = w_b + s_b
    nv = cfg.fmt == "nvfp4"
    sw_b, ss_b = bank_bytes_per_expert(cfg, cfg.shared_fmt or cfg.fmt)
    per_shared = (sw_b + ss_b) if L.shared is not None else 0
    router_b = cfg.E * cfg.d * 2
    R = replicas_for(cfg, args.replicas)
    layers = [base]
    for _ in range(R - 1):
        b2 = {}
        for bn, bank in base.banks.items():
            b2[bn] = None if bank is None else {
                k: (v.clone() if hasattr(v, "clone") else v) for k, v in bank.items()}
        layers.append(B.DeviceLayer.from_tensors(
            cfg, base.router_w.clone(),
            None if base.router_bias is None else base.router_bias.clone(),
            b2["routed"], b2["shared"]))
    descs = [l.descriptor(cfg.T) for l in layers]
    ws = B.alloc_workspace(descs[0], device=dev)
    out = torch.empty((cfg.T, cfg.d), dtype=torch.bfloat16, device=dev)
    idx_buf = torch.empty((cfg.T, cfg.k), dtype=torch.int32, device=dev)

    # ---- algorithmic bytes per pool entry: the layer, and its grouped gate/up launch
    gu_bytes, layer_bytes = [], []
    n_rows = cfg.T * cfg.k
    for xd in x_dev:
        B.layer_forward(descs[0], xd, ws, out=out, topk_idx=idx_buf)
        ur = np.unique(idx_buf.cpu().numpy()).size  # routed experts touched
        if nv:
            # gate/up stage: routed gate/up codes and scales, the shared expert's gate/up, x
            # (bf16, read to quantise), the quantised rows read by the GEMM, h written (fp32)
            gu = (ur * (2 * per_exp // 3) + 2 * per_shared // 3 + cfg.T * cfg.d * 2
                  + n_rows * cfg.d * 9 // 16 + n_rows * cfg.f * 4 + cfg.T * cfg.f * 2)
            lb = ur * per_exp + per_shared + router_b + 2 * cfg.T * cfg.d * 2
        else:
            u = ur + (1 if L.shared is not None else 0)
            gu = u * (2 * per_exp // 3) + cfg.T * cfg.d * 2 + (n_rows + cfg.T) * cfg.f * 2
            lb = u * per_exp + router_b + 2 * cfg.T * cfg.d * 2
        gu_bytes.append(gu)
        layer_bytes.append(lb)
    torch.cuda.synchronize()

    stream = torch.cuda.Stream(device=dev)
    fused = B.launches_per_call(descs[0]) == 1
    K = args.steps

    def step(i, marks=None):
        B.layer_forward(descs[i % R], x_dev[i % n_pool], ws, out=out, marks=marks, stream=stream)

    with torch.cuda.stream(stream):
        for i in range(args.warmup):
            step(i)
    torch.cuda.synchronize()

    # K steps captured once into CUDA graphs of up to G steps each (a decode step is a few
    # microseconds of GPU work; per-step host launches would dominate)
    G = 64
    plain = []
    for a0 in range(0, K, G):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=stream):
            for i in range(a0, min(K, a0 + G)):
                step(i)
        plain.append(g)
    # the grouped gate/up launch of the multi-kernel path, bracketed by stage marks (CUDA
    # events recorded on the launch stream; marks 2 and 3 enclose the gate/up stage)
    n_mark = min(K, 256)
    ev = []
    marked = []
    if not fused:
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
              for _ in range(n_mark)]
        for a, b in ev:  # torch creates the CUDA event on its first record
            a.record(stream)
            b.record(stream)
        for a0 in range(0, n_mark, G):
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=stream):
                for i in range(a0, min(n_mark, a0 + G)):
                    marks = [None] * B.N_MARKS
                    marks[2], marks[3] = ev[i]
                    step(i, marks)
            marked.append(g)
    with torch.cuda.stream(stream):  # one untimed pass over every graph
        for g in plain + marked:
            g.replay()
    torch.cuda.synchronize()

    def replay(graphs):
        with torch.cuda.stream(stream):
            for g in graphs:
                g.replay()

    # ---- timed regions: the K-step region replayed until min_seconds have passed
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
    torch.cuda.synchronize()
    region_ms = []
    with ClockSampler(local_rank) as clk:
        time.sleep(0.25)  # let the sampler start before the timed regions
        t_wall = time.perf_counter()
        torch.cuda.nvtx.range_push("timed")  # lets a profiler take the timed launches only
        while True:
            e0 = torch.cuda.Event(enable_timing=True)
            e1 = torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            replay(plain)
            e1.record(stream)
            e1.synchronize()
            region_ms.append(e0.elapsed_time(e1))
            if time.perf_counter() - t_wall >= args.min_seconds and len(region_ms) >= 3:
                break
        torch.cuda.nvtx.range_pop()
    if world > 1:
        dist.barrier()
    ms_region = float(np.median(region_ms))
    (ms_region,) = max_over_ranks([ms_region], device=dev)
    ms_per_step = ms_region / K

    # ---- dominant kernel: the single-kernel layer is the whole step; otherwise the gate/up
    # launch from the marked pass
    if fused:
        k_ms_avg = ms_per_step
        achieved = float(np.mean([layer_bytes[i % n_pool] for i in range(K)])) / (ms_per_step * 1e-3) / 1e9
        kernel_name = "decode_fused_kernel (whole layer, one launch)"
        prof_kernel = "decode_fused"
    else:
        torch.cuda.synchronize()
        replay(marked)
        torch.cuda.synchronize()
        k_ms = [ev[i][0].elapsed_time(ev[i][1]) for i in range(n_mark)]
        k_bytes = [gu_bytes[i % n_pool] for i in range(n_mark)]
        k_ms_avg = float(np.mean(k_ms))
        achieved = float(np.sum(k_bytes) / (np.sum(k_ms) * 1e-3) / 1e9)
        tc = cfg.T >= 16
        if nv:
            kernel_name = ("grouped gate/up + SwiGLU stage (FP4 tcgen05 kind::mxf4nvf4 with the "
                           "activation quantiser, and the bf16 shared expert)")
            prof_kernel = "nv_grouped"
        else:
            kernel_name = "grouped gate/up + SwiGLU" + (" (tcgen05, with its row gather)" if tc else "")
            prof_kernel = "tc_grouped" if tc else "gemv_tma"

    # ---- end to end through the public call with host buffers
    x_host = [torch.from_numpy(x.view(np.int16)).view(torch.bfloat16).pin_memory()
              for x in pool[:8]]
    out_host = torch.empty((cfg.T, cfg.d), dtype=torch.bfloat16).pin_memory()
    x_stage = torch.empty((cfg.T, cfg.d), dtype=torch.bfloat16, device=dev)
    e_steps = max(8, min(K, 200))

    def e2e_step(i):
        x_stage.copy_(x_host[i % len(x_host)], non_blocking=True)
        B.layer_forward(descs[i % R], x_stage, ws, out=out, stream=stream)
        out_host.copy_(out, non_blocking=True)

    # eager: one host launch sequence a step
    torch.cuda.synchronize()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        e0.record(stream)
        for i in range(e_steps):
            e2e_step(i)
        e1.record(stream)
    torch.cuda.synchronize()
    eager_ms = e0.elapsed_time(e1) / e_steps
    # as a decode loop runs it: the steps (each with its copies) captured in a CUDA graph
    GE = 32
    ge = torch.cuda.CUDAGraph()
    with torch.cuda.graph(ge, stream=stream):
        for i in range(GE):
            e2e_step(i)
    with torch.cuda.stream(stream):
        ge.replay()
    torch.cuda.synchronize()
    reps = max(1, e_steps // GE)
    with torch.cuda.stream(stream):
        e0.record(stream)
        for _ in range(reps):
            ge.replay()
        e1.record(stream)
    torch.cuda.synchronize()
    e2e_ms = e0.elapsed_time(e1) / (reps * GE)
    del ge
    (e2e_ms, eager_ms) = max_over_ranks([e2e_ms, eager_ms], device=dev)
    status = B.device_status(descs[0], ws)
    site = B.device_wait_site(descs[0], ws) if status else 0

    hbm, tc_burst, tc_sust, peak_kind = measured_peaks()
    lb = float(np.mean(layer_bytes))
    layer_gbs = lb / (ms_per_step * 1e-3) / 1e9
    flops = layer_flops(cfg)
    tflops = flops / (ms_per_step * 1e-3) / 1e12
    tensor = {"flops_per_step": flops, "achieved_tflops": tflops,
              "peak_sustained": tc_sust, "frac": tflops / tc_sust,
              "peak_burst": tc_burst, "frac_burst": tflops / tc_burst,
              "peak_nominal": TC_NOMINAL_TFLOPS, "frac_nominal": tflops / TC_NOMINAL_TFLOPS}
    if nv:
        # routed experts on the FP4 tensor cores (peak: the measured bf16 figure x the nominal
        # FP4/BF16 ratio), shared expert and router at the bf16 rate: the fraction is the time
        # the contraction needs at those peaks over the step time
        f_routed = 2 * 3 * cfg.d * cfg.f * cfg.T * cfg.k
        f_rest = flops - f_routed

        def ideal_s(peak_tf):
            return (f_routed / (FP4_OVER_BF16 * peak_tf) + f_rest / peak_tf) / 1e12

        step_s = ms_per_step * 1e-3
        tensor.update(frac=ideal_s(tc_sust) / step_s, frac_burst=ideal_s(tc_burst) / step_s,
                      frac_nominal=ideal_s(TC_NOMINAL_TFLOPS) / step_s,
                      fp4_flops_per_step=f_routed,
                      peak_fp4_sustained=FP4_OVER_BF16 * tc_sust,
                      peak_kind="fp4 = measured bf16 x 4 (nominal ratio) for the routed "
                                "experts, measured bf16 for the rest")
    roof = {"bound": "hbm", "kernel": kernel_name, "achieved": achieved, "peak": hbm,
            "unit": "GB/s", "frac": achieved / hbm, "peak_kind": peak_kind,
            "frac_nominal": achieved / HBM_NOMINAL_GBS,
            "traffic": profiled_traffic(cfg.name, prof_kernel),
            "avg_launch_ms": k_ms_avg,
            "layer_bytes": lb, "layer_achieved": layer_gbs, "layer_frac": layer_gbs / hbm,
            "layer_frac_nominal": layer_gbs / HBM_NOMINAL_GBS,
            "tensor": tensor}
    entry = {
        "metric": f"MoE-layer tokens/s ({cfg.name}, T={cfg.T})",
        "value": world * cfg.T / (ms_per_step * 1e-3),
        "unit": "tokens/s",
        "ms_per_step": ms_per_step,
        "steps": K,
        "regions": len(region_ms),
        "region_ms": {"median": ms_region, "min": float(np.min(region_ms)),
                      "max": float(np.max(region_ms))},
        "dtype": (f"{cfg.fmt} weights, bf16 activations, fp32 accumulate" if not nv else
                  "nvfp4 weights and activations (routed), bf16 shared expert, fp32 accumulate"),
        "config": workload_config(cfg, world, args.replicas),
        "roofline": roof,
        "e2e": {"value": world * cfg.T / (e2e_ms * 1e-3), "unit": "tokens/s",
                "h2d_bytes_per_step": cfg.T * cfg.d * 2, "d2h_bytes_per_step": cfg.T * cfg.d * 2,
                "mode": (f"CUDA graphs of {GE} steps, each: the step's hidden batch copied from "
                         "pinned host memory, moe_layer_forward, the output copied to pinned host "
                         "memory"),
                "eager_value": world * cfg.T / (eager_ms * 1e-3)},
        "gpu_launches_per_step": B.launches_per_call(descs[0]),
        "clocks": clk.summary(),
        "device_status": status,
    }
    if status:
        entry["device_wait_site"] = site
    if cfg.T >= 512:  # the tensor-core workloads: the contraction's share of the roofline
        roof["tc_frac"] = roof["tensor"]["frac"]
    del layers, base, descs, ws, x_dev
    torch.cuda.synchronize()
    torch.cuda.empty_cache()
    return entry, L, cfg


def main(argv=None):
    args = parse(argv)
    rank = int(os.environ.get("RANK", 0))
    world = int(os.environ.get("WORLD_SIZE", 1))
    local_rank = int(os.environ.get("LOCAL_RANK", 0))
    names = list(ALL_WORKLOADS) if args.workload == "all" else [args.workload]
    head = HEADLINE if args.workload == "all" else args.workload

    if args.impl == "reference":
        if rank != 0:
            return 0
        cfg = synth.CONFIGS[head]
        L = oracle_inputs(cfg)
        t0 = time.perf_counter()
        cb = cpu_baseline(cfg, L, args.cpu_seconds, one_thread=False)
        rate = cb["value"]
        line = {"impl": "reference", "metric": f"MoE-layer tokens/s ({cfg.name}, T={cfg.T})",
                "value": rate, "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
                "warmup": args.warmup, "ms_per_step": 1e3 * cfg.T / rate,
                "higher_is_better": True, "scaling": "weak",
                "vs_baseline": None, "dtype": "f64", "data": "synthetic",
                "config": workload_config(cfg, world, args.replicas),
                "cpu_baseline": cb,
                "e2e": {"value": rate, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                        "d2h_bytes_per_step": 0},
                "wall_s": time.perf_counter() - t0}
        print(json.dumps(line))
        return 0

    import torch
    torch.cuda.set_device(local_rank)
    if world > 1:
        import torch.distributed as dist
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=300),
                                device_id=torch.device("cuda", local_rank))
    from expert_routed_ffn_route_b200 import binding as B
    B.load_library()
    cache = BankCache()
    entries, inputs = {}, {}
    for n in names:
        entries[n], L, cfg = run_workload(n, args, world, local_rank, cache)
        inputs[n] = (L, cfg)
    if rank == 0 and world == 1 and not args.no_cpu:
        for n in names:
            L, cfg = inputs[n]
            entries[n]["cpu_baseline"] = cpu_baseline(cfg, L, args.cpu_seconds,
                                                      one_thread=(n == head))
    cache.banks.clear()
    h = entries[head]
    res = {
        "metric": h["metric"],
        "value": h["value"],
        "unit": "tokens/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": h["ms_per_step"],
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": h["dtype"],
        "data": "synthetic (seeded; shapes of the pages' model, random weights)",
        "config": h["config"],
        "roofline": h["roofline"],
        "e2e": h["e2e"],
        "gpu_launches": h["gpu_launches_per_step"] * args.steps,
        "clocks": h["clocks"],
        "device_status": h["device_status"],
        "timing": (f"median over {h['regions']} replays of the {args.steps}-step region "
                   f"(each >= {args.min_seconds} s in total), CUDA events on the launch stream"),
    }
    if "cpu_baseline" in h:
        res["cpu_baseline"] = h["cpu_baseline"]
    if len(names) > 1:
        res["workloads"] = entries
    if rank == 0:
        print(json.dumps(res))
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
