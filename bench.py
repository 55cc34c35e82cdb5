#!/usr/bin/env python
"""Benchmark of the expert-routed MoE FFN layer on B200.

A step is one full layer call (route -> plan -> grouped gate/up + SwiGLU -> grouped
down -> combine) over one batch of synthetic hidden states, on weights resident in
HBM. Default workload: 1-token decode (d=2560, E=512, top-10 + 1 shared, f=1024,
int4 g128). Prints ONE JSON line on rank 0.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME]
    python bench.py --impl reference ...   # the fp64 CPU oracle on host cores

L2: each step reads a different copy of the layer's weights (``replicas`` copies,
cycled) and a different hidden batch (a pool of 64), so no step finds its weights in
the 126 MB L2 (the inputs of the cycle are far larger than L2).
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
L2_BYTES = 126 * 2 ** 20
POOL = 64


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20000)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default="decode", choices=list(synth.CONFIGS))
    ap.add_argument("--replicas", type=int, default=0, help="weight copies cycled (0: auto)")
    ap.add_argument("--no-graph", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=12.0)
    ap.add_argument("--stage-times", action="store_true",
                    help="also report per-stage CUDA-event times (stage marks block overlap)")
    return ap.parse_args()


def measured_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as fh:
            d = json.load(fh)
        return float(d["hbm_gbs"]), "measured"
    return HBM_FALLBACK_GBS, "fallback"


def bank_bytes_per_expert(cfg):
    bits = synth.FMT_BITS[cfg.fmt]
    w = 3 * cfg.d * cfg.f * bits // 8
    s = 0 if cfg.fmt == "bf16" else 3 * cfg.d * cfg.f // cfg.group * 2
    return w, s


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
    "tc_grouped": ("tc_grouped.cu", "pipeline.cuh", "common.cuh"),
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


def profiled_traffic(workload, kernel="gemv_tma"):
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

def cpu_oracle_rate(cfg, L, seconds):
    """Tokens/s of the fp64 oracle on this host, on a bounded sample of the workload:
    whole calls of up to 1 token each on successive tokens until `seconds` pass."""
    from oracle import moe_oracle as O

    def bank_dict(b):
        if b is None:
            return None
        d = b.arrays()
        d.update(fmt=b.fmt, group=b.group)
        return d
    routed, shared = bank_dict(L.routed), bank_dict(L.shared)
    t0 = time.perf_counter()
    done = 0
    while True:
        t = done % L.x.shape[0]
        O.layer_forward(L.x[t:t + 1], L.router_w, L.router_bias, routed, shared, cfg.k)
        done += 1
        if time.perf_counter() - t0 >= seconds:
            break
    el = time.perf_counter() - t0
    cores = os.cpu_count()
    try:
        from threadpoolctl import threadpool_info
        cores = max([i.get("num_threads", 1) for i in threadpool_info()] or [1])
    except Exception:
        pass
    return done / el, cores, f"{done} single-token layer calls of '{cfg.name}' in {el:.1f} s"


def cpu_baseline(cfg, L, seconds):
    """The oracle's tokens/s with the host's BLAS threads (``value``) and with one thread
    (``value_1thread``, on a sample of a third of the time)."""
    rate, cores, sample = cpu_oracle_rate(cfg, L, seconds)
    out = {"value": rate, "unit": "tokens/s", "cores": cores, "kind": "oracle", "sample": sample}
    try:
        from threadpoolctl import threadpool_limits
    except Exception:
        return out
    with threadpool_limits(limits=1):
        r1, _, s1 = cpu_oracle_rate(cfg, L, seconds / 3)
    out.update(value_1thread=r1, sample_1thread=s1)
    return out


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

def run_ours(args, rank, world, local_rank):
    import torch
    from expert_routed_ffn_route_b200 import binding as B
    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    cfg = synth.CONFIGS[args.workload]
    B.load_library()

    # ---- inputs
    routed = synth.make_bank(cfg, "routed")
    shared = synth.make_bank(cfg, "shared")
    L = synth.make_layer(cfg, routed=routed, shared=shared)
    pool = [L.x] + [synth.make_hidden(cfg, L.router_w, L.router_bias, stream=f"pool{i}")
                    for i in range(1, POOL)]
    base = B.DeviceLayer(L, device=dev)
    x_dev = [torch.from_numpy(x.view(np.int16)).to(dev).view(torch.bfloat16) for x in pool]

    w_b, s_b = bank_bytes_per_expert(cfg)
    per_exp = w_b + s_b
    router_b = cfg.E * cfg.d * 2
    # replicas: enough weight copies that a cycle touches > 4x L2
    if args.replicas > 0:
        R = args.replicas
    else:
        touched = min(cfg.E, cfg.T * cfg.k) + 1
        step_bytes = touched * per_exp + router_b
        R = int(min(16, max(1, np.ceil(4 * L2_BYTES / step_bytes))))
    layers = [base]
    for _ in range(R - 1):
        b2 = {}
        for name, bank in base.banks.items():
            b2[name] = None if bank is None else {
                k: (v.clone() if hasattr(v, "clone") else v) for k, v in bank.items()}
        layers.append(B.DeviceLayer.from_tensors(
            cfg, base.router_w.clone(),
            None if base.router_bias is None else base.router_bias.clone(),
            b2["routed"], b2["shared"]))
    descs = [l.descriptor(cfg.T) for l in layers]
    ws = B.alloc_workspace(descs[0], device=dev)
    out = torch.empty((cfg.T, cfg.d), dtype=torch.bfloat16, device=dev)
    idx_buf = torch.empty((cfg.T, cfg.k), dtype=torch.int32, device=dev)

    # ---- algorithmic bytes of the dominant kernel (grouped gate/up) per pool entry
    gu_bytes, layer_bytes = [], []
    for xd in x_dev:
        B.layer_forward(descs[0], xd, ws, out=out, topk_idx=idx_buf)
        u = np.unique(idx_buf.cpu().numpy()).size + (1 if L.shared is not None else 0)
        gu = u * (2 * per_exp // 3) + cfg.T * cfg.d * 2 + (cfg.T * cfg.k + cfg.T) * cfg.f * 2
        gu_bytes.append(gu)
        layer_bytes.append(u * per_exp + router_b + 2 * cfg.T * cfg.d * 2)
    torch.cuda.synchronize()

    stream = torch.cuda.Stream(device=dev)
    n_mark = min(args.steps, 256)
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(n_mark)]
    for a, b in ev:  # torch creates the CUDA event on its first record
        a.record(stream)
        b.record(stream)

    # The dominant kernel: the single-kernel layer when a call is one launch (its marks
    # bracket the whole call), else the grouped gate/up kernel (marks 2 and 3).
    fused = B.launches_per_call(descs[0]) == 1
    mark_pair = (0, B.N_MARKS - 1) if fused else (2, 3)
    dom_bytes = layer_bytes if fused else gu_bytes

    def step(i, marked=False):
        marks = None
        if marked:
            marks = [None] * B.N_MARKS
            marks[mark_pair[0]], marks[mark_pair[1]] = ev[i % n_mark]
        B.layer_forward(descs[i % R], x_dev[i % POOL], ws, out=out, marks=marks, stream=stream)

    with torch.cuda.stream(stream):
        for i in range(args.warmup):
            step(i)
    torch.cuda.synchronize()

    # The K timed steps are captured once into CUDA graphs of up to G steps each (a
    # decode step is a few microseconds of GPU work; per-step host launches would
    # dominate). A second, shorter pass with stage marks around the gate/up kernel gives
    # that kernel's launch duration from CUDA events.
    G = 64
    plain, marked = [], []
    if not args.no_graph:
        for a0 in range(0, args.steps, G):
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=stream):
                for i in range(a0, min(args.steps, a0 + G)):
                    step(i)
            plain.append(g)
        for a0 in range(0, n_mark, G):
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=stream):
                for i in range(a0, min(n_mark, a0 + G)):
                    step(i, marked=True)
            marked.append(g)
        with torch.cuda.stream(stream):  # one untimed pass over every graph
            for g in plain + marked:
                g.replay()
        torch.cuda.synchronize()

    def run(graphs, n, with_marks):
        with torch.cuda.stream(stream):
            if graphs:
                for g in graphs:
                    g.replay()
            else:
                for i in range(n):
                    step(i, marked=with_marks)

    # ---- timed region
    t_start = torch.cuda.Event(enable_timing=True)
    t_end = torch.cuda.Event(enable_timing=True)
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
    torch.cuda.synchronize()
    with ClockSampler(local_rank) as clk:
        time.sleep(0.3)  # let the sampler start before the timed region
        torch.cuda.nvtx.range_push("timed")
        t_start.record(stream)
        run(plain, args.steps, False)
        t_end.record(stream)
        torch.cuda.synchronize()
        torch.cuda.nvtx.range_pop()
    if world > 1:
        dist.barrier()
    ms = t_start.elapsed_time(t_end)

    # dominant kernel: gate/up launches of the marked pass (CUDA events on the launch stream)
    torch.cuda.synchronize()
    run(marked, n_mark, True)
    torch.cuda.synchronize()
    k_ms = [ev[i][0].elapsed_time(ev[i][1]) for i in range(n_mark)]
    k_bytes = [dom_bytes[i % POOL] for i in range(n_mark)]
    gu_avg_ms = float(np.mean(k_ms))
    achieved = float(np.sum(k_bytes) / (np.sum(k_ms) * 1e-3) / 1e9)

    stage_ms = None
    if args.stage_times:
        n_st = min(args.steps, 200)
        sev = [[torch.cuda.Event(enable_timing=True) for _ in range(B.N_MARKS)]
               for _ in range(n_st)]
        for row in sev:  # torch creates the CUDA event on its first record
            for e_ in row:
                e_.record(stream)
        with torch.cuda.stream(stream):
            for i in range(n_st):
                B.layer_forward(descs[i % R], x_dev[i % POOL], ws, out=out, marks=sev[i],
                                stream=stream)
        torch.cuda.synchronize()
        names = ["route", "plan", "gate_up", "down", "combine"]
        stage_ms = {n: float(np.mean([sev[i][j].elapsed_time(sev[i][j + 1])
                                      for i in range(n_st // 2, n_st)]))
                    for j, n in enumerate(names)}

    # ---- end to end through the public call with host buffers
    x_host = [torch.from_numpy(x.view(np.int16)).view(torch.bfloat16).pin_memory()
              for x in pool[:8]]
    out_host = torch.empty((cfg.T, cfg.d), dtype=torch.bfloat16).pin_memory()
    x_stage = torch.empty((cfg.T, cfg.d), dtype=torch.bfloat16, device=dev)
    e_steps = min(args.steps, 200)
    torch.cuda.synchronize()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        e0.record(stream)
        for i in range(e_steps):
            x_stage.copy_(x_host[i % len(x_host)], non_blocking=True)
            B.layer_forward(descs[i % R], x_stage, ws, out=out, stream=stream)
            out_host.copy_(out, non_blocking=True)
        e1.record(stream)
    torch.cuda.synchronize()
    e2e_ms = e0.elapsed_time(e1) / e_steps
    status = B.device_status(descs[0], ws)

    ms, e2e_ms = max_over_ranks([ms, e2e_ms], device=dev)

    peak, peak_kind = measured_peaks()
    ms_per_step = ms / args.steps
    res = {
        "metric": f"MoE-layer tokens/s ({cfg.name}, T={cfg.T})",
        "value": world * cfg.T * args.steps / (ms * 1e-3),
        "unit": "tokens/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": ms_per_step,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": f"{cfg.fmt} weights, bf16 activations, fp32 accumulate",
        "data": "synthetic (seeded; shapes of the pages' model, random weights)",
        "config": {"workload": cfg.name, "T": cfg.T, "d": cfg.d, "E": cfg.E, "k": cfg.k,
                   "f": cfg.f, "n_shared": cfg.n_shared, "weights": f"{cfg.fmt} g{cfg.group}",
                   "parallelism": f"replicas x{world}",
                   "l2": f"inputs larger than L2: {R} weight copies x {POOL} hidden batches cycled",
                   "cuda_graph": not args.no_graph},
        "roofline": {"bound": "hbm",
                     "kernel": ("decode_fused_kernel (whole layer, one launch)" if fused
                                else "grouped gate/up + SwiGLU"),
                     "achieved": achieved, "peak": peak, "unit": "GB/s",
                     "frac": achieved / peak, "peak_kind": peak_kind,
                     "traffic": profiled_traffic(cfg.name, "decode_fused" if fused else
                                                 ("tc_grouped" if cfg.T >= 16 else "gemv_tma")),
                     "avg_launch_ms": gu_avg_ms,
                     "layer_frac": float(np.mean(layer_bytes)) / (ms_per_step * 1e-3) / 1e9 / peak},
        "e2e": {"value": world * cfg.T / (e2e_ms * 1e-3), "unit": "tokens/s",
                "h2d_bytes_per_step": cfg.T * cfg.d * 2, "d2h_bytes_per_step": cfg.T * cfg.d * 2},
        "gpu_launches": B.launches_per_call(descs[0]) * args.steps,
        "clocks": clk.summary(),
        "device_status": status,
        **({"stages_ms_eager": stage_ms} if stage_ms else {}),
    }
    return res, L, cfg


def main():
    args = parse()
    rank = int(os.environ.get("RANK", 0))
    world = int(os.environ.get("WORLD_SIZE", 1))
    local_rank = int(os.environ.get("LOCAL_RANK", 0))
    cfg = synth.CONFIGS[args.workload]

    if args.impl == "reference":
        if rank != 0:
            return 0
        L = synth.make_layer(cfg, routed=synth.make_bank(cfg, "routed", experts=[]),
                             shared=synth.make_bank(cfg, "shared"))
        # only the experts the sampled tokens touch are drawn (others are never read)
        from oracle import moe_oracle as O
        need = np.unique(O.select_topk(O.router_logits(L.x[:64], L.router_w, L.router_bias),
                                       cfg.k)[0])
        L.routed = synth.make_bank(cfg, "routed", experts=need)
        cb = cpu_baseline(cfg, L, args.cpu_seconds)
        rate = cb["value"]
        line = {"impl": "reference", "metric": f"MoE-layer tokens/s ({cfg.name}, T={cfg.T})",
                "value": rate, "unit": "tokens/s", "n_gpus": 0, "steps": args.steps,
                "warmup": args.warmup, "higher_is_better": True, "scaling": "weak",
                "vs_baseline": None, "dtype": "f64", "data": "synthetic",
                "config": {"workload": cfg.name, "T": cfg.T},
                "cpu_baseline": cb,
                "e2e": {"value": rate, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                        "d2h_bytes_per_step": 0}}
        print(json.dumps(line))
        return 0

    if world > 1:
        import torch
        import torch.distributed as dist
        from datetime import timedelta
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=timedelta(seconds=300),
                                device_id=torch.device("cuda", local_rank))
    res, L, cfg = run_ours(args, rank, world, local_rank)
    if rank == 0 and world == 1:
        res["cpu_baseline"] = cpu_baseline(cfg, L, args.cpu_seconds)
    if rank == 0:
        print(json.dumps(res))
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
