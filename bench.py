#!/usr/bin/env python
"""Benchmark of the BinaryAttention forward hot path on B200.

One step = the whole hot path over one batch of synthetic input already in
HBM: pack Q, pack K (sign bits + per-token scale), quantise V (channel-wise
int8), fused attention (binary QK, bias, online softmax, u8 P, integer PV).
Prints ONE JSON line on rank 0.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME]
    python bench.py --impl reference ...     # the CPU oracle, timed on host cores

Metric: effective TOPS = 4*B*H*N^2*d per step / step time (higher is better);
ms_per_step and the fused kernel's roofline fraction are reported alongside.
Multi-GPU (torchrun): the job is a global batch of N x B batch elements split
into contiguous slices of B, one per rank (bit_qk_attention_ba_b200.sharding;
the (b, h) units are independent, no collective on the data path); rank r's
slice is drawn with seed + its first global batch index.  value = all ranks'
operations / max-over-ranks time ("scaling": "weak": the per-GPU work is fixed).
"""
from __future__ import annotations

import argparse
import dataclasses
import glob
import hashlib
import json
import os
import re
import statistics
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from bit_qk_attention_ba_b200.sharding import shard_range  # noqa: E402
from bit_qk_attention_ba_b200.workloads import (BIAS_KIND, DECODE_WORKLOADS, WORKLOADS,  # noqa: E402
                                                make_decode_inputs, make_inputs)

METRIC = "binary attention effective TOPS (4*B*H*N^2*d per step)"
def dtype_of(w, variant):
    """The arithmetic the attention path runs for workload w: the QK kind the
    library picks (kind::f8f6f4 with +-1 e4m3 operands in the 128-key kernel,
    kind::i8 in the paired one, unless a variant is forced)."""
    pv = "u8 x s8 PV on tcgen05 kind::i8 (s32), fp32 scores and softmax"
    if variant == 1:
        return "b1 QK by XOR/popcount on CUDA cores, u8 x s8 PV by dp4a (s32), fp32 softmax"
    if variant == 2:
        return "b1 QK on warp mma.sync .b1 xor.popc, u8 x s8 PV on mma.sync (s32), fp32 softmax"
    f8 = variant == 4 or (variant == 0 and attn_kernel(w, variant)[0] == "attn_tc_kernel")
    if f8:
        return "+-1 e4m3 QK on tcgen05 kind::f8f6f4 (fp32 accumulate, exact), " + pv
    return "+-1 int8 QK on tcgen05 kind::i8 (s32 accumulate), " + pv
# The gate workloads reported beside the headline one, each timed on its own.
SIDE_WORKLOADS = ("deit_b384", "deit_s", "dit_xl2", "deit_t")
L2_BYTES = 126 * 2 ** 20
CSRC = os.path.join(ROOT, "bit_qk_attention_ba_b200", "csrc")


def attn_kernel(w, variant):
    """The fused attention kernel a workload runs, and its source file: the
    CUDA-core kernel for the popcount variant, the warp-MMA kernel for the .b1
    variant; otherwise, for a dense bias shared over a batch of two or more,
    the paired tensor-core kernel, else the 128-key one."""
    if variant == 1:
        return "attn_simt_kernel", os.path.join(CSRC, "ba_attn_simt.cu")
    if variant == 2:
        return "attn_b1_kernel", os.path.join(CSRC, "ba_attn_b1.cu")
    if w.bias == "dense" and w.B >= 2:
        return "attn_pair_kernel", os.path.join(CSRC, "ba_attn_tc_pair.cu")
    return "attn_tc_kernel", os.path.join(CSRC, "ba_attn_tc.cu")


# ------------------------------------------------------------------ helpers

def peaks():
    """Measured B200 peaks (generated file), else the recipe's fallback."""
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return dict(hbm_gbs=float(d["hbm_gbs"]), bf16=float(d["bf16_tflops"]),
                    bf16_sus=float(d.get("bf16_tflops_sustained", d["bf16_tflops"])), src="measured")
    return dict(hbm_gbs=6650.0, bf16=1590.0, bf16_sus=1400.0, src="fallback")


def attn_bytes(w, out_bytes):
    """Algorithmic bytes of one attention call: packed Q and K bits, both
    scales, int8 V, V scales, the bias (read once, shared over the batch), and
    the output."""
    BH, N, d = w.B * w.H, w.N, w.d
    W = (d + 31) // 32
    b = 2 * BH * N * W * 4 + 2 * BH * N * 4 + BH * N * d + BH * d * 4 + BH * N * d * out_bytes
    if w.bias == "dense":
        b += w.H * N * N * 4
    elif w.bias in ("relpos2d", "relpos2d_cls"):
        gh, gw = w.grid
        b += w.H * ((2 * gh - 1) * (2 * gw - 1) + (3 if w.bias == "relpos2d_cls" else 0)) * 4
    return b


def roofline(w, attn_t, out_bytes, variant):
    """Roofline of the fused attention call timed in isolation (CUDA events
    around ba_attention_fwd): tensor-bound when ops / int8 peak exceeds
    algorithmic bytes / HBM peak.  The int8 peak is 2 x the measured bf16 GEMM
    rate (the nominal B200 int8 : bf16 ratio), the burst figure since the call
    is timed alone; the fraction of the sustained figure is given beside it."""
    pk = peaks()
    int8_burst, int8_sus = 2.0 * pk["bf16"], 2.0 * pk["bf16_sus"]
    abytes = attn_bytes(w, out_bytes)
    t_tensor, t_hbm = w.ops / (int8_burst * 1e12), abytes / (pk["hbm_gbs"] * 1e9)
    if t_tensor >= t_hbm:
        ach = w.ops / attn_t / 1e12
        roof = {"bound": "tensor", "achieved": ach, "peak": int8_burst, "unit": "TOPS",
                "frac": ach / int8_burst, "frac_sustained": ach / int8_sus,
                "peak_source": "int8 = 2 x measured burst bf16 GEMM (%s); frac_sustained against 2 x the "
                               "sustained bf16 figure" % pk["src"]}
    else:
        ach = abytes / attn_t / 1e9
        roof = {"bound": "hbm", "achieved": ach, "peak": pk["hbm_gbs"], "unit": "GB/s",
                "frac": ach / pk["hbm_gbs"], "peak_source": "measured HBM copy (%s)" % pk["src"]}
    kname, ksrc = attn_kernel(w, variant)
    roof["kernel"] = kname
    roof["traffic"] = recorded_traffic(kname, ksrc, w.name)
    roof["kernel_us"] = attn_t * 1e6
    roof["algorithmic_bytes"] = abytes
    roof["ops"] = w.ops
    return roof


def _code_only(text):
    """Source text without comments and whitespace: what the compiler sees."""
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    text = re.sub(r"//[^\n]*", "", text)
    return re.sub(r"\s+", "", text)


def _included(path, seen):
    """path and every local header it includes ("..."), transitively, in order."""
    path = os.path.normpath(path)
    if path in seen or not os.path.exists(path):
        return
    seen.append(path)
    for inc in re.findall(r'^\s*#\s*include\s+"([^"]+)"', open(path).read(), flags=re.M):
        _included(os.path.join(os.path.dirname(path), inc), seen)


def source_hash(path):
    """Hash of a kernel source and the local headers it includes (transitively),
    comments and whitespace removed: an edit of comments alone keeps a
    recorded ncu summary valid, an edit of code the kernel compiles does not."""
    parts = []
    _included(path, parts)
    code = "".join(_code_only(open(p).read()) for p in parts)
    return hashlib.sha256(code.encode()).hexdigest()[:16]


def recorded_traffic(kernel, src, workload):
    """DRAM bytes per launch from a committed ncu summary, if it was taken on
    the current kernel source (else None)."""
    p = os.path.join(ROOT, "profiles", "%s_%s.txt" % (kernel, workload))
    if not os.path.exists(p):
        return None
    vals = {}
    for line in open(p):
        if ":" in line:
            k, v = line.split(":", 1)
            vals[k.strip()] = v.strip()
    if vals.get("source_sha256_16") != source_hash(src):
        return None
    try:
        return float(vals["dram_bytes_per_launch"])
    except (KeyError, ValueError):
        return None


class ClockSampler:
    """nvidia-smi clocks and throttle reasons sampled during the timed region."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.gpu = gpu_index
        self.proc = None
        self.lines = []

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(["nvidia-smi", "-i", str(self.gpu), "--query-gpu=" + self.FIELDS,
                                          "--format=csv,noheader,nounits", "-lms", "100"],
                                         stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.t = threading.Thread(target=self._read, daemon=True)
            self.t.start()
        except (OSError, FileNotFoundError):
            self.proc = None
        time.sleep(0.25)
        return self

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def __exit__(self, *a):
        if self.proc is not None:
            time.sleep(0.15)
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self):
        sm, smax, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in self.lines:
            f = [x.strip() for x in line.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                smax = float(f[2])
            except ValueError:
                continue
            for n, v in zip(names, f[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": smax, "reasons": [], "samples": 0}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": smax, "reasons": sorted(reasons),
                "samples": len(sm)}


def smi_id(dev):
    """nvidia-smi -i selector for a torch device (its UUID when available)."""
    import torch
    try:
        u = str(torch.cuda.get_device_properties(dev).uuid)
        if u:
            return u if u.startswith("GPU-") else "GPU-" + u
    except Exception:
        pass
    vis = os.environ.get("CUDA_VISIBLE_DEVICES", "")
    ids = [x for x in vis.split(",") if x.strip()]
    return ids[dev.index].strip() if dev.index < len(ids) else str(dev.index)


def dist_env():
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    return int(os.environ.get("RANK", "0")), int(os.environ.get("LOCAL_RANK", "0")), ws


def aggregate_tops(world, ops_per_rank, ms_per_step):
    """Whole-job effective TOPS: every rank runs one batch slice of the same
    size (weak scaling), timed by the slowest rank."""
    return world * ops_per_rank / (ms_per_step * 1e-3) / 1e12


def input_bytes(w):
    """Bytes of one step's inputs on the device (q, k, v and the bias)."""
    es = 2 if w.dtype == "bf16" else 4
    b = 3 * w.B * w.H * w.N * w.d * es
    if w.bias == "dense":
        b += w.H * w.N * w.ld * 4
    elif w.bias in ("relpos2d", "relpos2d_cls"):
        gh, gw = w.grid
        b += w.H * ((2 * gh - 1) * (2 * gw - 1) + (3 if w.bias == "relpos2d_cls" else 0)) * 4
    return b


def bench_config(w, world, variant):
    """The `config` object of the JSON line, the same for both arms."""
    return {"workload": w.name, "B": w.B, "H": w.H, "N": w.N, "d": w.d, "input_dtype": w.dtype,
            "bias": w.bias, "parallelism": "dp%d" % world, "global_batch": world * w.B,
            "split": "contiguous batch slices of %d per rank, no data-path collective" % w.B,
            "l2": "flushed between steps" if input_bytes(w) < 2 * L2_BYTES else "inputs larger than L2",
            "qk_variant": variant}


def max_over_ranks(x, world, device=None):
    """Max of a float over ranks (identity for one process)."""
    if world <= 1:
        return x
    import torch
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


# ------------------------------------------------------------------ our arm

def time_side_workload(w, variant, dev, steps=50, warmup=10):
    """A gate workload timed on its own: the pre-pass + attention step, the
    attention call alone, and the step replayed from one CUDA graph (CUDA
    events, median over the timed steps, the L2 flushed between steps when
    the inputs fit in it)."""
    import torch
    import bit_qk_attention_ba_b200 as ba
    inp = make_inputs(w)
    tdt = torch.bfloat16 if w.dtype == "bf16" else torch.float32
    q, k, v = (torch.from_numpy(inp[n]).to(tdt).to(dev) for n in ("q", "k", "v"))
    bias = None if inp["bias"] is None else torch.from_numpy(inp["bias"]).to(dev)
    kind, ld, grid = BIAS_KIND[w.bias], inp["ld"], w.grid
    pre = ba.prepass_qkv(q, k, v)
    out = torch.empty((w.B, w.H, w.N, w.d), dtype=tdt, device=dev)
    ws = ba.attention_workspace(w.B, w.H, w.N, w.d, kind, grid, device=dev)
    stream = torch.cuda.current_stream(dev)
    in_bytes = sum(t.numel() * t.element_size() for t in (q, k, v)) + (bias.numel() * 4 if bias is not None else 0)
    flush = torch.empty(2 * L2_BYTES // 4, dtype=torch.float32, device=dev) if in_bytes < 2 * L2_BYTES else None
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(steps)]

    def step(e=None):
        if e is not None:
            e[0].record(stream)
        ba.prepass_qkv(q, k, v, pre)
        if e is not None:
            e[1].record(stream)
        ba.attention_fwd(*pre, w.d, bias=bias, bias_kind=kind, ld=ld, grid=grid, out=out, variant=variant,
                         workspace=ws)
        if e is not None:
            e[2].record(stream)

    for _ in range(warmup):
        step()
    torch.cuda.synchronize(dev)
    for i in range(steps):
        if flush is not None:
            flush.zero_()
        step(ev[i])
    torch.cuda.synchronize(dev)
    step_ms = statistics.median(e[0].elapsed_time(e[2]) for e in ev)
    attn_ms = statistics.median(e[1].elapsed_time(e[2]) for e in ev)
    # The same step replayed from one CUDA graph (ba_fwd_graph_*): its kernels
    # run back to back, without a host launch per kernel.  A failure to build
    # the graph is reported in the line instead of ending the run.
    graph, graph_ms, graph_kernels, graph_error = None, None, None, None
    try:
        graph = ba.ForwardGraph(q, k, v, bias=bias, bias_kind=kind, ld=ld, grid=grid, out_dtype=tdt,
                                variant=variant)
    except Exception as e:          # noqa: BLE001 -- recorded in the JSON line
        graph_error = str(e)
    if graph is not None:
        gev = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(steps)]
        for _ in range(warmup):
            graph.launch()
        torch.cuda.synchronize(dev)
        for i in range(steps):
            if flush is not None:
                flush.zero_()
            gev[i][0].record(stream)
            graph.launch()
            gev[i][1].record(stream)
        torch.cuda.synchronize(dev)
        graph_ms = statistics.median(a.elapsed_time(b) for a, b in gev)
        graph_kernels = graph.kernels
        graph.close()
    roof = roofline(w, attn_ms * 1e-3, 2 if tdt == torch.bfloat16 else 4, variant)
    status = ba.check_device_status(dev)
    del q, k, v, bias, pre, out, ws, flush, graph
    torch.cuda.empty_cache()
    return {"B": w.B, "H": w.H, "N": w.N, "d": w.d, "bias": w.bias, "attention_us": attn_ms * 1e3,
            "step_us": step_ms * 1e3, "step_tops": w.ops / (step_ms * 1e-3) / 1e12,
            "graph_step_us": None if graph_ms is None else graph_ms * 1e3, "graph_kernels": graph_kernels,
            **({"graph_error": graph_error} if graph_error else {}),
            "attention_tops": w.ops / (attn_ms * 1e-3) / 1e12, "steps": steps, "warmup": warmup,
            "l2": "flushed between steps" if in_bytes < 2 * L2_BYTES else "inputs larger than L2",
            "roofline": roof, "device_status": status}


def time_backward(w, dev, steps=10, warmup=3):
    """The training-side backward (ba_attention_bwd: straight-through
    estimators, CUDA cores) on workload w: CUDA events around the call,
    median over the timed steps.  Ops counted: the four N x N x d
    contractions of an attention backward (dO V^T, P^T dO, dS K, dS^T Q),
    8 B H N^2 d; roofline: fp32 FMA on the CUDA cores (148 SMs x 128 lanes x
    2 flop x the SM clock)."""
    import torch
    import bit_qk_attention_ba_b200 as ba
    inp = make_inputs(w)
    tdt = torch.bfloat16 if w.dtype == "bf16" else torch.float32
    q, k, v = (torch.from_numpy(inp[n]).to(tdt).to(dev) for n in ("q", "k", "v"))
    bias = None if inp["bias"] is None else torch.from_numpy(inp["bias"]).to(dev)
    kind, ld, grid = BIAS_KIND[w.bias], inp["ld"], w.grid
    pre = ba.prepass_qkv(q, k, v)
    out = ba.attention_fwd(*pre, w.d, bias=bias, bias_kind=kind, ld=ld, grid=grid, out_dtype=torch.float32)
    dout = torch.randn(out.shape, generator=torch.Generator(device="cpu").manual_seed(0)).to(dev)
    grads = None
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
    stream = torch.cuda.current_stream(dev)
    for i in range(warmup + steps):
        e = ev[i - warmup] if i >= warmup else None
        if e:
            e[0].record(stream)
        grads = ba.attention_bwd(q, k, *pre, out, dout, bias=bias, bias_kind=kind, ld=ld, grid=grid, grads=grads)
        if e:
            e[1].record(stream)
    torch.cuda.synchronize(dev)
    ms = statistics.median(a.elapsed_time(b) for a, b in ev)
    ops = 8.0 * w.B * w.H * w.N * w.N * w.d
    peak = 148 * 128 * 2 * 1965e6 / 1e12
    status = ba.check_device_status(dev)
    return {"workload": w.name, "B": w.B, "H": w.H, "N": w.N, "d": w.d, "bias": w.bias, "ms": ms,
            "tops": ops / (ms * 1e-3) / 1e12, "launches": 4,
            "roofline": {"bound": "alu", "achieved": ops / (ms * 1e-3) / 1e12, "peak": peak, "unit": "TFLOP/s",
                         "frac": ops / (ms * 1e-3) / 1e12 / peak,
                         "peak_source": "fp32 FMA on CUDA cores: 148 SMs x 128 lanes x 2 flop x 1965 MHz",
                         "ops": ops},
            "device_status": status}


def run_ours(args, w, rank, local_rank, world):
    import torch
    import bit_qk_attention_ba_b200 as ba
    from bit_qk_attention_ba_b200 import _native as NAT

    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    if world > 1:
        import torch.distributed as dist
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=120), device_id=dev)

    # this rank's slice of the global batch (world x B elements)
    lo, hi = shard_range(world * w.B, world, rank)
    assert hi - lo == w.B
    inp = make_inputs(w, seed=w.seed + lo)
    tdt = torch.bfloat16 if w.dtype == "bf16" else torch.float32
    host = {n: torch.from_numpy(inp[n]).to(tdt).pin_memory() for n in ("q", "k", "v")}
    q, k, v = (host[n].to(dev) for n in ("q", "k", "v"))
    bias = None if inp["bias"] is None else torch.from_numpy(inp["bias"]).to(dev)
    host_bias = None if inp["bias"] is None else torch.from_numpy(inp["bias"]).pin_memory()
    kind, ld, grid = BIAS_KIND[w.bias], inp["ld"], w.grid
    out_dtype = tdt
    out_bytes = 2 if out_dtype == torch.bfloat16 else 4
    d = w.d
    pre = ba.prepass_qkv(q, k, v)
    bq, muq, bk, muk, vq, sv = pre
    out = torch.empty((w.B, w.H, w.N, d), dtype=out_dtype, device=dev)
    ws = ba.attention_workspace(w.B, w.H, w.N, d, kind, grid, device=dev)
    stream = torch.cuda.current_stream(dev)
    in_bytes = sum(t.numel() * t.element_size() for t in (q, k, v)) + (bias.numel() * 4 if bias is not None else 0)
    assert in_bytes == input_bytes(w)
    flush = None
    if in_bytes < 2 * L2_BYTES:
        flush = torch.empty(2 * L2_BYTES // 4, dtype=torch.float32, device=dev)

    a0 = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    a1 = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]

    def step(i=None):
        ba.prepass_qkv(q, k, v, pre)
        if i is not None:
            a0[i].record(stream)
        ba.attention_fwd(bq, muq, bk, muk, vq, sv, d, bias=bias, bias_kind=kind, ld=ld, grid=grid,
                         out=out, variant=args.variant, workspace=ws)
        if i is not None:
            a1[i].record(stream)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize(dev)
    if ba.check_device_status(dev) != 0:
        raise RuntimeError("device status set during warm-up")

    starts = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize(dev)
    with ClockSampler(smi_id(dev)) as clk:
        for i in range(args.steps):
            if flush is not None:
                flush.zero_()
            starts[i].record(stream)
            step(i)
            ends[i].record(stream)
        torch.cuda.synchronize(dev)
    if world > 1:
        torch.distributed.barrier()
    attn_ms = [x.elapsed_time(y) for x, y in zip(a0, a1)]
    total_ms = sum(s.elapsed_time(e) for s, e in zip(starts, ends))
    total_ms = max_over_ranks(total_ms, world, dev)
    status = ba.check_device_status(dev)
    clocks = clk.summary()

    # end to end through the public API: pinned host inputs -> device -> host output
    # A stream of batches: every step uploads its own inputs from pinned host
    # memory, runs ba.forward, and reads its output back to pinned host memory.
    # Two buffer sets and three streams (upload, compute, read-back) let the
    # upload of step i + 1 and the read-back of step i - 1 overlap step i's
    # kernels, as a serving loop would.
    NBUF = 2
    e_steps = max(3, min(args.steps, 20))
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    bufs = [dict(q=torch.empty_like(q), k=torch.empty_like(k), v=torch.empty_like(v),
                 b=torch.empty_like(bias) if bias is not None else None) for _ in range(NBUF)]
    host_outs = [torch.empty((w.B, w.H, w.N, d), dtype=out_dtype).pin_memory() for _ in range(NBUF)]
    s_up, s_back = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    ev_up = [torch.cuda.Event() for _ in range(NBUF)]
    ev_done = [torch.cuda.Event() for _ in range(NBUF)]
    ev_read = [torch.cuda.Event() for _ in range(NBUF)]

    def e2e_run(n):
        s_up.wait_stream(stream)
        s_back.wait_stream(stream)
        for i in range(n):
            j = i % NBUF
            bf = bufs[j]
            with torch.cuda.stream(s_up):
                if i >= NBUF:
                    s_up.wait_event(ev_done[j])        # step i - NBUF has consumed this buffer set
                for name in ("q", "k", "v"):
                    bf[name].copy_(host[name], non_blocking=True)
                if bf["b"] is not None:
                    bf["b"].copy_(host_bias, non_blocking=True)
                ev_up[j].record(s_up)
            stream.wait_event(ev_up[j])
            if i >= NBUF:
                stream.wait_event(ev_read[j])         # step i - NBUF's output is on the host
            o = ba.forward(bf["q"], bf["k"], bf["v"], bias=bf["b"], bias_kind=kind, ld=ld, grid=grid,
                           out_dtype=out_dtype, variant=args.variant, workspace=ws)
            ev_done[j].record(stream)
            with torch.cuda.stream(s_back):
                s_back.wait_event(ev_done[j])
                host_outs[j].copy_(o, non_blocking=True)
                ev_read[j].record(s_back)
            o.record_stream(s_back)
        stream.wait_stream(s_up)
        stream.wait_stream(s_back)

    e2e_run(NBUF)
    torch.cuda.synchronize(dev)
    e0.record(stream)
    e2e_run(e_steps)
    e1.record(stream)
    torch.cuda.synchronize(dev)
    e2e_ms = max_over_ranks(e0.elapsed_time(e1) / e_steps, world, dev)
    h2d = in_bytes
    d2h = host_outs[0].numel() * host_outs[0].element_size()

    ms = total_ms / args.steps
    ops = w.ops
    # the pre-pass (one fused launch, or pack Q, pack K and the V quantiser),
    # then either a warp-level attention kernel or the key staging (+ rel-pos
    # table staging) and the tensor-core one
    tc_path = ws is not None and args.variant not in (NAT.BA_QK_POPC, NAT.BA_QK_MMA_B1)
    fast_rp = kind == NAT.BA_BIAS_RELPOS2D and grid and grid[1] % 128 == 0
    launches_per_step = ba.prepass_launches(w.N, d, tdt) + (1 + (1 if fast_rp else 0) if tc_path else 0) + 1
    value = aggregate_tops(world, ops, ms)
    attn_t = statistics.median(attn_ms) * 1e-3
    # CUDA events bracket the whole ba_attention_fwd call: the key staging
    # pre-passes plus the fused kernel (the staging is the small remainder).
    roof = roofline(w, attn_t, out_bytes, args.variant)

    line = {
        "metric": METRIC, "value": value, "unit": "TOPS", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": dtype_of(w, args.variant), "data": "synthetic",
        "config": bench_config(w, world, args.variant),
        "roofline": roof,
        "e2e": {"value": world * ops / (e2e_ms * 1e-3) / 1e12, "unit": "TOPS", "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms,
                "pipeline": "2 buffer sets; upload, compute and read-back on three streams"},
        "gpu_launches": launches_per_step * args.steps,
        "clocks": clocks,
        "device_status": status,
    }
    if not args.no_backward:
        bw = w if args.backward_workload == "main" else WORKLOADS[args.backward_workload]
        line["backward"] = time_backward(bw, dev)
    if not args.no_side_workloads:
        # every rank times the same side workloads, so the ranks stay in step
        side = {}
        for name in SIDE_WORKLOADS:
            if name != w.name:
                side[name] = time_side_workload(WORKLOADS[name], args.variant, dev)
        line["workloads"] = side
    if rank == 0 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(w, inp, budget_s=args.cpu_seconds)
    if world > 1:
        torch.distributed.destroy_process_group()
    return line


# ------------------------------------------------------------------ decode shape

def decode_bytes(w, out_bytes):
    """Algorithmic bytes of one decode call: the cache (key bits, key scales,
    int8 value codes, value scales), the new queries' bits and scales, and the
    output."""
    BH, W = w.B * w.H, (w.d + 31) // 32
    return BH * w.Nk * (W * 4 + 4 + w.d) + BH * w.d * 4 + BH * w.Nq * (W * 4 + 4) + BH * w.Nq * w.d * out_bytes


def decode_config(w, world):
    return {"workload": w.name, "B": w.B, "H": w.H, "Nq": w.Nq, "Nk": w.Nk, "d": w.d,
            "input_dtype": w.dtype, "bias": "none", "parallelism": "replicas%d" % world,
            "l2": "cache larger than L2", "ops": "4*B*H*Nq*Nk*d per step"}


def run_decode(args, w, rank, local_rank, world):
    """One step = pack the new queries + the decode forward over the resident
    cache (packed key bits, key scales, int8 values: built once, as a KV cache
    is)."""
    import torch
    import bit_qk_attention_ba_b200 as ba

    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    if world > 1:
        import torch.distributed as dist
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=120), device_id=dev)
    inp = make_decode_inputs(w)
    tdt = torch.bfloat16 if w.dtype == "bf16" else torch.float32
    host_q = torch.from_numpy(inp["q"]).to(tdt).pin_memory()
    q = host_q.to(dev)
    bk, muk = ba.pack_qk(torch.from_numpy(inp["k"]).to(tdt).to(dev))
    vq, sv = ba.quant_v(torch.from_numpy(inp["v"]).to(tdt).to(dev))
    bq, muq = ba.pack_qk(q)
    out = torch.empty((w.B, w.H, w.Nq, w.d), dtype=tdt, device=dev)
    ws = ba.decode_workspace(w.B, w.H, w.Nq, w.Nk, w.d, device=dev)
    stream = torch.cuda.current_stream(dev)
    a0 = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    a1 = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]

    def step(i=None):
        ba.pack_qk(q, bq, muq)
        if i is not None:
            a0[i].record(stream)
        ba.attention_decode(bq, muq, bk, muk, vq, sv, w.d, out=out, workspace=ws)
        if i is not None:
            a1[i].record(stream)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize(dev)
    starts = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize(dev)
    with ClockSampler(smi_id(dev)) as clk:
        for i in range(args.steps):
            starts[i].record(stream)
            step(i)
            ends[i].record(stream)
        torch.cuda.synchronize(dev)
    if world > 1:
        torch.distributed.barrier()
    total_ms = max_over_ranks(sum(s.elapsed_time(e) for s, e in zip(starts, ends)), world, dev)
    attn_t = statistics.median(x.elapsed_time(y) for x, y in zip(a0, a1)) * 1e-3
    status = ba.check_device_status(dev)
    clocks = clk.summary()

    # end to end: the new queries come from pinned host memory, the output goes back
    host_out = torch.empty((w.B, w.H, w.Nq, w.d), dtype=tdt).pin_memory()
    e_steps = max(3, min(args.steps, 50))
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)

    def e2e_step():
        qd = host_q.to(dev, non_blocking=True)
        bqd, muqd = ba.pack_qk(qd)
        o = ba.attention_decode(bqd, muqd, bk, muk, vq, sv, w.d, out_dtype=tdt, workspace=ws)
        host_out.copy_(o, non_blocking=True)

    e2e_step()
    torch.cuda.synchronize(dev)
    e0.record(stream)
    for _ in range(e_steps):
        e2e_step()
    e1.record(stream)
    torch.cuda.synchronize(dev)
    e2e_ms = max_over_ranks(e0.elapsed_time(e1) / e_steps, world, dev)

    ms = total_ms / args.steps
    out_bytes = 2 if tdt == torch.bfloat16 else 4
    nbytes = decode_bytes(w, out_bytes)
    pk = peaks()
    roof = {"bound": "hbm", "achieved": nbytes / attn_t / 1e9, "peak": pk["hbm_gbs"], "unit": "GB/s",
            "kernel": "decode_pv_kernel",
            "traffic": recorded_traffic("decode_pv_kernel", os.path.join(CSRC, "ba_decode.cu"), w.name),
            "kernel_us": attn_t * 1e6,
            "peak_source": "measured HBM copy (%s)" % pk["src"], "algorithmic_bytes": nbytes,
            "note": "events around ba_attention_decode: two launches (split maxima; codes, PV and the splits added by the last CTA of a head)"}
    roof["frac"] = roof["achieved"] / roof["peak"]
    line = {
        "metric": METRIC, "value": aggregate_tops(world, w.ops, ms), "unit": "TOPS", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "b1 QK by XOR/popcount on CUDA cores, u8 x s8 PV by dp4a (s32), fp32 softmax",
        "data": "synthetic",
        "config": decode_config(w, world),
        "roofline": roof,
        "e2e": {"value": world * w.ops / (e2e_ms * 1e-3) / 1e12, "unit": "TOPS",
                "h2d_bytes_per_step": host_q.numel() * host_q.element_size(),
                "d2h_bytes_per_step": host_out.numel() * host_out.element_size(), "ms_per_step": e2e_ms,
                "cache": "resident on the device"},
        "gpu_launches": 3 * args.steps,            # pack the new queries, split maxima, codes + PV
        "clocks": clocks,
        "device_status": status,
    }
    if rank == 0 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline_decode(w, inp, budget_s=args.cpu_seconds)
    if world > 1:
        torch.distributed.destroy_process_group()
    return line


def cpu_baseline_decode(w, inp, budget_s=15.0):
    """The oracle's decode forward on the first heads (packing of the new
    queries included, the cache packed beforehand), scaled to all heads."""
    import oracle as O
    O.build()
    BH = w.B * w.H
    q = inp["q"].reshape(BH, w.Nq, w.d)
    k = inp["k"].reshape(BH, w.Nk, w.d)
    v = inp["v"].reshape(BH, w.Nk, w.d)
    heads, t, n = 1, 0.0, 0
    while True:
        bk, muk = O.pack(k[n:n + heads])
        vq, sv = O.quant_v(v[n:n + heads])
        t0 = time.perf_counter()
        bq, muq = O.pack(q[n:n + heads])
        O.attention_decode(bq, muq, bk, muk, vq, sv, w.H, w.d)
        t += time.perf_counter() - t0
        n += heads
        if t >= budget_s or n + heads > BH:
            break
        heads = min(heads * 2, BH - n)
    t_full = t * BH / n
    return {"value": w.ops / t_full / 1e12, "unit": "TOPS", "cores": 1, "kind": "oracle",
            "sample": "%d of %d heads (every cached key), %.1f s, scaled to all heads" % (n, BH, t),
            "seconds_full_workload_est": t_full}


# ------------------------------------------------------------------ CPU oracle

def cpu_baseline(w, inp, budget_s=15.0, heads=1):
    """Time the oracle as it stands on a bounded sample of this workload:
    pack/quantise the first `heads` heads, then the full forward of a block of
    query rows of those heads (every key), and scale to the whole workload."""
    import oracle as O
    O.build()
    d, N = w.d, w.N
    gh, gw = w.grid
    kind = BIAS_KIND[w.bias]
    q = inp["q"].reshape(-1, N, d)[:heads]
    k = inp["k"].reshape(-1, N, d)[:heads]
    v = inp["v"].reshape(-1, N, d)[:heads]
    t0 = time.perf_counter()
    bq, muq = O.pack(q)
    bk, muk = O.pack(k)
    vq, sv = O.quant_v(v)
    t_pre = time.perf_counter() - t0
    rows = min(N, 16)
    t0 = time.perf_counter()
    _, used = O.attention_fwd_rows(bq, muq, bk, muk, vq, sv, kind, inp["bias"], inp["ld"], gh, gw,
                                   heads, w.H, d, 0, rows)
    t_probe = time.perf_counter() - t0
    target = max(rows, min(N, int(rows * budget_s / max(t_probe, 1e-6))))
    t0 = time.perf_counter()
    _, used = O.attention_fwd_rows(bq, muq, bk, muk, vq, sv, kind, inp["bias"], inp["ld"], gh, gw,
                                   heads, w.H, d, 0, target)
    t_attn = time.perf_counter() - t0
    BH = w.B * w.H
    t_full = t_pre * BH / heads + t_attn * (BH * N) / (heads * target)
    # the DeiT-T workload (1 x 3 x 197 x 64) whole, on one core: the small
    # correctness configuration, timed in full
    wt = WORKLOADS["deit_t"]
    it = make_inputs(wt)
    t0 = time.perf_counter()
    O.forward(it["q"], it["k"], it["v"], BIAS_KIND[wt.bias], it["bias"], it["ld"], nthreads=1)
    t_small = time.perf_counter() - t0
    return {"value": w.ops / t_full / 1e12, "unit": "TOPS", "cores": used, "kind": "oracle",
            "sample": "%d head(s) x %d of %d query rows (all keys) + pre-passes of those heads, "
                      "%.1f s wall, scaled to the full workload" % (heads, target, N, t_pre + t_attn),
            "seconds_full_workload_est": t_full,
            "deit_t_one_core": {"seconds": t_small, "tops": wt.ops / t_small / 1e12, "cores": 1,
                                "sample": "the whole DeiT-T workload, pre-passes and forward"}}


def run_reference(args, w, rank, world):
    if rank != 0:
        return None
    inp = make_inputs(w)
    per_step = max(0.5, min(10.0, 150.0 / max(1, args.steps + args.warmup)))
    vals, walls = [], []
    for i in range(args.warmup + args.steps):
        t0 = time.perf_counter()
        cb = cpu_baseline(w, inp, budget_s=per_step)
        if i >= args.warmup:
            vals.append(cb)
            walls.append(time.perf_counter() - t0)
    value = statistics.median(c["value"] for c in vals)
    cb = dict(vals[-1])
    cb["value"] = value
    return {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "TOPS", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup,
        # each step is a bounded sample of the workload: its own wall time,
        # and the full workload's time at the sample's rate beside it
        "ms_per_step": statistics.median(walls) * 1e3,
        "ms_per_step_full_workload_est": w.ops / (value * 1e12) * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64 (oracle)",
        "data": "synthetic", "config": bench_config(w, world, args.variant),
        "cpu_baseline": cb,
        "e2e": {"value": value, "unit": "TOPS", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


def run_reference_decode(args, w, rank, world):
    if rank != 0:
        return None
    inp = make_decode_inputs(w)
    per_step = max(0.5, min(10.0, 150.0 / max(1, args.steps + args.warmup)))
    vals, walls = [], []
    for i in range(args.warmup + args.steps):
        t0 = time.perf_counter()
        cb = cpu_baseline_decode(w, inp, budget_s=per_step)
        if i >= args.warmup:
            vals.append(cb)
            walls.append(time.perf_counter() - t0)
    value = statistics.median(c["value"] for c in vals)
    cb = dict(vals[-1])
    cb["value"] = value
    return {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "TOPS", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": statistics.median(walls) * 1e3,
        "ms_per_step_full_workload_est": w.ops / (value * 1e12) * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64 (oracle)",
        "data": "synthetic",
        "config": decode_config(w, world),
        "cpu_baseline": cb,
        "e2e": {"value": value, "unit": "TOPS", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


def main(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--workload", default="hires16k", choices=sorted(WORKLOADS) + sorted(DECODE_WORKLOADS))
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--variant", type=int, default=0, help="QK path: 0 auto, 1 popc, 2 mma.sync b1, 3 tcgen05 i8, 4 tcgen05 f8")
    ap.add_argument("--cpu-seconds", type=float, default=15.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-backward", action="store_true", help="skip the training-side backward timing")
    ap.add_argument("--backward-workload", default="deit_b384",
                    help="workload of the backward timing ('main': the headline workload, after --batch/--heads)")
    ap.add_argument("--batch", type=int, default=0,
                    help="override the workload's batch size (smaller cases for profiler captures)")
    ap.add_argument("--heads", type=int, default=0, help="override the workload's head count (profiler captures)")
    ap.add_argument("--no-side-workloads", action="store_true",
                    help="skip the gate workloads timed beside the headline one")
    args = ap.parse_args(argv)
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    rank, local_rank, world = dist_env()
    if args.workload in DECODE_WORKLOADS:
        w = DECODE_WORKLOADS[args.workload]
        if args.batch or args.heads:
            w = dataclasses.replace(w, B=args.batch or w.B, H=args.heads or w.H)
        if args.impl == "reference":
            line = run_reference_decode(args, w, rank, world)
        else:
            line = run_decode(args, w, rank, local_rank, world)
        if rank == 0 and line is not None:
            print(json.dumps(line), flush=True)
        return
    w = WORKLOADS[args.workload]
    if args.batch or args.heads:
        w = w.scaled(B=args.batch or w.B, H=args.heads or w.H)
    if args.impl == "reference":
        line = run_reference(args, w, rank, world)
    else:
        line = run_ours(args, w, rank, local_rank, world)
    if rank == 0 and line is not None:
        print(json.dumps(line), flush=True)


if __name__ == "__main__":
    main()
