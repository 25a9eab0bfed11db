#!/usr/bin/env python
"""Benchmark of the batch-1 quantized decode path on B200.

Workloads (synthetic, seeded; shapes of the ntransformer news summary's
workloads, random weights of the Llama architecture):
  llama70b_q6k_decode (default)  80 layers, hidden 8192, 64 q / 8 kv heads, FFN 28672,
                                 Q6_K weights, fp16 KV cache prefilled to 8192 positions
  llama8b_q8_0_decode            32 layers, hidden 4096, 32 q / 8 kv heads, FFN 14336,
                                 Q8_0 weights, KV cache prefilled to 4096 positions
  llama70b_q4k_stream            70B shape in Q4_K, layers 0-35 resident, 36-79 streamed
                                 from pinned host memory through the two-slot HBM ring
  gemv_q8_0_4096                 Q8_0 GEMV 4096 x 4096 (rotating over weight copies)

One step = one decode step (one token); the metric is tokens per second.
`--impl reference` times the CPU oracle (as it stands) on a bounded sample of
the same workload instead.  Multi-GPU runs are independent replicas (the path
does not shard): each rank decodes its own sequence; value = tokens of all ranks
/ the slowest rank's time.
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

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

PEAKS_FALLBACK = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0}
METRIC = "batch-1 decode tok/s"


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    return PEAKS_FALLBACK["hbm_gbs"], "fallback"


# --------------------------------------------------------------------------- clocks

REASON_BITS = {0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap", 0x8: "hw_slowdown",
               0x10: "sync_boost", 0x20: "sw_thermal_slowdown", 0x40: "hw_thermal_slowdown",
               0x80: "hw_power_brake_slowdown", 0x100: "display_clock_setting"}


class ClockSampler:
    """nvidia-smi sampling of SM clock and throttle reasons during the timed region."""

    def __init__(self, index: int):
        self.index = index
        self.proc = None
        self.lines = []

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.index), "--query-gpu=clocks.sm,clocks.max.sm,clocks_event_reasons.active",
                 "--format=csv,noheader,nounits", "-lms", "100"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL,
                text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
        except OSError:
            self.proc = None
        return self

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def __exit__(self, *a):
        if self.proc:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self):
        sm, mx, reasons = [], None, set()
        for l in self.lines:
            parts = [p.strip() for p in l.split(",")]
            if len(parts) < 3:
                continue
            try:
                sm.append(float(parts[0]))
                mx = float(parts[1])
                bits = int(parts[2], 16)
            except ValueError:
                continue
            for b, name in REASON_BITS.items():
                if bits & b and name != "gpu_idle":
                    reasons.add(name)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unavailable"]}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx, "reasons": sorted(reasons), "samples": len(sm)}


# --------------------------------------------------------------------------- distributed

def dist_setup(n_gpus):
    rank, world = int(os.environ.get("RANK", "0")), int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    return rank, world, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(v, world):
    """The largest of the ranks' values (step times: the job is as slow as its slowest
    replica); NCCL reduces a device tensor, gloo a host one."""
    if world == 1:
        return v
    import torch
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([v], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


# --------------------------------------------------------------------------- workloads

def spec_for(name, layout="tiled"):
    import synth
    tiled = layout == "tiled"
    if name == "llama70b_q6k_decode":
        return synth.ModelSpec(**synth.LLAMA_70B_Q6_K, tiled=tiled)
    if name == "llama8b_q8_0_decode":
        return synth.ModelSpec(**synth.LLAMA_8B_Q8_0, tiled=tiled)
    if name == "llama70b_q4k_stream":
        return synth.ModelSpec(**synth.LLAMA_70B_Q4_K, tiled=tiled)
    raise ValueError(name)


def lib_qtype(spec):
    return spec.qtype | (16 if spec.tiled else 0)


def kv_read_bytes(spec):
    return spec.n_layers * 2 * spec.n_kv_heads * (spec.n_prefill + 1) * spec.head_dim * 2


def step_bytes(spec):
    """Algorithmic bytes of one decode step: packed weights read + KV cache read
    (positions 0..pos) + the embedding row (vectors are negligible)."""
    import synth
    w = spec.n_layers * spec.layer_weight_bytes() + spec.vocab * synth.row_bytes(spec.qtype, spec.hidden)
    return w + kv_read_bytes(spec) + synth.row_bytes(spec.qtype, spec.hidden)


def gemv_shapes(spec):
    """(rows, cols, launches per step) of the decode GEMVs."""
    return [(spec.qkv_rows, spec.hidden, spec.n_layers), (spec.hidden, spec.q_dim, spec.n_layers),
            (spec.ffn, spec.hidden, 2 * spec.n_layers), (spec.hidden, spec.ffn, spec.n_layers),
            (spec.vocab, spec.hidden, 1)]


# DRAM traffic (dram__bytes_read.sum + dram__bytes_write.sum, one ncu capture per
# shape, bytes per launch) of the tiled GEMV, and a hash of the kernel
# sources it was taken with: a changed kernel reports traffic as unknown (null).
GEMV_TRAFFIC_SRC_SHA = "d118f419951f3ecf"
GEMV_TRAFFIC = {"q6_k_t:10240x8192": 68896512, "q6_k_t:8192x8192": 55124992, "q6_k_t:28672x8192": 192979200,
                "q6_k_t:8192x28672": 192954624, "q6_k_t:128256x8192": 862085888, "q8_0_t:6144x4096": 26788864,
                "q8_0_t:4096x4096": 17875968, "q8_0_t:14336x4096": 62440448, "q8_0_t:4096x14336": 62481664,
                "q8_0_t:128256x4096": 558824960}


def gemv_sources_sha():
    import hashlib
    h = hashlib.sha256()
    d = os.path.join(os.path.dirname(os.path.abspath(__file__)), "quantized_weight_gemv_block_b200", "csrc")
    for f in ("qmma.cuh", "qmma.cu", "blocks.cuh", "common.cuh", "gemv.cuh"):
        with open(os.path.join(d, f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def measure_gemv_roofline(ntx, model, spec, stream, iters=3):
    """Time every decode GEMV of one step on its own (the same weights and shapes as
    the step, plain store epilogue, same stream) with CUDA events.  Per shape: bytes
    per launch (packed weights + x + y) and the average launch time, cycling over the
    layers so no launch finds its weights in L2.  The aggregate over a step's launches
    is the dominant kernel's achieved HBM bandwidth.  Only HBM-resident layers count;
    streamed layers are bound by the host link, which is reported on its own."""
    import torch
    import synth
    x = torch.randn(max(spec.hidden, spec.ffn, spec.q_dim), device="cuda")
    y = torch.empty(max(spec.vocab, spec.ffn, spec.qkv_rows), device="cuda")
    res = model.layers[:model.n_resident]
    shapes = [("qkv", [t["w_qkv"] for t in res], spec.qkv_rows, spec.hidden),
              ("o", [t["w_o"] for t in res], spec.hidden, spec.q_dim),
              ("gate_up", [t[k] for t in res for k in ("w_gate", "w_up")], spec.ffn, spec.hidden),
              ("down", [t["w_down"] for t in res], spec.hidden, spec.ffn),
              ("lm_head", [model.output], spec.vocab, spec.hidden)]
    q = lib_qtype(spec)
    fmt = {0: "q8_0", 1: "q4_0", 2: "q4_k", 3: "q6_k"}[spec.qtype] + ("_t" if spec.tiled else "")
    sha = gemv_sources_sha()
    out, tot_bytes, tot_ms, tot_launch, tot_traffic = {}, 0.0, 0.0, 0, 0.0
    with torch.cuda.stream(stream):
        for name, mats, r, c in shapes:
            per = r * synth.row_bytes(spec.qtype, c) + 4 * (c + r)
            n = max(len(mats) * iters, 4)
            for W in mats[:4]:
                ntx.ntx_gemv_q(q, W, r, c, x, y, stream.cuda_stream)
            torch.cuda.synchronize()
            # the n launches back to back in a CUDA graph, so the host's launch rate does
            # not bound the small shapes
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=stream):
                for i in range(n):
                    ntx.ntx_gemv_q(q, mats[i % len(mats)], r, c, x, y, stream.cuda_stream)
            g.replay()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            torch.cuda.synchronize()
            e0.record(stream)
            g.replay()
            e1.record(stream)
            torch.cuda.synchronize()
            del g
            ms = e0.elapsed_time(e1) / n
            launches = len(mats)    # launches of this shape in one decode step
            tr = GEMV_TRAFFIC.get(f"{fmt}:{r}x{c}") if sha == GEMV_TRAFFIC_SRC_SHA else None
            out[name] = {"shape": f"{fmt}:{r}x{c}", "bytes_per_launch": per, "avg_launch_us": ms * 1e3,
                         "achieved_gbs": per / (ms * 1e-3) / 1e9, "launches_per_step": launches,
                         "traffic_per_launch": tr}
            tot_bytes += per * launches
            tot_ms += ms * launches
            tot_launch += launches
            tot_traffic = None if (tr is None or tot_traffic is None) else tot_traffic + tr * launches
    agg = {"achieved": tot_bytes / (tot_ms * 1e-3) / 1e9, "bytes_per_launch": tot_bytes / tot_launch,
           "avg_launch_us": tot_ms * 1e3 / tot_launch,
           "traffic": None if tot_traffic is None else tot_traffic / tot_launch}
    return agg, out


def run_decode_bench(args, rank, world, local):
    import torch
    import quantized_weight_gemv_block_b200 as ntx
    from synth.device_model import DeviceModel

    name = args.workload
    spec = spec_for(name, args.layout)
    streamed = name == "llama70b_q4k_stream"
    n_res = 36 if streamed else None
    t0 = time.time()
    model = DeviceModel(spec, n_resident=n_res)
    setup_s = time.time() - t0
    token, pos = spec.token(), spec.n_prefill
    stream = torch.cuda.Stream()
    copy_stream = torch.cuda.Stream() if streamed else None
    logits = torch.empty(spec.vocab, dtype=torch.float32, device="cuda")
    # step word + embedding, per layer QKV, attention, split merge, O, gate/up, down, then the LM head
    launches_per_step = 2 + 6 * spec.n_layers + 1

    def step():
        if streamed:
            ntx.ntx_stream_layers(model.handle, token, pos, logits, stream.cuda_stream, copy_stream.cuda_stream, 0)
        else:
            ntx.ntx_decode_step(model.handle, token, pos, logits, stream.cuda_stream)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    barrier(world)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(local) as clk:
        e0.record(stream)
        for _ in range(args.steps):
            step()
        e1.record(stream)
        torch.cuda.synchronize()
    barrier(world)
    ms = e0.elapsed_time(e1) / args.steps
    ms = max_over_ranks(ms, world)
    dev_err = ntx.ntx_device_error()

    # end to end through the public API: token in from the host, logits back to pinned host memory
    host_logits = torch.empty(spec.vocab, dtype=torch.float32, pin_memory=True)
    e2e_steps = max(3, min(args.steps, 10))
    torch.cuda.synchronize()
    t_e2e = time.perf_counter()
    for _ in range(e2e_steps):
        step()
        with torch.cuda.stream(stream):
            host_logits.copy_(logits, non_blocking=True)
        stream.synchronize()
    e2e_ms = (time.perf_counter() - t_e2e) * 1e3 / e2e_steps
    e2e_ms = max_over_ranks(e2e_ms, world)

    out = {"ms_per_step": ms, "tok_s": world * 1e3 / ms, "e2e_tok_s": world * 1e3 / e2e_ms, "setup_s": setup_s,
           "clocks": clk.summary(), "launches": launches_per_step * args.steps, "device_error": dev_err,
           "bytes": step_bytes(spec), "spec": spec, "model": model, "stream": stream}
    if streamed:
        h2d, step_ms = ntx.ntx_stream_stats(model.handle)
        out["h2d_bytes"] = h2d
        out["h2d_gbs"] = h2d / (ms * 1e-3) / 1e9
        out["h2d_peak_gbs"] = measure_h2d()
    return out


def measure_h2d():
    """Pinned host -> device copy bandwidth of this machine (1 GiB, best of 3)."""
    import torch
    n = 1 << 30
    h = torch.empty(n, dtype=torch.uint8, pin_memory=True)
    d = torch.empty(n, dtype=torch.uint8, device="cuda")
    best = 0.0
    for _ in range(3):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        d.copy_(h, non_blocking=True)
        e1.record()
        torch.cuda.synchronize()
        best = max(best, n / (e0.elapsed_time(e1) * 1e-3) / 1e9)
    del h, d
    return best


def cpu_baseline(spec, budget_s=20.0):
    """The CPU oracle, as it stands, on a bounded sample of the decode step: whole
    layers at the workload's shape (weights generated before timing) and a slice of
    the LM head; extrapolated to one token."""
    import numpy as np
    import oracle
    from oracle import model as om
    import synth
    oracle.build()
    dims = oracle.dims_of(spec)
    t = om.layer_tensors(spec, 0)
    h = om.embedding_row(spec, spec.token()).copy()
    n_layers_timed, t_layers = 0, 0.0
    while t_layers < budget_s * 0.7 and n_layers_timed < spec.n_layers:
        t0 = time.perf_counter()
        oracle.decode_layer(dims, spec.qtype, h, spec.n_prefill, t["attn_norm"], t["w_qkv"], t["w_o"], t["ffn_norm"],
                            t["w_gate"], t["w_up"], t["w_down"], t["k_cache"], t["v_cache"])
        t_layers += time.perf_counter() - t0
        n_layers_timed += 1
    head_rows = max(256, spec.vocab // 32)
    norm, W = om.head_tensors(spec, (0, head_rows))
    t0 = time.perf_counter()
    oracle.lm_head(spec.qtype, norm, W, head_rows, spec.hidden, spec.rms_eps, h)
    t_head = (time.perf_counter() - t0) * spec.vocab / head_rows
    s_per_tok = t_layers / n_layers_timed * spec.n_layers + t_head
    return {"value": 1.0 / s_per_tok, "unit": "tok/s", "cores": oracle.threads(), "kind": "oracle",
            "sample": f"{n_layers_timed} of {spec.n_layers} layers (full shape, ctx {spec.n_prefill + 1}) "
                      f"+ {head_rows} of {spec.vocab} LM-head rows, extrapolated to one token"}


def gemv_bench(ntx, iters=50, tiled=True):
    """Q8_0 4096 x 4096 GEMV rotating over 16 weight copies (> 2 x L2)."""
    import torch
    import synth
    rows = cols = 4096
    qp = synth.sweep_qparams(synth.Q8_0)
    rb = synth.row_bytes(synth.Q8_0, cols)
    copies = [torch.empty(rows * rb, dtype=torch.uint8, device="cuda") for _ in range(16)]
    tmp = torch.empty(rows * rb, dtype=torch.uint8, device="cuda")
    for i, c in enumerate(copies):
        if tiled:
            synth.blocks_dev(tmp, synth.Q8_0, 0, 1, rows, cols, qp)
            ntx.ntx_repack_q(synth.Q8_0, tmp, c, rows, cols)
        else:
            synth.blocks_dev(c, synth.Q8_0, 0, 1, rows, cols, qp)
    q = synth.Q8_0 | (16 if tiled else 0)
    x = torch.empty(cols, device="cuda")
    synth.normal_f32_dev(x, 0, 2)
    y = torch.empty(rows, device="cuda")
    s = torch.cuda.Stream()
    for c in copies:
        ntx.ntx_gemv_q(q, c, rows, cols, x, y, s.cuda_stream)
    torch.cuda.synchronize()
    # back to back from a CUDA graph, so the host's launch rate does not bound them
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        for i in range(iters):
            ntx.ntx_gemv_q(q, copies[i % 16], rows, cols, x, y, s.cuda_stream)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(s):   # replay() launches on the current stream
        g.replay()
        torch.cuda.synchronize()
        e0.record(s)
        g.replay()
        e1.record(s)
    torch.cuda.synchronize()
    del g
    us = e0.elapsed_time(e1) * 1e3 / iters
    nbytes = rows * rb + 4 * (rows + cols)
    return {"us": us, "gbs": nbytes / (us * 1e-6) / 1e9}


def measure_read_ceiling(ntx, stream, nbytes=4 << 30, iters=10):
    """The practical HBM ceiling of the GEMV's data path: ntx_stream_read_probe (one CTA
    per SM, 1-D bulk copies into a shared-memory ring, no arithmetic) over a buffer much
    larger than L2, timed with CUDA events on the bench stream."""
    import torch
    buf = torch.empty(nbytes, dtype=torch.uint8, device="cuda")
    buf.fill_(1)
    for _ in range(3):
        ntx.ntx_stream_read_probe(buf, nbytes, stream.cuda_stream)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    e0.record(stream)
    for _ in range(iters):
        ntx.ntx_stream_read_probe(buf, nbytes, stream.cuda_stream)
    e1.record(stream)
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1) / iters
    del buf
    torch.cuda.empty_cache()
    return nbytes / (ms * 1e-3) / 1e9


def profile_gemv(what, launches):
    """A few launches of each listed GEMV (what = FMT:ROWSxCOLS[,FMT:ROWSxCOLS...],
    weights larger than L2 or ncu's cache flush between captured launches), nothing
    else: the case that profiler captures of the GEMV kernel run.  Per shape: one
    warm-up launch, then `launches` launches timed together with CUDA events."""
    import torch
    import synth
    import quantized_weight_gemv_block_b200 as ntx
    from quantized_weight_gemv_block_b200 import build
    build.build()
    synth.build_dev()
    for one in what.split(","):
        fmt, shape = one.split(":")
        rows, cols = (int(v) for v in shape.split("x"))
        tiled = fmt.endswith("_t")
        q = synth.qtype_of(fmt[:-2] if tiled else fmt)
        W = torch.empty(rows * synth.row_bytes(q, cols), dtype=torch.uint8, device="cuda")
        synth.blocks_dev(W, q, 0, 1, rows, cols, synth.sweep_qparams(q))
        if tiled:
            Wt = torch.empty_like(W)
            ntx.ntx_repack_q(q, W, Wt, rows, cols)
            W = Wt
            q |= 16
        x = torch.empty(cols, device="cuda")
        synth.normal_f32_dev(x, 0, 2)
        y = torch.empty(rows, device="cuda")
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        ntx.ntx_gemv_q(q, W, rows, cols, x, y)
        torch.cuda.synchronize()
        e0.record()
        for _ in range(launches):
            ntx.ntx_gemv_q(q, W, rows, cols, x, y)
        e1.record()
        torch.cuda.synchronize()
        us = e0.elapsed_time(e1) * 1e3 / launches
        print(json.dumps({"gemv": one, "bytes": W.numel(), "us": us, "gbs": W.numel() / (us * 1e-6) / 1e9}))
        del W, x, y
        torch.cuda.empty_cache()


def profile_attn(what, launches):
    """A few launches of the split-KV decode attention on one shape (random fp16 KV
    cache, L2 flushed between launches), nothing else: the case that profiler
    captures of the attention kernel run.  what = QHEADS:KVHEADS:CONTEXT."""
    import torch
    import quantized_weight_gemv_block_b200 as ntx
    from quantized_weight_gemv_block_b200 import build
    build.build()
    nq, nkv, ctx = (int(v) for v in what.split(":"))
    hd = 128
    g = torch.Generator(device="cuda").manual_seed(7)
    q = torch.randn(nq * hd, device="cuda", generator=g)
    k = torch.randn(nkv * ctx * hd, device="cuda", generator=g).half()
    v = torch.randn(nkv * ctx * hd, device="cuda", generator=g).half()
    out = torch.empty(nq * hd, device="cuda")
    wsb = ntx.ntx_attn_workspace_bytes(nq, nkv, hd, ctx)
    ws = torch.empty(wsb, dtype=torch.uint8, device="cuda")
    flush = torch.empty(256 << 20, dtype=torch.uint8, device="cuda")
    times = []
    for i in range(launches + 1):
        flush.fill_(i & 0xFF)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        ntx.ntx_attn_decode(q, k, v, out, nq, nkv, hd, ctx, ctx, ws, wsb)
        e1.record()
        torch.cuda.synchronize()
        if i:
            times.append(e0.elapsed_time(e1) * 1e3)
    us = sorted(times)[len(times) // 2]
    kv = 2 * nkv * ctx * hd * 2
    print(json.dumps({"attn": what, "kv_bytes": kv, "us_median": us, "gbs": kv / (us * 1e-6) / 1e9}))


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ntx", choices=["ntx", "reference"])
    ap.add_argument("--workload", default="llama70b_q6k_decode",
                    choices=["llama70b_q6k_decode", "llama8b_q8_0_decode", "llama70b_q4k_stream"])
    ap.add_argument("--layout", default="tiled", choices=["tiled", "gguf"],
                    help="weights handed to the library as tiled (repacked once at load) or GGUF-style blocks")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-extras", action="store_true")
    ap.add_argument("--profile-gemv", default=None, metavar="FMT:ROWSxCOLS[,...]",
                    help="only run the GEMV kernel on one matrix (for profilers), e.g. q6_k:28672x8192")
    ap.add_argument("--profile-attn", default=None, metavar="QHEADS:KVHEADS:CONTEXT",
                    help="only run the decode attention on one shape (for profilers), e.g. 64:8:8193")
    args = ap.parse_args()
    if args.profile_gemv:
        return profile_gemv(args.profile_gemv, args.steps)
    if args.profile_attn:
        return profile_attn(args.profile_attn, args.steps)
    if args.warmup < 3:
        args.warmup = 3

    if args.impl == "reference":
        # the CPU oracle needs no process group: rank 0 alone runs it, the others exit
        rank, world, local = int(os.environ.get("RANK", "0")), int(os.environ.get("WORLD_SIZE", "1")), 0
    else:
        rank, world, local = dist_setup(args.gpus)
    spec = spec_for(args.workload, args.layout)
    config = {"workload": args.workload, "layers": spec.n_layers, "hidden": spec.hidden, "ffn": spec.ffn,
              "q_heads": spec.n_q_heads, "kv_heads": spec.n_kv_heads, "vocab": spec.vocab, "format": ["q8_0", "q4_0",
              "q4_k", "q6_k"][spec.qtype], "layout": args.layout, "context": spec.n_prefill + 1, "batch": 1,
              "l2": "inputs larger than L2 (weights %.1f GB per step)" % (step_bytes(spec) / 1e9),
              "parallelism": "replicas" if world > 1 else "single"}

    if args.impl == "reference":
        if rank != 0:
            return
        cb = None
        vals = []
        for i in range(args.warmup + args.steps):
            cb = cpu_baseline(spec, budget_s=6.0)
            if i >= args.warmup:
                vals.append(cb["value"])
        v = statistics.median(vals)
        cb["value"] = v
        print(json.dumps({"metric": METRIC, "value": v, "unit": "tok/s", "n_gpus": args.gpus, "steps": args.steps,
                          "warmup": args.warmup, "ms_per_step": 1e3 / v, "higher_is_better": True,
                          "scaling": "weak", "vs_baseline": None, "dtype": "f32", "data": "synthetic",
                          "impl": "reference", "config": config, "cpu_baseline": cb,
                          "e2e": {"value": v, "unit": "tok/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}))
        return

    import torch
    import quantized_weight_gemv_block_b200 as ntx
    from quantized_weight_gemv_block_b200 import build
    import synth
    build.build()
    synth.build_dev()
    torch.cuda.set_device(local)
    r = run_decode_bench(args, rank, world, local)
    spec, model, stream = r["spec"], r["model"], r["stream"]
    peak, peak_kind = load_peaks()

    line = {"metric": METRIC, "value": r["tok_s"], "unit": "tok/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": r["ms_per_step"], "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f32", "data": "synthetic (seeded random weights and KV cache)",
            "config": config, "clocks": r["clocks"], "gpu_launches": r["launches"],
            "e2e": {"value": r["e2e_tok_s"], "unit": "tok/s", "h2d_bytes_per_step": 8,
                    "d2h_bytes_per_step": 4 * spec.vocab}}
    step_gbs = r["bytes"] / (r["ms_per_step"] * 1e-3) / 1e9
    line["step_hbm"] = {"bytes_per_step": r["bytes"], "achieved_gbs": step_gbs, "frac_of_%s" % peak_kind:
                        step_gbs / peak, "frac_of_8000": step_gbs / 8000.0}
    if args.workload == "llama70b_q4k_stream":
        line["host_link"] = {"h2d_bytes_per_step": r["h2d_bytes"], "achieved_gbs": r["h2d_gbs"],
                             "measured_pinned_h2d_gbs": r["h2d_peak_gbs"], "frac": r["h2d_gbs"] / r["h2d_peak_gbs"]}
    if rank == 0:
        agg, per_shape = measure_gemv_roofline(ntx, model, spec, stream)
        line["roofline"] = {"bound": "hbm", "kernel": "qmma_kernel<%s> (all GEMV launches of one step)" % config["format"],
                            "achieved": agg["achieved"], "peak": peak, "peak_kind": peak_kind, "unit": "GB/s",
                            "frac": agg["achieved"] / peak, "traffic": agg["traffic"],
                            "bytes_per_launch": agg["bytes_per_launch"], "avg_launch_us": agg["avg_launch_us"]}
        line["gemv_shapes"] = per_shape
        ceil_gbs = measure_read_ceiling(ntx, stream)
        line["read_ceiling"] = {"kernel": "ntx_stream_read_probe (bulk-copy ring, one CTA per SM, no arithmetic)",
                                "gbs": ceil_gbs, "frac_of_%s" % peak_kind: ceil_gbs / peak}
        line["roofline"]["frac_of_read_ceiling"] = agg["achieved"] / ceil_gbs
        if not args.no_extras:
            line["gemv_q8_0_4096x4096"] = {"tiled": gemv_bench(ntx, tiled=True), "gguf": gemv_bench(ntx, tiled=False)}
        if not args.no_cpu_baseline:
            line["cpu_baseline"] = cpu_baseline(spec)
        if r["device_error"]:
            line["device_error"] = r["device_error"]
        print(json.dumps(line))
    model.close()
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
