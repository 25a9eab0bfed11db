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
  gemv_sweep                     the quantized GEMV sweep at the Llama-8B layer shapes in Q4_0
                                 and Q4_K (both layouts) and the single Q8_0 4096 x 4096 GEMV,
                                 weights rotated over copies larger than 2 x L2; metric GB/s

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

def spec_for(name, layout="tiled", layers=None, extra_ctx=0):
    """The workload's model; `layers` shortens it (profiler captures only); `extra_ctx` adds
    KV-cache positions past the decode position (room for multi-token verify passes)."""
    import synth
    tiled = layout == "tiled"
    base = {"llama70b_q6k_decode": synth.LLAMA_70B_Q6_K, "llama8b_q8_0_decode": synth.LLAMA_8B_Q8_0,
            "llama70b_q4k_stream": synth.LLAMA_70B_Q4_K}[name]
    kw = dict(base)
    if layers:
        kw["n_layers"] = layers
    kw["max_ctx"] += extra_ctx
    return synth.ModelSpec(**kw, tiled=tiled)


def lib_qtype(spec):
    return spec.qtype | (16 if spec.tiled else 0)


def kv_read_bytes(spec):
    return spec.n_layers * 2 * spec.n_kv_heads * (spec.n_prefill + 1) * spec.head_dim * 2


def step_bytes(spec):
    """Algorithmic bytes of one decode step: packed weights read + KV cache read
    (positions 0..pos) + the embedding row (vectors are negligible)."""
    import synth
    w = sum(spec.layer_weight_bytes(l) for l in range(spec.n_layers))
    w += spec.vocab * synth.row_bytes(spec.qtype_of("output"), spec.hidden)
    return w + kv_read_bytes(spec) + synth.row_bytes(spec.qtype_of("tok_embd"), spec.hidden)


def gemv_kinds(spec):
    """The step's fused GEMV launches per kind: (name, replay kind, rows, cols, matrices per
    launch, launches per step, algorithmic bytes per launch).  Bytes = packed weights read +
    the fp32 vectors read and written (+ the fp16 K / V rows the QKV epilogue appends)."""
    import synth
    h, f, qd, L = spec.hidden, spec.ffn, spec.q_dim, spec.n_layers
    rb = lambda c: synth.row_bytes(spec.qtype, c)
    kvd = spec.n_kv_heads * spec.head_dim
    return [("qkv", 0, spec.qkv_rows, h, 1, L, spec.qkv_rows * rb(h) + 4 * (2 * h + qd) + 2 * 2 * kvd),
            ("o", 1, h, qd, 1, L, h * rb(qd) + 4 * (qd + 2 * h)),
            ("gate_up", 2, f, h, 2, L, 2 * f * rb(h) + 4 * (2 * h + f)),
            ("down", 3, h, f, 1, L, h * rb(f) + 4 * (f + 2 * h)),
            ("lm_head", 4, spec.vocab, h, 1, 1, spec.vocab * rb(h) + 4 * (2 * h + spec.vocab))]


# DRAM traffic (dram__bytes_read.sum + dram__bytes_write.sum, one ncu capture of the step's
# fused launch of each kind, bytes per launch) of the tiled GEMV, and a hash of the kernel
# sources it was taken with: a changed kernel reports traffic as unknown (null).  Captured with
#   ncu --metrics dram__bytes_read.sum,dram__bytes_write.sum,gpu__time_duration.sum \
#       --clock-control none -k regex:qmma_kernel -c 40 --csv --log-file traffic.csv \
#       python bench.py --workload <workload> --layers 2 --profile-step-gemv --warmup 3
# (the last five launches: QKV, O, gate/up, down, LM head).
GEMV_TRAFFIC_SRC_SHA = "edad805671c881a8"
GEMV_TRAFFIC = {
    "q6_k_t:qkv:10240x8192": 68951296,
    "q6_k_t:o:8192x8192": 55166464,
    "q6_k_t:gate_up:28672x8192": 385856512,
    "q6_k_t:down:8192x28672": 192995840,
    "q6_k_t:lm_head:128256x8192": 862166272,
    "q8_0_t:qkv:6144x4096": 26833920,
    "q8_0_t:o:4096x4096": 17900032,
    "q8_0_t:gate_up:14336x4096": 124950272,
    "q8_0_t:down:4096x14336": 62517760,
    "q8_0_t:lm_head:128256x4096": 558389248,
    "q4_k_t:qkv:10240x8192": 47322624,
    "q4_k_t:o:8192x8192": 37869568,
    "q4_k_t:gate_up:28672x8192": 264761600,
    "q4_k_t:down:8192x28672": 132520960,
    "q4_k_t:lm_head:128256x8192": 591300352,
}


def gemv_sources_sha():
    import hashlib
    h = hashlib.sha256()
    d = os.path.join(os.path.dirname(os.path.abspath(__file__)), "quantized_weight_gemv_block_b200", "csrc")
    for f in ("qmma.cuh", "qmma.cu", "blocks.cuh", "common.cuh", "gemv.cuh"):
        with open(os.path.join(d, f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def fmt_name(spec):
    return {0: "q8_0", 1: "q4_0", 2: "q4_k", 3: "q6_k"}[spec.qtype] + ("_t" if spec.tiled else "")


def measure_gemv_roofline(ntx, model, spec, stream, logits, rounds=5):
    """Time the step's own fused GEMV launches, kind by kind: ntx_model_replay_gemv enqueues
    them exactly as the decode step does (same kernels, prologues, epilogues, programmatic
    launch), cycling over the resident layers so no launch finds its weights in L2; n of
    them are captured in a CUDA graph and replayed on the bench stream between CUDA events.
    Per kind: average launch time (median over `rounds` replays) and algorithmic bytes per
    launch.  The launch-weighted aggregate over one step is the dominant kernel's achieved
    HBM bandwidth.  Only HBM-resident layers count (streamed ones are bound by the host link)."""
    import torch
    fmt = fmt_name(spec)
    sha = gemv_sources_sha()
    nres = model.n_resident
    out, tot_bytes, tot_ms, tot_launch, tot_traffic = {}, 0.0, 0.0, 0, 0.0
    for name, kind, r, c, nmat, per_step, per in gemv_kinds(spec):
        if kind != 4 and nres < 1:
            continue
        launches = per_step if kind == 4 else nres     # launches of this kind in one step's resident part
        n = max(3 * launches, 8) if kind != 4 else 8
        with torch.cuda.stream(stream):
            ntx.ntx_model_replay_gemv(model.handle, kind, min(n, 4), logits, stream.cuda_stream)
            torch.cuda.synchronize()
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=stream):
                ntx.ntx_model_replay_gemv(model.handle, kind, n, logits, stream.cuda_stream)
            g.replay()
            torch.cuda.synchronize()
            times = []
            for _ in range(rounds):
                e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                e0.record(stream)
                g.replay()
                e1.record(stream)
                torch.cuda.synchronize()
                times.append(e0.elapsed_time(e1) / n)
            del g
        ms = statistics.median(times)
        shape = f"{fmt}:{'2x' if nmat == 2 else ''}{r}x{c}"
        tr = GEMV_TRAFFIC.get(f"{fmt}:{name}:{r}x{c}") if sha == GEMV_TRAFFIC_SRC_SHA else None
        out[name] = {"shape": shape, "fused": ["rmsnorm+rope+kv_append", "residual_add", "rmsnorm+swiglu",
                                                "residual_add", "rmsnorm"][kind],
                     "bytes_per_launch": per, "avg_launch_us": ms * 1e3, "best_launch_us": min(times) * 1e3,
                     "achieved_gbs": per / (ms * 1e-3) / 1e9, "launches_per_step": launches,
                     "traffic_per_launch": tr}
        tot_bytes += per * launches
        tot_ms += ms * launches
        tot_launch += launches
        tot_traffic = None if (tr is None or tot_traffic is None) else tot_traffic + tr * launches
    agg = {"achieved": tot_bytes / (tot_ms * 1e-3) / 1e9, "bytes_per_launch": tot_bytes / tot_launch,
           "avg_launch_us": tot_ms * 1e3 / tot_launch, "launches": tot_launch,
           "traffic": None if tot_traffic is None else tot_traffic / tot_launch}
    return agg, out


def run_decode_bench(args, rank, world, local):
    import torch
    import quantized_weight_gemv_block_b200 as ntx
    from synth.device_model import DeviceModel

    name = args.workload
    # speculative passes verify k positions from the decode position on: room for 4 passes
    spec = spec_for(name, args.layout, args.layers, extra_ctx=4 * args.speculative)
    streamed = name == "llama70b_q4k_stream"
    n_res = 36 if streamed else None
    t0 = time.time()
    model = DeviceModel(spec, n_resident=n_res)
    setup_s = time.time() - t0
    token, pos = spec.token(), spec.n_prefill
    stream = torch.cuda.Stream()
    copy_stream = torch.cuda.Stream() if streamed else None
    logits = torch.empty(spec.vocab, dtype=torch.float32, device="cuda")
    # step word + embedding, per layer QKV, attention (+ split merge), O, gate/up, down, LM head
    launches_per_step = ntx.ntx_model_step_launches(model.handle)

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

    # end to end through the public API, the same number of steps: token in from the host,
    # logits back to pinned host memory, the host waiting for each step
    host_logits = torch.empty(spec.vocab, dtype=torch.float32, pin_memory=True)
    torch.cuda.synchronize()
    t_e2e = time.perf_counter()
    for _ in range(args.steps):
        step()
        with torch.cuda.stream(stream):
            host_logits.copy_(logits, non_blocking=True)
        stream.synchronize()
    e2e_ms = (time.perf_counter() - t_e2e) * 1e3 / args.steps
    e2e_ms = max_over_ranks(e2e_ms, world)

    # per-step spread: >= 50 replays, each between its own pair of events
    replay_ms = []
    for _ in range(max(50, args.steps)):
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        step()
        b.record(stream)
        replay_ms.append((a, b))
    torch.cuda.synchronize()
    replay_ms = sorted(a.elapsed_time(b) for a, b in replay_ms)

    out = {"ms_per_step": ms, "tok_s": world * 1e3 / ms, "e2e_tok_s": world * 1e3 / e2e_ms, "e2e_ms": e2e_ms,
           "setup_s": setup_s, "clocks": clk.summary(), "launches": launches_per_step * args.steps,
           "device_error": dev_err, "bytes": step_bytes(spec), "spec": spec, "model": model, "stream": stream,
           "logits": logits,
           "replays": {"n": len(replay_ms), "median_ms": statistics.median(replay_ms), "best_ms": replay_ms[0],
                       "worst_ms": replay_ms[-1]}}
    if streamed:
        h2d, step_ms = ntx.ntx_stream_stats(model.handle)
        out["h2d_bytes"] = h2d
        out["h2d_gbs"] = h2d / (ms * 1e-3) / 1e9
        out["h2d_peak_gbs"] = measure_h2d()
    if args.speculative:
        out["speculative"] = run_speculative(ntx, model, spec, token, pos, args.speculative, stream, copy_stream,
                                             max(3, args.steps // 2))
    return out


def run_speculative(ntx, model, spec, token, pos, k, stream, copy_stream, n_calls):
    """Self-speculative decoding: n_calls steps of (draft k - 1 tokens with the resident
    layers, verify k tokens in one pass), each timed with CUDA events on the compute stream.
    With random weights the draft's picks agree with the full model's by chance only, so the
    measured tokens per pass say nothing about trained models; the verify pass's positions
    per second (k per pass) is what full acceptance would give."""
    import torch
    cs = stream.cuda_stream
    ks = copy_stream.cuda_stream if copy_stream is not None else None
    times, counts, t, p = [], [], token, pos
    for i in range(n_calls + 1):
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        out = ntx.ntx_speculative_step(model.handle, t, p, k, None, cs, ks)
        b.record(stream)
        torch.cuda.synchronize()
        if i:     # the first call allocates the pass buffers
            times.append(a.elapsed_time(b))
            counts.append(len(out))
        t = out[-1]
        p = spec.n_prefill + ((p - spec.n_prefill + len(out)) % max(1, spec.max_ctx - spec.n_prefill - k))
    ms = statistics.median(times)
    return {"k": k, "calls": n_calls, "median_ms_per_call": ms, "tokens_per_call": statistics.mean(counts),
            "tok_s": sum(counts) / (sum(times) * 1e-3), "verify_positions_per_s_at_full_acceptance": k / (ms * 1e-3),
            "note": "random weights: acceptance is by chance; see verify_positions_per_s_at_full_acceptance"}


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


CPU_SAMPLE_LAYERS = 4     # whole layers the CPU baseline times per token (both arms alike)


def cpu_baseline(spec, n_layers_timed=CPU_SAMPLE_LAYERS):
    """The CPU oracle, as it stands, on a bounded sample of the decode step: the first
    `n_layers_timed` whole layers at the workload's shape (weights generated before timing)
    and 1/32 of the LM-head rows; the per-token time is extrapolated from them (layers x
    n_layers / n_layers_timed, head x 32)."""
    import oracle
    from oracle import model as om
    oracle.build()
    dims = oracle.dims_of(spec)
    h = om.embedding_row(spec, spec.token()).copy()
    n = min(n_layers_timed, spec.n_layers)
    t_layers = 0.0
    for layer in range(n):
        t = om.layer_tensors(spec, layer)
        t0 = time.perf_counter()
        qts = [spec.qtype_of(k, layer) for k in ("w_qkv", "w_o", "w_gate", "w_down")]
        oracle.decode_layer(dims, qts, h, spec.n_prefill, t["attn_norm"], t["w_qkv"], t["w_o"], t["ffn_norm"],
                            t["w_gate"], t["w_up"], t["w_down"], t["k_cache"], t["v_cache"])
        t_layers += time.perf_counter() - t0
    head_rows = max(256, spec.vocab // 32)
    norm, W = om.head_tensors(spec, (0, head_rows))
    t0 = time.perf_counter()
    oracle.lm_head(spec.qtype_of("output"), norm, W, head_rows, spec.hidden, spec.rms_eps, h)
    t_head = (time.perf_counter() - t0) * spec.vocab / head_rows
    s_per_tok = t_layers / n * spec.n_layers + t_head
    return {"value": 1.0 / s_per_tok, "unit": "tok/s", "cores": oracle.threads(), "kind": "oracle",
            "extrapolated": True,
            "sample": f"{n} of {spec.n_layers} layers (full shape, ctx {spec.n_prefill + 1}) "
                      f"+ {head_rows} of {spec.vocab} LM-head rows timed, extrapolated to one token"}


SWEEP_SHAPES = [("qkv", 6144, 4096), ("o", 4096, 4096), ("gate_or_up", 14336, 4096), ("down", 4096, 14336),
                ("lm_head", 128256, 4096)]


def gemv_rotation_bench(ntx, qtype, rows, cols, tiled, stream, n_launch=48, rounds=5):
    """One GEMV shape on its own: enough weight copies that one pass over them exceeds
    2 x L2 (so every launch streams its weights from HBM), n_launch launches cycling over
    the copies captured in a CUDA graph (programmatic launch between them, as in the step)
    and replayed `rounds` times between CUDA events; the median and best per-launch times."""
    import math
    import torch
    import synth
    l2 = torch.cuda.get_device_properties(torch.cuda.current_device()).L2_cache_size
    rb = synth.row_bytes(qtype, cols)
    nbytes = rows * rb
    n_copies = max(2, math.ceil(2 * l2 / nbytes) + 1)
    qp = synth.sweep_qparams(qtype)
    base = torch.empty(nbytes, dtype=torch.uint8, device="cuda")
    synth.blocks_dev(base, qtype, 0, 1, rows, cols, qp)
    if tiled:
        t = torch.empty_like(base)
        ntx.ntx_repack_q(qtype, base, t, rows, cols)
        base = t
    copies = [base] + [base.clone() for _ in range(n_copies - 1)]
    q = qtype | (16 if tiled else 0)
    x = torch.empty(cols, device="cuda")
    synth.normal_f32_dev(x, 0, 2)
    y = torch.empty(rows, device="cuda")
    with torch.cuda.stream(stream):
        for c in copies[:4]:
            ntx.ntx_gemv_q(q, c, rows, cols, x, y, stream.cuda_stream)
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=stream):
            for i in range(n_launch):
                ntx.ntx_gemv_q(q, copies[i % n_copies], rows, cols, x, y, stream.cuda_stream)
        g.replay()
        torch.cuda.synchronize()
        times = []
        for _ in range(rounds):
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            g.replay()
            e1.record(stream)
            torch.cuda.synchronize()
            times.append(e0.elapsed_time(e1) * 1e3 / n_launch)
        del g
    del copies, base
    torch.cuda.empty_cache()
    per = nbytes + 4 * (rows + cols)
    us = statistics.median(times)
    return {"bytes_per_launch": per, "us": us, "best_us": min(times), "gbs": per / (us * 1e-6) / 1e9,
            "copies": n_copies}


def gemv_sweep(ntx, stream, peak, peak_kind, ceiling):
    """The quantized GEMV sweep at the Llama-8B layer shapes (4096 -> 6144 fused QKV,
    4096 -> 4096 O, 4096 -> 14336 gate or up, 14336 -> 4096 down, 4096 -> 128256 LM head)
    in Q4_0 and Q4_K, in both layouts, plus the single Q8_0 4096 x 4096 GEMV."""
    import synth
    rows_out = []
    for qname, q in (("q4_0", synth.Q4_0), ("q4_k", synth.Q4_K)):
        for layout in ("tiled", "gguf"):
            for name, rows, cols in SWEEP_SHAPES:
                r = gemv_rotation_bench(ntx, q, rows, cols, layout == "tiled", stream)
                r.update({"format": qname, "layout": layout, "shape": name, "rows": rows, "cols": cols,
                          "frac_of_%s" % peak_kind: r["gbs"] / peak, "frac_of_read_ceiling": r["gbs"] / ceiling})
                rows_out.append(r)
    single = {}
    for layout in ("tiled", "gguf"):
        r = gemv_rotation_bench(ntx, synth.Q8_0, 4096, 4096, layout == "tiled", stream)
        r.update({"frac_of_%s" % peak_kind: r["gbs"] / peak, "frac_of_read_ceiling": r["gbs"] / ceiling})
        single[layout] = r
    # the further formats at the same shapes: Q5_K in its tiled layout, F16 and F32 rows
    further = []
    for qname, q, tiled in (("q5_k", synth.Q5_K, True), ("f16", synth.F16, False), ("f32", synth.F32, False)):
        for name, rows, cols in SWEEP_SHAPES:
            r = gemv_rotation_bench(ntx, q, rows, cols, tiled, stream)
            r.update({"format": qname, "layout": "tiled" if tiled else "rows", "shape": name, "rows": rows,
                      "cols": cols, "frac_of_%s" % peak_kind: r["gbs"] / peak,
                      "frac_of_read_ceiling": r["gbs"] / ceiling})
            further.append(r)
    return rows_out, single, further


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


DTYPE = "i8*i24->i32+f32"
DTYPE_DETAIL = ("weights: packed block codes (4/6/8-bit) unpacked to int8; GEMV: integer dot products (dp4a) "
                "of the codes with x as 24-bit fixed point (three int8 limbs, one exponent per 32-column step), "
                "exact int32 block sums, block scales and sums in fp32; attention: fp16 KV cache, fp32 softmax and "
                "accumulation (fp16 tensor-core products of exact split operands); activations fp32")
ROOFLINE_FRAC_LIMIT = 1.2   # a GEMV timed above 1.2 x the copy peak is not doing the work: refuse the figure


def print_line(line):
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ntx", choices=["ntx", "reference"])
    ap.add_argument("--workload", default="llama70b_q6k_decode",
                    choices=["llama70b_q6k_decode", "llama8b_q8_0_decode", "llama70b_q4k_stream", "gemv_sweep"])
    ap.add_argument("--layout", default="tiled", choices=["tiled", "gguf"],
                    help="weights handed to the library as tiled (repacked once at load) or GGUF-style blocks")
    ap.add_argument("--layers", type=int, default=None,
                    help="shorten the model to this many layers (profiler captures only; the line says so)")
    ap.add_argument("--speculative", type=int, default=0, metavar="K",
                    help="also time self-speculative decoding steps verifying K tokens per pass")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-extras", action="store_true")
    ap.add_argument("--profile-gemv", default=None, metavar="FMT:ROWSxCOLS[,...]",
                    help="only run the GEMV kernel on one matrix (for profilers), e.g. q6_k:28672x8192")
    ap.add_argument("--profile-attn", default=None, metavar="QHEADS:KVHEADS:CONTEXT",
                    help="only run the decode attention on one shape (for profilers), e.g. 64:8:8193")
    ap.add_argument("--profile-step-gemv", action="store_true",
                    help="build the model, run --warmup steps, then one launch of each of the step's fused GEMV "
                         "kinds (for profilers; use with --layers)")
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
    peak, peak_kind = load_peaks()

    if args.workload == "gemv_sweep":
        return run_sweep(args, rank, world, local, peak, peak_kind)

    spec = spec_for(args.workload, args.layout, args.layers)
    config = {"workload": args.workload, "layers": spec.n_layers, "hidden": spec.hidden, "ffn": spec.ffn,
              "q_heads": spec.n_q_heads, "kv_heads": spec.n_kv_heads, "vocab": spec.vocab, "format": ["q8_0", "q4_0",
              "q4_k", "q6_k"][spec.qtype], "layout": args.layout, "context": spec.n_prefill + 1, "batch": 1,
              "l2": "inputs larger than L2 (weights %.1f GB per step)" % (step_bytes(spec) / 1e9),
              "parallelism": "replicas" if world > 1 else "single"}
    if args.layers:
        config["shortened_for_profiling"] = True

    if args.impl == "reference":
        if rank != 0:
            return
        cb = None
        vals = []
        for i in range(args.warmup + args.steps):
            cb = cpu_baseline(spec)
            if i >= args.warmup:
                vals.append(cb["value"])
        v = statistics.median(vals)
        cb["value"] = v
        print_line({"metric": METRIC, "value": v, "unit": "tok/s", "n_gpus": args.gpus, "steps": args.steps,
                    "warmup": args.warmup, "ms_per_step": 1e3 / v, "higher_is_better": True,
                    "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
                    "impl": "reference", "config": config, "cpu_baseline": cb,
                    "note": "each step times a sample of one token (cpu_baseline.sample) and extrapolates",
                    "e2e": {"value": v, "unit": "tok/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}})
        return

    import torch
    import quantized_weight_gemv_block_b200 as ntx
    from quantized_weight_gemv_block_b200 import build
    import synth
    build.build()
    synth.build_dev()
    torch.cuda.set_device(local)
    if args.profile_step_gemv:
        return profile_step_gemv(args, spec)
    r = run_decode_bench(args, rank, world, local)
    spec, model, stream = r["spec"], r["model"], r["stream"]

    line = {"metric": METRIC, "value": r["tok_s"], "unit": "tok/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": r["ms_per_step"], "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": DTYPE, "dtype_detail": DTYPE_DETAIL,
            "data": "synthetic (seeded random weights and KV cache)",
            "config": config, "clocks": r["clocks"], "gpu_launches": r["launches"],
            "e2e": {"value": r["e2e_tok_s"], "unit": "tok/s", "h2d_bytes_per_step": 8,
                    "d2h_bytes_per_step": 4 * spec.vocab, "steps": args.steps,
                    "not_faster_than_device_timed": r["e2e_tok_s"] <= r["tok_s"] * 1.01},
            "replays": r["replays"]}
    step_gbs = r["bytes"] / (r["ms_per_step"] * 1e-3) / 1e9
    line["step_hbm"] = {"bytes_per_step": r["bytes"], "achieved_gbs": step_gbs, "frac_of_%s" % peak_kind:
                        step_gbs / peak, "frac_of_8000": step_gbs / 8000.0}
    if args.workload == "llama70b_q4k_stream":
        line["host_link"] = {"h2d_bytes_per_step": r["h2d_bytes"], "achieved_gbs": r["h2d_gbs"],
                             "measured_pinned_h2d_gbs": r["h2d_peak_gbs"], "frac": r["h2d_gbs"] / r["h2d_peak_gbs"]}
    if "speculative" in r:
        line["speculative"] = r["speculative"]
    if rank == 0:
        agg, per_kind = measure_gemv_roofline(ntx, model, spec, stream, r["logits"])
        frac = agg["achieved"] / peak
        line["roofline"] = {"bound": "hbm",
                            "kernel": "qmma_kernel<%s> (the step's fused GEMV launches, all kinds, launch-weighted)"
                                      % fmt_name(spec),
                            "achieved": agg["achieved"], "peak": peak, "peak_kind": peak_kind, "unit": "GB/s",
                            "frac": frac, "traffic": agg["traffic"],
                            "bytes_per_launch": agg["bytes_per_launch"], "avg_launch_us": agg["avg_launch_us"],
                            "launches_per_step": agg["launches"]}
        if frac > ROOFLINE_FRAC_LIMIT:
            line["roofline"]["rejected"] = "achieved above %.1f x the copy peak: the timed kernel is not doing " \
                                           "the work" % ROOFLINE_FRAC_LIMIT
            line["roofline"]["frac"] = None
        line["gemv_kinds"] = per_kind
        ceil_gbs = measure_read_ceiling(ntx, stream)
        line["read_ceiling"] = {"kernel": "ntx_stream_read_probe (bulk-copy ring, one CTA per SM, no arithmetic)",
                                "gbs": ceil_gbs, "frac_of_%s" % peak_kind: ceil_gbs / peak}
        line["roofline"]["frac_of_read_ceiling"] = agg["achieved"] / ceil_gbs
        if not args.no_extras:
            line["gemv_q8_0_4096x4096"] = {lay: gemv_rotation_bench(ntx, synth.Q8_0, 4096, 4096, lay == "tiled",
                                                                    stream) for lay in ("tiled", "gguf")}
        if not args.no_cpu_baseline:
            line["cpu_baseline"] = cpu_baseline(spec)
        if r["device_error"]:
            line["device_error"] = r["device_error"]
        print_line(line)
    model.close()
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


def run_sweep(args, rank, world, local, peak, peak_kind):
    """--workload gemv_sweep: the GEMV sweep's line (metric: quantized GEMV HBM GB/s)."""
    config = {"workload": "gemv_sweep", "shapes": [f"{c}->{r}" for _, r, c in SWEEP_SHAPES],
              "formats": ["q4_0", "q4_k"], "layouts": ["tiled", "gguf"], "batch": 1,
              "l2": "weights rotated over copies larger than 2 x L2", "parallelism": "single"}
    if args.impl == "reference":
        if rank != 0:
            return
        import numpy as np
        import oracle
        import synth
        oracle.build()
        vals = []
        for i in range(args.warmup + args.steps):
            tot_b, tot_s = 0, 0.0
            for qname, q in (("q4_0", synth.Q4_0), ("q4_k", synth.Q4_K)):
                for name, rows, cols in SWEEP_SHAPES:
                    n = 64
                    W = synth.blocks_host(q, 0, 1, n, cols, synth.sweep_qparams(q))
                    x = synth.normal_f32_host(0, 2, cols)
                    t0 = time.perf_counter()
                    oracle.gemv(q, W, n, cols, x)
                    tot_s += time.perf_counter() - t0
                    tot_b += W.size
            if i >= args.warmup:
                vals.append(tot_b / tot_s / 1e9)
        v = statistics.median(vals)
        print_line({"metric": "quantized GEMV GB/s", "value": v, "unit": "GB/s", "n_gpus": args.gpus,
                    "steps": args.steps, "warmup": args.warmup, "higher_is_better": True, "scaling": "weak",
                    "vs_baseline": None, "dtype": "f64", "data": "synthetic", "impl": "reference", "config": config,
                    "cpu_baseline": {"value": v, "unit": "GB/s", "cores": oracle.threads(), "kind": "oracle",
                                     "sample": "64 rows of each sweep shape and format"},
                    "e2e": {"value": v, "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}})
        return
    import torch
    import quantized_weight_gemv_block_b200 as ntx
    from quantized_weight_gemv_block_b200 import build
    import synth
    build.build()
    synth.build_dev()
    torch.cuda.set_device(local)
    stream = torch.cuda.Stream()
    ceil_gbs = measure_read_ceiling(ntx, stream)
    with ClockSampler(local) as clk:
        rows_out, single, further = gemv_sweep(ntx, stream, peak, peak_kind, ceil_gbs)
    tiled = [r for r in rows_out if r["layout"] == "tiled"]
    tot_b = sum(r["bytes_per_launch"] for r in tiled)
    tot_us = sum(r["us"] for r in tiled)
    v = tot_b / (tot_us * 1e-6) / 1e9
    top = max(tiled, key=lambda r: r["bytes_per_launch"])
    line = {"metric": "quantized GEMV HBM GB/s", "value": v, "unit": "GB/s", "n_gpus": world, "steps": 5,
            "warmup": 1, "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": DTYPE,
            "data": "synthetic (seeded random blocks, x ~ N(0,1))", "config": config, "clocks": clk.summary(),
            "gpu_launches": 48 * 5 * (len(rows_out) + 2 + len(further)),
            "roofline": {"bound": "hbm", "kernel": "qmma_kernel (tiled Q4_0 / Q4_K, all sweep shapes, one launch each)",
                         "achieved": v, "peak": peak, "peak_kind": peak_kind, "unit": "GB/s", "frac": v / peak,
                         "traffic": None, "frac_of_read_ceiling": v / ceil_gbs,
                         "largest_shape": {"shape": f"{top['format']}:{top['rows']}x{top['cols']}",
                                           "gbs": top["gbs"]}},
            "read_ceiling": {"gbs": ceil_gbs}, "sweep": rows_out, "gemv_q8_0_4096x4096": single,
            "further_formats": further}
    print_line(line)


def profile_step_gemv(args, spec):
    """The step's fused GEMV kinds, one launch each, after `warmup` decode steps of a
    (shortened) model: the case that profiler captures of the fused instances run."""
    import torch
    import quantized_weight_gemv_block_b200 as ntx
    from synth.device_model import DeviceModel
    model = DeviceModel(spec)
    logits = torch.empty(spec.vocab, dtype=torch.float32, device="cuda")
    for _ in range(args.warmup):
        ntx.ntx_decode_step(model.handle, spec.token(), spec.n_prefill, logits)
    torch.cuda.synchronize()
    for name, kind, *_ in gemv_kinds(spec):
        ntx.ntx_model_replay_gemv(model.handle, kind, 1, logits)
        torch.cuda.synchronize()
        print(json.dumps({"profiled": name}), flush=True)
    model.close()


if __name__ == "__main__":
    main()
