"""Throughput of the compressed-expert routed MoE layer on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]

One step = one forward of the layer (route/bucket, gate/up + SwiGLU, down +
weighted combine, final cast) over one batch of synthetic tokens, with the
weights and the step's inputs already resident in HBM.  The default workload
is the single-token MXFP4 decode of the MiMo-shaped layer (hidden 4096,
inter 2048, 256 experts, top-8).  Every rank runs its own replica on its own
tokens (the path partitions by batch; no collective on the data path), so
``value`` is the total over ranks and ``scaling`` is "weak".

Rank 0 prints one JSON line.  ``--impl reference`` times the oracle (the f64
CPU restatement) on the host cores instead, on a bounded sample per step.
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

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import synth  # noqa: E402

PEAKS_FILE = os.path.join(ROOT, "MEASURED_PEAKS.json")
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}

# DRAM traffic (dram__bytes_read.sum + dram__bytes_write.sum) of the dominant
# kernel per launch, from one ncu capture of the named source (summary under
# profiles/); reported only while that source is byte-identical, else null.
NCU_TRAFFIC = {
    "decode_mxfp4": (("bit_quantized_moe_routed_b200/csrc/decode_mx.cu",
                      "bit_quantized_moe_routed_b200/csrc/async.cuh",
                      "bit_quantized_moe_routed_b200/csrc/decode_common.cuh",
                      "bit_quantized_moe_routed_b200/csrc/internal.cuh",
                      "include/moeq.h"),
                     "0cca0e038c0ed780604c13d445697ac9d59ca7bc78d4644098ff1218d86fd098",
                     107049216.0 + 358144.0, "profiles/dec_fused_mx_decode_mxfp4.md"),
}


def ncu_traffic(workload):
    """(bytes per launch, summary file) while the kernel's sources (its file and
    the headers it includes, hashed in order) are those that were profiled."""
    import hashlib
    ent = NCU_TRAFFIC.get(workload)
    if ent is None:
        return None, None
    srcs, sha, traffic, summary = ent
    h = hashlib.sha256()
    try:
        for src in srcs:
            with open(os.path.join(os.path.dirname(os.path.abspath(__file__)), src), "rb") as f:
                h.update(f.read())
    except OSError:
        return None, None
    return (traffic, summary) if h.hexdigest() == sha else (None, None)


# workload -> (config name, overrides)
WORKLOADS = {
    "decode_mxfp4": ("decode_mxfp4", {}),
    "decode_mxfp4_t8": ("decode_mxfp4", dict(T=8)),
    "decode_vq_t1": ("decode_vq", dict(T=1)),
    "decode_vq_t4": ("decode_vq", dict(T=4)),
    "decode_vq_t8": ("decode_vq", dict(T=8)),
    "decode_vq_t1_r0": ("decode_vq", dict(T=1, fmt="vq13")),
    "decode_gvq1_t1": ("decode_vq", dict(T=1, fmt="gvq1r8")),
    "decode_gvq1_t8": ("decode_vq", dict(T=8, fmt="gvq1r8")),
    "decode_vq_t8_r0": ("decode_vq", dict(T=8, fmt="vq13")),
    "prefill_mxfp4_zipf": ("prefill_mxfp4_zipf", {}),
    "prefill_vq_overflow": ("prefill_vq_overflow", {}),
    # reduced layers (64 experts, 512 tokens; under 2 GB on the device) for
    # counter captures of the tensor-core kernels; not bench lines
    "prefill_mxfp4_zipf_e64_t512": ("prefill_mxfp4_zipf", dict(E=64, T=512)),
    "prefill_vq_overflow_e64_t512": ("prefill_vq_overflow", dict(E=64, T=512)),
    "prefill_gvq1_overflow": ("prefill_vq_overflow", dict(fmt="gvq1r8")),
}


def workload_cfg(name):
    base, over = WORKLOADS[name]
    return synth.get_cfg(base, **over)


def is_decode(cfg):
    return cfg.T <= 8


# ------------------------------------------------------------------ algorithmic work

def proj_bytes(cfg, p):
    """Compressed bytes of one expert's projection p."""
    N, K = cfg.shape(p)
    if cfg.fmt == "mxfp4":
        return N * (K // 2 + K // 32)
    if cfg.fmt.startswith("gvq1"):
        b = N * (synth.gvq1_code_row_bytes(K) + K // 64)   # 12-bit stream + bit-12 plane: 13 bits per 8 weights
    else:
        b = N * synth.idx13_row_bytes(K)
    if cfg.fmt in ("vq13r8", "gvq1r8"):
        b += N * (K // 8)
    if cfg.gains:
        b += 2 * N
    return b


def book_bytes(cfg):
    if cfg.fmt == "mxfp4":
        return 0
    if cfg.fmt.startswith("gvq1"):   # 1-byte entries
        return 8192 * 8 + (256 * 8 if cfg.fmt == "gvq1r8" else 0)
    return 8192 * 16 + (256 * 16 if cfg.fmt == "vq13r8" else 0)


def flops(cfg, n_routes):
    return 2 * n_routes * 3 * cfg.H * cfg.I


# ------------------------------------------------------------------ inputs

def step_inputs(cfg, n_steps, seed=0):
    """Per-step routings and activations.  Single-token decode rotates 32
    disjoint expert sets so no expert's weights are reused within 32 steps
    (3.4 GB of MXFP4 weights stream between reuses: larger than L2);
    multi-token decode draws a fresh routing per step; prefill reuses one
    batch (each step streams 2-3.4 GB of weights, larger than L2)."""
    if cfg.T == 1:
        ids, w = synth.gen_disjoint_routing_schedule(cfg, n_steps, seed=seed)
        xs = np.stack([synth.gen_activations(cfg, seed=seed + 1 + i) for i in range(min(n_steps, 64))])
        xs = xs[np.arange(n_steps) % len(xs)]
        how = "inputs larger than L2: 32 disjoint expert sets rotate, a set recurs after 31 others"
    elif is_decode(cfg):
        ids = np.empty((n_steps, cfg.T, cfg.k), np.int32)
        w = np.empty((n_steps, cfg.T, cfg.k), np.float32)
        xs = []
        for i in range(n_steps):
            ids[i], w[i] = synth.gen_routing(cfg, seed=seed + 1 + i)
            xs.append(synth.gen_activations(cfg, seed=seed + 1 + i))
        xs = np.stack(xs)
        how = "inputs larger than L2: a fresh routing per step (~30-60 experts, 150-470 MB of weights)"
    else:
        i0, w0 = synth.gen_routing(cfg, seed=seed)
        x0 = synth.gen_activations(cfg, seed=seed)
        ids = np.broadcast_to(i0, (n_steps,) + i0.shape)
        w = np.broadcast_to(w0, (n_steps,) + w0.shape)
        xs = np.broadcast_to(x0, (n_steps,) + x0.shape)
        how = "inputs larger than L2: every step streams all routed experts' weights (GBs)"
    return xs, ids, w, how


# ------------------------------------------------------------------ clocks

CLOCK_FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
                "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
                "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")


class ClockSampler:
    def __init__(self, gpu_index):
        self.gpu = gpu_index
        self.proc = None
        # the raw samples go to MOEQ_CLOCKS_DIR when set, else the temp directory
        out_dir = os.environ.get("MOEQ_CLOCKS_DIR") or tempfile.gettempdir()
        self.path = os.path.join(out_dir, f"moeq_clocks_rank{gpu_index}_{os.getpid()}.csv")

    def start(self):
        try:
            self.f = open(self.path, "w")
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={CLOCK_FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=self.f, stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.f.close()
        sm, smax, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in open(self.path):
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                smax.append(float(parts[2]))
            except ValueError:
                continue
            for n, v in zip(names, parts[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(smax), "reasons": sorted(reasons),
                "samples": len(sm)}


# ------------------------------------------------------------------ reference arm (the oracle)

def run_reference(args, cfg):
    import oracle
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    L = synth.gen_layer(cfg)
    n_total = args.warmup + args.steps
    xs, ids, w, how = step_inputs(cfg, n_total)
    # size each step's sample so the whole run stays within ~150 s of CPU time
    probe_t = time.perf_counter()
    oracle.forward(L, xs[0][:1], ids[0][:1], w[0][:1])
    per_token = time.perf_counter() - probe_t
    budget = 150.0 / n_total
    tok_per_step = int(max(1, min(cfg.T, budget // max(per_token, 1e-6))))
    times = []
    for i in range(n_total):
        tok = np.arange(tok_per_step, dtype=np.int32) + (i * tok_per_step) % max(1, cfg.T - tok_per_step + 1)
        tok = tok % cfg.T
        t0 = time.perf_counter()
        oracle.forward(L, xs[i], ids[i], w[i], tokens=tok)
        dt = time.perf_counter() - t0
        if i >= args.warmup:
            times.append(dt)
    total = sum(times)
    value = tok_per_step * args.steps / total
    sample = f"{tok_per_step} of {cfg.T} tokens per step (all their routes), steps {args.steps}"
    line = {
        "impl": "reference", "metric": "MoE-layer tokens/s", "value": value, "unit": "tokens/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1000 * total / args.steps, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": config_obj(args, cfg, how),
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": oracle.num_threads(), "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def reduce_times(ms, e2e_s, world, dev):
    """The timed regions' durations, maximised over the ranks (every rank ran
    the same steps on its own GPU: replicas, no collective in the data path)."""
    if world <= 1:
        return ms, e2e_s
    import torch
    import torch.distributed as dist
    tt = torch.tensor([ms, e2e_s], device=dev, dtype=torch.float64)
    dist.all_reduce(tt, op=dist.ReduceOp.MAX)
    return float(tt[0]), float(tt[1])


def job_tokens_per_s(world, tokens_per_step, steps, ms):
    """Whole-job throughput: the tokens all ranks processed over the slowest rank's time."""
    return world * tokens_per_step * steps / (ms / 1e3)


def config_obj(args, cfg, how):
    return {"workload": args.workload, "hidden": cfg.H, "inter": cfg.I, "experts": cfg.E, "top_k": cfg.k,
            "tokens_per_step": cfg.T, "format": cfg.fmt, "act": cfg.act, "routing": cfg.routing,
            "seed": 0, "l2": how, "parallelism": f"replicas x{args.gpus} (one per GPU, no collective)"}


# ------------------------------------------------------------------ cpu baseline (our arm)

def cpu_baseline(cfg, L, xs, ids, w, seconds=12.0):
    import oracle
    done_tok, t_used, i = 0, 0.0, 0
    per_call = max(1, min(cfg.T, 2))
    while t_used < seconds and i < 10000:
        tok = (np.arange(per_call, dtype=np.int32) + i * per_call) % cfg.T
        t0 = time.perf_counter()
        oracle.forward(L, xs[i % len(xs)], ids[i % len(ids)], w[i % len(w)], tokens=tok)
        t_used += time.perf_counter() - t0
        done_tok += per_call
        i += 1
    return {"value": done_tok / t_used, "unit": "tokens/s", "cores": oracle.num_threads(), "kind": "oracle",
            "sample": f"{done_tok} tokens ({i} calls of {per_call} token(s) with all their routes), "
                      f"{t_used:.1f} s on the host"}


# ------------------------------------------------------------------ our arm

# Workloads the default run times after the headline one, one layer at a
# time (each layer is freed before the next is built): the prefill
# micro-batches and the VQ decode batch sizes.
EXTRA_WORKLOADS = ("decode_mxfp4_t8", "prefill_mxfp4_zipf", "prefill_vq_overflow", "prefill_gvq1_overflow",
                   "decode_vq_t1", "decode_vq_t4", "decode_vq_t8", "decode_gvq1_t1", "decode_gvq1_t8")


def load_peaks():
    if os.path.exists(PEAKS_FILE):
        return json.load(open(PEAKS_FILE)), "measured"
    return FALLBACK_PEAKS, "fallback"


def gather_roofline(cfg, d_mean, launch_ms, peaks):
    """The shared-memory bound of a VQ decode gate/up launch: the codeword
    bytes it gathers from the resident books (per 8 weights one base entry,
    plus one residual entry with R8; 16-byte bf16 entries for VQ13, 8-byte
    E4M3 entries for GVQ1) over the launch's duration, against the shared-
    memory bandwidth of all SMs (148 x 128 bytes per clock at the maximum SM
    clock)."""
    entry = 8 if cfg.fmt.startswith("gvq1") else 16
    per_vec = entry * (2 if cfg.fmt.endswith("r8") else 1)
    nbytes = d_mean * 2 * cfg.I * (cfg.H // 8) * per_vec
    achieved = nbytes / (launch_ms / 1e3) / 1e9
    peak = 148 * 128 * float(peaks.get("sm_max_mhz", 1965.0)) * 1e6 / 1e9
    return {"bound": "shared-memory gathers", "achieved": achieved, "peak": peak, "unit": "GB/s",
            "frac": achieved / peak, "per_launch_bytes": nbytes,
            "per_unit": f"{per_vec} gathered bytes per 8 weights of gate and up",
            "peak_source": "derived: 148 SMs x 128 B per clock x sm_max_mhz"}


def roofline(cfg, workload, ids_h, warmup, n_total, launch_ms, ms_step, peaks, peak_src, phase_how):
    """The dominant kernel's roofline and whole-step figures.

    Decode: algorithmic bytes = distinct experts per step x compressed bytes
    per expert of the projections the kernel streams (all three for the
    one-launch MXFP4 step; gate+up, + codebooks, for VQ), against the
    measured HBM copy bandwidth.  Prefill: 2 x routes x 2 x H x I flop, against the measured
    burst bf16 GEMM rate (the kernel runs for milliseconds inside a
    sub-second graph, not under a seconds-long power-capped load)."""
    n_steps = n_total - warmup
    if is_decode(cfg):
        d_mean = float(np.mean([len(np.unique(ids_h[i][(ids_h[i] >= 0) & (ids_h[i] < cfg.E)]))
                                for i in range(warmup, n_total)]))
        if cfg.fmt == "mxfp4":
            # one kernel does the whole step: its bytes are all three
            # projections, and its average duration is the step's device time
            # over the K replayed launches (gaps between launches included)
            kernel = "decode step (one launch: routing, gate/up + SwiGLU, down, combine)"
            bytes_k = d_mean * sum(proj_bytes(cfg, p) for p in range(3))
            per_unit = "compressed gate+up+down bytes of one expert"
            launch_ms = ms_step
            phase_how = "one launch per step: CUDA events around the K replayed steps, divided by K"
        else:
            kernel = "gate/up + SwiGLU"
            bytes_k = d_mean * (proj_bytes(cfg, 0) + proj_bytes(cfg, 1)) + book_bytes(cfg)
            per_unit = "compressed gate+up bytes of one expert (+ codebooks once per launch)"
        achieved = bytes_k / (launch_ms / 1e3) / 1e9
        peak = float(peaks["hbm_gbs"])
        traffic, traffic_src = ncu_traffic(workload)
        roof = {"kernel": kernel, "bound": "hbm", "achieved": achieved, "peak": peak,
                "unit": "GB/s", "frac": achieved / peak, "traffic": traffic,
                "peak_source": f"{peak_src} hbm_gbs", "per_launch_bytes": bytes_k,
                "per_unit": per_unit, "units_per_launch": d_mean, "launch_ms": launch_ms, "timing": phase_how}
        if cfg.fmt != "mxfp4":
            roof["gather"] = gather_roofline(cfg, d_mean, launch_ms, peaks)
        if traffic_src:
            roof["traffic_source"] = traffic_src
        step_bytes = d_mean * sum(proj_bytes(cfg, p) for p in range(3)) + book_bytes(cfg)
        extra = {"step_weight_gbs": step_bytes / (ms_step / 1e3) / 1e9,
                 "step_hbm_frac": step_bytes / (ms_step / 1e3) / 1e9 / peak}
    else:
        n_routes = int(((ids_h[warmup:] >= 0) & (ids_h[warmup:] < cfg.E)).sum()) / n_steps
        fl_gu = 2 * n_routes * 2 * cfg.H * cfg.I
        achieved = fl_gu / (launch_ms / 1e3) / 1e12
        peak = float(peaks["bf16_tflops"])
        traffic, traffic_src = ncu_traffic(workload)
        roof = {"kernel": "gate/up + SwiGLU", "bound": "tensor", "achieved": achieved, "peak": peak,
                "unit": "TFLOP/s", "frac": achieved / peak, "traffic": traffic,
                "peak_source": f"{peak_src} bf16_tflops (burst)", "per_launch_flops": fl_gu,
                "per_unit": "2 x 2 x H x I flop per route", "units_per_launch": n_routes,
                "launch_ms": launch_ms, "timing": phase_how}
        if traffic_src:
            roof["traffic_source"] = traffic_src
        extra = {"step_tflops": flops(cfg, n_routes) / (ms_step / 1e3) / 1e12,
                 "step_tensor_frac": flops(cfg, n_routes) / (ms_step / 1e3) / 1e12 / peak}
    return roof, extra


def measure(workload, steps, warmup, world, rank, local, barrier, cpu_seconds, with_cpu):
    """Time `steps` forwards of one workload (after `warmup` eager ones) as one
    replayed CUDA graph, then the per-phase durations, then the host-buffer
    entry point.  Returns this rank's figures; the caller reduces over ranks."""
    import torch
    from bit_quantized_moe_routed_b200 import moeq

    cfg = workload_cfg(workload)
    L = synth.gen_layer(cfg)
    lay = moeq.Layer(cfg.H, cfg.I, cfg.E, cfg.k, cfg.T, cfg.fmt, cfg.act, device=local)
    lay.upload(L)
    n_total = warmup + steps
    xs_h, ids_h, w_h, how = step_inputs(cfg, n_total, seed=rank)
    dev = torch.device("cuda", local)
    to_x = (lambda a: torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16)) \
        if cfg.act == "bf16" else (lambda a: torch.from_numpy(np.ascontiguousarray(a)))
    uniq = 1 if not is_decode(cfg) else n_total
    xs = to_x(xs_h[:uniq]).to(dev)
    ids = torch.from_numpy(np.ascontiguousarray(ids_h[:uniq])).to(dev)
    ws = torch.from_numpy(np.ascontiguousarray(w_h[:uniq])).to(dev)
    outs = torch.empty((uniq, cfg.T, cfg.H), dtype=xs.dtype, device=dev)

    def step(i):
        j = i % uniq
        lay.forward(xs[j], ids[j], ws[j], out=outs[j])

    # warm-up: W eager steps
    l0 = lay.kernel_launches()
    for i in range(warmup):
        step(i)
    torch.cuda.synchronize()
    launches_per_step = (lay.kernel_launches() - l0) // warmup

    # capture the K timed steps as one CUDA graph
    cap = torch.cuda.Stream(device=dev)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=cap):
        for i in range(warmup, n_total):
            step(i)
    g.replay()                      # untimed: graph upload
    torch.cuda.synchronize()

    # clock soak (~1 s of the same work), then the timed replay
    sampler = ClockSampler(local)
    sampler.start()
    t_end = time.time() + 1.0
    while time.time() < t_end:
        g.replay()
        torch.cuda.synchronize()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    barrier()
    torch.cuda.synchronize()
    # CUDAGraph.replay launches on the current stream: time it there
    e0.record()
    g.replay()
    e1.record()
    torch.cuda.synchronize()
    barrier()
    ms = e0.elapsed_time(e1)
    for _ in range(3):
        g.replay()
    torch.cuda.synchronize()
    clocks = sampler.stop()

    # per-phase kernel durations over the same K steps (a second graph with
    # event-record nodes between the kernels, on the launching stream)
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(5)] for _ in range(steps)]
    for row in ev:              # torch creates the CUDA event at its first record
        for e in row:
            e.record()
    torch.cuda.synchronize()
    g2 = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g2, stream=cap):
        for n, i in enumerate(range(warmup, n_total)):
            j = i % uniq
            lay.forward_profiled(xs[j], ids[j], ws[j], outs[j], ev[n])
    g2.replay()
    torch.cuda.synchronize()
    g2.replay()
    torch.cuda.synchronize()
    phase_ms = [sum(ev[n][p].elapsed_time(ev[n][p + 1]) for n in range(steps)) / steps for p in range(4)]
    phase_how = "event-record nodes between the kernels of a replayed graph of the same K steps"

    # end to end through the host-buffer entry point (pinned host memory)
    xh = torch.from_numpy(np.ascontiguousarray(xs_h[0])).pin_memory()
    ih = torch.from_numpy(np.ascontiguousarray(ids_h[0])).pin_memory()
    wh = torch.from_numpy(np.ascontiguousarray(w_h[0])).pin_memory()
    oh = torch.empty_like(xh).pin_memory()
    h_bytes = xh.numel() * xh.element_size() + ih.numel() * 4 + wh.numel() * 4
    d_bytes = oh.numel() * oh.element_size()
    e2e_steps = min(steps, 200)
    for _ in range(3):
        lay.forward_host_ptr(xh.data_ptr(), ih.data_ptr(), wh.data_ptr(), cfg.T, oh.data_ptr())
    barrier()
    t0 = time.perf_counter()
    for _ in range(e2e_steps):
        lay.forward_host_ptr(xh.data_ptr(), ih.data_ptr(), wh.data_ptr(), cfg.T, oh.data_ptr())
    e2e_s = time.perf_counter() - t0
    status = lay.status()
    del g, g2
    lay.close()
    res = {"cfg": cfg, "how": how, "ms": ms, "e2e_s": e2e_s, "e2e_steps": e2e_steps, "phase_ms": phase_ms,
           "phase_how": phase_how, "launches_per_step": launches_per_step, "clocks": clocks,
           "h_bytes": h_bytes, "d_bytes": d_bytes, "ids_h": ids_h, "status": status}
    if with_cpu and rank == 0:
        res["cpu_baseline"] = cpu_baseline(cfg, L, xs_h, ids_h, w_h, seconds=cpu_seconds)
    return res


# f32 FMA peak of the CUDA cores: 148 SMs x 128 FP32 lanes x 2 flop x 1.965 GHz (the recipe's unit
# counts and maximum SM clock), for kernels bound by plain ALU arithmetic
ALU_F32_TFLOPS = 148 * 128 * 2 * 1.965e9 / 1e12


def time_graph(fn, steps, warmup, dev):
    """Device time (ms) of `steps` calls of fn captured in one CUDA graph,
    after `warmup` eager calls; CUDA events on the replaying stream."""
    import torch
    for _ in range(warmup):
        fn()
    torch.cuda.synchronize()
    cap = torch.cuda.Stream(device=dev)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=cap):
        for _ in range(steps):
            fn()
    g.replay()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    g.replay()
    e1.record()
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1)
    del g
    return ms


def measure_router(T, steps, warmup, local, peaks, peak_src):
    """The router kernel (moeq_router, sigmoid weights) on the MiMo shape:
    tokens/s, and its roofline -- the f32 router matrix (E x H x 4 bytes,
    the algorithmic bytes; the kernel reads it as three bf16 terms) at one
    token, 2 T E H flop at prefill sizes."""
    import torch
    from bit_quantized_moe_routed_b200 import moeq
    cfg = synth.get_cfg("decode_mxfp4", T=T)
    dev = torch.device("cuda", local)
    lay = moeq.Layer(cfg.H, cfg.I, cfg.E, cfg.k, T, "mxfp4", "bf16", device=local)
    lay.router_upload(synth.gen_router(cfg), "sigmoid")
    x = torch.from_numpy(synth.gen_activations(cfg).view(np.int16)).view(torch.bfloat16).to(dev)
    ids = torch.empty((T, cfg.k), dtype=torch.int32, device=dev)
    w = torch.empty((T, cfg.k), dtype=torch.float32, device=dev)
    n0 = lay.kernel_launches()
    ms = time_graph(lambda: moeq.lib().moeq_router(lay.handle, moeq.C.c_void_p(x.data_ptr()), T,
                                                  moeq.C.c_void_p(ids.data_ptr()), moeq.C.c_void_p(w.data_ptr()),
                                                  None, moeq._stream_ptr(None)), steps, warmup, dev)
    launches = (lay.kernel_launches() - n0) // (steps + warmup)
    per = ms / steps / 1e3
    if T <= 8:
        nbytes = cfg.E * cfg.H * 4 + T * cfg.H * 2
        roof = {"kernel": "router (logits, top-k, weights)", "bound": "hbm", "achieved": nbytes / per / 1e9,
                "peak": float(peaks["hbm_gbs"]), "unit": "GB/s", "traffic": None,
                "per_unit": "the f32 router matrix (E x H x 4 bytes) and the step's activations",
                "peak_source": f"{peak_src} hbm_gbs"}
    else:
        fl = 2.0 * T * cfg.E * cfg.H
        roof = {"kernel": "router (logits, top-k, weights)", "bound": "tensor", "achieved": fl / per / 1e12,
                "peak": float(peaks["bf16_tflops"]), "unit": "TFLOP/s", "traffic": None,
                "per_unit": "2 x E x H flop per token (the kernel issues three bf16 MMAs per product)",
                "peak_source": f"{peak_src} bf16_tflops (burst)"}
    roof["frac"] = roof["achieved"] / roof["peak"]
    lay.close()
    return {"metric": "router tokens/s", "value": T / per, "unit": "tokens/s", "steps": steps, "warmup": warmup,
            "ms_per_step": ms / steps, "dtype": "bf16 x, f32 router", "config": {"workload": f"router_t{T}",
            "hidden": cfg.H, "experts": cfg.E, "top_k": cfg.k, "tokens_per_step": T, "score": "sigmoid"},
            "roofline": roof, "gpu_launches": int(launches * steps)}


def measure_encoder(steps, warmup, local, with_cpu):
    """The VQ encoder (moeq_vq_encode, VQ13+R8, unit column weights) on one
    MiMo expert's three matrices: weights/s, against the f32 FMA peak with
    the algorithmic flops 16 x (8192 + 256) per 8-vector (the expanded
    distance's dot product over both books)."""
    import torch
    from bit_quantized_moe_routed_b200 import moeq
    cfg = synth.get_cfg("decode_vq", E=1)
    L = synth.gen_layer(cfg, seed=7)
    dev = torch.device("cuda", local)
    rng = np.random.default_rng(7)
    mats = []
    for p in range(3):
        N, K = cfg.shape(p)
        W = torch.from_numpy(rng.normal(0.0, 0.02, size=(N, K)).astype(np.float32)).to(dev)
        mats.append((W, torch.empty((N, K * 13 // 64), dtype=torch.uint8, device=dev),
                     torch.empty((N, K // 8), dtype=torch.uint8, device=dev)))
    b13 = torch.from_numpy(L.book13.view(np.int16)).to(dev)
    b8 = torch.from_numpy(L.book8.view(np.int16)).to(dev)
    P = moeq.C.c_void_p

    def fn():
        for W, o13, o8 in mats:
            moeq.lib().moeq_vq_encode(P(W.data_ptr()), W.shape[0], W.shape[1], None, None, P(b13.data_ptr()),
                                      P(b8.data_ptr()), P(o13.data_ptr()), P(o8.data_ptr()), moeq._stream_ptr(None))
    ms = time_graph(fn, steps, warmup, dev)
    n_w = sum(W.numel() for W, _, _ in mats)
    per = ms / steps / 1e3
    fl = 16.0 * (8192 + 256) * (n_w / 8)
    roof = {"kernel": "vq_encode_kernel", "bound": "alu", "achieved": fl / per / 1e12, "peak": ALU_F32_TFLOPS,
            "unit": "TFLOP/s", "frac": fl / per / 1e12 / ALU_F32_TFLOPS, "traffic": None,
            "per_unit": "16 x (8192 + 256) flop per 8-weight vector",
            "peak_source": "derived: 148 SMs x 128 FP32 lanes x 2 flop x 1.965 GHz"}
    line = {"metric": "VQ encode weights/s", "value": n_w / per, "unit": "weights/s", "steps": steps,
            "warmup": warmup, "ms_per_step": ms / steps, "dtype": "f32", "config": {
                "workload": "vq_encode_expert", "matrices": "gate, up [2048][4096], down [4096][2048]",
                "format": "vq13r8", "weights": "N(0, 0.02^2)", "column_weights": None},
            "roofline": roof, "gpu_launches": 3 * steps}
    if with_cpu:
        import oracle.vq_encode as ve
        W0 = mats[0][0][:2].cpu().numpy()
        t0 = time.perf_counter()
        ve.encode_rows(W0, L.book13, L.book8)
        dt = time.perf_counter() - t0
        line["cpu_baseline"] = {"value": W0.size / dt, "unit": "weights/s", "cores": os.cpu_count(),
                                "kind": "oracle", "sample": f"2 rows of the gate matrix ({W0.size} weights), "
                                f"{dt:.1f} s"}
    return line


def summarize(args, workload, r, world, steps, warmup, peaks, peak_src):
    """The contract's fields for one measured workload (times already reduced over ranks)."""
    cfg = r["cfg"]
    ms_step = r["ms"] / steps
    roof, extra = roofline(cfg, workload, r["ids_h"], warmup, warmup + steps, r["phase_ms"][1], ms_step,
                           peaks, peak_src, r["phase_how"])
    a = argparse.Namespace(**vars(args))
    a.workload = workload
    line = {
        "metric": "MoE-layer tokens/s", "value": job_tokens_per_s(world, cfg.T, steps, r["ms"]),
        "unit": "tokens/s", "n_gpus": world, "steps": steps, "warmup": warmup, "ms_per_step": ms_step,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "bf16" if cfg.act == "bf16" else "f32", "data": "synthetic",
        "config": config_obj(a, cfg, r["how"]),
        "roofline": roof, "phase_ms": dict(zip(["route", "gateup", "down_combine", "cast"], r["phase_ms"])),
        "step": extra,
        "e2e": {"value": job_tokens_per_s(world, cfg.T, r["e2e_steps"], r["e2e_s"] * 1e3), "unit": "tokens/s",
                "h2d_bytes_per_step": r["h_bytes"], "d2h_bytes_per_step": r["d_bytes"], "steps": r["e2e_steps"],
                "how": "moeq_forward_host per step: pinned H2D of x/ids/w, forward, D2H of out, sync"},
        "gpu_launches": int(r["launches_per_step"] * steps),
        "clocks": r["clocks"],
        "device_status": r["status"],
    }
    if "cpu_baseline" in r:
        line["cpu_baseline"] = r["cpu_baseline"]
    return line


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--workload", default="decode_mxfp4", choices=sorted(WORKLOADS))
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-extra", action="store_true",
                    help="time only --workload (by default the prefill and VQ workloads follow the headline one)")
    ap.add_argument("--extra-steps", type=int, default=30, help="timed steps of each extra workload")
    args = ap.parse_args()
    assert args.warmup >= 3, "at least 3 warm-up steps"
    cfg = workload_cfg(args.workload)
    world = int(os.environ.get("WORLD_SIZE", "1"))
    if args.impl == "reference":
        return run_reference(args, cfg)

    import torch
    import torch.distributed as dist
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))

    def barrier():
        if world > 1:
            dist.barrier()

    peaks, peak_src = load_peaks()
    with_cpu = not args.no_cpu_baseline and world == 1
    r = measure(args.workload, args.steps, args.warmup, world, rank, local, barrier, 12.0, with_cpu)
    r["ms"], r["e2e_s"] = reduce_times(r["ms"], r["e2e_s"], world, dev)
    line = summarize(args, args.workload, r, world, args.steps, args.warmup, peaks, peak_src) if rank == 0 else None

    # The extra workloads follow the headline one; a failure in one of them is
    # reported in its entry and does not cost the headline line.
    extra = {}

    def run_extra(name, fn):
        try:
            res = fn()
        except Exception as exc:   # noqa: BLE001 -- reported, not hidden
            res = {"error": f"{type(exc).__name__}: {exc}"[:300]}
        torch.cuda.empty_cache()
        if rank == 0 and res is not None:
            extra[name] = res

    def layer_extra(name):
        rx = measure(name, args.extra_steps, args.warmup, world, rank, local, barrier, 6.0, with_cpu)
        rx["ms"], rx["e2e_s"] = reduce_times(rx["ms"], rx["e2e_s"], world, dev)
        if rank != 0:
            return None
        lx = summarize(args, name, rx, world, args.extra_steps, args.warmup, peaks, peak_src)
        for key in ("metric", "n_gpus", "higher_is_better", "scaling", "vs_baseline", "data"):
            lx.pop(key, None)
        return lx

    extra_names = () if (args.no_extra or args.workload != "decode_mxfp4") else EXTRA_WORKLOADS
    for name in extra_names:
        run_extra(name, lambda name=name: layer_extra(name))

    if extra_names:
        # the steps on either side of the layer: the router and the VQ encoder
        for T in (1, 2048):
            run_extra(f"router_t{T}", lambda T=T: measure_router(T, args.extra_steps, args.warmup, local, peaks,
                                                                  peak_src))
        run_extra("vq_encode_expert", lambda: measure_encoder(3, 3, local, with_cpu))

    if rank == 0:
        if extra:
            line["workloads"] = extra
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
