#!/usr/bin/env python
"""Throughput of the MoE-layer forward on B200, as one JSON line.

python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference] [--workload NAME]

A step is one moe_forward over one batch (route, permute, grouped GEMM 1/3 +
SwiGLU, grouped GEMM 2, combine, statistics) of the named workload, default
the Mixtral-8x7B-shaped prefill layer (T=4096, d=4096, E=8, d_ff=14336,
top-2, bf16). Inputs are seeded synthetic tensors resident in HBM; between
timed steps a 512 MiB buffer is written and then a second 512 MiB buffer is
read, so L2 holds none of the step's data and no dirty lines whose write-back
would be charged to the step (the 2.8 GB of expert weights exceed L2 anyway). Steps are timed with CUDA events on the launching
stream and summed; the job time is the max over ranks. With N > 1 every rank
is an independent data-parallel replica over its own tokens (weak scaling)
and the per-expert statistics are summed over ranks with one NCCL
all-reduce per step.

Also reported: end to end through host buffers (pinned H2D copy of x, the
forward, D2H of the output, all inside the timed region), a per-stage
breakdown, the roofline of the dominant kernel (grouped GEMM 1/3 + SwiGLU)
against the measured bf16 peak, SM clocks sampled during the timed region,
and (rank 0, N = 1) the CPU oracle timed on a bounded token sample.
--impl reference times the CPU oracle alone (this build's reference arm).
"""

from __future__ import annotations

import argparse
import datetime
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from mixture_experts_layer_62_b200 import inputs  # noqa: E402

METRIC = "MoE-layer fwd tokens/s & TFLOP/s vs bf16 peak; small-batch decode HBM GB/s"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
TRAFFIC_FILE = os.path.join(ROOT, "profiles", "traffic.json")
CSRC = os.path.join(ROOT, "mixture_experts_layer_62_b200", "csrc")
GEMM_SRC = os.path.join(CSRC, "gemm_sm100.cu")
GEMV_SRC = os.path.join(CSRC, "gemv_sm100.cu")


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as fh:
            d = json.load(fh)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def flops_per_step(cfg, rows=None):
    """Algorithmic FLOPs: 2 T k 3 d d_ff (routed) + 2 T d E (router) + shared."""
    T, d, dff, E, k, dfs = cfg["T"], cfg["d"], cfg["d_ff"], cfg["E"], cfg["k"], cfg["d_ff_shared"]
    R = T * k if rows is None else rows
    return 2.0 * R * 3 * d * dff + 2.0 * T * d * E + 2.0 * T * 3 * d * dfs


def up_flops(cfg, rows):
    return 2.0 * rows * cfg["d"] * 2 * cfg["d_ff"] + 2.0 * cfg["T"] * cfg["d"] * 2 * cfg["d_ff_shared"]


def down_flops(cfg, rows):
    return 2.0 * rows * cfg["d_ff"] * cfg["d"] + 2.0 * cfg["T"] * cfg["d_ff_shared"] * cfg["d"]


class ClockSampler:
    """nvidia-smi samples of SM clock and throttle reasons while running.

    Each sample carries nvidia-smi's own timestamp; mark() and stop() take
    the host time at the two ends of the timed region, and only the samples
    inside it are summarised (the sampler starts before the region and
    stops after it, and an idle GPU's clock says nothing about the work)."""

    FIELDS = ["timestamp", "clocks.sm", "clocks.max.sm", "power.draw", "clocks_event_reasons.hw_slowdown",
              "clocks_event_reasons.hw_thermal_slowdown", "clocks_event_reasons.sw_thermal_slowdown",
              "clocks_event_reasons.sw_power_cap"]
    REASONS = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]

    def __init__(self, gpu_index):
        self.gpu_index = gpu_index
        self.proc = None
        self.lines = []
        self.thread = None
        self.t0 = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={','.join(self.FIELDS)}", "--format=csv,noheader,nounits",
                 "-lms", "20", "-i", str(self.gpu_index)],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
            return
        self.thread = threading.Thread(target=self._read, daemon=True)
        self.thread.start()
        time.sleep(0.2)

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def mark(self):
        """The timed region starts now."""
        self.t0 = time.time()

    def stop(self):
        """Summary of the samples taken since mark() (all samples when mark()
        was not called)."""
        if self.proc is None:
            return None
        t1 = time.time()
        time.sleep(0.1)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        if self.thread:
            self.thread.join(timeout=2)
        return self.summarise(self.lines, self.t0, t1)

    @classmethod
    def summarise(cls, lines, t0=None, t1=None):
        sm, mx, reasons, outside = [], None, set(), 0
        for ln in lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) != len(cls.FIELDS):
                continue
            try:
                ts = datetime.datetime.strptime(parts[0], "%Y/%m/%d %H:%M:%S.%f").timestamp()
                clk = float(parts[1])
                mx = float(parts[2])
            except ValueError:
                continue
            if t0 is not None and not (t0 <= ts <= t1):
                outside += 1
                continue
            sm.append(clk)
            for name, val in zip(cls.REASONS, parts[4:]):
                if val.lower().startswith("active"):
                    reasons.add(name)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": mx, "reasons": [], "samples": 0,
                    "note": "no nvidia-smi sample fell inside the timed region"}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx, "reasons": sorted(reasons), "samples": len(sm)}


def gpu_index_for(local_rank):
    vis = os.environ.get("CUDA_VISIBLE_DEVICES")
    if vis:
        ids = [v.strip() for v in vis.split(",") if v.strip()]
        if local_rank < len(ids) and ids[local_rank].isdigit():
            return int(ids[local_rank])
    return local_rank


def traffic_for(kernel, workload):
    """DRAM bytes per launch from the committed ncu summary, if it still
    describes the current kernel source."""
    if not os.path.exists(TRAFFIC_FILE):
        return None
    with open(TRAFFIC_FILE) as fh:
        d = json.load(fh)
    src = GEMV_SRC if kernel.startswith("gemv") else GEMM_SRC
    src_hash = hashlib.sha256(open(src, "rb").read()).hexdigest()
    ent = d.get(kernel, {}).get(workload)
    if not ent or ent.get("source_sha256") != src_hash:
        return None
    return ent.get("dram_bytes_per_launch")


def blas_threads():
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 0) for i in threadpool_info() if i.get("user_api") == "blas"]
        if n:
            return max(n)
    except Exception:
        pass
    return os.cpu_count()


def oracle_sample(cfg, L, n_tokens, seed=0, needed_experts=None):
    """Time the CPU oracle: routing of all tokens plus the expert math of a
    seeded sample of n_tokens tokens. Every array the oracle reads is in
    float64 on the host before the clock starts (the weights of the experts
    the sample can touch, x, W_r), so the timed region holds the oracle's
    own arithmetic only, not dtype conversions. Returns (tokens, seconds,
    seconds of the routing-only pass over all tokens)."""
    from oracle import moe_oracle as O
    x = L["x"].double().cpu().numpy()
    W_r = L["W_r"].double().cpu().numpy()
    bias = None if L["bias"] is None else L["bias"].double().cpu().numpy()
    rng = np.random.default_rng(seed)
    tokens = np.sort(rng.choice(cfg["T"], size=min(n_tokens, cfg["T"]), replace=False))
    experts = range(cfg["E"]) if needed_experts is None else sorted(set(needed_experts(tokens)))

    class _Host(dict):
        # an expert the oracle's own routing picks beyond the prefetched set
        # (a near-tie) is copied on demand
        def __init__(self, W):
            super().__init__({e: W[e].double().cpu().numpy() for e in experts})
            self.W = W

        def __missing__(self, e):
            v = self[e] = self.W[e].double().cpu().numpy()
            return v

    W1, W3, W2 = _Host(L["W1"]), _Host(L["W3"]), _Host(L["W2"])
    sh = {}
    if cfg["d_ff_shared"]:
        sh = {n: L[n].double().cpu().numpy() for n in ("Ws1", "Ws3", "Ws2")}
    args = (x, W_r, W1, W3, W2, cfg["k"], cfg["cf"], bias, cfg["bias_mode"], sh.get("Ws1"), sh.get("Ws3"),
            sh.get("Ws2"))
    t0 = time.perf_counter()
    O.moe_forward(*args, tokens=np.zeros(0, dtype=np.int64))     # routing, permutation, statistics only
    t_route = time.perf_counter() - t0
    t0 = time.perf_counter()
    O.moe_forward(*args, tokens=tokens)
    dt = time.perf_counter() - t0
    return len(tokens), dt, t_route


def touched_experts(st):
    return sum(1 for c in st.counts if c > 0)


def decode_bytes(cfg, st):
    """Bytes one forward must move: every touched expert's three matrices,
    the router, x and y (the weight-read bound of small-batch decode)."""
    d, dff, E, T = cfg["d"], cfg["d_ff"], cfg["E"], cfg["T"]
    eb = 2 if cfg["dtype"] == "bf16" else 4
    b = touched_experts(st) * 3 * d * dff * eb + d * E * eb + 2 * T * d * eb
    if cfg["d_ff_shared"]:
        b += 3 * d * cfg["d_ff_shared"] * eb
    return b


def stage_bytes(cfg, rows):
    """Algorithmic bytes of the HBM-bound stages, as their stage entry points
    run them: route reads x and W_r and writes the fp32 logits, idx and
    gates; permute reads x and writes the `rows` kept rows of Xp, pos and
    row_token; combine reads those rows of O (and the shared expert's rows)
    and writes y."""
    T, d, E, k = cfg["T"], cfg["d"], cfg["E"], cfg["k"]
    eb = 2 if cfg["dtype"] == "bf16" else 4
    route = T * d * eb + d * E * eb + T * E * 4 + T * k * 8
    permute = T * d * eb + rows * d * eb + T * k * 4 + rows * 4
    combine = rows * d * eb + T * k * 8 + T * d * eb + (T * d * eb if cfg["d_ff_shared"] else 0)
    return {"route": route, "permute": permute, "combine": combine}


def hbm_stages(cfg, rows, stages_ms, peaks):
    """Achieved HBM bandwidth of route, permute and combine: their
    algorithmic bytes over their stage times (CUDA events around each stage
    entry point, L2 cleared between iterations)."""
    out = {}
    for name, b in stage_bytes(cfg, rows).items():
        ms = stages_ms.get(name)
        if not ms:
            continue
        gbs = b / (ms / 1e3) / 1e9
        out[name] = {"bytes": b, "ms": ms, "gbs": gbs, "frac": gbs / peaks["hbm_gbs"]}
    return out


KERNEL_NAMES = {
    "pair": ("tc_pair_gemm<SWIGLU> (grouped GEMM 1/3 + SwiGLU, CTA pairs)", "tc_pair_gemm_swiglu"),
    "grid_split": ("tc_grouped_gemm<SWIGLU> (grouped GEMM 1/3 + SwiGLU, small groups on their own CTAs)",
                   "tc_grouped_gemm_swiglu"),
    "single": ("tc_grouped_gemm<SWIGLU> (grouped GEMM 1/3 + SwiGLU)", "tc_grouped_gemm_swiglu"),
    "split_k": ("tc_grouped_gemm<SWIGLU> (grouped GEMM 1/3 + SwiGLU, split-K)", "tc_grouped_gemm_swiglu"),
    "interleaved": ("tc_grouped_gemm<SWIGLU> (grouped GEMM 1/3 + SwiGLU, small groups interleaved)",
                    "tc_grouped_gemm_swiglu"),
    "simt": ("simt_gemm_kernel<true> (grouped GEMM 1/3 + SwiGLU, CUDA cores)", "simt_gemm_swiglu"),
    "gemv": ("gemv_swiglu_kernel (grouped GEMM 1/3 + SwiGLU as weight-streaming GEMVs)", "gemv_swiglu"),
}


def workload_roofline(cfg, workload, stages, st, peaks, peak_src, variant="single"):
    """Roofline of the dominant kernel, grouped GEMM 1/3 + SwiGLU."""
    rows = st.rows
    up_ms = stages["expert_up"]
    down_ms = stages["expert_down"]
    fl = up_flops(cfg, rows)
    eb = 2 if cfg["dtype"] == "bf16" else 4
    n_touch = touched_experts(st)
    up_bytes = n_touch * 2 * cfg["d"] * cfg["d_ff"] * eb
    up_bytes += rows * cfg["d"] * eb + rows * cfg["d_ff"] * eb
    if cfg["d_ff_shared"]:
        up_bytes += 2 * cfg["d"] * cfg["d_ff_shared"] * eb + cfg["T"] * cfg["d"] * eb + cfg["T"] * cfg["d_ff_shared"] * eb
    t = up_ms / 1e3
    tflops, gbs = fl / t / 1e12, up_bytes / t / 1e9
    peak_tf, peak_bw = peaks["bf16_tflops"], peaks["hbm_gbs"]
    t_compute, t_memory = fl / (peak_tf * 1e12), up_bytes / (peak_bw * 1e9)
    kname, tkey = KERNEL_NAMES[variant]
    common = {"kernel": kname, "gemm_variant": variant, "ms_per_launch": up_ms,
              "flops_per_launch": fl, "bytes_per_launch": up_bytes,
              "roofline_time_ms": 1e3 * max(t_compute, t_memory),
              "frac_of_roofline_time": max(t_compute, t_memory) / t,
              "traffic": traffic_for(tkey, workload),
              "down_proj": {"ms_per_launch": down_ms, "tflops": down_flops(cfg, rows) / (down_ms / 1e3) / 1e12}}
    if t_memory > t_compute:
        return {"bound": "hbm", "achieved": gbs, "peak": peak_bw, "unit": "GB/s", "frac": gbs / peak_bw,
                "peak_source": f"{peak_src} HBM copy", **common}
    return {"bound": "tensor", "achieved": tflops, "peak": peak_tf, "unit": "TFLOP/s", "frac": tflops / peak_tf,
            "peak_source": f"{peak_src} bf16 burst",
            "frac_of_sustained": tflops / peaks.get("bf16_tflops_sustained", peak_tf), **common}


def run_reference(args, cfg, rank):
    """The reference arm: the CPU oracle as it stands, on a bounded sample of
    the workload per step; rank 0 only."""
    if rank != 0:
        return
    dev = "cuda" if torch.cuda.is_available() else "cpu"
    L = inputs.make_layer(cfg, seed=0, device="cpu", weights_device=dev)
    n = args.ref_sample
    for i in range(args.warmup):
        oracle_sample(cfg, L, n, seed=1000 + i)
    total_tok, total_t, total_route = 0, 0.0, 0.0
    for i in range(args.steps):
        nt, dt, tr = oracle_sample(cfg, L, n, seed=i)
        total_tok += nt
        total_t += dt
        total_route += tr
    value = total_tok / total_t
    cores = blas_threads()
    sample = (f"per step: routing of all {cfg['T']} tokens + expert math of {n} seeded random tokens; "
              f"routing alone {1e3 * total_route / args.steps:.0f} ms, expert math "
              f"{1e3 * (total_t - total_route) / total_tok:.1f} ms per token")
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * total_t / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic", "config": config_of(cfg, args),
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": cores, "kind": "oracle", "sample": sample,
                         "route_ms": 1e3 * total_route / args.steps,
                         "expert_ms_per_token": 1e3 * (total_t - total_route) / total_tok},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


class L2Flush:
    """Evicts L2 between timed steps: writes a 512 MiB buffer, then reads
    another 512 MiB buffer, so that L2 is left holding clean lines of an
    unrelated buffer (neither the step's data nor dirty lines whose write-back
    the next timed step would pay for)."""

    def __init__(self, dev):
        self.w = torch.empty(512 << 20, dtype=torch.uint8, device=dev)
        self.r = torch.ones(128 << 20, dtype=torch.float32, device=dev)

    def __call__(self):
        self.w.fill_(1)
        self.r.amax()


def config_of(cfg, args):
    return {"workload": args.workload, "T_per_gpu": cfg["T"], "d": cfg["d"], "d_ff": cfg["d_ff"], "E": cfg["E"],
            "k": cfg["k"], "capacity_factor": cfg["cf"], "bias_mode": cfg["bias_mode"],
            "d_ff_shared": cfg["d_ff_shared"], "global_batch_tokens": cfg["T"] * args.gpus,
            "parallelism": f"dp{args.gpus} replicas" if args.gpus > 1 else "single GPU",
            "l2": "between timed steps a 512 MiB buffer written, then another 512 MiB read (L2 left clean); "
                  "the weights read per step also exceed L2",
            "launch": "eager" if getattr(args, "no_graph", False) else "cuda_graph (captured moe_forward, replayed)",
            "pad_rows": getattr(args, "pad_rows", 0)}


def launches_per_forward(cfg, pad_rows=0, train=0):
    """Kernels one moe_forward launches, from the library's own choice of
    router (moe_router_variant)."""
    if cfg["T"] == 0:
        return 1
    import mixture_experts_layer_62_b200 as moe
    p = moe.problem(cfg["T"], cfg["d"], cfg["d_ff"], cfg["E"], cfg["k"], cfg.get("cf", 0.0), cfg["dtype"],
                    cfg.get("bias_mode", 0), cfg["d_ff_shared"], pad_rows=pad_rows, train=train)
    router = moe.router_variant(p)
    if router == "small":
        # partial router logits, routing finisher, grouped GEMM 1/3, grouped GEMM 2, combine
        return 5
    # router: one fused kernel (logits and selection), or transpose W_r,
    # logits (tensor or CUDA cores), select; then scan, permute+gather,
    # (padding fill,) grouped GEMM 1/3, grouped GEMM 2, combine
    return (6 if router.startswith("fused") else 8) + (1 if pad_rows else 0)


def time_steps(step, steps, warmup, dev, stream, flush, barrier, local_rank):
    """Total device milliseconds of `steps` calls of step(): `warmup` untimed
    calls, then each timed call bracketed by CUDA events on the launching
    stream, with an L2 flush before it (outside the events); barrier and
    synchronize on both sides. SM clocks are sampled during the timed calls."""
    for _ in range(warmup):
        step()
    torch.cuda.synchronize(dev)
    barrier()
    sampler = ClockSampler(gpu_index_for(local_rank))
    sampler.start()
    torch.cuda.synchronize(dev)
    barrier()
    sampler.mark()
    evs = []
    for _ in range(steps):
        flush()
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        step()
        e1.record(stream)
        evs.append((e0, e1))
    torch.cuda.synchronize(dev)
    barrier()
    clocks = sampler.stop()
    return sum(a.elapsed_time(b) for a, b in evs), clocks


def pass_roofline(cfg, st, ms_per_step, peaks):
    """Roofline of the whole forward: the slower of its FLOPs (executed rows)
    at the bf16 peak and its compulsory bytes (every touched expert's
    weights, the router, x and y) at the HBM peak, over the measured step."""
    fl = flops_per_step(cfg, st.rows)
    by = decode_bytes(cfg, st)
    t_c = fl / (peaks["bf16_tflops"] * 1e12)
    t_m = by / (peaks["hbm_gbs"] * 1e9)
    t = ms_per_step / 1e3
    return {"bound": "tensor" if t_c >= t_m else "hbm", "flops": fl, "bytes": by,
            "roofline_ms": 1e3 * max(t_c, t_m), "frac": max(t_c, t_m) / t,
            "tflops": fl / t / 1e12, "hbm_gbs": by / t / 1e9}


# The other configurations of the benchmark, measured in the same process
# after the headline workload (one GPU): the decode sweep's batch sizes that
# carry the HBM target, the DeepSeek-V3-shaped layer and the skewed layer
# with capacity drops.
EXTRA_WORKLOADS = ("decode_t1", "decode_t2", "decode_t4", "decode_t8", "skewed_capacity", "deepseek_v3")


def measure_extra(name, args, moe, dev, stream, flush, peaks, peak_src, weight_cache):
    """One more workload, timed like the headline (graph replay, L2 flushed
    between steps, CUDA events); returns its summary."""
    cfg = inputs.workload(name)
    key = (cfg["d"], cfg["d_ff"], cfg["E"], cfg["dtype"], cfg["d_ff_shared"])
    if key in weight_cache:
        # same shapes and seed: the same weights, x and W_r drawn for this T
        L = dict(weight_cache[key])
        x, W_r, bias = inputs.make_routing_inputs(cfg, seed=0)
        L.update(x=x.to(dev), W_r=W_r.to(dev), bias=None if bias is None else bias.to(dev))
    else:
        weight_cache.clear()
        torch.cuda.empty_cache()
        L = inputs.make_layer(cfg, seed=0, device="cpu", weights_device=dev)
        L = {k_: (v.to(dev) if isinstance(v, torch.Tensor) else v) for k_, v in L.items()}
        weight_cache[key] = {n: L[n] for n in ("W1", "W3", "W2", "Ws1", "Ws3", "Ws2")}
    p = moe.problem(cfg["T"], cfg["d"], cfg["d_ff"], cfg["E"], cfg["k"], cfg["cf"], cfg["dtype"], cfg["bias_mode"],
                    cfg["d_ff_shared"])
    layer = moe.MoELayer(p, L["W_r"], L["W1"], L["W3"], L["W2"], bias=L["bias"], Ws1=L["Ws1"], Ws3=L["Ws3"],
                         Ws2=L["Ws2"])
    x = L["x"]
    for _ in range(args.warmup):
        layer(x)
    torch.cuda.synchronize(dev)
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        layer(x)
    torch.cuda.synchronize(dev)
    # at least about 100 ms of timed steps, so that the 20 ms clock samples
    # fall inside the timed region even for a decode step of a tenth of a ms
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(3):
        graph.replay()
    e1.record(stream)
    torch.cuda.synchronize(dev)
    est_ms = max(e0.elapsed_time(e1) / 3, 1e-3)
    steps = min(2000, max(args.steps, int(math.ceil(100.0 / est_ms))))
    total_ms, clocks = time_steps(graph.replay, steps, args.warmup, dev, stream, flush, lambda: None, 0)
    st = layer.read_stats()
    if st.status != moe.MOE_OK:
        raise SystemExit(f"{name}: device status {st.status}: {moe.error_string(st.status)}")
    ms = total_ms / steps
    stages = breakdown(moe, p, cfg, L, dev, stream, flush, iters=max(3, min(10, args.steps)))
    out = {"ms_per_step": ms, "steps": steps, "tokens_per_s": cfg["T"] / (ms / 1e3), "T": cfg["T"],
           "roofline": workload_roofline(cfg, name, stages, st, peaks, peak_src, moe.gemm_variant(p)),
           "router_variant": moe.router_variant(p),
           "pass_roofline": pass_roofline(cfg, st, ms, peaks), "stages_ms": stages,
           "hbm_stages": hbm_stages(cfg, st.rows, stages, peaks), "clocks": clocks,
           "routing": {"rows": st.rows, "dropped": st.dropped, "capacity": st.capacity, "l_aux": st.l_aux,
                       "max_over_mean": st.max_over_mean, "experts_touched": touched_experts(st),
                       "counts": st.counts if cfg["E"] <= 16 else None,
                       "kept": st.kept if cfg["E"] <= 16 else None},
           "gpu_launches": launches_per_forward(cfg) * steps}
    if cfg["T"] <= 64:
        out["forward_hbm_gbs"] = decode_bytes(cfg, st) / (ms / 1e3) / 1e9
        out["forward_hbm_frac"] = out["forward_hbm_gbs"] / peaks["hbm_gbs"]
    del graph, layer
    return out


def main():
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=100)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="mixtral_prefill")
    ap.add_argument("--cpu-sample", type=int, default=1024, help="tokens of the timed CPU-oracle sample")
    ap.add_argument("--ref-sample", type=int, default=256, help="tokens per step of the reference arm")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-extra", action="store_true",
                    help="measure the headline workload only (by default one GPU also measures " +
                         ", ".join(EXTRA_WORKLOADS) + ")")
    ap.add_argument("--no-graph", action="store_true", help="launch the forward eagerly in the timed loop")
    ap.add_argument("--train", action="store_true",
                    help="time a training step (forward + backward) instead of the forward")
    ap.add_argument("--pad-rows", type=int, default=0, choices=[0, 64, 128],
                    help="pad every expert's rows to a multiple of this (the MegaBlocks layout), for comparison")
    args = ap.parse_args()
    if args.warmup < 3:
        raise SystemExit("--warmup must be >= 3")

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if world != args.gpus:
        if world == 1 and args.gpus > 1:
            raise SystemExit("--gpus N > 1 must be launched with torch.distributed.run (one rank per GPU)")
    cfg = inputs.workload(args.workload)

    if args.impl == "reference":
        run_reference(args, cfg, rank)
        return

    import mixture_experts_layer_62_b200 as moe
    import torch.distributed as dist
    from mixture_experts_layer_62_b200 import parallel
    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    if world > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=120), device_id=dev)

    # each rank: its own tokens (seed = rank), the same weights (seed 0)
    L = inputs.make_layer(cfg, seed=0, device="cpu", weights_device=dev)
    if rank > 0:
        x_r, _, _ = inputs.make_routing_inputs(cfg, seed=rank)
        L["x"] = x_r
    L = {k_: (v.to(dev) if isinstance(v, torch.Tensor) else v) for k_, v in L.items()}
    p = moe.problem(cfg["T"], cfg["d"], cfg["d_ff"], cfg["E"], cfg["k"], cfg["cf"], cfg["dtype"], cfg["bias_mode"],
                    cfg["d_ff_shared"], pad_rows=args.pad_rows)
    layer = moe.MoELayer(p, L["W_r"], L["W1"], L["W3"], L["W2"], bias=L["bias"], Ws1=L["Ws1"], Ws3=L["Ws3"],
                         Ws2=L["Ws2"])
    x = L["x"]
    E = cfg["E"]
    flush = L2Flush(dev)
    stream = torch.cuda.current_stream(dev)
    if args.train:
        if world > 1:
            raise SystemExit("--train runs on one GPU")
        run_train(args, cfg, moe, L, dev, stream, flush)
        return

    # the forward is captured once in a CUDA graph and replayed (the library's
    # launches are asynchronous and allocation-free, so they capture as is)
    for _ in range(args.warmup):
        layer(x)
    torch.cuda.synchronize(dev)
    fwd = (lambda: layer(x))
    if not args.no_graph:
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph):
            layer(x)
        torch.cuda.synchronize(dev)
        fwd = graph.replay

    def step():
        fwd()
        if world > 1:
            # the one exchange of data-parallel replicas: global load statistics
            v = parallel._local_vector(layer.stats, E, cfg["T"])
            dist.all_reduce(v)

    def barrier():
        if world > 1:
            dist.barrier()

    # ---- device-timed steps ----
    total_ms, clocks = time_steps(step, args.steps, args.warmup, dev, stream, flush, barrier, local_rank)
    t = torch.tensor([total_ms], dtype=torch.float64, device=dev)
    if world > 1:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    job_ms = float(t.item())
    st = layer.read_stats()
    gst = parallel.global_stats(layer.stats, E, cfg["k"], cfg["T"]) if world > 1 else None
    if st.status != moe.MOE_OK:
        raise SystemExit(f"device status {st.status}: {moe.error_string(st.status)}")
    tokens_total = cfg["T"] * world * args.steps
    value = tokens_total / (job_ms / 1e3)
    ms_per_step = job_ms / args.steps
    rows = st.rows
    tflops = flops_per_step(cfg, rows) * world * args.steps / (job_ms / 1e3) / 1e12

    # ---- per-stage breakdown (stage entry points, events between) ----
    # (right after the timed steps, under the same flush-separated load: the
    # end-to-end loop below keeps the GPU busy without gaps, and under the
    # power cap the clock is lower after it)
    stages = breakdown(moe, p, cfg, L, dev, stream, flush, iters=max(3, min(10, args.steps)))

    # ---- end to end through host buffers ----
    x_host = x.cpu().pin_memory()
    e2e_sampler = ClockSampler(gpu_index_for(local_rank))
    e2e_sampler.start()
    e2e_ms = e2e_pipelined(layer, x_host, dev, stream, args.steps, before_timed=barrier, sampler=e2e_sampler)
    e2e_clocks = e2e_sampler.stop()
    barrier()
    t = torch.tensor([e2e_ms], dtype=torch.float64, device=dev)
    if world > 1:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    e2e_value = tokens_total / (float(t.item()) / 1e3)
    nbytes = x.numel() * x.element_size()

    peaks, peak_src = load_peaks()
    roofline = workload_roofline(cfg, args.workload, stages, st, peaks, peak_src, moe.gemm_variant(p))
    if cfg["T"] <= 64:
        # decode: weight-read bound; the headline figure is HBM bandwidth
        roofline["forward_hbm_gbs"] = decode_bytes(cfg, st) / (ms_per_step / 1e3) / 1e9
        roofline["forward_hbm_frac"] = roofline["forward_hbm_gbs"] / peaks["hbm_gbs"]

    line = {
        "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16" if cfg["dtype"] == "bf16" else "f32", "data": "synthetic",
        "config": config_of(cfg, args), "tflops": tflops,
        "tflops_frac_of_peak": tflops / peaks["bf16_tflops"],
        "roofline": roofline,
        "e2e": {"value": e2e_value, "unit": "tokens/s", "h2d_bytes_per_step": nbytes,
                "d2h_bytes_per_step": nbytes, "ms_per_step": float(t.item()) / args.steps,
                "schedule": "double-buffered: the copy-in of step i+1 and the copy-out of step i-1 run on "
                            "their own streams beside the forward of step i; one timed region from the "
                            "first copy-in to the last copy-out; no L2 flush (the weights exceed L2)",
                "clocks": e2e_clocks},
        "gpu_launches": launches_per_forward(cfg, args.pad_rows) * args.steps,
        "router_variant": moe.router_variant(p),
        "clocks": clocks,
        "stages_ms": stages,
        "hbm_stages": hbm_stages(cfg, rows, stages, peaks),
        "routing": {"rows": rows, "dropped": st.dropped, "l_aux": st.l_aux, "max_over_mean": st.max_over_mean,
                    "experts_touched": touched_experts(st), "counts": st.counts if E <= 16 else None,
                    "kept": st.kept if E <= 16 else None},
    }
    if gst is not None:
        line["global_stats"] = {"T": gst.T, "l_aux": gst.l_aux, "dropped": gst.dropped,
                                "max_over_mean": gst.max_over_mean}
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        gidx = moe.workspace_view(layer.workspace, p, "idx").cpu().numpy()
        n, dt, tr = oracle_sample(cfg, L, args.cpu_sample,
                                  needed_experts=lambda toks: gidx[toks].reshape(-1).tolist())
        line["cpu_baseline"] = {"value": n / dt, "unit": "tokens/s", "cores": blas_threads(), "kind": "oracle",
                                "sample": f"routing of all {cfg['T']} tokens + expert math of {n} seeded random "
                                          f"tokens ({dt:.1f} s)",
                                "route_ms": 1e3 * tr, "expert_ms_per_token": 1e3 * (dt - tr) / n}
    line["pass_roofline"] = pass_roofline(cfg, st, ms_per_step, peaks)
    if not args.no_graph:
        del graph
    if world == 1 and not args.no_extra and args.workload == "mixtral_prefill" and not args.pad_rows:
        cache = {(cfg["d"], cfg["d_ff"], cfg["E"], cfg["dtype"], cfg["d_ff_shared"]):
                 {n: L[n] for n in ("W1", "W3", "W2", "Ws1", "Ws3", "Ws2")}}
        del layer
        line["workloads"] = {name: measure_extra(name, args, moe, dev, stream, flush, peaks, peak_src, cache)
                             for name in EXTRA_WORKLOADS}
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(line), flush=True)


def e2e_pipelined(layer, x_host, dev, stream, steps, before_timed=None, sampler=None):
    """Milliseconds for `steps` forwards through host buffers, as a serving
    loop runs them: each step copies its input rows from pinned host memory
    and its output rows back to pinned host memory; the copy-in of step i+1
    (one stream) and the copy-out of step i-1 (another) overlap the forward
    of step i, with two device buffers each for inputs and outputs. The
    timed region opens before the first copy-in and closes after the last
    copy-out, on the forward's stream."""
    T, d = x_host.shape
    dt = x_host.dtype
    s_in = torch.cuda.Stream(dev)
    s_out = torch.cuda.Stream(dev)
    x_dev = [torch.empty((T, d), dtype=dt, device=dev) for _ in range(2)]
    o_dev = [torch.empty((T, d), dtype=dt, device=dev) for _ in range(2)]
    o_host = [torch.empty((T, d), dtype=dt).pin_memory() for _ in range(2)]

    def run(n):
        in_done, comp_done, out_done = [None] * n, [None] * n, [None] * n
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        s_in.wait_event(e0)
        s_out.wait_event(e0)

        def copy_in(i):
            with torch.cuda.stream(s_in):
                if i >= 2:
                    s_in.wait_event(comp_done[i - 2])   # x_dev[i % 2] no longer read
                x_dev[i % 2].copy_(x_host, non_blocking=True)
                in_done[i] = torch.cuda.Event()
                in_done[i].record(s_in)

        copy_in(0)
        for i in range(n):
            if i + 1 < n:
                copy_in(i + 1)
            stream.wait_event(in_done[i])
            if i >= 2:
                stream.wait_event(out_done[i - 2])      # o_dev[i % 2] copied out
            layer(x_dev[i % 2], out=o_dev[i % 2], stream=stream)
            comp_done[i] = torch.cuda.Event()
            comp_done[i].record(stream)
            with torch.cuda.stream(s_out):
                s_out.wait_event(comp_done[i])
                o_host[i % 2].copy_(o_dev[i % 2], non_blocking=True)
                out_done[i] = torch.cuda.Event()
                out_done[i].record(s_out)
        stream.wait_event(out_done[n - 1])
        e1.record(stream)
        torch.cuda.synchronize(dev)
        return e0.elapsed_time(e1)

    run(3)
    if before_timed is not None:
        before_timed()
    if sampler is not None:
        sampler.mark()
    return run(steps)


def run_train(args, cfg, moe, L, dev, stream, flush):
    """Training step: forward with the pre-activations kept, then the backward
    of <dy, y> + alpha L_aux + beta L_z (both captured in one CUDA graph),
    on the padded-row layout the backward needs; rank 0 prints one JSON line."""
    T, d, dff, E, k = cfg["T"], cfg["d"], cfg["d_ff"], cfg["E"], cfg["k"]
    pad = args.pad_rows or 128
    p = moe.problem(T, d, dff, E, k, cfg["cf"], cfg["dtype"], cfg["bias_mode"], cfg["d_ff_shared"],
                    pad_rows=pad, train=1)
    ws = moe.alloc_workspace(p, dev)
    st = moe.alloc_stats(E, dev)
    bws = moe.alloc_backward_workspace(p, dev)
    out = torch.empty((T, d), dtype=L["x"].dtype, device=dev)
    g = torch.Generator().manual_seed(1)
    dy = torch.randn((T, d), generator=g).to(L["x"].dtype).to(dev)
    dx = torch.empty_like(L["x"])
    dW_r = torch.empty((d, E), device=dev)
    dW1 = torch.empty((E, dff, d), device=dev)
    dW3 = torch.empty((E, dff, d), device=dev)
    dW2 = torch.empty((E, d, dff), device=dev)
    dfs = cfg["d_ff_shared"]
    dWs = [torch.empty((dfs, d), device=dev), torch.empty((dfs, d), device=dev),
           torch.empty((d, dfs), device=dev)] if dfs else [None, None, None]

    def fwd():
        moe.forward(p, L["x"], L["W_r"], L["W1"], L["W3"], L["W2"], out, st, ws, bias=L["bias"], Ws1=L["Ws1"],
                    Ws3=L["Ws3"], Ws2=L["Ws2"])

    def bwd():
        moe.backward(p, L["x"], L["W_r"], L["W1"], L["W3"], L["W2"], dy, dx, dW_r, dW1, dW3, dW2, st, ws, bws,
                     alpha=0.01, beta=0.001, Ws1=L["Ws1"], Ws3=L["Ws3"], Ws2=L["Ws2"], dWs1=dWs[0], dWs3=dWs[1],
                     dWs2=dWs[2])

    for _ in range(args.warmup):
        fwd()
        bwd()
    torch.cuda.synchronize(dev)
    graphs = {}
    for name, fn in (("step", lambda: (fwd(), bwd())), ("fwd", fwd), ("bwd", bwd)):
        gr = torch.cuda.CUDAGraph()
        with torch.cuda.graph(gr):
            fn()
        graphs[name] = gr
    torch.cuda.synchronize(dev)

    def timed(gr, n):
        evs = []
        for _ in range(n):
            flush()
            a = torch.cuda.Event(enable_timing=True)
            b = torch.cuda.Event(enable_timing=True)
            a.record(stream)
            gr.replay()
            b.record(stream)
            evs.append((a, b))
        torch.cuda.synchronize(dev)
        return sum(a.elapsed_time(b) for a, b in evs) / n

    for _ in range(3):
        graphs["step"].replay()
    sampler = ClockSampler(gpu_index_for(0))
    sampler.start()
    sampler.mark()
    step_ms = timed(graphs["step"], args.steps)
    clocks = sampler.stop()
    fwd_ms = timed(graphs["fwd"], max(3, args.steps // 3))
    bwd_ms = timed(graphs["bwd"], max(3, args.steps // 3))
    s = moe.read_stats(st, E)
    if s.status != moe.MOE_OK:
        raise SystemExit(f"device status {s.status}: {moe.error_string(s.status)}")
    R = s.rows
    fl_fwd = flops_per_step(cfg, R)
    # backward: dH and dXp (2 R d d_ff + 4 R d d_ff), dW2 and [dW1; dW3] (the same), router 2 x 2 T d E,
    # and the shared expert's four GEMMs over all T rows
    fl_bwd = 2.0 * (2.0 * R * d * dff + 4.0 * R * d * dff) + 4.0 * T * d * E + 2.0 * 6.0 * T * d * dfs
    peaks, peak_src = load_peaks()
    tf_step = (fl_fwd + fl_bwd) / (step_ms / 1e3) / 1e12
    tf_bwd = fl_bwd / (bwd_ms / 1e3) / 1e12
    cpu = None
    if not args.no_cpu_baseline:
        cpu = train_cpu_baseline(cfg, L, min(args.cpu_sample, 64))
    line = {
        "metric": "MoE-layer training step (fwd+bwd) tokens/s & TFLOP/s vs bf16 peak", "impl": "ours",
        "value": T / (step_ms / 1e3), "unit": "tokens/s", "n_gpus": 1, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": step_ms, "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic", "config": dict(config_of(cfg, args), pad_rows=pad, train=1, alpha=0.01, beta=0.001),
        "tflops": tf_step, "tflops_frac_of_peak": tf_step / peaks["bf16_tflops"],
        "tflops_frac_of_sustained": tf_step / peaks.get("bf16_tflops_sustained", peaks["bf16_tflops"]),
        "peak_source": peak_src,
        "forward": {"ms": fwd_ms, "tflops": fl_fwd / (fwd_ms / 1e3) / 1e12},
        "backward": {"ms": bwd_ms, "tflops": tf_bwd},
        # the backward pass as the unit: its four grouped GEMMs are 99 % of its FLOPs
        "roofline": {"bound": "tensor", "kernel": "backward pass (tc_bwd_gemm x 4 + router/gather kernels)",
                     "achieved": tf_bwd, "peak": peaks["bf16_tflops"], "unit": "TFLOP/s",
                     "frac": tf_bwd / peaks["bf16_tflops"], "peak_source": f"{peak_src} bf16 burst",
                     "frac_of_sustained": tf_bwd / peaks.get("bf16_tflops_sustained", peaks["bf16_tflops"]),
                     "flops_per_launch": fl_bwd, "traffic": None},
        "cpu_baseline": cpu,
        "gpu_launches": (launches_per_forward(cfg, pad, train=1) + 10 + (6 if dfs else 0)) * args.steps,
        "clocks": clocks,
    }
    print(json.dumps(line), flush=True)


def train_cpu_baseline(cfg, L, n_tokens, seed=0):
    """The backward oracle on a seeded token sample: routing of all tokens,
    expert forward and backward of the sampled tokens only (dy is zero on the
    others), timed on the host cores."""
    from oracle import moe_oracle as O
    from oracle import moe_backward_oracle as BO
    rng = np.random.default_rng(seed)
    tokens = np.sort(rng.choice(cfg["T"], size=min(n_tokens, cfg["T"]), replace=False))
    x = L["x"].float().cpu().numpy()[tokens]
    W_r = L["W_r"].float().cpu().numpy()
    bias = None if L["bias"] is None else L["bias"].float().cpu().numpy()
    z = O.router_logits(x, W_r)
    key = O.selection_key(z, bias, cfg["bias_mode"])
    used = sorted(set(O.topk_lowest_index(key, cfg["k"]).reshape(-1).tolist()))

    class _Host(dict):
        def __init__(self, W):
            super().__init__({e: W[e].float().cpu().numpy() for e in used})
            self.W = W

        def __missing__(self, e):
            v = self[e] = self.W[e].float().cpu().numpy()
            return v

    W1, W3, W2 = _Host(L["W1"]), _Host(L["W3"]), _Host(L["W2"])
    sh = {n: (None if L[n] is None else L[n].float().cpu().numpy()) for n in ("Ws1", "Ws3", "Ws2")}
    dy = rng.standard_normal(x.shape)
    t0 = time.perf_counter()
    BO.moe_backward(x, W_r, W1, W3, W2, cfg["k"], dy, 0.0, bias, cfg["bias_mode"], **sh, alpha=0.01, beta=0.001)
    dt = time.perf_counter() - t0
    return {"value": len(tokens) / dt, "unit": "tokens/s", "cores": blas_threads(), "kind": "oracle",
            "sample": f"forward + backward of {len(tokens)} seeded random tokens as their own batch "
                      f"(no capacity), {dt:.1f} s"}


def breakdown(moe, p, cfg, L, dev, stream, flush, iters):
    """Average device time of each stage, each launched through its own entry point."""
    T, d, dff, E, k, dfs = cfg["T"], cfg["d"], cfg["d_ff"], cfg["E"], cfg["k"], cfg["d_ff_shared"]
    dt = L["x"].dtype
    ws = moe.alloc_workspace(p, dev)
    st = moe.alloc_stats(E, dev)
    idx = torch.empty((T, k), dtype=torch.int32, device=dev)
    gate = torch.empty((T, k), dtype=torch.float32, device=dev)
    pos = torch.empty((T, k), dtype=torch.int32, device=dev)
    indptr = torch.empty((E + 1,), dtype=torch.int32, device=dev)
    R = moe.permuted_rows(p)
    row_token = torch.empty((R,), dtype=torch.int32, device=dev)
    xp = torch.empty((R, d), dtype=dt, device=dev)
    h = torch.empty((R, dff), dtype=dt, device=dev)
    o = torch.empty((R, d), dtype=dt, device=dev)
    hs = torch.empty((T, dfs), dtype=dt, device=dev) if dfs else None
    s = torch.empty((T, d), dtype=dt, device=dev) if dfs else None
    out = torch.empty((T, d), dtype=dt, device=dev)
    names = ["route", "permute", "expert_up", "expert_down", "combine"]
    acc = {n: 0.0 for n in names}

    def run(record):
        evs = [torch.cuda.Event(enable_timing=True) for _ in range(len(names) + 1)]
        evs[0].record(stream)
        moe.route(p, L["x"], L["W_r"], idx, gate, st, ws, bias=L["bias"])
        evs[1].record(stream)
        moe.permute(p, L["x"], idx, pos, indptr, row_token, xp, st, ws)
        evs[2].record(stream)
        moe.expert_up(p, xp, indptr, L["W1"], L["W3"], h, ws, x=L["x"], Ws1=L["Ws1"], Ws3=L["Ws3"], hs=hs)
        evs[3].record(stream)
        moe.expert_down(p, h, indptr, L["W2"], o, ws, hs=hs, Ws2=L["Ws2"], s=s)
        evs[4].record(stream)
        moe.combine(p, o, pos, gate, out, s=s)
        evs[5].record(stream)
        return evs

    for _ in range(2):
        run(False)
    allev = []
    for _ in range(iters):
        flush()
        allev.append(run(True))
    torch.cuda.synchronize(dev)
    for evs in allev:
        for i, n in enumerate(names):
            acc[n] += evs[i].elapsed_time(evs[i + 1])
    return {n: acc[n] / iters for n in names}


if __name__ == "__main__":
    main()
