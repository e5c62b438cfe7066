"""Seeded synthetic inputs shaped like the workloads of the MoE notes.

This module only draws random tensors; it holds none of the layer's
arithmetic. Both the CUDA path and the CPU oracle are fed from it.

Recipe (every tensor has its own generator, seeded from (seed, tensor name)):
  x            ~ N(0, 1)                 [T, d]
  W_r          ~ N(0, 1/d)               [d, E]
  W1, W3, Ws1, Ws3 ~ N(0, 1/d)           [E, d_ff, d] / [d_ff_s, d]
  W2, Ws2      ~ N(0, 1/d_ff)            [E, d, d_ff] / [d, d_ff_s]
  bias         PROB mode: U(-0.1, 0.1); LOGIT mode (skewed workload): the
               calibrated vector stored in tests/golden/zipf_bias_skewed.txt
drawn in fp32 and rounded once to the workload's dtype. x, W_r and the bias
are always drawn on the CPU (so routing inputs are identical on every
machine); the expert weights are drawn on ``weights_device`` expert by
expert (the CUDA generator when that is a GPU).
"""

from __future__ import annotations

import math
import os
import zlib

import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
ZIPF_BIAS_FILE = os.path.join(ROOT, "tests", "golden", "zipf_bias_skewed.txt")

# The workloads of the notes (sizes as named in the benchmark configuration).
WORKLOADS = {
    # toy layer, fp32, no capacity
    "toy_fp32": dict(T=1024, d=128, d_ff=256, E=8, k=2, cf=0.0, dtype="f32", bias_mode=0, d_ff_shared=0),
    # Mixtral-8x7B-shaped layer, bf16 prefill
    "mixtral_prefill": dict(T=4096, d=4096, d_ff=14336, E=8, k=2, cf=0.0, dtype="bf16", bias_mode=0,
                            d_ff_shared=0),
    # DeepSeek-V3-shaped fine-grained layer: 256 routed top-8 + 1 shared expert,
    # selection on softmax score + bias
    "deepseek_v3": dict(T=8192, d=7168, d_ff=2048, E=256, k=8, cf=0.0, dtype="bf16", bias_mode=2,
                        d_ff_shared=2048),
    # Mixtral shape, Zipf(1.2)-skewed routing via a selection bias on the
    # logits, capacity factor 1.25
    "skewed_capacity": dict(T=16384, d=4096, d_ff=14336, E=8, k=2, cf=1.25, dtype="bf16", bias_mode=1,
                            d_ff_shared=0),
    # half the Mixtral width, half the tokens: a training step that holds
    # about 2.5 GB on the device (the size for full profiler captures)
    "train_small": dict(T=2048, d=2048, d_ff=7168, E=8, k=2, cf=0.0, dtype="bf16", bias_mode=0, d_ff_shared=0),
}
DECODE_TOKENS = (1, 2, 4, 8, 16, 32)


def decode_workload(T: int) -> dict:
    """Mixtral-shaped decode step with T tokens (uniform random router)."""
    return dict(T=T, d=4096, d_ff=14336, E=8, k=2, cf=0.0, dtype="bf16", bias_mode=0, d_ff_shared=0)


def workload(name: str) -> dict:
    if name.startswith("decode_t"):
        return decode_workload(int(name[len("decode_t"):]))
    return dict(WORKLOADS[name])


def torch_dtype(cfg):
    return torch.bfloat16 if cfg["dtype"] == "bf16" else torch.float32


def _seed(seed: int, name: str) -> int:
    return (int(seed) * 1_000_003 + zlib.crc32(name.encode())) % (1 << 62)


def _gen(device, seed, name):
    g = torch.Generator(device=device)
    g.manual_seed(_seed(seed, name))
    return g


def normal(shape, std, seed, name, device="cpu", dtype=torch.float32):
    g = _gen(device, seed, name)
    t = torch.randn(shape, generator=g, device=device, dtype=torch.float32)
    if std != 1.0:
        t.mul_(std)
    return t.to(dtype)


def stacked_normal(E, rows, cols, std, seed, name, device="cpu", dtype=torch.float32):
    """[E, rows, cols], expert by expert from one generator (bounded scratch)."""
    out = torch.empty((E, rows, cols), dtype=dtype, device=device)
    g = _gen(device, seed, name)
    for e in range(E):
        out[e] = (torch.randn((rows, cols), generator=g, device=device, dtype=torch.float32) * std).to(dtype)
    return out


def load_zipf_bias(E: int):
    vals = []
    with open(ZIPF_BIAS_FILE) as fh:
        for line in fh:
            line = line.strip()
            if line and not line.startswith("#"):
                vals.extend(float(v) for v in line.split())
    if len(vals) != E:
        raise ValueError(f"{ZIPF_BIAS_FILE} holds {len(vals)} values, expected {E}")
    return torch.tensor(vals, dtype=torch.float32)


def make_routing_inputs(cfg, seed=0):
    """x, W_r and bias on the CPU."""
    dt = torch_dtype(cfg)
    T, d, E = cfg["T"], cfg["d"], cfg["E"]
    x = normal((T, d), 1.0, seed, "x", dtype=dt)
    W_r = normal((d, E), 1.0 / math.sqrt(d), seed, "W_r", dtype=dt)
    bias = None
    if cfg["bias_mode"] == 2:
        g = _gen("cpu", seed, "bias")
        bias = (torch.rand((E,), generator=g, dtype=torch.float32) * 0.2 - 0.1)
    elif cfg["bias_mode"] == 1:
        bias = load_zipf_bias(E)
    return x, W_r, bias


def make_layer(cfg, seed=0, device="cpu", weights_device=None):
    """All inputs of one layer as a dict of tensors (x, W_r, bias on `device`)."""
    wdev = weights_device or device
    dt = torch_dtype(cfg)
    d, dff, E, dfs = cfg["d"], cfg["d_ff"], cfg["E"], cfg["d_ff_shared"]
    x, W_r, bias = make_routing_inputs(cfg, seed)
    out = dict(x=x.to(device), W_r=W_r.to(device), bias=None if bias is None else bias.to(device))
    out["W1"] = stacked_normal(E, dff, d, 1.0 / math.sqrt(d), seed, "W1", wdev, dt)
    out["W3"] = stacked_normal(E, dff, d, 1.0 / math.sqrt(d), seed, "W3", wdev, dt)
    out["W2"] = stacked_normal(E, d, dff, 1.0 / math.sqrt(dff), seed, "W2", wdev, dt)
    if dfs:
        out["Ws1"] = normal((dfs, d), 1.0 / math.sqrt(d), seed, "Ws1", wdev, dt)
        out["Ws3"] = normal((dfs, d), 1.0 / math.sqrt(d), seed, "Ws3", wdev, dt)
        out["Ws2"] = normal((d, dfs), 1.0 / math.sqrt(dfs), seed, "Ws2", wdev, dt)
    else:
        out["Ws1"] = out["Ws3"] = out["Ws2"] = None
    return out
