"""Helpers of the GPU parity tests: run the CUDA path, run the oracle on the
same inputs, and measure the differences the way the acceptance bars state
them."""

from __future__ import annotations

import numpy as np
import torch

import mixture_experts_layer_62_b200 as moe
from mixture_experts_layer_62_b200 import inputs
from oracle import moe_oracle as O

# Acceptance bars: max relative output error (per token in L2, and per
# element against the largest element of its row), and L_aux.
TOL_BF16 = 2e-2
TOL_F32 = 1e-5
TOL_LAUX = 1e-4
# End-to-end routing: tokens whose k-th / (k+1)-th key margin is below this
# are excluded from index comparisons (GPU fp32 logits vs oracle fp64 logits).
MARGIN = 1e-3


def np32(t: torch.Tensor) -> np.ndarray:
    return t.detach().float().cpu().numpy()


class LazyExperts:
    """W[e] as float32 numpy, copied from the device on first use."""

    def __init__(self, W, keep=4):
        self.W = W
        self.keep = keep
        self.cache = {}

    def __getitem__(self, e):
        e = int(e)
        if e not in self.cache:
            if len(self.cache) >= self.keep:
                self.cache.pop(next(iter(self.cache)))
            self.cache[e] = self.W[e].float().cpu().numpy()
        return self.cache[e]


def problem_of(cfg):
    return moe.problem(cfg["T"], cfg["d"], cfg["d_ff"], cfg["E"], cfg["k"], cfg["cf"], cfg["dtype"],
                       cfg["bias_mode"], cfg["d_ff_shared"], cfg.get("gate", 0), cfg.get("drop", 0),
                       cfg.get("pad", 0))


def gpu_forward(cfg, L, device="cuda"):
    p = problem_of(cfg)
    ws = moe.alloc_workspace(p, device)
    st = moe.alloc_stats(cfg["E"], device)
    out = torch.empty((cfg["T"], cfg["d"]), dtype=inputs.torch_dtype(cfg), device=device)
    moe.forward(p, L["x"], L["W_r"], L["W1"], L["W3"], L["W2"], out, st, ws, bias=L["bias"],
                Ws1=L["Ws1"], Ws3=L["Ws3"], Ws2=L["Ws2"])
    torch.cuda.synchronize()
    return p, out, st, ws


def to_device(L, device="cuda"):
    return {k_: (v.to(device) if isinstance(v, torch.Tensor) else v) for k_, v in L.items()}


def oracle_weights(L):
    """Expert weights indexable by expert for the oracle (lazy for big ones)."""
    W = {}
    for n in ("W1", "W3", "W2"):
        W[n] = LazyExperts(L[n])
    for n in ("Ws1", "Ws3", "Ws2"):
        W[n] = None if L[n] is None else np32(L[n])
    return W


def token_rel_err(y, ref):
    """max_t ||y_t - ref_t|| / ||ref_t|| over rows with ref_t != 0, and the
    largest |y_t| over rows where ref_t == 0 (must be exactly 0)."""
    y = np.asarray(y, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    nr = np.linalg.norm(ref, axis=1)
    nz = nr > 0
    rel = 0.0
    if nz.any():
        rel = float(np.max(np.linalg.norm(y[nz] - ref[nz], axis=1) / nr[nz]))
    zero_rows_max = float(np.abs(y[~nz]).max()) if (~nz).any() else 0.0
    return rel, zero_rows_max


def elem_rel_err(y, ref):
    """max over rows with ref_t != 0 and elements i of |y_ti - ref_ti| /
    max_i |ref_ti|, and the global max|y - ref| / max|ref|.

    Unlike the per-token L2 norm, this sees a single wrong column: at d = 4096
    a column that is entirely wrong moves a token's L2 error by only about
    1/sqrt(d) = 0.016, but moves the element error by the column's own size
    relative to its row's largest element."""
    y = np.asarray(y, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    if ref.size == 0:
        return 0.0, 0.0
    rmax = np.abs(ref).max(axis=1)
    nz = rmax > 0
    per_row = 0.0
    if nz.any():
        per_row = float((np.abs(y[nz] - ref[nz]).max(axis=1) / rmax[nz]).max())
    gmax = float(np.abs(ref).max())
    glob = float(np.abs(y - ref).max() / gmax) if gmax > 0 else float(np.abs(y).max())
    return per_row, glob


def assert_rows_close(y, ref, tol, what=""):
    """The output bar, applied three ways: per-token relative L2 error, per
    element against its row's largest element, and the global elementwise
    max|dy|/max|y|, all below tol; rows whose reference is 0 (fully dropped
    tokens without a shared expert) must be exactly 0. Returns the three."""
    rel, zmax = token_rel_err(y, ref)
    elem, glob = elem_rel_err(y, ref)
    assert rel < tol, (what, "token L2", rel)
    assert elem < tol, (what, "element / row max", elem)
    assert glob < tol, (what, "global element", glob)
    assert zmax == 0.0, (what, "zero rows", zmax)
    return rel, elem, glob


def key_margin(key, k):
    """Gap between the k-th and (k+1)-th largest key of every row (inf if k == E)."""
    key = np.asarray(key, dtype=np.float64)
    if k >= key.shape[1]:
        return np.full(key.shape[0], np.inf)
    part = -np.sort(-key, axis=1)
    return part[:, k - 1] - part[:, k]
