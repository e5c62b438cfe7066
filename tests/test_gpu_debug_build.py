"""The debug build (libmoe_debug.so): same results, plus device-side bounds
checks that turn an out-of-range index into MOE_ERR_BOUNDS instead of a fault.

The debug library is loaded in a child process (MOE_LIBRARY=debug). There:
  * whole forwards on valid inputs (the CTA-pair and single-CTA kernels, the
    split-K and GEMV decode paths) give the release library's bits and MOE_OK;
  * the expert stage handed group offsets that decrease, or that end past
    the permuted rows, records MOE_ERR_BOUNDS, schedules no tile and writes
    nothing: every row of the output keeps its sentinel value.
Only the debug library ever runs the invalid offsets: its check in the
schedule kernel runs before any tile reads them. The release library is
never given them.
"""

import math
import os
import subprocess
import sys

import numpy as np
import pytest
import torch

import mixture_experts_layer_62_b200 as moe

pytestmark = pytest.mark.gpu
ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
DEV = "cuda"

FORWARDS = [dict(T=2048, d=256, d_ff=384, E=4, k=2, cf=0.0),      # CTA pairs
            dict(T=300, d=256, d_ff=384, E=8, k=2, cf=0.6),       # single-CTA tiles, capacity drops
            dict(T=40, d=512, d_ff=512, E=8, k=2, cf=0.0),        # split-K, general router
            dict(T=4, d=512, d_ff=512, E=8, k=2, cf=0.0)]         # GEMVs, small-batch router


def _layer(c, seed):
    g = torch.Generator().manual_seed(seed)
    T, d, dff, E = c["T"], c["d"], c["d_ff"], c["E"]
    return [torch.randn((T, d), generator=g).to(torch.bfloat16),
            (torch.randn((d, E), generator=g) / math.sqrt(d)).to(torch.bfloat16),
            (torch.randn((E, dff, d), generator=g) / math.sqrt(d)).to(torch.bfloat16),
            (torch.randn((E, dff, d), generator=g) / math.sqrt(d)).to(torch.bfloat16),
            (torch.randn((E, d, dff), generator=g) / math.sqrt(dff)).to(torch.bfloat16)]


def run_forwards():
    out = {}
    for i, c in enumerate(FORWARDS):
        x, W_r, W1, W3, W2 = [t.to(DEV) for t in _layer(c, 40 + i)]
        p = moe.problem(c["T"], c["d"], c["d_ff"], c["E"], c["k"], c["cf"], "bf16")
        ws = moe.alloc_workspace(p, DEV)
        st = moe.alloc_stats(c["E"], DEV)
        y = torch.empty((c["T"], c["d"]), dtype=torch.bfloat16, device=DEV)
        moe.forward(p, x, W_r, W1, W3, W2, y, st, ws)
        torch.cuda.synchronize()
        out[f"y{i}"] = y.view(torch.int16).cpu().numpy()
        out[f"status{i}"] = np.array([moe.read_stats(st, c["E"]).status])
        out[f"variant{i}"] = np.array([moe.gemm_variant(p)])
    return out


def run_bad_offsets():
    """The expert stage with invalid group offsets (debug library only)."""
    out = {}
    E, d, d_ff, T = 4, 256, 256, 200
    g = torch.Generator().manual_seed(9)
    rows = 2 * T
    xp = torch.randn((rows, d), generator=g).to(torch.bfloat16).to(DEV)
    W = (torch.randn((E, d_ff, d), generator=g) / math.sqrt(d)).to(torch.bfloat16).to(DEV)
    W2 = (torch.randn((E, d, d_ff), generator=g) / math.sqrt(d_ff)).to(torch.bfloat16).to(DEV)
    p = moe.problem(T, d, d_ff, E, 2, 0.0, "bf16")
    for name, offs in (("decreasing", [0, 150, 100, 300, 400]), ("past_rows", [0, 100, 200, 300, rows + 64])):
        ws = moe.alloc_workspace(p, DEV)
        st = moe.alloc_stats(E, DEV)
        o = torch.full((rows, d), 7.0, dtype=torch.bfloat16, device=DEV)
        moe.experts(p, xp, torch.tensor(offs, dtype=torch.int32, device=DEV), W, W, W2, o, ws, stats=st)
        torch.cuda.synchronize()
        out[f"status_{name}"] = np.array([moe.read_stats(st, E).status])
        out[f"untouched_{name}"] = np.array([bool((o == 7.0).all().item())])
    return out


SCRIPT = r"""
import sys
import numpy as np
sys.path.insert(0, sys.argv[2])
sys.path.insert(0, sys.argv[2] + "/tests")
import mixture_experts_layer_62_b200 as moe
assert moe.LIB_PATH.endswith("libmoe_debug.so"), moe.LIB_PATH
from test_gpu_debug_build import run_forwards, run_bad_offsets
out = run_forwards()
out.update(run_bad_offsets())
np.savez(sys.argv[1], **out)
"""


def test_debug_build_matches_release_and_catches_bad_offsets(tmp_path):
    path = tmp_path / "debug.npz"
    env = dict(os.environ, MOE_LIBRARY="debug")
    r = subprocess.run([sys.executable, "-c", SCRIPT, str(path), ROOT], env=env, capture_output=True, text=True,
                       timeout=600)
    assert r.returncode == 0, r.stdout + r.stderr
    dbg = dict(np.load(path))
    rel = run_forwards()      # this process: the release library
    assert moe.LIB_PATH.endswith("libmoe.so")
    for i in range(len(FORWARDS)):
        assert int(dbg[f"status{i}"][0]) == moe.MOE_OK
        assert str(dbg[f"variant{i}"][0]) == str(rel[f"variant{i}"][0])
        assert np.array_equal(dbg[f"y{i}"], rel[f"y{i}"]), i
    assert {str(rel[f"variant{i}"][0]) for i in range(len(FORWARDS))} == {"pair", "single", "split_k", "gemv"}
    for name in ("decreasing", "past_rows"):
        assert int(dbg[f"status_{name}"][0]) == moe.MOE_ERR_BOUNDS, name
        assert bool(dbg[f"untouched_{name}"][0]), name
