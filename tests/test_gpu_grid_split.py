"""The opt-in two-class schedules of the single-CTA grouped GEMMs.

With 32 or more experts and fewer than 512 rows per expert on average:
  * MOE_SMALL_CTAS=n (grid split) runs the groups of at most 128 rows as
    operand-swapped tiles (the weight rows as the MMA's M operand, the
    group's rows in 32-row boxes as its N operand) on the first n CTAs, and
    the other groups on the rest;
  * MOE_INTERLEAVE=1 spreads those groups' ordinary tiles evenly through the
    others' in one order, their weights loaded with an evict-first L2 policy.
The overrides are read once per process, so each runs in a child process;
its outputs are checked here against the oracle, element by element, at the
bf16 bar, over groups of every size around the 32-row boundaries, with and
without the shared expert, and in a whole forward.
"""

import math
import os
import subprocess
import sys

import numpy as np
import pytest
import torch

from oracle import moe_oracle as O
from parity_util import TOL_BF16, assert_rows_close

pytestmark = pytest.mark.gpu
ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

CASES = [(256, 384, [0, 1, 5, 31, 32, 33, 64, 65, 96, 97, 128, 129, 200, 300, 0, 7] + [3] * 16, 128, 800),
         (512, 256, [2, 40, 129, 700, 17, 0, 1, 90] * 4, 0, 2000),
         (256, 14336, [2500, 3, 7] + [1] * 29, 0, 1300)]


def _inputs(i, d, d_ff, counts, dfs, T):
    E = len(counts)
    g = torch.Generator().manual_seed(300 + i)
    rows = 2 * T
    assert sum(counts) <= rows
    xp = torch.randn((rows, d), generator=g).to(torch.bfloat16)
    W1 = (torch.randn((E, d_ff, d), generator=g) / math.sqrt(d)).to(torch.bfloat16)
    W3 = (torch.randn((E, d_ff, d), generator=g) / math.sqrt(d)).to(torch.bfloat16)
    W2 = (torch.randn((E, d, d_ff), generator=g) / math.sqrt(d_ff)).to(torch.bfloat16)
    x = torch.randn((T, d), generator=g).to(torch.bfloat16)
    sh = {}
    if dfs:
        sh = dict(Ws1=(torch.randn((dfs, d), generator=g) / math.sqrt(d)).to(torch.bfloat16),
                  Ws3=(torch.randn((dfs, d), generator=g) / math.sqrt(d)).to(torch.bfloat16),
                  Ws2=(torch.randn((d, dfs), generator=g) / math.sqrt(dfs)).to(torch.bfloat16))
    return xp, W1, W3, W2, x, sh


SCRIPT = r"""
import math, sys
import numpy as np
import torch
sys.path.insert(0, sys.argv[2])
sys.path.insert(0, sys.argv[2] + "/tests")
import mixture_experts_layer_62_b200 as moe
from test_gpu_grid_split import CASES, _inputs
DEV = "cuda"
out = {}
for i, (d, d_ff, counts, dfs, T) in enumerate(CASES):
    E = len(counts)
    xp, W1, W3, W2, x, sh = _inputs(i, d, d_ff, counts, dfs, T)
    p = moe.problem(T, d, d_ff, E, 2, 0.0, "bf16", 0, dfs)
    assert moe.gemm_variant(p) == sys.argv[3]
    ws = moe.alloc_workspace(p, DEV)
    st = moe.alloc_stats(E, DEV)
    o = torch.zeros((2 * T, d), dtype=torch.bfloat16, device=DEV)
    s = torch.zeros((T, d), dtype=torch.bfloat16, device=DEV) if dfs else None
    indptr = torch.tensor(np.concatenate([[0], np.cumsum(counts)]), dtype=torch.int32, device=DEV)
    moe.experts(p, xp.to(DEV), indptr, W1.to(DEV), W3.to(DEV), W2.to(DEV), o, ws, x=x.to(DEV), s=s, stats=st,
                **{n: v.to(DEV) for n, v in sh.items()})
    torch.cuda.synchronize()
    assert moe.read_stats(st, E).status == moe.MOE_OK
    out[f"o{i}"] = o[:sum(counts)].float().cpu().numpy()
    if dfs:
        out[f"s{i}"] = s.float().cpu().numpy()
# a whole forward (the schedule written by the scan of the forward pass)
from test_gpu_grid_split import _forward_layer, FWD
T, d, d_ff, E, k, cf = FWD
L = _forward_layer()
p = moe.problem(T, d, d_ff, E, k, cf, "bf16", 1, 0)
assert moe.gemm_variant(p) == sys.argv[3]
ws = moe.alloc_workspace(p, DEV)
st = moe.alloc_stats(E, DEV)
y = torch.empty((T, d), dtype=torch.bfloat16, device=DEV)
moe.forward(p, L["x"].to(DEV), L["W_r"].to(DEV), L["W1"].to(DEV), L["W3"].to(DEV), L["W2"].to(DEV), y, st, ws,
            bias=L["bias"].to(DEV))
torch.cuda.synchronize()
assert moe.read_stats(st, E).status == moe.MOE_OK
out["y"] = y.float().cpu().numpy()
out["logits"] = moe.workspace_view(ws, p, "logits").cpu().numpy()
out["idx"] = moe.workspace_view(ws, p, "idx").cpu().numpy()
np.savez(sys.argv[1], **out)
"""

FWD = (900, 128, 384, 64, 6, 0.8)


def _forward_layer():
    T, d, d_ff, E, k, cf = FWD
    g = torch.Generator().manual_seed(77)
    return dict(x=torch.randn((T, d), generator=g).to(torch.bfloat16),
                W_r=(torch.randn((d, E), generator=g) / math.sqrt(d)).to(torch.bfloat16),
                W1=(torch.randn((E, d_ff, d), generator=g) / math.sqrt(d)).to(torch.bfloat16),
                W3=(torch.randn((E, d_ff, d), generator=g) / math.sqrt(d)).to(torch.bfloat16),
                W2=(torch.randn((E, d, d_ff), generator=g) / math.sqrt(d_ff)).to(torch.bfloat16),
                bias=torch.linspace(0.5, -0.5, E))


@pytest.mark.parametrize("env_var,value,variant", [("MOE_SMALL_CTAS", "24", "grid_split"),
                                                 ("MOE_INTERLEAVE", "1", "interleaved")])
def test_two_class_schedules_match_the_oracle(tmp_path, env_var, value, variant):
    path = tmp_path / "split.npz"
    env = dict(os.environ, **{env_var: value})
    r = subprocess.run([sys.executable, "-c", SCRIPT, str(path), ROOT, variant], env=env, capture_output=True,
                       text=True, timeout=900)
    assert r.returncode == 0, r.stdout + r.stderr
    got = dict(np.load(path))
    for i, (d, d_ff, counts, dfs, T) in enumerate(CASES):
        xp, W1, W3, W2, x, sh = _inputs(i, d, d_ff, counts, dfs, T)
        ip = np.concatenate([[0], np.cumsum(counts)])
        for e in range(len(counts)):
            lo, hi = ip[e], ip[e + 1]
            if hi > lo:
                ref = O.swiglu_expert(xp[lo:hi].float().numpy(), W1[e].float().numpy(), W3[e].float().numpy(),
                                      W2[e].float().numpy())
                assert_rows_close(got[f"o{i}"][lo:hi], ref, TOL_BF16, f"case {i} expert {e}")
        if dfs:
            ref = O.swiglu_expert(x.float().numpy(), sh["Ws1"].float().numpy(), sh["Ws3"].float().numpy(),
                                  sh["Ws2"].float().numpy())
            assert_rows_close(got[f"s{i}"], ref, TOL_BF16, f"case {i} shared")
    # the forward: routing bit-exact from the GPU's logits, outputs element by element
    T, d, d_ff, E, k, cf = FWD
    L = _forward_layer()
    res = O.moe_forward(L["x"].float().numpy(), None, {e: L["W1"][e].float().numpy() for e in range(E)},
                        {e: L["W3"][e].float().numpy() for e in range(E)},
                        {e: L["W2"][e].float().numpy() for e in range(E)}, k, cf, L["bias"].numpy(), O.BIAS_LOGIT,
                        logits=got["logits"], key_dtype=np.float32)
    assert np.array_equal(got["idx"], res.routing.idx)
    assert res.stats.dropped > 0
    assert_rows_close(got["y"], res.y, TOL_BF16, "forward")
