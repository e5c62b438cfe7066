"""The fused router's two forms against the oracle.

Up to 64 experts (fewer than 64 for bf16, which takes tensor cores from 64
up), moe_route computes the logits and the selection in one kernel:
  * bf16 rows whose W_r^T fits the kernel's shared-memory budget eight
    experts at a time take the warp-MMA form (bf16 products, fp32 sums);
  * fp32, and wider bf16 rows, take the FMA form;
  * MOE_ROUTER_MMA=0 forces the FMA form for bf16. The switch is read once
    per process, so those cases run in a child process.
For every token of each case:
  * the logits, element by element, against the fp64 logits ("Week 2 Day 2:
    Mixture of Experts" §1.3, z = W_r^T x) within the fp32-accumulation bar:
    each logit is a d-term sum of products exact in fp32, and 1e-5 *
    sum_i |x_i w_i| is far above rounding and far below a wrong term;
  * indices bit-exact, gates to fp32 rounding, against the oracle's
    selection from the GPU's own logits (the key formed in fp32 on both
    sides);
  * counts exact, P and L_aux against the oracle's statistics.
The shapes cover the ragged edges of the MMA form: rows that end inside a
staged 128-element item (bf16 rows are a multiple of 64), chunks of fewer
than 32 tokens, expert counts that are not a multiple of 8 or 16 (one
expert; 20 in passes of 8, 8 and 4), and up to five passes over x.
"""

import math
import os
import subprocess
import sys

import numpy as np
import pytest
import torch

import mixture_experts_layer_62_b200 as moe
from oracle import moe_oracle as O
from parity_util import TOL_LAUX

pytestmark = pytest.mark.gpu
ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
DEV = "cuda"

# (T, d, E, k, bias_mode, dtype)
CASES = {
    "mixtral_4096x4096_E8": (4096, 4096, 8, 2, 0, "bf16"),
    "d192_ragged_item": (1000, 192, 8, 2, 1, "bf16"),
    "E6_T77": (77, 64, 6, 2, 0, "bf16"),
    "E16_k4": (500, 256, 16, 4, 1, "bf16"),
    "E40_partial_groups": (300, 512, 40, 4, 0, "bf16"),
    "E56_d1024": (257, 1024, 56, 8, 1, "bf16"),
    "E16_two_passes_d4992": (129, 4992, 16, 2, 0, "bf16"),
    "E40_five_passes_d4992": (70, 4992, 40, 4, 1, "bf16"),
    "E20_three_passes_d4992": (50, 4992, 20, 3, 1, "bf16"),
    "E1_k1": (100, 256, 1, 1, 0, "bf16"),
    "d6016_fma_form": (64, 6016, 8, 2, 0, "bf16"),
    "f32_E12": (100, 200, 12, 3, 1, "f32"),
    "f32_E40": (90, 128, 40, 4, 1, "f32"),
    "d6016_E48_fma_form": (70, 6016, 48, 6, 0, "bf16"),
    "T1": (1, 4096, 8, 2, 0, "bf16"),
}
FORCED_FMA = ["mixtral_4096x4096_E8", "d192_ragged_item", "E40_partial_groups"]
# the form moe_route takes for each case (moe_router_variant)
FMA_CASES = {"d6016_fma_form", "f32_E12", "f32_E40", "d6016_E48_fma_form"}


def _inputs(name):
    T, d, E, k, bm, dt = CASES[name]
    g = torch.Generator().manual_seed(sum(map(ord, name)))
    tdt = torch.bfloat16 if dt == "bf16" else torch.float32
    x = torch.randn((T, d), generator=g).to(tdt)
    W_r = (torch.randn((d, E), generator=g) / math.sqrt(d)).to(tdt)
    bias = (torch.rand((E,), generator=g) - 0.5) * 0.2 if bm else None
    return x, W_r, bias


def check_case(name, form=None):
    """Runs moe_route on one case and checks it against the oracle; the
    router form moe_route takes must be `form` (by default the one the case
    is listed for)."""
    T, d, E, k, bm, dt = CASES[name]
    x, W_r, bias = _inputs(name)
    p = moe.problem(T, d, 64, E, k, 0.0, dt, bm)
    want = form or ("fused_fma" if name in FMA_CASES else "fused_mma")
    assert moe.router_variant(p, forward=False) == want, name
    ws = moe.alloc_workspace(p, DEV)
    st = moe.alloc_stats(E, DEV)
    idx = torch.empty((T, k), dtype=torch.int32, device=DEV)
    gate = torch.empty((T, k), dtype=torch.float32, device=DEV)
    logits = torch.empty((T, E), dtype=torch.float32, device=DEV)
    moe.route(p, x.to(DEV), W_r.to(DEV), idx, gate, st, ws, bias=None if bias is None else bias.to(DEV),
              logits=logits)
    torch.cuda.synchronize()
    z = logits.cpu().numpy()
    x64 = x.float().numpy().astype(np.float64)
    W64 = W_r.float().numpy().astype(np.float64)
    z64 = O.router_logits(x64, W64)
    absdot = np.abs(x64) @ np.abs(W64)
    err = np.abs(z64 - z)
    assert (err <= 1e-5 * absdot + 1e-30).all(), (name, float(np.max(err / absdot)))
    b = None if bias is None else bias.numpy().astype(np.float32)
    r = O.route(z, k, b, bm, key_dtype=np.float32)
    assert np.array_equal(idx.cpu().numpy(), r.idx), name
    assert np.allclose(gate.cpu().numpy(), r.gate, rtol=2e-6, atol=1e-7), name
    s = moe.read_stats(st, E)
    ls = O.load_stats(O.permute(r.idx, E), r.probs, T, k, None, z=z)
    assert s.status == moe.MOE_OK
    assert s.counts == ls.counts.tolist(), name
    assert np.allclose(s.P, ls.P, rtol=1e-5, atol=1e-7), name
    assert s.l_aux == pytest.approx(ls.l_aux, rel=TOL_LAUX)
    return z


@pytest.mark.parametrize("name", list(CASES))
def test_fused_router(name):
    check_case(name)


def test_fused_router_is_deterministic():
    a = check_case("mixtral_4096x4096_E8")
    b = check_case("mixtral_4096x4096_E8")
    assert np.array_equal(a, b)


SCRIPT = r"""
import sys
sys.path.insert(0, sys.argv[1])
sys.path.insert(0, sys.argv[1] + "/tests")
from test_gpu_router import check_case
for name in sys.argv[2:]:
    check_case(name, form="fused_fma")
print("ok")
"""


def test_fma_form_forced():
    env = dict(os.environ, MOE_ROUTER_MMA="0")
    r = subprocess.run([sys.executable, "-c", SCRIPT, ROOT, *FORCED_FMA], env=env, capture_output=True, text=True,
                       timeout=600, cwd=ROOT)
    assert r.returncode == 0 and r.stdout.strip().endswith("ok"), r.stdout[-2000:] + r.stderr[-4000:]
