"""CTA-pair tiles (256 rows, cta_group::2) against single-CTA tiles (128 rows).

The grouped GEMMs switch to CTA pairs when the experts average at least 512
rows; the environment variable MOE_CTA_PAIR=0 keeps the single-CTA kernel
(read once per process). Both kernels accumulate every output element over
the same K blocks in the same order, so the same inputs give the same bits.
Each setting runs in its own process on the same seeded inputs; the outputs
are compared bit for bit, including groups that span more than one band of M
blocks (where the two kernels order their tiles differently).
"""

import os
import subprocess
import sys

import numpy as np
import pytest

pytestmark = pytest.mark.gpu
ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

SCRIPT = r"""
import math, sys
import numpy as np
import torch
sys.path.insert(0, sys.argv[2])
import mixture_experts_layer_62_b200 as moe

DEV = "cuda"
out = {}
cases = [(512, 384, [600, 0, 1300, 257], 1100), (256, 14336, [2600, 3], 1302),
         (7168, 256, [70, 2300], 1185), (128, 128, [1, 1023], 512)]
for i, (d, d_ff, counts, T) in enumerate(cases):
    E = len(counts)
    g = torch.Generator().manual_seed(100 + i)
    rows = T * 2
    xp = torch.randn((rows, d), generator=g).to(torch.bfloat16).to(DEV)
    W1 = (torch.randn((E, d_ff, d), generator=g) / math.sqrt(d)).to(torch.bfloat16).to(DEV)
    W3 = (torch.randn((E, d_ff, d), generator=g) / math.sqrt(d)).to(torch.bfloat16).to(DEV)
    W2 = (torch.randn((E, d, d_ff), generator=g) / math.sqrt(d_ff)).to(torch.bfloat16).to(DEV)
    indptr = torch.tensor(np.concatenate([[0], np.cumsum(counts)]), dtype=torch.int32, device=DEV)
    p = moe.problem(T, d, d_ff, E, 2, 0.0, "bf16")
    ws = moe.alloc_workspace(p, DEV)
    st = moe.alloc_stats(E, DEV)
    o = torch.zeros((rows, d), dtype=torch.bfloat16, device=DEV)
    moe.experts(p, xp, indptr, W1, W3, W2, o, ws, stats=st)
    torch.cuda.synchronize()
    assert moe.read_stats(st, E).status == moe.MOE_OK
    out[f"experts{i}"] = o[:sum(counts)].view(torch.int16).cpu().numpy()
# a whole forward with capacity drops
T, d, d_ff, E, k = 3000, 256, 384, 4, 2
g = torch.Generator().manual_seed(7)
x = torch.randn((T, d), generator=g).to(torch.bfloat16).to(DEV)
W_r = (torch.randn((d, E), generator=g) / math.sqrt(d)).to(torch.bfloat16).to(DEV)
W1 = (torch.randn((E, d_ff, d), generator=g) / math.sqrt(d)).to(torch.bfloat16).to(DEV)
W3 = (torch.randn((E, d_ff, d), generator=g) / math.sqrt(d)).to(torch.bfloat16).to(DEV)
W2 = (torch.randn((E, d, d_ff), generator=g) / math.sqrt(d_ff)).to(torch.bfloat16).to(DEV)
p = moe.problem(T, d, d_ff, E, k, 0.9, "bf16")
ws = moe.alloc_workspace(p, DEV)
st = moe.alloc_stats(E, DEV)
y = torch.empty((T, d), dtype=torch.bfloat16, device=DEV)
moe.forward(p, x, W_r, W1, W3, W2, y, st, ws)
torch.cuda.synchronize()
assert moe.read_stats(st, E).status == moe.MOE_OK
out["forward"] = y.view(torch.int16).cpu().numpy()
np.savez(sys.argv[1], **out)
"""


def _run(path, pair):
    env = dict(os.environ, MOE_CTA_PAIR="1" if pair else "0")
    r = subprocess.run([sys.executable, "-c", SCRIPT, str(path), ROOT], env=env, capture_output=True, text=True,
                       timeout=600)
    assert r.returncode == 0, r.stdout + r.stderr
    return dict(np.load(path))


def test_pair_and_single_cta_tiles_agree_bit_for_bit(tmp_path):
    single = _run(tmp_path / "single.npz", pair=False)
    pair = _run(tmp_path / "pair.npz", pair=True)
    assert single.keys() == pair.keys()
    for name in single:
        a, b = single[name], pair[name]
        assert np.array_equal(a, b), (name, int((a != b).sum()), a.size)
