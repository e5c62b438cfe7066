"""The allocation-free permutation entry point (moe_permute_noalloc).

It exists for callers that cannot allocate device memory where they run the
layer (a runtime plugin handed only its input and output buffers, or a
latency-critical loop in which cudaMalloc could block or synchronise the
device): it runs moe_permute's kernels with the scratch in a fixed array
inside the library instead of a caller workspace.

The GPU test calls it through the C ABI twice in a row, on different inputs,
and compares every output with the existing workspace-based moe_permute on the
same inputs: integers and gathered rows must be bit-identical, the tolerance
all permutation tests use. The second call runs on the scratch left by the
first, so a stale-scratch dependence would show. It passes on its own in a
fresh process (its first call does the per-device set-up) and after the rest
of the suite.
"""

import ctypes

import numpy as np
import pytest
import torch

import mixture_experts_layer_62_b200 as moe
from oracle import moe_oracle as O

DEV = "cuda"


def _inputs(T, E, k, d, skew, seed):
    rng = np.random.default_rng(seed)
    z = rng.standard_normal((T, E))
    z[:, 0] += skew
    idx = O.topk_lowest_index(z, k).astype(np.int32)
    g = torch.Generator().manual_seed(seed)
    x = torch.randn((T, d), generator=g).to(torch.bfloat16)
    return torch.from_numpy(idx).to(DEV), x.to(DEV)


def _outputs(T, E, k, d):
    return dict(pos=torch.full((T, k), -5, dtype=torch.int32, device=DEV),
                indptr=torch.full((E + 1,), -5, dtype=torch.int32, device=DEV),
                row_token=torch.full((T * k,), -5, dtype=torch.int32, device=DEV),
                xp=torch.zeros((T * k, d), dtype=torch.bfloat16, device=DEV),
                stats=moe.alloc_stats(E, DEV))


@pytest.mark.gpu
def test_noalloc_matches_permute_on_two_calls_in_a_row():
    cases = [dict(T=3000, E=64, k=8, d=256, cf=1.0, skew=1.5, seed=1),
             dict(T=1000, E=8, k=2, d=128, cf=0.0, skew=0.0, seed=2)]
    for c in cases:
        T, E, k, d = c["T"], c["E"], c["k"], c["d"]
        p = moe.problem(T, d, 64, E, k, c["cf"], "bf16")
        idx, x = _inputs(T, E, k, d, c["skew"], c["seed"])
        a = _outputs(T, E, k, d)
        moe.permute_noalloc(p, x, idx, a["pos"], a["indptr"], a["row_token"], a["xp"], a["stats"])
        b = _outputs(T, E, k, d)
        ws = moe.alloc_workspace(p, DEV)
        moe.permute(p, x, idx, b["pos"], b["indptr"], b["row_token"], b["xp"], b["stats"], ws)
        torch.cuda.synchronize()
        for name in ("pos", "indptr", "xp", "stats"):
            assert torch.equal(a[name], b[name]), name
        R = int(b["indptr"][-1])
        assert torch.equal(a["row_token"][:R], b["row_token"][:R])
        s = moe.read_stats(a["stats"], E)
        assert s.status == moe.MOE_OK and s.rows == R
        if c["cf"] > 0:
            assert s.dropped > 0


def test_noalloc_rejects_problems_beyond_its_scratch():
    # host-side check, nothing launched: E * ceil(T / 32) must stay <= 131072
    p = moe.problem(16416, 256, 64, 256, 8, 0.0, "bf16")     # 513 chunks x 256 experts
    fake = ctypes.c_void_p(1 << 20)
    fn = moe.lib.moe_permute_noalloc
    fn.argtypes = [ctypes.POINTER(moe.Problem)] + [ctypes.c_void_p] * 8
    fn.restype = ctypes.c_int
    assert fn(ctypes.byref(p), fake, fake, fake, fake, fake, fake, fake, None) == moe.MOE_ERR_UNSUPPORTED
    p = moe.problem(16, 256, 64, 4, 5)                         # k > E
    assert fn(ctypes.byref(p), fake, fake, fake, fake, fake, fake, fake, None) == moe.MOE_ERR_INVALID_ARG
