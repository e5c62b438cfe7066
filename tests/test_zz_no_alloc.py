"""The allocation-free permutation entry point (moe_permute_noalloc).

It exists for callers that cannot allocate device memory where they run the
layer (a runtime plugin handed only its input and output buffers, or a
latency-critical loop in which cudaMalloc could block or synchronise the
device): it runs moe_permute's kernels with the scratch in a fixed array
inside the library instead of a caller workspace.

The GPU test calls it through the C ABI twice in a row, on different inputs,
and compares every output with the existing workspace-based moe_permute on the
same inputs, and with the oracle's permutation of the same expert selection:
integers and gathered rows must be bit-identical, the tolerance all
permutation tests use. The second call runs on the scratch left by the
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


def _inputs(T, E, k, d, skew, seed, dtype):
    rng = np.random.default_rng(seed)
    z = rng.standard_normal((T, E))
    z[:, 0] += skew
    idx = O.topk_lowest_index(z, k).astype(np.int32)
    g = torch.Generator().manual_seed(seed)
    x = torch.randn((T, d), generator=g).to(dtype)
    return idx, torch.from_numpy(idx).to(DEV), x.to(DEV)


def _outputs(T, E, k, d, dtype):
    return dict(pos=torch.full((T, k), -5, dtype=torch.int32, device=DEV),
                indptr=torch.full((E + 1,), -5, dtype=torch.int32, device=DEV),
                row_token=torch.full((T * k,), -5, dtype=torch.int32, device=DEV),
                xp=torch.zeros((T * k, d), dtype=dtype, device=DEV),
                stats=moe.alloc_stats(E, DEV))


@pytest.mark.gpu
def test_noalloc_matches_permute_on_two_calls_in_a_row():
    # bf16 and fp32 rows, with and without capacity, token and slot drop
    # order (the slot order keeps k counts per chunk and expert in the array)
    cases = [dict(T=3000, E=64, k=8, d=256, cf=1.0, skew=1.5, seed=1, dtype="bf16", drop=0),
             dict(T=1000, E=8, k=2, d=128, cf=0.0, skew=0.0, seed=2, dtype="bf16", drop=0),
             dict(T=2500, E=16, k=4, d=64, cf=0.8, skew=1.0, seed=3, dtype="f32", drop=1),
             dict(T=777, E=32, k=2, d=192, cf=0.5, skew=2.0, seed=4, dtype="bf16", drop=1)]
    for c in cases:
        T, E, k, d = c["T"], c["E"], c["k"], c["d"]
        dt = torch.bfloat16 if c["dtype"] == "bf16" else torch.float32
        p = moe.problem(T, d, 64, E, k, c["cf"], c["dtype"], drop_order=c["drop"])
        idx_np, idx, x = _inputs(T, E, k, d, c["skew"], c["seed"], dt)
        a = _outputs(T, E, k, d, dt)
        moe.permute_noalloc(p, x, idx, a["pos"], a["indptr"], a["row_token"], a["xp"], a["stats"])
        b = _outputs(T, E, k, d, dt)
        ws = moe.alloc_workspace(p, DEV)
        moe.permute(p, x, idx, b["pos"], b["indptr"], b["row_token"], b["xp"], b["stats"], ws)
        torch.cuda.synchronize()
        # the existing entry point: every output bit-identical
        for name in ("pos", "indptr", "xp", "stats"):
            assert torch.equal(a[name], b[name]), name
        R = int(b["indptr"][-1])
        assert torch.equal(a["row_token"][:R], b["row_token"][:R])
        # the oracle's permutation of the same selection: bit-exact as well
        C = O.capacity(c["cf"], T, k, E)
        perm = O.permute(idx_np, E, C, c["drop"])
        assert np.array_equal(a["pos"].cpu().numpy(), perm.pos)
        assert np.array_equal(a["indptr"].cpu().numpy(), perm.indptr)
        assert np.array_equal(a["row_token"].cpu().numpy()[:R], perm.row_token)
        assert torch.equal(a["xp"][:R].cpu(), x.cpu()[torch.from_numpy(perm.row_token)])
        s = moe.read_stats(a["stats"], E)
        assert s.status == moe.MOE_OK and s.rows == R
        assert s.counts == perm.counts.tolist() and s.kept == perm.kept.tolist()
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


def test_noalloc_checks_problems_like_permute():
    # host-side checks, nothing launched: on every problem that moe_permute
    # rejects before looking at its workspace, both entry points return the
    # same code
    fake = ctypes.c_void_p(1 << 20)
    noalloc = moe.lib.moe_permute_noalloc
    noalloc.argtypes = [ctypes.POINTER(moe.Problem)] + [ctypes.c_void_p] * 8
    noalloc.restype = ctypes.c_int
    lib = moe._lib()
    bad = [
        moe.problem(64, 256, 64, 8, 2, float("inf"), "bf16"),      # infinite capacity factor
        moe.problem(64, 256, 64, 8, 2, float("nan"), "bf16"),
        moe.problem(64, 72, 64, 8, 2, 0.0, "bf16"),               # bf16 rows need d % 64 == 0
        moe.problem(64, 12, 64, 8, 2, 0.0, "f32"),                # fp32 rows need d % 8 == 0
        moe.problem(64, 256, 64, 4, 5),                           # k > E
        moe.problem(-1, 256, 64, 8, 2),
        moe.problem(64, 256, 64, 512, 16, drop_order=1),          # slot counts beyond the limit
    ]
    p = moe.problem(64, 256, 64, 8, 2)
    p.pad_rows = 3                                               # neither 0, 64 nor 128
    bad.append(p)
    p = moe.problem(64, 256, 64, 8, 2)
    p.train = 2
    bad.append(p)
    p = moe.problem(64, 256, 64, 8, 2)
    p.dtype = 7
    bad.append(p)
    for p in bad:
        want = lib.moe_permute(ctypes.byref(p), fake, fake, fake, fake, fake, fake, fake, fake, 1 << 30, None)
        got = noalloc(ctypes.byref(p), fake, fake, fake, fake, fake, fake, fake, None)
        assert want != moe.MOE_OK and got == want, (want, got)
