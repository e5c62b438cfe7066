"""GPU parity of every stage of the CUDA path against the CPU oracle.

Stage by stage (same inputs on both sides):
  route from given logits   indices bit-exact (NONE / LOGIT keys are formed
                            in fp32 on both sides), gates to fp32 rounding
  permutation               pos, indptr, row_token, counts, kept bit-exact,
                            gathered rows bit-exact
  expert GEMMs              per-row relative error under the bf16 bar
  combine                   to fp32 / bf16 rounding
End to end: small shapes over all tokens, the full-size workloads on sampled
tokens (routing over all tokens), determinism, and stage composition.
"""

import math
import os

import numpy as np
import pytest
import torch

import mixture_experts_layer_62_b200 as moe
from mixture_experts_layer_62_b200 import inputs
from oracle import moe_oracle as O
from parity_util import (MARGIN, TOL_BF16, TOL_F32, TOL_LAUX, LazyExperts, assert_rows_close, gpu_forward,
                         key_margin, np32, oracle_weights, problem_of, to_device)

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _dt(name):
    return torch.bfloat16 if name == "bf16" else torch.float32


# --------------------------------------------------------------------------
# routing from given logits
# --------------------------------------------------------------------------

@pytest.mark.parametrize("T,E,k,mode,gm", [
    (1000, 8, 2, 0, 0), (777, 8, 2, 1, 0), (300, 64, 8, 0, 0), (513, 256, 8, 1, 0), (64, 256, 8, 0, 0),
    (40, 5, 5, 0, 0), (33, 1, 1, 0, 0), (1, 8, 2, 1, 0), (95, 512, 16, 0, 0), (200, 32, 1, 1, 0),
    (500, 8, 1, 0, 1), (300, 64, 2, 1, 1), (129, 256, 8, 0, 1),
])
def test_route_from_logits_bit_exact(T, E, k, mode, gm):
    rng = np.random.default_rng(T * 31 + E)
    z = rng.standard_normal((T, E)).astype(np.float32) * 2
    if E >= 3:
        z[::7, 1:3] = z[::7, 0:1]           # exact ties: the lower index must win
    bias = rng.uniform(-0.5, 0.5, E).astype(np.float32) if mode else None
    p = moe.problem(T, 64, 64, E, k, 0.0, "bf16", mode, gate_mode=gm)
    ws = moe.alloc_workspace(p, DEV)
    st = moe.alloc_stats(E, DEV)
    idx = torch.empty((T, k), dtype=torch.int32, device=DEV)
    gate = torch.empty((T, k), dtype=torch.float32, device=DEV)
    moe.route_from_logits(p, torch.from_numpy(z).to(DEV), idx, gate, st, ws,
                          bias=None if bias is None else torch.from_numpy(bias).to(DEV))
    torch.cuda.synchronize()
    r = O.route(z, k, bias, mode, key_dtype=np.float32, gate_mode=gm)
    assert np.array_equal(idx.cpu().numpy(), r.idx)
    assert np.allclose(gate.cpu().numpy(), r.gate, rtol=2e-6, atol=1e-7)
    s = moe.read_stats(st, E)
    perm = O.permute(r.idx, E)
    ls = O.load_stats(perm, r.probs, T, k, None, z=z)
    assert s.status == moe.MOE_OK
    assert s.counts == ls.counts.tolist()
    assert np.allclose(s.P, ls.P, rtol=1e-5, atol=1e-7)
    assert s.l_aux == pytest.approx(ls.l_aux, rel=TOL_LAUX)
    assert s.z_loss == pytest.approx(ls.z_loss, rel=1e-5)
    assert s.entropy == pytest.approx(ls.entropy, rel=1e-5, abs=1e-6)
    assert s.top_gap == pytest.approx(ls.top_gap, rel=1e-5, abs=1e-6)
    assert s.rows == T * k and s.dropped == 0 and s.capacity == -1


@pytest.mark.parametrize("T,E,k", [(500, 64, 8), (257, 256, 8), (100, 16, 4)])
def test_route_from_logits_prob_bias(T, E, k):
    # key = softmax(z) + b: the softmax is formed with each side's exp, so the
    # comparison excludes rows whose k-th / (k+1)-th key gap is within rounding
    rng = np.random.default_rng(E + k)
    z = rng.standard_normal((T, E)).astype(np.float32)
    bias = rng.uniform(-0.1, 0.1, E).astype(np.float32)
    p = moe.problem(T, 64, 64, E, k, 0.0, "bf16", moe.BIAS_PROB)
    ws = moe.alloc_workspace(p, DEV)
    st = moe.alloc_stats(E, DEV)
    idx = torch.empty((T, k), dtype=torch.int32, device=DEV)
    gate = torch.empty((T, k), dtype=torch.float32, device=DEV)
    moe.route_from_logits(p, torch.from_numpy(z).to(DEV), idx, gate, st, ws, bias=torch.from_numpy(bias).to(DEV))
    torch.cuda.synchronize()
    r = O.route(z, k, bias, O.BIAS_PROB)
    key = O.selection_key(z, bias, O.BIAS_PROB)
    m = key_margin(key, k)
    ok = m > 1e-6
    g_idx = idx.cpu().numpy()
    assert ok.mean() > 0.95
    assert np.array_equal(np.sort(g_idx[ok], axis=1), np.sort(r.idx[ok], axis=1))
    kg = np.take_along_axis(key, g_idx.astype(np.int64), axis=1)
    assert (np.diff(kg, axis=1) <= 1e-6).all()          # descending up to rounding
    # near-tie rows: the GPU's set must still be a valid top-k within rounding
    kth = -np.sort(-key, axis=1)[:, k - 1]
    for t in np.nonzero(~ok)[0]:
        assert (key[t, g_idx[t]] >= kth[t] - 1e-6).all()
    # gates matched by expert (slot order of near-tied keys may differ)
    for t in np.nonzero(ok)[0][:200]:
        want = dict(zip(r.idx[t].tolist(), r.gate[t].tolist()))
        for j in range(k):
            assert gate[t, j].item() == pytest.approx(want[int(g_idx[t, j])], rel=2e-6, abs=1e-7)


# --------------------------------------------------------------------------
# permutation
# --------------------------------------------------------------------------

@pytest.mark.parametrize("T,E,k,cf,dtype,drop", [
    (1000, 8, 2, 0.0, "bf16", 0), (1000, 8, 2, 0.6, "bf16", 0), (31, 4, 2, 0.5, "f32", 0), (1, 8, 2, 0.0, "bf16", 0),
    (2049, 256, 8, 1.0, "bf16", 0), (300, 64, 8, 0.3, "f32", 0), (64, 3, 3, 0.9, "bf16", 0),
    (4096, 8, 2, 1.25, "bf16", 0),
    (1000, 8, 2, 0.6, "bf16", 1), (2049, 256, 8, 1.0, "bf16", 1), (77, 6, 3, 0.4, "f32", 1), (1, 8, 2, 0.3, "bf16", 1),
])
def test_permute_bit_exact(T, E, k, cf, dtype, drop):
    rng = np.random.default_rng(T + E * 7)
    z = rng.standard_normal((T, E))
    z[:, 0] += 1.0                                    # skew toward expert 0 so capacity bites
    idx_np = O.topk_lowest_index(z, k)
    d = 128 if dtype == "bf16" else 64
    x = torch.randn((T, d), dtype=torch.float32).to(_dt(dtype)).to(DEV)
    p = moe.problem(T, d, 64, E, k, cf, dtype, drop_order=drop)
    ws = moe.alloc_workspace(p, DEV)
    st = moe.alloc_stats(E, DEV)
    idx = torch.from_numpy(idx_np.astype(np.int32)).to(DEV)
    pos = torch.empty((T, k), dtype=torch.int32, device=DEV)
    indptr = torch.empty((E + 1,), dtype=torch.int32, device=DEV)
    row_token = torch.full((T * k,), -7, dtype=torch.int32, device=DEV)
    xp = torch.zeros((T * k, d), dtype=_dt(dtype), device=DEV)
    moe.permute(p, x, idx, pos, indptr, row_token, xp, st, ws)
    torch.cuda.synchronize()
    C = O.capacity(cf, T, k, E)
    perm = O.permute(idx_np, E, C, drop)
    assert np.array_equal(pos.cpu().numpy(), perm.pos)
    assert np.array_equal(indptr.cpu().numpy(), perm.indptr)
    R = int(perm.indptr[-1])
    assert np.array_equal(row_token.cpu().numpy()[:R], perm.row_token)
    s = moe.read_stats(st, E)
    assert s.counts == perm.counts.tolist() and s.kept == perm.kept.tolist()
    assert s.rows == R and s.dropped == int((perm.counts - perm.kept).sum())
    assert s.capacity == (-1 if C is None else C)
    # gathered rows are bit copies of their token rows
    assert torch.equal(xp[:R].cpu(), x.cpu()[torch.from_numpy(perm.row_token)])


@pytest.mark.parametrize("T,E,k,cf,dtype,pad", [
    (1000, 8, 2, 0.6, "bf16", 128), (300, 64, 8, 0.0, "bf16", 64), (77, 6, 3, 0.4, "f32", 128),
    (2049, 256, 8, 1.0, "bf16", 128), (1, 8, 2, 0.0, "bf16", 64),
])
def test_permute_padded_bit_exact(T, E, k, cf, dtype, pad):
    rng = np.random.default_rng(T + E * 11)
    z = rng.standard_normal((T, E))
    z[:, 0] += 1.0
    idx_np = O.topk_lowest_index(z, k)
    d = 128 if dtype == "bf16" else 64
    x = torch.randn((T, d), dtype=torch.float32).to(_dt(dtype)).to(DEV)
    p = moe.problem(T, d, 64, E, k, cf, dtype, pad_rows=pad)
    Rmax = moe.permuted_rows(p)
    assert Rmax == T * k + E * (pad - 1)
    ws = moe.alloc_workspace(p, DEV)
    st = moe.alloc_stats(E, DEV)
    idx = torch.from_numpy(idx_np.astype(np.int32)).to(DEV)
    pos = torch.empty((T, k), dtype=torch.int32, device=DEV)
    indptr = torch.empty((E + 1,), dtype=torch.int32, device=DEV)
    row_token = torch.full((Rmax,), -7, dtype=torch.int32, device=DEV)
    xp = torch.full((Rmax, d), 3.0, dtype=_dt(dtype), device=DEV)     # padding must be overwritten
    moe.permute(p, x, idx, pos, indptr, row_token, xp, st, ws)
    torch.cuda.synchronize()
    C = O.capacity(cf, T, k, E)
    perm = O.permute(idx_np, E, C, O.DROP_TOKEN, pad=pad)
    assert np.array_equal(pos.cpu().numpy(), perm.pos)
    assert np.array_equal(indptr.cpu().numpy(), perm.indptr)
    R = int(perm.indptr[-1])
    assert R % pad == 0 or R == 0
    rt = row_token.cpu().numpy()
    assert np.array_equal(rt[:R], perm.row_token)
    s = moe.read_stats(st, E)
    assert s.kept == perm.kept.tolist() and s.rows == int(perm.kept.sum())
    xh = xp[:R].cpu()
    real = torch.from_numpy(perm.row_token >= 0)
    assert torch.equal(xh[real], x.cpu()[torch.from_numpy(perm.row_token[perm.row_token >= 0])])
    assert (xh[~real] == 0).all()


def test_padded_forward_equals_dense():
    # same kernels per row: padding moves rows to other tiles but computes
    # every kept row the same way (no split-K at these sizes)
    for cfg in (dict(T=600, d=256, d_ff=384, E=8, k=2, cf=0.7, dtype="bf16", bias_mode=1, d_ff_shared=0),
                dict(T=200, d=128, d_ff=128, E=32, k=4, cf=0.0, dtype="bf16", bias_mode=2, d_ff_shared=128),
                dict(T=300, d=64, d_ff=128, E=6, k=2, cf=0.0, dtype="f32", bias_mode=0, d_ff_shared=0)):
        L = to_device(_small_layer(cfg, seed=21))
        outs = []
        for pad in (0, 64, 128):
            p, out, st, ws = gpu_forward(dict(cfg, pad=pad), L)
            assert moe.read_stats(st, cfg["E"]).status == moe.MOE_OK
            outs.append(out.cpu())
        assert torch.equal(outs[0], outs[1]) and torch.equal(outs[0], outs[2])


# --------------------------------------------------------------------------
# expert GEMMs (tcgen05 for bf16, CUDA cores for fp32)
# --------------------------------------------------------------------------

@pytest.mark.parametrize("dtype,d,d_ff,counts,shared,T", [
    ("bf16", 512, 384, [0, 130, 1, 257], 128, 100),          # empty group, ragged tails, 8 k-blocks
    ("bf16", 256, 128, [128, 128, 128], 0, 64),              # exact tiles
    ("bf16", 1024, 256, [300], 0, 10),                       # 16 k-blocks: ring wraps 4 times
    ("bf16", 128, 512, [5, 0, 0, 700, 3], 192, 257),         # shared width != routed width
    ("f32", 128, 256, [0, 70, 1, 129], 64, 50),
    # groups wider than one band of M blocks (the GEMM runs a group's rows in
    # bands of about 32 MB): GEMM 1/3 with K = 7168 (17 blocks a band) over 18
    # blocks, GEMM 2 with K = 14336 (9 blocks a band) over 10 blocks
    ("bf16", 7168, 256, [70, 2300], 0, 10),
    ("bf16", 256, 14336, [1200, 3], 0, 10),
    # at least 512 rows per expert on average: CTA-pair tiles of 256 rows
    # (ragged, empty and single-row groups; the shared expert; a group of 11
    # pair M blocks over a band of 8 at K = 14336)
    ("bf16", 512, 384, [600, 0, 1300, 257], 0, 1100),
    ("bf16", 256, 256, [700, 900], 128, 800),
    ("bf16", 256, 14336, [2600, 3], 0, 10),
    ("bf16", 128, 128, [1, 1023], 0, 512),
    # at least 32 experts, mixed group sizes (every 32-row boundary: 1, 32,
    # 33, 64, 65, 96, 97, 128 rows), with and without the shared expert, and a
    # large group over several bands of M blocks at K = 14336 (the runs of the
    # same cases with the two-class schedules are in test_gpu_grid_split.py)
    ("bf16", 256, 384, [0, 1, 5, 31, 32, 33, 64, 65, 96, 97, 128, 129, 200, 300, 0, 7] + [3] * 16, 128, 800),
    ("bf16", 512, 256, [2, 40, 129, 700, 17, 0, 1, 90] * 4, 0, 2000),
    ("bf16", 256, 14336, [2500, 3, 7] + [1] * 29, 0, 10),
    # at most 16 permuted rows, no shared expert: GEMM 1/3 as weight-streaming
    # GEMVs up to 8 rows (one- to eight-row groups, empty groups, K = 64: one
    # half-size item per row and fewer items than K warps, N = 64: fewer
    # output groups than CTAs), split-K tiles above
    ("bf16", 512, 384, [0, 3, 0, 5], 0, 4),
    ("bf16", 256, 512, [16], 0, 16),
    ("bf16", 64, 128, [3, 0, 9, 4], 0, 8),
    ("bf16", 1024, 64, [1, 1, 0, 1, 1, 1, 1, 1], 0, 4),
])
def test_experts_stage(dtype, d, d_ff, counts, shared, T):
    E = len(counts)
    k = min(2, E)
    Tt = max(T, (sum(counts) + k - 1) // k)
    rows = Tt * k
    assert sum(counts) <= rows
    g = torch.Generator().manual_seed(d + d_ff)
    dt = _dt(dtype)
    xp = torch.randn((rows, d), generator=g).to(dt)
    W1 = (torch.randn((E, d_ff, d), generator=g) / math.sqrt(d)).to(dt)
    W3 = (torch.randn((E, d_ff, d), generator=g) / math.sqrt(d)).to(dt)
    W2 = (torch.randn((E, d, d_ff), generator=g) / math.sqrt(d_ff)).to(dt)
    x = torch.randn((Tt, d), generator=g).to(dt)
    sh = {}
    if shared:
        sh = dict(Ws1=(torch.randn((shared, d), generator=g) / math.sqrt(d)).to(dt),
                  Ws3=(torch.randn((shared, d), generator=g) / math.sqrt(d)).to(dt),
                  Ws2=(torch.randn((d, shared), generator=g) / math.sqrt(shared)).to(dt))
    indptr_np = np.concatenate([[0], np.cumsum(counts)]).astype(np.int32)
    p = moe.problem(Tt, d, d_ff, E, k, 0.0, dtype, 0, shared)
    ws = moe.alloc_workspace(p, DEV)
    st = moe.alloc_stats(E, DEV)
    o = torch.full((rows, d), float("nan"), dtype=dt, device=DEV)
    s = torch.empty((Tt, d), dtype=dt, device=DEV) if shared else None
    moe.experts(p, xp.to(DEV), torch.from_numpy(indptr_np).to(DEV), W1.to(DEV), W3.to(DEV), W2.to(DEV), o, ws,
                x=x.to(DEV), s=s, stats=st, **{n: v.to(DEV) for n, v in sh.items()})
    torch.cuda.synchronize()
    assert moe.read_stats(st, E).status == moe.MOE_OK
    tol = TOL_BF16 if dtype == "bf16" else TOL_F32
    on = o.float().cpu().numpy()
    for e in range(E):
        lo, hi = indptr_np[e], indptr_np[e + 1]
        if hi == lo:
            continue
        ref = O.swiglu_expert(xp[lo:hi].float().numpy(), W1[e].float().numpy(), W3[e].float().numpy(),
                              W2[e].float().numpy())
        assert_rows_close(on[lo:hi], ref, tol, f"expert {e}")
    # rows past the last group are never written
    R = indptr_np[-1]
    if R < rows:
        assert torch.isnan(o[R:].float()).all()
    if shared:
        ref = O.swiglu_expert(x.float().numpy(), sh["Ws1"].float().numpy(), sh["Ws3"].float().numpy(),
                              sh["Ws2"].float().numpy())
        assert_rows_close(s.float().cpu().numpy(), ref, tol, "shared expert")


# --------------------------------------------------------------------------
# combine
# --------------------------------------------------------------------------

@pytest.mark.parametrize("dtype,T,d,k,shared", [("bf16", 300, 256, 2, False), ("f32", 77, 64, 3, True),
                                                 ("bf16", 65, 7168, 8, True)])
def test_combine(dtype, T, d, k, shared):
    rng = np.random.default_rng(T + d)
    R = T * k
    perm_rows = rng.permutation(R)
    pos = perm_rows.reshape(T, k).astype(np.int32)
    pos[rng.random((T, k)) < 0.2] = -1
    pos[3] = -1                                           # a fully dropped token
    gate = rng.random((T, k)).astype(np.float32)
    dt = _dt(dtype)
    O_rows = torch.randn((R, d)).to(dt)
    S = torch.randn((T, d)).to(dt) if shared else None
    p = moe.problem(T, d, 64, 8, k, 0.0, dtype)
    out = torch.empty((T, d), dtype=dt, device=DEV)
    moe.combine(p, O_rows.to(DEV), torch.from_numpy(pos).to(DEV), torch.from_numpy(gate).to(DEV), out,
                s=None if S is None else S.to(DEV))
    torch.cuda.synchronize()
    ref = O.unpermute_combine(O_rows.float().numpy(), pos, gate, None if S is None else S.float().numpy())
    got = out.float().cpu().numpy()
    if dtype == "bf16":
        assert np.allclose(got, ref, rtol=2 ** -8, atol=1e-6)
    else:
        assert np.allclose(got, ref, rtol=1e-6, atol=1e-6)
    if not shared:
        assert np.abs(got[3]).max() == 0.0


# --------------------------------------------------------------------------
# end to end, small shapes, all tokens
# --------------------------------------------------------------------------

SMALL = [
    dict(T=300, d=256, d_ff=384, E=8, k=2, cf=0.0, dtype="bf16", bias_mode=0, d_ff_shared=0),
    dict(T=130, d=128, d_ff=128, E=64, k=8, cf=0.0, dtype="bf16", bias_mode=2, d_ff_shared=128),
    dict(T=1000, d=256, d_ff=256, E=8, k=2, cf=0.6, dtype="bf16", bias_mode=1, d_ff_shared=0),
    dict(T=33, d=128, d_ff=128, E=1, k=1, cf=0.0, dtype="bf16", bias_mode=0, d_ff_shared=0),
    dict(T=50, d=128, d_ff=192, E=4, k=4, cf=0.0, dtype="bf16", bias_mode=0, d_ff_shared=0),
    dict(T=1, d=512, d_ff=256, E=8, k=2, cf=0.0, dtype="bf16", bias_mode=0, d_ff_shared=0),
    dict(T=64, d=256, d_ff=128, E=256, k=8, cf=0.0, dtype="bf16", bias_mode=2, d_ff_shared=256),
    dict(T=257, d=64, d_ff=128, E=6, k=3, cf=0.25, dtype="f32", bias_mode=1, d_ff_shared=64),
    # T*k <= 128 rows: moe_forward may split K of both GEMMs (fp32 partials)
    dict(T=16, d=1024, d_ff=512, E=8, k=2, cf=0.0, dtype="bf16", bias_mode=0, d_ff_shared=0),
    dict(T=5, d=256, d_ff=1024, E=4, k=2, cf=0.0, dtype="bf16", bias_mode=1, d_ff_shared=0),
    # T*k <= 64, E % 8 == 0, E <= 64: the small-batch router
    dict(T=20, d=256, d_ff=256, E=64, k=2, cf=0.5, dtype="bf16", bias_mode=1, d_ff_shared=0),
    dict(T=8, d=512, d_ff=256, E=16, k=4, cf=0.0, dtype="bf16", bias_mode=2, d_ff_shared=0),
    dict(T=3, d=128, d_ff=128, E=8, k=8, cf=0.0, dtype="bf16", bias_mode=0, d_ff_shared=0),
    # T <= 8 on the small router, with every routing variant
    dict(T=8, d=256, d_ff=256, E=8, k=2, cf=0.5, dtype="bf16", bias_mode=1, d_ff_shared=0, gate=1, drop=1),
    dict(T=7, d=256, d_ff=384, E=32, k=2, cf=0.75, dtype="bf16", bias_mode=1, d_ff_shared=0),
    dict(T=6, d=128, d_ff=256, E=64, k=8, cf=0.0, dtype="bf16", bias_mode=0, d_ff_shared=0),
    dict(T=4, d=192, d_ff=256, E=8, k=2, cf=0.0, dtype="bf16", bias_mode=0, d_ff_shared=0),
    # routing variants: Switch full-softmax gates, GShard slot-priority drops
    dict(T=500, d=256, d_ff=256, E=8, k=1, cf=1.0, dtype="bf16", bias_mode=0, d_ff_shared=0, gate=1, drop=0),
    dict(T=700, d=128, d_ff=256, E=16, k=2, cf=0.7, dtype="bf16", bias_mode=1, d_ff_shared=0, gate=0, drop=1),
    dict(T=24, d=256, d_ff=128, E=8, k=2, cf=0.6, dtype="bf16", bias_mode=1, d_ff_shared=0, gate=1, drop=1),
    dict(T=200, d=64, d_ff=64, E=6, k=3, cf=0.5, dtype="f32", bias_mode=0, d_ff_shared=0, gate=1, drop=1),
    # at least 512 rows per expert on average: CTA-pair tiles of 256 rows
    dict(T=2048, d=256, d_ff=384, E=4, k=2, cf=0.0, dtype="bf16", bias_mode=0, d_ff_shared=0),
    dict(T=3000, d=128, d_ff=256, E=4, k=2, cf=0.9, dtype="bf16", bias_mode=1, d_ff_shared=0, gate=1, drop=1),
    dict(T=1024, d=128, d_ff=128, E=2, k=1, cf=0.0, dtype="bf16", bias_mode=2, d_ff_shared=128),
    dict(T=600, d=192, d_ff=320, E=1, k=1, cf=0.0, dtype="bf16", bias_mode=0, d_ff_shared=0),
    # 32 or more experts, many small groups
    dict(T=400, d=256, d_ff=256, E=32, k=4, cf=0.0, dtype="bf16", bias_mode=2, d_ff_shared=0),
    # the largest expert count (MOE_MAX_E: tensor-core router, 512 groups)
    # and the largest k (MOE_MAX_K)
    dict(T=300, d=256, d_ff=128, E=512, k=8, cf=0.0, dtype="bf16", bias_mode=2, d_ff_shared=128),
    dict(T=100, d=128, d_ff=128, E=64, k=16, cf=0.0, dtype="bf16", bias_mode=0, d_ff_shared=0),
    dict(T=900, d=128, d_ff=384, E=64, k=6, cf=0.8, dtype="bf16", bias_mode=1, d_ff_shared=128, gate=1),
    # padded (MegaBlocks) layout: every expert's rows rounded up to 128 or 64
    dict(T=300, d=256, d_ff=384, E=8, k=2, cf=0.0, dtype="bf16", bias_mode=0, d_ff_shared=0, pad=128),
    dict(T=1000, d=256, d_ff=256, E=8, k=2, cf=0.6, dtype="bf16", bias_mode=1, d_ff_shared=0, pad=64),
    dict(T=130, d=128, d_ff=128, E=64, k=8, cf=0.0, dtype="bf16", bias_mode=2, d_ff_shared=128, pad=128),
    dict(T=20, d=256, d_ff=256, E=8, k=2, cf=0.0, dtype="bf16", bias_mode=0, d_ff_shared=0, pad=128),
    dict(T=257, d=64, d_ff=128, E=6, k=3, cf=0.25, dtype="f32", bias_mode=1, d_ff_shared=64, pad=128),
]


def _small_layer(cfg, seed):
    g = torch.Generator().manual_seed(seed)
    dt = _dt(cfg["dtype"])
    T, d, dff, E, dfs = cfg["T"], cfg["d"], cfg["d_ff"], cfg["E"], cfg["d_ff_shared"]
    L = dict(x=torch.randn((T, d), generator=g).to(dt),
             W_r=(torch.randn((d, E), generator=g) / math.sqrt(d)).to(dt),
             W1=(torch.randn((E, dff, d), generator=g) / math.sqrt(d)).to(dt),
             W3=(torch.randn((E, dff, d), generator=g) / math.sqrt(d)).to(dt),
             W2=(torch.randn((E, d, dff), generator=g) / math.sqrt(dff)).to(dt),
             bias=None, Ws1=None, Ws3=None, Ws2=None)
    if cfg["bias_mode"] == 1:
        L["bias"] = torch.linspace(1.0, -1.0, E)
    elif cfg["bias_mode"] == 2:
        L["bias"] = torch.rand((E,), generator=g) * 0.2 - 0.1
    if dfs:
        L["Ws1"] = (torch.randn((dfs, d), generator=g) / math.sqrt(d)).to(dt)
        L["Ws3"] = (torch.randn((dfs, d), generator=g) / math.sqrt(d)).to(dt)
        L["Ws2"] = (torch.randn((d, dfs), generator=g) / math.sqrt(dfs)).to(dt)
    return L


def _check_forward(cfg, L_cpu, tokens=None, check_own_routing=True):
    """Run the CUDA forward and compare with the oracle; returns the errors."""
    L = to_device(L_cpu)
    p, out, st, ws = gpu_forward(cfg, L)
    T, k, E = cfg["T"], cfg["k"], cfg["E"]
    s = moe.read_stats(st, E)
    assert s.status == moe.MOE_OK
    logits = moe.workspace_view(ws, p, "logits").cpu().numpy()
    g_idx = moe.workspace_view(ws, p, "idx").cpu().numpy()
    g_pos = moe.workspace_view(ws, p, "pos").cpu().numpy()
    x_np = np32(L_cpu["x"])
    bias = None if L_cpu["bias"] is None else L_cpu["bias"].float().numpy()
    W = oracle_weights(L_cpu)
    # (1) oracle consuming the GPU's logits: routing, drops, outputs
    exact_key = cfg["bias_mode"] != O.BIAS_PROB
    res = O.moe_forward(x_np, None, W["W1"], W["W3"], W["W2"], k, cfg["cf"], bias, cfg["bias_mode"],
                        W["Ws1"], W["Ws3"], W["Ws2"], logits=logits, tokens=tokens,
                        key_dtype=np.float32 if exact_key else np.float64,
                        gate_mode=cfg.get("gate", 0), drop_order=cfg.get("drop", 0),
                        pad=cfg.get("pad") or None)
    if exact_key:
        assert np.array_equal(g_idx, res.routing.idx)
        assert np.array_equal(g_pos, res.perm.pos)
        assert s.counts == res.stats.counts.tolist()
        assert s.kept == res.stats.kept.tolist()
        assert s.dropped == res.stats.dropped
        good = np.ones(T, dtype=bool)
    else:
        # softmax keys are formed with each side's exp: compare the selected
        # set away from k-th/(k+1)-th near-ties; inside the set, near-tied keys
        # may be ordered either way, so check the order against rounding
        m = key_margin(res.routing.key, k)
        good = m > 1e-6
        assert good.mean() > 0.99
        assert np.array_equal(np.sort(g_idx[good], axis=1), np.sort(res.routing.idx[good], axis=1))
        kg = np.take_along_axis(res.routing.key, g_idx.astype(np.int64), axis=1)
        assert (np.diff(kg, axis=1) <= 1e-6).all()
        assert cfg["cf"] <= 0, "PROB-key parity with capacity needs a drop-set argument"
    assert s.l_aux == pytest.approx(res.stats.l_aux, rel=TOL_LAUX)
    assert s.z_loss == pytest.approx(res.stats.z_loss, rel=1e-4)
    assert s.entropy == pytest.approx(res.stats.entropy, rel=1e-4, abs=1e-6)
    assert s.top_gap == pytest.approx(res.stats.top_gap, rel=1e-4, abs=1e-6)
    toks = res.tokens
    sel = good[toks]
    got_all = out.float().cpu().numpy()
    got = got_all[toks]
    tol = TOL_BF16 if cfg["dtype"] == "bf16" else TOL_F32
    rel, _, _ = assert_rows_close(got[sel], res.y[sel], tol, "oracle on the GPU's logits")
    # (2) the GPU's logits against the fp32-accumulation bound: each logit is
    # a d-term dot product of values exact in fp32, so any fp32 summation
    # order is within gamma_d * sum_i |x_i w_i| (gamma_d = d u / (1 - d u),
    # u = 2^-24, 2.4e-4 at d = 4096); summation errors of random sign grow
    # like sqrt(d) u, so 1e-5 * sum_i |x_i w_i| is a bar well above real
    # rounding and far below a wrong term or weight
    W_r64 = np32(L_cpu["W_r"]).astype(np.float64)
    z64 = O.router_logits(x_np, W_r64)
    absdot = np.abs(x_np.astype(np.float64)) @ np.abs(W_r64)
    assert (np.abs(z64 - logits) <= 1e-5 * absdot + 1e-30).all(), float(np.max(np.abs(z64 - logits) / absdot))
    # (3) the oracle's own fp64 routing: indices equal away from near-ties,
    # and the outputs of every token whose selection and kept slots both
    # sides agree on, element by element
    if check_own_routing:
        key64 = O.selection_key(z64, bias, cfg["bias_mode"])
        own = O.topk_lowest_index(key64, k)
        far = key_margin(key64, k) >= MARGIN
        assert np.array_equal(g_idx[far], own[far])
        res64 = O.moe_forward(x_np, W_r64, W["W1"], W["W3"], W["W2"], k, cfg["cf"], bias, cfg["bias_mode"],
                              W["Ws1"], W["Ws3"], W["Ws2"], tokens=toks, gate_mode=cfg.get("gate", 0),
                              drop_order=cfg.get("drop", 0), pad=cfg.get("pad") or None)
        # the same experts, kept the same way (slot order may differ where
        # keys inside the selected set are within rounding of each other: the
        # output is a sum over slots)
        def kept_sets(idx, pos):
            return np.sort(np.where(pos >= 0, idx, -1), axis=1)
        o_idx, o_pos = res64.routing.idx[toks], res64.perm.pos[toks]
        same = far[toks] & (np.sort(g_idx[toks], axis=1) == np.sort(o_idx, axis=1)).all(axis=1) \
            & (kept_sets(g_idx[toks], g_pos[toks]) == kept_sets(o_idx, o_pos)).all(axis=1)
        # away from near-ties the selections agree everywhere; the kept sets
        # differ only where another token's flipped near-tie moved a pair across
        # the capacity boundary
        assert same[far[toks]].mean() >= 0.9, (same[far[toks]].mean(), far.mean())
        assert_rows_close(got[same], res64.y[same], tol, "oracle on its own fp64 routing")
    return rel


@pytest.mark.parametrize("cfg", SMALL, ids=[f"T{c['T']}_E{c['E']}_k{c['k']}_{c['dtype']}_b{c['bias_mode']}"
                                            f"_cf{c['cf']}_s{c['d_ff_shared']}_g{c.get('gate', 0)}"
                                            f"_d{c.get('drop', 0)}_p{c.get('pad', 0)}" for c in SMALL])
def test_forward_small(cfg):
    _check_forward(cfg, _small_layer(cfg, cfg["T"] + cfg["E"]))


def test_forward_zero_tokens():
    cfg = dict(T=0, d=128, d_ff=128, E=8, k=2, cf=1.0, dtype="bf16", bias_mode=0, d_ff_shared=0)
    p = problem_of(cfg)
    ws = moe.alloc_workspace(p, DEV)
    st = moe.alloc_stats(8, DEV)
    W = torch.zeros((8, 128, 128), dtype=torch.bfloat16, device=DEV)
    W_r = torch.zeros((128, 8), dtype=torch.bfloat16, device=DEV)
    # zero-size tensors may carry a null pointer: pass 16-byte aligned stand-ins
    x = torch.empty((1, 128), dtype=torch.bfloat16, device=DEV)
    out = torch.empty((1, 128), dtype=torch.bfloat16, device=DEV)
    moe.forward(p, x, W_r, W, W, W, out, st, ws)
    torch.cuda.synchronize()
    s = moe.read_stats(st, 8)
    assert s.status == 0 and s.rows == 0 and s.counts == [0] * 8 and s.l_aux == 0.0


def test_forward_toy_fp32_full():
    cfg = inputs.workload("toy_fp32")
    L = inputs.make_layer(cfg, seed=0)
    rel = _check_forward(cfg, L)
    assert rel < TOL_F32


# --------------------------------------------------------------------------
# determinism and stage composition
# --------------------------------------------------------------------------

def test_forward_is_deterministic():
    cfg = dict(T=1000, d=256, d_ff=256, E=8, k=2, cf=0.6, dtype="bf16", bias_mode=1, d_ff_shared=128)
    L = to_device(_small_layer(cfg, 5))
    _, out1, st1, _ = gpu_forward(cfg, L)
    _, out2, st2, _ = gpu_forward(cfg, L)
    assert torch.equal(out1, out2)
    assert torch.equal(st1, st2)


def test_stages_compose_to_forward():
    cfg = dict(T=500, d=256, d_ff=384, E=16, k=4, cf=0.8, dtype="bf16", bias_mode=1, d_ff_shared=128)
    L = to_device(_small_layer(cfg, 9))
    p, out, st, ws = gpu_forward(cfg, L)
    T, d, E, k = cfg["T"], cfg["d"], cfg["E"], cfg["k"]
    ws2 = moe.alloc_workspace(p, DEV)
    st2 = moe.alloc_stats(E, DEV)
    idx = torch.empty((T, k), dtype=torch.int32, device=DEV)
    gate = torch.empty((T, k), dtype=torch.float32, device=DEV)
    logits = torch.empty((T, E), dtype=torch.float32, device=DEV)
    moe.route(p, L["x"], L["W_r"], idx, gate, st2, ws2, bias=L["bias"], logits=logits)
    pos = torch.empty((T, k), dtype=torch.int32, device=DEV)
    indptr = torch.empty((E + 1,), dtype=torch.int32, device=DEV)
    row_token = torch.empty((T * k,), dtype=torch.int32, device=DEV)
    xp = torch.empty((T * k, d), dtype=torch.bfloat16, device=DEV)
    moe.permute(p, L["x"], idx, pos, indptr, row_token, xp, st2, ws2)
    o = torch.empty((T * k, d), dtype=torch.bfloat16, device=DEV)
    s = torch.empty((T, d), dtype=torch.bfloat16, device=DEV)
    moe.experts(p, xp, indptr, L["W1"], L["W3"], L["W2"], o, ws2, x=L["x"], Ws1=L["Ws1"], Ws3=L["Ws3"],
                Ws2=L["Ws2"], s=s)
    out2 = torch.empty_like(out)
    moe.combine(p, o, pos, gate, out2, s=s)
    torch.cuda.synchronize()
    assert torch.equal(moe.workspace_view(ws, p, "idx"), idx)
    assert torch.equal(moe.workspace_view(ws, p, "pos"), pos)
    assert torch.equal(out, out2)


@pytest.mark.parametrize("cfg", [
    dict(T=4, d=512, d_ff=512, E=8, k=2, cf=0.0, dtype="bf16", bias_mode=0, d_ff_shared=0),
    dict(T=40, d=512, d_ff=512, E=8, k=2, cf=0.0, dtype="bf16", bias_mode=0, d_ff_shared=0),
    dict(T=600, d=256, d_ff=384, E=16, k=4, cf=0.8, dtype="bf16", bias_mode=1, d_ff_shared=128),
], ids=["decode_gemv_pdl", "decode_split_pdl", "general_pdl"])
def test_forward_captures_in_a_cuda_graph(cfg):
    # moe_forward is asynchronous and allocation-free: captured once and
    # replayed, it gives the eager call's bits
    L = to_device(_small_layer(cfg, 21))
    p, out, st, ws = gpu_forward(cfg, L)
    out_g = torch.empty_like(out)
    st_g = moe.alloc_stats(cfg["E"], DEV)
    ws_g = moe.alloc_workspace(p, DEV)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        moe.forward(p, L["x"], L["W_r"], L["W1"], L["W3"], L["W2"], out_g, st_g, ws_g, bias=L["bias"],
                    Ws1=L["Ws1"], Ws3=L["Ws3"], Ws2=L["Ws2"])
    for _ in range(2):
        out_g.zero_()
        g.replay()
    torch.cuda.synchronize()
    assert torch.equal(out, out_g)
    assert torch.equal(st, st_g)
    del g


# --------------------------------------------------------------------------
# full-size workloads: routing on all tokens, outputs on sampled tokens
# --------------------------------------------------------------------------

def _sample_tokens(pos, indptr, rng, n_random):
    """Every expert's first and last kept rows, rows at the capacity edge,
    fully dropped tokens, and random tokens."""
    T = pos.shape[0]
    picks = set(rng.choice(T, size=min(n_random, T), replace=False).tolist())
    R = int(indptr[-1])
    row_of = {}
    for t in range(T):
        for j in range(pos.shape[1]):
            if pos[t, j] >= 0:
                row_of[int(pos[t, j])] = t
    for e in range(len(indptr) - 1):
        lo, hi = int(indptr[e]), int(indptr[e + 1])
        rows = [r for r in (lo, hi - 1) if r in row_of]
        while hi - 1 > lo and hi - 1 not in row_of:   # padded layout: last kept row
            hi -= 1
        if hi - 1 in row_of:
            rows.append(hi - 1)
        picks.update(row_of[r] for r in rows)
    dropped = np.nonzero((pos < 0).all(axis=1))[0]
    picks.update(dropped[:4].tolist())
    return np.array(sorted(picks))


@pytest.mark.parametrize("name,n_random,pad", [("mixtral_prefill", 24, 0), ("skewed_capacity", 16, 0),
                                               ("deepseek_v3", 6, 0), ("mixtral_prefill", 8, 128)])
def test_forward_full_size(name, n_random, pad):
    cfg = dict(inputs.workload(name), pad=pad)
    # the kernel each full-size workload exercises
    want = {"mixtral_prefill": "single" if pad else "pair", "skewed_capacity": "pair", "deepseek_v3": "single"}
    if not any(v in os.environ for v in ("MOE_CTA_PAIR", "MOE_SMALL_CTAS", "MOE_INTERLEAVE")):
        assert moe.gemm_variant(problem_of(cfg)) == want[name]
    L = inputs.make_layer(cfg, seed=0, device="cpu", weights_device=DEV)
    Ld = to_device(L)
    p, out, st, ws = gpu_forward(cfg, Ld)
    pos = moe.workspace_view(ws, p, "pos").cpu().numpy()
    indptr = moe.workspace_view(ws, p, "indptr").cpu().numpy()
    rng = np.random.default_rng(0)
    toks = _sample_tokens(pos, indptr, rng, n_random)
    if name == "deepseek_v3":
        toks = toks[:40]
    _check_forward(cfg, L, tokens=toks)
    s = moe.read_stats(st, cfg["E"])
    if name == "skewed_capacity":
        assert s.capacity == 5120 and s.dropped > 0


def test_decode_experts_touched_fraction():
    # the decode sweep's routing, with a fresh router matrix per trial: the
    # mean fraction of experts the GPU router touches matches
    # 1 - (C(E-1, k) / C(E, k))^T within 3 sigma of the trials' mean
    E, k, d, trials = 8, 2, 4096, 1000
    g = torch.Generator(device=DEV)
    g.manual_seed(1234)
    for T in inputs.DECODE_TOKENS:
        p = moe.problem(T, d, 14336, E, k, 0.0, "bf16", 0, 0)
        ws = moe.alloc_workspace(p, DEV)
        st = moe.alloc_stats(E, DEV)
        x = torch.randn((T, d), generator=g, device=DEV).to(torch.bfloat16)
        idx = torch.empty((T, k), dtype=torch.int32, device=DEV)
        gate = torch.empty((T, k), dtype=torch.float32, device=DEV)
        picks = torch.empty((trials, T, k), dtype=torch.int32, device=DEV)
        for i in range(trials):
            W_r = (torch.randn((d, E), generator=g, device=DEV) / math.sqrt(d)).to(torch.bfloat16)
            moe.route(p, x, W_r, idx, gate, st, ws)
            picks[i].copy_(idx)
        torch.cuda.synchronize()
        pk = picks.cpu().numpy().reshape(trials, T * k)
        assert ((pk >= 0) & (pk < E)).all()
        fr = np.array([len(set(row.tolist())) / E for row in pk])
        expect = O.fraction_experts_touched(E, k, T)
        # standard deviation of one trial's fraction under uniform k-subsets:
        # N = experts touched, P(e missed) = q^T, P(e and e' missed) = r^T
        q = math.comb(E - 1, k) / math.comb(E, k)
        r = math.comb(E - 2, k) / math.comb(E, k)
        pt = 1 - q ** T
        var_n = E * pt * (1 - pt) + E * (E - 1) * (1 - 2 * q ** T + r ** T - pt * pt)
        sigma = math.sqrt(max(var_n, 0.0)) / E / math.sqrt(trials)
        assert abs(fr.mean() - expect) <= 3 * sigma + 1e-12, (T, fr.mean(), expect, sigma)


@pytest.mark.parametrize("T", inputs.DECODE_TOKENS)
def test_forward_decode(T):
    cfg = inputs.workload(f"decode_t{T}")
    L = inputs.make_layer(cfg, seed=0, device="cpu", weights_device=DEV)
    _check_forward(cfg, L)
