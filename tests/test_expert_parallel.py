"""Expert parallelism on CPU: world sizes 2 and 4 over gloo.

Every rank routes and permutes its own token shard (with the oracle, on the
CPU), then plan / dispatch / run_local_experts / combine_back move the rows
to the ranks that own their experts and back, and forward_overlapped does
the same exchange in rounds that overlap the local experts. The local experts use only
the owner's slice of the weights. Each rank's output must equal the oracle's
single-process forward of its tokens with all the experts, drops included.
"""

import math
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from mixture_experts_layer_62_b200 import expert_parallel as ep
from mixture_experts_layer_62_b200 import parallel
from oracle import moe_oracle as O

T, d, d_ff, E, k, CF = 157, 16, 24, 8, 2, 1.0


def _layer():
    rng = np.random.default_rng(3)
    x = rng.standard_normal((T, d))
    W_r = rng.standard_normal((d, E)) / math.sqrt(d)
    W1 = rng.standard_normal((E, d_ff, d)) / math.sqrt(d)
    W3 = rng.standard_normal((E, d_ff, d)) / math.sqrt(d)
    W2 = rng.standard_normal((E, d, d_ff)) / math.sqrt(d_ff)
    return x, W_r, W1, W3, W2


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=__import__("datetime").timedelta(seconds=60))
    try:
        x, W_r, W1, W3, W2 = _layer()
        lo, hi = parallel.shard_range(T, world, rank)
        xr = x[lo:hi]
        e_lo, e_hi = ep.expert_range(E, world, rank)
        W1l, W3l, W2l = W1[e_lo:e_hi], W3[e_lo:e_hi], W2[e_lo:e_hi]   # this rank's experts only

        # routing and permutation of the rank's own tokens (per-rank capacity)
        r = O.route(O.router_logits(xr, W_r), k)
        perm = O.permute(r.idx, E, O.capacity(CF, hi - lo, k, E))
        xp = torch.from_numpy(xr[perm.row_token])
        p = ep.plan(torch.from_numpy(perm.indptr), E)
        assert p.rows_out == int(perm.indptr[-1])

        rows = ep.dispatch(xp, p)

        def experts_fn(block, offsets):
            b = block.numpy()
            out = np.empty((b.shape[0], d))
            for e in range(p.E_local):
                s, t = int(offsets[e]), int(offsets[e + 1])
                if t > s:
                    out[s:t] = O.swiglu_expert(b[s:t], W1l[e], W3l[e], W2l[e])
            return torch.from_numpy(out)

        expert_out = ep.run_local_experts(rows, p, experts_fn, d)
        o = torch.zeros((p.rows_out, d), dtype=torch.float64)
        ep.combine_back(expert_out, p, o)
        y = O.unpermute_combine(o.numpy(), perm.pos, r.gate)

        # the overlapped exchange (rounds of paired sends and receives, one
        # block's experts running while the next block moves) gives the same
        # rows in the same places
        o2 = torch.full((p.rows_out, d), float("nan"), dtype=torch.float64)
        ep.forward_overlapped(xp, p, experts_fn, o2)
        same = bool(torch.equal(o, o2))

        ref = O.moe_forward(xr, W_r, W1, W3, W2, k, CF)
        err = float(np.abs(y - ref.y).max() / max(1e-30, np.abs(ref.y).max()))
        q.put((rank, err, int(perm.kept.sum()), int(ref.stats.dropped), p.rows_in, same))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 4])
def test_expert_parallel_matches_single_process(world):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for pr in procs:
        pr.start()
    res = [q.get(timeout=120) for _ in range(world)]
    for pr in procs:
        pr.join(timeout=60)
        assert pr.exitcode == 0
    res.sort()
    assert all(err < 1e-12 for _, err, _, _, _, _ in res), res
    assert all(same for *_, same in res), res
    # some pairs were dropped by the per-rank capacity, and every kept row
    # was computed by exactly one owner
    assert sum(dr for _, _, _, dr, _, _ in res) > 0
    assert sum(kept for _, _, kept, _, _, _ in res) == sum(n for _, _, _, _, n, _ in res)


def test_expert_range_requires_an_even_split():
    assert ep.expert_range(8, 4, 3) == (6, 8)
    with pytest.raises(ValueError):
        ep.expert_range(8, 3, 0)


def _fake_library(monkeypatch, E_l, dd, dff, calls, allocs):
    """The library's expert stage as a CPU fake that checks what it is
    handed (a problem of n tokens, one slot each, over the local experts;
    int32 offsets; a workspace at least moe_workspace_size) and computes
    with the oracle; workspace allocations are recorded."""
    import mixture_experts_layer_62_b200 as moe

    def ws_size(p):
        return 1000 + 10 * p.T

    def fake_experts(p, xp, indptr, w1, w3, w2, o, ws, **kw):
        assert (p.T, p.d, p.d_ff, p.E, p.k) == (xp.shape[0], dd, dff, E_l, 1)
        assert indptr.dtype == torch.int32 and indptr.shape == (E_l + 1,) and int(indptr[-1]) == xp.shape[0]
        assert ws.numel() >= ws_size(p)
        assert kw.get("stats") is not None
        ip = indptr.tolist()
        for e in range(E_l):
            if ip[e + 1] > ip[e]:
                o[ip[e]:ip[e + 1]] = torch.from_numpy(O.swiglu_expert(
                    xp[ip[e]:ip[e + 1]].numpy(), w1[e].numpy(), w3[e].numpy(), w2[e].numpy()))
        calls.append(xp.shape[0])

    real_empty = torch.empty

    def counting_empty(*shape, dtype=None, device=None, **kw):
        t = real_empty(*shape, dtype=dtype, **kw)
        if dtype == torch.uint8:
            allocs.append(t.numel())
        return t

    monkeypatch.setattr(moe, "experts", fake_experts)
    monkeypatch.setattr(moe, "workspace_size", ws_size)
    monkeypatch.setattr(moe, "alloc_stats", lambda E, device=None: real_empty(64, dtype=torch.uint8))
    monkeypatch.setattr(moe, "problem", lambda T, d, d_ff, E, k, cf, dtype: types_ns(T, d, d_ff, E, k))
    monkeypatch.setattr(ep.torch, "empty", counting_empty)


def _weights(rng, E_l, dd, dff):
    return (torch.from_numpy(rng.standard_normal((E_l, dff, dd))),
            torch.from_numpy(rng.standard_normal((E_l, dff, dd))),
            torch.from_numpy(rng.standard_normal((E_l, dd, dff))))


def test_library_experts_fn_wiring(monkeypatch):
    rng = np.random.default_rng(5)
    E_l, dd, dff = 3, 8, 12
    W1, W3, W2 = _weights(rng, E_l, dd, dff)
    calls, allocs = [], []
    _fake_library(monkeypatch, E_l, dd, dff, calls, allocs)
    fn = ep.library_experts_fn(W1, W3, W2)
    block = torch.from_numpy(rng.standard_normal((7, dd)))
    offsets = torch.tensor([0, 2, 2, 7], dtype=torch.int64)
    got = fn(block, offsets).numpy()
    want = np.concatenate([O.swiglu_expert(block[0:2].numpy(), W1[0].numpy(), W3[0].numpy(), W2[0].numpy()),
                           O.swiglu_expert(block[2:7].numpy(), W1[2].numpy(), W3[2].numpy(), W2[2].numpy())])
    assert np.allclose(got, want, rtol=0, atol=1e-12) and calls == [7]


@pytest.mark.parametrize("max_rows", [None, 40])
def test_library_experts_fn_keeps_one_workspace(monkeypatch, max_rows):
    # block sizes change from step to step: one workspace is held, replaced
    # only when a block needs more (or sized once from max_rows)
    rng = np.random.default_rng(6)
    E_l, dd, dff = 2, 8, 8
    W1, W3, W2 = _weights(rng, E_l, dd, dff)
    calls, allocs = [], []
    _fake_library(monkeypatch, E_l, dd, dff, calls, allocs)
    fn = ep.library_experts_fn(W1, W3, W2, max_rows=max_rows)
    sizes = [7, 3, 12, 5, 12, 9, 30, 1, 30, 2]
    for n in sizes:
        block = torch.from_numpy(rng.standard_normal((n, dd)))
        offsets = torch.tensor([0, n // 2, n], dtype=torch.int64)
        fn(block, offsets)
    assert calls == sizes
    if max_rows is None:
        assert allocs == [1000 + 10 * n for n in (7, 12, 30)]      # grows, never per size
    else:
        assert allocs == [1000 + 10 * max_rows]                   # once, up front
    assert fn.state["ws"].numel() == allocs[-1]


def types_ns(T, d, d_ff, E, k):
    import types
    return types.SimpleNamespace(T=T, d=d, d_ff=d_ff, E=E, k=k)


# rows per (source rank, expert) with empty pairs: rank 2 sends nothing,
# owner 1 gets nothing from ranks 0 and 3, rank 3 keeps everything local
_COUNTS = {0: [3, 0, 0, 0, 1, 2, 0, 0],
           1: [0, 1, 0, 0, 0, 0, 2, 1],
           2: [0, 0, 0, 0, 0, 0, 0, 0],
           3: [0, 0, 0, 0, 0, 0, 4, 0]}


def _edge_worker(rank, world, port, q):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=__import__("datetime").timedelta(seconds=60))
    try:
        counts = _COUNTS[rank]
        indptr = torch.tensor(np.concatenate([[0], np.cumsum(counts)]), dtype=torch.int64)
        n = int(indptr[-1])
        xp = torch.arange(n * 4, dtype=torch.float64).reshape(n, 4) + 100.0 * rank
        p = ep.plan(indptr, 8)
        e_lo, _ = ep.expert_range(8, world, rank)

        def experts_fn(block, offsets):
            # expert e of this owner scales its rows by (global expert id + 1)
            out = torch.empty_like(block)
            for e in range(p.E_local):
                s, t = int(offsets[e]), int(offsets[e + 1])
                out[s:t] = block[s:t] * (e_lo + e + 1)
            return out

        o = torch.zeros((n, 4), dtype=torch.float64)
        ep.combine_back(ep.run_local_experts(ep.dispatch(xp, p), p, experts_fn, 4), p, o)
        o2 = torch.full((n, 4), float("nan"), dtype=torch.float64)
        ep.forward_overlapped(xp, p, experts_fn, o2)
        scale = torch.repeat_interleave(torch.arange(1, 9, dtype=torch.float64), torch.tensor(counts))
        q.put((rank, bool(torch.equal(o, o2)), bool(torch.equal(o2, xp * scale[:, None]))))
    finally:
        dist.destroy_process_group()


def test_overlapped_exchange_with_empty_pairs():
    world = 4
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_edge_worker, args=(r, world, port, q)) for r in range(world)]
    for pr in procs:
        pr.start()
    res = sorted(q.get(timeout=120) for _ in range(world))
    for pr in procs:
        pr.join(timeout=60)
        assert pr.exitcode == 0
    assert all(a and b for _, a, b in res), res
