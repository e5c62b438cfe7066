"""Data-parallel replicas on CPU: world_size 2 over gloo.

Each rank routes its own token shard with the oracle, packs the statistics
into the library's statistics-block layout and calls global_stats (one
all-reduce); the result must equal the oracle's statistics of the whole
batch: counts exactly, f and P to fp32 rounding, L_aux within 1e-6.
"""

import math
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from mixture_experts_layer_62_b200 import parallel
from oracle import moe_oracle as O

T, d, E, k = 203, 32, 8, 2


def _data():
    rng = np.random.default_rng(0)
    x = rng.standard_normal((T, d))
    W_r = rng.standard_normal((d, E)) / math.sqrt(d)
    return x, W_r


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=__import__("datetime").timedelta(seconds=60))
    try:
        x, W_r = _data()
        lo, hi = parallel.shard_range(T, world, rank)
        z = O.router_logits(x[lo:hi], W_r)
        r = O.route(z, k)
        perm = O.permute(r.idx, E, O.capacity(0.0, hi - lo, k, E))
        st = O.load_stats(perm, r.probs, hi - lo, k, None)
        blk = parallel.stats_block_from_parts(st.counts.tolist(), st.kept.tolist(), st.P.tolist())
        g = parallel.global_stats(blk, E, k, hi - lo)
        q.put((rank, g.T, g.counts.tolist(), g.f.tolist(), g.P.tolist(), g.l_aux, g.max_over_mean))
    finally:
        dist.destroy_process_group()


def test_shard_range_covers_every_token_once():
    for Tg in (0, 1, 7, 203, 4096):
        for world in (1, 2, 3, 8):
            got = []
            for r in range(world):
                lo, hi = parallel.shard_range(Tg, world, r)
                got.extend(range(lo, hi))
            assert got == list(range(Tg))


def test_global_stats_two_gloo_ranks_match_full_batch():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    results = [q.get(timeout=120) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    x, W_r = _data()
    z = O.router_logits(x, W_r)
    r = O.route(z, k)
    perm = O.permute(r.idx, E)
    ref = O.load_stats(perm, r.probs, T, k, None)
    for rank, Tg, counts, f, P, l_aux, mom in results:
        assert Tg == T
        assert counts == ref.counts.tolist()
        assert np.allclose(f, ref.f, rtol=0, atol=1e-15)
        assert np.allclose(P, ref.P, rtol=1e-6)
        assert l_aux == pytest.approx(ref.l_aux, rel=1e-6)
        assert mom == pytest.approx(ref.max_over_mean)
    # both ranks hold the same global statistics
    assert results[0][1:] == results[1][1:]


def test_global_stats_single_process_is_identity():
    blk = parallel.stats_block_from_parts([3, 1, 0, 2], [3, 1, 0, 1], [0.5, 0.2, 0.1, 0.2], dropped=1)
    g = parallel.global_stats(blk, 4, 2, 3)
    assert g.counts.tolist() == [3, 1, 0, 2] and g.kept.tolist() == [3, 1, 0, 1] and g.dropped == 1
    assert g.f.tolist() == [0.5, 1 / 6, 0.0, 1 / 3]
    assert g.l_aux == pytest.approx(4 * (0.5 * 0.5 + 0.2 / 6 + 0.2 / 3), rel=1e-6)


# --- data-parallel training: global f, scaled alpha/beta, summed gradients ---

d_ff = 6
ALPHA, BETA = 0.3, 0.05


def _train_data():
    rng = np.random.default_rng(1)
    x, W_r = _data()
    W1 = rng.standard_normal((E, d_ff, d)) / math.sqrt(d)
    W3 = rng.standard_normal((E, d_ff, d)) / math.sqrt(d)
    W2 = rng.standard_normal((E, d, d_ff)) / math.sqrt(d_ff)
    dy = rng.standard_normal((T, d))
    return x, W_r, W1, W3, W2, dy


def _train_worker(rank, world, port, q):
    from oracle import moe_backward_oracle as BO
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=__import__("datetime").timedelta(seconds=60))
    try:
        x, W_r, W1, W3, W2, dy = _train_data()
        lo, hi = parallel.shard_range(T, world, rank)
        # the replica's forward statistics, exchanged
        z = O.router_logits(x[lo:hi], W_r)
        r = O.route(z, k)
        perm = O.permute(r.idx, E)
        st = O.load_stats(perm, r.probs, hi - lo, k, None)
        blk = parallel.stats_block_from_parts(st.counts.tolist(), st.kept.tolist(), st.P.tolist())
        g = parallel.global_stats(blk, E, k, hi - lo)
        parallel.set_global_f(blk, E, g)
        f_blk = blk[48 + 12 * E:48 + 16 * E].view(torch.float32).double().numpy()
        s = parallel.loss_scale(hi - lo, g.T)
        res = BO.moe_backward(x[lo:hi], W_r, W1, W3, W2, k, dy[lo:hi], alpha=ALPHA * s, beta=BETA * s, f=f_blk)
        grads = [torch.from_numpy(a.copy()) for a in (res.dW_r, res.dW1, res.dW3, res.dW2)]
        parallel.allreduce_gradients(grads)
        q.put((rank, lo, hi, res.dx, [t.numpy() for t in grads], f_blk))
    finally:
        dist.destroy_process_group()


def test_data_parallel_gradients_equal_full_batch_backward():
    from oracle import moe_backward_oracle as BO
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_train_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    results = [q.get(timeout=120) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    x, W_r, W1, W3, W2, dy = _train_data()
    ref = BO.moe_backward(x, W_r, W1, W3, W2, k, dy, alpha=ALPHA, beta=BETA)
    for rank, lo, hi, dx, grads, f_blk in results:
        # the global f went through the block in fp32
        assert np.allclose(f_blk, ref.forward.stats.f, rtol=1e-7, atol=0)
        assert np.allclose(dx, ref.dx[lo:hi], rtol=1e-6, atol=1e-9)
        for got, want in zip(grads, (ref.dW_r, ref.dW1, ref.dW3, ref.dW2)):
            assert np.allclose(got, want, rtol=1e-6, atol=1e-9)
