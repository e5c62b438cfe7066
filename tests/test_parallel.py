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
