"""The multi-rank paths with the library's kernels, as two ranks on one GPU.

Two processes share cuda:0; their exchanges (the statistics all-reduce of
the data-parallel replicas, the dispatch and combine all-to-alls of expert
parallelism) run over gloo on CPU tensors, so no kernel of one rank ever
waits on the other's. What these tests add to the CPU-only multi-rank tests
is the GPU side: statistics blocks written by the library's own kernels, and
each owner's experts run by the library's grouped GEMMs.

* Data parallel: every rank runs moe_forward on its contiguous shard; the
  statistics blocks the kernels wrote go through parallel.global_stats (one
  all-reduce); the global counts, P and L_aux must be the oracle's statistics
  of the whole batch, routed from the same logits.
* Expert parallel ("Lecture 21 · LLM: Mixture-of-Experts" §5.1): every rank
  routes and permutes its tokens with the library, plan / dispatch move the
  permuted rows to the owners of their experts, the owner's experts run with
  library_experts_fn (moe_experts on the owner's weight slice), combine_back
  returns them and moe_combine finishes the layer. Each rank's output must
  match, element by element, the oracle's single-process forward of its
  tokens with all the experts, capacity drops included; forward_overlapped
  (the same exchange in rounds that overlap the experts) must put the same
  expert outputs in the same rows.
"""

import math
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

pytestmark = pytest.mark.gpu

T, d, d_ff, E, k, CF = 600, 256, 384, 4, 2, 1.0


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _layer():
    g = torch.Generator().manual_seed(11)
    x = torch.randn((T, d), generator=g).to(torch.bfloat16)
    W_r = (torch.randn((d, E), generator=g) / math.sqrt(d)).to(torch.bfloat16)
    W1 = (torch.randn((E, d_ff, d), generator=g) / math.sqrt(d)).to(torch.bfloat16)
    W3 = (torch.randn((E, d_ff, d), generator=g) / math.sqrt(d)).to(torch.bfloat16)
    W2 = (torch.randn((E, d, d_ff), generator=g) / math.sqrt(d_ff)).to(torch.bfloat16)
    return x, W_r, W1, W3, W2


def _init(rank, world, port):
    import datetime
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=120))
    torch.cuda.set_device(0)


def _dp_worker(rank, world, port, q):
    _init(rank, world, port)
    try:
        import mixture_experts_layer_62_b200 as moe
        from mixture_experts_layer_62_b200 import parallel
        x, W_r, W1, W3, W2 = _layer()
        lo, hi = parallel.shard_range(T, world, rank)
        dev = torch.device("cuda", 0)
        p = moe.problem(hi - lo, d, d_ff, E, k, CF, "bf16")
        layer = moe.MoELayer(p, W_r.to(dev), W1.to(dev), W3.to(dev), W2.to(dev))
        layer(x[lo:hi].to(dev))
        torch.cuda.synchronize()
        assert layer.read_stats().status == moe.MOE_OK
        logits = moe.workspace_view(layer.workspace, p, "logits").cpu().numpy()
        g = parallel.global_stats(layer.stats.cpu(), E, k, hi - lo)
        q.put((rank, logits, g.T, g.counts.tolist(), g.kept.tolist(), g.P.tolist(), g.l_aux, g.dropped, None))
    except Exception as e:   # reported to the parent, which fails the test
        q.put((rank, None, None, None, None, None, None, None, repr(e)))
    finally:
        dist.destroy_process_group()


def _ep_worker(rank, world, port, q):
    _init(rank, world, port)
    try:
        import mixture_experts_layer_62_b200 as moe
        from mixture_experts_layer_62_b200 import expert_parallel as ep
        from mixture_experts_layer_62_b200 import parallel
        x, W_r, W1, W3, W2 = _layer()
        dev = torch.device("cuda", 0)
        lo, hi = parallel.shard_range(T, world, rank)
        Tr = hi - lo
        p = moe.problem(Tr, d, d_ff, E, k, CF, "bf16")
        ws = moe.alloc_workspace(p, dev)
        st = moe.alloc_stats(E, dev)
        xr = x[lo:hi].to(dev)
        idx = torch.empty((Tr, k), dtype=torch.int32, device=dev)
        gate = torch.empty((Tr, k), dtype=torch.float32, device=dev)
        logits = torch.empty((Tr, E), dtype=torch.float32, device=dev)
        pos = torch.empty((Tr, k), dtype=torch.int32, device=dev)
        indptr = torch.empty((E + 1,), dtype=torch.int32, device=dev)
        row_token = torch.empty((Tr * k,), dtype=torch.int32, device=dev)
        xp = torch.empty((Tr * k, d), dtype=torch.bfloat16, device=dev)
        moe.route(p, xr, W_r.to(dev), idx, gate, st, ws, logits=logits)
        moe.permute(p, xr, idx, pos, indptr, row_token, xp, st, ws)
        torch.cuda.synchronize()
        # exchange over gloo on host copies; the experts run on the GPU
        plan = ep.plan(indptr.cpu(), E)
        rows = ep.dispatch(xp.cpu(), plan).to(dev)
        e_lo, e_hi = ep.expert_range(E, world, rank)
        fn = ep.library_experts_fn(W1[e_lo:e_hi].contiguous().to(dev), W3[e_lo:e_hi].contiguous().to(dev),
                                   W2[e_lo:e_hi].contiguous().to(dev), max_rows=T * k)
        expert_out = ep.run_local_experts(rows, plan, fn, d)
        torch.cuda.synchronize()
        status = moe.read_stats(fn.state["stats"], e_hi - e_lo).status
        o = torch.zeros((Tr * k, d), dtype=torch.bfloat16)
        ep.combine_back(expert_out.cpu(), plan, o)
        y = torch.empty((Tr, d), dtype=torch.bfloat16, device=dev)
        moe.combine(p, o.to(dev), pos, gate, y)
        torch.cuda.synchronize()
        # the overlapped exchange: each block's experts run on the GPU while
        # the next block's rows move; the same rows in the same places
        o2 = torch.full((Tr * k, d), float("nan"), dtype=torch.bfloat16)
        ep.forward_overlapped(xp.cpu(), plan, lambda blk, offs: fn(blk.to(dev), offs).cpu(), o2)
        same = bool(torch.equal(o[:plan.rows_out], o2[:plan.rows_out]))
        q.put((rank, y.float().cpu().numpy(), logits.cpu().numpy(), idx.cpu().numpy(), status,
               plan.rows_in, int(indptr[-1].item()), same, None))
    except Exception as e:
        q.put((rank, None, None, None, None, None, None, None, repr(e)))
    finally:
        dist.destroy_process_group()


def _spawn(target, world):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=target, args=(r, world, port, q)) for r in range(world)]
    for pr in procs:
        pr.start()
    res = [q.get(timeout=300) for _ in range(world)]
    for pr in procs:
        pr.join(timeout=120)
        assert pr.exitcode == 0
    res.sort(key=lambda r: r[0])
    for r in res:
        assert r[-1] is None, r[-1]
    return res


def test_data_parallel_stats_from_library_blocks():
    from oracle import moe_oracle as O
    res = _spawn(_dp_worker, 2)
    logits = np.concatenate([r[1] for r in res])
    # the whole batch as one: the oracle's statistics on the ranks' logits
    # (counts and kept per replica capacity: sums of the ranks' own)
    r_all = O.route(logits, k, key_dtype=np.float32)
    counts = np.bincount(r_all.idx.ravel(), minlength=E)
    P = r_all.probs.mean(axis=0)
    f = counts / (T * k)
    kept, dropped = np.zeros(E, dtype=np.int64), 0
    from mixture_experts_layer_62_b200 import parallel
    for rank in range(2):
        lo, hi = parallel.shard_range(T, 2, rank)
        rr = O.route(logits[lo:hi], k, key_dtype=np.float32)
        perm = O.permute(rr.idx, E, O.capacity(CF, hi - lo, k, E))
        kept += perm.kept
        dropped += int((perm.counts - perm.kept).sum())
    for r in res:
        _, _, gT, gcounts, gkept, gP, gl_aux, gdropped, _ = r
        assert gT == T
        assert gcounts == counts.tolist()
        assert gkept == kept.tolist() and gdropped == dropped
        assert np.allclose(gP, P, rtol=1e-5, atol=1e-7)
        assert gl_aux == pytest.approx(E * float(np.sum(f * P)), rel=1e-4)


def test_expert_parallel_forward_with_library_experts():
    from oracle import moe_oracle as O
    from mixture_experts_layer_62_b200 import parallel
    from parity_util import TOL_BF16, assert_rows_close
    res = _spawn(_ep_worker, 2)
    x, W_r, W1, W3, W2 = _layer()
    W = {n: {e: w[e].float().numpy() for e in range(E)} for n, w in (("W1", W1), ("W3", W3), ("W2", W2))}
    total_in, total_out, drops = 0, 0, 0
    for rank, y, logits, idx, status, rows_in, rows_out, same, _ in res:
        assert status == 0
        assert same, f"rank {rank}: the overlapped exchange differs from dispatch / combine_back"
        lo, hi = parallel.shard_range(T, 2, rank)
        ref = O.moe_forward(x[lo:hi].float().numpy(), None, W["W1"], W["W3"], W["W2"], k, CF, logits=logits,
                            key_dtype=np.float32)
        assert np.array_equal(idx, ref.routing.idx)
        drops += ref.stats.dropped
        assert_rows_close(y, ref.y, TOL_BF16, f"rank {rank}")
        total_in += rows_in
        total_out += rows_out
    assert total_in == total_out     # every kept row went to exactly one owner and came back
    assert drops > 0                 # the per-rank capacity dropped some pairs
