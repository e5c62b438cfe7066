"""Failure detection on the GPU without a fault: the bounded waits.

Every mbarrier wait inside the tensor-core kernels gives up after a
wall-clock limit, records MOE_ERR_TIMEOUT in the call's status word, drains
the copies and MMAs it already started (under a separate, long limit), frees
its tensor memory and returns. These tests make the waits run out on purpose
by setting the limit to 1 ns through the C ABI (moe_set_wait_limit): every
wait that is not satisfied at its first probe gives up. Nothing else is
changed, no wait is removed and no flag is left unset. The host then reads
the status word, restores the default limit, and checks that the next call on
the same context is correct against the oracle.
"""

import math

import numpy as np
import pytest
import torch

import mixture_experts_layer_62_b200 as moe
from oracle import moe_oracle as O
from parity_util import TOL_BF16, assert_rows_close, gpu_forward, np32, oracle_weights, to_device

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _expert_stage_inputs(seed=3):
    E, d, d_ff = 4, 256, 384
    counts = [100, 50, 150, 100]           # 400 rows: no split-K, ragged M blocks
    rows = sum(counts)
    g = torch.Generator().manual_seed(seed)
    xp = torch.randn((rows, d), generator=g).to(torch.bfloat16)
    W1 = (torch.randn((E, d_ff, d), generator=g) / math.sqrt(d)).to(torch.bfloat16)
    W3 = (torch.randn((E, d_ff, d), generator=g) / math.sqrt(d)).to(torch.bfloat16)
    W2 = (torch.randn((E, d, d_ff), generator=g) / math.sqrt(d_ff)).to(torch.bfloat16)
    indptr = np.concatenate([[0], np.cumsum(counts)]).astype(np.int32)
    return E, d, d_ff, rows, xp, W1, W3, W2, indptr


def _run_stage(p, E, d, rows, xp, W1, W3, W2, indptr):
    ws = moe.alloc_workspace(p, DEV)
    st = moe.alloc_stats(E, DEV)
    o = torch.zeros((rows, d), dtype=torch.bfloat16, device=DEV)
    moe.experts(p, xp.to(DEV), torch.from_numpy(indptr).to(DEV), W1.to(DEV), W3.to(DEV), W2.to(DEV), o, ws,
                stats=st)
    torch.cuda.synchronize()
    return o, moe.read_stats(st, E)


def test_expert_stage_wait_runs_out_then_recovers():
    E, d, d_ff, rows, xp, W1, W3, W2, indptr = _expert_stage_inputs()
    p = moe.problem(rows // 2, d, d_ff, E, 2, 0.0, "bf16")
    prev = moe.set_wait_limit(1)
    try:
        _, s = _run_stage(p, E, d, rows, xp, W1, W3, W2, indptr)
    finally:
        moe.set_wait_limit(prev)
    assert s.status == moe.MOE_ERR_TIMEOUT, s.status
    assert moe.error_string(s.status) == "device-side bounded wait timed out"
    # the context is intact: the same call with the normal limit is correct
    for _ in range(2):
        o, s = _run_stage(p, E, d, rows, xp, W1, W3, W2, indptr)
        assert s.status == moe.MOE_OK
        on = o.float().cpu().numpy()
        for e in range(E):
            lo, hi = indptr[e], indptr[e + 1]
            ref = O.swiglu_expert(xp[lo:hi].float().numpy(), W1[e].float().numpy(), W3[e].float().numpy(),
                                  W2[e].float().numpy())
            assert_rows_close(on[lo:hi], ref, TOL_BF16, f"expert {e}")


def _layer(T, d, d_ff, E, seed):
    g = torch.Generator().manual_seed(seed)
    return dict(x=torch.randn((T, d), generator=g).to(torch.bfloat16),
                W_r=(torch.randn((d, E), generator=g) / math.sqrt(d)).to(torch.bfloat16),
                W1=(torch.randn((E, d_ff, d), generator=g) / math.sqrt(d)).to(torch.bfloat16),
                W3=(torch.randn((E, d_ff, d), generator=g) / math.sqrt(d)).to(torch.bfloat16),
                W2=(torch.randn((E, d, d_ff), generator=g) / math.sqrt(d_ff)).to(torch.bfloat16),
                bias=None, Ws1=None, Ws3=None, Ws2=None)


@pytest.mark.parametrize("T", [300, 4])      # the general path, and the decode path with split-K
def test_forward_wait_runs_out_then_recovers(T):
    cfg = dict(T=T, d=256, d_ff=256, E=8, k=2, cf=0.0, dtype="bf16", bias_mode=0, d_ff_shared=0)
    L_cpu = _layer(T, 256, 256, 8, seed=T)
    L = to_device(L_cpu)
    prev = moe.set_wait_limit(1)
    try:
        _, _, st, _ = gpu_forward(cfg, L)
    finally:
        moe.set_wait_limit(prev)
    assert moe.read_stats(st, 8).status == moe.MOE_ERR_TIMEOUT
    # next forwards (same buffers recreated, same context): correct, twice
    outs = []
    for _ in range(2):
        p, out, st, ws = gpu_forward(cfg, L)
        s = moe.read_stats(st, 8)
        assert s.status == moe.MOE_OK
        outs.append(out.cpu())
    assert torch.equal(outs[0], outs[1])
    logits = moe.workspace_view(ws, p, "logits").cpu().numpy()
    W = oracle_weights(L_cpu)
    res = O.moe_forward(np32(L_cpu["x"]), None, W["W1"], W["W3"], W["W2"], 2, 0.0, logits=logits,
                        key_dtype=np.float32)
    assert np.array_equal(moe.workspace_view(ws, p, "idx").cpu().numpy(), res.routing.idx)
    assert_rows_close(outs[0].float().numpy(), res.y, TOL_BF16, "forward after a timed-out call")
