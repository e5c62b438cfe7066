"""Expert parallelism over W ranks: dispatch and combine as all-to-alls.

Rank r owns the experts [r E/W, (r + 1) E/W) ("Lecture 21 · LLM:
Mixture-of-Experts" §4, expert parallelism: every GPU holds E/W experts,
tokens travel to their experts' GPU and back). Each rank routes and permutes
its own tokens (``moe_route`` and ``moe_permute`` of the library, or the
fused pass up to the permutation). The permutation is expert-major, so the
rows bound for one owner form one contiguous slice of Xp, already in the
owner's expert order; no packing step is needed. Then:

1. ``plan``: an all-to-all of the per-expert row counts (E numbers a rank)
   tells every owner how many rows of each of its experts each source sends.
2. ``dispatch``: an all-to-all of the rows; the owner's buffer holds one
   block per source, each block grouped by the owner's experts.
3. ``run_local_experts``: the owner runs its experts over each source's block
   (one grouped GEMM call per block, with the block's own offsets), so the
   outputs stay in the order the rows came in.
4. ``combine_back``: an all-to-all returns every block to its source, where
   it lands exactly where the single-GPU pass puts its expert outputs (O, in
   the permuted order), and the library's combine finishes the layer.

``forward_overlapped`` does steps 2-4 in rounds of paired sends and
receives (rank r exchanges with r + i and r - i in round i), so the grouped
GEMMs of one source's block run while the next block's rows, and the
previous block's outputs, are on the wire.

Capacity is applied by each source on its own tokens (per-device capacity,
as for the data-parallel replicas). The collectives and point-to-point
transfers are issued by torch.distributed (NCCL on GPUs, gloo on CPU
tensors); the same functions serve both. The overlap is per block; a single
kernel that moves tiles over peer memory while it multiplies is not built
here.
"""

from __future__ import annotations

from dataclasses import dataclass
from typing import Callable, List

import torch
import torch.distributed as dist


def expert_range(E: int, world: int, rank: int):
    """Experts [lo, hi) owned by `rank` (E must divide evenly)."""
    if E % world:
        raise ValueError(f"{E} experts do not split evenly over {world} ranks")
    n = E // world
    return rank * n, (rank + 1) * n


@dataclass
class EPPlan:
    world: int
    E: int
    E_local: int
    send_rows: List[int]        # rows this rank sends to each owner
    recv_rows: List[int]        # rows this rank receives from each source
    recv_counts: torch.Tensor   # [world, E_local] int64: rows per (source, local expert)

    @property
    def rows_out(self) -> int:
        return sum(self.send_rows)

    @property
    def rows_in(self) -> int:
        return sum(self.recv_rows)

    def block_offsets(self, src: int) -> torch.Tensor:
        """Row offsets [E_local + 1] of source `src`'s block, per local expert."""
        c = self.recv_counts[src]
        return torch.cat([torch.zeros(1, dtype=torch.int64), torch.cumsum(c, 0)])


def plan(indptr: torch.Tensor, E: int, group=None) -> EPPlan:
    """Exchange per-expert row counts. `indptr` [E + 1] is this rank's
    permutation offsets (kept rows, expert-major)."""
    world = dist.get_world_size(group)
    lo, hi = expert_range(E, world, 0)
    E_local = hi - lo
    ip = indptr.to(torch.int64)
    counts = ip[1:] - ip[:-1]                           # [E], owner-major
    recv = torch.empty_like(counts)
    dist.all_to_all_single(recv, counts, group=group)   # [world * E_local], source-major
    send_rows = counts.view(world, E_local).sum(1).cpu().tolist()
    recv_counts = recv.view(world, E_local).cpu()
    recv_rows = recv_counts.sum(1).tolist()
    return EPPlan(world, E, E_local, [int(v) for v in send_rows], [int(v) for v in recv_rows], recv_counts)


def dispatch(xp: torch.Tensor, p: EPPlan, group=None) -> torch.Tensor:
    """Send the permuted rows to their owners; returns the rows received,
    one block per source in rank order."""
    out = xp.new_empty((p.rows_in,) + tuple(xp.shape[1:]))
    dist.all_to_all_single(out, xp[:p.rows_out].contiguous(), output_split_sizes=p.recv_rows,
                           input_split_sizes=p.send_rows, group=group)
    return out


def run_local_experts(rows: torch.Tensor, p: EPPlan,
                      experts_fn: Callable[[torch.Tensor, torch.Tensor], torch.Tensor], d_out: int) -> torch.Tensor:
    """Apply the local experts block by block: experts_fn(block_rows,
    offsets) returns the block's expert outputs [n, d_out], rows in the
    block's order, offsets [E_local + 1] int64 on the host."""
    out = rows.new_empty((p.rows_in, d_out))
    at = 0
    for src in range(p.world):
        n = p.recv_rows[src]
        if n:
            out[at:at + n] = experts_fn(rows[at:at + n], p.block_offsets(src))
        at += n
    return out


def combine_back(expert_out: torch.Tensor, p: EPPlan, o: torch.Tensor, group=None) -> torch.Tensor:
    """Return every block to its source; fills o[:rows_out] (this rank's
    expert outputs in its own permuted order) and returns o."""
    dist.all_to_all_single(o[:p.rows_out], expert_out.contiguous(), output_split_sizes=p.send_rows,
                           input_split_sizes=p.recv_rows, group=group)
    return o


def _peer(rank: int, group) -> int:
    return rank if group is None else dist.get_global_rank(group, rank)


def forward_overlapped(xp: torch.Tensor, p: EPPlan,
                       experts_fn: Callable[[torch.Tensor, torch.Tensor], torch.Tensor], o: torch.Tensor,
                       group=None) -> torch.Tensor:
    """dispatch + run_local_experts + combine_back with the transfers
    overlapping the grouped GEMMs.

    The exchange runs in rounds. In round r (1 <= r < W) this rank sends its
    rows for owner (rank + r) mod W and receives the rows of source
    (rank - r) mod W; the return of round r sends that source its outputs
    and receives this rank's outputs from owner (rank + r) mod W. The
    rank's own rows (round 0) are computed first, while round 1's dispatch
    is in flight; after that, the block of round r is computed while round
    r + 1's dispatch and round r - 1's return are in flight. Every rank
    posts the same sequence of paired send/receive groups (D1, D2, R1, D3,
    R2, ...), so on a backend that runs one rank's transfers in order (NCCL)
    every send meets its receive. Each block goes through experts_fn exactly
    as in run_local_experts, so o[:rows_out] gets the same values as
    dispatch, run_local_experts and combine_back give. Returns o."""
    world = p.world
    rank = dist.get_rank(group)
    d = xp.shape[1]
    send_off = [0]
    for n in p.send_rows:
        send_off.append(send_off[-1] + n)
    keep = []   # tensors in flight must outlive their transfers

    def src_of(r):
        return (rank - r) % world

    def dst_of(r):
        return (rank + r) % world

    def exchange(send_t, send_to, n_send, recv_t, recv_from, n_recv):
        ops = []
        if n_send:
            ops.append(dist.P2POp(dist.isend, send_t, _peer(send_to, group), group))
        if n_recv:
            ops.append(dist.P2POp(dist.irecv, recv_t, _peer(recv_from, group), group))
        keep.append((send_t, recv_t))
        return dist.batch_isend_irecv(ops) if ops else []

    recv_buf = {}

    def post_dispatch(r):
        dst, src = dst_of(r), src_of(r)
        recv_buf[src] = xp.new_empty((p.recv_rows[src], d))
        return exchange(xp[send_off[dst]:send_off[dst + 1]].contiguous(), dst, p.send_rows[dst],
                        recv_buf[src], src, p.recv_rows[src])

    def wait(works):
        for w in works:
            w.wait()

    pending_d = post_dispatch(1) if world > 1 else []
    # round 0: this rank's rows for its own experts
    if p.send_rows[rank]:
        o[send_off[rank]:send_off[rank + 1]] = experts_fn(xp[send_off[rank]:send_off[rank + 1]],
                                                          p.block_offsets(rank))
    pending_r = []
    for r in range(1, world):
        wait(pending_d)
        pending_d = post_dispatch(r + 1) if r + 1 < world else []
        src, dst = src_of(r), dst_of(r)
        rows = recv_buf.pop(src)
        out_blk = experts_fn(rows, p.block_offsets(src)) if p.recv_rows[src] else rows.new_empty((0, o.shape[1]))
        recv_t = o[send_off[dst]:send_off[dst + 1]]
        pending_r.append(exchange(out_blk.contiguous(), src, p.recv_rows[src], recv_t, dst, p.send_rows[dst]))
    for works in pending_r:
        wait(works)
    return o


def library_experts_fn(W1_local: torch.Tensor, W3_local: torch.Tensor, W2_local: torch.Tensor,
                       max_rows: int | None = None):
    """An experts_fn for run_local_experts that runs the owner's experts with
    the library's grouped GEMMs (moe_experts, GEMM 1/3 + SwiGLU then GEMM 2)
    on the device of the weights: W1_local, W3_local [E_local, d_ff, d],
    W2_local [E_local, d, d_ff]. A block of n rows is one call with a
    problem of n tokens, one slot each, over the E_local experts.

    The function holds one workspace. With ``max_rows`` (the largest block a
    source can send, e.g. its tokens times k) it is sized once, up front;
    without, it is replaced only when a block needs more than it holds, so
    the memory held is that of the largest block seen, however the block
    sizes vary from step to step. The calls share one statistics block,
    ``fn.state["stats"]``, whose status word records a device-side error
    (a bounded wait of a tensor-core kernel that gave up)."""
    import mixture_experts_layer_62_b200 as moe

    E_local, d_ff, d = W1_local.shape
    dev = W1_local.device
    state = {"ws": None, "stats": moe.alloc_stats(E_local, dev)}

    def ensure(n, dtype):
        need = moe.workspace_size(moe.problem(n, d, d_ff, E_local, 1, 0.0, dtype))
        ws = state["ws"]
        if ws is None or ws.numel() < need:
            state["ws"] = None                      # release the old buffer before the new one
            state["ws"] = torch.empty(need, dtype=torch.uint8, device=dev)
        return state["ws"]

    if max_rows is not None:
        ensure(int(max_rows), W1_local.dtype)

    def fn(block: torch.Tensor, offsets: torch.Tensor) -> torch.Tensor:
        n = block.shape[0]
        p = moe.problem(n, d, d_ff, E_local, 1, 0.0, block.dtype)
        ws = ensure(n, block.dtype)
        indptr = offsets.to(device=block.device, dtype=torch.int32)
        out = torch.empty((n, d), dtype=block.dtype, device=block.device)
        moe.experts(p, block.contiguous(), indptr, W1_local, W3_local, W2_local, out, ws, stats=state["stats"])
        return out

    fn.state = state
    return fn
