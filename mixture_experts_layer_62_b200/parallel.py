"""Data-parallel replicas of the MoE layer: token sharding and the one
exchange step, the global load statistics.

Every rank holds the full layer (one Mixtral-shaped layer is 2.8 GB, a
DeepSeek-V3-shaped one 22.6 GB, of the B200's 180 GB) and runs moe_forward on
its own contiguous shard of tokens; tokens are independent ("Week 2 Day 2:
Mixture of Experts" §1.3), so outputs need no communication. Capacity is
per replica (each rank truncates its own pairs, the per-device reading of
"Lecture 21 · LLM: Mixture-of-Experts" §3.5).

The statistics of the balance loss are defined over the whole batch
("Week 2 Day 2" §3.2: f_i over all T tokens, P_i the mean probability), so
the replicas exchange them: one all-reduce of 4E + 2 numbers per step —
counts, kept, the sum of router probabilities (P_e * T_r) and the token and
drop totals — after which every rank holds f, P and L_aux of the global
batch. The same code runs on NCCL (CUDA tensors) and gloo (CPU tensors).
"""

from __future__ import annotations

from dataclasses import dataclass

import torch
import torch.distributed as dist

STATS_HEADER_BYTES = 48


def shard_range(T_global: int, world: int, rank: int):
    """Contiguous token range [lo, hi) of one rank (sizes differ by at most 1)."""
    base, rem = divmod(T_global, world)
    lo = rank * base + min(rank, rem)
    hi = lo + base + (1 if rank < rem else 0)
    return lo, hi


@dataclass
class GlobalStats:
    T: int
    counts: torch.Tensor      # [E] int64
    kept: torch.Tensor        # [E] int64
    f: torch.Tensor           # [E] float64, c_e / (T k)
    P: torch.Tensor           # [E] float64, mean router probability
    l_aux: float              # E * sum f P
    dropped: int
    max_over_mean: float


def _local_vector(stats_block: torch.Tensor, E: int, T_local: int) -> torch.Tensor:
    """[counts, kept, P*T, T, dropped] of one statistics block, float64."""
    body = stats_block[STATS_HEADER_BYTES:STATS_HEADER_BYTES + 16 * E]
    counts = body[:4 * E].view(torch.int32).to(torch.float64)
    kept = body[4 * E:8 * E].view(torch.int32).to(torch.float64)
    P = body[8 * E:12 * E].view(torch.float32).to(torch.float64)
    dropped = stats_block[12:16].view(torch.int32).to(torch.float64)
    T = torch.tensor([float(T_local)], dtype=torch.float64, device=stats_block.device)
    return torch.cat([counts, kept, P * float(T_local), T, dropped])


def global_stats(stats_block: torch.Tensor, E: int, k: int, T_local: int, group=None) -> GlobalStats:
    """Sum the per-replica statistics over the process group (one all-reduce)."""
    v = _local_vector(stats_block, E, T_local)
    if dist.is_available() and dist.is_initialized():
        dist.all_reduce(v, op=dist.ReduceOp.SUM, group=group)
    v = v.cpu()
    counts = v[:E].round().to(torch.int64)
    kept = v[E:2 * E].round().to(torch.int64)
    psum = v[2 * E:3 * E]
    T = int(round(float(v[3 * E])))
    dropped = int(round(float(v[3 * E + 1])))
    f = counts.to(torch.float64) / float(T * k) if T > 0 else torch.zeros(E, dtype=torch.float64)
    P = psum / float(T) if T > 0 else torch.zeros(E, dtype=torch.float64)
    l_aux = float(E * torch.sum(f * P))
    mean = T * k / E
    mom = float(counts.max()) / mean if T > 0 else 0.0
    return GlobalStats(T=T, counts=counts, kept=kept, f=f, P=P, l_aux=l_aux, dropped=dropped, max_over_mean=mom)


# ---- data-parallel training --------------------------------------------------
#
# A replica's backward differentiates its own tokens' share of the global
# loss L = sum_t <dy_t, y_t> + alpha L_aux + beta L_z. L_aux uses the global
# f and the global token count ("Week 2 Day 2" §3.2: f and P over the whole
# batch), so before moe_backward a replica writes the global f into its
# statistics block and scales alpha and beta by T_local / T_global (the
# backward divides by its own T); afterwards one all-reduce (sum) of each
# weight gradient gives every replica the gradient of the global loss. dx
# stays local.

def set_global_f(stats_block: torch.Tensor, E: int, g: GlobalStats) -> None:
    """Overwrite the f array of a statistics block with the global f."""
    body = stats_block[STATS_HEADER_BYTES:STATS_HEADER_BYTES + 16 * E]
    body[12 * E:16 * E].view(torch.float32).copy_(g.f.to(torch.float32).to(stats_block.device))


def loss_scale(T_local: int, T_global: int) -> float:
    """Factor for alpha and beta on a replica holding T_local of T_global tokens."""
    return float(T_local) / float(T_global) if T_global > 0 else 0.0


def allreduce_gradients(grads, group=None) -> None:
    """Sum each gradient tensor over the replicas, in place."""
    if dist.is_available() and dist.is_initialized():
        for t in grads:
            dist.all_reduce(t, op=dist.ReduceOp.SUM, group=group)


def stats_block_from_parts(counts, kept, P, dropped=0, capacity=-1, device="cpu") -> torch.Tensor:
    """Build a statistics block (the library's layout) from host values; used
    to feed global_stats from statistics computed elsewhere."""
    E = len(counts)
    blk = torch.zeros(STATS_HEADER_BYTES + 16 * E, dtype=torch.uint8)
    hdr = blk[:STATS_HEADER_BYTES].view(torch.int32)
    hdr[1] = int(capacity)
    hdr[2] = int(sum(kept))
    hdr[3] = int(dropped)
    hdr[4] = int(max(counts)) if E else 0
    body = blk[STATS_HEADER_BYTES:]
    body[:4 * E].view(torch.int32)[:] = torch.tensor(list(counts), dtype=torch.int32)
    body[4 * E:8 * E].view(torch.int32)[:] = torch.tensor(list(kept), dtype=torch.int32)
    body[8 * E:12 * E].view(torch.float32)[:] = torch.tensor(list(P), dtype=torch.float32)
    return blk.to(device)
