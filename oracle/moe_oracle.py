"""CPU oracle for the forward pass of one sparse Mixture-of-Experts layer.

TEST INFRASTRUCTURE ONLY. This module is the slow, plain definition that the
CUDA library is checked against. Only the test suite, the smoke check in
``__graft_entry__`` and the CPU-baseline leg of ``bench.py`` may import it. The
product path (the C-ABI library and its Python binding) never imports, calls or
falls back to it, and it shares no code with that path.

Everything here is numpy in float64 (the inputs are float32 or the float32
value of bf16 numbers, so the conversion is exact). Each function cites the
passage of the source notes it follows. Page keys used in the citations:

* [CME295 W2D2]    "Week 2 Day 2: Mixture of Experts" course notes (CME295)
* [MoE tutorial]   "混合专家模型" (Mixture-of-Experts) tutorial, FANDEX
* [CS336 L04]      "Stanford CS336 Lecture 04: Detailed Explanation of the MoE Architecture"
* [CMU 15-779 L21] "Lecture 21 · LLM: Mixture-of-Experts (architectures, kernels, parallelism)"
* [W11 routing]    "W11 · MoE routing and parallel cost" lesson

Readings taken where the notes are silent or disagree (each is listed in the
design notes of the repository as well):

* capacity uses the form with k: C = ceil(cf * T * k / E) ([CMU 15-779 L21]
  §3.5 capacity equation; [W11 routing] §3). The form without k in
  [CME295 W2D2] §3.3 is not used.
* a pair over capacity is dropped in token order inside its expert (the order
  of the expert-major prefix sum, [CMU 15-779 L21] §3.3); the surviving gates
  are not renormalised and a fully dropped token gets a zero output row.
* gates are the softmax over the k selected raw logits ([CME295 W2D2] §1.3);
  the selection bias never enters the gates ([CME295 W2D2] §4.2).
* f_e = c_e / (T k) with pre-drop counts, so that uniform routing gives
  L_aux = 1 (alpha omitted); P_e is the mean full softmax over raw logits
  ([CME295 W2D2] §3.2).
* the expert is SwiGLU without biases: W2 (SiLU(W1 x) * (W3 x)), SiLU(a) =
  a * sigmoid(a) ([CME295 W2D2] §2.1 table, "3 d d_ff" parameters, no bias).
* top-k ties go to the lower expert index.

Parity pins: every function below is pinned by the CPU tests in
``tests/test_oracle_pins.py`` (worked examples of the notes, closed forms,
special cases and a dense-masked brute force). The one-token worked example of
[CMU 15-779 L21] §2.1 (experts {0, 5}, weights 0.743 / 0.257) and the 0.30
top-k-vs-dense difference of [CME295 W2D2] §1.3 print no inputs: parity
unpinned for those two values; only the invariants they illustrate are pinned.
"""

from __future__ import annotations

import math
from dataclasses import dataclass, field
from typing import Optional

import numpy as np

# Selection-bias modes (numbering shared with the C header by value only).
BIAS_NONE = 0   # key = z
BIAS_LOGIT = 1  # key = z + b      ([MoE tutorial] route(): bias on raw scores)
BIAS_PROB = 2   # key = softmax(z) + b   ([CS336 L04] §2.3.3c: bias on s_{i,t})

# Gate modes.
GATE_SELECTED = 0  # softmax over the k selected raw logits ([CME295 W2D2] §1.3)
GATE_FULL = 1      # full-softmax probability of each selected expert, not
                   # renormalised (Switch top-1, [CMU 15-779 L21] §2.5)

# Drop orders under capacity.
DROP_TOKEN = 0     # rank inside an expert in token order ([CMU 15-779 L21] §3.3)
DROP_SLOT = 1      # GShard Algorithm 1: every token's first choice before any
                   # second choice ([CMU 15-779 L21] §3.5)


# --------------------------------------------------------------------------
# Router
# --------------------------------------------------------------------------

def router_logits(x, W_r):
    """z_t = W_r^T x_t for every token (one score per expert).

    [CME295 W2D2] §1.3, first routing equation; W_r has shape [d, E].
    x: [T, d]; returns [T, E] float64.
    """
    x = np.asarray(x, dtype=np.float64)
    W_r = np.asarray(W_r, dtype=np.float64)
    return x @ W_r


def softmax_rows(z):
    """Row-wise softmax, max-subtracted ([W11 routing] §1: p = softmax(W_r x))."""
    z = np.asarray(z, dtype=np.float64)
    m = z.max(axis=1, keepdims=True)
    e = np.exp(z - m)
    return e / e.sum(axis=1, keepdims=True)


def selection_key(z, bias, bias_mode, dtype=np.float64):
    """The score that top-k ranks.

    * BIAS_NONE:  z                    ([CME295 W2D2] §1.3, T = TopK(z, k))
    * BIAS_LOGIT: z + b                ([CME295 W2D2] §4.2, TopK(z + b, k);
                                        [MoE tutorial] route(), biased scores)
    * BIAS_PROB:  softmax(z) + b       ([CS336 L04] §2.3.3c, s_{i,t} + b_i)

    ``dtype`` fixes the precision in which the key is formed. An integer
    decision (the selected index) is taken in the kernel's precision when the
    result is compared bit for bit, so callers pass np.float32 there.
    """
    z = np.asarray(z, dtype=dtype)
    if bias_mode == BIAS_NONE:
        return z
    b = np.asarray(bias, dtype=dtype).reshape(1, -1)
    if bias_mode == BIAS_LOGIT:
        return (z + b).astype(dtype)
    if bias_mode == BIAS_PROB:
        zz = z.astype(dtype)
        m = zz.max(axis=1, keepdims=True)
        e = np.exp(zz - m).astype(dtype)
        p = (e / e.sum(axis=1, keepdims=True, dtype=dtype)).astype(dtype)
        return (p + b).astype(dtype)
    raise ValueError(f"unknown bias_mode {bias_mode}")


def topk_lowest_index(key, k):
    """Indices of the k largest keys per row, in descending key order.

    Greedy top-k ([CMU 15-779 L21] §2.1: top-k picks the k highest scores).
    Equal keys go to the lower expert index (a stable sort on -key keeps the
    index order among equals, as the sorted(..., key=-b) in [MoE tutorial]
    route() does).
    """
    key = np.asarray(key)
    order = np.argsort(-key, axis=1, kind="stable")
    return order[:, :k].astype(np.int64)


def gates_from_selected(z, idx):
    """g_i = exp(z_i) / sum_{j in T} exp(z_j) over the selected set, i in T.

    [CME295 W2D2] §1.3 gate equation; computed max-subtracted as in
    [MoE tutorial] route() ("softmax over the raw scores of the chosen
    experts"). Returns [T, k] float64 in slot order.
    """
    z = np.asarray(z, dtype=np.float64)
    chosen = np.take_along_axis(z, idx, axis=1)
    m = chosen.max(axis=1, keepdims=True)
    e = np.exp(chosen - m)
    return e / e.sum(axis=1, keepdims=True)


def gates_full_softmax(z, idx):
    """g_i = softmax(z)_i for each selected i, not renormalised over the
    selected set: the Switch Transformer's top-1 gate y = p_i(x) E_i(x)
    ([CMU 15-779 L21] §2.5; [CME295 W2D2] §1.3: Switch with k = 1 takes the
    full softmax probability; [CS336 L04] §2.1.2, g_{i,t} = s_{i,t})."""
    return np.take_along_axis(softmax_rows(z), idx, axis=1)


@dataclass
class Routing:
    idx: np.ndarray        # [T, k] int64, descending key order
    gate: np.ndarray       # [T, k] float64
    probs: np.ndarray      # [T, E] float64, full softmax of raw z
    key: np.ndarray        # [T, E] the ranked key


def route(z, k, bias=None, bias_mode=BIAS_NONE, key_dtype=np.float64, gate_mode=GATE_SELECTED):
    """Routing from logits: selection key, top-k, gates and full softmax.

    [CME295 W2D2] §1.3 and §4.2; [MoE tutorial] route().
    """
    z = np.asarray(z)
    key = selection_key(z, bias, bias_mode, dtype=key_dtype)
    idx = topk_lowest_index(key, k)
    gate = gates_from_selected(z, idx) if gate_mode == GATE_SELECTED else gates_full_softmax(z, idx)
    probs = softmax_rows(z)
    return Routing(idx=idx, gate=gate, probs=probs, key=key)


# --------------------------------------------------------------------------
# Capacity and permutation
# --------------------------------------------------------------------------

def capacity(capacity_factor, T, k, E):
    """C = ceil(cf * N * k / E); None (no limit) when cf <= 0.

    [CMU 15-779 L21] §3.5 capacity equation; [W11 routing] §3. The factor is
    taken through float32 first, the precision in which callers hand it over.
    """
    cf = float(np.float32(capacity_factor))
    if cf <= 0.0:
        return None
    return int(math.ceil(cf * T * k / E))


@dataclass
class Permutation:
    pos: np.ndarray        # [T, k] int64 destination row, -1 if dropped
    indptr: np.ndarray     # [E+1] int64 over kept rows (CSR row offsets)
    counts: np.ndarray     # [E] int64 pairs routed to e before capacity
    kept: np.ndarray       # [E] int64 pairs kept
    row_token: np.ndarray  # [R] int64 source token of each permuted row
    row_slot: np.ndarray   # [R] int64 slot j of each permuted row
    rank: np.ndarray       # [T, k] int64 rank of the pair inside its expert


def permute(idx, E, C=None, drop_order=DROP_TOKEN, pad=None):
    """Permutation indices by prefix sum, with capacity truncation.

    [CMU 15-779 L21] §3.3: build the N x E 0/1 selection mask, flatten it
    expert-major (transpose, then rows), take the inclusive cumulative sum and
    reshape back; the destination row of a selected pair is that sum minus
    one, and the CSR indptr is 0 followed by the last sum of every expert
    column. A pair's rank inside its expert is its destination row minus the
    expert's first row, i.e. token order.

    Capacity ([CMU 15-779 L21] §3.5, [W11 routing] §3): a pair whose rank is
    >= C is dropped. The kept pairs are renumbered with the same expert-major
    order, so their rows are indptr_kept[e] + rank.

    drop_order = DROP_SLOT (GShard's Algorithm 1, [CMU 15-779 L21] §3.5:
    all first choices before the second choices, the rank again a prefix
    sum): the mask gets a slot axis, [k, N, E] with mask[j, t, e] = 1 iff
    idx[t, j] = e, and is flattened expert-major as (e, j, t), so inside an
    expert the pairs are ordered by slot, then token.

    pad = P (MegaBlocks, [CMU 15-779 L21] §3.6: every expert's row count is
    padded to a multiple of the block size inside the permutation): the
    indptr is the prefix sum of ceil(kept_e / P) * P; the padding rows follow
    each expert's kept rows and belong to no token (row_token -1).
    """
    idx = np.asarray(idx, dtype=np.int64)
    T, k = idx.shape
    if drop_order == DROP_SLOT:
        mask3 = np.zeros((k, T, E), dtype=np.int64)
        for t in range(T):
            for j in range(k):
                mask3[j, t, idx[t, j]] = 1
        flat = mask3.transpose(2, 0, 1).reshape(-1)            # (e, j, t)
        cs3 = np.cumsum(flat).reshape(E, k, T)                  # inclusive
        indptr_full = np.zeros(E + 1, dtype=np.int64)
        indptr_full[1:] = cs3[:, k - 1, T - 1] if T > 0 else 0
        counts = indptr_full[1:] - indptr_full[:-1]

        def rank_of(t, j, e):
            return cs3[e, j, t] - 1 - indptr_full[e]
    else:
        mask = np.zeros((T, E), dtype=np.int64)
        for t in range(T):
            for j in range(k):
                mask[t, idx[t, j]] = 1
        flat = mask.T.reshape(-1)                    # expert-major
        cs = np.cumsum(flat).reshape(E, T).T         # [T, E] inclusive prefix sums
        indptr_full = np.zeros(E + 1, dtype=np.int64)
        indptr_full[1:] = cs[T - 1, :] if T > 0 else 0
        counts = indptr_full[1:] - indptr_full[:-1]

        def rank_of(t, j, e):
            return cs[t, e] - 1 - indptr_full[e]

    kept = counts.copy() if C is None else np.minimum(counts, C)
    indptr = np.zeros(E + 1, dtype=np.int64)
    rows_e = kept if not pad else -(-kept // pad) * pad
    indptr[1:] = np.cumsum(rows_e)

    pos = np.full((T, k), -1, dtype=np.int64)
    rank = np.zeros((T, k), dtype=np.int64)
    for t in range(T):
        for j in range(k):
            e = idx[t, j]
            r = rank_of(t, j, e)
            rank[t, j] = r
            if C is None or r < C:
                pos[t, j] = indptr[e] + r
    R = int(indptr[E])
    row_token = np.full(R, -1, dtype=np.int64)
    row_slot = np.full(R, -1, dtype=np.int64)
    for t in range(T):
        for j in range(k):
            if pos[t, j] >= 0:
                row_token[pos[t, j]] = t
                row_slot[pos[t, j]] = j
    return Permutation(pos=pos, indptr=indptr, counts=counts, kept=kept,
                       row_token=row_token, row_slot=row_slot, rank=rank)


# --------------------------------------------------------------------------
# Experts
# --------------------------------------------------------------------------

def block_sparse_topology(rows_per_expert, block, blocks_per_expert):
    """Block-sparse metadata of the padded expert matrix (MegaBlocks,
    [CMU 15-779 L21] §3.6, Figure 5): the rows of expert e, padded to a
    multiple of ``block``, form block rows that are nonzero exactly in the
    expert's own ``blocks_per_expert`` block columns. Nonzero blocks are
    numbered row-major. Returns (BCSR row offsets, column index of every
    block, row index of every block (the COO part), transpose index: the
    block numbers listed column by column, rows ascending).
    """
    rows = np.asarray(rows_per_expert, dtype=np.int64)
    brows_e = -(-rows // block)                     # block rows per expert
    row_expert = np.repeat(np.arange(len(rows)), brows_e)
    nbr = int(brows_e.sum())
    offsets = np.arange(nbr + 1, dtype=np.int64) * blocks_per_expert
    col = np.concatenate([row_expert[r] * blocks_per_expert + np.arange(blocks_per_expert)
                          for r in range(nbr)]) if nbr else np.zeros(0, dtype=np.int64)
    row = np.repeat(np.arange(nbr), blocks_per_expert)
    # column-major listing: stable sort of the blocks by column
    transpose = np.argsort(col, kind="stable")
    return offsets, col.astype(np.int64), row.astype(np.int64), transpose.astype(np.int64)


def silu(a):
    """SiLU(a) = a * sigmoid(a) (the gate of SwiGLU)."""
    a = np.asarray(a, dtype=np.float64)
    with np.errstate(over="ignore"):
        return a / (1.0 + np.exp(-a))


def swiglu_expert(X, W1e, W3e, W2e):
    """One SwiGLU expert, no biases: W2 (SiLU(W1 x) * (W3 x)).

    [CME295 W2D2] §1.3 (experts are SwiGLU FFNs) and §2.1 (3 d d_ff parameters
    per expert, no bias). Weights in nn.Linear layout: W1e, W3e [d_ff, d],
    W2e [d, d_ff]. X: [n, d] rows; returns [n, d] float64.
    """
    X = np.asarray(X, dtype=np.float64)
    W1e = np.asarray(W1e, dtype=np.float64)
    W3e = np.asarray(W3e, dtype=np.float64)
    W2e = np.asarray(W2e, dtype=np.float64)
    H = silu(X @ W1e.T) * (X @ W3e.T)
    return H @ W2e.T


# --------------------------------------------------------------------------
# Load statistics
# --------------------------------------------------------------------------

def l_aux(f, P, alpha=1.0):
    """L_aux = alpha * E * sum_i f_i P_i ([CME295 W2D2] §3.2; [CS336 L04]
    §2.3.3a with N = number of experts)."""
    f = np.asarray(f, dtype=np.float64)
    P = np.asarray(P, dtype=np.float64)
    E = f.shape[0]
    return float(alpha * E * np.sum(f * P))


def router_z_loss(z):
    """L_z = (1/T) sum_t (log sum_i exp z_{t,i})^2 ([CME295 W2D2] §3.4;
    [CS336 L04] §3.1: it penalises the overall size of the router logits)."""
    z = np.asarray(z, dtype=np.float64)
    m = z.max(axis=1, keepdims=True)
    lse = m[:, 0] + np.log(np.exp(z - m).sum(axis=1))
    return float(np.mean(lse ** 2)) if z.shape[0] else 0.0


def router_entropy(probs):
    """Mean over tokens of the router distribution's entropy, -sum_i p log p
    ([W11 routing] §5, "router entropy"); 0 log 0 = 0."""
    p = np.asarray(probs, dtype=np.float64)
    with np.errstate(divide="ignore", invalid="ignore"):
        h = -np.where(p > 0, p * np.log(p), 0.0).sum(axis=1)
    return float(h.mean()) if p.shape[0] else 0.0


def router_top_gap(probs):
    """Mean over tokens of the gap between the largest and second-largest
    router probability ([W11 routing] §5, "top-1/top-2 gap"); with one expert
    the second is taken as 0."""
    p = np.asarray(probs, dtype=np.float64)
    if p.shape[0] == 0:
        return 0.0
    if p.shape[1] == 1:
        return float(p[:, 0].mean())
    srt = -np.sort(-p, axis=1)
    return float(np.mean(srt[:, 0] - srt[:, 1]))


@dataclass
class LoadStats:
    counts: np.ndarray     # [E] pairs routed before capacity
    kept: np.ndarray       # [E] pairs kept
    f: np.ndarray          # [E] c_e / (T k)
    P: np.ndarray          # [E] mean full-softmax probability
    l_aux: float           # E * sum f P
    dropped: int           # sum (c_e - kept_e)
    max_count: int
    max_over_mean: float   # max_e c_e / (T k / E)
    capacity: Optional[int]
    z_loss: float = 0.0    # router z-loss
    entropy: float = 0.0   # mean router entropy
    top_gap: float = 0.0   # mean top-1 minus top-2 probability


def load_stats(perm: Permutation, probs, T, k, C, z=None):
    """Per-expert load statistics of one batch.

    f and P per [CME295 W2D2] §3.2 (f counts all k choices, P is the mean
    router probability); counts, drops and max/mean load per [W11 routing]
    §3 and §5.
    """
    E = perm.counts.shape[0]
    counts = perm.counts
    f = counts / float(T * k) if T > 0 else np.zeros(E)
    P = np.asarray(probs, dtype=np.float64).mean(axis=0) if T > 0 else np.zeros(E)
    mean_load = T * k / E
    return LoadStats(counts=counts, kept=perm.kept, f=f, P=P,
                     l_aux=l_aux(f, P), dropped=int(np.sum(counts - perm.kept)),
                     max_count=int(counts.max()) if E else 0,
                     max_over_mean=float(counts.max() / mean_load) if T > 0 else 0.0,
                     capacity=C,
                     z_loss=router_z_loss(z) if z is not None else 0.0,
                     entropy=router_entropy(probs) if T > 0 else 0.0,
                     top_gap=router_top_gap(probs) if T > 0 else 0.0)


# --------------------------------------------------------------------------
# The layer
# --------------------------------------------------------------------------

@dataclass
class ForwardResult:
    routing: Routing
    perm: Permutation
    stats: LoadStats
    y: np.ndarray                      # [len(tokens), d] float64
    tokens: np.ndarray                 # token ids whose output rows are in y
    extra: dict = field(default_factory=dict)


def moe_forward(x, W_r, W1, W3, W2, k, capacity_factor=0.0, bias=None,
                bias_mode=BIAS_NONE, Ws1=None, Ws3=None, Ws2=None,
                logits=None, tokens=None, key_dtype=np.float64,
                gate_mode=GATE_SELECTED, drop_order=DROP_TOKEN, pad=None, idx=None):
    """Forward pass of one MoE layer, the sparse per-pair definition.

    Steps in the order of [CMU 15-779 L21] §3.2 (route, permute, compute per
    expert, un-permute and mix):

    1. z = W_r^T x ([CME295 W2D2] §1.3), unless ``logits`` are given.
    2. selection key and top-k; gates = softmax over the selected raw logits.
    3. capacity and permutation by prefix sum.
    4. every kept pair (t, j) evaluates its expert on x_t.
    5. y_t = sum over kept slots j in slot order of g_{t,j} f_{e}(x_t), plus the
       always-on shared expert when given ([CME295 W2D2] §4.1; [CS336 L04]
       §2.1.3b).

    ``W1``, ``W3``, ``W2`` are indexable by expert (``W1[e]`` -> [d_ff, d]);
    ``idx`` [T, k], when given, replaces the top-k selection (for checking a
    selection made by another implementation from the same logits);
    ``tokens`` restricts step 4-5 to a subset of tokens (routing, permutation
    and statistics always cover all tokens). Returns a ForwardResult whose
    ``y`` rows follow ``tokens``.
    """
    x = np.asarray(x)
    T = x.shape[0]
    E = np.asarray(W_r).shape[1] if logits is None else np.asarray(logits).shape[1]
    z = router_logits(x, W_r) if logits is None else np.asarray(logits, dtype=np.float64)
    if logits is not None and key_dtype == np.float32:
        z_key = np.asarray(logits, dtype=np.float32)
    else:
        z_key = z
    key = selection_key(z_key, bias, bias_mode, dtype=key_dtype)
    if idx is None:
        idx = topk_lowest_index(key, k)
    else:   # a selection decided elsewhere (the gates still follow from z)
        idx = np.asarray(idx, dtype=np.int64)
    gate = gates_from_selected(z, idx) if gate_mode == GATE_SELECTED else gates_full_softmax(z, idx)
    probs = softmax_rows(z)
    routing = Routing(idx=idx, gate=gate, probs=probs, key=key)

    C = capacity(capacity_factor, T, k, E)
    perm = permute(idx, E, C, drop_order, pad)
    stats = load_stats(perm, probs, T, k, C, z=z)

    if tokens is None:
        tokens = np.arange(T)
    tokens = np.asarray(tokens, dtype=np.int64)
    d = x.shape[1]
    n = len(tokens)
    # contrib[j, i] = g_{t,j} f_{e_{t,j}}(x_t) for token t = tokens[i], zero if
    # the pair was dropped. Experts are evaluated one at a time on the rows
    # routed to them; each row of a stacked product equals the per-pair
    # product, rows never mix.
    contrib = np.zeros((k, n, d), dtype=np.float64)
    for e in range(E):
        rows, slots = [], []
        for i, t in enumerate(tokens):
            for j in range(k):
                if idx[t, j] == e and perm.pos[t, j] >= 0:
                    rows.append(i)
                    slots.append(j)
        if not rows:
            continue
        X = np.asarray(x[tokens[rows]], dtype=np.float64)
        Oe = swiglu_expert(X, W1[e], W3[e], W2[e])
        for r, (i, j) in enumerate(zip(rows, slots)):
            contrib[j, i] = gate[tokens[i], j] * Oe[r]
    # sum in slot order j = 0 .. k-1
    y = np.zeros((n, d), dtype=np.float64)
    for j in range(k):
        y = y + contrib[j]
    if Ws1 is not None:
        S = swiglu_expert(np.asarray(x[tokens], dtype=np.float64), Ws1, Ws3, Ws2)
        y = y + S
    return ForwardResult(routing=routing, perm=perm, stats=stats, y=y, tokens=tokens)


def unpermute_combine(O_rows, pos, gate, S=None):
    """Un-permute and mix: y_t = sum_{j < k, pos[t,j] >= 0} g_{t,j} O[pos[t,j]]
    in slot order, plus the shared-expert row S_t when given.

    [CMU 15-779 L21] §3.2 step 4 (restore token order, weight by the gates);
    [CME295 W2D2] §4.1 (the shared expert is added for every token).
    O_rows: [R, d] expert outputs in permuted order; pos, gate: [T, k].
    """
    O_rows = np.asarray(O_rows, dtype=np.float64)
    pos = np.asarray(pos)
    gate = np.asarray(gate, dtype=np.float64)
    T, k = pos.shape
    d = O_rows.shape[1] if O_rows.ndim == 2 else (np.asarray(S).shape[1] if S is not None else 0)
    y = np.zeros((T, d), dtype=np.float64)
    for t in range(T):
        for j in range(k):
            if pos[t, j] >= 0:
                y[t] = y[t] + gate[t, j] * O_rows[pos[t, j]]
    if S is not None:
        y = y + np.asarray(S, dtype=np.float64)
    return y


# --------------------------------------------------------------------------
# Closed forms the notes print
# --------------------------------------------------------------------------

def fraction_experts_touched(E, k, B):
    """Expected fraction of experts chosen by at least one of B tokens, each
    token picking a uniformly random k-subset of E experts:
    1 - (C(E-1, k) / C(E, k))^B. ([CME295 W2D2] §2.3 table, top-2 of 8.)"""
    miss_one = math.comb(E - 1, k) / math.comb(E, k)
    return 1.0 - miss_one ** B


def expected_experts_touched(E, k, B):
    """E (1 - (1 - k/E)^B): expected experts touched when every token picks
    each expert independently with probability k/E ([CMU 15-779 L21] §3.1;
    exercise 4 uses it for 256 experts, top-8, B = 32)."""
    return E * (1.0 - (1.0 - k / E) ** B)


@dataclass
class ModelShape:
    layers: int
    d: int
    n_heads: int
    n_kv_heads: int
    head_dim: int
    E: int
    k: int
    d_ff: int
    vocab: int
    tied_embeddings: bool = False
    norms_per_layer: int = 2
    final_norm: bool = True


def param_counts(s: ModelShape):
    """Total and active parameters of a decoder with SwiGLU MoE FFNs.

    Per layer: attention Q, O (d x h*dh) and K, V (d x kv*dh); E experts of
    3 d d_ff; a router d x E; RMSNorm weights. Plus embeddings (two matrices
    unless tied) and the final norm. Active counts k experts instead of E.
    ([CME295 W2D2] §2.1, Mixtral 8x7B count.)
    """
    attn = 2 * s.d * s.n_heads * s.head_dim + 2 * s.d * s.n_kv_heads * s.head_dim
    expert = 3 * s.d * s.d_ff
    router = s.d * s.E
    norms = s.norms_per_layer * s.d
    emb = (1 if s.tied_embeddings else 2) * s.vocab * s.d
    final = s.d if s.final_norm else 0
    total = s.layers * (attn + s.E * expert + router + norms) + emb + final
    active = s.layers * (attn + s.k * expert + router + norms) + emb + final
    return total, active


MIXTRAL_8X7B = ModelShape(layers=32, d=4096, n_heads=32, n_kv_heads=8,
                          head_dim=128, E=8, k=2, d_ff=14336, vocab=32000)
