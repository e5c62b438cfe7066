"""Dense-masked brute force of the MoE layer, for tiny token counts.

Test-only cross-check of the oracle, written independently of it: every
expert is evaluated on every token and the gate matrix zeroes the unselected
and dropped pairs (formulation 0, "every expert computes", of [CMU 15-779 L21]
§3.4). Each step uses a different procedure from the oracle's:

* top-k by k rounds of arg-max with masking (np.argmax returns the first,
  i.e. lowest, index among equal maxima) instead of a stable sort;
* gates as the full softmax renormalised over the selected pair set
  ([CMU 15-779 L21] §2.1, s_i = g_{e_i} / sum_j g_{e_j}) instead of a softmax
  over the selected logits;
* capacity by a running per-expert counter over the pairs in visiting order
  (token by token, or, for GShard's slot priority, all first choices before
  any second choice) instead of a prefix sum;
* destination rows by sorting the kept pairs on (expert, visiting order);
* experts by explicit per-token loops over the hidden units;
* z-loss, entropy and top-1/top-2 gap by explicit per-token loops.
"""

from __future__ import annotations

import math

import numpy as np


def _softmax(v):
    m = max(v)
    ex = [math.exp(a - m) for a in v]
    s = sum(ex)
    return [a / s for a in ex]


def brute_forward(x, W_r, W1, W3, W2, k, cf=0.0, bias=None, bias_mode=0,
                  Ws1=None, Ws3=None, Ws2=None, gate_mode=0, drop_order=0):
    x = np.asarray(x, dtype=np.float64)
    W_r = np.asarray(W_r, dtype=np.float64)
    T, d = x.shape
    E = W_r.shape[1]
    z = np.einsum("td,de->te", x, W_r)

    # selection key and top-k by repeated arg-max
    idx = np.zeros((T, k), dtype=np.int64)
    for t in range(T):
        if bias_mode == 0:
            key = z[t].copy()
        elif bias_mode == 1:
            key = z[t] + np.asarray(bias, dtype=np.float64)
        else:
            key = np.asarray(_softmax(list(z[t]))) + np.asarray(bias, dtype=np.float64)
        for j in range(k):
            e = int(np.argmax(key))
            idx[t, j] = e
            key[e] = -np.inf

    # gates: full softmax renormalised over the selected set (gate_mode 0),
    # or the full-softmax probability itself (gate_mode 1)
    gate = np.zeros((T, k))
    for t in range(T):
        p = _softmax(list(z[t]))
        den = sum(p[idx[t, j]] for j in range(k)) if gate_mode == 0 else 1.0
        for j in range(k):
            gate[t, j] = p[idx[t, j]] / den

    # capacity by running counters in token order
    C = None
    cf32 = float(np.float32(cf))
    if cf32 > 0:
        C = int(math.ceil(cf32 * T * k / E))
    used = [0] * E
    keep = np.zeros((T, k), dtype=bool)
    counts = np.zeros(E, dtype=np.int64)
    # visiting order: token by token (drop_order 0), or all first choices,
    # then all second choices, ... (drop_order 1)
    order = ([(t, j) for t in range(T) for j in range(k)] if drop_order == 0
             else [(t, j) for j in range(k) for t in range(T)])
    for t, j in order:
        e = idx[t, j]
        counts[e] += 1
        if C is None or used[e] < C:
            keep[t, j] = True
            used[e] += 1

    # destination rows: kept pairs sorted by expert, then in visiting order
    rank_in_order = {tj: r for r, tj in enumerate(order)}
    pairs = sorted((idx[t, j], rank_in_order[(t, j)], t, j) for t in range(T) for j in range(k) if keep[t, j])
    pairs = [(e, t, j) for e, _, t, j in pairs]
    pos = np.full((T, k), -1, dtype=np.int64)
    for r, (_, t, j) in enumerate(pairs):
        pos[t, j] = r

    # every expert on every token, by explicit loops over hidden units
    def expert(v, A, B, Cm):
        A = np.asarray(A, dtype=np.float64)
        B = np.asarray(B, dtype=np.float64)
        Cm = np.asarray(Cm, dtype=np.float64)
        h = np.zeros(A.shape[0])
        for u in range(A.shape[0]):
            a = float(np.dot(A[u], v))
            b = float(np.dot(B[u], v))
            h[u] = (a / (1.0 + math.exp(-a)) if a > -700 else 0.0) * b
        return Cm @ h

    G = np.zeros((T, E))
    for t in range(T):
        for j in range(k):
            if keep[t, j]:
                G[t, idx[t, j]] = gate[t, j]
    y = np.zeros((T, d))
    for e in range(E):
        if not G[:, e].any():
            continue
        for t in range(T):
            if G[t, e] != 0.0:
                y[t] += G[t, e] * expert(x[t], W1[e], W3[e], W2[e])
    if Ws1 is not None:
        for t in range(T):
            y[t] += expert(x[t], Ws1, Ws3, Ws2)

    p_all = np.array([_softmax(list(z[t])) for t in range(T)])
    f = counts / (T * k)
    P = p_all.mean(axis=0)
    # router statistics by explicit loops
    zl = ent = gap = 0.0
    for t in range(T):
        lse = math.log(sum(math.exp(v) for v in z[t]))
        zl += lse * lse
        ent += -sum(pv * math.log(pv) for pv in p_all[t] if pv > 0)
        srt = sorted(p_all[t], reverse=True)
        gap += srt[0] - (srt[1] if E > 1 else 0.0)
    return dict(z=z, idx=idx, gate=gate, pos=pos, keep=keep, counts=counts,
                kept=np.array(used), y=y, f=f, P=P, l_aux=E * float(np.sum(f * P)),
                capacity=C, z_loss=zl / T, entropy=ent / T, top_gap=gap / T)
