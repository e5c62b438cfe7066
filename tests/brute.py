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
* capacity by a running per-expert counter over tokens in order instead of a
  prefix sum;
* destination rows by sorting the kept pairs on (expert, token);
* experts by explicit per-token loops over the hidden units.
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
                  Ws1=None, Ws3=None, Ws2=None):
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

    # gates: full softmax renormalised over the selected set
    gate = np.zeros((T, k))
    for t in range(T):
        p = _softmax(list(z[t]))
        den = sum(p[idx[t, j]] for j in range(k))
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
    for t in range(T):
        for j in range(k):
            e = idx[t, j]
            counts[e] += 1
            if C is None or used[e] < C:
                keep[t, j] = True
                used[e] += 1

    # destination rows: kept pairs sorted by (expert, token)
    pairs = sorted((idx[t, j], t, j) for t in range(T) for j in range(k) if keep[t, j])
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
    return dict(z=z, idx=idx, gate=gate, pos=pos, keep=keep, counts=counts,
                kept=np.array(used), y=y, f=f, P=P, l_aux=E * float(np.sum(f * P)),
                capacity=C)
