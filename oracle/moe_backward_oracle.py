"""CPU oracle for the backward pass of one sparse Mixture-of-Experts layer.

TEST INFRASTRUCTURE ONLY, like ``oracle/moe_oracle.py`` (whose forward it
reuses): only the test suite, ``__graft_entry__.smoke()`` and ``bench.py``'s
CPU legs may import it; the CUDA library never does.

The loss whose gradient is taken is

    L = sum_t <dy_t, y_t>  +  alpha * L_aux  +  beta * L_z

with y the layer output, L_aux = E sum_e f_e P_e (f frozen: counts are not
differentiable, [CME295 W2D2] §3.2) and L_z the router z-loss
((1/T) sum_t logsumexp(z_t)^2, [CME295 W2D2] §3.4). The expert selection (top-k
over the biased or unbiased key, capacity drops) is a discrete choice and
carries no gradient; the selection bias gets none ([CME295 W2D2] §4.2: it
only steers which experts are picked).

Everything is numpy float64, one expert at a time; each step is written out
from the chain rule of the forward definition:

* combine y_t = sum_j g_{t,j} o_{t,j}: dg_{t,j} = <dy_t, o_{t,j}> and
  do_{t,j} = g_{t,j} dy_t (kept pairs only);
* expert o = W2 h, h = SiLU(a) * b, a = W1 x, b = W3 x:
  dW2 += do h^T, dh = W2^T do, da = dh * b * SiLU'(a), db = dh * SiLU(a),
  dW1 += da x^T, dW3 += db x^T, dx += W1^T da + W3^T db,
  with SiLU'(a) = sigma(a) (1 + a (1 - sigma(a)));
* gates, softmax over the k selected raw logits ([CME295 W2D2] §1.3):
  dz_{t,e_j} += g_j (dg_j - sum_l g_l dg_l); for the full-softmax (Switch)
  gates g_j = p_{t,e_j}: dz_t += p_t * (v_t - <p_t, v_t>), v_{t,e_j} = dg_j;
* balance loss, the notes' closed form ([CME295 W2D2] §3.2):
  dL_aux/dz_{t,i} = (E / T) p_{t,i} (f_i - sum_j p_{t,j} f_j);
* z-loss: dL_z/dz_{t,i} = (2 / T) lse_t p_{t,i};
* router z = W_r^T x: dW_r = x^T dz, dx += dz W_r^T.

Parity pins (``tests/test_backward_pins.py``): central finite differences of
the forward oracle's loss in every input on small layers, the notes' aux-loss
gradient against finite differences of L_aux with f frozen, the special case
E = k = 1 (a dense SwiGLU FFN, gate 1), and the bias update's hand example.
"""

from __future__ import annotations

from dataclasses import dataclass
from typing import Optional

import numpy as np

from oracle import moe_oracle as O


def silu_grad(a):
    """d/da of a * sigma(a) = sigma(a) (1 + a (1 - sigma(a)))."""
    a = np.asarray(a, dtype=np.float64)
    with np.errstate(over="ignore"):
        s = 1.0 / (1.0 + np.exp(-a))
    return s * (1.0 + a * (1.0 - s))


def expert_backward(X, dO, W1e, W3e, W2e):
    """Gradients of one SwiGLU expert over its rows X [n, d] given dO [n, d]
    (already gate-scaled): returns (dX, dW1, dW3, dW2, O) with O = the
    ungated expert output of the rows."""
    X = np.asarray(X, dtype=np.float64)
    dO = np.asarray(dO, dtype=np.float64)
    W1e = np.asarray(W1e, dtype=np.float64)
    W3e = np.asarray(W3e, dtype=np.float64)
    W2e = np.asarray(W2e, dtype=np.float64)
    A = X @ W1e.T
    B = X @ W3e.T
    H = O.silu(A) * B
    dW2 = dO.T @ H
    dH = dO @ W2e
    dA = dH * B * silu_grad(A)
    dB = dH * O.silu(A)
    dW1 = dA.T @ X
    dW3 = dB.T @ X
    dX = dA @ W1e + dB @ W3e
    return dX, dW1, dW3, dW2, H @ W2e.T


def router_dz(z, idx, keep, dgate, gate_mode, f, alpha, beta):
    """Gradient of the loss w.r.t. the router logits z [T, E]: gates,
    balance loss (f frozen) and z-loss, each as in the module docstring."""
    z = np.asarray(z, dtype=np.float64)
    T, E = z.shape
    p = O.softmax_rows(z)
    dz = np.zeros((T, E))
    k = idx.shape[1]
    for t in range(T):
        dg = np.where(keep[t], dgate[t], 0.0)
        if gate_mode == O.GATE_SELECTED:
            zs = z[t, idx[t]]
            g = np.exp(zs - zs.max())
            g = g / g.sum()
            s = float(np.dot(g, dg))
            for j in range(k):
                dz[t, idx[t, j]] += g[j] * (dg[j] - s)
        else:
            v = np.zeros(E)
            for j in range(k):
                v[idx[t, j]] += dg[j]
            dz[t] += p[t] * (v - np.dot(p[t], v))
    if T > 0 and alpha != 0.0:
        pf = p @ f
        dz += alpha * (E / T) * p * (f[None, :] - pf[:, None])
    if T > 0 and beta != 0.0:
        m = z.max(axis=1, keepdims=True)
        lse = m[:, 0] + np.log(np.exp(z - m).sum(axis=1))
        dz += beta * (2.0 / T) * lse[:, None] * p
    return dz


@dataclass
class BackwardResult:
    dx: np.ndarray
    dW_r: np.ndarray
    dW1: np.ndarray
    dW3: np.ndarray
    dW2: np.ndarray
    dWs1: Optional[np.ndarray]
    dWs3: Optional[np.ndarray]
    dWs2: Optional[np.ndarray]
    dz: np.ndarray        # [T, E] router-logit gradient
    dgate: np.ndarray     # [T, k] <dy_t, o_{t,j}> (0 for dropped pairs)
    forward: O.ForwardResult


def moe_backward(x, W_r, W1, W3, W2, k, dy, capacity_factor=0.0, bias=None, bias_mode=O.BIAS_NONE,
                 Ws1=None, Ws3=None, Ws2=None, alpha=0.0, beta=0.0, gate_mode=O.GATE_SELECTED,
                 drop_order=O.DROP_TOKEN, logits=None, key_dtype=np.float64, idx=None, f=None):
    """Gradients of L = <dy, y> + alpha L_aux + beta L_z w.r.t. x, W_r and the
    expert weights. ``W1``, ``W3``, ``W2`` are indexable by expert; ``f``
    replaces the batch's own f in L_aux (a data-parallel replica uses the
    global one)."""
    x = np.asarray(x, dtype=np.float64)
    dy = np.asarray(dy, dtype=np.float64)
    T, d = x.shape
    W_r64 = None if W_r is None else np.asarray(W_r, dtype=np.float64)
    fwd = O.moe_forward(x, W_r, W1, W3, W2, k, capacity_factor, bias, bias_mode, logits=logits,
                        key_dtype=key_dtype, gate_mode=gate_mode, drop_order=drop_order, idx=idx)
    idx, gate = fwd.routing.idx, fwd.routing.gate
    pos = fwd.perm.pos
    keep = pos >= 0
    E = fwd.stats.counts.shape[0]
    z = O.router_logits(x, W_r) if logits is None else np.asarray(logits, dtype=np.float64)

    d_ff = np.asarray(W1[0]).shape[0]
    dx = np.zeros((T, d))
    dW1 = np.zeros((E, d_ff, d))
    dW3 = np.zeros((E, d_ff, d))
    dW2 = np.zeros((E, d, d_ff))
    dgate = np.zeros((T, k))
    for e in range(E):
        pairs = [(t, j) for t in range(T) for j in range(k) if idx[t, j] == e and keep[t, j]]
        if not pairs:
            continue
        ts = np.array([t for t, _ in pairs])
        js = np.array([j for _, j in pairs])
        dO_rows = gate[ts, js][:, None] * dy[ts]
        dX, g1, g3, g2, O_rows = expert_backward(x[ts], dO_rows, W1[e], W3[e], W2[e])
        dW1[e], dW3[e], dW2[e] = g1, g3, g2
        dgate[ts, js] = np.einsum("nd,nd->n", dy[ts], O_rows)
        np.add.at(dx, ts, dX)

    dWs1 = dWs3 = dWs2 = None
    if Ws1 is not None:
        dXs, dWs1, dWs3, dWs2, _ = expert_backward(x, dy, Ws1, Ws3, Ws2)
        dx += dXs

    dz = router_dz(z, idx, keep, dgate, gate_mode, fwd.stats.f if f is None else np.asarray(f, dtype=np.float64),
                   alpha, beta)
    dW_r = x.T @ dz
    if W_r64 is not None:
        dx += dz @ W_r64.T
    return BackwardResult(dx=dx, dW_r=dW_r, dW1=dW1, dW3=dW3, dW2=dW2, dWs1=dWs1, dWs3=dWs3, dWs2=dWs2,
                          dz=dz, dgate=dgate, forward=fwd)


def loss(x, W_r, W1, W3, W2, k, dy, f_frozen, capacity_factor=0.0, bias=None, bias_mode=O.BIAS_NONE,
         Ws1=None, Ws3=None, Ws2=None, alpha=0.0, beta=0.0, gate_mode=O.GATE_SELECTED,
         drop_order=O.DROP_TOKEN):
    """The scalar L whose gradient moe_backward returns, with the balance
    loss's f frozen at ``f_frozen`` (for finite-difference checks)."""
    fwd = O.moe_forward(x, W_r, W1, W3, W2, k, capacity_factor, bias, bias_mode, Ws1, Ws3, Ws2,
                        gate_mode=gate_mode, drop_order=drop_order)
    z = O.router_logits(x, W_r)
    E = z.shape[1]
    P = O.softmax_rows(z).mean(axis=0)
    val = float(np.sum(np.asarray(dy, dtype=np.float64) * fwd.y))
    val += alpha * E * float(np.sum(f_frozen * P))
    val += beta * O.router_z_loss(z)
    return val, fwd


def bias_update(bias, counts, gamma, T, k):
    """Auxiliary-loss-free balancing ([CMU 15-779 L21] §2.4, DeepSeek-V3):
    after a step, an expert whose load is above the mean T k / E has its
    selection bias lowered by gamma, one below the mean raised by gamma; one
    exactly at the mean keeps its bias."""
    b = np.asarray(bias, dtype=np.float64).copy()
    c = np.asarray(counts, dtype=np.float64)
    mean = T * k / c.shape[0]
    b -= gamma * np.sign(c - mean)
    return b
