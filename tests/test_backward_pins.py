"""Pins of the backward oracle (CPU): its analytic gradients against central
finite differences of the forward oracle's loss, the notes' closed-form
balance-loss gradient, and the auxiliary-loss-free bias update."""

import math

import numpy as np
import pytest

from oracle import moe_oracle as O
from oracle import moe_backward_oracle as B


def _layer(rng, T, d, E, d_ff, shared=False):
    x = rng.standard_normal((T, d))
    W_r = rng.standard_normal((d, E)) / math.sqrt(d) * 2.0
    W1 = rng.standard_normal((E, d_ff, d)) / math.sqrt(d)
    W3 = rng.standard_normal((E, d_ff, d)) / math.sqrt(d)
    W2 = rng.standard_normal((E, d, d_ff)) / math.sqrt(d_ff)
    sh = {}
    if shared:
        sh = dict(Ws1=rng.standard_normal((d_ff, d)) / math.sqrt(d),
                  Ws3=rng.standard_normal((d_ff, d)) / math.sqrt(d),
                  Ws2=rng.standard_normal((d, d_ff)) / math.sqrt(d_ff))
    return x, W_r, W1, W3, W2, sh


def _fd(fn, arr, eps=1e-6):
    """Central differences of the scalar fn() in every entry of arr (in place)."""
    g = np.zeros_like(arr)
    it = np.nditer(arr, flags=["multi_index"])
    for _ in it:
        i = it.multi_index
        old = arr[i]
        arr[i] = old + eps
        up = fn()
        arr[i] = old - eps
        dn = fn()
        arr[i] = old
        g[i] = (up - dn) / (2 * eps)
    return g


CASES = [
    dict(T=6, d=5, E=4, k=2, d_ff=3, cf=0.0, gate=O.GATE_SELECTED, shared=False, alpha=0.0, beta=0.0),
    dict(T=7, d=4, E=4, k=2, d_ff=3, cf=0.75, gate=O.GATE_SELECTED, shared=True, alpha=0.3, beta=0.05),
    dict(T=5, d=4, E=3, k=1, d_ff=2, cf=0.0, gate=O.GATE_FULL, shared=False, alpha=0.2, beta=0.0),
    dict(T=6, d=3, E=5, k=3, d_ff=2, cf=0.6, gate=O.GATE_FULL, shared=False, alpha=0.0, beta=0.1),
]


@pytest.mark.parametrize("c", CASES)
def test_gradients_match_finite_differences(c):
    rng = np.random.default_rng(100 + c["T"] * 7 + c["E"])
    x, W_r, W1, W3, W2, sh = _layer(rng, c["T"], c["d"], c["E"], c["d_ff"], c["shared"])
    dy = rng.standard_normal((c["T"], c["d"]))
    kw = dict(capacity_factor=c["cf"], alpha=c["alpha"], beta=c["beta"], gate_mode=c["gate"], **sh)
    res = B.moe_backward(x, W_r, W1, W3, W2, c["k"], dy, **kw)
    # routing must be far from ties so that the perturbations do not flip it
    z = O.router_logits(x, W_r)
    srt = -np.sort(-z, axis=1)
    if c["k"] < c["E"]:
        assert (srt[:, c["k"] - 1] - srt[:, c["k"]]).min() > 1e-4
    if c["cf"] > 0:
        assert res.forward.stats.dropped > 0
    f0 = res.forward.stats.f.copy()
    idx0 = res.forward.routing.idx.copy()

    def L():
        val, fwd = B.loss(x, W_r, W1, W3, W2, c["k"], dy, f0, **kw)
        assert np.array_equal(fwd.routing.idx, idx0)
        return val

    for name, arr, got in [("x", x, res.dx), ("W_r", W_r, res.dW_r), ("W1", W1, res.dW1),
                           ("W3", W3, res.dW3), ("W2", W2, res.dW2)] + (
            [("Ws1", sh["Ws1"], res.dWs1), ("Ws3", sh["Ws3"], res.dWs3), ("Ws2", sh["Ws2"], res.dWs2)]
            if c["shared"] else []):
        want = _fd(L, arr)
        scale = max(1.0, np.abs(want).max())
        assert np.abs(got - want).max() < 1e-6 * scale, name


def test_balance_loss_gradient_is_the_notes_closed_form():
    # [CME295 W2D2] §3.2: dL_aux/dz_{t,i} = (alpha E / T) p_{t,i} (f_i - sum_j p_{t,j} f_j)
    rng = np.random.default_rng(5)
    T, E, alpha = 9, 6, 0.7
    z = rng.standard_normal((T, E)) * 1.5
    f = rng.dirichlet(np.ones(E))
    idx = O.topk_lowest_index(z, 2)
    dz = B.router_dz(z, idx, np.zeros_like(idx, dtype=bool), np.zeros(idx.shape), O.GATE_SELECTED, f, alpha, 0.0)

    def laux():
        return alpha * E * float(np.sum(f * O.softmax_rows(z).mean(axis=0)))
    want = _fd(laux, z)
    assert np.allclose(dz, want, rtol=1e-6, atol=1e-9)
    # exercise 5's partial derivative with respect to P_1 is E f_1
    g = np.array([0.7, 0.1, 0.1, 0.1])
    assert 4 * g[0] == pytest.approx(2.8)


def test_z_loss_gradient_matches_finite_differences():
    rng = np.random.default_rng(6)
    z = rng.standard_normal((5, 7)) * 3
    dz = B.router_dz(z, O.topk_lowest_index(z, 2), np.zeros((5, 2), bool), np.zeros((5, 2)),
                     O.GATE_SELECTED, np.zeros(7), 0.0, 0.4)
    want = _fd(lambda: 0.4 * O.router_z_loss(z), z)
    assert np.allclose(dz, want, rtol=1e-6, atol=1e-9)


def test_selected_gates_of_a_single_choice_carry_no_gradient():
    # k = 1 with the selected softmax: the gate is 1 whatever z is
    rng = np.random.default_rng(7)
    x, W_r, W1, W3, W2, _ = _layer(rng, 6, 4, 4, 3)
    res = B.moe_backward(x, W_r, W1, W3, W2, 1, rng.standard_normal((6, 4)))
    assert np.abs(res.dz).max() == 0.0 and np.abs(res.dW_r).max() == 0.0


def test_bias_update_hand_example():
    # [CMU 15-779 L21] §2.4: above the mean load -> b - gamma, below -> b + gamma
    b = B.bias_update([0.5, 0.0, -0.2, 0.1], [5, 1, 2, 0], 0.001, T=4, k=2)   # mean load 2
    assert b.tolist() == pytest.approx([0.499, 0.001, -0.2, 0.101], abs=1e-15)


def test_planted_silu_derivative_mistake_is_caught(monkeypatch):
    rng = np.random.default_rng(8)
    x, W_r, W1, W3, W2, _ = _layer(rng, 5, 4, 3, 2)
    dy = rng.standard_normal((5, 4))
    monkeypatch.setattr(B, "silu_grad", lambda a: 1.0 / (1.0 + np.exp(-np.asarray(a))))   # sigma only
    res = B.moe_backward(x, W_r, W1, W3, W2, 2, dy)
    f0 = res.forward.stats.f

    def L():
        return B.loss(x, W_r, W1, W3, W2, 2, dy, f0)[0]
    assert not np.allclose(res.dW1, _fd(L, W1), rtol=1e-4, atol=1e-8)
