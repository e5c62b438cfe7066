"""Pins of the CPU oracle to what the notes fix (CPU only, no GPU).

Each test names the passage it checks. Together they are chosen so that a
plausible slip in the oracle (a dropped k in the capacity, token-major instead
of expert-major numbering, gates without renormalisation, ties broken upward,
a missing shared expert, a transposed weight) fails at least one of them; the
last group plants such slips in a copy of the oracle and checks that a pin
catches each one.
"""

import math

import numpy as np
import pytest

from golden_io import load
from brute import brute_forward
from oracle import moe_oracle as O


def _rand_layer(rng, T, d, E, d_ff, shared=False):
    x = rng.standard_normal((T, d))
    W_r = rng.standard_normal((d, E)) / math.sqrt(d)
    W1 = rng.standard_normal((E, d_ff, d)) / math.sqrt(d)
    W3 = rng.standard_normal((E, d_ff, d)) / math.sqrt(d)
    W2 = rng.standard_normal((E, d, d_ff)) / math.sqrt(d_ff)
    sh = {}
    if shared:
        sh = dict(Ws1=rng.standard_normal((d_ff, d)) / math.sqrt(d),
                  Ws3=rng.standard_normal((d_ff, d)) / math.sqrt(d),
                  Ws2=rng.standard_normal((d, d_ff)) / math.sqrt(d_ff))
    return x, W_r, W1, W3, W2, sh


# --- permutation: worked examples ([CMU 15-779 L21] §3.3 and exercise 2) ---

def test_prefix_sum_worked_example():
    g = load("prefix_sum_worked_example.txt")
    perm = O.permute(g["idx"], g["E"])
    assert perm.pos.tolist() == g["pos"].tolist()
    assert perm.indptr.tolist() == g["indptr"].tolist()
    # the slides' intermediate: the expert-major inclusive cumsum, reshaped back
    T, E = g["idx"].shape[0], g["E"]
    mask = np.zeros((T, E), dtype=np.int64)
    for t in range(T):
        mask[t, g["idx"][t]] = 1
    cs = np.cumsum(mask.T.reshape(-1)).reshape(E, T).T
    assert cs.tolist() == g["cumsum"].tolist()


def test_exercise2_permutation():
    g = load("exercise2_permutation.txt")
    perm = O.permute(g["idx"], g["E"])
    assert perm.pos.tolist() == g["pos"].tolist()
    assert perm.indptr.tolist() == g["indptr"].tolist()
    # every destination row is used exactly once and maps back to its token
    R = perm.indptr[-1]
    assert sorted(perm.pos.reshape(-1).tolist()) == list(range(R))
    for t in range(perm.pos.shape[0]):
        for j in range(perm.pos.shape[1]):
            assert perm.row_token[perm.pos[t, j]] == t


def test_permutation_order_independent_of_slot_order():
    # the destination rows depend on the chosen set, not on the slot order
    g = load("exercise2_permutation.txt")
    flipped = g["idx"][:, ::-1]
    perm = O.permute(flipped, g["E"])
    assert perm.pos[:, ::-1].tolist() == g["pos"].tolist()


# --- capacity ([CMU 15-779 L21] §3.5 and exercise 3; [W11 routing] §3) ---

def test_exercise3_capacity():
    g = load("exercise3_capacity.txt")
    C = O.capacity(g["cf"], g["N"], g["k"], g["E"])
    assert C == g["C"]
    # construct a routing in which expert 0 receives exactly `busiest` pairs
    N, E, k = g["N"], g["E"], g["k"]
    idx = np.zeros((N, k), dtype=np.int64)
    rng = np.random.default_rng(0)
    for t in range(N):
        if t < g["busiest"]:
            other = 1 + rng.integers(0, E - 1)
            idx[t] = [0, other]
        else:
            idx[t] = 1 + rng.choice(E - 1, size=2, replace=False)
    perm = O.permute(idx, E, C)
    assert perm.counts[0] == g["busiest"]
    assert perm.counts[0] - perm.kept[0] == g["dropped_busiest"]
    # the first C pairs in token order survive, the rest are dropped
    rows0 = [t for t in range(N) if 0 in idx[t]]
    assert all(perm.pos[t, 0] >= 0 for t in rows0[:C])
    assert all(perm.pos[t, 0] == -1 for t in rows0[C:])
    assert E * g["busiest"] == g["dynamic_rows"]
    assert N * k == g["needed_rows"]
    assert round(g["dynamic_rows"] / g["needed_rows"], 2) == g["ratio"]


def test_capacity_skewed_config_value():
    # Mixtral shape, T = 16384, top-2 of 8, cf = 1.25 -> ceil(1.25 * 16384 * 2 / 8) = 5120
    assert O.capacity(1.25, 16384, 2, 8) == 5120
    assert O.capacity(0.0, 16384, 2, 8) is None
    assert O.capacity(-1.0, 16384, 2, 8) is None


def test_kept_rows_are_dense_and_expert_major():
    rng = np.random.default_rng(3)
    T, E, k = 300, 6, 2
    z = rng.standard_normal((T, E))
    idx = O.topk_lowest_index(z, k)
    C = O.capacity(0.9, T, k, E)
    perm = O.permute(idx, E, C)
    assert (perm.kept == np.minimum(perm.counts, C)).all()
    R = perm.indptr[-1]
    assert sorted(p for p in perm.pos.reshape(-1) if p >= 0) == list(range(R))
    for e in range(E):
        toks = perm.row_token[perm.indptr[e]:perm.indptr[e + 1]]
        assert (np.diff(toks) > 0).all()           # token order inside an expert
        assert all(e in idx[t] for t in toks)


# --- load statistics ([CME295 W2D2] §3.2; [CMU 15-779 L21] §2.4 and exercise 5) ---

def test_exercise5_laux_and_gradient():
    g = load("exercise5_laux.txt")
    assert O.l_aux(g["f"], g["P"]) == pytest.approx(g["l_aux"], abs=1e-12)
    h = 1e-6
    grads = []
    for i in range(4):
        P = g["P"].astype(float).copy()
        P[i] += h
        grads.append((O.l_aux(g["f"], P) - O.l_aux(g["f"], g["P"])) / h)
    assert grads[0] == pytest.approx(g["dl_dP1"], rel=1e-5)
    for gi in grads[1:]:
        assert gi == pytest.approx(g["dl_dP_other"], rel=1e-5)


def test_laux_uniform_and_collapse():
    g = load("load_balance_uniform.txt")
    for E in (4, 8, 256):
        u = np.full(E, 1.0 / E)
        assert O.l_aux(u, u, alpha=g["alpha"]) == pytest.approx(g["uniform"], abs=1e-12)
        f = np.zeros(E)
        f[0] = 1.0
        P = np.full(E, 1e-4 / (E - 1))
        P[0] = 1 - 1e-4
        assert O.l_aux(f, P) == pytest.approx(E, rel=1e-3)


def test_load_stats_uniform_routing_gives_one():
    # 8 tokens, 8 experts, token t picks {t, t+1}: every expert gets 2 pairs;
    # with equal probabilities L_aux = E * sum (1/E)(1/E) = 1
    E, k, T = 8, 2, 8
    idx = np.array([[t, (t + 1) % E] for t in range(T)])
    perm = O.permute(idx, E)
    st = O.load_stats(perm, np.full((T, E), 1.0 / E), T, k, None)
    assert st.l_aux == pytest.approx(1.0, abs=1e-15)
    assert st.f.tolist() == [1.0 / E] * E
    assert st.dropped == 0 and st.max_over_mean == 1.0


def test_call_count_and_mean_load():
    g = load("counts_and_load.txt")
    rng = np.random.default_rng(1)
    z = rng.standard_normal((g["calls_T"], g["calls_E"]))
    perm = O.permute(O.topk_lowest_index(z, g["calls_k"]), g["calls_E"])
    assert perm.counts.sum() == g["calls"]
    z = rng.standard_normal((g["load_N"], g["load_E"]))
    perm = O.permute(O.topk_lowest_index(z, g["load_k"]), g["load_E"])
    assert perm.counts.mean() == g["mean_load"]


# --- gates and top-k ([CME295 W2D2] §1.3 and §4.2; [MoE tutorial] route()) ---

def test_gates_equal_renormalised_full_softmax():
    # [CMU 15-779 L21] §2.1: s_i = g_{e_i} / sum_j g_{e_j} with g = softmax(z)
    rng = np.random.default_rng(2)
    z = rng.standard_normal((50, 8)) * 3
    idx = O.topk_lowest_index(z, 2)
    g = O.gates_from_selected(z, idx)
    p = O.softmax_rows(z)
    ps = np.take_along_axis(p, idx, axis=1)
    assert np.allclose(g, ps / ps.sum(axis=1, keepdims=True), rtol=1e-13, atol=0)
    assert np.allclose(g.sum(axis=1), 1.0, rtol=0, atol=1e-15)
    assert (g[:, 0] >= g[:, 1]).all()   # descending key order with no bias


def test_tie_break_lowest_index():
    # equal router columns give exactly equal logits; the lower index wins
    rng = np.random.default_rng(4)
    d, E = 16, 6
    W_r = rng.standard_normal((d, E))
    x = rng.standard_normal((10, d))
    big = np.abs(W_r).sum(axis=1) * 0 + 10.0
    W_r[:, 2] = big
    W_r[:, 4] = big
    x = np.abs(x)
    z = O.router_logits(x, W_r)
    assert (z[:, 2] == z[:, 4]).all()
    idx = O.topk_lowest_index(z, 2)
    assert (idx[:, 0] == 2).all() and (idx[:, 1] == 4).all()
    idx1 = O.topk_lowest_index(z, 1)
    assert (idx1[:, 0] == 2).all()
    # all-equal logits pick 0..k-1 in order
    assert O.topk_lowest_index(np.zeros((3, 8)), 3).tolist() == [[0, 1, 2]] * 3


def test_bias_selects_but_gates_use_raw_scores():
    z = np.array([[2.0, 1.0, 0.0]])
    r = O.route(z, 2, bias=[0.0, 0.0, 5.0], bias_mode=O.BIAS_LOGIT)
    assert r.idx.tolist() == [[2, 0]]
    e2 = math.exp(2.0)
    assert r.gate[0].tolist() == pytest.approx([1 / (1 + e2), e2 / (1 + e2)], rel=1e-14)
    # bias on the softmax score ([CS336 L04] §2.3.3c): softmax(z) = (.665, .245, .090)
    r = O.route(z, 2, bias=[0.0, 0.5, 0.0], bias_mode=O.BIAS_PROB)
    assert r.idx.tolist() == [[1, 0]]
    e1 = math.exp(1.0)
    assert r.gate[0].tolist() == pytest.approx([e1 / (e1 + e2), e2 / (e1 + e2)], rel=1e-14)
    # no bias: plain top-k of z
    r = O.route(z, 2)
    assert r.idx.tolist() == [[0, 1]]


# --- the layer: special cases and brute force ---

def test_single_expert_top1_is_dense_swiglu():
    # [CME295 W2D2] §B: with E = 1, k = 1 the layer equals a dense SwiGLU FFN
    rng = np.random.default_rng(5)
    x, W_r, W1, W3, W2, _ = _rand_layer(rng, 20, 16, 1, 24)
    res = O.moe_forward(x, W_r, W1, W3, W2, k=1)
    a = x @ W1[0].T
    dense = ((a / (1 + np.exp(-a))) * (x @ W3[0].T)) @ W2[0].T
    assert np.array_equal(res.routing.gate, np.ones((20, 1)))
    assert np.allclose(res.y, dense, rtol=1e-14, atol=1e-14)


def test_k_equal_E_is_dense_mixture():
    # k = E: the selected-softmax gates are the full softmax; the layer is the
    # dense mixture sum_e softmax(z)_e f_e(x) ([CME295 W2D2] §1.3)
    rng = np.random.default_rng(6)
    T, d, E, d_ff = 12, 16, 5, 20
    x, W_r, W1, W3, W2, _ = _rand_layer(rng, T, d, E, d_ff)
    res = O.moe_forward(x, W_r, W1, W3, W2, k=E)
    p = O.softmax_rows(x @ W_r)
    dense = np.zeros((T, d))
    for e in range(E):
        a = x @ W1[e].T
        dense += p[:, e:e + 1] * (((a / (1 + np.exp(-a))) * (x @ W3[e].T)) @ W2[e].T)
    assert np.allclose(res.y, dense, rtol=1e-12, atol=1e-13)


@pytest.mark.parametrize("case", [
    dict(T=40, d=16, E=8, d_ff=24, k=2, cf=0.0, mode=0, shared=False),
    dict(T=64, d=12, E=6, d_ff=20, k=3, cf=0.75, mode=0, shared=False),
    dict(T=33, d=8, E=16, d_ff=16, k=4, cf=1.0, mode=2, shared=True),
    dict(T=50, d=8, E=8, d_ff=8, k=2, cf=1.25, mode=1, shared=False),
    dict(T=17, d=8, E=4, d_ff=8, k=1, cf=0.5, mode=1, shared=True),
    dict(T=48, d=8, E=6, d_ff=8, k=3, cf=0.6, mode=0, shared=False, gate=1, drop=1),
    dict(T=30, d=8, E=8, d_ff=8, k=1, cf=0.5, mode=1, shared=False, gate=1, drop=0),
    dict(T=41, d=8, E=4, d_ff=8, k=2, cf=0.7, mode=2, shared=True, gate=0, drop=1),
])
def test_oracle_matches_dense_masked_brute_force(case):
    rng = np.random.default_rng(case["T"] * 7 + case["E"])
    x, W_r, W1, W3, W2, sh = _rand_layer(rng, case["T"], case["d"], case["E"],
                                         case["d_ff"], case["shared"])
    bias = rng.uniform(-0.5, 0.5, case["E"]) if case["mode"] else None
    if case["mode"] == 1:
        bias = bias * 4
    gm, do = case.get("gate", 0), case.get("drop", 0)
    res = O.moe_forward(x, W_r, W1, W3, W2, k=case["k"], capacity_factor=case["cf"],
                        bias=bias, bias_mode=case["mode"], gate_mode=gm, drop_order=do, **sh)
    b = brute_forward(x, W_r, W1, W3, W2, k=case["k"], cf=case["cf"], bias=bias,
                      bias_mode=case["mode"], gate_mode=gm, drop_order=do, **sh)
    assert np.array_equal(res.routing.idx, b["idx"])
    assert np.array_equal(res.perm.pos, b["pos"])
    assert np.array_equal(res.perm.counts, b["counts"])
    assert np.array_equal(res.perm.kept, b["kept"])
    assert res.stats.capacity == b["capacity"]
    assert np.allclose(res.routing.gate, b["gate"], rtol=1e-13, atol=0)
    scale = np.abs(b["y"]).max()
    assert np.abs(res.y - b["y"]).max() <= 1e-12 * scale
    assert res.stats.l_aux == pytest.approx(b["l_aux"], rel=1e-12)
    if case["cf"] > 0:
        assert res.stats.dropped == int((b["counts"] - b["kept"]).sum())
    assert res.stats.z_loss == pytest.approx(b["z_loss"], rel=1e-12)
    assert res.stats.entropy == pytest.approx(b["entropy"], rel=1e-12)
    assert res.stats.top_gap == pytest.approx(b["top_gap"], rel=1e-12)


def test_fully_dropped_token_gets_zero_row():
    rng = np.random.default_rng(8)
    T, d, E, d_ff = 32, 8, 4, 8
    x, W_r, W1, W3, W2, _ = _rand_layer(rng, T, d, E, d_ff)
    W_r[:] = 0.0
    W_r[:, 0] = 1.0
    W_r[:, 1] = 0.5
    x = np.abs(x) + 0.1   # every token prefers experts 0 then 1
    res = O.moe_forward(x, W_r, W1, W3, W2, k=2, capacity_factor=0.25)
    C = res.stats.capacity
    assert C == 4
    dropped_both = [t for t in range(T) if (res.perm.pos[t] < 0).all()]
    assert dropped_both == list(range(C, T))
    assert np.abs(res.y[dropped_both]).max() == 0.0


def test_token_subset_matches_full():
    rng = np.random.default_rng(9)
    x, W_r, W1, W3, W2, sh = _rand_layer(rng, 30, 8, 4, 8, shared=True)
    full = O.moe_forward(x, W_r, W1, W3, W2, k=2, capacity_factor=0.6, **sh)
    sub = O.moe_forward(x, W_r, W1, W3, W2, k=2, capacity_factor=0.6, tokens=[29, 0, 7], **sh)
    # BLAS may block different row counts differently: equal up to rounding
    assert np.allclose(sub.y, full.y[[29, 0, 7]], rtol=1e-13, atol=1e-15)


def test_unpermute_combine_reproduces_layer_output():
    # expert outputs computed in permuted row order and mixed back give the
    # per-pair layer output ([CMU 15-779 L21] §3.2 four steps)
    rng = np.random.default_rng(13)
    x, W_r, W1, W3, W2, sh = _rand_layer(rng, 40, 8, 6, 8, shared=True)
    res = O.moe_forward(x, W_r, W1, W3, W2, k=3, capacity_factor=0.7, **sh)
    perm = res.perm
    R = perm.indptr[-1]
    O_rows = np.zeros((R, 8))
    for e in range(6):
        lo, hi = perm.indptr[e], perm.indptr[e + 1]
        if hi > lo:
            O_rows[lo:hi] = O.swiglu_expert(x[perm.row_token[lo:hi]], W1[e], W3[e], W2[e])
    S = O.swiglu_expert(x, sh["Ws1"], sh["Ws3"], sh["Ws2"])
    y = O.unpermute_combine(O_rows, perm.pos, res.routing.gate, S)
    assert np.allclose(y, res.y, rtol=1e-12, atol=1e-13)
    assert res.stats.dropped > 0


# --- routing variants ([CMU 15-779 L21] §2.5 and §3.5; [CME295 W2D2] §3.4; [W11 routing] §5) ---

def test_z_loss_and_max_probability_match_printed_values():
    # 8 experts, logits N(0, std^2): the page's z-loss 6.2 / 59.6 / 988.9 and mean
    # largest probability 0.355 -> 0.949 come from a finite sample; the expected
    # values over a large sample sit within 6 % of them
    g = load("z_loss_table.txt")
    rng = np.random.default_rng(7)
    for std, want in zip(g["std"], g["z_loss"]):
        z = rng.standard_normal((50000, g["E"])) * std
        assert O.router_z_loss(z) == pytest.approx(want, rel=0.06)
    z = rng.standard_normal((50000, g["E"]))
    assert O.softmax_rows(z).max(axis=1).mean() == pytest.approx(g["max_prob_std1"], rel=0.03)
    z = rng.standard_normal((50000, g["E"])) * 20
    assert O.softmax_rows(z).max(axis=1).mean() == pytest.approx(g["max_prob_std20"], rel=0.03)


def test_router_statistics_closed_forms():
    for E in (2, 8, 64):
        z = np.zeros((5, E))
        assert O.router_z_loss(z) == pytest.approx(math.log(E) ** 2, rel=1e-14)
        p = O.softmax_rows(z)
        assert O.router_entropy(p) == pytest.approx(math.log(E), rel=1e-14)
        assert O.router_top_gap(p) == 0.0
        # a shift c of every logit moves log-sum-exp by c
        assert O.router_z_loss(z + 3.0) == pytest.approx((math.log(E) + 3.0) ** 2, rel=1e-14)
        zd = np.zeros((3, E))
        zd[:, 0] = 80.0                       # one dominant expert
        pd = O.softmax_rows(zd)
        assert O.router_entropy(pd) < 1e-30 + 1e-20 * E
        assert O.router_top_gap(pd) == pytest.approx(1.0, abs=1e-30)


def test_full_softmax_gates_are_switch_top1():
    # k = 1 with gates renormalised over the selected set is always 1 (the
    # router gets no gradient); the Switch gate is the full-softmax probability
    rng = np.random.default_rng(14)
    z = rng.standard_normal((20, 8)) * 2
    idx = O.topk_lowest_index(z, 1)
    assert np.array_equal(O.gates_from_selected(z, idx), np.ones((20, 1)))
    full = O.gates_full_softmax(z, idx)
    assert np.allclose(full[:, 0], O.softmax_rows(z).max(axis=1), rtol=1e-15)
    assert (full < 1).all()
    # top-2 full gates sum to the two largest probabilities
    idx2 = O.topk_lowest_index(z, 2)
    srt = -np.sort(-O.softmax_rows(z), axis=1)
    assert np.allclose(O.gates_full_softmax(z, idx2).sum(axis=1), srt[:, 0] + srt[:, 1], rtol=1e-14)


def test_slot_priority_drop_order_worked_example():
    # GShard's Algorithm 1: all first choices are placed before any second
    # choice. Three tokens, two experts, top-2, capacity 2:
    # x0 -> (0, 1), x1 -> (1, 0), x2 -> (0, 1)
    idx = np.array([[0, 1], [1, 0], [0, 1]])
    tok = O.permute(idx, 2, 2, O.DROP_TOKEN)
    slot = O.permute(idx, 2, 2, O.DROP_SLOT)
    # token order keeps x0 and x1 in both experts; x2 loses both pairs
    assert tok.pos.tolist() == [[0, 2], [3, 1], [-1, -1]]
    # slot priority: expert 0 keeps x0 (1st) and x2 (1st) and drops x1's 2nd
    # choice; expert 1 keeps x1 (1st) and x0 (2nd) and drops x2's 2nd choice
    assert slot.pos.tolist() == [[0, 3], [2, -1], [1, -1]]
    assert slot.counts.tolist() == [3, 3] and slot.kept.tolist() == [2, 2]


def test_drop_orders_agree_without_capacity_and_for_top1():
    rng = np.random.default_rng(15)
    z = rng.standard_normal((200, 8))
    idx = O.topk_lowest_index(z, 3)
    a = O.permute(idx, 8, None, O.DROP_TOKEN)
    b = O.permute(idx, 8, None, O.DROP_SLOT)
    assert np.array_equal(a.indptr, b.indptr)
    for e in range(8):   # same pairs per expert, possibly in another order
        sa = {tuple(x) for x in np.argwhere(idx == e).tolist()}
        rows_b = set(range(b.indptr[e], b.indptr[e + 1]))
        assert {tuple(x) for x in np.argwhere((idx == e) & np.isin(b.pos, list(rows_b))).tolist()} == sa
    idx1 = O.topk_lowest_index(z, 1)
    assert np.array_equal(O.permute(idx1, 8, 20, O.DROP_TOKEN).pos, O.permute(idx1, 8, 20, O.DROP_SLOT).pos)


def test_megablocks_figure5_topology():
    g = load("megablocks_figure5.txt")
    off, col, row, tr = O.block_sparse_topology(g["rows"], g["block"], g["blocks_per_expert"])
    assert off.tolist() == g["offsets"].tolist()
    assert col.tolist() == g["col"].tolist()
    assert row.tolist() == g["row"].tolist()
    assert tr.tolist() == g["transpose"].tolist()


def test_padded_permutation_follows_figure5_rows():
    # one pick per token so that the experts get the figure's 3 / 1 / 6 rows;
    # padded to blocks of 2 they hold 4 / 2 / 6 rows, the figure's 6 block rows
    g = load("megablocks_figure5.txt")
    idx = np.array([[0], [2], [0], [2], [1], [2], [0], [2], [2], [2]])
    perm = O.permute(idx, 3, None, O.DROP_TOKEN, pad=g["block"])
    assert perm.kept.tolist() == g["rows"].tolist()
    assert perm.indptr.tolist() == [0, 4, 6, 12]
    assert (perm.indptr[1:] - perm.indptr[:-1]).sum() // g["block"] == len(g["offsets"]) - 1
    assert perm.pos[:, 0].tolist() == [0, 6, 1, 7, 4, 8, 2, 9, 10, 11]
    assert perm.row_token.tolist() == [0, 2, 6, -1, 4, -1, 1, 3, 5, 7, 8, 9]
    # without padding the same pairs are numbered densely
    assert O.permute(idx, 3).indptr.tolist() == [0, 3, 4, 10]


def test_padding_does_not_change_the_layer_output():
    rng = np.random.default_rng(16)
    x, W_r, W1, W3, W2, _ = _rand_layer(rng, 40, 16, 8, 8)
    a = O.moe_forward(x, W_r, W1, W3, W2, k=2, capacity_factor=1.0)
    b = O.moe_forward(x, W_r, W1, W3, W2, k=2, capacity_factor=1.0, pad=4)
    assert np.array_equal(a.y, b.y)
    assert np.array_equal(a.perm.kept, b.perm.kept)
    assert (b.perm.indptr % 4 == 0).all() and b.perm.indptr[-1] >= a.perm.indptr[-1]


# --- closed forms ([CME295 W2D2] §2.3; [CMU 15-779 L21] §3.1 and exercise 4; §2.1 counts) ---

def test_experts_touched_table():
    g = load("experts_touched_table.txt")
    got = [round(100 * O.fraction_experts_touched(g["E"], g["k"], B), 1) for B in g["B"]]
    assert got == g["percent"].tolist()


def test_experts_touched_by_routing_simulation():
    # route random tokens through the oracle's top-k; the mean touched fraction
    # at B = 8 must sit within 4 sigma of the closed form
    rng = np.random.default_rng(10)
    E, k, B, trials = 8, 2, 8, 4000
    fr = np.empty(trials)
    for i in range(trials):
        idx = O.topk_lowest_index(rng.standard_normal((B, E)), k)
        fr[i] = len(set(idx.reshape(-1).tolist())) / E
    expect = O.fraction_experts_touched(E, k, B)
    assert abs(fr.mean() - expect) < 4 * fr.std() / math.sqrt(trials)


def test_exercise4_decode_touched():
    g = load("exercise4_decode_touched.txt")
    assert round(O.expected_experts_touched(g["E"], g["k"], g["B"])) == g["touched"]


def test_mixtral_param_counts():
    g = load("mixtral_param_counts.txt")
    total, active = O.param_counts(O.MIXTRAL_8X7B)
    assert total == g["total"]
    assert active == g["active"]
    s = O.MIXTRAL_8X7B
    assert round(3 * s.d * s.d_ff / 1e6, 1) == g["expert_M"]
    assert s.d * s.E == g["router"]
    attn = 2 * s.d * s.n_heads * s.head_dim + 2 * s.d * s.n_kv_heads * s.head_dim
    assert round(attn / 1e6, 1) == g["attention_per_layer_M"]


# --- planted mistakes: each must be caught by a pin above ---

def test_planted_capacity_without_k_is_caught(monkeypatch):
    g = load("exercise3_capacity.txt")
    monkeypatch.setattr(O, "capacity", lambda cf, T, k, E: int(math.ceil(cf * T / E)))
    assert O.capacity(g["cf"], g["N"], g["k"], g["E"]) != g["C"]


def test_planted_token_major_numbering_is_caught():
    g = load("prefix_sum_worked_example.txt")
    idx, E = g["idx"], g["E"]
    T = idx.shape[0]
    mask = np.zeros((T, E), dtype=np.int64)
    for t in range(T):
        mask[t, idx[t]] = 1
    cs = np.cumsum(mask.reshape(-1)).reshape(T, E)     # token-major: wrong order
    pos = np.array([[cs[t, e] - 1 for e in idx[t]] for t in range(T)])
    assert pos.tolist() != g["pos"].tolist()


def test_planted_unnormalised_gates_are_caught(monkeypatch):
    rng = np.random.default_rng(11)
    x, W_r, W1, W3, W2, _ = _rand_layer(rng, 20, 8, 6, 8)
    b = brute_forward(x, W_r, W1, W3, W2, k=2)

    def wrong(z, idx):
        return np.take_along_axis(O.softmax_rows(z), idx, axis=1)
    monkeypatch.setattr(O, "gates_from_selected", wrong)
    res = O.moe_forward(x, W_r, W1, W3, W2, k=2)
    assert not np.allclose(res.y, b["y"], rtol=1e-6)


def test_planted_upward_tie_break_is_caught(monkeypatch):
    def wrong(key, k):
        key = np.asarray(key)
        order = np.argsort(-key[:, ::-1], axis=1, kind="stable")
        return (key.shape[1] - 1 - order)[:, :k]
    monkeypatch.setattr(O, "topk_lowest_index", wrong)
    assert O.topk_lowest_index(np.zeros((1, 8)), 2).tolist() != [[0, 1]]


def test_planted_missing_shared_expert_is_caught():
    rng = np.random.default_rng(12)
    x, W_r, W1, W3, W2, sh = _rand_layer(rng, 10, 8, 4, 8, shared=True)
    b = brute_forward(x, W_r, W1, W3, W2, k=2, **sh)
    res = O.moe_forward(x, W_r, W1, W3, W2, k=2)   # shared expert left out
    assert not np.allclose(res.y, b["y"], rtol=1e-6)


def test_planted_slot_order_ignored_is_caught(monkeypatch):
    idx = np.array([[0, 1], [1, 0], [0, 1]])
    orig = O.permute
    monkeypatch.setattr(O, "permute", lambda idx_, E, C, drop_order=O.DROP_TOKEN: orig(idx_, E, C, O.DROP_TOKEN))
    assert O.permute(idx, 2, 2, O.DROP_SLOT).pos.tolist() != [[0, 3], [2, -1], [1, -1]]


def test_planted_unsquared_z_loss_is_caught(monkeypatch):
    def wrong(z):
        z = np.asarray(z, dtype=np.float64)
        m = z.max(axis=1, keepdims=True)
        return float(np.mean(m[:, 0] + np.log(np.exp(z - m).sum(axis=1))))
    monkeypatch.setattr(O, "router_z_loss", wrong)
    assert O.router_z_loss(np.zeros((5, 8))) != pytest.approx(math.log(8) ** 2, rel=1e-14)
