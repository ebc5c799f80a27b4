"""Pins for the CPU oracle: each test checks it against something other than
itself — a worked example printed by the pages, brute force on tiny inputs, a
textbook special case, or an invariant the method fixes."""
import itertools
import json
import math
import os

import numpy as np
import pytest

import oracle as O

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _rng(seed):
    return np.random.default_rng(seed)


def _tiny_layer(seed, n=16, d=8, H=6):
    r = _rng(seed)
    return dict(
        W1=r.standard_normal((n, d)), b1=r.standard_normal(n) - 0.5,
        W2T=r.standard_normal((n, d)), b2=r.standard_normal(d),
        Wp1=r.standard_normal((H, d)), bp1=r.standard_normal(H) * 0.1,
        Wp2=r.standard_normal((n, H)), bp2=r.standard_normal(n) - 0.3)


# ---------------------------------------------------------------------------
# brute-force loop nests on tiny shapes
def _loops_dense(W1, b1, W2T, b2, x):
    n, d = len(W1), len(W1[0])
    y = [float(b2[c]) for c in range(d)]
    for j in range(n):
        z = float(b1[j])
        for c in range(d):
            z += float(W1[j][c]) * float(x[c])
        a = z if z > 0 else 0.0
        for c in range(d):
            y[c] += a * float(W2T[j][c])
    return y


def test_dense_ffn_matches_loop_nest():
    L = _tiny_layer(1)
    X = _rng(2).standard_normal((3, 8))
    got = O.dense_ffn(L["W1"], L["b1"], L["W2T"], L["b2"], X)
    for t in range(3):
        want = _loops_dense(L["W1"].tolist(), L["b1"], L["W2T"].tolist(), L["b2"], X[t])
        np.testing.assert_allclose(got[t], want, rtol=1e-13, atol=1e-13)


def test_predictor_matches_loop_nest_and_sigmoid():
    L = _tiny_layer(3)
    x = _rng(4).standard_normal(8)
    h = O.predictor_hidden(L["Wp1"], x, L["bp1"])[0]
    l = O.predictor_logits(L["Wp2"], h, L["bp2"])[0]
    for k in range(6):
        s = float(L["bp1"][k]) + sum(float(L["Wp1"][k][c]) * float(x[c]) for c in range(8))
        assert h[k] == pytest.approx(max(s, 0.0), abs=1e-13)
    sel = []
    for i in range(16):
        s = float(L["bp2"][i]) + sum(float(L["Wp2"][i][k]) * float(h[k]) for k in range(6))
        assert l[i] == pytest.approx(s, abs=1e-12)
        if 1.0 / (1.0 + math.exp(-s)) > 0.5:      # the sigmoid decision itself
            sel.append(i)
    idx, k = O.neuron_table(O.predicted_mask(l))
    assert idx.tolist() == sel and k == len(sel)


def test_threshold_is_strict_at_zero():
    assert O.predicted_mask([0.0, -0.0, 1e-300, -1e-300]).tolist() == [False, False, True, False]


def test_union_mask_is_or_of_per_token_masks():
    L = _tiny_layer(5)
    X = _rng(6).standard_normal((5, 8))
    idx, k, logits = O.predict(L["Wp1"], L["Wp2"], L["bp2"], X, L["bp1"])
    union = set()
    for t in range(5):
        it, _, _ = O.predict(L["Wp1"], L["Wp2"], L["bp2"], X[t], L["bp1"])
        union |= set(it.tolist())
    assert idx.tolist() == sorted(union) and k == len(union)
    assert np.all(np.diff(idx) > 0)


# ---------------------------------------------------------------------------
# invariants of the sparse FFN
def test_full_mask_reproduces_dense():
    L = _tiny_layer(7, n=64, d=32)
    X = _rng(8).standard_normal((4, 32))
    ys = O.sparse_ffn(L["W1"], L["b1"], L["W2T"], L["b2"], X, np.arange(64))
    yd = O.dense_ffn(L["W1"], L["b1"], L["W2T"], L["b2"], X)
    np.testing.assert_allclose(ys, yd, rtol=1e-12, atol=1e-12)


def test_superset_of_positive_set_reproduces_dense_bitwise():
    L = _tiny_layer(9, n=64, d=32)
    x = _rng(10).standard_normal(32)
    z = O.fc1_preactivation(L["W1"], L["b1"], x)[0]
    pos = np.nonzero(z > 0)[0]
    y_pos = O.sparse_ffn(L["W1"], L["b1"], L["W2T"], L["b2"], x, pos)
    r = _rng(11)
    for _ in range(20):
        extra = np.nonzero(r.random(64) < 0.5)[0]
        sup = np.union1d(pos, extra)
        y_sup = O.sparse_ffn(L["W1"], L["b1"], L["W2T"], L["b2"], x, sup)
        assert np.array_equal(y_sup, y_pos)          # skipped terms are exact zeros
    yd = O.dense_ffn(L["W1"], L["b1"], L["W2T"], L["b2"], x)
    np.testing.assert_allclose(y_pos, yd, rtol=1e-12, atol=1e-12)


def test_skipped_neurons_contribute_exactly_zero():
    L = _tiny_layer(12, n=32, d=16)
    X = _rng(13).standard_normal((2, 16))
    idx = np.array([1, 4, 5, 17, 30])
    y0 = O.sparse_ffn(L["W1"], L["b1"], L["W2T"], L["b2"], X, idx)
    W1, W2T, b1 = L["W1"].copy(), L["W2T"].copy(), L["b1"].copy()
    off = np.setdiff1d(np.arange(32), idx)
    W1[off] += 1e3
    W2T[off] *= -7.0
    b1[off] += 50.0
    y1 = O.sparse_ffn(W1, b1, W2T, L["b2"], X, idx)
    assert np.array_equal(y0, y1)


def test_empty_table_gives_b2():
    L = _tiny_layer(14)
    x = _rng(15).standard_normal(8)
    y = O.sparse_ffn(L["W1"], L["b1"], L["W2T"], L["b2"], x, np.array([], dtype=np.int64))
    assert np.array_equal(y[0], L["b2"])


@pytest.mark.slow
def test_all_masks_n16_brute_force():
    """Every one of the 2^16 neuron subsets at n=16: the result depends only on
    the subset's positive neurons, and equals the dense FFN exactly when the
    subset contains every positive neuron."""
    n, d = 16, 4
    L = _tiny_layer(16, n=n, d=d)
    x = _rng(17).standard_normal(d)
    z = O.fc1_preactivation(L["W1"], L["b1"], x)[0]
    pos = frozenset(np.nonzero(z > 0)[0].tolist())
    assert 0 < len(pos) < n
    yd = O.dense_ffn(L["W1"], L["b1"], L["W2T"], L["b2"], x)[0]
    by_pos = {}
    for bits in range(1 << n):
        idx = [j for j in range(n) if bits >> j & 1]
        y = O.sparse_ffn(L["W1"], L["b1"], L["W2T"], L["b2"], x, np.array(idx, dtype=np.int64))[0]
        key = frozenset(idx) & pos
        if key in by_pos:
            assert np.array_equal(by_pos[key], y)
        else:
            by_pos[key] = y
        covers = pos <= set(idx)
        assert np.allclose(y, yd, rtol=1e-12, atol=1e-12) == covers
    assert len(by_pos) == 1 << len(pos)


# ---------------------------------------------------------------------------
# the pages' worked example
def test_worked_example_fig3():
    g = json.load(open(os.path.join(GOLDEN, "fig3_worked_example.json")))
    e = g["expected"]
    h = O.predictor_hidden(g["Wp1"], g["x"], g["bp1"])[0]
    assert h.tolist() == e["hidden"]
    l = O.predictor_logits(g["Wp2"], h, g["bp2"])[0]
    assert l.tolist() == e["logits"]
    idx, k, _ = O.predict(g["Wp1"], g["Wp2"], g["bp2"], g["x"], g["bp1"])
    assert idx.tolist() == g["printed_by_the_pages"]["predicted_active"] == e["idx"] and k == 3
    z = O.fc1_preactivation(g["W1"], g["b1"], g["x"])[0]
    assert z.tolist() == e["preactivation"]
    for j in g["printed_by_the_pages"]["hot_but_not_predicted"]:
        assert z[j] > 0 and j not in idx.tolist()
    y = O.sparse_ffn(g["W1"], g["b1"], g["W2T"], g["b2"], g["x"], idx)[0]
    assert y.tolist() == e["y_sparse"]
    yd = O.dense_ffn(g["W1"], g["b1"], g["W2T"], g["b2"], g["x"])[0]
    assert yd.tolist() == e["y_dense"]
    counts = O.activation_counts(g["W1"], g["b1"], g["profile_tokens"])
    assert counts.tolist() == e["profile_counts"]
    perm = O.hot_first_order(counts)
    assert perm.tolist() == e["hot_first_perm"]
    assert sorted(perm[:3].tolist()) == g["printed_by_the_pages"]["hot_neurons"]


# ---------------------------------------------------------------------------
# profiling and placement
def test_activation_counts_loop_nest():
    L = _tiny_layer(18, n=12, d=5)
    X = _rng(19).standard_normal((30, 5))
    got = O.activation_counts(L["W1"], L["b1"], X)
    for j in range(12):
        c = 0
        for t in range(30):
            s = float(L["b1"][j]) + sum(float(L["W1"][j][q]) * float(X[t][q]) for q in range(5))
            c += s > 0
        assert got[j] == c


def test_hot_first_order_sort_and_ties():
    c = np.array([3, 7, 7, 0, 3, 9, 0, 7], dtype=np.uint32)
    perm = O.hot_first_order(c)
    assert perm.tolist() == sorted(range(8), key=lambda i: (-int(c[i]), i))
    assert perm.tolist() == [5, 1, 2, 7, 0, 4, 3, 6]


def test_reorder_is_permutation_invariant():
    n, d, H = 48, 16, 8
    L = _tiny_layer(20, n=n, d=d, H=H)
    X = _rng(21).standard_normal((3, d))
    prof = _rng(22).standard_normal((64, d))
    counts = O.activation_counts(L["W1"], L["b1"], prof)
    perm = O.hot_first_order(counts)
    assert sorted(perm.tolist()) == list(range(n))
    P = {k: (O.permute_rows(v, perm) if k in ("W1", "b1", "W2T", "Wp2", "bp2") else v) for k, v in L.items()}
    assert np.all(np.diff(O.permute_rows(counts, perm).astype(np.int64)) <= 0)
    idx0, k0, _, y0 = O.step(L, X)
    idx1, k1, _, y1 = O.step(P, X)
    assert k0 == k1 and sorted(perm[idx1].tolist()) == idx0.tolist()
    np.testing.assert_allclose(y1, y0, rtol=1e-12, atol=1e-12)


# ---------------------------------------------------------------------------
# chaining reading
def test_chain_closed_forms():
    u = np.full((1, 64), 0.75)
    out = O.chain(u, np.zeros((1, 64)))
    assert np.allclose(out, 0.75 / math.sqrt(0.75 ** 2 + O.RMS_EPS), rtol=1e-15)
    r = _rng(23)
    x, y = r.standard_normal((3, 128)), r.standard_normal((3, 128))
    out = O.chain(x, y)
    ms = np.mean((x + y) ** 2, axis=1)
    np.testing.assert_allclose(np.sqrt(np.mean(out ** 2, axis=1)), np.sqrt(ms / (ms + O.RMS_EPS)), rtol=1e-13)
    np.testing.assert_allclose(out * np.sqrt(ms + O.RMS_EPS)[:, None], x + y, rtol=1e-13)


def test_dealt_order_hand_example():
    # counts: neuron 4 hottest, then 1, 6, 0, 3, 2, 5 (ties by index)
    counts = np.array([5, 8, 1, 4, 9, 1, 7], dtype=np.uint32)
    assert O.hot_first_order(counts).tolist() == [4, 1, 6, 0, 3, 2, 5]
    # 3 ranges over 7 slots: [0,2) [2,4) [4,7); deal 4->r0, 1->r1, 6->r2, 0->r0, 3->r1, 2->r2, 5->r2
    assert O.dealt_order(counts, 3).tolist() == [4, 0, 1, 3, 6, 2, 5]
    assert O.dealt_order(counts, 1).tolist() == O.hot_first_order(counts).tolist()


# ---------------------------------------------------------------------------
# look-ahead prediction
def _hand_lookahead_layer():
    # identity predictor (h = ReLU(x), logit_i = h_i): neuron i is predicted iff x_i > 0;
    # FC1 = identity (a_j = ReLU(x_j)); FC2 rows e1*3 and e0*5: y = [5 a_1, 3 a_0]
    return dict(W1=np.eye(2), b1=np.zeros(2), W2T=np.array([[0.0, 3.0], [5.0, 0.0]]), b2=np.zeros(2),
                Wp1=np.eye(2), bp1=np.zeros(2), Wp2=np.eye(2), bp2=np.zeros(2))


def test_lookahead_hand_example():
    L = _hand_lookahead_layer()
    x0 = np.array([1.0, -1.0])
    # layer 0: both readings predict from x0 -> {0}; y0 = [0, 3]
    idx0, k0, _, y0 = O.step_lookahead(L, x0, x0)
    assert idx0.tolist() == [0] and k0 == 1
    np.testing.assert_array_equal(y0[0], [0.0, 3.0])
    x1 = O.chain(x0, y0)[0]
    s = math.sqrt(2.5 + O.RMS_EPS)
    np.testing.assert_allclose(x1, [1.0 / s, 2.0 / s], rtol=1e-15)
    # layer 1 on x1: its own input fires both neurons, the previous input only neuron 0
    idx_s, k_s, _, y_s = O.step(L, x1)
    idx_l, k_l, _, y_l = O.step_lookahead(L, x0, x1)
    assert idx_s.tolist() == [0, 1] and idx_l.tolist() == [0]
    np.testing.assert_allclose(y_s[0], [10.0 / s, 3.0 / s], rtol=1e-15)
    np.testing.assert_allclose(y_l[0], [0.0, 3.0 / s], rtol=1e-15)


def test_lookahead_set_depends_only_on_predictor_input():
    L = _tiny_layer(31)
    r = _rng(32)
    xp, x, x2 = r.standard_normal(8), r.standard_normal(8), r.standard_normal(8)
    idx_a, _, log_a, y_a = O.step_lookahead(L, xp, x)
    idx_b, _, log_b, y_b = O.step_lookahead(L, xp, x2)
    assert idx_a.tolist() == idx_b.tolist()
    np.testing.assert_array_equal(log_a, log_b)
    # the FFN part is the sparse FFN of the FFN input over that set
    np.testing.assert_array_equal(y_b, O.sparse_ffn(L["W1"], L["b1"], L["W2T"], L["b2"], x2, idx_a))
    # same input on both sides: the plain step, bit for bit
    i0, k0, l0, y0 = O.step(L, x)
    i1, k1, l1, y1 = O.step_lookahead(L, x, x)
    assert i0.tolist() == i1.tolist() and k0 == k1
    np.testing.assert_array_equal(l0, l1)
    np.testing.assert_array_equal(y0, y1)
