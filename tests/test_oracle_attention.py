"""Pins of the attention-head predictor / head-sparse attention oracle against
things other than itself: explicit loop nests, closed forms of the softmax
average, the textbook matrix form of multi-head attention, and the invariants
the DejaVu appendix fixes (a skipped head contributes nothing; K/V filled late
from the stored token inputs equal those computed when the token arrived)."""
import math

import numpy as np

import oracle.attention as A
import workload as wl

ident = lambda a: np.asarray(a, dtype=np.float64)
fp16 = lambda a: wl.widen(wl.round_to(np.asarray(a, dtype=np.float64), 0), 0)


def rnd(shape, seed, scale=1.0):
    return np.random.default_rng(seed).standard_normal(shape) * scale


def weights(nh, dh, d, seed, bias=True):
    r = lambda s, k: rnd(s, seed * 10 + k, 1.0 / math.sqrt(s[-1]))
    Wt = dict(Wq=r((nh * dh, d), 1), Wk=r((nh * dh, d), 2), Wv=r((nh * dh, d), 3), Wo=r((d, nh * dh), 4))
    for k, name in enumerate(("bq", "bk", "bv")):
        Wt[name] = rnd(nh * dh, seed * 10 + 5 + k, 0.1) if bias else None
    Wt["bo"] = rnd(d, seed * 10 + 8, 0.1) if bias else None
    return Wt


def test_attend_matches_loop_nest():
    for T, dh, seed in ((1, 4, 0), (5, 8, 1), (9, 3, 2)):
        q, K, V = rnd(dh, seed), rnd((T, dh), seed + 10), rnd((T, dh), seed + 20)
        s = [sum(q[i] * K[p][i] for i in range(dh)) / math.sqrt(dh) for p in range(T)]
        e = [math.exp(v) for v in s]
        z = sum(e)
        want = [sum(e[p] / z * V[p][i] for p in range(T)) for i in range(dh)]
        assert np.allclose(A.attend(q, K, V), want, rtol=0, atol=1e-12)


def test_attend_closed_forms():
    dh = 6
    V = rnd((7, dh), 3)
    # a single position returns its value row exactly
    assert np.array_equal(A.attend(rnd(dh, 1), rnd((1, dh), 2), V[:1]), V[0])
    # equal keys: every weight is 1/T, the output is the mean of the values
    K = np.tile(rnd(dh, 4), (7, 1))
    assert np.allclose(A.attend(rnd(dh, 5), K, V), V.mean(axis=0), rtol=0, atol=1e-14)
    # one score far above the rest: the output is that position's value
    K = np.zeros((7, dh)); K[3, 0] = 1.0
    q = np.zeros(dh); q[0] = 800.0
    assert np.allclose(A.attend(q, K, V), V[3], rtol=0, atol=1e-12)


def test_head_logits_loop_nest_and_sigmoid_threshold():
    d, Ha, nh = 12, 7, 9
    Wa1, Wa2, ba1, ba2, y = rnd((Ha, d), 1), rnd((nh, Ha), 2), rnd(Ha, 3), rnd(nh, 4), rnd(d, 5)
    h = [max(0.0, sum(Wa1[j][i] * y[i] for i in range(d)) + ba1[j]) for j in range(Ha)]
    want = [sum(Wa2[k][j] * h[j] for j in range(Ha)) + ba2[k] for k in range(nh)]
    got = A.head_logits(Wa1, Wa2, y, ba1, ba2)[0]
    assert np.allclose(got, want, rtol=0, atol=1e-12)
    sig = [1.0 / (1.0 + math.exp(-v)) for v in want]
    assert A.selected_heads(got).tolist() == [k for k in range(nh) if sig[k] > 0.5]
    # a batch selects the union of its tokens' heads; an exact zero logit is not selected
    L = np.array([[0.0, 1.0, -1.0], [-2.0, -1.0, 0.5]])
    assert A.selected_heads(L).tolist() == [1, 2]


def test_sparse_with_all_heads_equals_dense_matrix_form():
    nh, dh, d, T = 4, 8, 20, 6
    Wt = weights(nh, dh, d, 7)
    Y = rnd((T, d), 8)
    cache = A.KVCache(nh, dh, d, T, ident)
    for t in range(T):
        got = A.mha_sparse_step(Wt, cache, Y[t], np.arange(nh))
        want = A.mha_dense(Wt, Y[:t + 1], nh, dh, ident)
        assert np.allclose(got, want, rtol=0, atol=1e-12), t


def test_late_filled_kv_equals_kv_at_arrival():
    """Heads picked at random each step: the output equals dense attention
    restricted to the picked heads (whose K/V the dense form computes for every
    position), and every cache row present equals its direct computation."""
    nh, dh, d, T = 6, 4, 16, 9
    Wt = weights(nh, dh, d, 11)
    Y = rnd((T, d), 12)
    r = np.random.default_rng(13)
    for round_kv in (ident, fp16):
        cache = A.KVCache(nh, dh, d, T, round_kv)
        for t in range(T):
            heads = np.sort(r.choice(nh, int(r.integers(0, nh + 1)), replace=False))
            got = A.mha_sparse_step(Wt, cache, Y[t], heads)
            want = A.mha_dense(Wt, Y[:t + 1], nh, dh, round_kv, heads=heads)
            assert np.allclose(got, want, rtol=0, atol=1e-12), (t, heads)
            for h in heads:
                assert cache.filled[h, :t + 1].all()
        for h in range(nh):
            for p in range(T):
                if cache.filled[h, p]:
                    assert np.array_equal(cache.K[h, p], round_kv(A.head_rows(Wt["Wk"], Wt["bk"], h, dh, Y[p])))
                    assert np.array_equal(cache.V[h, p], round_kv(A.head_rows(Wt["Wv"], Wt["bv"], h, dh, Y[p])))


def test_skipped_heads_contribute_exactly_nothing():
    nh, dh, d, T = 5, 4, 12, 5
    Wt = weights(nh, dh, d, 21)
    Y = rnd((T, d), 22)
    keep = np.array([0, 3])
    outs = []
    for perturb in (False, True):
        W = {k: (None if v is None else v.copy()) for k, v in Wt.items()}
        if perturb:
            for h in (1, 2, 4):
                rows = slice(h * dh, (h + 1) * dh)
                for name in ("Wq", "Wk", "Wv"):
                    W[name][rows] += 3.0
                W["Wo"][:, rows] -= 2.0
        cache = A.KVCache(nh, dh, d, T, ident)
        outs.append([A.mha_sparse_step(W, cache, Y[t], keep) for t in range(T)])
    assert all(np.array_equal(a, b) for a, b in zip(*outs))
    # no head selected: the output is the bias alone
    cache = A.KVCache(nh, dh, d, 1, ident)
    assert np.array_equal(A.mha_sparse_step(Wt, cache, Y[0], []), Wt["bo"])
