"""CPU oracle for the attention-head predictor and head-sparse attention decode
(DejaVu's SP_A) — TEST INFRASTRUCTURE ONLY, like the rest of ``oracle``.

Plain numpy in fp64, written to be checked by eye against the DejaVu appendix of
"LLM模型之PowerInfer1.0" (blog-zz7.pages.dev):

* equation (-1): the layer's attention input y selects the heads,
  ``S_A <- SP_A(y)``, and the attention block runs only on those heads,
  ``y~ <- MHA_{S_A}(y)``;
* SP_A is a two-layer MLP whose output layer has one unit per head, each
  followed by a sigmoid that makes a binary "select / do not select" decision;
* KV-cache misses: the layer keeps a copy of every past token's input; when a
  head that was skipped earlier is selected, its missing K/V entries are
  computed from those stored inputs before it attends.

Readings where the pages leave a step open (all pinned by tests):

* SP_A's hidden activation is ReLU (as for the FFN predictor) and the sigmoid
  > 0.5 decision is the equivalent strict ``logit > 0``;
* MHA is standard scaled dot-product attention of one new token over the
  layer's cache: per head h with width dh, ``q = Wq_h y + bq_h``, ``k_p = Wk_h
  y_p + bk_h``, ``v_p = Wv_h y_p + bv_h`` for positions p = 0..t (the new token
  included), ``o_h = softmax_p(q . k_p / sqrt(dh)) v``, and the output
  ``y~ = bo + sum_{h in S_A} Wo[:, h] o_h`` (Wo's dh columns of head h); a
  head outside S_A contributes nothing;
* the cache stores K and V rounded to the storage dtype (like the weights and
  the layer inputs); q, the scores, the softmax and o stay in full precision;
* no positional encoding on this path (OPT adds learned positions to the
  embeddings before the first layer).
"""
from __future__ import annotations

import numpy as np


def _f64(a) -> np.ndarray:
    return np.asarray(a, dtype=np.float64)


def head_logits(Wa1, Wa2, y, ba1=None, ba2=None) -> np.ndarray:
    """SP_A: ``l = Wa2 ReLU(Wa1 y + ba1) + ba2``, one logit per head ([B, nh])."""
    Y = np.atleast_2d(_f64(y))
    h = Y @ _f64(Wa1).T
    if ba1 is not None:
        h = h + _f64(ba1)[None, :]
    h = np.maximum(h, 0.0)
    out = h @ _f64(Wa2).T
    if ba2 is not None:
        out = out + _f64(ba2)[None, :]
    return out


def selected_heads(logits) -> np.ndarray:
    """Heads whose sigmoid output exceeds 0.5 for any token (logit > 0), ascending."""
    L = np.atleast_2d(_f64(logits))
    return np.nonzero(np.any(L > 0.0, axis=0))[0].astype(np.int32)


def head_rows(W, b, h: int, dh: int, y) -> np.ndarray:
    """The head's dh outputs of a projection: ``W[h dh:(h+1) dh] y + b[...]``."""
    rows = slice(h * dh, (h + 1) * dh)
    out = _f64(W)[rows] @ _f64(y)
    if b is not None:
        out = out + _f64(b)[rows]
    return out


def attend(q, K, V) -> np.ndarray:
    """One head: ``softmax_p(q . K[p] / sqrt(dh)) V`` with the max subtracted
    before exponentiating (the same function, numerically safe)."""
    q, K, V = _f64(q), _f64(K), _f64(V)
    s = K @ q / np.sqrt(q.size)
    w = np.exp(s - s.max())
    return (w / w.sum()) @ V


class KVCache:
    """One layer's decode state: the stored inputs of every past token, and per
    head the K/V rows computed so far (in the storage dtype's values) with a
    flag per position saying whether the row exists."""

    def __init__(self, nh: int, dh: int, d: int, tmax: int, round_kv):
        self.nh, self.dh, self.d, self.tmax = nh, dh, d, tmax
        self.Y = np.zeros((tmax, d))
        self.K = np.zeros((nh, tmax, dh))
        self.V = np.zeros((nh, tmax, dh))
        self.filled = np.zeros((nh, tmax), dtype=bool)
        self.t = 0                     # tokens stored so far
        self.round_kv = round_kv       # fp64 -> the stored values (storage-dtype rounding)


def mha_sparse_step(Wt, cache: KVCache, y, heads) -> np.ndarray:
    """Decode one token through the attention block restricted to ``heads``
    (equation (-1)): store y; for each selected head fill its missing K/V rows
    from the stored inputs, then attend over positions 0..t; sum the selected
    heads' output projections.  ``Wt``: dict with Wq, bq, Wk, bk, Wv, bv ([nh
    dh, d] and [nh dh]), Wo ([d, nh dh]) and bo ([d]); biases may be None."""
    t = cache.t
    assert t < cache.tmax
    cache.Y[t] = _f64(y)
    cache.t = t + 1
    dh = cache.dh
    out = np.zeros(cache.d) if Wt.get("bo") is None else _f64(Wt["bo"]).copy()
    Wo = _f64(Wt["Wo"])
    for h in np.asarray(heads, dtype=np.int64):
        h = int(h)
        for p in range(t + 1):
            if not cache.filled[h, p]:
                cache.K[h, p] = cache.round_kv(head_rows(Wt["Wk"], Wt.get("bk"), h, dh, cache.Y[p]))
                cache.V[h, p] = cache.round_kv(head_rows(Wt["Wv"], Wt.get("bv"), h, dh, cache.Y[p]))
                cache.filled[h, p] = True
        q = head_rows(Wt["Wq"], Wt.get("bq"), h, dh, cache.Y[t])
        o = attend(q, cache.K[h, :t + 1], cache.V[h, :t + 1])
        out += Wo[:, h * dh:(h + 1) * dh] @ o
    return out


def mha_dense(Wt, Yhist, nh: int, dh: int, round_kv, heads=None) -> np.ndarray:
    """Textbook multi-head attention of the last token of ``Yhist`` [t+1, d]
    over all of them, in matrix form (all heads at once): Q, K, V projections of
    the whole history, per-head scaled scores and softmax, concatenated head
    outputs times Wo.  ``heads`` restricts the output sum to those heads (all by
    default); K and V pass through ``round_kv`` as they would in a cache."""
    Y = _f64(Yhist)
    bias = lambda name, w: 0.0 if Wt.get(name) is None else _f64(Wt[name])[None, :]
    Q = Y @ _f64(Wt["Wq"]).T + bias("bq", Wt["Wq"])
    K = round_kv(Y @ _f64(Wt["Wk"]).T + bias("bk", Wt["Wk"]))
    V = round_kv(Y @ _f64(Wt["Wv"]).T + bias("bv", Wt["Wv"]))
    T = Y.shape[0]
    q = Q[-1].reshape(nh, dh)                      # [nh, dh]
    Kh = K.reshape(T, nh, dh).transpose(1, 0, 2)   # [nh, T, dh]
    Vh = V.reshape(T, nh, dh).transpose(1, 0, 2)
    S = np.einsum("hd,htd->ht", q, Kh) / np.sqrt(dh)
    P = np.exp(S - S.max(axis=1, keepdims=True))
    P = P / P.sum(axis=1, keepdims=True)
    O = np.einsum("ht,htd->hd", P, Vh)             # [nh, dh]
    mask = np.zeros(nh, dtype=bool)
    mask[np.arange(nh) if heads is None else np.asarray(heads, dtype=np.int64)] = True
    O = O * mask[:, None]
    out = _f64(Wt["Wo"]) @ O.reshape(nh * dh)
    if Wt.get("bo") is not None:
        out = out + _f64(Wt["bo"])
    return out
