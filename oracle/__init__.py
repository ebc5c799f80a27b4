"""CPU oracle for activation-sparse FFN decoding — TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline leg
may import this package.  The CUDA library never does, and this package never
imports the CUDA library: the two share nothing but the seeded input
generator in ``workload/``.

Everything here is plain numpy in fp64, written to be checked by eye against
the pages.  Inputs are the stored fp16/bf16 values widened exactly to fp64.
Page titles used in citations:

* [PI1] "LLM模型之PowerInfer1.0" (blog-zz7.pages.dev), sections 2.1, 3.2, 4.1,
  4.2, 4.4, 5.1–5.2 and the DejaVu appendix with its equation (-1) and the
  closing question on why down-projection uses AXPY.
* [SPX] "Técnicas dispersas para una aceleración 100X en la inferencia de
  modelos de lenguaje grandes" (blogs.novita.ai/es), on ReLU activation
  sparsity, batch effects and the PowerInfer worked example.
* [UAI] "PowerInfer: Nhanh Large Language Model với GPU Tiêu dùng" (unite.ai/vi),
  on neuron tables.

Readings where the pages leave a step open (all pinned by tests unless noted):

* predictor hidden activation is ReLU, hidden bias ``bp1`` (default 0);
* the sigmoid > 0.5 decision is taken as the equivalent strict ``logit > 0``;
* for a batch, the neuron set is the union of the per-token predicted sets and
  every token is computed on every neuron of the union;
* the neuron table is ascending in physical (stored-row) order;
* an empty set gives ``y = b2``;
* the layer chaining used by multi-layer runs is
  ``x' = round_dtype((x + y) / sqrt(mean((x + y)^2) + eps))`` with eps = 1e-6;
* under look-ahead prediction the set of layer l+1 comes from layer l+1's own
  predictor applied to layer l's input (equation (-2) writes the predictor with
  the earlier layer's index, but its outputs are layer l+1's neurons), and the
  first layer, having no earlier input, predicts from its own.

Parity of the predictor's *quality* (recall against the true active set) is
unpinned: with random weights there is nothing to claim, and no function here
computes it.
"""
from __future__ import annotations

import numpy as np


def _f64(a) -> np.ndarray:
    return np.asarray(a, dtype=np.float64)


def _tokens(x) -> np.ndarray:
    x = _f64(x)
    return x[None, :] if x.ndim == 1 else x


def relu(v: np.ndarray) -> np.ndarray:
    """[PI1] §2.1: ReLU gates FC1's output, keeping positive values, zeroing the rest."""
    return np.maximum(v, 0.0)


# ---------------------------------------------------------------------------
# the X-H-O predictor
def predictor_hidden(Wp1, x, bp1=None) -> np.ndarray:
    """Hidden layer of the two-layer X-H-O MLP predictor ([PI1] §1 item 2.1,
    §4.1; DejaVu appendix): ``h_t = ReLU(Wp1 x_t + bp1)``, shape [B, H]."""
    X = _tokens(x)
    pre = X @ _f64(Wp1).T
    if bp1 is not None:
        pre = pre + _f64(bp1)[None, :]
    return relu(pre)


def predictor_logits(Wp2, h, bp2=None) -> np.ndarray:
    """Output layer of the predictor: one logit per FFN neuron, ``l_t = Wp2 h_t + bp2``,
    shape [B, n] ([PI1] DejaVu appendix: one sigmoid output per unit)."""
    out = _f64(h) @ _f64(Wp2).T
    if bp2 is not None:
        out = out + _f64(bp2)[None, :]
    return out


def predicted_mask(logits) -> np.ndarray:
    """Per-neuron decision for a batch: neuron i is selected when any token's
    sigmoid output exceeds 0.5, i.e. ``logit > 0`` ([PI1] DejaVu appendix,
    binary decision per output; union over the batch per [SPX] on batch size)."""
    L = np.atleast_2d(_f64(logits))
    return np.any(L > 0.0, axis=0)


def neuron_table(mask) -> tuple[np.ndarray, int]:
    """Compact a mask into the neuron table: ascending physical indices of the
    selected neurons and their count ([PI1] §4.2, [UAI] neuron tables)."""
    m = np.asarray(mask, dtype=bool)
    idx = np.nonzero(m)[0].astype(np.int32)
    return idx, int(idx.size)


def predict(Wp1, Wp2, bp2, x, bp1=None):
    """Predictor + threshold + compaction for one layer: returns (idx, count, logits)."""
    h = predictor_hidden(Wp1, x, bp1)
    l = predictor_logits(Wp2, h, bp2)
    idx, k = neuron_table(predicted_mask(l))
    return idx, k, l


# ---------------------------------------------------------------------------
# the FFN block
def fc1_preactivation(W1, b1, x, rows=None) -> np.ndarray:
    """``z_{t,j} = W1[j] . x_t + b1_j`` ([PI1] §2.1: each FC1 output is the dot
    product of the input with one neuron's row); [B, len(rows)] or [B, n]."""
    W = _f64(W1)
    b = _f64(b1)
    if rows is not None:
        W = W[rows]
        b = b[rows]
    return _tokens(x) @ W.T + b[None, :]


def dense_ffn(W1, b1, W2T, b2, x) -> np.ndarray:
    """Dense ReLU FFN, ``y_t = W2 ReLU(W1 x_t + b1) + b2`` with ``W2 = W2T^T``
    ([PI1] §2.1, Figure 1 description); [B, d]."""
    a = relu(fc1_preactivation(W1, b1, x))
    y = a @ _f64(W2T)
    if b2 is not None:
        y = y + _f64(b2)[None, :]
    return y


def sparse_ffn(W1, b1, W2T, b2, x, idx, row_ids=None) -> np.ndarray:
    """Neuron-aware FFN ([PI1] §4.4 and the closing AXPY question): for each
    neuron j of the table, in ascending order, ``a = ReLU(W1[j] . x + b1_j)`` (a
    vec_dot over FC1's row) and ``y += a * W2T[j]`` (an AXPY over the neuron's
    contiguous column of FC2).  Neurons outside the table contribute nothing.

    ``row_ids`` maps physical neuron j to its row in ``W1``/``W2T`` when only
    some rows are held (``W1[row_ids.index(j)]``); ``b1`` is always full length.
    """
    X = _tokens(x)
    B, d = X.shape
    y = np.zeros((B, d), dtype=np.float64)
    if b2 is not None:
        y += _f64(b2)[None, :]
    W1 = _f64(W1)
    W2T = _f64(W2T)
    b1 = _f64(b1)
    where = None
    if row_ids is not None:
        where = {int(r): i for i, r in enumerate(np.asarray(row_ids))}
    for j in np.asarray(idx, dtype=np.int64):
        r = int(j) if where is None else where[int(j)]
        a = relu(X @ W1[r] + b1[int(j)])          # [B]
        y += a[:, None] * W2T[r][None, :]
    return y


def step(layer, x):
    """One layer: predict (hidden, logits, union mask, neuron table) then the
    neuron-aware FFN over the table ([PI1] DejaVu equation (-1): S_M from the
    predictor on the FFN input, then the MLP restricted to S_M)."""
    idx, k, logits = predict(layer["Wp1"], layer["Wp2"], layer["bp2"], x, layer.get("bp1"))
    y = sparse_ffn(layer["W1"], layer["b1"], layer["W2T"], layer.get("b2"), x, idx)
    return idx, k, logits, y


def step_lookahead(layer, x_pred, x):
    """One layer under look-ahead prediction ([PI1] DejaVu appendix, equation (-2)
    and the closing list on DejaVu's speed: the sparsity of layer l+1 is predicted
    from layer l's input while layer l computes).  The layer's own predictor is
    applied to ``x_pred`` (the previous layer's input; the layer's own input for
    the first layer) and the FFN runs on ``x`` restricted to that set."""
    idx, k, logits = predict(layer["Wp1"], layer["Wp2"], layer["bp2"], x_pred, layer.get("bp1"))
    y = sparse_ffn(layer["W1"], layer["b1"], layer["W2T"], layer.get("b2"), x, idx)
    return idx, k, logits, y


# ---------------------------------------------------------------------------
# offline profiling and hot-first placement
def activation_counts(W1, b1, X) -> np.ndarray:
    """Offline profile ([PI1] §5.1): for every profiling token, each neuron whose
    FC1 output is positive has its count incremented; returns uint32 counts."""
    z = fc1_preactivation(W1, b1, X)
    return np.sum(z > 0.0, axis=0).astype(np.uint32)


def hot_first_order(counts) -> np.ndarray:
    """Neuron placement by impact ([PI1] §5.2 equation (1): impact = profiled
    activation frequency): permutation ``perm`` (new slot -> original neuron)
    ordering neurons by count descending, ties by original index ascending."""
    c = np.asarray(counts, dtype=np.int64)
    return np.lexsort((np.arange(c.size), -c)).astype(np.int32)


def dealt_order(counts, parts: int) -> np.ndarray:
    """Hot-first order dealt over ``parts`` contiguous slot ranges: range c holds
    slots [floor(n c/parts), floor(n (c+1)/parts)); the i-th hottest neuron (per
    hot_first_order) goes to range i mod parts, into its next free slot.  A
    placement choice of this library (impact-ordered, [PI1] §5.2 equation (1)),
    spreading hot neurons evenly over the ranges."""
    hot = hot_first_order(counts)
    n = hot.size
    bounds = [n * c // parts for c in range(parts + 1)]
    fill = [bounds[c] for c in range(parts)]
    perm = np.empty(n, dtype=np.int32)
    c = 0
    for neuron in hot:
        while fill[c] >= bounds[c + 1]:      # range already full: next range
            c = (c + 1) % parts
        perm[fill[c]] = neuron
        fill[c] += 1
        c = (c + 1) % parts
    return perm


def permute_rows(a, perm) -> np.ndarray:
    """Apply the neuron table: row ``s`` of the result is row ``perm[s]``."""
    return np.asarray(a)[np.asarray(perm, dtype=np.int64)]


# ---------------------------------------------------------------------------
# multi-layer chaining (a reading, see module docstring)
RMS_EPS = 1e-6


def chain(x, y, eps: float = RMS_EPS) -> np.ndarray:
    """Next layer's input in fp64: ``(x + y) / sqrt(mean((x + y)^2) + eps)``,
    per token; rounding to the storage dtype is left to the caller."""
    u = _tokens(x) + _f64(y)
    rms = np.sqrt(np.mean(u * u, axis=1, keepdims=True) + eps)
    return u / rms
