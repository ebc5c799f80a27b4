"""Shared helpers for the GPU parity tests: seeded inputs from ``workload``,
expected values from ``oracle`` only, results from the CUDA library."""
import math

import numpy as np

import oracle as O
import workload as wl

REL_L2_BAR = 1e-3      # the contract on FFN outputs, applied to every token
LOGIT_BAND = 1e-4      # neurons whose logit lies this close to 0 may go either way
# Internal bar on a layer's y when the GPU and the oracle see the same input.  The
# kernels accumulate in fp32 (relative error ~1e-7 over these sums); the union path
# feeds fp32 activations to the 16-bit MMA as a hi/lo pair of the storage type, whose
# residual is at most 2^-22 (fp16) or 2^-18 (bf16) of the value, ~2e-6 rms for bf16.
Y_INTERNAL_BAR = 1e-5
# Internal bar on the last y of a stack.  After layer 0 the oracle's chained input is
# its own fp64 rounding of x + y, the kernel's a rounding of an fp32 value that is
# within ~1e-6 relative of it; the two round apart on the few elements that fall that
# close to a rounding boundary (about d 1e-6 / ulp of them).  One such element moves
# the next y by about ulp |W1| / rms(a) ~ ulp / (0.7 sqrt(d)) relative: ~2e-5 for fp16
# (ulp 2^-10 near 1) and ~3e-4 for bf16 (ulp 2^-7) at d ~ 1000-4000.  So a stack's
# last y gets 1e-4 in fp16 and only the contract itself, 1e-3, in bf16.
STACK_Y_INTERNAL_BAR = 1e-4
STACK_Y_INTERNAL_BAR_BF16 = REL_L2_BAR


def rel_l2(got, want):
    got = np.asarray(got, dtype=np.float64)
    want = np.asarray(want, dtype=np.float64)
    den = np.linalg.norm(want)
    return np.linalg.norm(got - want) / (den if den > 0 else 1.0)


def check_y(got, want, internal=Y_INTERNAL_BAR):
    """The 1e-3 relative-L2 bound on every token (rows of [B, d]) plus the tighter
    internal bar on the whole tensor; returns the whole-tensor error."""
    got = np.atleast_2d(np.asarray(got, dtype=np.float64))
    want = np.atleast_2d(np.asarray(want, dtype=np.float64))
    assert got.shape == want.shape, (got.shape, want.shape)
    assert np.all(np.isfinite(got)), "non-finite output"
    per = [rel_l2(got[t], want[t]) for t in range(got.shape[0])]
    worst = int(np.argmax(per))
    assert per[worst] <= REL_L2_BAR, "token %d: rel L2 %.3g" % (worst, per[worst])
    err = rel_l2(got, want)
    assert err <= internal, "rel L2 %.3g above the internal bar %.0e" % (err, internal)
    return err


def ulp_of(v, bf16):
    """Spacing of the storage type at |v| (subnormal spacing below the normal range)."""
    m, emin = (7, -126) if bf16 else (10, -14)
    a = np.abs(np.asarray(v, dtype=np.float64))
    e = np.floor(np.log2(np.maximum(a, 2.0 ** emin)))
    return np.exp2(e - m)


def check_x(got_bits, want64, bf16, stack=False, slack=None):
    """A chained input in the storage dtype: every token within the contract and
    every element within 2 ulp of the oracle's value (both sides round once, from
    fp32 and fp64 values that differ slightly).  ``slack`` (absolute, per element)
    adds the part of the difference the layer's y error carries into x: where x
    and y nearly cancel, an error far below the contract in y is many ulps of the
    small result.  For the output of a stack of independently chained oracle
    inputs (``stack``), 2 ulp of 1.0 more."""
    got = wl.widen(got_bits, bf16)
    want = np.asarray(want64, dtype=np.float64)
    assert got.shape == want.shape
    for t in range(got.shape[0]):
        assert rel_l2(got[t], want[t]) <= REL_L2_BAR, t
    bound = 2 * ulp_of(want, bf16) + (2 * ulp_of(1.0, bf16) if stack else 0.0)
    if slack is not None:
        bound = bound + slack
    bad = np.abs(got - want) > bound
    assert not bad.any(), "x differs beyond 2 ulp at %d elements, e.g. %s" % (
        bad.sum(), list(zip(got[bad][:3], want[bad][:3])))


def torch_layer(h: wl.HostLayer, device="cuda"):
    """Upload a full host layer (bit-exact) as torch tensors."""
    cfg = h.cfg
    t = lambda a: wl.to_torch(a, cfg, device)
    return dict(W1=t(h.W1), b1=t(h.b1), W2T=t(h.W2T), b2=t(h.b2), Wp1=t(h.Wp1), bp1=t(h.bp1),
                Wp2=t(h.Wp2), bp2=t(h.bp2))


def oracle_layer(h: wl.HostLayer):
    return dict(W1=h.f64("W1"), b1=h.f64("b1"), W2T=h.f64("W2T"), b2=h.f64("b2"), Wp1=h.f64("Wp1"),
                bp1=h.f64("bp1"), Wp2=h.f64("Wp2"), bp2=h.f64("bp2"))


def ambiguous(logits):
    """Neurons whose union decision max_t l_t lies within LOGIT_BAND of zero."""
    m = np.atleast_2d(logits).max(axis=0)
    return set(np.nonzero(np.abs(m) < LOGIT_BAND)[0].tolist())


def check_table(idx_gpu, k_gpu, idx_or, logits):
    """Bit-exact neuron table outside the near-threshold band; returns the
    ambiguous neurons on which the two sides differ."""
    idx_gpu = np.asarray(idx_gpu[:k_gpu])
    assert np.all(np.diff(idx_gpu) > 0), "table not strictly ascending"
    amb = ambiguous(logits)
    diff = set(idx_gpu.tolist()) ^ set(np.asarray(idx_or).tolist())
    assert diff <= amb, "tables differ outside the near-threshold band: %s" % sorted(diff - amb)[:10]
    keep_g = [j for j in idx_gpu.tolist() if j not in amb]
    keep_o = [j for j in np.asarray(idx_or).tolist() if j not in amb]
    assert keep_g == keep_o
    return diff


def x_tokens(cfg, B, aux, layer=0):
    bits = wl.tokens(cfg, B, aux=aux, layer=layer)
    return bits, wl.widen(bits, cfg.bf16)


def bits_of(t):
    """Storage bits (uint16) of a float16/bfloat16 torch tensor."""
    import torch
    return t.detach().cpu().view(torch.int16).numpy().view(np.uint16)


class HostOracle:
    """The oracle's view of one small layer held in full on the host."""

    def __init__(self, h: wl.HostLayer):
        self.L = oracle_layer(h)

    def predict(self, x64):
        L = self.L
        return O.predict(L["Wp1"], L["Wp2"], L["bp2"], x64, L["bp1"])

    def ffn(self, x64, table):
        L = self.L
        return O.sparse_ffn(L["W1"], L["b1"], L["W2T"], L["b2"], x64, table)


class RowsOracle:
    """The oracle's view of one full-size layer filled on the device by the
    device twin of the generator: the whole predictor is regenerated on the host,
    and of W1/W2T only the rows a table names (b2 = 0 in the workloads)."""

    def __init__(self, cfg, layer, rate=None):
        self.cfg, self.layer = cfg, layer
        bf = cfg.bf16
        p, Wp1, bp1, Wp2, bp2 = wl.host_predictor(cfg, layer, rate=rate)
        self.Wp1, self.bp1 = wl.widen(Wp1, bf), wl.widen(bp1, bf)
        self.Wp2, self.bp2 = wl.widen(Wp2, bf), wl.widen(bp2, bf)
        self.b1 = wl.widen(wl.fc1_bias(p, bf), bf)

    def predict(self, x64):
        return O.predict(self.Wp1, self.Wp2, self.bp2, x64, self.bp1)

    def ffn(self, x64, table):
        cfg = self.cfg
        table = np.asarray(table, dtype=np.int64)
        sc = 1.0 / math.sqrt(cfg.d)
        W1 = wl.widen(wl.fill_rows(wl.stream_id(wl.T_W1, self.layer), cfg.d, table, sc, cfg.bf16), cfg.bf16)
        W2T = wl.widen(wl.fill_rows(wl.stream_id(wl.T_W2T, self.layer), cfg.d, table, sc, cfg.bf16), cfg.bf16)
        return O.sparse_ffn(W1, self.b1, W2T, np.zeros(cfg.d), x64, table, row_ids=table)


def prefix_runner(layers, x_in, cfg, lookahead=False):
    """Runs spffn_decode (or its look-ahead form) over the first k layers of the
    stack on the same input and returns the storage bits of x_k and that run's
    y (the y of layer k-1).  Every decode path is deterministic, so these are the
    full run's own intermediate values."""
    def run(k):
        import torch
        import activation_sparse_ffn_predictor_b200 as sp
        B = x_in.shape[0]
        x_out = torch.empty_like(x_in)
        y = torch.empty(B, cfg.d, dtype=torch.float32, device=x_in.device)
        counts = torch.full((k,), -1, dtype=torch.int32, device=x_in.device)
        sp.decode(layers[:k], x_in, x_out, y, counts, lookahead=lookahead)
        torch.cuda.synchronize()
        return bits_of(x_out), y.cpu().numpy()
    return run


def check_stack(layers, oracles, cfg, x64, y, x_out, counts, lookahead=False, run_prefix=None):
    """A whole decode step against the oracle, layer by layer, on every layer,
    with the oracle fed the GPU's own input of each layer.

    ``run_prefix(k)`` (see prefix_runner) gives the GPU's x_k and the y of
    layer k-1; the full run gives the last ones.  For every layer l:
    - its table (read back through spffn_layer_table) must equal the oracle's
      prediction from the GPU's x_l (from x_{l-1} under look-ahead; layer 0 from
      x_0) outside the near-threshold band, and its count must be its length;
      inside the band the GPU's table is one of the valid answers, and the
      oracle's FFN is taken over the table the GPU used;
    - y_l must match the oracle's FFN of the GPU's x_l per token (the contract)
      and overall within the internal bar;
    - x_{l+1} must be the oracle's chaining of (x_l, y_l) within 2 ulp.
    Returns the number of layers whose tables differed inside the band."""
    kc = counts.cpu().numpy()
    L = len(layers)
    if run_prefix is None:
        assert L == 1, "a stack needs run_prefix to obtain its intermediate layer inputs"
    outs = [run_prefix(k) for k in range(1, L)] + [(bits_of(x_out), y.cpu().numpy())]
    xs = [x64] + [wl.widen(o[0], cfg.bf16) for o in outs]
    in_band = 0
    for l, (Ly, Or) in enumerate(zip(layers, oracles)):
        xp = xs[max(l - 1, 0)] if lookahead else xs[l]
        idx_or, k_or, logits = Or.predict(xp)
        k = int(kc[l])
        assert 0 <= k <= cfg.n, (l, k)
        tab = Ly.table(k).cpu().numpy()
        diff = check_table(tab, k, idx_or, logits)
        assert abs(k - k_or) <= len(diff), (l, k, k_or)
        in_band += bool(diff)
        y_or = Or.ffn(xs[l], tab if diff else idx_or)
        check_y(outs[l][1], y_or)
        # x_{l+1} = round(u rs) with u = x_l + y: the GPU's y error moves u by |dy|
        u = xs[l] + y_or
        rs = 1.0 / np.sqrt(np.mean(u * u, axis=1, keepdims=True) + O.RMS_EPS)
        slack = 1.01 * rs * np.abs(np.asarray(outs[l][1], dtype=np.float64) - y_or) + 1e-12
        check_x(outs[l][0], wl.widen(wl.round_to(O.chain(xs[l], y_or), cfg.bf16), cfg.bf16), cfg.bf16,
                slack=slack)
    return in_band
