"""Shared helpers for the GPU parity tests: seeded inputs from ``workload``,
expected values from ``oracle`` only, results from the CUDA library."""
import numpy as np

import oracle as O
import workload as wl

REL_L2_BAR = 1e-3      # bound on FFN outputs
LOGIT_BAND = 1e-4      # neurons whose logit lies this close to 0 may go either way


def rel_l2(got, want):
    got = np.asarray(got, dtype=np.float64)
    want = np.asarray(want, dtype=np.float64)
    den = np.linalg.norm(want)
    return np.linalg.norm(got - want) / (den if den > 0 else 1.0)


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
