"""Hot-neuron L2 residency (spffn_set_l2_hot_rows): the cache-eviction hints on
the small-batch decode kernel's copies change where bytes are cached, never the
arithmetic.  With the hints on, decode (plain, look-ahead and on caller tables)
gives bit-identical results to the run without them, and the run matches the
oracle layer by layer."""
import numpy as np
import pytest

import activation_sparse_ffn_predictor_b200 as sp
import oracle as O
import workload as wl
from _gpu import HostOracle, bits_of, check_stack, oracle_layer, prefix_runner, torch_layer, x_tokens

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu


def dealt_layers(cfg, Lc, B):
    """Layers placed hot-first and dealt over the kernel's ranges, from a profile."""
    hs = [wl.host_layer(cfg, l) for l in range(Lc)]
    G = sp.Layer(**torch_layer(hs[0]), max_batch=B).num_partials
    out = []
    for l, h in enumerate(hs):
        Xp = wl.widen(wl.tokens(cfg, 64, aux=l, tensor=wl.T_XPROF), cfg.bf16)
        counts = O.activation_counts(h.f64("W1"), h.f64("b1"), Xp)
        perm = O.dealt_order(counts, G)
        for name in ("W1", "W2T", "Wp2", "b1", "bp2"):
            setattr(h, name, np.ascontiguousarray(getattr(h, name)[perm]))
        out.append(h)
    return out


@pytest.mark.parametrize("B,lookahead", [(1, False), (1, True), (2, False)])
def test_hot_row_hints_keep_results_bitwise(B, lookahead):
    cfg = wl.CONFIGS[0]
    Lc = 3
    hs = dealt_layers(cfg, Lc, B)
    layers = [sp.Layer(**torch_layer(h), max_batch=B) for h in hs]
    xb, x64 = x_tokens(cfg, B, aux=61)
    dt = torch.float16
    outs = []
    try:
        for rows in (0, 2):
            sp.set_l2_hot_rows(rows)
            assert sp.l2_hot_rows() == rows
            x_out = torch.empty(B, cfg.d, dtype=dt, device="cuda")
            y = torch.empty(B, cfg.d, dtype=torch.float32, device="cuda")
            counts = torch.full((Lc,), -1, dtype=torch.int32, device="cuda")
            sp.decode(layers, wl.to_torch(xb, cfg), x_out, y, counts, lookahead=lookahead)
            torch.cuda.synchronize()
            for L in layers:
                assert L.last_device_error() == (sp.OK, 0)
            outs.append((bits_of(x_out), y.cpu().numpy(), counts.cpu().numpy(),
                         [L.table(int(k)).cpu().numpy() for L, k in zip(layers, counts.cpu().numpy())]))
    finally:
        sp.set_l2_hot_rows(0)
    a, b = outs
    assert np.array_equal(a[0], b[0]) and np.array_equal(a[1], b[1]) and np.array_equal(a[2], b[2])
    assert all(np.array_equal(u, v) for u, v in zip(a[3], b[3]))
    check_stack(layers, [HostOracle(h) for h in hs], cfg, x64, torch.from_numpy(b[1]),
                torch.from_numpy(b[0].view(np.int16)).view(torch.float16), torch.from_numpy(b[2]),
                lookahead=lookahead, run_prefix=prefix_runner(layers, wl.to_torch(xb, cfg), cfg, lookahead))


def test_hot_row_hints_on_caller_tables():
    cfg = wl.CONFIGS[0]
    Lc, B = 2, 1
    hs = dealt_layers(cfg, Lc, B)
    layers = [sp.Layer(**torch_layer(h), max_batch=B) for h in hs]
    xb, x64 = x_tokens(cfg, B, aux=62)
    OL = oracle_layer(hs[0])
    z = O.fc1_preactivation(OL["W1"], OL["b1"], x64)
    tab0 = np.nonzero(np.any(z > 0, axis=0))[0].astype(np.int32)
    tabs = [torch.from_numpy(tab0).cuda(), torch.from_numpy(tab0[::2].copy()).cuda()]
    tc = torch.tensor([tab0.size, tab0[::2].size], dtype=torch.int32, device="cuda")
    outs = []
    try:
        for rows in (0, 3):
            sp.set_l2_hot_rows(rows)
            x_out = torch.empty(B, cfg.d, dtype=torch.float16, device="cuda")
            y = torch.empty(B, cfg.d, dtype=torch.float32, device="cuda")
            sp.decode_tables(layers, wl.to_torch(xb, cfg), tabs, tc, x_out, y)
            torch.cuda.synchronize()
            outs.append((bits_of(x_out), y.cpu().numpy()))
    finally:
        sp.set_l2_hot_rows(0)
    assert np.array_equal(outs[0][0], outs[1][0]) and np.array_equal(outs[0][1], outs[1][1])


def test_hot_row_setting_rejects_negative():
    assert sp.library().spffn_set_l2_hot_rows(-1) == sp.ERR_INVALID_ARG
    assert sp.l2_hot_rows() == 0
