"""Decode on caller-supplied neuron tables, no predictor (spffn_decode_tables):
each layer's table is the oracle's true activation set (z > 0) of its own
chained input; y and the final x against the oracle over the same tables.
Covers the persistent kernel (B <= 2) and the per-layer path (B = 3), table order
(a table is a set) and out-of-range entries (skipped, latched)."""
import numpy as np
import pytest

import activation_sparse_ffn_predictor_b200 as sp
import oracle as O
import workload as wl
from _gpu import STACK_Y_INTERNAL_BAR, STACK_Y_INTERNAL_BAR_BF16, bits_of, check_x, check_y, oracle_layer, torch_layer, x_tokens

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

CASES = {
    "block-d1024-n4096-L4": (wl.CONFIGS[0], 4),
    "ragged-bf16-d1088-n4128-H320-L3": (wl.FFNConfig("ragged", 1, 1088, 4128, 320, "bf16", 1.0, 0.2), 3),
}


def oracle_true_chain(cfg, hs, x64):
    xs, tabs, ys = [x64], [], []
    for h in hs:
        OL = oracle_layer(h)
        z = O.fc1_preactivation(OL["W1"], OL["b1"], xs[-1])
        tab = np.nonzero(np.any(z > 0, axis=0))[0].astype(np.int32)
        y = O.sparse_ffn(OL["W1"], OL["b1"], OL["W2T"], OL["b2"], xs[-1], tab)
        tabs.append(tab)
        ys.append(y)
        xs.append(wl.widen(wl.round_to(O.chain(xs[-1], y), cfg.bf16), cfg.bf16))
    return tabs, ys, xs


def run_tables(cfg, layers, xb, tabs, B):
    dt = torch.bfloat16 if cfg.bf16 else torch.float16
    x_out = torch.empty(B, cfg.d, dtype=dt, device="cuda")
    y = torch.empty(B, cfg.d, dtype=torch.float32, device="cuda")
    counts = torch.full((len(tabs),), -1, dtype=torch.int32, device="cuda")
    tt = [torch.from_numpy(np.ascontiguousarray(t, dtype=np.int32)).cuda() if len(t) else
          torch.zeros(1, dtype=torch.int32, device="cuda") for t in tabs]
    tc = torch.tensor([len(t) for t in tabs], dtype=torch.int32, device="cuda")
    sp.decode_tables(layers, wl.to_torch(xb, cfg), tt, tc, x_out, y, counts)
    torch.cuda.synchronize()
    return x_out, y, counts


@pytest.mark.parametrize("B", [1, 2, 3])
@pytest.mark.parametrize("name", list(CASES))
def test_decode_tables_true_sets_match_oracle(name, B):
    cfg, Lc = CASES[name]
    hs = [wl.host_layer(cfg, l) for l in range(Lc)]
    layers = [sp.Layer(**torch_layer(h), max_batch=B) for h in hs]
    xb, x64 = x_tokens(cfg, B, aux=1100 + B)
    tabs, ys, xs = oracle_true_chain(cfg, hs, x64)
    x_out, y, counts = run_tables(cfg, layers, xb, tabs, B)
    assert counts.cpu().numpy().tolist() == [len(t) for t in tabs]
    check_y(y.cpu().numpy(), ys[-1], internal=STACK_Y_INTERNAL_BAR_BF16 if cfg.bf16 else STACK_Y_INTERNAL_BAR)
    check_x(bits_of(x_out), xs[-1], cfg.bf16, stack=True)
    for L in layers:
        assert L.last_device_error() == (sp.OK, 0)


@pytest.mark.parametrize("B", [1, 3])
def test_decode_tables_order_and_bad_entries(B):
    cfg, Lc = CASES["block-d1024-n4096-L4"]
    hs = [wl.host_layer(cfg, l) for l in range(2)]
    layers = [sp.Layer(**torch_layer(h), max_batch=B) for h in hs]
    xb, x64 = x_tokens(cfg, B, aux=1200 + B)
    tabs, ys, xs = oracle_true_chain(cfg, hs, x64)
    r = np.random.default_rng(B)
    shuffled = [r.permutation(t).astype(np.int32) for t in tabs]
    x_out, y, counts = run_tables(cfg, layers, xb, shuffled, B)
    check_y(y.cpu().numpy(), ys[-1], internal=STACK_Y_INTERNAL_BAR_BF16 if cfg.bf16 else STACK_Y_INTERNAL_BAR)
    for L in layers:
        assert L.last_device_error() == (sp.OK, 0)
    # out-of-range entries in layer 0's table: skipped (the result is unchanged) and latched
    bad = [np.concatenate([[cfg.n + 3], tabs[0], [-7]]).astype(np.int32), tabs[1]]
    x_out, y, counts = run_tables(cfg, layers, xb, bad, B)
    check_y(y.cpu().numpy(), ys[-1], internal=STACK_Y_INTERNAL_BAR_BF16 if cfg.bf16 else STACK_Y_INTERNAL_BAR)
    s, code = layers[0].last_device_error()
    assert s == sp.ERR_DEVICE_CHECK and code & 2
