"""Full-size parity (needs a B200): the five workloads' layer shapes, filled in
HBM by the device generator; the oracle regenerates on the host exactly the
tensors it needs (whole predictor, only the selected FFN rows) and checks the
sampled layers/steps."""
import math

import numpy as np
import pytest

import activation_sparse_ffn_predictor_b200 as sp
import oracle as O
import workload as wl
from _gpu import check_table, check_y, x_tokens

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu


def test_device_generator_matches_host():
    for cfg in (wl.CONFIGS[1], wl.CONFIGS[2]):
        dl = wl.device_layer(cfg, 3)
        h_p, Wp1, bp1, Wp2, bp2 = wl.host_predictor(cfg, 3)
        bits = lambda t: t.cpu().view(torch.int16).numpy().view(np.uint16)
        assert np.array_equal(bits(dl.Wp1), Wp1)
        assert np.array_equal(bits(dl.Wp2), Wp2)
        assert np.array_equal(bits(dl.bp2), bp2)
        rows = np.array([0, 1, 777, cfg.n - 1])
        sc = 1.0 / math.sqrt(cfg.d)
        assert np.array_equal(bits(dl.W1)[rows], wl.fill_rows(wl.stream_id(wl.T_W1, 3), cfg.d, rows, sc, cfg.bf16))
        assert np.array_equal(bits(dl.W2T)[rows], wl.fill_rows(wl.stream_id(wl.T_W2T, 3), cfg.d, rows, sc, cfg.bf16))
        del dl
        torch.cuda.empty_cache()


def _oracle_layer_rows(cfg, layer, x64, rate=None):
    """Oracle for one full-size layer: returns (idx, logits, y, W-rows)."""
    p, Wp1, bp1, Wp2, bp2 = wl.host_predictor(cfg, layer, rate=rate)
    bf = cfg.bf16
    idx, k, logits = O.predict(wl.widen(Wp1, bf), wl.widen(Wp2, bf), wl.widen(bp2, bf), x64, wl.widen(bp1, bf))
    return p, idx, logits


def _rows_y(cfg, layer, p, x64, table):
    sc = 1.0 / math.sqrt(cfg.d)
    table = np.asarray(table, dtype=np.int64)
    W1 = wl.widen(wl.fill_rows(wl.stream_id(wl.T_W1, layer), cfg.d, table, sc, cfg.bf16), cfg.bf16)
    W2T = wl.widen(wl.fill_rows(wl.stream_id(wl.T_W2T, layer), cfg.d, table, sc, cfg.bf16), cfg.bf16)
    b1 = wl.widen(wl.fc1_bias(p, cfg.bf16), cfg.bf16)
    return O.sparse_ffn(W1, b1, W2T, np.zeros(cfg.d), x64, table, row_ids=table)


@pytest.mark.parametrize("cfg_id,B,rate", [(2, 16, None), (2, 4, None), (3, 1, 0.20), (3, 1, 0.01), (4, 32, None)])
def test_fullsize_layer_step(cfg_id, B, rate):
    cfg = wl.CONFIGS[cfg_id]
    layer = 5
    dl = wl.device_layer(cfg, layer, rate=rate)
    L = sp.Layer.from_device_layer(dl, max_batch=B)
    xb, x64 = x_tokens(cfg, B, aux=1000 + B, layer=layer)
    idx = torch.empty(cfg.n, dtype=torch.int32, device="cuda")
    cnt = torch.zeros(1, dtype=torch.int32, device="cuda")
    y = torch.empty(B, cfg.d, dtype=torch.float32, device="cuda")
    L.step(wl.to_torch(xb, cfg), idx, cnt, y)
    torch.cuda.synchronize()
    k = int(cnt.item())
    p, idx_or, logits = _oracle_layer_rows(cfg, layer, x64, rate)
    diff = check_table(idx.cpu().numpy(), k, idx_or, logits)
    sel = idx.cpu().numpy()[:k] if diff else idx_or
    y_or = _rows_y(cfg, layer, p, x64, sel)
    check_y(y.cpu().numpy(), y_or)
    assert L.last_device_error() == (sp.OK, 0)
    L.close()
    del dl, L
    torch.cuda.empty_cache()


def test_fullsize_true_mask_forward():
    """Config-3 shape with the mask taken from the true pre-activation (z > 0):
    forward over it reproduces the dense FFN."""
    cfg = wl.CONFIGS[3]
    layer, rate = 2, 0.05
    dl = wl.device_layer(cfg, layer, rate=rate)
    L = sp.Layer.from_device_layer(dl, max_batch=1)
    xb, x64 = x_tokens(cfg, 1, aux=31, layer=layer)
    h = wl.host_layer(cfg, layer, rate=rate)
    z = O.fc1_preactivation(h.f64("W1"), h.f64("b1"), x64)[0]
    truth = np.nonzero(z > 0)[0].astype(np.int32)
    assert 0.02 * cfg.n < truth.size < 0.09 * cfg.n
    y = torch.empty(1, cfg.d, dtype=torch.float32, device="cuda")
    L.forward(wl.to_torch(xb, cfg), torch.from_numpy(truth).cuda(),
              torch.tensor([truth.size], dtype=torch.int32, device="cuda"), y)
    yd = O.dense_ffn(h.f64("W1"), h.f64("b1"), h.f64("W2T"), None, x64)
    check_y(y.cpu().numpy(), yd)
    L.close()
    del dl, L, h
    torch.cuda.empty_cache()
