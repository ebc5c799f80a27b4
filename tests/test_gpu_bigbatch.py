"""Union tensor-core path at batch 48..256 (token groups of the split-activation
modes, chunked epilogue) vs the CPU oracle: union tables bit-exact outside the
near-threshold band, FFN outputs within the relative-L2 bar, caller tables, and
the unsupported-shape error for batches above 32 off the union path."""
import numpy as np
import pytest

import activation_sparse_ffn_predictor_b200 as sp
import oracle as O
import workload as wl
from _gpu import check_table, check_y, oracle_layer, torch_layer, x_tokens

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

CASES = {
    "f16-d1024-n4096-H256": wl.CONFIGS[0],
    "bf16-d512-n2048-H128": wl.FFNConfig("u-bf16", 1, 512, 2048, 128, "bf16", 1.0, 0.02),
}
_cache = {}


def setup(name, max_batch=256):
    if name not in _cache:
        cfg = CASES[name]
        h = wl.host_layer(cfg, 0)
        T = torch_layer(h)
        _cache[name] = (cfg, h, oracle_layer(h), T, sp.Layer(**T, max_batch=max_batch))
    return _cache[name]


@pytest.mark.parametrize("B", [48, 128, 130, 200, 256])
@pytest.mark.parametrize("name", list(CASES))
def test_bigbatch_step_parity(name, B):
    cfg, h, OL, T, L = setup(name)
    xb, x64 = x_tokens(cfg, B, aux=700 + B)
    idx = torch.full((cfg.n,), -5, dtype=torch.int32, device="cuda")
    cnt = torch.zeros(1, dtype=torch.int32, device="cuda")
    y = torch.empty(B, cfg.d, dtype=torch.float32, device="cuda")
    L.step(wl.to_torch(xb, cfg), idx, cnt, y)
    torch.cuda.synchronize()
    k = int(cnt.item())
    idx_or, k_or, logits = O.predict(OL["Wp1"], OL["Wp2"], OL["bp2"], x64, OL["bp1"])
    diff = check_table(idx.cpu().numpy(), k, idx_or, logits)
    sel = idx.cpu().numpy()[:k] if diff else idx_or
    y_or = O.sparse_ffn(OL["W1"], OL["b1"], OL["W2T"], OL["b2"], x64, sel)
    check_y(y.cpu().numpy(), y_or)
    assert L.last_device_error() == (sp.OK, 0)


@pytest.mark.parametrize("B", [64, 256])
def test_bigbatch_forward_caller_tables(B):
    cfg, h, OL, T, L = setup("f16-d1024-n4096-H256")
    xb, x64 = x_tokens(cfg, B, aux=800 + B)
    x = wl.to_torch(xb, cfg)
    r = np.random.default_rng(B)
    for tab in (np.arange(cfg.n), np.sort(r.choice(cfg.n, 333, replace=False)), np.array([cfg.n - 1])):
        idx = torch.from_numpy(np.ascontiguousarray(tab, dtype=np.int32)).cuda()
        cnt = torch.tensor([len(tab)], dtype=torch.int32, device="cuda")
        y = torch.empty(B, cfg.d, dtype=torch.float32, device="cuda")
        L.forward(x, idx, cnt, y)
        y_or = O.sparse_ffn(OL["W1"], OL["b1"], OL["W2T"], OL["b2"], x64, tab)
        check_y(y.cpu().numpy(), y_or)
    # the full table is the dense FFN
    y_dense = O.dense_ffn(OL["W1"], OL["b1"], OL["W2T"], OL["b2"], x64)
    idx = torch.arange(cfg.n, dtype=torch.int32, device="cuda")
    y = torch.empty(B, cfg.d, dtype=torch.float32, device="cuda")
    L.forward(x, idx, torch.tensor([cfg.n], dtype=torch.int32, device="cuda"), y)
    check_y(y.cpu().numpy(), y_dense)
    assert L.last_device_error() == (sp.OK, 0)


def test_bigbatch_is_deterministic():
    cfg, h, OL, T, L = setup("f16-d1024-n4096-H256")
    xb, _ = x_tokens(cfg, 200, aux=9)
    x = wl.to_torch(xb, cfg)
    outs = []
    for _ in range(2):
        idx = torch.empty(cfg.n, dtype=torch.int32, device="cuda")
        cnt = torch.zeros(1, dtype=torch.int32, device="cuda")
        y = torch.empty(200, cfg.d, dtype=torch.float32, device="cuda")
        L.step(x, idx, cnt, y)
        k = int(cnt.item())
        outs.append((y.cpu(), idx[:k].cpu()))
    assert all(torch.equal(a, b) for a, b in zip(outs[0], outs[1]))


def test_batch_above_32_needs_the_union_path():
    # d % 128 != 0: the union path does not apply, so B = 48 is unsupported (host-side check)
    cfg = wl.FFNConfig("rag", 1, 1088, 4128, 320, "f16", 1.0, 0.02)
    T = torch_layer(wl.host_layer(cfg, 0))
    L = sp.Layer(**T, max_batch=48)
    xb, _ = x_tokens(cfg, 48, aux=1)
    idx = torch.empty(cfg.n, dtype=torch.int32, device="cuda")
    cnt = torch.zeros(1, dtype=torch.int32, device="cuda")
    with pytest.raises(sp.SpffnError) as e:
        L.predict(wl.to_torch(xb, cfg), idx, cnt)
    assert e.value.status == sp.ERR_UNSUPPORTED
    # 32 tokens still run on the per-phase kernels
    L.predict(wl.to_torch(wl.tokens(cfg, 32, aux=2), cfg), idx, cnt)
    torch.cuda.synchronize()
    assert L.last_device_error() == (sp.OK, 0)


def _mixed_tables(n, seed):
    r = np.random.default_rng(seed)
    dense = np.arange(256, 512)                                          # two full blocks
    edge = 1024 + np.sort(r.choice(128, 64, replace=False))             # a block exactly half full
    below = 1280 + np.sort(r.choice(128, 63, replace=False))            # one member short of dense
    sparse = np.sort(r.choice(np.arange(2048, n), 300, replace=False))
    tab = np.concatenate([dense, edge, below, sparse])
    shuffled = r.permutation(tab)
    return tab, shuffled


@pytest.mark.parametrize("B", [16, 64])
def test_union_forward_dense_and_sparse_blocks(B):
    # tables mixing full, half-full and sparse 128-neuron blocks, in ascending and in
    # shuffled order (a table is a set): dense blocks load as 2-D tiles, the rest gathered
    cfg, h, OL, T, L = setup("f16-d1024-n4096-H256")
    xb, x64 = x_tokens(cfg, B, aux=900 + B)
    x = wl.to_torch(xb, cfg)
    tab, shuffled = _mixed_tables(cfg.n, B)
    y_or = O.sparse_ffn(OL["W1"], OL["b1"], OL["W2T"], OL["b2"], x64, np.sort(tab))
    for t in (tab, shuffled):
        idx = torch.from_numpy(np.ascontiguousarray(t, dtype=np.int32)).cuda()
        cnt = torch.tensor([len(t)], dtype=torch.int32, device="cuda")
        y = torch.empty(B, cfg.d, dtype=torch.float32, device="cuda")
        L.forward(x, idx, cnt, y)
        check_y(y.cpu().numpy(), y_or)
    assert L.last_device_error() == (sp.OK, 0)
