"""Union-mask tensor-core path (batch 16..32) vs the CPU oracle: predictor
GEMMs, union table, FC1/FC2 over gathered rows."""
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
    "bf16-d512-n2048-H128": wl.FFNConfig("u-bf16", 1, 512, 2048, 128, "bf16", 1.0, 0.05),
    "f16-d1024-n4128-H320-ragged": wl.FFNConfig("u-rag", 1, 1024, 4128, 320, "f16", 1.0, 0.02),
}
_cache = {}


def setup(name, B):
    if (name, B) not in _cache:
        cfg = CASES[name]
        h = wl.host_layer(cfg, 0)
        T = torch_layer(h)
        _cache[(name, B)] = (cfg, h, oracle_layer(h), T, sp.Layer(**T, max_batch=B))
    return _cache[(name, B)]


@pytest.mark.parametrize("B", [16, 20, 32])
@pytest.mark.parametrize("name", list(CASES))
def test_union_step_parity(name, B):
    cfg, h, OL, T, L = setup(name, B)
    xb, x64 = x_tokens(cfg, B, aux=500 + B)
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


@pytest.mark.parametrize("B", [16, 32])
def test_union_forward_tables(B):
    cfg, h, OL, T, L = setup("f16-d1024-n4096-H256", B)
    xb, x64 = x_tokens(cfg, B, aux=600 + B)
    x = wl.to_torch(xb, cfg)
    z = O.fc1_preactivation(OL["W1"], OL["b1"], x64)
    truth = np.nonzero(np.any(z > 0, axis=0))[0]
    r = np.random.default_rng(B)
    for tab in (truth, np.sort(r.choice(cfg.n, 77, replace=False)), np.arange(cfg.n), np.array([5])):
        idx = torch.from_numpy(np.ascontiguousarray(tab, dtype=np.int32)).cuda()
        cnt = torch.tensor([len(tab)], dtype=torch.int32, device="cuda")
        y = torch.empty(B, cfg.d, dtype=torch.float32, device="cuda")
        L.forward(x, idx, cnt, y)
        y_or = O.sparse_ffn(OL["W1"], OL["b1"], OL["W2T"], OL["b2"], x64, tab)
        check_y(y.cpu().numpy(), y_or)
    # empty table: y = b2 (zero here)
    y = torch.full((B, cfg.d), 7.0, dtype=torch.float32, device="cuda")
    L.forward(x, idx, torch.tensor([0], dtype=torch.int32, device="cuda"), y)
    assert torch.count_nonzero(y).item() == 0
    assert L.last_device_error() == (sp.OK, 0)


def test_union_is_deterministic():
    cfg, h, OL, T, L = setup("f16-d1024-n4096-H256", 32)
    xb, _ = x_tokens(cfg, 32, aux=9)
    x = wl.to_torch(xb, cfg)
    outs = []
    for _ in range(3):
        idx = torch.empty(cfg.n, dtype=torch.int32, device="cuda")
        cnt = torch.zeros(1, dtype=torch.int32, device="cuda")
        y = torch.empty(32, cfg.d, dtype=torch.float32, device="cuda")
        L.step(x, idx, cnt, y)
        k = int(cnt.item())
        outs.append((y.cpu(), idx[:k].cpu(), cnt.cpu()))   # entries past the count are not written
    for o in outs[1:]:
        assert all(torch.equal(a, b) for a, b in zip(outs[0], o))


def test_union_edge_cases_empty_clamped_and_out_of_range():
    cfg, h, OL, T, L = setup("f16-d1024-n4096-H256", 16)
    xb, x64 = x_tokens(cfg, 16, aux=31)
    x = wl.to_torch(xb, cfg)
    y = torch.empty(16, cfg.d, dtype=torch.float32, device="cuda")
    idx = torch.arange(cfg.n, dtype=torch.int32, device="cuda")
    L.last_device_error()
    # empty table: y = b2 (zero here), no error
    L.forward(x, idx, torch.tensor([0], dtype=torch.int32, device="cuda"), y)
    assert torch.count_nonzero(y).item() == 0
    assert L.last_device_error() == (sp.OK, 0)
    # count > n: clamped to n (the dense FFN), latched
    L.forward(x, idx, torch.tensor([cfg.n + 9], dtype=torch.int32, device="cuda"), y)
    yd = O.dense_ffn(OL["W1"], OL["b1"], OL["W2T"], OL["b2"], x64)
    check_y(y.cpu().numpy(), yd)
    s, code = L.last_device_error()
    assert s == sp.ERR_DEVICE_CHECK and code & 1
    # out-of-range entries are skipped and latched
    bad = torch.tensor([3, cfg.n + 4, 7, -1, 9], dtype=torch.int32, device="cuda")
    L.forward(x, bad, torch.tensor([5], dtype=torch.int32, device="cuda"), y)
    y_or = O.sparse_ffn(OL["W1"], OL["b1"], OL["W2T"], OL["b2"], x64, [3, 7, 9])
    check_y(y.cpu().numpy(), y_or)
    s, code = L.last_device_error()
    assert s == sp.ERR_DEVICE_CHECK and code & 2
    assert L.last_device_error() == (sp.OK, 0)
