"""CUDA library vs the CPU oracle on the same seeded inputs (needs a B200).

Neuron tables must agree bit-exactly except for neurons whose oracle logit is
within 1e-4 of the threshold; FFN outputs within relative L2 1e-3."""
import numpy as np
import pytest

import activation_sparse_ffn_predictor_b200 as sp
import oracle as O
import workload as wl
from _gpu import REL_L2_BAR, check_table, check_y, oracle_layer, rel_l2, torch_layer, x_tokens

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

# Sizes the oracle finishes in seconds that still span several tiles and a ragged tail.
SMALL = {
    "block-d1024-n4096": wl.CONFIGS[0],
    "ragged-bf16-d1088-n4128-H320": wl.FFNConfig("ragged", 1, 1088, 4128, 320, "bf16", 1.0, 0.2),
    "bf16-d512-n2048-H128": wl.FFNConfig("small-bf16", 1, 512, 2048, 128, "bf16", 1.0, 0.05),
    "tiny-d64-n32-H64": wl.FFNConfig("tiny", 1, 64, 32, 64, "f16", 1.2, 0.3),
}

_cache = {}


def setup(name, B, layer=0):
    key = (name, B, layer)
    if key not in _cache:
        cfg = SMALL[name]
        h = wl.host_layer(cfg, layer)
        T = torch_layer(h)
        L = sp.Layer(**T, max_batch=B)
        _cache[key] = (cfg, h, oracle_layer(h), T, L)
    return _cache[key]


@pytest.mark.parametrize("B", [1, 3, 8, 16, 32])
@pytest.mark.parametrize("name", list(SMALL))
def test_predict_and_step_parity(name, B):
    cfg, h, OL, T, L = setup(name, B)
    xb, x64 = x_tokens(cfg, B, aux=100 + B)
    x = wl.to_torch(xb, cfg)
    idx = torch.full((cfg.n,), -7, dtype=torch.int32, device="cuda")
    cnt = torch.zeros(1, dtype=torch.int32, device="cuda")
    y = torch.empty(B, cfg.d, dtype=torch.float32, device="cuda")
    L.step(x, idx, cnt, y)
    torch.cuda.synchronize()
    k = int(cnt.item())
    idx_or, k_or, logits = O.predict(OL["Wp1"], OL["Wp2"], OL["bp2"], x64, OL["bp1"])
    diff = check_table(idx.cpu().numpy(), k, idx_or, logits)
    # the GPU's table is a valid answer; the oracle computes y for it
    sel = np.asarray(idx.cpu().numpy()[:k]) if diff else idx_or
    y_or = O.sparse_ffn(OL["W1"], OL["b1"], OL["W2T"], OL["b2"], x64, sel)
    check_y(y.cpu().numpy(), y_or)
    assert L.last_device_error() == (sp.OK, 0)


@pytest.mark.parametrize("B", [1, 5, 32])
@pytest.mark.parametrize("name", ["block-d1024-n4096", "ragged-bf16-d1088-n4128-H320"])
def test_forward_given_table(name, B):
    """forward() on tables the oracle chooses: its own prediction, the true
    positive set (reproduces the dense FFN), a shuffled random subset."""
    cfg, h, OL, T, L = setup(name, B)
    xb, x64 = x_tokens(cfg, B, aux=200 + B)
    x = wl.to_torch(xb, cfg)
    z = O.fc1_preactivation(OL["W1"], OL["b1"], x64)
    truth = np.nonzero(np.any(z > 0, axis=0))[0]
    r = np.random.default_rng(B)
    rand = r.permutation(np.nonzero(r.random(cfg.n) < 0.3)[0])
    tables = {"true-mask": truth, "random-shuffled": rand, "all": np.arange(cfg.n)}
    for tag, tab in tables.items():
        idx = torch.from_numpy(np.ascontiguousarray(tab, dtype=np.int32)).cuda()
        cnt = torch.tensor([len(tab)], dtype=torch.int32, device="cuda")
        y = torch.empty(B, cfg.d, dtype=torch.float32, device="cuda")
        L.forward(x, idx, cnt, y)
        y_or = O.sparse_ffn(OL["W1"], OL["b1"], OL["W2T"], OL["b2"], x64, tab)
        check_y(y.cpu().numpy(), y_or)
        if tag in ("true-mask", "all"):
            yd = O.dense_ffn(OL["W1"], OL["b1"], OL["W2T"], OL["b2"], x64)
            check_y(y.cpu().numpy(), yd)


def test_forward_is_deterministic():
    cfg, h, OL, T, L = setup("block-d1024-n4096", 8)
    xb, _ = x_tokens(cfg, 8, aux=7)
    x = wl.to_torch(xb, cfg)
    idx = torch.arange(0, cfg.n, 3, dtype=torch.int32, device="cuda")
    cnt = torch.tensor([idx.numel()], dtype=torch.int32, device="cuda")
    ys = []
    for _ in range(3):
        y = torch.empty(8, cfg.d, dtype=torch.float32, device="cuda")
        L.forward(x, idx, cnt, y)
        ys.append(y.cpu())
    assert torch.equal(ys[0], ys[1]) and torch.equal(ys[1], ys[2])


def test_edge_cases_empty_clamped_and_out_of_range():
    cfg = SMALL["tiny-d64-n32-H64"]
    h = wl.host_layer(cfg, 0)
    h.b2 = wl.round_to(np.linspace(-1, 1, cfg.d), 0)      # non-zero FC2 bias
    OL = oracle_layer(h)
    T = torch_layer(h)
    L = sp.Layer(**T, max_batch=2)
    xb, x64 = x_tokens(cfg, 2, aux=3)
    x = wl.to_torch(xb, cfg)
    y = torch.empty(2, cfg.d, dtype=torch.float32, device="cuda")
    idx = torch.arange(cfg.n, dtype=torch.int32, device="cuda")
    # empty table: y = b2 exactly, no error
    L.forward(x, idx, torch.tensor([0], dtype=torch.int32, device="cuda"), y)
    assert np.array_equal(y.cpu().numpy(), np.tile(OL["b2"].astype(np.float32), (2, 1)))
    assert L.last_device_error() == (sp.OK, 0)
    # count > n: clamped to n (the dense FFN), latched
    L.forward(x, idx, torch.tensor([cfg.n + 9], dtype=torch.int32, device="cuda"), y)
    yd = O.dense_ffn(OL["W1"], OL["b1"], OL["W2T"], OL["b2"], x64)
    check_y(y.cpu().numpy(), yd)
    s, code = L.last_device_error()
    assert s == sp.ERR_DEVICE_CHECK and code & 1
    # negative count: clamped to 0
    L.forward(x, idx, torch.tensor([-4], dtype=torch.int32, device="cuda"), y)
    assert np.array_equal(y.cpu().numpy(), np.tile(OL["b2"].astype(np.float32), (2, 1)))
    assert L.last_device_error()[0] == sp.ERR_DEVICE_CHECK
    # out-of-range entries are skipped and latched
    bad = torch.tensor([3, 40, 7, -1, 9], dtype=torch.int32, device="cuda")
    L.forward(x, bad, torch.tensor([5], dtype=torch.int32, device="cuda"), y)
    y_or = O.sparse_ffn(OL["W1"], OL["b1"], OL["W2T"], OL["b2"], x64, [3, 7, 9])
    check_y(y.cpu().numpy(), y_or)
    s, code = L.last_device_error()
    assert s == sp.ERR_DEVICE_CHECK and code & 2
    assert L.last_device_error() == (sp.OK, 0)      # reading clears it


@pytest.mark.parametrize("dtype", ["f16", "bf16"])
def test_chain_parity(dtype):
    cfg = wl.FFNConfig("c", 1, 1088, 64, 64, dtype, 1.0, 0.1)
    h = wl.host_layer(cfg, 0)
    L = sp.Layer(**torch_layer(h), max_batch=4)
    xb, x64 = x_tokens(cfg, 4, aux=11)
    y64 = wl.float_tokens(cfg, 4, aux=12).astype(np.float64)
    xn = torch.empty(4, cfg.d, dtype=torch.bfloat16 if cfg.bf16 else torch.float16, device="cuda")
    L.chain(wl.to_torch(xb, cfg), torch.from_numpy(y64.astype(np.float32)).cuda(), xn)
    want = wl.round_to(O.chain(x64, y64), cfg.bf16)
    got = xn.cpu().view(torch.int16).numpy().view(np.uint16)
    ulps = np.abs(got.astype(np.int32) - want.astype(np.int32))
    assert ulps.max() <= 1 and (ulps > 0).mean() < 0.01
    assert rel_l2(wl.widen(got, cfg.bf16), wl.widen(want, cfg.bf16)) <= REL_L2_BAR


def test_profile_counts_and_permutation():
    cfg = SMALL["block-d1024-n4096"]
    cfg_, h, OL, T, L = setup("block-d1024-n4096", 1)
    Xb = wl.tokens(cfg, 300, aux=5, tensor=wl.T_XPROF)
    X64 = wl.widen(Xb, cfg.bf16)
    counts = torch.zeros(cfg.n, dtype=torch.int32, device="cuda")
    L.profile_counts(wl.to_torch(Xb[:200], cfg), counts)
    L.profile_counts(wl.to_torch(Xb[200:], cfg), counts)     # accumulates
    got = counts.cpu().numpy().astype(np.int64)
    want = O.activation_counts(OL["W1"], OL["b1"], X64).astype(np.int64)
    z = O.fc1_preactivation(OL["W1"], OL["b1"], X64)
    slack = (np.abs(z) < 1e-4).sum(axis=0)
    assert np.all(np.abs(got - want) <= slack)
    assert got.sum() > 0
    perm = O.hot_first_order(want)
    assert np.array_equal(sp.reorder(want.astype(np.uint32)), perm)
    pt = torch.from_numpy(perm).cuda()
    dst = torch.empty_like(T["W1"])
    sp.permute_rows(T["W1"], dst, pt)
    assert torch.equal(dst.cpu(), T["W1"].cpu()[torch.from_numpy(perm).long()])
    vb = torch.empty_like(T["b1"])
    sp.permute_vector(T["b1"], vb, pt)
    assert torch.equal(vb.cpu(), T["b1"].cpu()[torch.from_numpy(perm).long()])


def test_reordered_layer_gives_same_output():
    """Hot-first placement changes only where neurons sit: outputs agree, and
    the table maps back through perm."""
    cfg, h, OL, T, L = setup("block-d1024-n4096", 1)
    X64 = wl.widen(wl.tokens(cfg, 256, aux=9, tensor=wl.T_XPROF), 0)
    perm = O.hot_first_order(O.activation_counts(OL["W1"], OL["b1"], X64))
    pt = torch.from_numpy(perm).cuda()
    P = {}
    for k in ("W1", "W2T", "Wp2"):
        P[k] = torch.empty_like(T[k])
        sp.permute_rows(T[k], P[k], pt)
    for k in ("b1", "bp2"):
        P[k] = torch.empty_like(T[k])
        sp.permute_vector(T[k], P[k], pt)
    for k in ("b2", "Wp1", "bp1"):
        P[k] = T[k]
    LP = sp.Layer(**P, max_batch=1)
    xb, x64 = x_tokens(cfg, 1, aux=77)
    x = wl.to_torch(xb, cfg)
    outs = []
    for lay in (L, LP):
        idx = torch.empty(cfg.n, dtype=torch.int32, device="cuda")
        cnt = torch.zeros(1, dtype=torch.int32, device="cuda")
        y = torch.empty(1, cfg.d, dtype=torch.float32, device="cuda")
        lay.step(x, idx, cnt, y)
        outs.append((idx.cpu().numpy()[:int(cnt.item())], y.cpu().numpy()))
    assert sorted(perm[outs[1][0]].tolist()) == outs[0][0].tolist()
    assert rel_l2(outs[1][1], outs[0][1]) <= 1e-5
    # hot slots come first: the reordered table is concentrated at low slots
    assert np.median(outs[1][0]) < np.median(outs[0][0])
