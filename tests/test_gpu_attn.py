"""Head-sparse attention decode with the attention-head predictor (DejaVu's
SP_A, equation (-1) of the DejaVu appendix in "LLM模型之PowerInfer1.0") against
the oracle, step by step over a token sequence:

* the selected heads: bit-exact (ascending) outside the 1e-4 logit band;
* the cache after the step: the stored token, which rows exist (a selected head
  gets every missing row up to the new position, a skipped head gets none) and
  each row's K/V values within 1 ulp of the oracle's (both round a dot product
  to the storage dtype, from fp32 and fp64);
* the step's output: per token within the contract and within the internal bar
  of the oracle's attention over the GPU's validated cache rows.
Plus: a full cache, CUDA-graph replay, reset, and the OPT-66B attention shape."""
import numpy as np
import pytest

import activation_sparse_ffn_predictor_b200 as sp
import oracle.attention as A
import workload as wl
from _gpu import LOGIT_BAND, check_y, ulp_of

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

CASES = {
    "d1024-h16-dh64": wl.ATTN_CONFIGS[0],
    "bf16-d512-h8-dh48-Ha128": wl.AttnConfig("a-bf16", 1, 512, 8, 48, 128, "bf16", 0.4, 0, 24),
    "d256-h6-dh8": wl.AttnConfig("a-tiny", 1, 256, 6, 8, 64, "f16", 0.5, 0, 12),
}


def make_layer(cfg, h):
    T = lambda a: wl.to_torch(a, cfg)
    return sp.AttnLayer(T(h.Wq), T(h.Wk), T(h.Wv), T(h.WoT), T(h.Wa1), T(h.Wa2), nh=cfg.nh, tmax=cfg.tmax,
                        ba2=T(h.ba2))


def round_kv(cfg):
    return lambda a: wl.widen(wl.round_to(np.asarray(a, dtype=np.float64), cfg.bf16), cfg.bf16)


def oracle_weights(h):
    return dict(Wq=h.f64("Wq"), Wk=h.f64("Wk"), Wv=h.f64("Wv"), Wo=h.f64("WoT").T, bq=None, bk=None, bv=None,
                bo=None)


def bits(t):
    return t.detach().cpu().view(torch.int16).numpy().view(np.uint16)


def run_and_check(cfg, steps, aux):
    h = wl.host_attn(cfg, 0)
    layer = make_layer(cfg, h)
    Wt = oracle_weights(h)
    Wa1, Wa2, ba2 = h.f64("Wa1"), h.f64("Wa2"), h.f64("ba2")
    cache = A.KVCache(cfg.nh, cfg.dh, cfg.d, cfg.tmax, round_kv(cfg))
    Yb = wl.attn_tokens(cfg, steps, aux=aux)
    heads = torch.full((cfg.nh,), -1, dtype=torch.int32, device="cuda")
    count = torch.full((1,), -1, dtype=torch.int32, device="cuda")
    out = torch.empty(cfg.d, dtype=torch.float32, device="cuda")
    seen_counts = []
    for t in range(steps):
        y64 = wl.widen(Yb[t], cfg.bf16)
        layer.step(wl.to_torch(Yb[t], cfg), heads, count, out)
        torch.cuda.synchronize()
        k = int(count.item())
        got = heads[:k].cpu().numpy()
        assert np.all(np.diff(got) > 0)
        logits = A.head_logits(Wa1, Wa2, y64, None, ba2)[0]
        want = A.selected_heads(logits)
        band = set(np.nonzero(np.abs(logits) < LOGIT_BAND)[0].tolist())
        assert set(got.tolist()) ^ set(want.tolist()) <= band, (t, got, want)
        seen_counts.append(k)
        # the oracle's own cache step on the heads the GPU used (a valid answer)
        A.mha_sparse_step(Wt, cache, y64, got)
        K, V, filled, Yc, tt = layer.cache()
        assert int(tt.item()) == t + 1
        assert np.array_equal(filled.cpu().numpy()[:, :t + 1].astype(bool), cache.filled[:, :t + 1])
        assert np.array_equal(bits(Yc[t]), Yb[t])
        Kg = wl.widen(bits(K), cfg.bf16)
        Vg = wl.widen(bits(V), cfg.bf16)
        for hh in got.tolist():
            for G_, O_ in ((Kg, cache.K), (Vg, cache.V)):
                gv, ov = G_[hh, :t + 1], O_[hh, :t + 1]
                assert np.all(np.abs(gv - ov) <= ulp_of(ov, cfg.bf16) + 1e-5), (t, hh)
        # the step's output from the GPU's validated rows
        want_out = np.zeros(cfg.d)
        for hh in got.tolist():
            q = A.head_rows(Wt["Wq"], None, hh, cfg.dh, y64)
            o = A.attend(q, Kg[hh, :t + 1], Vg[hh, :t + 1])
            want_out += Wt["Wo"][:, hh * cfg.dh:(hh + 1) * cfg.dh] @ o
        if k == 0:
            assert np.array_equal(out.cpu().numpy(), np.zeros(cfg.d, dtype=np.float32))
        else:
            check_y(out.cpu().numpy()[None, :], want_out[None, :])
    assert layer.last_device_error() == (sp.OK, 0)
    return layer, seen_counts


@pytest.mark.parametrize("name", list(CASES))
def test_attn_sequence_matches_oracle(name):
    cfg = CASES[name]
    layer, ks = run_and_check(cfg, min(cfg.tmax, 20), aux=31)
    # the sequence exercised both skipped heads and lazily filled ones
    assert 0 < sum(ks) < cfg.nh * len(ks)


def test_attn_full_cache_latches_and_writes_bias():
    cfg = CASES["d256-h6-dh8"]
    h = wl.host_attn(cfg, 0)
    layer = make_layer(cfg, h)
    Yb = wl.attn_tokens(cfg, cfg.tmax + 1, aux=5)
    heads = torch.zeros(cfg.nh, dtype=torch.int32, device="cuda")
    count = torch.zeros(1, dtype=torch.int32, device="cuda")
    out = torch.empty(cfg.d, dtype=torch.float32, device="cuda")
    for t in range(cfg.tmax):
        layer.step(wl.to_torch(Yb[t], cfg), heads, count, out)
    torch.cuda.synchronize()
    assert layer.last_device_error() == (sp.OK, 0)
    layer.step(wl.to_torch(Yb[cfg.tmax], cfg), heads, count, out)
    torch.cuda.synchronize()
    assert int(count.item()) == 0
    assert np.array_equal(out.cpu().numpy(), np.zeros(cfg.d, dtype=np.float32))
    assert int(layer.cache()[4].item()) == cfg.tmax
    s, code = layer.last_device_error()
    assert s == sp.ERR_DEVICE_CHECK and code & (1 << 4)


def test_attn_graph_replay_and_reset_are_bitwise_repeatable():
    cfg = CASES["d1024-h16-dh64"]
    steps = 10
    h = wl.host_attn(cfg, 0)
    Yb = wl.attn_tokens(cfg, steps, aux=77)
    y_in = torch.empty(cfg.d, dtype=torch.float16, device="cuda")
    heads = torch.zeros(cfg.nh, dtype=torch.int32, device="cuda")
    count = torch.zeros(1, dtype=torch.int32, device="cuda")
    out = torch.empty(cfg.d, dtype=torch.float32, device="cuda")
    # eager reference
    layer = make_layer(cfg, h)
    ref = []
    for t in range(steps):
        y_in.copy_(wl.to_torch(Yb[t], cfg))
        layer.step(y_in, heads, count, out)
        ref.append((out.cpu().numpy().copy(), int(count.item())))
    # after a reset the same steps give the same bits, through one captured graph
    s = torch.cuda.Stream()
    layer.reset(stream=s)
    s.synchronize()
    assert int(layer.cache()[4].item()) == 0 and int(layer.cache()[2].sum().item()) == 0
    y_in.copy_(wl.to_torch(Yb[0], cfg))
    with torch.cuda.stream(s):
        layer.step(y_in, heads, count, out, stream=s)         # step 0, eager (also warms up)
    s.synchronize()
    assert np.array_equal(out.cpu().numpy(), ref[0][0])
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        layer.step(y_in, heads, count, out, stream=s)
    # capture does not run the step: the cache still holds one token
    assert int(layer.cache()[4].item()) == 1
    for t in range(1, steps):
        y_in.copy_(wl.to_torch(Yb[t], cfg))
        g.replay()
        torch.cuda.synchronize()
        assert int(count.item()) == ref[t][1]
        assert np.array_equal(out.cpu().numpy(), ref[t][0]), t
    assert layer.last_device_error() == (sp.OK, 0)
    del g


def test_attn_launch_count():
    assert sp.attn_step_kernel_launches() == 5


def test_attn_opt66b_shape():
    """The OPT-66B attention shape (72 heads of 128, d = 9216, predictor 1024)."""
    cfg = wl.ATTN_CONFIGS[1].with_(tmax=16)
    run_and_check(cfg, 8, aux=3)
    torch.cuda.empty_cache()
