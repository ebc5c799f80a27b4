"""Whole-stack decode, plain (spffn_decode) and with look-ahead prediction
(spffn_decode_lookahead, DejaVu appendix equation (-2) of "LLM模型之PowerInfer1.0"),
against the oracle chaining its own layer inputs: every layer's neuron table
(bit-exact outside the near-threshold band) and count, the last layer's y and
the final x.  Where a table differs from the oracle's only inside that band the
oracle continues on the GPU's table, so every layer is compared on every seed.
Covers the persistent kernel (B <= 2), the per-layer path (B = 3) and the union
tensor-core path (B = 16, 64 and 200)."""
import pytest

import activation_sparse_ffn_predictor_b200 as sp
import workload as wl
from _gpu import HostOracle, check_stack, prefix_runner, torch_layer, x_tokens

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

CASES = {
    "block-d1024-n4096-L4": (wl.CONFIGS[0], 4),
    "ragged-bf16-d1088-n4128-H320-L3": (wl.FFNConfig("ragged", 1, 1088, 4128, 320, "bf16", 1.0, 0.2), 3),
    "tiny-d64-n32-H64-L3": (wl.FFNConfig("tiny", 1, 64, 32, 64, "f16", 1.2, 0.3), 3),
    "wide-d10240-n2048-H64-L2": (wl.FFNConfig("wide", 1, 10240, 2048, 64, "f16", 1.2, 0.1), 2),
    "bigH-d512-n1024-H8192-L2": (wl.FFNConfig("bigH", 1, 512, 1024, 8192, "bf16", 1.0, 0.1), 2),
}


def run_and_check(cfg, Lc, B, aux, lookahead, max_batch=None):
    hs = [wl.host_layer(cfg, l) for l in range(Lc)]
    layers = [sp.Layer(**torch_layer(h), max_batch=max_batch or B) for h in hs]
    xb, x64 = x_tokens(cfg, B, aux=aux)
    dt = torch.bfloat16 if cfg.bf16 else torch.float16
    x_out = torch.empty(B, cfg.d, dtype=dt, device="cuda")
    y = torch.empty(B, cfg.d, dtype=torch.float32, device="cuda")
    counts = torch.full((Lc,), -1, dtype=torch.int32, device="cuda")
    x_in = wl.to_torch(xb, cfg)
    sp.decode(layers, x_in, x_out, y, counts, lookahead=lookahead)
    torch.cuda.synchronize()
    for L in layers:
        assert L.last_device_error() == (sp.OK, 0)
    kc = counts.cpu().numpy()
    check_stack(layers, [HostOracle(h) for h in hs], cfg, x64, y, x_out, counts, lookahead=lookahead,
                run_prefix=prefix_runner(layers, x_in, cfg, lookahead))
    return kc


@pytest.mark.parametrize("lookahead", [False, True])
@pytest.mark.parametrize("B", [1, 2, 3])
@pytest.mark.parametrize("name", list(CASES))
def test_decode_tables_match_oracle(name, B, lookahead):
    cfg, Lc = CASES[name]
    run_and_check(cfg, Lc, B, aux=500 + B, lookahead=lookahead)


@pytest.mark.parametrize("B", [16, 64, 200])
@pytest.mark.parametrize("lookahead", [False, True])
def test_union_decode_tables_match_oracle(lookahead, B):
    run_and_check(wl.CONFIGS[0], 3, B, aux=516 + B, lookahead=lookahead, max_batch=B)


def test_lookahead_changes_the_sets():
    # the two modes agree on layer 0 and (for this seed) differ on a later layer
    cfg, Lc = CASES["block-d1024-n4096-L4"]
    k_std = run_and_check(cfg, Lc, 1, aux=9, lookahead=False)
    k_la = run_and_check(cfg, Lc, 1, aux=9, lookahead=True)
    assert k_std[0] == k_la[0]
    assert any(k_std[l] != k_la[l] for l in range(1, Lc))


def test_lookahead_decode_in_cuda_graph_is_repeatable():
    cfg, Lc = CASES["block-d1024-n4096-L4"]
    hs = [wl.host_layer(cfg, l) for l in range(Lc)]
    layers = [sp.Layer(**torch_layer(h), max_batch=1) for h in hs]
    x_in = torch.empty(1, cfg.d, dtype=torch.float16, device="cuda")
    x_out = torch.empty_like(x_in)
    y = torch.empty(1, cfg.d, dtype=torch.float32, device="cuda")
    counts = torch.zeros(Lc, dtype=torch.int32, device="cuda")
    s = torch.cuda.Stream()
    x_in.copy_(wl.to_torch(wl.tokens(cfg, 1, aux=3), cfg))
    with torch.cuda.stream(s):
        sp.decode(layers, x_in, x_out, y, counts, stream=s, lookahead=True)
    s.synchronize()
    first = (y.cpu(), x_out.cpu(), counts.cpu())
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        sp.decode(layers, x_in, x_out, y, counts, stream=s, lookahead=True)
    for _ in range(2):
        g.replay()
        torch.cuda.synchronize()
        assert all(torch.equal(a, b) for a, b in zip(first, (y.cpu(), x_out.cpu(), counts.cpu())))
    del g
