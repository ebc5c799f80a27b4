"""Whole-stack decode (spffn_decode, the launch the bench times) vs the oracle
chaining its layer inputs: every layer's neuron table and count, the last
layer's y and the final x (the oracle continues on the GPU's table where the two
differ only inside the near-threshold band)."""
import pytest

import activation_sparse_ffn_predictor_b200 as sp
import workload as wl
from _gpu import HostOracle, check_stack, prefix_runner, torch_layer, x_tokens

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

CASES = {
    "block-d1024-n4096-L4": (wl.CONFIGS[0], 4),
    "ragged-bf16-d1088-n4128-H320-L3": (wl.FFNConfig("ragged", 1, 1088, 4128, 320, "bf16", 1.0, 0.2), 3),
    "tiny-d64-n32-H64-L2": (wl.FFNConfig("tiny", 1, 64, 32, 64, "f16", 1.2, 0.3), 2),
    "wide-d10240-n2048-H64-L2": (wl.FFNConfig("wide", 1, 10240, 2048, 64, "f16", 1.2, 0.1), 2),
    "bigH-d512-n1024-H8192-L2": (wl.FFNConfig("bigH", 1, 512, 1024, 8192, "bf16", 1.0, 0.1), 2),
}


def run_case(cfg, Lc, B, aux):
    hs = [wl.host_layer(cfg, l) for l in range(Lc)]
    Ts = [torch_layer(h) for h in hs]
    layers = [sp.Layer(**T, max_batch=B) for T in Ts]
    xb, x64 = x_tokens(cfg, B, aux=aux)
    dt = torch.bfloat16 if cfg.bf16 else torch.float16
    x_out = torch.empty(B, cfg.d, dtype=dt, device="cuda")
    y = torch.empty(B, cfg.d, dtype=torch.float32, device="cuda")
    counts = torch.full((Lc,), -1, dtype=torch.int32, device="cuda")
    x_in = wl.to_torch(xb, cfg)
    sp.decode(layers, x_in, x_out, y, counts)
    torch.cuda.synchronize()
    return hs, layers, x64, x_in, x_out, y, counts


@pytest.mark.parametrize("B", [1, 2, 3])
@pytest.mark.parametrize("name", list(CASES))
def test_decode_matches_oracle_chain(name, B):
    cfg, Lc = CASES[name]
    hs, layers, x64, x_in, x_out, y, counts = run_case(cfg, Lc, B, aux=300 + B)
    for L in layers:
        assert L.last_device_error() == (sp.OK, 0)
    check_stack(layers, [HostOracle(h) for h in hs], cfg, x64, y, x_out, counts,
                run_prefix=prefix_runner(layers, x_in, cfg))


def test_decode_is_deterministic_and_repeatable():
    cfg, Lc = CASES["block-d1024-n4096-L4"]
    outs = []
    for _ in range(2):
        hs, layers, x64, x_in, x_out, y, counts = run_case(cfg, Lc, 1, aux=77)
        outs.append((x_out.cpu(), y.cpu(), counts.cpu()))
    assert all(torch.equal(a, b) for a, b in zip(outs[0], outs[1]))


def test_decode_in_cuda_graph_replays():
    cfg, Lc = CASES["block-d1024-n4096-L4"]
    hs = [wl.host_layer(cfg, l) for l in range(Lc)]
    layers = [sp.Layer(**torch_layer(h), max_batch=1) for h in hs]
    x_in = torch.empty(1, cfg.d, dtype=torch.float16, device="cuda")
    x_out = torch.empty_like(x_in)
    y = torch.empty(1, cfg.d, dtype=torch.float32, device="cuda")
    counts = torch.zeros(Lc, dtype=torch.int32, device="cuda")
    s = torch.cuda.Stream()
    x_in.copy_(wl.to_torch(wl.tokens(cfg, 1, aux=1), cfg))
    with torch.cuda.stream(s):
        sp.decode(layers, x_in, x_out, y, counts, stream=s)
    s.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        sp.decode(layers, x_in, x_out, y, counts, stream=s)
    ref = {}
    for aux in (1, 2, 1):
        x_in.copy_(wl.to_torch(wl.tokens(cfg, 1, aux=aux), cfg))
        g.replay()
        torch.cuda.synchronize()
        if aux in ref:
            assert torch.equal(ref[aux], y.cpu())
        ref[aux] = y.cpu()
    assert not torch.equal(ref[1], ref[2])
    del g
