"""The persistent union-path decode: one launch for the whole stack at
3 <= B <= 128 (below 16 the MMA's columns are padded), against the oracle layer by layer (every layer's neuron table
bit-exact outside the near-threshold band and its count, the last y, the final
x).  Shapes cover a ragged last tile in every phase (n and H not multiples of
128, B not a multiple of 16) in fp16 and bf16, a context sized for a larger
batch than the call uses, an empty neuron set, and bitwise-repeatable CUDA
graph replays."""
import numpy as np
import pytest

import activation_sparse_ffn_predictor_b200 as sp
import workload as wl
from _gpu import HostOracle, bits_of, check_stack, prefix_runner, torch_layer, x_tokens

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

@pytest.fixture(autouse=True)
def whole_stack_mode():
    """These tests run the whole-stack kernel at every batch it serves (the
    default dispatch uses per-layer launches)."""
    sp.set_union_stack(sp.UNION_STACK)
    yield
    sp.set_union_stack(sp.UNION_AUTO)


CASES = {
    "block-d1024-n4096-H256-L3": (wl.CONFIGS[0], 3),
    "ragged-bf16-d1152-n4128-H320-L3": (wl.FFNConfig("uragged", 1, 1152, 4128, 320, "bf16", 1.0, 0.1), 3),
    # one layer: the kernel's y against the oracle on the same input (internal bar 1e-5)
    "ragged-bf16-d1152-n4128-H320-L1": (wl.FFNConfig("uragged", 1, 1152, 4128, 320, "bf16", 1.0, 0.1), 1),
    "block-d1024-n4096-H256-L1": (wl.CONFIGS[0], 1),
}


def run(cfg, hs, B, aux, max_batch=None):
    layers = [sp.Layer(**torch_layer(h), max_batch=max_batch or B) for h in hs]
    assert sp.decode_kernel_launches(layers, B) == 1          # the whole stack in one launch
    xb, x64 = x_tokens(cfg, B, aux=aux)
    dt = torch.bfloat16 if cfg.bf16 else torch.float16
    x_out = torch.empty(B, cfg.d, dtype=dt, device="cuda")
    y = torch.empty(B, cfg.d, dtype=torch.float32, device="cuda")
    counts = torch.full((len(hs),), -1, dtype=torch.int32, device="cuda")
    x_in = wl.to_torch(xb, cfg)
    sp.decode(layers, x_in, x_out, y, counts)
    torch.cuda.synchronize()
    for L in layers:
        assert L.last_device_error() == (sp.OK, 0)
    return layers, x64, x_out, y, counts, prefix_runner(layers, x_in, cfg)


@pytest.mark.parametrize("B", [3, 8, 16, 20, 48, 100, 128])
@pytest.mark.parametrize("name", list(CASES))
def test_union_stack_matches_oracle(name, B):
    cfg, Lc = CASES[name]
    hs = [wl.host_layer(cfg, l) for l in range(Lc)]
    layers, x64, x_out, y, counts, pre = run(cfg, hs, B, aux=800 + B)
    check_stack(layers, [HostOracle(h) for h in hs], cfg, x64, y, x_out, counts, run_prefix=pre)


def test_union_stack_context_sized_for_a_larger_batch():
    cfg, Lc = CASES["block-d1024-n4096-H256-L3"]
    hs = [wl.host_layer(cfg, l) for l in range(Lc)]
    layers, x64, x_out, y, counts, pre = run(cfg, hs, 24, aux=900, max_batch=128)
    check_stack(layers, [HostOracle(h) for h in hs], cfg, x64, y, x_out, counts, run_prefix=pre)


def test_union_stack_empty_set():
    """Every predictor logit far below 0: no neuron is selected in any layer, so
    y = b2 and each layer only renormalises its input."""
    cfg, Lc = CASES["block-d1024-n4096-H256-L3"]
    hs = [wl.host_layer(cfg, l) for l in range(Lc)]
    for h in hs:
        h.bp2 = wl.round_to(np.full(cfg.n, -60.0), cfg.bf16)
    layers, x64, x_out, y, counts, pre = run(cfg, hs, 16, aux=901)
    assert counts.cpu().numpy().tolist() == [0] * Lc
    check_stack(layers, [HostOracle(h) for h in hs], cfg, x64, y, x_out, counts, run_prefix=pre)


def test_union_stack_graph_replays_are_bitwise_repeatable():
    cfg, Lc = CASES["block-d1024-n4096-H256-L3"]
    B = 32
    hs = [wl.host_layer(cfg, l) for l in range(Lc)]
    layers = [sp.Layer(**torch_layer(h), max_batch=B) for h in hs]
    x_in = torch.empty(B, cfg.d, dtype=torch.float16, device="cuda")
    x_out = torch.empty_like(x_in)
    y = torch.empty(B, cfg.d, dtype=torch.float32, device="cuda")
    counts = torch.zeros(Lc, dtype=torch.int32, device="cuda")
    s = torch.cuda.Stream()
    x_in.copy_(wl.to_torch(wl.tokens(cfg, B, aux=11), cfg))
    with torch.cuda.stream(s):
        sp.decode(layers, x_in, x_out, y, counts, stream=s)
    s.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        sp.decode(layers, x_in, x_out, y, counts, stream=s)
    seen = {}
    for aux in (11, 12, 11):
        x_in.copy_(wl.to_torch(wl.tokens(cfg, B, aux=aux), cfg))
        g.replay()
        torch.cuda.synchronize()
        got = (bits_of(x_out).copy(), y.cpu().numpy().copy(), counts.cpu().numpy().copy())
        if aux in seen:
            assert all(np.array_equal(a, b) for a, b in zip(seen[aux], got))
        seen[aux] = got
    assert not np.array_equal(seen[11][1], seen[12][1])
    for L in layers:
        assert L.last_device_error() == (sp.OK, 0)
    del g
