"""The union path's neuron table as the FC1 launch ranks it from the mask words inside
spffn_decode (batch >= 3), at its two extremes, against the oracle chain:
- no neuron selected in any layer (count 0, y = b2);
- every neuron selected, with more 128-row tiles than CTAs (so some CTAs hold two tiles,
  one split each) and a ragged last tile."""
import dataclasses

import numpy as np
import pytest

import activation_sparse_ffn_predictor_b200 as sp
import workload as wl
from _gpu import HostOracle, check_stack, prefix_runner, torch_layer, x_tokens

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

B = 4


def decode_with_bias(cfg, Lc, bp2_value, aux):
    """Decode Lc layers whose predictor output bias is bp2_value for every neuron; returns
    the per-layer counts after checking every layer against the oracle."""
    hs = []
    for l in range(Lc):
        h = wl.host_layer(cfg, l)
        hs.append(dataclasses.replace(h, bp2=wl.round_to(np.full(cfg.n, bp2_value), cfg.bf16)))
    layers = [sp.Layer(**torch_layer(h), max_batch=B) for h in hs]
    assert sp.decode_kernel_launches(layers, B) > 1            # the per-layer union launches
    xb, x64 = x_tokens(cfg, B, aux=aux)
    x_in = wl.to_torch(xb, cfg)
    dt = torch.bfloat16 if cfg.bf16 else torch.float16
    x_out = torch.empty(B, cfg.d, dtype=dt, device="cuda")
    y = torch.empty(B, cfg.d, dtype=torch.float32, device="cuda")
    counts = torch.full((Lc,), -1, dtype=torch.int32, device="cuda")
    sp.decode(layers, x_in, x_out, y, counts)
    torch.cuda.synchronize()
    for L in layers:
        assert L.last_device_error() == (sp.OK, 0)
    check_stack(layers, [HostOracle(h) for h in hs], cfg, x64, y, x_out, counts,
                run_prefix=prefix_runner(layers, x_in, cfg))
    return counts.cpu().numpy(), y.cpu().numpy()


def test_no_neuron_selected():
    cfg = wl.CONFIGS[0]
    counts, y = decode_with_bias(cfg, 2, -1.0e3, aux=611)
    assert counts.tolist() == [0, 0]
    assert np.all(y == 0.0)                                    # b2 = 0 in the workloads


def test_every_neuron_selected_more_tiles_than_ctas():
    # 20416 neurons: 160 tiles of 128 rows (the last one ragged), more than the SM count
    cfg = wl.FFNConfig("allsel-d1024-n20416-H256", 2, 1024, 20416, 256, "f16", 1.2, 0.1)
    counts, _ = decode_with_bias(cfg, 2, 1.0e3, aux=612)
    assert counts.tolist() == [cfg.n, cfg.n]
