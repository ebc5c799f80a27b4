"""The decode paths at the shapes the benchmark times, compared with the oracle
layer by layer: every layer's neuron table (bit-exact outside the near-threshold
band) and count, the last layer's y (per token and against the internal bar) and
the final x.  Layers are filled in HBM by the device generator; the oracle
regenerates the whole predictor and exactly the FFN rows each table names.

One case per instantiation of the whole-stack kernel that a benchmark line
reports (hidden units per lane HV = ceil(H / 256)):

    OPT-6.7B shape  d4096 n16384 H1024 fp16   B = 1 and 2, HV = 4, with and
                                              without look-ahead
    OPT-13B shape   d5120 n20480 H1024 bf16   B = 1, HV = 4, with and without
                                              look-ahead
    OPT-30B shape   d7168 n28672 H1024 fp16   B = 1 (three predictor and three
                                              FFN slots), rate 5%
    OPT-66B shape   d9216 n36864 H2048 fp16   B = 1 (HV = 8), and B = 32 on the
                                              union tensor-core path
and the whole-stack union kernel at the OPT-13B shape (bf16, B = 4 and 16) and
the OPT-66B shape (fp16, B = 32, the default benchmark line).
"""
import pytest

import activation_sparse_ffn_predictor_b200 as sp
import workload as wl
from _gpu import RowsOracle, check_stack, prefix_runner, x_tokens

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

#            config, layers, batch, look-ahead, rate
CASES = {
    "opt6.7b-B1": (1, 3, 1, False, None),
    "opt6.7b-B1-lookahead": (1, 3, 1, True, None),
    "opt6.7b-B2": (1, 3, 2, False, None),
    "opt6.7b-B2-lookahead": (1, 2, 2, True, None),
    "opt13b-bf16-B1": (2, 3, 1, False, None),
    "opt13b-bf16-B1-lookahead": (2, 3, 1, True, None),
    "opt30b-B1-r0.05": (3, 3, 1, False, 0.05),
    "opt13b-bf16-B4-union": (2, 2, 4, False, None),
    "opt13b-bf16-B16-union": (2, 2, 16, False, None),
    "opt66b-B1": (4, 2, 1, False, None),
    "opt66b-B32-union": (4, 2, 32, False, None),
}


@pytest.mark.parametrize("name", list(CASES))
def test_timed_path_matches_oracle(name):
    cid, Lc, B, lookahead, rate = CASES[name]
    cfg = wl.CONFIGS[cid]
    dls = [wl.device_layer(cfg, l, rate=rate) for l in range(Lc)]
    layers = [sp.Layer.from_device_layer(d, max_batch=B) for d in dls]
    # the default dispatch, as in the benchmark: B <= 2 the whole stack in one persistent
    # launch, from 3 tokens per-layer tensor-core launches (five per layer and token group)
    want_launches = 1 if B <= 2 else Lc * (3 + 2 * ((B + 127) // 128))
    assert sp.decode_kernel_launches(layers, B) == want_launches
    xb, x64 = x_tokens(cfg, B, aux=4000 + 17 * cid + B)
    dt = torch.bfloat16 if cfg.bf16 else torch.float16
    x_out = torch.empty(B, cfg.d, dtype=dt, device="cuda")
    y = torch.empty(B, cfg.d, dtype=torch.float32, device="cuda")
    counts = torch.full((Lc,), -1, dtype=torch.int32, device="cuda")
    x_in = wl.to_torch(xb, cfg)
    sp.decode(layers, x_in, x_out, y, counts, lookahead=lookahead)
    torch.cuda.synchronize()
    for L in layers:
        assert L.last_device_error() == (sp.OK, 0)
    oracles = [RowsOracle(cfg, l, rate=rate) for l in range(Lc)]
    check_stack(layers, oracles, cfg, x64, y, x_out, counts, lookahead=lookahead,
                run_prefix=prefix_runner(layers, x_in, cfg, lookahead))
    for L in layers:
        L.close()
    del dls, layers
    torch.cuda.empty_cache()


@pytest.mark.parametrize("cid,Lc,B,mode", [(4, 2, 32, 1), (2, 2, 16, 1), (2, 2, 4, 1), (2, 2, 4, 0)])
def test_other_union_dispatch_matches_oracle(cid, Lc, B, mode):
    """The whole-stack kernel (mode 1, which the default does not pick) and
    explicit per-layer launches (mode 0)."""
    cfg = wl.CONFIGS[cid]
    dls = [wl.device_layer(cfg, l) for l in range(Lc)]
    layers = [sp.Layer.from_device_layer(d, max_batch=B) for d in dls]
    try:
        sp.set_union_stack(mode)
        assert sp.decode_kernel_launches(layers, B) == (1 if mode == 1 else Lc * 5)
        xb, x64 = x_tokens(cfg, B, aux=4100 + cid)
        dt = torch.bfloat16 if cfg.bf16 else torch.float16
        x_out = torch.empty(B, cfg.d, dtype=dt, device="cuda")
        y = torch.empty(B, cfg.d, dtype=torch.float32, device="cuda")
        counts = torch.full((Lc,), -1, dtype=torch.int32, device="cuda")
        x_in = wl.to_torch(xb, cfg)
        sp.decode(layers, x_in, x_out, y, counts)
        torch.cuda.synchronize()
        for L in layers:
            assert L.last_device_error() == (sp.OK, 0)
        oracles = [RowsOracle(cfg, l) for l in range(Lc)]
        check_stack(layers, oracles, cfg, x64, y, x_out, counts, run_prefix=prefix_runner(layers, x_in, cfg))
    finally:
        sp.set_union_stack(sp.UNION_AUTO)
    for L in layers:
        L.close()
    del dls, layers
    torch.cuda.empty_cache()
