"""The bounded-wait failure path of the persistent whole-stack kernels, made to
run out on purpose without any fault: a short grid-barrier wait limit plus a
grid barrier that expects one more arrival than there are CTAs
(spffn_set_wait_test).  The kernel must give up, latch SPFFN_ERR_TIMEOUT with
the barrier bit, drain its copies and return; the next normal decode on the
same contexts must be clean and match the oracle.  Covers the small-batch kernel
(B = 1, with and without look-ahead) and the union-path kernel (B = 16)."""
import pytest

import activation_sparse_ffn_predictor_b200 as sp
import workload as wl
from _gpu import HostOracle, check_stack, prefix_runner, torch_layer, x_tokens

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

ERR_BARRIER_TIMEOUT = 1 << 2


@pytest.mark.parametrize("B,lookahead", [(1, False), (1, True), (16, False)])
def test_unmeetable_grid_barrier_times_out_and_context_recovers(B, lookahead):
    cfg = wl.CONFIGS[0]
    Lc = 2
    hs = [wl.host_layer(cfg, l) for l in range(Lc)]
    layers = [sp.Layer(**torch_layer(h), max_batch=B) for h in hs]
    sp.set_union_stack(sp.UNION_STACK)          # B = 16: the whole-stack union kernel
    assert sp.decode_kernel_launches(layers, B) == 1
    xb, x64 = x_tokens(cfg, B, aux=91)
    x_in = wl.to_torch(xb, cfg)
    x_out = torch.empty(B, cfg.d, dtype=torch.float16, device="cuda")
    y = torch.empty(B, cfg.d, dtype=torch.float32, device="cuda")
    counts = torch.full((Lc,), -1, dtype=torch.int32, device="cuda")
    lib = sp.library()
    try:
        assert lib.spffn_set_wait_test(5_000_000, 1) == sp.OK        # 5 ms, unmeetable barrier
        sp.decode(layers, x_in, x_out, y, counts, lookahead=lookahead)
        torch.cuda.synchronize()
    finally:
        assert lib.spffn_set_wait_test(0, 0) == sp.OK
        sp.set_union_stack(sp.UNION_STACK)
    s, code = layers[0].last_device_error()
    assert s == sp.ERR_TIMEOUT, (s, code)
    assert code & ERR_BARRIER_TIMEOUT, code
    # the same contexts decode normally afterwards
    counts.fill_(-1)
    sp.decode(layers, x_in, x_out, y, counts, lookahead=lookahead)
    torch.cuda.synchronize()
    for L in layers:
        assert L.last_device_error() == (sp.OK, 0)
    check_stack(layers, [HostOracle(h) for h in hs], cfg, x64, y, x_out, counts, lookahead=lookahead,
                run_prefix=prefix_runner(layers, x_in, cfg, lookahead))
    sp.set_union_stack(sp.UNION_AUTO)
