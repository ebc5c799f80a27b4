"""spffn_forward_noalloc, the allocation-free forward for callers that cannot
call cudaMalloc (code inside another allocator's arena or under a fixed
device-memory budget; its scratch is the library's fixed device array).
Through the C-ABI, on two calls in a row at each batch, its output matches the
oracle's sparse FFN over the same table (every token within the contract, the
whole tensor within the internal bar) and spffn_forward's output on the same
layer and table.  Collected last, so a run that stops at the first failure has
already run every other test."""
import ctypes

import numpy as np
import pytest

import activation_sparse_ffn_predictor_b200 as sp
import oracle as O
import workload as wl
from _gpu import check_y, oracle_layer, rel_l2, torch_layer

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("B", [1, 3, 32])
def test_forward_noalloc_matches_oracle_and_forward_twice(B):
    # B = 1 and 32: spffn_forward runs the persistent kernel and the union tensor-core
    # path there; the allocation-free call always runs the per-phase split kernels
    cfg = wl.CONFIGS[0]
    h = wl.host_layer(cfg, 0)
    OL = oracle_layer(h)
    L = sp.Layer(**torch_layer(h), max_batch=B)
    lib = sp.library()
    r = np.random.default_rng(11 + B)
    for call in range(2):
        xb = wl.tokens(cfg, B, aux=700 + 10 * B + call)
        x = wl.to_torch(xb, cfg)
        tab = np.sort(r.choice(cfg.n, 300 + 50 * call, replace=False)).astype(np.int32)
        idx = torch.from_numpy(tab).cuda()
        cnt = torch.tensor([tab.size], dtype=torch.int32, device="cuda")
        y_ref = torch.empty(B, cfg.d, dtype=torch.float32, device="cuda")
        y = torch.full((B, cfg.d), float("nan"), dtype=torch.float32, device="cuda")
        L.forward(x, idx, cnt, y_ref)
        s = torch.cuda.current_stream().cuda_stream
        st = lib.spffn_forward_noalloc(ctypes.byref(L.cfg), ctypes.byref(L.weights), x.data_ptr(), B,
                                       idx.data_ptr(), cnt.data_ptr(), y.data_ptr(), s)
        assert st == sp.OK, st
        torch.cuda.synchronize()
        got = y.cpu().numpy()
        want = O.sparse_ffn(OL["W1"], OL["b1"], OL["W2T"], OL["b2"], wl.widen(xb, cfg.bf16), tab)
        check_y(got, want)
        assert rel_l2(got, y_ref.cpu().numpy()) <= 1e-5


def test_forward_noalloc_rejects_oversize_on_host():
    """Beyond the fixed scratch (B * d * 4 bytes > 1 MiB) the call fails before
    touching the device."""
    lib = sp.library()
    cfg = sp.Config(9216, 4096, 256, 32, 0, 0)
    fake = 1 << 40
    w = sp.Weights(fake, fake, fake, None, fake, None, fake, None)
    st = lib.spffn_forward_noalloc(ctypes.byref(cfg), ctypes.byref(w), fake, 32, fake, fake, fake, None)
    assert st == sp.ERR_UNSUPPORTED
    assert lib.spffn_forward_noalloc(ctypes.byref(cfg), ctypes.byref(w), fake, 0, fake, fake, fake, None) \
        == sp.ERR_INVALID_ARG
