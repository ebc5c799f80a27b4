"""spffn_forward_noalloc, the allocation-free forward for callers that cannot
call cudaMalloc (its scratch is the library's fixed device array): through the
C-ABI, its output matches spffn_forward's on the same layer and table, on two
calls in a row.  Collected last, so a run that stops at the first failure has
already run every other test."""
import ctypes

import numpy as np
import pytest

import activation_sparse_ffn_predictor_b200 as sp
import workload as wl
from _gpu import REL_L2_BAR, rel_l2, torch_layer

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu


def test_forward_noalloc_matches_forward_twice():
    cfg = wl.CONFIGS[0]
    B = 3
    h = wl.host_layer(cfg, 0)
    L = sp.Layer(**torch_layer(h), max_batch=B)
    lib = sp.library()
    r = np.random.default_rng(11)
    for call in range(2):
        x = wl.to_torch(wl.tokens(cfg, B, aux=700 + call), cfg)
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
        assert torch.isfinite(y).all()
        assert rel_l2(y.cpu().numpy(), y_ref.cpu().numpy()) <= REL_L2_BAR


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
