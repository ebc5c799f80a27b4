"""bench.py's dense comparison arm (cuBLAS on the same weights) computes the
dense FFN and the chaining the oracle defines."""
import pytest

import bench
import oracle as O
import workload as wl
from _gpu import rel_l2

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

# cuBLAS hands back z = W1 x + b1 and y in fp16.  Each rounding is at most 2^-11
# relative per element, so together they stay under about 1e-3 rel-L2 on y.
# The bound leaves a factor of two for cuBLAS's own fp32 summation order.
DENSE_BAR = 2e-3


def test_dense_arm_matches_oracle():
    cfg = wl.CONFIGS[0]
    dl = wl.device_layer(cfg, 0, device="cuda")
    h = wl.host_layer(cfg, 0)
    xb = wl.tokens(cfg, 3, aux=77)
    x = wl.to_torch(xb, cfg, "cuda")
    x64 = wl.widen(xb, cfg.bf16)
    y = bench.dense_layer(dl, x)
    y_or = O.dense_ffn(h.f64("W1"), h.f64("b1"), h.f64("W2T"), h.f64("b2"), x64)
    assert rel_l2(y.cpu().numpy(), y_or) <= DENSE_BAR
    x1 = bench.dense_stack([dl], x, torch.float16)
    assert x1.dtype == torch.float16 and x1.shape == x.shape
    assert rel_l2(x1.float().cpu().numpy(), O.chain(x64, y_or)) <= DENSE_BAR

