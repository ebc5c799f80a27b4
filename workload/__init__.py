"""Seeded synthetic inputs for activation-sparse FFN decoding.

This module is the only code shared by the CUDA library's tests/bench and the
CPU oracle.  It draws random numbers and shapes them into the workloads the
configurations describe; it computes none of the method's arithmetic (no
predictor, no mask, no FFN).

Recipe (one layer, storage dtype f16 or bf16; every random number comes from the
counter-based generator in ``wl_gen.h``, Philox4x32-10 + Box-Muller):

* ``W1[n,d]``, ``W2T[n,d]``  ~ N(0, 1/d)   (FC1 rows and neuron-major FC2 rows)
* ``Wp1[H,d]`` ~ N(0, 1/d), ``Wp2[n,H]`` ~ N(0, 1/H)   (predictor, N(0, 1/fan_in))
* ``x[B,d]`` ~ N(0, 1) per decode step
* activation rate of neuron i: ``p_i = min(0.99, c * r_i^-alpha)`` with rank
  ``r_i`` from a seeded permutation (hot neurons start scattered) and ``c``
  found by fp64 bisection so that ``mean(p) = rate``
* ``b1_i = -Phi^-1(1 - p_i)`` so that ``P(W1[i].x + b1_i > 0) ~= p_i``
* ``bp2_i = -(m S1_i + sqrt(v S2_i) Phi^-1(1 - p_i))`` with ``S1_i``/``S2_i`` the
  fp64 row sums of ``Wp2[i]`` and of its squares, ``m = 1/sqrt(2 pi)`` and
  ``v = 1/2 - 1/(2 pi)`` (mean and variance of ReLU of a unit normal), so that
  the predicted rate of neuron i is also ~= ``p_i``
* ``b2 = 0``, ``bp1 = 0``

Tensors are returned as ``uint16`` arrays holding the storage bits.
"""
from __future__ import annotations

import ctypes
import math
import os
from dataclasses import dataclass, field, replace
from typing import Optional, Sequence

import numpy as np

from . import build as _build

SEED = 20241208

# Stream ids: (layer << 32) | (tensor << 24) | aux.
T_W1, T_W2T, T_WP1, T_WP2, T_X, T_XPROF, T_PERM, T_Y = 1, 2, 3, 4, 5, 6, 7, 8
# attention layers: projections, output projection (head-major), head predictor, tokens
T_WQ, T_WK, T_WV, T_WOT, T_WA1, T_WA2, T_XA = 9, 10, 11, 12, 13, 14, 15

PMAX = 0.99
RELU_MEAN = 1.0 / math.sqrt(2.0 * math.pi)
RELU_VAR = 0.5 - 1.0 / (2.0 * math.pi)


def stream_id(tensor: int, layer: int = 0, aux: int = 0) -> int:
    assert 0 <= aux < (1 << 24) and 0 <= tensor < 256 and 0 <= layer < (1 << 31)
    return (layer << 32) | (tensor << 24) | aux


@dataclass(frozen=True)
class FFNConfig:
    """Shape of one synthetic FFN layer stack."""
    name: str
    layers: int
    d: int
    n: int
    H: int
    dtype: str          # "f16" or "bf16"
    alpha: float
    rate: float
    batch: int = 1
    steps: int = 16
    rates: tuple = ()   # sweep values, when the workload has one
    batches: tuple = ()

    @property
    def bf16(self) -> int:
        return 1 if self.dtype == "bf16" else 0

    def with_(self, **kw) -> "FFNConfig":
        return replace(self, **kw)


# The five workloads: a single block, then OPT-6.7B/13B/30B/66B-shaped stacks.
CONFIGS = {
    0: FFNConfig("block-d1024-n4096", 1, 1024, 4096, 256, "f16", 1.2, 0.10, 1, 16),
    1: FFNConfig("opt6.7b-d4096-n16384-L32", 32, 4096, 16384, 1024, "f16", 1.2, 0.05, 1, 128),
    2: FFNConfig("opt13b-d5120-n20480-L40", 40, 5120, 20480, 1024, "bf16", 1.0, 0.05, 1, 64,
                 batches=(1, 4, 8, 16)),
    3: FFNConfig("opt30b-d7168-n28672-L48", 48, 7168, 28672, 1024, "f16", 1.2, 0.05, 1, 16,
                 rates=(0.20, 0.10, 0.05, 0.01)),
    4: FFNConfig("opt66b-d9216-n36864-L64", 64, 9216, 36864, 2048, "f16", 1.0, 0.01, 32, 32),
}


# ---------------------------------------------------------------------------
# host library
_lib = None


def host_lib():
    global _lib
    if _lib is None:
        path = _build.build_host()
        lib = ctypes.CDLL(path)
        u64, i64, dbl, i32 = ctypes.c_uint64, ctypes.c_int64, ctypes.c_double, ctypes.c_int
        vp = ctypes.c_void_p
        lib.wl_philox.argtypes = [vp, vp, vp]
        lib.wl_normal_f64.argtypes = [u64, u64, u64, i64, vp]
        lib.wl_fill.argtypes = [u64, u64, u64, i64, dbl, i32, vp]
        lib.wl_fill_rows.argtypes = [u64, u64, i64, vp, i64, dbl, i32, vp]
        lib.wl_row_stats.argtypes = [vp, i64, i64, i32, vp, vp]
        lib.wl_round_f64.argtypes = [vp, i64, i32, vp]
        lib.wl_widen.argtypes = [vp, i64, i32, vp]
        lib.wl_u64_keys.argtypes = [u64, u64, i64, vp]
        for f in (lib.wl_philox, lib.wl_normal_f64, lib.wl_fill, lib.wl_fill_rows,
                  lib.wl_row_stats, lib.wl_round_f64, lib.wl_widen, lib.wl_u64_keys):
            f.restype = None
        _lib = lib
    return _lib


def _ptr(a: np.ndarray):
    assert a.flags["C_CONTIGUOUS"]
    return a.ctypes.data_as(ctypes.c_void_p)


def philox4x32_10(ctr: Sequence[int], key: Sequence[int]) -> list:
    c = np.asarray(ctr, dtype=np.uint32)
    k = np.asarray(key, dtype=np.uint32)
    o = np.zeros(4, dtype=np.uint32)
    host_lib().wl_philox(_ptr(c), _ptr(k), _ptr(o))
    return [int(v) for v in o]


def normals(stream: int, count: int, e0: int = 0, seed: int = SEED) -> np.ndarray:
    out = np.empty(count, dtype=np.float64)
    host_lib().wl_normal_f64(seed, stream, e0, count, _ptr(out))
    return out


def fill(stream: int, count: int, scale: float, bf16: int, e0: int = 0, seed: int = SEED) -> np.ndarray:
    out = np.empty(count, dtype=np.uint16)
    host_lib().wl_fill(seed, stream, e0, count, scale, bf16, _ptr(out))
    return out


def fill_rows(stream: int, cols: int, rows: np.ndarray, scale: float, bf16: int,
              seed: int = SEED) -> np.ndarray:
    rows = np.ascontiguousarray(rows, dtype=np.int64)
    out = np.empty((rows.size, cols), dtype=np.uint16)
    if rows.size:
        host_lib().wl_fill_rows(seed, stream, cols, _ptr(rows), rows.size, scale, bf16, _ptr(out))
    return out


def row_stats(w_bits: np.ndarray, bf16: int):
    w = np.ascontiguousarray(w_bits, dtype=np.uint16)
    rows, cols = w.shape
    s1 = np.empty(rows, dtype=np.float64)
    s2 = np.empty(rows, dtype=np.float64)
    host_lib().wl_row_stats(_ptr(w), rows, cols, bf16, _ptr(s1), _ptr(s2))
    return s1, s2


def round_to(x: np.ndarray, bf16: int) -> np.ndarray:
    x = np.ascontiguousarray(x, dtype=np.float64)
    out = np.empty(x.shape, dtype=np.uint16)
    host_lib().wl_round_f64(_ptr(x), x.size, bf16, _ptr(out))
    return out


def widen(bits: np.ndarray, bf16: int) -> np.ndarray:
    """Storage bits -> exact fp64 values."""
    b = np.ascontiguousarray(bits, dtype=np.uint16)
    out = np.empty(b.shape, dtype=np.float64)
    host_lib().wl_widen(_ptr(b), b.size, bf16, _ptr(out))
    return out


# ---------------------------------------------------------------------------
# per-neuron rates and biases
def neuron_ranks(n: int, layer: int, seed: int = SEED) -> np.ndarray:
    """Seeded permutation: rank (1 = hottest) of each neuron in its physical slot."""
    keys = np.empty(n, dtype=np.uint64)
    host_lib().wl_u64_keys(seed, stream_id(T_PERM, layer), n, _ptr(keys))
    order = np.argsort(keys, kind="stable")
    rank = np.empty(n, dtype=np.int64)
    rank[order] = np.arange(1, n + 1, dtype=np.int64)
    return rank


def power_law_rates(n: int, alpha: float, rate: float, layer: int, seed: int = SEED) -> np.ndarray:
    """p_i = min(PMAX, c r_i^-alpha), c by fp64 bisection so that mean(p) = rate."""
    r = neuron_ranks(n, layer, seed).astype(np.float64) ** (-alpha)
    lo, hi = 0.0, float(n) * 2.0
    for _ in range(200):
        c = 0.5 * (lo + hi)
        m = np.minimum(PMAX, c * r).mean()
        if m < rate:
            lo = c
        else:
            hi = c
    return np.minimum(PMAX, 0.5 * (lo + hi) * r)


def _ndtri(q: np.ndarray) -> np.ndarray:
    from scipy.special import ndtri
    return ndtri(q)


def fc1_bias(p: np.ndarray, bf16: int) -> np.ndarray:
    return round_to(-_ndtri(1.0 - p), bf16)


def predictor_bias(s1: np.ndarray, s2: np.ndarray, p: np.ndarray, bf16: int) -> np.ndarray:
    b = -(RELU_MEAN * s1 + np.sqrt(RELU_VAR * s2) * _ndtri(1.0 - p))
    return round_to(b, bf16)


# ---------------------------------------------------------------------------
# host layers
@dataclass
class HostLayer:
    """One layer's inputs as storage bits (uint16).  ``rows`` set => W1/W2T hold
    only those rows (in that order); everything else is full size."""
    cfg: FFNConfig
    layer: int
    p: np.ndarray
    b1: np.ndarray
    b2: np.ndarray
    Wp1: np.ndarray
    bp1: np.ndarray
    Wp2: np.ndarray
    bp2: np.ndarray
    W1: np.ndarray
    W2T: np.ndarray
    rows: Optional[np.ndarray] = None

    def f64(self, name: str) -> np.ndarray:
        return widen(getattr(self, name), self.cfg.bf16)


def host_predictor(cfg: FFNConfig, layer: int, seed: int = SEED, rate: Optional[float] = None):
    bf = cfg.bf16
    p = power_law_rates(cfg.n, cfg.alpha, cfg.rate if rate is None else rate, layer, seed)
    Wp1 = fill(stream_id(T_WP1, layer), cfg.H * cfg.d, 1.0 / math.sqrt(cfg.d), bf, seed=seed)
    Wp1 = Wp1.reshape(cfg.H, cfg.d)
    Wp2 = fill(stream_id(T_WP2, layer), cfg.n * cfg.H, 1.0 / math.sqrt(cfg.H), bf, seed=seed)
    Wp2 = Wp2.reshape(cfg.n, cfg.H)
    s1, s2 = row_stats(Wp2, bf)
    bp2 = predictor_bias(s1, s2, p, bf)
    bp1 = np.zeros(cfg.H, dtype=np.uint16)
    return p, Wp1, bp1, Wp2, bp2


def host_layer(cfg: FFNConfig, layer: int = 0, rows: Optional[np.ndarray] = None,
               seed: int = SEED, rate: Optional[float] = None) -> HostLayer:
    bf = cfg.bf16
    p, Wp1, bp1, Wp2, bp2 = host_predictor(cfg, layer, seed, rate)
    sc = 1.0 / math.sqrt(cfg.d)
    if rows is None:
        W1 = fill(stream_id(T_W1, layer), cfg.n * cfg.d, sc, bf, seed=seed).reshape(cfg.n, cfg.d)
        W2T = fill(stream_id(T_W2T, layer), cfg.n * cfg.d, sc, bf, seed=seed).reshape(cfg.n, cfg.d)
    else:
        rows = np.asarray(rows, dtype=np.int64)
        W1 = fill_rows(stream_id(T_W1, layer), cfg.d, rows, sc, bf, seed)
        W2T = fill_rows(stream_id(T_W2T, layer), cfg.d, rows, sc, bf, seed)
    b1 = fc1_bias(p, bf)
    b2 = np.zeros(cfg.d, dtype=np.uint16)
    return HostLayer(cfg, layer, p, b1, b2, Wp1, bp1, Wp2, bp2, W1, W2T, rows)


def tokens(cfg: FFNConfig, B: int, aux: int, layer: int = 0, tensor: int = T_X,
           seed: int = SEED) -> np.ndarray:
    """[B, d] storage bits of N(0,1) decode inputs for stream (tensor, layer, aux)."""
    return fill(stream_id(tensor, layer, aux), B * cfg.d, 1.0, cfg.bf16, seed=seed).reshape(B, cfg.d)


def float_tokens(cfg: FFNConfig, B: int, aux: int, layer: int = 0, seed: int = SEED) -> np.ndarray:
    """[B, d] fp32 values (N(0,1) rounded to fp32), e.g. a stand-in FFN output."""
    return normals(stream_id(T_Y, layer, aux), B * cfg.d, seed=seed).astype(np.float32).reshape(B, cfg.d)


# ---------------------------------------------------------------------------
# device layers (torch is used only to own device memory)
_dlib = None


def device_lib():
    global _dlib
    if _dlib is None:
        path = _build.build_device()
        lib = ctypes.CDLL(path)
        u64, i64, dbl, i32, vp = ctypes.c_uint64, ctypes.c_int64, ctypes.c_double, ctypes.c_int, ctypes.c_void_p
        lib.wl_dev_fill.argtypes = [u64, u64, u64, i64, dbl, i32, vp, vp]
        lib.wl_dev_fill.restype = ctypes.c_int
        lib.wl_dev_row_stats.argtypes = [vp, i64, i64, i32, vp, vp, vp]
        lib.wl_dev_row_stats.restype = ctypes.c_int
        _dlib = lib
    return _dlib


def _torch_dtype(cfg):
    import torch
    return torch.bfloat16 if cfg.bf16 else torch.float16


def device_fill(t, stream: int, scale: float, bf16: int, seed: int = SEED, e0: int = 0):
    import torch
    s = torch.cuda.current_stream().cuda_stream
    rc = device_lib().wl_dev_fill(seed, stream, e0, t.numel(), scale, bf16, ctypes.c_void_p(t.data_ptr()),
                                  ctypes.c_void_p(s))
    if rc != 0:
        raise RuntimeError("wl_dev_fill failed: cuda error %d" % rc)
    return t


def device_row_stats(w, bf16: int):
    import torch
    rows, cols = w.shape
    s1 = torch.empty(rows, dtype=torch.float64, device=w.device)
    s2 = torch.empty(rows, dtype=torch.float64, device=w.device)
    s = torch.cuda.current_stream().cuda_stream
    rc = device_lib().wl_dev_row_stats(ctypes.c_void_p(w.data_ptr()), rows, cols, bf16,
                                       ctypes.c_void_p(s1.data_ptr()), ctypes.c_void_p(s2.data_ptr()),
                                       ctypes.c_void_p(s))
    if rc != 0:
        raise RuntimeError("wl_dev_row_stats failed: cuda error %d" % rc)
    return s1.cpu().numpy(), s2.cpu().numpy()


@dataclass
class DeviceLayer:
    W1: object
    b1: object
    W2T: object
    b2: object
    Wp1: object
    bp1: object
    Wp2: object
    bp2: object
    p: np.ndarray


def device_layer(cfg: FFNConfig, layer: int, device="cuda", seed: int = SEED,
                 rate: Optional[float] = None, out: Optional[DeviceLayer] = None) -> DeviceLayer:
    """Fill one layer directly in HBM with the same bits ``host_layer`` gives."""
    import torch
    dt = _torch_dtype(cfg)
    bf = cfg.bf16
    p = power_law_rates(cfg.n, cfg.alpha, cfg.rate if rate is None else rate, layer, seed)
    if out is None:
        out = DeviceLayer(
            W1=torch.empty(cfg.n, cfg.d, dtype=dt, device=device),
            b1=torch.empty(cfg.n, dtype=dt, device=device),
            W2T=torch.empty(cfg.n, cfg.d, dtype=dt, device=device),
            b2=torch.zeros(cfg.d, dtype=dt, device=device),
            Wp1=torch.empty(cfg.H, cfg.d, dtype=dt, device=device),
            bp1=torch.zeros(cfg.H, dtype=dt, device=device),
            Wp2=torch.empty(cfg.n, cfg.H, dtype=dt, device=device),
            bp2=torch.empty(cfg.n, dtype=dt, device=device),
            p=p)
    out.p = p
    sc = 1.0 / math.sqrt(cfg.d)
    device_fill(out.W1, stream_id(T_W1, layer), sc, bf, seed)
    device_fill(out.W2T, stream_id(T_W2T, layer), sc, bf, seed)
    device_fill(out.Wp1, stream_id(T_WP1, layer), sc, bf, seed)
    device_fill(out.Wp2, stream_id(T_WP2, layer), 1.0 / math.sqrt(cfg.H), bf, seed)
    s1, s2 = device_row_stats(out.Wp2, bf)
    out.b1.copy_(torch.from_numpy(fc1_bias(p, bf).view(np.int16)).view(dt))
    out.bp2.copy_(torch.from_numpy(predictor_bias(s1, s2, p, bf).view(np.int16)).view(dt))
    out.b2.zero_()
    out.bp1.zero_()
    return out


def to_torch(bits: np.ndarray, cfg: FFNConfig, device="cuda"):
    """Storage bits -> torch tensor of the storage dtype (bit-exact copy)."""
    import torch
    t = torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(_torch_dtype(cfg))
    return t.to(device)


# ---------------------------------------------------------------------------
# attention layers with an attention-head predictor
@dataclass(frozen=True)
class AttnConfig:
    """Shape of a synthetic attention stack: d model width, nh heads of width dh,
    Ha predictor hidden units, per-head selection rate, tokens already in the
    cache before timing (context) and cache capacity (tmax)."""
    name: str
    layers: int
    d: int
    nh: int
    dh: int
    Ha: int
    dtype: str
    rate: float
    context: int
    tmax: int

    @property
    def bf16(self) -> int:
        return 1 if self.dtype == "bf16" else 0

    def with_(self, **kw) -> "AttnConfig":
        return replace(self, **kw)


# A small block and the OPT-66B attention shape (72 heads of 128), with the head
# rate of about 20% the DejaVu appendix reports.
ATTN_CONFIGS = {
    0: AttnConfig("attn-d1024-h16", 1, 1024, 16, 64, 256, "f16", 0.25, 24, 64),
    1: AttnConfig("attn-opt66b-d9216-h72-L64", 64, 9216, 72, 128, 1024, "f16", 0.20, 1024, 1280),
}


@dataclass
class HostAttn:
    """One attention layer's weights as storage bits; biases of Q/K/V/O are zero."""
    cfg: AttnConfig
    layer: int
    Wq: np.ndarray
    Wk: np.ndarray
    Wv: np.ndarray
    WoT: np.ndarray
    Wa1: np.ndarray
    Wa2: np.ndarray
    ba2: np.ndarray

    def f64(self, name: str) -> np.ndarray:
        return widen(getattr(self, name), self.cfg.bf16)


def attn_head_bias(cfg: AttnConfig, Wa2: np.ndarray) -> np.ndarray:
    """ba2 calibrated like the FFN predictor's so each head is selected at ``rate``."""
    s1, s2 = row_stats(Wa2, cfg.bf16)
    return predictor_bias(s1, s2, np.full(cfg.nh, cfg.rate), cfg.bf16)


def host_attn(cfg: AttnConfig, layer: int = 0, seed: int = SEED) -> HostAttn:
    bf, rows = cfg.bf16, cfg.nh * cfg.dh
    sd = 1.0 / math.sqrt(cfg.d)
    m = lambda t, r, c, sc: fill(stream_id(t, layer), r * c, sc, bf, seed=seed).reshape(r, c)
    Wa2 = m(T_WA2, cfg.nh, cfg.Ha, 1.0 / math.sqrt(cfg.Ha))
    return HostAttn(cfg, layer, m(T_WQ, rows, cfg.d, sd), m(T_WK, rows, cfg.d, sd), m(T_WV, rows, cfg.d, sd),
                    m(T_WOT, rows, cfg.d, 1.0 / math.sqrt(rows)), m(T_WA1, cfg.Ha, cfg.d, sd), Wa2,
                    attn_head_bias(cfg, Wa2))


def attn_rows(cfg: AttnConfig, tensor: int, layer: int, rows, seed: int = SEED) -> np.ndarray:
    """Storage bits of the given rows of one projection ([len(rows), d])."""
    sc = 1.0 / math.sqrt(cfg.nh * cfg.dh) if tensor == T_WOT else 1.0 / math.sqrt(cfg.d)
    return fill_rows(stream_id(tensor, layer), cfg.d, np.asarray(rows, dtype=np.int64), sc, cfg.bf16, seed)


@dataclass
class DeviceAttn:
    Wq: object
    Wk: object
    Wv: object
    WoT: object
    Wa1: object
    Wa2: object
    ba2: object


def device_attn(cfg: AttnConfig, layer: int, device="cuda", seed: int = SEED) -> DeviceAttn:
    """Fill one attention layer directly in HBM with the same bits host_attn gives."""
    import torch
    dt = _torch_dtype(cfg)
    bf, rows = cfg.bf16, cfg.nh * cfg.dh
    sd = 1.0 / math.sqrt(cfg.d)
    e = lambda r, c: torch.empty(r, c, dtype=dt, device=device)
    out = DeviceAttn(e(rows, cfg.d), e(rows, cfg.d), e(rows, cfg.d), e(rows, cfg.d), e(cfg.Ha, cfg.d),
                     e(cfg.nh, cfg.Ha), torch.empty(cfg.nh, dtype=dt, device=device))
    device_fill(out.Wq, stream_id(T_WQ, layer), sd, bf, seed)
    device_fill(out.Wk, stream_id(T_WK, layer), sd, bf, seed)
    device_fill(out.Wv, stream_id(T_WV, layer), sd, bf, seed)
    device_fill(out.WoT, stream_id(T_WOT, layer), 1.0 / math.sqrt(rows), bf, seed)
    device_fill(out.Wa1, stream_id(T_WA1, layer), sd, bf, seed)
    device_fill(out.Wa2, stream_id(T_WA2, layer), 1.0 / math.sqrt(cfg.Ha), bf, seed)
    s1, s2 = device_row_stats(out.Wa2, bf)
    out.ba2.copy_(torch.from_numpy(predictor_bias(s1, s2, np.full(cfg.nh, cfg.rate), bf).view(np.int16)).view(dt))
    return out


def attn_tokens(cfg: AttnConfig, T: int, aux: int, layer: int = 0, seed: int = SEED) -> np.ndarray:
    """[T, d] storage bits of N(0,1) attention inputs."""
    return fill(stream_id(T_XA, layer, aux), T * cfg.d, 1.0, cfg.bf16, seed=seed).reshape(T, cfg.d)
