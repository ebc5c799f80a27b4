"""Activation-sparse FFN decoding on NVIDIA B200 — Python binding.

A thin ``ctypes`` layer over ``libspffn.so`` (C-ABI in ``include/spffn.h``):
it only marshals arguments.  Every step of the path — predictor, threshold,
compaction, FC1, FC2, reduction, chaining, profiling, row permutation — runs in
the library's CUDA kernels.  PyTorch is used only to own device memory and
streams.  There is no CPU fallback: if the library is missing and cannot be
built, importing the binding's functions raises.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional, Sequence

import numpy as np

from . import build as _build

__all__ = ["SpffnError", "Layer", "AttnLayer", "attn_step_kernel_launches", "decode", "decode_tables", "decode_kernel_launches", "forward_noalloc",
           "reorder", "reorder_dealt", "permute_rows", "permute_vector", "set_trace", "trace_marks",
           "set_l2_hot_rows", "l2_hot_rows", "set_union_stack", "union_stack",
           "workspace_bytes", "library", "F16", "BF16"]

F16, BF16 = 0, 1
OK, ERR_INVALID_ARG, ERR_UNSUPPORTED, ERR_WORKSPACE, ERR_CUDA, ERR_DEVICE_CHECK, ERR_TIMEOUT = range(7)

EXPORTS = ("spffn_workspace_bytes", "spffn_create", "spffn_destroy", "spffn_predict", "spffn_forward",
           "spffn_step", "spffn_chain", "spffn_decode", "spffn_profile_counts", "spffn_reorder",
           "spffn_permute_rows", "spffn_permute_vector", "spffn_last_device_error", "spffn_status_string",
           "spffn_num_partials", "spffn_decode_kernel_launches", "spffn_set_trace", "spffn_trace_marks",
           "spffn_last_cuda_error_string", "spffn_reorder_dealt", "spffn_forward_noalloc",
           "spffn_decode_lookahead", "spffn_layer_table", "spffn_decode_tables", "spffn_set_wait_test", "spffn_set_l2_hot_rows", "spffn_l2_hot_rows",
           "spffn_set_union_stack", "spffn_union_stack",
           "spffn_attn_workspace_bytes", "spffn_attn_create", "spffn_attn_destroy", "spffn_attn_reset",
           "spffn_attn_step", "spffn_attn_cache", "spffn_attn_step_kernel_launches", "spffn_attn_last_device_error")


class SpffnError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        super().__init__("%s: %s (status %d)" % (what, _status_string(status), status))


class Config(ctypes.Structure):
    _fields_ = [("d", ctypes.c_int32), ("n", ctypes.c_int32), ("H", ctypes.c_int32),
                ("max_batch", ctypes.c_int32), ("dtype", ctypes.c_int32), ("flags", ctypes.c_uint32)]


class Weights(ctypes.Structure):
    _fields_ = [(k, ctypes.c_void_p) for k in ("W1", "b1", "W2T", "b2", "Wp1", "bp1", "Wp2", "bp2")]


class AttnConfig(ctypes.Structure):
    _fields_ = [("d", ctypes.c_int32), ("nh", ctypes.c_int32), ("dh", ctypes.c_int32), ("Ha", ctypes.c_int32),
                ("tmax", ctypes.c_int32), ("dtype", ctypes.c_int32), ("flags", ctypes.c_uint32)]


class AttnWeights(ctypes.Structure):
    _fields_ = [(k, ctypes.c_void_p) for k in ("Wq", "bq", "Wk", "bk", "Wv", "bv", "WoT", "bo", "Wa1", "ba1",
                                                "Wa2", "ba2")]


class AttnCacheView(ctypes.Structure):
    _fields_ = [("K", ctypes.c_void_p), ("V", ctypes.c_void_p), ("filled", ctypes.c_void_p), ("Y", ctypes.c_void_p),
                ("t", ctypes.c_void_p)]


_lib = None


def library(path: Optional[str] = None):
    """Load (building in-tree first if it is missing or stale) libspffn.so."""
    global _lib
    if _lib is not None:
        return _lib
    so = path or _build.SO
    if path is None and _build.stale():
        try:
            _build.build()
        except Exception as e:  # no nvcc here: the library must already exist
            if not os.path.exists(so):
                raise RuntimeError("libspffn.so is missing and could not be built: %s" % e) from e
    lib = ctypes.CDLL(so)
    vp, i32, sz = ctypes.c_void_p, ctypes.c_int32, ctypes.c_size_t
    st = ctypes.c_int
    sig = {
        "spffn_workspace_bytes": (sz, [ctypes.POINTER(Config)]),
        "spffn_create": (st, [ctypes.POINTER(Config), ctypes.POINTER(Weights), vp, sz, ctypes.POINTER(vp)]),
        "spffn_destroy": (st, [vp]),
        "spffn_predict": (st, [vp, vp, i32, vp, vp, vp]),
        "spffn_forward": (st, [vp, vp, i32, vp, vp, vp, vp]),
        "spffn_step": (st, [vp, vp, i32, vp, vp, vp, vp]),
        "spffn_chain": (st, [vp, vp, vp, i32, vp, vp]),
        "spffn_decode": (st, [ctypes.POINTER(vp), i32, vp, i32, vp, vp, vp, vp]),
        "spffn_decode_lookahead": (st, [ctypes.POINTER(vp), i32, vp, i32, vp, vp, vp, vp]),
        "spffn_layer_table": (st, [vp, ctypes.POINTER(vp)]),
        "spffn_decode_tables": (st, [ctypes.POINTER(vp), i32, vp, i32, ctypes.POINTER(vp), vp, vp, vp, vp, vp]),
        "spffn_profile_counts": (st, [vp, vp, i32, vp, vp]),
        "spffn_reorder": (st, [vp, i32, vp]),
        "spffn_reorder_dealt": (st, [vp, i32, i32, vp]),
        "spffn_forward_noalloc": (st, [ctypes.POINTER(Config), ctypes.POINTER(Weights), vp, i32, vp, vp, vp, vp]),
        "spffn_permute_rows": (st, [vp, vp, i32, i32, vp, vp]),
        "spffn_permute_vector": (st, [vp, vp, i32, vp, vp]),
        "spffn_last_device_error": (st, [vp, ctypes.POINTER(ctypes.c_uint32), vp]),
        "spffn_status_string": (ctypes.c_char_p, [st]),
        "spffn_num_partials": (i32, [vp]),
        "spffn_decode_kernel_launches": (i32, [ctypes.POINTER(vp), i32, i32]),
        "spffn_set_trace": (st, [vp, sz]),
        "spffn_set_wait_test": (st, [ctypes.c_uint64, i32]),
        "spffn_set_l2_hot_rows": (st, [i32]),
        "spffn_set_union_stack": (st, [i32]),
        "spffn_union_stack": (i32, []),
        "spffn_l2_hot_rows": (i32, []),
        "spffn_trace_marks": (i32, []),
        "spffn_last_cuda_error_string": (ctypes.c_char_p, []),
        "spffn_attn_workspace_bytes": (sz, [ctypes.POINTER(AttnConfig)]),
        "spffn_attn_create": (st, [ctypes.POINTER(AttnConfig), ctypes.POINTER(AttnWeights), vp, sz, ctypes.POINTER(vp)]),
        "spffn_attn_destroy": (st, [vp]),
        "spffn_attn_reset": (st, [vp, vp]),
        "spffn_attn_step": (st, [vp, vp, vp, vp, vp, vp]),
        "spffn_attn_cache": (st, [vp, ctypes.POINTER(AttnCacheView)]),
        "spffn_attn_step_kernel_launches": (i32, []),
        "spffn_attn_last_device_error": (st, [vp, ctypes.POINTER(ctypes.c_uint32), vp]),
    }
    for name, (res, args) in sig.items():
        f = getattr(lib, name)
        f.restype = res
        f.argtypes = args
    _lib = lib
    return lib


def _status_string(s: int) -> str:
    try:
        return library().spffn_status_string(s).decode()
    except Exception:
        return "status"


def _check(status: int, what: str):
    if status != OK:
        if status == ERR_CUDA:
            what = "%s [%s]" % (what, library().spffn_last_cuda_error_string().decode())
        raise SpffnError(status, what)


def _p(t) -> Optional[int]:
    """Device pointer of a CUDA tensor (None stays NULL)."""
    if t is None:
        return None
    if not getattr(t, "is_cuda", False):
        raise TypeError("expected a CUDA tensor, got %r" % (type(t),))
    if not t.is_contiguous():
        raise ValueError("tensor must be contiguous")
    return t.data_ptr()


def _stream(stream) -> Optional[int]:
    if stream is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    return getattr(stream, "cuda_stream", stream)


def _dtype_code(t) -> int:
    import torch
    if t.dtype == torch.float16:
        return F16
    if t.dtype == torch.bfloat16:
        return BF16
    raise TypeError("storage dtype must be float16 or bfloat16, got %s" % t.dtype)


def workspace_bytes(d: int, n: int, H: int, max_batch: int, dtype: int = F16) -> int:
    cfg = Config(d, n, H, max_batch, dtype, 0)
    return int(library().spffn_workspace_bytes(ctypes.byref(cfg)))


class Layer:
    """One FFN layer bound to the library (wraps an ``spffn_ctx``).

    Weight tensors (CUDA, row-major, float16 or bfloat16): ``W1[n,d]``, ``b1[n]``,
    ``W2T[n,d]`` (neuron-major FC2), ``b2[d]`` or None, ``Wp1[H,d]``, ``bp1[H]``
    or None, ``Wp2[n,H]``, ``bp2[n]`` or None.  The workspace is a zero-filled
    uint8 CUDA tensor (allocated here when not given).
    """

    def __init__(self, W1, b1, W2T, b2, Wp1, bp1, Wp2, bp2, max_batch: int = 1, workspace=None):
        import torch
        n, d = W1.shape
        H = Wp1.shape[0]
        self.d, self.n, self.H, self.max_batch = int(d), int(n), int(H), int(max_batch)
        self.dtype = _dtype_code(W1)
        self.cfg = Config(self.d, self.n, self.H, self.max_batch, self.dtype, 0)
        self._keep = [W1, b1, W2T, b2, Wp1, bp1, Wp2, bp2]
        self.weights = Weights(_p(W1), _p(b1), _p(W2T), _p(b2), _p(Wp1), _p(bp1), _p(Wp2), _p(bp2))
        need = int(library().spffn_workspace_bytes(ctypes.byref(self.cfg)))
        if need == 0:
            raise SpffnError(ERR_INVALID_ARG, "spffn_workspace_bytes (bad shape)")
        if workspace is None:
            workspace = torch.zeros(need, dtype=torch.uint8, device=W1.device)
        self.workspace = workspace
        ctx = ctypes.c_void_p()
        _check(library().spffn_create(ctypes.byref(self.cfg), ctypes.byref(self.weights),
                                      _p(workspace), workspace.numel(), ctypes.byref(ctx)), "spffn_create")
        self.ctx = ctx

    @classmethod
    def from_device_layer(cls, L, max_batch: int = 1, workspace=None):
        return cls(L.W1, L.b1, L.W2T, L.b2, L.Wp1, L.bp1, L.Wp2, L.bp2, max_batch, workspace)

    def close(self):
        if getattr(self, "ctx", None):
            library().spffn_destroy(self.ctx)
            self.ctx = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    @property
    def num_partials(self) -> int:
        return int(library().spffn_num_partials(self.ctx))

    def predict(self, x, idx, count, stream=None):
        _check(library().spffn_predict(self.ctx, _p(x), x.shape[0], _p(idx), _p(count), _stream(stream)),
               "spffn_predict")

    def forward(self, x, idx, count, y, stream=None):
        _check(library().spffn_forward(self.ctx, _p(x), x.shape[0], _p(idx), _p(count), _p(y),
                                       _stream(stream)), "spffn_forward")

    def step(self, x, idx, count, y, stream=None):
        _check(library().spffn_step(self.ctx, _p(x), x.shape[0], _p(idx), _p(count), _p(y), _stream(stream)),
               "spffn_step")

    def chain(self, x, y, x_next, stream=None):
        _check(library().spffn_chain(self.ctx, _p(x), _p(y), x.shape[0], _p(x_next), _stream(stream)),
               "spffn_chain")

    def profile_counts(self, X, counts, stream=None):
        _check(library().spffn_profile_counts(self.ctx, _p(X), X.shape[0], _p(counts), _stream(stream)),
               "spffn_profile_counts")

    def table(self, count: int):
        """The neuron table the last decode left in this layer's workspace: an
        int32 view of its first ``count`` entries (spffn_layer_table)."""
        import torch
        ptr = ctypes.c_void_p()
        _check(library().spffn_layer_table(self.ctx, ctypes.byref(ptr)), "spffn_layer_table")
        off = int(ptr.value) - self.workspace.data_ptr()
        return self.workspace[off:off + 4 * int(count)].view(torch.int32)

    def last_device_error(self, stream=None):
        code = ctypes.c_uint32(0)
        s = library().spffn_last_device_error(self.ctx, ctypes.byref(code), _stream(stream))
        return s, int(code.value)


class AttnLayer:
    """One attention layer with its head predictor (wraps an ``spffn_attn_ctx``).

    Weight tensors (CUDA, row-major, float16 or bfloat16): ``Wq, Wk, Wv[nh*dh, d]``,
    ``WoT[nh*dh, d]`` (output projection stored head-major), ``Wa1[Ha, d]``,
    ``Wa2[nh, Ha]``; biases ``bq, bk, bv[nh*dh]``, ``bo[d]``, ``ba1[Ha]``,
    ``ba2[nh]`` or None.  The workspace (cache included) is a zero-filled uint8
    CUDA tensor, allocated here when not given.
    """

    def __init__(self, Wq, Wk, Wv, WoT, Wa1, Wa2, nh: int, tmax: int, bq=None, bk=None, bv=None, bo=None,
                 ba1=None, ba2=None, workspace=None):
        import torch
        rows, d = Wq.shape
        self.d, self.nh, self.dh, self.Ha, self.tmax = int(d), int(nh), int(rows) // int(nh), int(Wa1.shape[0]), int(tmax)
        self.dtype = _dtype_code(Wq)
        self.cfg = AttnConfig(self.d, self.nh, self.dh, self.Ha, self.tmax, self.dtype, 0)
        self._keep = [Wq, bq, Wk, bk, Wv, bv, WoT, bo, Wa1, ba1, Wa2, ba2]
        self.weights = AttnWeights(*[_p(t) for t in self._keep])
        need = int(library().spffn_attn_workspace_bytes(ctypes.byref(self.cfg)))
        if need == 0:
            raise SpffnError(ERR_INVALID_ARG, "spffn_attn_workspace_bytes (bad shape)")
        if workspace is None:
            workspace = torch.zeros(need, dtype=torch.uint8, device=Wq.device)
        self.workspace = workspace
        ctx = ctypes.c_void_p()
        _check(library().spffn_attn_create(ctypes.byref(self.cfg), ctypes.byref(self.weights), _p(workspace),
                                           workspace.numel(), ctypes.byref(ctx)), "spffn_attn_create")
        self.ctx = ctx

    def close(self):
        if getattr(self, "ctx", None):
            library().spffn_attn_destroy(self.ctx)
            self.ctx = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    def step(self, y, heads, count, out, stream=None):
        """One decode step: y [d] -> out [d] (fp32); heads [nh], count [1] (int32)."""
        _check(library().spffn_attn_step(self.ctx, _p(y), _p(heads), _p(count), _p(out), _stream(stream)),
               "spffn_attn_step")

    def reset(self, stream=None):
        _check(library().spffn_attn_reset(self.ctx, _stream(stream)), "spffn_attn_reset")

    def cache(self):
        """(K, V, filled, Y, t) views of the cache as torch tensors on the workspace."""
        import torch
        v = AttnCacheView()
        _check(library().spffn_attn_cache(self.ctx, ctypes.byref(v)), "spffn_attn_cache")
        base = self.workspace.data_ptr()
        dt = torch.bfloat16 if self.dtype == BF16 else torch.float16
        def view(ptr, nbytes):
            off = int(ptr) - base
            return self.workspace[off:off + nbytes]
        kv = self.nh * self.tmax * self.dh
        K = view(v.K, 2 * kv).view(dt).view(self.nh, self.tmax, self.dh)
        V = view(v.V, 2 * kv).view(dt).view(self.nh, self.tmax, self.dh)
        filled = view(v.filled, self.nh * self.tmax).view(self.nh, self.tmax)
        Y = view(v.Y, 2 * self.tmax * self.d).view(dt).view(self.tmax, self.d)
        t = view(v.t, 4).view(torch.int32)
        return K, V, filled, Y, t

    def last_device_error(self, stream=None):
        code = ctypes.c_uint32(0)
        s = library().spffn_attn_last_device_error(self.ctx, ctypes.byref(code), _stream(stream))
        return s, int(code.value)


def attn_step_kernel_launches() -> int:
    return int(library().spffn_attn_step_kernel_launches())


def forward_noalloc(layer: Layer, x, idx, count, y, stream=None):
    """spffn_forward for `layer`'s weights without its context or workspace
    (scratch in the library's fixed device array; see include/spffn.h)."""
    _check(library().spffn_forward_noalloc(ctypes.byref(layer.cfg), ctypes.byref(layer.weights), _p(x), x.shape[0],
                                           _p(idx), _p(count), _p(y), _stream(stream)), "spffn_forward_noalloc")


def decode(layers: Sequence[Layer], x_in, x_out, y, counts=None, stream=None, lookahead: bool = False):
    """One decode step through the stack (spffn_decode; with ``lookahead`` the
    set of layer l+1 is predicted from x_l, spffn_decode_lookahead)."""
    arr = (ctypes.c_void_p * len(layers))(*[l.ctx.value for l in layers])
    fn = library().spffn_decode_lookahead if lookahead else library().spffn_decode
    _check(fn(arr, len(layers), _p(x_in), x_in.shape[0], _p(x_out), _p(y), _p(counts), _stream(stream)),
           "spffn_decode_lookahead" if lookahead else "spffn_decode")


def decode_tables(layers: Sequence[Layer], x_in, tables, tab_counts, x_out, y, counts=None, stream=None):
    """One decode step on caller-supplied neuron tables, no predictor
    (spffn_decode_tables): ``tables`` is a sequence of L int32 CUDA tensors,
    ``tab_counts`` an int32 CUDA tensor [L] of their lengths."""
    arr = (ctypes.c_void_p * len(layers))(*[l.ctx.value for l in layers])
    tabs = (ctypes.c_void_p * len(tables))(*[_p(t) for t in tables])
    _check(library().spffn_decode_tables(arr, len(layers), _p(x_in), x_in.shape[0], tabs, _p(tab_counts),
                                         _p(x_out), _p(y), _p(counts), _stream(stream)), "spffn_decode_tables")


def decode_kernel_launches(layers: Sequence[Layer], B: int) -> int:
    arr = (ctypes.c_void_p * len(layers))(*[l.ctx.value for l in layers])
    return int(library().spffn_decode_kernel_launches(arr, len(layers), B))


def set_trace(buf=None):
    """Bind (or unbind with None) a uint64 CUDA tensor that whole-stack decode
    launches fill with per-(CTA, layer, mark) %globaltimer stamps."""
    if buf is None:
        _check(library().spffn_set_trace(None, 0), "spffn_set_trace")
    else:
        _check(library().spffn_set_trace(_p(buf), buf.numel() * buf.element_size()), "spffn_set_trace")


def trace_marks() -> int:
    return int(library().spffn_trace_marks())


def set_l2_hot_rows(rows_per_range: int):
    """Keep the first ``rows_per_range`` slots of every dealt range (the hottest
    neurons after the hot-first dealt placement) in L2 during small-batch decode
    (spffn_set_l2_hot_rows; 0 turns the cache hints off)."""
    _check(library().spffn_set_l2_hot_rows(int(rows_per_range)), "spffn_set_l2_hot_rows")


def l2_hot_rows() -> int:
    return int(library().spffn_l2_hot_rows())


UNION_PER_LAYER, UNION_STACK, UNION_AUTO = 0, 1, 2


def set_union_stack(mode: int):
    """How decode runs 3 <= B <= 128 (spffn_set_union_stack): UNION_STACK (one
    persistent launch), UNION_PER_LAYER, or UNION_AUTO (the default: the faster
    of the two on the measured shapes, per-layer launches at every batch)."""
    _check(library().spffn_set_union_stack(int(mode)), "spffn_set_union_stack")


def union_stack() -> int:
    return int(library().spffn_union_stack())


def reorder(counts: np.ndarray) -> np.ndarray:
    c = np.ascontiguousarray(counts, dtype=np.uint32)
    perm = np.empty(c.size, dtype=np.int32)
    _check(library().spffn_reorder(c.ctypes.data_as(ctypes.c_void_p), c.size,
                                   perm.ctypes.data_as(ctypes.c_void_p)), "spffn_reorder")
    return perm


def reorder_dealt(counts: np.ndarray, parts: int) -> np.ndarray:
    c = np.ascontiguousarray(counts, dtype=np.uint32)
    perm = np.empty(c.size, dtype=np.int32)
    _check(library().spffn_reorder_dealt(c.ctypes.data_as(ctypes.c_void_p), c.size, parts,
                                         perm.ctypes.data_as(ctypes.c_void_p)), "spffn_reorder_dealt")
    return perm


def permute_rows(src, dst, perm, stream=None):
    rows = src.shape[0]
    row_bytes = src[0].numel() * src.element_size()
    _check(library().spffn_permute_rows(_p(src), _p(dst), rows, row_bytes, _p(perm), _stream(stream)),
           "spffn_permute_rows")


def permute_vector(src, dst, perm, stream=None):
    _check(library().spffn_permute_vector(_p(src), _p(dst), src.numel(), _p(perm), _stream(stream)),
           "spffn_permute_vector")
