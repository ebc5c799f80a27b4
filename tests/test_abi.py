"""The C-ABI library on CPU: it loads, exports every declared entry point, and
its host-side logic (validation, workspace sizing, hot-first reorder) behaves."""
import ctypes
import os
import re

import numpy as np
import pytest

import activation_sparse_ffn_predictor_b200 as sp
import oracle as O

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared_symbols():
    out = []
    for f in sorted(os.listdir(os.path.join(ROOT, "include"))):
        if f.endswith(".h"):
            txt = open(os.path.join(ROOT, "include", f)).read()
            txt = re.sub(r"/\*.*?\*/", "", txt, flags=re.S)
            out += re.findall(r"^\s*[A-Za-z_][\w\s\*]*?\b(spffn_\w+)\s*\(", txt, flags=re.M)
    return sorted(set(out))


def test_library_exports_every_declared_symbol():
    lib = sp.library()
    syms = declared_symbols()
    assert len(syms) >= 15
    for s in syms:
        assert hasattr(lib, s), s
    assert set(sp.EXPORTS) <= set(syms)


def test_library_is_built_for_sm100a_only():
    """The build compiles every source for sm_100a and nothing else."""
    from activation_sparse_ffn_predictor_b200 import build
    flags = " ".join(build.FLAGS)
    assert "-gencode arch=compute_100a,code=sm_100a" in flags
    assert flags.count("-gencode") == 1 and "-arch" not in build.FLAGS


def test_status_strings():
    lib = sp.library()
    assert lib.spffn_status_string(0) == b"ok"
    assert lib.spffn_status_string(3).startswith(b"workspace")


def test_workspace_bytes_validation():
    ok = sp.workspace_bytes(4096, 16384, 1024, 1)
    assert ok > 16384 // 32 * 4 + 1024 * 4
    assert sp.workspace_bytes(4096, 16384, 1024, 32) > ok
    assert sp.workspace_bytes(4096, 16384, 1024, 256) > sp.workspace_bytes(4096, 16384, 1024, 32)
    for bad in [(4000, 16384, 1024, 1), (4096, 16383, 1024, 1), (4096, 16384, 1000, 1),
                (4096, 16384, 1024, 0), (4096, 16384, 1024, 257), (32, 64, 64, 1)]:
        assert sp.workspace_bytes(*bad) == 0, bad
    assert sp.workspace_bytes(4096, 16384, 1024, 1, dtype=2) == 0


def test_create_rejects_bad_arguments_on_host():
    lib = sp.library()
    cfg = sp.Config(1024, 4096, 256, 1, 0, 0)
    need = lib.spffn_workspace_bytes(ctypes.byref(cfg))
    fake = 1 << 40  # never dereferenced by create
    w = sp.Weights(fake, fake, fake, None, fake, None, fake, fake)
    ctx = ctypes.c_void_p()
    assert lib.spffn_create(ctypes.byref(cfg), ctypes.byref(w), fake, need - 1, ctypes.byref(ctx)) == sp.ERR_WORKSPACE
    assert lib.spffn_create(ctypes.byref(cfg), ctypes.byref(w), fake + 16, need, ctypes.byref(ctx)) == sp.ERR_WORKSPACE
    bad = sp.Weights(fake + 2, fake, fake, None, fake, None, fake, fake)
    assert lib.spffn_create(ctypes.byref(cfg), ctypes.byref(bad), fake, need, ctypes.byref(ctx)) == sp.ERR_INVALID_ARG
    miss = sp.Weights(None, fake, fake, None, fake, None, fake, fake)
    assert lib.spffn_create(ctypes.byref(cfg), ctypes.byref(miss), fake, need, ctypes.byref(ctx)) == sp.ERR_INVALID_ARG
    assert lib.spffn_create(ctypes.byref(cfg), ctypes.byref(w), fake, need, ctypes.byref(ctx)) == sp.OK
    # entry points validate before enqueuing anything
    assert lib.spffn_predict(ctx, fake, 0, fake, fake, None) == sp.ERR_INVALID_ARG
    assert lib.spffn_predict(ctx, fake, 2, fake, fake, None) == sp.ERR_INVALID_ARG
    assert lib.spffn_forward(ctx, fake + 8, 1, fake, fake, fake, None) == sp.ERR_INVALID_ARG
    assert lib.spffn_forward(ctx, fake, 1, None, fake, fake, None) == sp.ERR_INVALID_ARG
    assert lib.spffn_chain(ctx, fake, fake, 1, fake, None) == sp.ERR_INVALID_ARG     # aliasing
    arr = (ctypes.c_void_p * 1)(ctx.value)
    assert lib.spffn_decode(arr, 0, fake, 1, fake + 256, fake, None, None) == sp.ERR_INVALID_ARG
    assert lib.spffn_permute_rows(fake, fake + 4096, 8, 20, fake, None) == sp.ERR_INVALID_ARG
    assert lib.spffn_destroy(ctx) == sp.OK
    assert lib.spffn_destroy(None) == sp.OK


def test_reorder_matches_oracle():
    r = np.random.default_rng(0)
    for n in (1, 7, 64, 5000):
        c = r.integers(0, 6, n).astype(np.uint32)   # many ties
        assert np.array_equal(sp.reorder(c), O.hot_first_order(c))


def test_reorder_dealt_matches_oracle():
    r = np.random.default_rng(1)
    for n, parts in ((7, 3), (64, 148), (4096, 148), (16384, 148), (1000, 7)):
        c = r.integers(0, 50, n).astype(np.uint32)
        got = sp.reorder_dealt(c, parts)
        want = O.dealt_order(c, parts)
        assert np.array_equal(got, want)
        assert sorted(got.tolist()) == list(range(n))
