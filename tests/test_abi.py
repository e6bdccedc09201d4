"""The C ABI library on the host: it loads, exports every declared entry point,
and its host-side arithmetic (config checks, workspace and KV-byte figures)
behaves as documented.  No GPU needed."""
import ctypes
import os
import re

import pytest

from cross_loop_sparsity_b200 import build as fl_build
from cross_loop_sparsity_b200 import flashloop as fl
from cross_loop_sparsity_b200 import synth

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def L():
    fl_build.build()
    return fl.lib()


def _declared():
    src = open(os.path.join(ROOT, "include", "flashloop.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b((?:flashloop|fl_test|fl_gemm)_[a-z_]+)\s*\(", src)))


def test_every_declared_symbol_is_exported(L):
    names = _declared()
    assert len(names) >= 20
    for n in names:
        assert hasattr(L, n), n


def test_binding_covers_every_symbol():
    assert set(_declared()) == set(fl._SIG)


def _cfg(name, **kw):
    cfg = synth.config(name)
    return fl.make_config(cfg, kw.pop("mb", cfg.batch), kw.pop("ctx", cfg.max_ctx + 64),
                          kw.pop("mt", cfg.batch * cfg.seq_len), **kw)


def test_workspace_bytes_valid_and_invalid(L):
    for name in ("c1", "c2", "c3", "c5"):
        assert fl.workspace_bytes(_cfg(name)) > 0
    bad = [dict(d_model=100), dict(head_dim=96), dict(n_kv_heads=3), dict(resid_bits=3), dict(group_size=48),
           dict(rho=0.0), dict(rho=1.5), dict(c_cols=0), dict(n_loops=0), dict(n_loops=17), dict(max_batch=0),
           dict(ffn_dim=10)]
    for b in bad:
        c = _cfg("c1")
        for k, v in b.items():
            setattr(c, k, v)
        assert fl.workspace_bytes(c) == 0, b


def _kv_per_token_layer(cfg, bits):
    """Bytes per token and layer of the cache layout, from its definition."""
    kv_rows = 2 * cfg.n_kv_heads
    if bits == 16:
        return kv_rows * cfg.n_loops * cfg.head_dim * 2
    base = cfg.head_dim * 2
    resid = cfg.head_dim * bits // 8 + (cfg.head_dim // cfg.group_size) * 2
    return kv_rows * (base + (cfg.n_loops - 1) * resid)


@pytest.mark.parametrize("name,lazy,dense", [("c1", 1888, 4096), ("c2", 3680, 8192), ("c3", 2592, 4096),
                                             ("c4", 7264, 16384), ("c5", 5856, 16384), ("c5_int2", 4064, 16384)])
def test_kv_bytes_per_token(L, name, lazy, dense):
    cfg = synth.config(name)
    c = _cfg(name)
    tot, per, den = fl.kv_bytes_for(c)
    assert per == lazy == _kv_per_token_layer(cfg, cfg.resid_bits)
    assert den == dense == _kv_per_token_layer(cfg, 16)
    assert tot == int(per * cfg.n_layers * c.max_batch * c.max_ctx)


def test_status_strings(L):
    for s in range(8):
        assert L.flashloop_status_string(s)


def test_init_rejects_bad_arguments_without_touching_the_gpu(L):
    c = _cfg("c1")
    ctx = ctypes.c_void_p()
    w = fl.Weights()   # all NULL
    st = L.flashloop_init(ctypes.byref(c), ctypes.byref(w), None, 0, None, ctypes.byref(ctx))
    assert st == 1 and not ctx.value
    c.head_dim = 96
    st = L.flashloop_init(ctypes.byref(c), ctypes.byref(w), None, 0, None, ctypes.byref(ctx))
    assert st == 1


def test_unit_entry_points_reject_bad_sizes(L):
    assert L.fl_test_quantize(None, 1, 128, 64, 4, None, None, None) == 1
    assert L.fl_test_topk(None, 1, 10, 3, None, None) == 1
    assert L.fl_test_gemm(None, None, None, 1, 1, 8, 0, None, 0, None) == 1
    assert L.fl_test_gemm_scratch_bytes(65, 128, 64, 1) == 0


def test_last_loop_kv_bytes_are_one_pass(L):
    """last_loop keeps one pass of dense KV: K times fewer bytes than per_loop."""
    from cross_loop_sparsity_b200 import flashloop as fl
    cfg = synth.config("c2").with_(resid_bits=16)
    per = fl.kv_bytes_for(fl.make_config(cfg, 8, 4097))
    last = fl.kv_bytes_for(fl.make_config(cfg.with_(kv_mode=1), 8, 4097))
    assert per[1] == per[2] == cfg.n_loops * last[1]
    assert last[2] == per[2] and per[0] == cfg.n_loops * last[0]
    # last_loop is a dense-path mode: the lazy path rejects it
    bad = fl.make_config(cfg.with_(resid_bits=4, kv_mode=1), 8, 4097)
    assert L.flashloop_workspace_bytes(bad) == 0


@pytest.mark.parametrize("name,floor", [("c2", 3.5), ("c5", 5.0), ("c5_int2", 5.0)])
def test_sparse_residual_storage_kv_bytes(L, name, floor):
    """Residual rows for the recomputed tokens only (a pool sized to the
    context's recompute rate plus the batch's new tokens) and a 4-byte row index
    per (layer, loop, position): bf16 base + (K-1) x (pool fraction x row bytes
    + 4) per token and layer."""
    cfg = synth.config(name)
    rows = synth.sparse_rows(cfg, cfg.batch)
    c = fl.make_config(cfg.with_(resid_rows=rows), cfg.batch, cfg.max_ctx)
    tot, per, dense = fl.kv_bytes_for(c)
    kv, hd, K = 2 * cfg.n_kv_heads, cfg.head_dim, cfg.n_loops
    row = hd * cfg.resid_bits / 8 + (hd // cfg.group_size) * 2
    assert per == pytest.approx(kv * hd * 2 + (K - 1) * (kv * row * rows / cfg.max_ctx + 4))
    assert dense / per >= floor
    # the dense layout of the same config keeps every position's residual rows
    _, per_dense_layout, _ = fl.kv_bytes_for(fl.make_config(cfg, cfg.batch, cfg.max_ctx))
    assert per < per_dense_layout
    assert L.flashloop_workspace_bytes(ctypes.byref(c)) > 0
    # the pool cannot be larger than the context, and is a lazy-path layout
    assert L.flashloop_workspace_bytes(ctypes.byref(fl.make_config(cfg.with_(resid_rows=cfg.max_ctx + 1), cfg.batch,
                                                                   cfg.max_ctx))) == 0
    assert L.flashloop_workspace_bytes(ctypes.byref(fl.make_config(cfg.with_(resid_rows=rows, resid_bits=16),
                                                                   cfg.batch, cfg.max_ctx))) == 0
