"""The C-ABI library loads, exports every entry point include/lfm3.h declares, and refuses bad
arguments on the host (no GPU needed: lfm3_create touches no device memory)."""
import ctypes as C
import os
import re

import pytest

from conftest import ROOT


@pytest.fixture(scope="module")
def L():
    from attention_decoder_b200 import build
    build.build(verbose=False)  # no-op when liblfm3.so is current
    from attention_decoder_b200 import _lib
    return _lib


def declared_symbols():
    text = open(os.path.join(ROOT, "include", "lfm3.h")).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(lfm3_[a-z_]+)\s*\(", text)))


def test_every_declared_symbol_is_exported(L):
    lib = L.lib()
    decl = declared_symbols()
    assert decl == sorted(L.SYMBOLS)
    for name in decl:
        assert hasattr(lib, name), name


def _config(L, **kw):
    from lfm3_inputs import lfm3_1p7b
    g = lfm3_1p7b()
    cfg = L.lfm3_config()
    cfg.n_layers = g.n_layers
    for i, t in enumerate(g.layer_types):
        cfg.layer_type[i] = t
    cfg.d_model, cfg.d_ffn, cfg.n_q, cfg.n_kv, cfg.head_dim = 2048, 7680, 16, 4, 128
    cfg.conv_taps, cfg.window, cfg.vocab = 7, 256, 128000
    cfg.theta_full, cfg.theta_sliding, cfg.rope_pairs_full, cfg.eps = 1e6, 1e4, 32, 1e-5
    cfg.has_head, cfg.ffn_format, cfg.page_size, cfg.n_pages = 1, 0, 64, 64
    cfg.max_streams, cfg.max_pages_per_stream, cfg.max_chunk, cfg.max_batch = 1, 64, 2048, 1
    for k, v in kw.items():
        setattr(cfg, k, v)
    return cfg


def _weights(L, n_layers=24, null_field=None):
    layers = (L.lfm3_layer_weights * n_layers)()
    fake = 0x10000  # never dereferenced by lfm3_create
    for i in range(n_layers):
        for name, ctype in L.lfm3_layer_weights._fields_:
            if ctype is C.c_void_p:
                setattr(layers[i], name, fake)
        if null_field:
            setattr(layers[i], null_field, None)
    w = L.lfm3_weights()
    w.embed = fake
    w.final_norm = fake
    w.layers = C.cast(layers, C.POINTER(L.lfm3_layer_weights))
    return w, layers


def _create(L, cfg, w):
    ctx = C.c_void_p()
    ws = C.c_size_t()
    st = L.lfm3_create(C.byref(cfg), C.byref(w), C.byref(ws), C.byref(ctx))
    return st, ctx, ws.value


def test_create_accepts_the_lfm3_geometry_and_sizes_the_workspace(L):
    w, keep = _weights(L)
    st, ctx, ws = _create(L, _config(L), w)
    try:
        assert st == 0
        assert ctx.value
        # at least the fp32 residual + bf16 activations of 2048 rows and the rotary tables
        assert ws > 2048 * 2048 * 4 + 4 * 4096 * 64 * 4
        assert L.lfm3_last_error(ctx) == b""
    finally:
        L.lfm3_free(ctx)


@pytest.mark.parametrize("field,value,status,word", [
    ("d_model", 4096, -5, b"d_model"),
    ("head_dim", 64, -5, b"head_dim"),
    ("window", 512, -5, b"window"),
    ("conv_taps", 3, -5, b"conv_taps"),
    ("vocab", 1000, -5, b"vocab"),
    ("n_layers", 0, -2, b"n_layers"),
    ("max_chunk", 4096, -2, b"max_chunk"),
    ("max_batch", 65, -2, b"max_batch"),
    ("ffn_format", 7, -5, b"Ffn"),
])
def test_create_refuses_by_name(L, field, value, status, word):
    w, keep = _weights(L)
    st, ctx, ws = _create(L, _config(L, **{field: value}), w)
    assert st == status
    assert not ctx.value
    assert word in L.lfm3_last_error(None)


def test_create_refuses_missing_weights(L):
    w, keep = _weights(L, null_field="o_proj")
    st, ctx, _ = _create(L, _config(L), w)
    assert st == -1 and not ctx.value
    assert b"NULL" in L.lfm3_last_error(None)


def test_calls_before_binding_a_workspace_are_refused(L):
    w, keep = _weights(L)
    st, ctx, ws = _create(L, _config(L), w)
    assert st == 0
    try:
        state = L.lfm3_state()
        assert L.lfm3_prefill(ctx, C.byref(state), 0, None, None, 1, None, None, None, None) == -7
        assert b"workspace" in L.lfm3_last_error(ctx)
        # a misaligned workspace is refused before any device call
        assert L.lfm3_bind_workspace(ctx, C.c_void_p(0x10001), ws) == -1
        assert L.lfm3_bind_workspace(ctx, C.c_void_p(0x10000), ws - 1) == -1
    finally:
        L.lfm3_free(ctx)
