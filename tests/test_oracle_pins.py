"""Pins of the CPU oracle against things other than itself (CPU only).

Each test ties one oracle function to a library routine, a closed form, brute
force or a figure the pages print, so that a dropped term, a wrong sign or
index or a transposed operand in the oracle fails here.
"""
import math

import numpy as np
import pytest
import torch
import torch.nn.functional as Fn

from conftest import read_golden
from lfm3_inputs import (CONV, FULL, SLIDING, lfm3_1p7b, lfm3_slice3, tiny_geometry, make_weights,
                         nvfp4_draw, rng_for, bf16_bits)
from oracle import Lfm3Oracle, rms_norm, rope_inv_freq, apply_rope, e2m1_value, e4m3_value, nvfp4_dequant
from oracle.lfm3 import causal_conv_full, causal_conv_chunk, sigmoid, silu, _bf16
from oracle.nvfp4 import nvfp4_unpack_codes, nvfp4_block_values


# ---------------------------------------------------------------- geometry and the export's totals

def test_geometry_matches_pages():
    gold = read_golden("lfm3_geometry.txt")
    g = lfm3_1p7b()
    assert g.n_layers == gold["n_layers"]
    assert (g.d_model, g.d_ffn, g.n_q, g.n_kv, g.head_dim) == (
        gold["d_model"], gold["d_ffn"], gold["n_q"], gold["n_kv"], gold["head_dim"])
    assert g.conv_taps == gold["conv_taps"] and g.conv_taps - 1 == gold["conv_state_cols"]
    assert (g.count(CONV), g.count(FULL), g.count(SLIDING)) == (gold["n_conv"], gold["n_full"], gold["n_sliding"])
    assert g.window == gold["window"] and g.vocab == gold["vocab"]
    assert g.theta_full == gold["theta_full"] and g.theta_sliding == gold["theta_sliding"]
    assert g.rope_pairs_full == gold["rope_pairs_full"] and g.rope_pairs_full * 2 == g.head_dim // 2
    assert g.n_q == gold["gate_outputs"] and g.eps == gold["eps"]


def _nvfp4_export_totals(g):
    """Tensor count and bytes of a weight-only NVFP4 export of geometry g: FFN w1/w3/w2 as
    packed E2M1 (half a byte each) + one E4M3 byte per 16 weights + fp32 weight_scale_2 and
    input_scale; everything else bf16; q, k, v, gate as separate tensors."""
    D, F, d = g.d_model, g.d_ffn, g.head_dim
    tensors = 2  # embedding, final norm
    nbytes = 2 * (g.vocab * D + D)
    for kind in g.layer_types:
        tensors += 4
        nbytes += 2 * 4 * D
        if kind == CONV:
            tensors += 3
            nbytes += 2 * (3 * D * D + D * g.conv_taps + D * D)
        else:
            tensors += 7
            nbytes += 2 * (g.n_q * d * D + 2 * g.n_kv * d * D + g.n_q * D + 2 * d + D * g.n_q * d)
        for (n, k) in ((F, D), (F, D), (D, F)):
            tensors += 4
            nbytes += n * k // 2 + n * k // 16 + 4 + 4
    return tensors, nbytes


def test_nvfp4_export_total_pins_geometry_and_g16():
    gold = read_golden("nvfp4_export_header.txt")
    t, b = _nvfp4_export_totals(lfm3_1p7b())
    assert t == gold["text_tensors"]
    assert b == gold["total_bytes"]
    # a group size of 32, or a 7168-wide FFN, would miss the published total
    g = lfm3_1p7b(d_ffn=7168)
    assert _nvfp4_export_totals(g)[1] != gold["total_bytes"]


def test_generator_weight_bytes_match_export_layout():
    # the generator's NVFP4 arrays have exactly the export's per-tensor sizes
    codes, scales = nvfp4_draw(0, "x", 32, 64)
    assert codes.shape == (32, 32) and scales.shape == (32, 4)


# ---------------------------------------------------------------- NVFP4

def test_e2m1_table_is_ocp():
    gold = open(__file__.replace("test_oracle_pins.py", "golden/e2m1_ocp.txt")).read().split("\n")
    vals = [float(v) for line in gold if line and not line.startswith("#") for v in line.split()]
    assert len(vals) == 16
    for c in range(16):
        assert e2m1_value(c) == vals[c]
        assert math.copysign(1.0, e2m1_value(c)) == math.copysign(1.0, vals[c])


def test_e4m3_all_bytes_against_torch():
    b = torch.arange(256, dtype=torch.uint8)
    ref = b.view(torch.float8_e4m3fn).to(torch.float64).numpy()
    mine = np.array([e4m3_value(i) for i in range(256)])
    nan = np.isnan(ref)
    assert np.array_equal(nan, np.isnan(mine))
    assert nan.sum() == 2  # 0x7F and 0xFF
    assert np.array_equal(ref[~nan], mine[~nan])


def test_nvfp4_nibble_order_matches_generator():
    n, k = 8, 64
    codes, scales = nvfp4_draw(3, "w", n, k)
    drawn = rng_for(3, "w.codes").integers(0, 16, size=(n, k), dtype=np.uint8)
    assert np.array_equal(nvfp4_unpack_codes(codes), drawn)


def test_nvfp4_dequant_bruteforce_and_bf16_exact():
    n, k = 16, 128
    codes, scales = nvfp4_draw(5, "w", n, k)
    s = 2.0 ** -8
    w = nvfp4_dequant(codes, scales, s)
    drawn = rng_for(5, "w.codes").integers(0, 16, size=(n, k), dtype=np.uint8)
    sc = torch.from_numpy(scales).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    table = [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]
    for i in range(n):
        for j in range(k):
            c = int(drawn[i, j])
            v = (-1.0 if c & 8 else 1.0) * table[c & 7]
            assert w[i, j] == v * sc[i, j // 16] * s
    # E2M1 x E4M3 products are exact in bf16 (<= 6 significant bits)
    bv = nvfp4_block_values(codes, scales)
    assert np.array_equal(_bf16(bf16_bits(bv)), bv)
    # scales were drawn log-uniform in [2^-6, 2^2] and rounded to E4M3
    assert sc.min() >= 2.0 ** -6 and sc.max() <= 4.0


# ---------------------------------------------------------------- RMSNorm, SiLU, sigmoid

def test_rms_norm_against_torch_and_closed_form():
    r = np.random.default_rng(0)
    x = r.standard_normal((5, 64))
    g = 1 + 0.02 * r.standard_normal(64)
    ref = Fn.rms_norm(torch.from_numpy(x), (64,), weight=torch.from_numpy(g), eps=1e-5).numpy()
    assert np.allclose(rms_norm(x, g, 1e-5), ref, rtol=1e-12, atol=1e-12)
    c = 0.3
    y = rms_norm(np.full(8, c), np.ones(8), 1e-5)
    assert np.allclose(y, c / math.sqrt(c * c + 1e-5))


def test_silu_sigmoid_against_torch():
    x = np.linspace(-30, 30, 101)
    assert np.allclose(silu(x), Fn.silu(torch.from_numpy(x)).numpy(), rtol=1e-13, atol=1e-15)
    assert np.allclose(sigmoid(x), torch.sigmoid(torch.from_numpy(x)).numpy(), rtol=1e-13, atol=1e-15)


# ---------------------------------------------------------------- conv

def test_causal_conv_against_numpy_convolve_and_torch_conv1d():
    r = np.random.default_rng(1)
    T, C, taps = 23, 5, 7
    bx = r.standard_normal((T, C))
    w = r.standard_normal((C, taps))
    z = causal_conv_full(bx, w)
    for c in range(C):
        # full convolution of the sequence with the reversed taps, first T outputs
        ref = np.convolve(bx[:, c], w[c, ::-1])[:T]
        assert np.allclose(z[:, c], ref, rtol=1e-12, atol=1e-12)
    # torch Conv1d [channels, 1, taps] with padding taps-1, first T outputs
    t = Fn.conv1d(torch.from_numpy(bx.T[None]), torch.from_numpy(w[:, None, :]), padding=taps - 1, groups=C)
    assert np.allclose(z, t[0, :, :T].numpy().T, rtol=1e-12, atol=1e-12)


@pytest.mark.parametrize("cut", [0, 1, 3, 6, 7, 12, 22])
def test_conv_state_carry_equals_one_shot(cut):
    r = np.random.default_rng(2)
    T, C, taps = 23, 4, 7
    bx = r.standard_normal((T, C))
    w = r.standard_normal((C, taps))
    z_all = causal_conv_full(bx, w)
    st = np.zeros((taps - 1, C))
    z1, st = causal_conv_chunk(st, bx[:cut], w)
    # the carried state is the last 6 columns of B*x (zeros before the start)
    padded = np.concatenate([np.zeros((taps - 1, C)), bx])
    assert np.array_equal(st, padded[cut:cut + taps - 1])
    z2, st = causal_conv_chunk(st, bx[cut:], w)
    assert np.allclose(np.concatenate([z1, z2]), z_all, rtol=1e-12, atol=1e-12)


# ---------------------------------------------------------------- rotary

def test_inv_freq_closed_form():
    f = rope_inv_freq(1e6, 128, 32)
    assert f[0] == 1.0
    assert math.isclose(f[1], 1e6 ** (-2 / 128), rel_tol=1e-15)
    assert math.isclose(f[31], 1e6 ** (-62 / 128), rel_tol=1e-15)
    assert np.all(f[32:] == 0)
    s = rope_inv_freq(1e4, 128, 64)
    assert math.isclose(s[63], 1e4 ** (-126 / 128), rel_tol=1e-15) and np.all(s > 0)


def test_rope_against_complex_rotation():
    r = np.random.default_rng(3)
    T, H, d = 9, 3, 128
    x = r.standard_normal((T, H, d))
    pos = np.array([0, 1, 2, 17, 255, 256, 1000, 8191, 32767])
    for theta, pairs in ((1e6, 32), (1e4, 64)):
        f = rope_inv_freq(theta, d, pairs)
        y = apply_rope(x, pos, f)
        z = x[..., :64] + 1j * x[..., 64:]
        zr = z * np.exp(1j * pos[:, None, None] * f[None, None, :])
        assert np.allclose(y[..., :64], zr.real, atol=1e-12)
        assert np.allclose(y[..., 64:], zr.imag, atol=1e-12)


def test_partial_rope_passes_through_32_63_and_96_127():
    r = np.random.default_rng(4)
    x = r.standard_normal((4, 2, 128))
    pos = np.array([5, 77, 300, 4000])
    y = apply_rope(x, pos, rope_inv_freq(1e6, 128, 32))
    assert np.array_equal(y[..., 32:64], x[..., 32:64])
    assert np.array_equal(y[..., 96:128], x[..., 96:128])
    # dims 0..31 pair with 64..95 (not "the first 64 dims")
    assert not np.allclose(y[..., 64:96], x[..., 64:96])
    # unit vector e0 at position p turns into (cos p, sin p) on dims (0, 64)
    e = np.zeros((1, 1, 128)); e[0, 0, 0] = 1.0
    p = 3
    ye = apply_rope(e, np.array([p]), rope_inv_freq(1e4, 128, 64))
    assert math.isclose(ye[0, 0, 0], math.cos(p)) and math.isclose(ye[0, 0, 64], math.sin(p))


def test_rope_relative_position_and_norm():
    r = np.random.default_rng(5)
    q = r.standard_normal((1, 1, 128))
    k = r.standard_normal((1, 1, 128))
    f = rope_inv_freq(1e4, 128, 64)
    dots = []
    for base in (0, 13, 1000):
        qa = apply_rope(q, np.array([base + 40]), f)
        ka = apply_rope(k, np.array([base + 7]), f)
        dots.append(float(np.sum(qa * ka)))
        assert math.isclose(np.linalg.norm(qa), np.linalg.norm(q), rel_tol=1e-12)
    assert np.allclose(dots, dots[0], rtol=1e-9)


# ---------------------------------------------------------------- attention

def _sdpa_reference(q, k, v, pos, window, gate):
    """torch SDPA (float64) with repeat-kv GQA and a boolean causal/window mask."""
    Hq, Hkv = q.shape[1], k.shape[1]
    tq = torch.from_numpy(q).permute(1, 0, 2)
    tk = torch.from_numpy(k).permute(1, 0, 2).repeat_interleave(Hq // Hkv, dim=0)
    tv = torch.from_numpy(v).permute(1, 0, 2).repeat_interleave(Hq // Hkv, dim=0)
    tp = torch.from_numpy(pos)
    diff = tp[:, None] - tp[None, :]
    mask = diff >= 0
    if window is not None:
        mask &= diff < window
    o = Fn.scaled_dot_product_attention(tq, tk, tv, attn_mask=mask)     # scale 1/sqrt(d)
    o = o.permute(1, 0, 2).numpy()
    return o * sigmoid(gate)[:, :, None]


@pytest.mark.parametrize("window", [None, 8, 3])
def test_attention_against_torch_sdpa(window):
    g = tiny_geometry()
    W = make_weights(g, 0)
    o = Lfm3Oracle(W)
    r = np.random.default_rng(6)
    T = 20
    q = r.standard_normal((T, g.n_q, g.head_dim))
    k = r.standard_normal((T, g.n_kv, g.head_dim))
    v = r.standard_normal((T, g.n_kv, g.head_dim))
    gate = r.standard_normal((T, g.n_q))
    pos = np.arange(T)
    mine = o._attend(q, pos, k, v, pos, window, gate).reshape(T, g.n_q, g.head_dim)
    assert np.allclose(mine, _sdpa_reference(q, k, v, pos, window, gate), rtol=1e-10, atol=1e-12)


def test_sliding_equals_full_when_sequence_fits_window():
    # "under 256 tokens the window never bites"
    g = tiny_geometry()
    o = Lfm3Oracle(make_weights(g, 0))
    r = np.random.default_rng(7)
    T = g.window
    q = r.standard_normal((T, g.n_q, g.head_dim))
    k = r.standard_normal((T, g.n_kv, g.head_dim))
    v = r.standard_normal((T, g.n_kv, g.head_dim))
    gate = r.standard_normal((T, g.n_q))
    pos = np.arange(T)
    assert np.array_equal(o._attend(q, pos, k, v, pos, g.window, gate), o._attend(q, pos, k, v, pos, None, gate))
    q2 = r.standard_normal((T + 1, g.n_q, g.head_dim))
    k2 = r.standard_normal((T + 1, g.n_kv, g.head_dim))
    v2 = r.standard_normal((T + 1, g.n_kv, g.head_dim))
    g2 = r.standard_normal((T + 1, g.n_q))
    p2 = np.arange(T + 1)
    assert not np.allclose(o._attend(q2, p2, k2, v2, p2, g.window, g2), o._attend(q2, p2, k2, v2, p2, None, g2))


def test_gate_limits():
    g = tiny_geometry()
    o = Lfm3Oracle(make_weights(g, 0))
    r = np.random.default_rng(8)
    T = 6
    q = r.standard_normal((T, g.n_q, g.head_dim))
    k = r.standard_normal((T, g.n_kv, g.head_dim))
    v = r.standard_normal((T, g.n_kv, g.head_dim))
    pos = np.arange(T)
    assert np.allclose(o._attend(q, pos, k, v, pos, None, np.full((T, g.n_q), -800.0)), 0.0, atol=1e-300)
    ungated = Lfm3Oracle(make_weights(g, 0), gate=False)._attend(q, pos, k, v, pos, None, np.zeros((T, g.n_q)))
    assert np.allclose(o._attend(q, pos, k, v, pos, None, np.full((T, g.n_q), 800.0)), ungated, rtol=1e-15)


# ---------------------------------------------------------------- blocks against torch primitives

def _t(a):
    return torch.from_numpy(np.asarray(a, dtype=np.float64))


def test_conv_block_against_torch_modules():
    g = tiny_geometry()
    W = make_weights(g, 0)
    o = Lfm3Oracle(W)
    O = o.layers[0]
    assert O["kind"] == CONV
    r = np.random.default_rng(9)
    T, D = 15, g.d_model
    xn = r.standard_normal((T, D))
    # LFM2-style ShortConv: in_proj -> chunk(B, C, x) over channels -> B*x -> Conv1d(groups=D,
    # padding=taps-1)[..., :T] -> C*conv -> out_proj
    bcx = Fn.linear(_t(xn), _t(O["in_proj"])).T
    B, C, X = bcx.chunk(3, dim=0)
    conv = Fn.conv1d((B * X)[None], _t(O["conv"])[:, None, :], padding=g.conv_taps - 1, groups=D)[0, :, :T]
    ref = Fn.linear((C * conv).T, _t(O["out_proj"])).numpy()
    assert np.allclose(o._conv_full(xn, O), ref, rtol=1e-10, atol=1e-12)


@pytest.mark.parametrize("kind", [FULL, SLIDING])
def test_attention_block_against_torch_modules(kind):
    g = tiny_geometry()
    W = make_weights(g, 0)
    o = Lfm3Oracle(W)
    li = [i for i, t in enumerate(g.layer_types) if t == kind][0]
    O = o.layers[li]
    r = np.random.default_rng(10)
    T, D, d = 19, g.d_model, g.head_dim
    xn = r.standard_normal((T, D))
    pos = np.arange(T)
    x = _t(xn)
    q = Fn.linear(x, _t(O["q_proj"])).view(T, g.n_q, d)
    k = Fn.linear(x, _t(O["k_proj"])).view(T, g.n_kv, d)
    v = Fn.linear(x, _t(O["v_proj"])).view(T, g.n_kv, d)
    gate = Fn.linear(x, _t(O["gate_proj"]))
    q = Fn.rms_norm(q, (d,), weight=_t(O["q_norm"]), eps=g.eps)
    k = Fn.rms_norm(k, (d,), weight=_t(O["k_norm"]), eps=g.eps)
    pairs = g.rope_pairs_full if kind == FULL else d // 2
    theta = g.theta_full if kind == FULL else g.theta_sliding
    f = np.array([theta ** (-2 * i / d) if i < pairs else 0.0 for i in range(d // 2)])
    rot = np.exp(1j * pos[:, None, None] * f[None, None, :])

    def rope(a):
        a = a.numpy()
        z = (a[..., :d // 2] + 1j * a[..., d // 2:]) * rot
        return np.concatenate([z.real, z.imag], axis=-1)
    att = _sdpa_reference(rope(q), rope(k), v.numpy(), pos, g.window if kind == SLIDING else None, gate.numpy())
    ref = Fn.linear(_t(att.reshape(T, -1)), _t(O["o_proj"])).numpy()
    assert np.allclose(o._attn_full(xn, O, pos, kind), ref, rtol=1e-9, atol=1e-12)


def test_swiglu_ffn_against_torch_and_nvfp4_equals_its_dequantised_bf16():
    g = tiny_geometry()
    W = make_weights(g, 0)
    o = Lfm3Oracle(W)
    O = o.layers[0]
    r = np.random.default_rng(11)
    hn = r.standard_normal((7, g.d_model))
    h = _t(hn)
    ref = Fn.linear(Fn.silu(Fn.linear(h, _t(O["w1"]))) * Fn.linear(h, _t(O["w3"])), _t(O["w2"])).numpy()
    assert np.allclose(o._ffn(hn, O), ref, rtol=1e-10, atol=1e-12)
    # NVFP4 FFN == a bf16 FFN holding the exactly dequantised weights
    Wq = make_weights(g, 0, ffn="nvfp4")
    oq = Lfm3Oracle(Wq)
    Wb = make_weights(g, 0)
    for L, Lq in zip(Wb["layers"], Wq["layers"]):
        for nm, s in (("w1", "w13_scale2"), ("w3", "w13_scale2"), ("w2", "w2_scale2")):
            deq = nvfp4_dequant(Lq[nm + "_codes"], Lq[nm + "_scales"], Lq[s])
            L[nm] = bf16_bits(deq.astype(np.float32))
            assert np.array_equal(_bf16(L[nm]).astype(np.float64), deq)
    ob = Lfm3Oracle(Wb)
    tok = np.arange(10) * 7 % g.vocab
    a = oq.forward_full(tokens=tok, logits="all")
    b = ob.forward_full(tokens=tok, logits="all")
    assert np.allclose(a["logits"], b["logits"], rtol=1e-12, atol=1e-12)


def test_sandwich_norm_structure():
    g = tiny_geometry(layer_types=(CONV,), has_head=False)

    def weights():
        # at width 64 the N(0, 0.02) conv branch is far below sqrt(eps); scale it up to
        # unit RMS so that the norm's scale invariance is visible
        W = make_weights(g, 0)
        L = W["layers"][0]
        for nm, f in (("in_proj", 5.0), ("conv", 50.0), ("out_proj", 5.0)):
            L[nm] = bf16_bits(_bf16(L[nm]) * f)
        return W
    W = weights()
    r = np.random.default_rng(12)
    x = r.standard_normal((9, g.d_model))
    base = Lfm3Oracle(W).forward_full(x0=x)["hidden"][-1]
    # the mixer output passes through post_operator_norm, so scaling the mixer's input norm
    # gain (a cubic change of the conv output) leaves the block unchanged up to eps
    W2 = weights()
    W2["layers"][0]["op_norm"] = bf16_bits(_bf16(W["layers"][0]["op_norm"]) * 4.0)
    assert np.allclose(Lfm3Oracle(W2).forward_full(x0=x)["hidden"][-1], base, rtol=1e-4, atol=1e-4)
    # zero post-norm gains make the block the identity
    W3 = make_weights(g, 0)
    W3["layers"][0]["post_op_norm"] = np.zeros_like(W3["layers"][0]["post_op_norm"])
    W3["layers"][0]["post_ffn_norm"] = np.zeros_like(W3["layers"][0]["post_ffn_norm"])
    assert np.array_equal(Lfm3Oracle(W3).forward_full(x0=x)["hidden"][-1], x)
    # each residual branch adds a unit-RMS (times gain) vector
    W4 = weights()
    W4["layers"][0]["post_ffn_norm"] = np.zeros_like(W4["layers"][0]["post_ffn_norm"])
    W4["layers"][0]["post_op_norm"] = bf16_bits(np.ones(g.d_model, np.float32))
    d = Lfm3Oracle(W4).forward_full(x0=x)["hidden"][-1] - x
    assert np.allclose(np.sqrt(np.mean(d * d, axis=1)), 1.0, rtol=1e-3)


# ---------------------------------------------------------------- bf16 activation boundaries

def test_round_bf16_against_torch_and_ties():
    from oracle import round_bf16
    r = np.random.default_rng(13)
    x = (r.standard_normal(10000) * np.exp(r.uniform(-20, 20, 10000))).astype(np.float32).astype(np.float64)
    ref = torch.from_numpy(x.astype(np.float32)).to(torch.bfloat16).to(torch.float64).numpy()
    assert np.array_equal(round_bf16(x), ref)
    # idempotent, exact on bf16 values, ties to even (1 + 2^-8 lies halfway between 1 and 1 + 2^-7)
    assert np.array_equal(round_bf16(ref), ref)
    assert round_bf16(1.0 + 2.0 ** -8) == 1.0
    assert round_bf16(1.0 + 3 * 2.0 ** -8) == 1.0 + 2.0 ** -6
    assert round_bf16(-(1.0 + 2.0 ** -8 + 2.0 ** -30)) == -(1.0 + 2.0 ** -7)


def test_bf16_boundary_mode_keeps_the_invariants_and_stores_bf16_state():
    from oracle import round_bf16
    g = tiny_geometry()
    W = make_weights(g, 0)
    tok = np.arange(21) * 5 % g.vocab
    o = Lfm3Oracle(W, bf16=True)
    full = o.forward_full(tokens=tok, logits="all")
    st = o.new_state()
    parts = [o.forward_chunk(st, tokens=tok[:9], logits="all")] + \
            [o.forward_chunk(st, tokens=tok[t:t + 1], logits="all") for t in range(9, 21)]
    assert np.allclose(np.concatenate([p["logits"] for p in parts]), full["logits"], rtol=1e-10, atol=1e-10)
    # the carried conv columns and the cached keys/values are bf16 values
    for a in st.conv + st.full_k + st.full_v + st.ring_k + st.ring_v:
        assert np.array_equal(round_bf16(a), a)
    # close to the unrounded definition, but not equal to it
    exact = Lfm3Oracle(W).forward_full(tokens=tok, logits="all")
    d = np.abs(full["hidden"][-1] - exact["hidden"][-1]).max() / np.abs(exact["hidden"][-1]).max()
    assert 1e-5 < d < 5e-2


@pytest.mark.parametrize("n_real,n_pad", [(1, 63), (5, 59), (6, 58), (37, 27), (64, 0)])
def test_pad_tail_state_is_columns_n_to_n_plus_6_of_the_padded_window(n_real, n_pad):
    """coreai-model-zoo note "lfm3-1.7b-port", pad-tail paragraph: a chunk padded at its end reads
    its new conv state from columns [n, n + 6) of [state | Bx], n = the real rows. The oracle's
    chunked conv, run on the real rows alone, commits exactly those columns of the padded window
    whatever the pads hold, and the real rows' conv outputs do not see the pads."""
    r = np.random.default_rng(14)
    C = 24
    w = r.standard_normal((C, 7))
    state = r.standard_normal((6, C))
    bx = r.standard_normal((n_real, C))
    pads = np.full((n_pad, C), np.nan)
    win = np.concatenate([state, bx, pads], axis=0)
    z, st_new = causal_conv_chunk(state, bx, w)
    assert np.array_equal(win[n_real:n_real + 6], st_new)
    pads = r.standard_normal((n_pad, C)) * 1e3
    z_pad, _ = causal_conv_chunk(state, np.concatenate([bx, pads], axis=0), w)
    assert np.array_equal(z_pad[:n_real], z)
