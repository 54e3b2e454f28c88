"""Pins of the oracle's MLX affine decoding (CPU only): the pages' export total, brute-force bit
extraction, the dequantisation formula, and an affine FFN against the same FFN holding the
dequantised weights."""
import numpy as np
import pytest

from conftest import read_golden
from lfm3_inputs import CONV, lfm3_1p7b, tiny_geometry, make_weights, affine_draw
from oracle import Lfm3Oracle, affine_unpack, affine_dequant


def _mlx_export_totals(g, bits, group):
    """Tensors and bytes of an MLX affine text export of geometry g: the embedding and every
    linear as packed codes + bf16 scales + bf16 biases per group; norms, q/k norms and the conv
    kernel bf16; q, k, v, o and the gate as separate linears; the head tied to the embedding."""
    D, F, d = g.d_model, g.d_ffn, g.head_dim

    def lin(n, k):
        return n * k * bits // 8 + 2 * 2 * (n * k // group)
    tensors, nbytes = 3 + 1, lin(g.vocab, D) + 2 * D
    for kind in g.layer_types:
        tensors += 4 + 9
        nbytes += 2 * 4 * D + 2 * lin(F, D) + lin(D, F)
        if kind == CONV:
            tensors += 3 + 3 + 1
            nbytes += lin(3 * D, D) + lin(D, D) + 2 * D * g.conv_taps
        else:
            tensors += 5 * 3 + 2
            nbytes += lin(g.n_q * d, D) + 2 * lin(g.n_kv * d, D) + lin(D, g.n_q * d) + lin(g.n_q, D) + 2 * 2 * d
    return tensors, nbytes


def test_mlx4_export_total_pins_groups_of_64_and_bf16_scales():
    gold = read_golden("mlx4_export_header.txt")
    t, b = _mlx_export_totals(lfm3_1p7b(), gold["bits"], gold["group"])
    assert (t, b) == (gold["text_tensors"], gold["total_bytes"])
    # groups of 32, or fp32 scales, or a bf16 gate projection would miss the published total
    assert _mlx_export_totals(lfm3_1p7b(), 4, 32)[1] != gold["total_bytes"]


@pytest.mark.parametrize("bits", [4, 6, 8])
def test_unpack_against_brute_force_bits(bits):
    packed, s, b = affine_draw(3, f"unpack{bits}", 5, 128, bits)
    raw = packed.view(np.uint8)
    got = affine_unpack(packed, bits, 128)
    for r in range(5):
        stream = int.from_bytes(raw[r].tobytes(), "little")
        for c in range(128):
            assert got[r, c] == (stream >> (bits * c)) & ((1 << bits) - 1)
    # every code value occurs and none exceeds the width
    assert got.max() < (1 << bits)


@pytest.mark.parametrize("bits", [4, 6, 8])
def test_dequant_is_scale_times_code_plus_bias_per_group_of_64(bits):
    packed, s, b = affine_draw(4, f"deq{bits}", 3, 192, bits)
    q = affine_unpack(packed, bits, 192)
    w = affine_dequant(packed, s, b, bits, 192)
    sf = (s.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    bf = (b.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    for r in range(3):
        for c in range(192):
            assert w[r, c] == sf[r, c // 64] * float(q[r, c]) + bf[r, c // 64]
    # the draws span about +-0.02, like the bf16 weights
    assert 0.005 < np.abs(w).mean() < 0.03


def test_affine_ffn_equals_the_ffn_of_its_dequantised_weights():
    g = tiny_geometry(d_ffn=128)  # both FFN widths in whole groups of 64
    Wa = make_weights(g, 0, ffn="affine4")
    oa = Lfm3Oracle(Wa)
    tok = np.arange(12) * 5 % g.vocab
    a = oa.forward_full(tokens=tok, logits="all")
    # the same model with float64 FFN weights put in directly
    ob = Lfm3Oracle(make_weights(g, 0))
    for O, L in zip(ob.layers, Wa["layers"]):
        for nm, cols in (("w1", g.d_model), ("w3", g.d_model), ("w2", g.d_ffn)):
            O[nm] = affine_dequant(L[nm + "_codes"], L[nm + "_scales"], L[nm + "_biases"], 4, cols)
    b = ob.forward_full(tokens=tok, logits="all")
    assert np.allclose(a["logits"], b["logits"], rtol=1e-12, atol=1e-12)
