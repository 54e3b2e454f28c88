"""The prompt-pass FLOP count the bench divides by its device time, pinned to an independent count:
projection FLOPs from the element counts of the weight arrays themselves, attention FLOPs from an
explicit enumeration of the (query, key) pairs each layer type lets through."""
import numpy as np

import bench
from lfm3_inputs import make_weights
from lfm3_inputs.gen import CONV, FULL, SLIDING, lfm3_1p7b, tiny_geometry

PROJECTIONS = ("in_proj", "out_proj", "q_proj", "k_proj", "v_proj", "gate_proj", "o_proj", "w1", "w3", "w2")


def direct_count(g, W, n):
    proj = sum(2 * n * L[k].size for L in W["layers"] for k in PROJECTIONS if k in L)
    q = np.arange(n)[:, None]
    k = np.arange(n)[None, :]
    attn = 0
    for t in g.layer_types:
        if t == CONV:
            continue
        seen = k <= q
        if t == SLIDING:
            seen &= q - k < g.window
        # Q K^T and P V: 2 multiply-adds per head dimension per pair, for every query head
        attn += int(seen.sum()) * g.n_q * g.head_dim * 2 * 2
    head = 2 * W["embed"].size  # the tied head on the last row only
    return proj + attn + head


def test_prefill_flops_matches_weight_shapes_and_enumerated_pairs():
    g = tiny_geometry()
    W = make_weights(g, 0)
    for n in (1, 7, 8, 9, 37):  # around and past the window of 8
        assert bench.prefill_flops(g, n) == direct_count(g, W, n), n


def test_prefill_flops_full_geometry_8k():
    """The 8k prompt of the full geometry: 25.76 TFLOP, of which the causal full-attention half is 1.6495."""
    g = lfm3_1p7b()
    f = bench.prefill_flops(g, 8192)
    assert abs(f / 1e12 - 25.758) < 1e-3
    full_attn = 6 * 8192 * 8193 // 2 * 16 * 128 * 4
    assert g.count(FULL) == 6 and abs(full_attn / 1e12 - 1.64947) < 1e-5
