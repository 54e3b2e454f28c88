"""Geometry and seeded draws for the LFM3 workloads (no decoder arithmetic here).

Geometry: 24 layers at width 2048, FFN 7680, 16 query / 4 KV heads of 128,
vocabulary 128000 with a tied head (TensorFold issue #1491, "Architecture";
coreai-model-zoo note "lfm3-1.7b-port", LFM2.5 -> LFM3 diff table). The layer
pattern (0-based) puts sliding-window attention at 1, 5, 9, 13, 17, full
attention at 3, 7, 11, 15, 19, 21 and the gated short conv everywhere else:
13 conv, 6 full and 5 sliding layers, as the diff table counts them.
"""
from __future__ import annotations

import os
import zlib
from concurrent.futures import ThreadPoolExecutor
from dataclasses import dataclass, field, replace

import numpy as np

CONV, FULL, SLIDING = 0, 1, 2

_SLIDING_AT = (1, 5, 9, 13, 17)
_FULL_AT = (3, 7, 11, 15, 19, 21)


def _lfm3_layer_types() -> tuple:
    t = []
    for i in range(24):
        t.append(SLIDING if i in _SLIDING_AT else FULL if i in _FULL_AT else CONV)
    return tuple(t)


@dataclass(frozen=True)
class Lfm3Geometry:
    """Shape of one LFM3 decoder. ``rope_pairs_full`` is how many of the
    head_dim/2 rotary pairs turn on full-attention layers (half of them)."""

    layer_types: tuple = field(default_factory=_lfm3_layer_types)
    d_model: int = 2048
    d_ffn: int = 7680
    n_q: int = 16
    n_kv: int = 4
    head_dim: int = 128
    conv_taps: int = 7
    window: int = 256
    vocab: int = 128000
    theta_full: float = 1.0e6
    theta_sliding: float = 1.0e4
    rope_pairs_full: int = 32
    eps: float = 1.0e-5
    has_head: bool = True

    @property
    def n_layers(self) -> int:
        return len(self.layer_types)

    def count(self, kind: int) -> int:
        return sum(1 for t in self.layer_types if t == kind)

    def index_in_kind(self, layer: int) -> int:
        """Position of ``layer`` among the layers of its own type."""
        kind = self.layer_types[layer]
        return sum(1 for t in self.layer_types[:layer] if t == kind)

    @property
    def qkvg_rows(self) -> int:
        return self.n_q * self.head_dim + 2 * self.n_kv * self.head_dim + self.n_q


def lfm3_1p7b(**kw) -> Lfm3Geometry:
    """The full 24-layer LFM3-1.7B geometry."""
    return replace(Lfm3Geometry(), **kw)


def lfm3_slice3(**kw) -> Lfm3Geometry:
    """Three-block slice at width 2048: conv, sliding (theta 1e4, all pairs),
    full (theta 1e6, half the pairs); inputs are vectors, so no embedding/head."""
    return replace(Lfm3Geometry(), layer_types=(CONV, SLIDING, FULL), has_head=False, **kw)


def tiny_geometry(**kw) -> Lfm3Geometry:
    """A small geometry for the oracle's own CPU tests (same structure)."""
    base = dict(layer_types=(CONV, SLIDING, FULL, CONV, SLIDING, FULL), d_model=64, d_ffn=96,
                n_q=4, n_kv=2, head_dim=16, conv_taps=7, window=8, vocab=97,
                rope_pairs_full=4)
    base.update(kw)
    return Lfm3Geometry(**base)


# ----------------------------------------------------------------------------------------
# draws


def rng_for(seed: int, tag: str) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(np.random.SeedSequence([int(seed), zlib.crc32(tag.encode())])))


def bf16_bits(x) -> np.ndarray:
    """Round float32 values to bf16 (nearest, ties to even) and return the bit patterns."""
    f = np.ascontiguousarray(x, dtype=np.float32)
    u = f.view(np.uint32)
    r = ((u >> 16) & 1) + np.uint32(0x7FFF)
    return ((u + r) >> 16).astype(np.uint16)


def _normal_bf16(seed, tag, shape, std, mean=0.0):
    g = rng_for(seed, tag)
    v = g.standard_normal(int(np.prod(shape)), dtype=np.float32)
    if std != 1.0:
        v *= np.float32(std)
    if mean != 0.0:
        v += np.float32(mean)
    return bf16_bits(v).reshape(shape)


def _e4m3_nearest_bytes(vals: np.ndarray) -> np.ndarray:
    """Encode positive normal values (2^-6 <= v < 448) as E4M3 bytes, nearest, ties to even.
    Only used to draw synthetic block scales; the decoders read the bytes."""
    v = np.asarray(vals, dtype=np.float64)
    m, e = np.frexp(v)                     # v = m * 2^e, m in [0.5, 1)
    e = e - 1                              # v = (2m) * 2^e, 2m in [1, 2)
    mant = np.rint((2.0 * m - 1.0) * 8.0)  # ties to even
    carry = mant >= 8
    mant = np.where(carry, 0, mant)
    e = np.where(carry, e + 1, e)
    assert np.all(e >= -6) and np.all(e <= 8)
    return ((e + 7).astype(np.uint8) << 3) | mant.astype(np.uint8)


def nvfp4_draw(seed: int, tag: str, n: int, k: int):
    """One NVFP4 weight [n, k]: E2M1 codes uniform over all 16 (incl. -0), packed two
    per byte along k (element 2b in the low nibble, 2b+1 in the high nibble); one E4M3
    block scale per 16 consecutive k, drawn as 2^u, u ~ U(-6, 2), rounded to E4M3."""
    assert k % 16 == 0
    g = rng_for(seed, tag + ".codes")
    codes = g.integers(0, 16, size=(n, k), dtype=np.uint8)
    packed = (codes[:, 0::2] | (codes[:, 1::2] << 4)).astype(np.uint8)
    g2 = rng_for(seed, tag + ".scales")
    u = g2.uniform(-6.0, 2.0, size=(n, k // 16))
    scales = _e4m3_nearest_bytes(np.exp2(u))
    return np.ascontiguousarray(packed), np.ascontiguousarray(scales)


NVFP4_TENSOR_SCALE = np.float32(2.0 ** -8)


def affine_draw(seed: int, tag: str, n: int, k: int, bits: int):
    """One MLX-style affine weight [n, k] in groups of 64 along k: codes uniform over the
    2^bits values, packed as one little-endian bit stream per row into uint32 words; per group a
    bf16 scale s = 2^u * 0.04 / (2^bits - 1), u ~ U(-1, 1), and a bf16 bias drawn around
    -s * (2^bits - 1) / 2, so that s * q + b spans about +-0.02 like the bf16 weights."""
    assert k % 64 == 0 and (k * bits) % 32 == 0
    g = rng_for(seed, tag + ".codes")
    codes = g.integers(0, 1 << bits, size=(n, k), dtype=np.uint8)
    bitsarr = ((codes[:, :, None] >> np.arange(bits, dtype=np.uint8)[None, None, :]) & 1).reshape(n, k * bits)
    packed = np.packbits(bitsarr, axis=1, bitorder="little").view(np.uint32)
    g2 = rng_for(seed, tag + ".scales")
    s = (np.exp2(g2.uniform(-1.0, 1.0, size=(n, k // 64))) * (0.04 / ((1 << bits) - 1))).astype(np.float32)
    g3 = rng_for(seed, tag + ".biases")
    b = (-s * ((1 << bits) - 1) / 2.0 * (1.0 + 0.05 * g3.standard_normal((n, k // 64)))).astype(np.float32)
    return np.ascontiguousarray(packed), bf16_bits(s), bf16_bits(b)


def make_weights(geom: Lfm3Geometry, seed: int = 0, ffn: str = "bf16", threads: int | None = None) -> dict:
    """Random-init weights: linear and conv weights N(0, 0.02), norm gains 1 + N(0, 0.02),
    all rounded to bf16 once. ``ffn='nvfp4'`` draws the FFN (w1, w3, w2) as NVFP4.
    Each tensor has its own seeded stream, so tensors are drawn in parallel threads."""
    if ffn not in ("bf16", "nvfp4", "affine4", "affine6", "affine8"):
        raise ValueError(ffn)
    D, F, d = geom.d_model, geom.d_ffn, geom.head_dim
    W = {"geometry": geom, "ffn": ffn, "layers": []}
    jobs = []  # (container, key, callable)
    if geom.has_head:
        jobs.append((W, "embed", lambda: _normal_bf16(seed, "embed", (geom.vocab, D), 0.02)))
        jobs.append((W, "final_norm", lambda: _normal_bf16(seed, "final_norm", (D,), 0.02, 1.0)))
    for li, kind in enumerate(geom.layer_types):
        p = f"layer{li}."
        L = {"kind": kind}
        W["layers"].append(L)

        def normal(key, shape, std, mean=0.0, L=L, p=p):
            jobs.append((L, key, lambda: _normal_bf16(seed, p + key, shape, std, mean)))

        for nm in ("op_norm", "post_op_norm", "ffn_norm", "post_ffn_norm"):
            normal(nm, (D,), 0.02, 1.0)
        if kind == CONV:
            normal("in_proj", (3 * D, D), 0.02)
            normal("conv", (D, geom.conv_taps), 0.02)
            normal("out_proj", (D, D), 0.02)
        else:
            normal("q_proj", (geom.n_q * d, D), 0.02)
            normal("k_proj", (geom.n_kv * d, D), 0.02)
            normal("v_proj", (geom.n_kv * d, D), 0.02)
            normal("gate_proj", (geom.n_q, D), 0.02)
            normal("q_norm", (d,), 0.02, 1.0)
            normal("k_norm", (d,), 0.02, 1.0)
            normal("o_proj", (D, geom.n_q * d), 0.02)
        if ffn == "bf16":
            normal("w1", (F, D), 0.02)
            normal("w3", (F, D), 0.02)
            normal("w2", (D, F), 0.02)
        elif ffn.startswith("affine"):
            bits = int(ffn[6:])
            L["affine_bits"] = bits
            for nm, (n, k) in (("w1", (F, D)), ("w3", (F, D)), ("w2", (D, F))):
                jobs.append((L, nm, lambda nm=nm, n=n, k=k, p=p: affine_draw(seed, p + nm, n, k, bits)))
        else:
            for nm, (n, k) in (("w1", (F, D)), ("w3", (F, D)), ("w2", (D, F))):
                jobs.append((L, nm, lambda nm=nm, n=n, k=k, p=p: nvfp4_draw(seed, p + nm, n, k)))
            L["w13_scale2"] = NVFP4_TENSOR_SCALE
            L["w2_scale2"] = NVFP4_TENSOR_SCALE
    workers = threads or min(16, os.cpu_count() or 1)
    with ThreadPoolExecutor(max_workers=workers) as ex:
        results = list(ex.map(lambda j: j[2](), jobs))
    for (box, key, _), val in zip(jobs, results):
        if isinstance(val, tuple) and len(val) == 3:
            box[key + "_codes"], box[key + "_scales"], box[key + "_biases"] = val
        elif isinstance(val, tuple):
            box[key + "_codes"], box[key + "_scales"] = val
        else:
            box[key] = val
    return W


def make_tokens(seed: int, tag: str, n: int, vocab: int) -> np.ndarray:
    return rng_for(seed, tag).integers(0, vocab, size=n, dtype=np.int64).astype(np.int32)


def make_embeds(seed: int, tag: str, n: int, d_model: int) -> np.ndarray:
    """Input vectors ~ N(0, 1), rounded to bf16 (bit patterns)."""
    return _normal_bf16(seed, tag, (n, d_model), 1.0)


def page_permutation(seed: int, tag: str, n_pages: int) -> np.ndarray:
    return rng_for(seed, tag).permutation(n_pages).astype(np.int32)


def context_lengths(seed: int, tag: str, n_streams: int, lo: int, hi: int) -> np.ndarray:
    """Per-stream context lengths uniform in [lo, hi]."""
    return rng_for(seed, tag).integers(lo, hi + 1, size=n_streams, dtype=np.int64).astype(np.int32)


def synthetic_state(geom: Lfm3Geometry, seed: int, contexts) -> dict:
    """Decode state as if ``contexts[s]`` tokens had already been consumed, drawn instead
    of prefilled: keys/values and conv columns are bf16 N(0, 1). Logical order only
    (positions ascending); laying it out in pages or rings is the consumer's job.

    Returns {'conv': [n_conv][S][taps-1][D] (oldest column first),
             'full_k'/'full_v': [n_full][S] arrays [ctx, n_kv, d],
             'slide_k'/'slide_v': [n_sliding][S] arrays [min(ctx, W), n_kv, d] for the
             last positions ctx-min(ctx,W) .. ctx-1}."""
    S = len(contexts)
    D, d, kv = geom.d_model, geom.head_dim, geom.n_kv
    out = {"conv": _normal_bf16(seed, "state.conv", (geom.count(CONV), S, geom.conv_taps - 1, D), 1.0),
           "full_k": [], "full_v": [], "slide_k": [], "slide_v": []}
    for j in range(geom.count(FULL)):
        out["full_k"].append([_normal_bf16(seed, f"state.full{j}.k.s{s}", (int(c), kv, d), 1.0)
                              for s, c in enumerate(contexts)])
        out["full_v"].append([_normal_bf16(seed, f"state.full{j}.v.s{s}", (int(c), kv, d), 1.0)
                              for s, c in enumerate(contexts)])
    for j in range(geom.count(SLIDING)):
        out["slide_k"].append([_normal_bf16(seed, f"state.slide{j}.k.s{s}", (min(int(c), geom.window), kv, d), 1.0)
                               for s, c in enumerate(contexts)])
        out["slide_v"].append([_normal_bf16(seed, f"state.slide{j}.v.s{s}", (min(int(c), geom.window), kv, d), 1.0)
                               for s, c in enumerate(contexts)])
    return out
