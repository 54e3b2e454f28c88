"""Seeded synthetic inputs for the LFM3-1.7B hybrid decoder.

This module is shared by the CPU oracle and the CUDA path. It holds only the
geometry of the workloads and the seeded random draws (weights, token ids,
input vectors, page permutations, context lengths); it holds none of the
decoder's arithmetic. Every array it returns is raw storage: bf16 values as
their 16-bit patterns (``np.uint16``), NVFP4 weights as packed E2M1 nibbles and
E4M3 scale bytes (``np.uint8``) plus an fp32 tensor scale.

Draws come from NumPy's ``Generator(PCG64(SeedSequence([seed, crc32(tag)])))``,
one stream per named tensor, so any tensor can be regenerated alone.
"""
from .gen import (  # noqa: F401
    CONV, FULL, SLIDING,
    Lfm3Geometry, lfm3_1p7b, lfm3_slice3, tiny_geometry,
    rng_for, bf16_bits, make_weights, make_tokens, make_embeds,
    nvfp4_draw, affine_draw, page_permutation, context_lengths, synthetic_state,
)
