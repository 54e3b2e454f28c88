"""MLX affine weight decoding (the 4-, 6- and 8-bit text exports).

TEST INFRASTRUCTURE ONLY (see the package docstring).

TensorFold issue #1491, "Checkpoint handling": the text 4/6/8-bit exports "use affine groups of
64". A weight row is cut into groups of 64 consecutive inputs; each group has one scale s and
one bias b (bf16), and an element with code q (an unsigned integer of `bits` bits) stands for
    w = s * q + b
which is evaluated here in float64 (the plain definition; the GPU keeps it exact as
s * (sum of q x) + b * (sum of x) over the group). TensorFold PR #1508's NVFP4 admission commit
reports the MLX 4-bit header as 594 tensors and 973,008,384 bytes, which the pins reproduce
with the embedding and every linear in this format, bf16 scales and biases, and the conv kernel
and norms in bf16.

Packing (a layout this library chooses; the pages do not give one): each row is one
little-endian bit stream, code i at bits [bits * i, bits * i + bits), stored as uint32 words
[rows, cols * bits / 32]; scales and biases are bf16 [rows, cols / 64].
"""
import numpy as np

GROUP = 64


def affine_unpack(packed, bits: int, cols: int) -> np.ndarray:
    """uint32 words [rows, cols * bits / 32] -> codes uint8 [rows, cols]."""
    w = np.ascontiguousarray(packed, dtype=np.uint32)
    rows = w.shape[0]
    stream = w.view(np.uint8).reshape(rows, -1)                 # little-endian bytes of each row
    bitsarr = np.unpackbits(stream, axis=1, bitorder="little")  # bit j of the row at column j
    idx = np.arange(cols)[:, None] * bits + np.arange(bits)[None, :]
    weights = (1 << np.arange(bits)).astype(np.uint32)
    return (bitsarr[:, idx] * weights).sum(axis=2).astype(np.uint8)


def affine_dequant(packed, scales_bits, biases_bits, bits: int, cols: int) -> np.ndarray:
    """w[r, c] = s[r, c // 64] * q[r, c] + b[r, c // 64], float64."""
    q = affine_unpack(packed, bits, cols).astype(np.float64)
    s = (np.asarray(scales_bits, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    b = (np.asarray(biases_bits, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    return q * np.repeat(s, GROUP, axis=1) + np.repeat(b, GROUP, axis=1)
