"""NVFP4 weight decoding, written from the element-format definitions.

TEST INFRASTRUCTURE ONLY (see the package docstring).

The checkpoint stores only the FFN (w1, w3, w2) as NVFP4: E2M1 codes in groups
of 16 with one E4M3 block scale per group and one fp32 tensor scale; the
static input scale is read but not applied, so activations stay bf16
(TensorFold PR #1508, "What" and the NVFP4 admission commit; weight-only).

Element formats (OCP Microscaling Formats spec, v1.0):
* E2M1: bit 3 sign, bits 2..1 exponent (bias 1), bit 0 mantissa. Exponent 0 is
  subnormal: 0.5 * m. Otherwise 2^(e-1) * (1 + m/2). No inf/NaN.
* E4M3 ("fn"): bit 7 sign, bits 6..3 exponent (bias 7), bits 2..0 mantissa.
  Exponent 0 is subnormal: 2^-6 * m/8. Exponent 15 with mantissa 7 is NaN;
  there is no infinity.

Packing (a layout this library chooses; the pages do not give one): two codes per byte
along the input dimension, element 2b in the low nibble and 2b+1 in the high
nibble; scales row-major [rows, cols/16].
"""
import numpy as np


def e2m1_value(code: int) -> float:
    code = int(code) & 0xF
    s = -1.0 if code & 0x8 else 1.0
    e = (code >> 1) & 0x3
    m = code & 0x1
    if e == 0:
        return s * 0.5 * m
    return s * (2.0 ** (e - 1)) * (1.0 + 0.5 * m)


def e4m3_value(byte: int) -> float:
    byte = int(byte) & 0xFF
    s = -1.0 if byte & 0x80 else 1.0
    e = (byte >> 3) & 0xF
    m = byte & 0x7
    if e == 0xF and m == 0x7:
        return float("nan")
    if e == 0:
        return s * (2.0 ** -6) * (m / 8.0)
    return s * (2.0 ** (e - 7)) * (1.0 + m / 8.0)


E2M1_TABLE = np.array([e2m1_value(c) for c in range(16)], dtype=np.float64)
E4M3_TABLE = np.array([e4m3_value(b) for b in range(256)], dtype=np.float64)


def nvfp4_unpack_codes(packed: np.ndarray) -> np.ndarray:
    """[rows, cols/2] bytes -> [rows, cols] 4-bit codes."""
    packed = np.asarray(packed, dtype=np.uint8)
    rows, half = packed.shape
    codes = np.empty((rows, 2 * half), dtype=np.uint8)
    codes[:, 0::2] = packed & 0x0F
    codes[:, 1::2] = packed >> 4
    return codes


def nvfp4_block_values(packed: np.ndarray, scales: np.ndarray) -> np.ndarray:
    """E2M1 value times its block's E4M3 scale, per weight (no tensor scale).
    The product of a 2-bit and a 4-bit significand is exact in float32."""
    codes = nvfp4_unpack_codes(packed)
    vals = E2M1_TABLE[codes]
    sc = E4M3_TABLE[np.asarray(scales, dtype=np.uint8)]
    vals = vals * np.repeat(sc, 16, axis=1)
    return vals.astype(np.float32)


def nvfp4_dequant(packed: np.ndarray, scales: np.ndarray, tensor_scale: float) -> np.ndarray:
    """Full dequantisation w = e2m1(code) * e4m3(block scale) * tensor scale, float64."""
    return nvfp4_block_values(packed, scales).astype(np.float64) * float(tensor_scale)
