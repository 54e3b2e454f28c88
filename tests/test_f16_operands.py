"""The arithmetic the NVFP4 kernels rely on when they multiply on f16 operands, checked exhaustively
with NumPy (no GPU): every E2M1 x E4M3 product is exact in f16, and the bf16 activations the f16
copies are made of convert exactly inside f16's normal range.

The kernels expand a code pair with the hardware E2M1 -> f16 conversion, multiply by the block's
E4M3 scale converted to f16, and feed f16 activations (bf16 values stored as f16) to the MMA; the
fp32 tensor scale multiplies the fp32 sums. The element formats are the OCP Microscaling ones
(E2M1: 1 sign, 2 exponent bits with bias 1, 1 mantissa bit; E4M3: 1 sign, 4 exponent bits with
bias 7, 3 mantissa bits, no infinity)."""
import numpy as np

from oracle.nvfp4 import e2m1_value, e4m3_value


def _bf16_to_f64(bits):
    return (np.asarray(bits, dtype=np.uint32) << 16).view(np.float32).astype(np.float64)


def test_every_e2m1_code_and_e4m3_scale_is_an_f16_value():
    for c in range(16):
        v = e2m1_value(c)
        assert float(np.float16(v)) == v
    for b in range(256):
        v = e4m3_value(b)
        if np.isnan(v):
            continue
        assert float(np.float16(v)) == v, b


def test_every_code_times_scale_product_is_exact_in_f16():
    codes = np.array([e2m1_value(c) for c in range(16)])
    scales = np.array([e4m3_value(b) for b in range(256)])
    scales = scales[~np.isnan(scales)]
    prod = codes[:, None] * scales[None, :]            # exact in float64
    assert np.all(prod.astype(np.float16).astype(np.float64) == prod)
    # the extremes: 6 x 448 = 2688 (far below 65504) and 0.5 x 2^-9 = 2^-10 (above f16's
    # smallest normal, 2^-14), so no product is subnormal or overflows in f16
    nz = np.abs(prod[prod != 0])
    assert nz.max() == 2688.0 and nz.min() == 2.0 ** -10


def test_bf16_values_in_f16_normal_range_convert_exactly():
    # every bf16 bit pattern whose magnitude lies in [2^-14, 65504]
    bits = np.arange(1 << 16, dtype=np.uint32)
    x = _bf16_to_f64(bits)
    inside = np.isfinite(x) & (np.abs(x) >= 2.0 ** -14) & (np.abs(x) <= 65504.0)
    assert inside.sum() > 7000
    assert np.all(x[inside].astype(np.float16).astype(np.float64) == x[inside])
    # just past the range a value is no longer representable (the reading the header states)
    big = x[np.isfinite(x) & (np.abs(x) > 65504.0)]
    with np.errstate(over="ignore"):
        assert np.all(np.isinf(big.astype(np.float16)))


def test_bf16_values_below_the_normal_range_lose_at_most_half_an_f16_subnormal_step():
    bits = np.arange(1 << 16, dtype=np.uint32)
    x = _bf16_to_f64(bits)
    small = np.isfinite(x) & (np.abs(x) < 2.0 ** -14)
    err = np.abs(x[small].astype(np.float16).astype(np.float64) - x[small])
    assert err.max() <= 2.0 ** -25  # half of the subnormal spacing 2^-24
