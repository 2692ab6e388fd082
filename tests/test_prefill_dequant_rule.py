"""The prefill GEMM's Q4 -> bf16 dequantisation rule, checked on the CPU with its
steps restated: a 4-bit code q placed in the low mantissa bits of the bf16
constant 0x4300 (128.0, whose last mantissa bit is worth 1) reads as 128 + q;
subtracting 128 leaves q exactly; then w = d q + m is rounded once to bf16 (d and
m already bf16). The result is within half a bf16 unit of d q + m."""
import numpy as np


def bf16_bits_to_f64(bits):
    return (np.asarray(bits, dtype=np.uint32) << 16).view(np.float32).astype(np.float64)


def round_bf16(v):
    """Round float64 values to bf16 (nearest even) through float32 (exact here:
    the values have at most 24 significant bits before the final rounding)."""
    f = np.asarray(v, dtype=np.float64).astype(np.float32)
    u = f.view(np.uint32).astype(np.uint64)
    u = ((u + 0x7FFF + ((u >> 16) & 1)) >> 16) << 16
    return u.astype(np.uint32).view(np.float32).astype(np.float64)


def test_magic_constant_encodes_the_code():
    q = np.arange(16)
    v = bf16_bits_to_f64(0x4300 | q)
    assert np.array_equal(v, 128.0 + q)
    assert np.array_equal(v - 128.0, q)       # representable, so the subtraction is exact


def test_one_rounding_of_d_q_plus_m():
    rs = np.random.default_rng(4)
    d = round_bf16(rs.uniform(0.002, 0.01, 4000))
    m = round_bf16(-7.5 * d)
    q = rs.integers(0, 16, 4000).astype(np.float64)
    exact = d * q + m                          # exact in float64: a 16-bit-wide fixed-point sum
    w = round_bf16(exact)
    ulp = np.abs(exact) * 2.0 ** -8            # a bf16 unit is at most 2^-7 relative
    assert np.all(np.abs(w - exact) <= ulp + 1e-30)
    # q = 0 returns m itself
    assert np.array_equal(round_bf16(d * 0 + m), m)
