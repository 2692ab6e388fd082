"""The integer arithmetic of the decode contraction, checked on the CPU with its
rules restated: activations quantised to X with |X| <= 8,355,711 (24-bit fixed
point per 32-element block), split into three balanced signed 8-bit limbs,
multiplied by the codes on the integer tensor cores and recombined. Every step
must be exact for the block sums to be exact integers."""
import numpy as np

QMAX = 8_355_711   # 127 * 65536 + 127 * 256 + 127


def limbs3(X):
    """Balanced base-256 digits of X, as the decode kernels form them."""
    X = np.asarray(X, dtype=np.int64)
    l0 = ((X + 128) & 255) - 128
    X1 = (X - l0) >> 8
    l1 = ((X1 + 128) & 255) - 128
    l2 = (X1 - l1) >> 8
    return l2, l1, l0


def i2f_small(v):
    """int -> float through the 1.5 * 2^23 magic number (valid for |v| < 2^22)."""
    bits = (np.int64(0x4B400000) + np.asarray(v, dtype=np.int64)).astype(np.uint32)
    return bits.view(np.float32) - np.float32(12582912.0)


def test_limbs_reconstruct_exactly_and_fit_signed_bytes():
    rs = np.random.default_rng(1)
    X = np.concatenate([np.arange(-QMAX, -QMAX + 70000), np.arange(-70000, 70000), np.arange(QMAX - 70000, QMAX + 1),
                        rs.integers(-QMAX, QMAX + 1, 200000)])
    l2, l1, l0 = limbs3(X)
    for l in (l2, l1, l0):
        assert l.min() >= -128 and l.max() <= 127
    assert np.array_equal(65536 * l2 + 256 * l1 + l0, X)


def test_magic_conversion_is_exact_over_its_range():
    v = np.arange(-(1 << 22), 1 << 22, dtype=np.int64)
    assert np.array_equal(i2f_small(v).astype(np.int64), v)


def test_block_sums_stay_in_the_exact_ranges():
    # Q2 codes 0..3, Q4 codes 0..15; |limb| <= 128; 32 products per block
    hi_q2 = 32 * 3 * (128 * 256 + 128)      # |256 * sum q l2 + sum q l1|
    hi_q4 = 32 * 15 * (128 * 256 + 128)
    assert hi_q2 < (1 << 22)                # the magic conversion is exact (Q2)
    assert hi_q4 < (1 << 24)                # an ordinary int -> fp32 conversion is exact (Q4)
    assert 32 * QMAX < (1 << 31)            # the block sum of X fits int32


def test_recombined_columns_equal_the_code_activation_product():
    """The hi lanes form (256 * sum q l2 + sum q l1) * 256 and the lo lanes
    sum q l0; their sum is sum q X for every block, exactly."""
    rs = np.random.default_rng(2)
    for bits in (2, 4):
        q = rs.integers(0, 1 << bits, (1000, 32))
        X = rs.integers(-QMAX, QMAX + 1, (1000, 32))
        X[:10] = QMAX
        X[10:20] = -QMAX
        l2, l1, l0 = limbs3(X)
        d2, d1, d0 = (q * l2).sum(1), (q * l1).sum(1), (q * l0).sum(1)
        hi = (256 * d2 + d1) * 256
        assert np.array_equal(hi + d0, (q * X).sum(1)), bits


def test_limb_pair_recombination_is_exact_for_4_bit_codes():
    """The epilogue forms hi * 256 + lo as fma(f(hi), 256, f(lo)) from the two
    block sums of a limb pair. For 4-bit codes each sum is at most
    32 * 15 * 128 = 61,440 in magnitude: both convert exactly through the magic
    number, f(hi) * 256 is exact, and the exact result stays below 2^24, so the
    fused multiply-add's single rounding is no rounding at all."""
    bound = 32 * 15 * 128
    rs = np.random.default_rng(2)
    hi = np.concatenate([[-bound, bound, 0, -1, 1], rs.integers(-bound, bound + 1, 100000)])
    lo = np.concatenate([[bound, -bound, 0, 1, -1], rs.integers(-bound, bound + 1, 100000)])
    exact = hi.astype(np.int64) * 256 + lo
    assert np.abs(exact).max() < 2 ** 24
    assert np.array_equal(i2f_small(hi).astype(np.int64), hi) and np.array_equal(i2f_small(lo).astype(np.int64), lo)
    # fma in float32 of exactly representable operands whose exact result fits
    # 24 bits: the float64 evaluation is the exact value, and it survives float32
    fused = i2f_small(hi).astype(np.float64) * 256.0 + i2f_small(lo).astype(np.float64)
    assert np.array_equal(fused.astype(np.float32).astype(np.int64), exact)


def test_limb_pair_recombination_is_exact_in_one_step_for_2_bit_codes():
    """With 2-bit codes the epilogue forms hi * 256 + lo in integers and
    converts it through the magic number 1.5 * 2^23 in one step, which is exact
    only below 2^22: each block sum is at most 32 * 3 * 128 = 12,288."""
    bound = 32 * 3 * 128
    rs = np.random.default_rng(3)
    hi = np.concatenate([[-bound, bound, 0], rs.integers(-bound, bound + 1, 100000)])
    lo = np.concatenate([[-bound, bound, 0], rs.integers(-bound, bound + 1, 100000)])
    v = hi.astype(np.int64) * 256 + lo
    assert np.abs(v).max() < 2 ** 22
    assert np.array_equal(i2f_small(v).astype(np.int64), v)


def test_router_partial_fixed_point_rounds_once_to_the_nearest_integer():
    """Router slice partials become integers in units of 2^-32 through one
    fused multiply-add with 1.5 * 2^52 (its ulp is 1): for |p| < 2^19 the
    product p * 2^32 is exact and below 2^51, so the integer read from the
    sum's bits is p * 2^32 rounded to nearest (ties to even); 4096 such
    integers (H = 65,536) add without overflowing 64 bits."""
    rs = np.random.default_rng(11)
    p = np.concatenate([rs.uniform(-2.0 ** 19, 2.0 ** 19, 20000), rs.standard_normal(20000) * 1e-3,
                        [2.0 ** 19 - 1e-6, -(2.0 ** 19 - 1e-6), 0.0, -0.0, 2.0 ** -33, 3 * 2.0 ** -33, -(2.0 ** -33)]])
    magic = np.float64(1.5 * 2.0 ** 52)
    t = p * 2.0 ** 32 + magic            # the product is exact, the sum rounds once (float64)
    v = t.view(np.int64) - magic.view(np.int64)
    assert np.array_equal(v, np.rint(p * 2.0 ** 32).astype(np.int64))   # rint: to nearest, ties to even
    assert 4096 * (2 ** 51 - 1) < 2 ** 63      # each |v| <= 2^51 - 1
