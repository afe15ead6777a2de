"""Host-side checks of the two floating-point identities the preparation kernels rely on,
restated in numpy (IEEE fp32, round to nearest even) over every finite fp16 value.

1. Exact channel sums.  For x a finite fp16 value, one rounding add of C = 1.5 * 2^17 gives
   t = C + h with h = x rounded to a multiple of 2^-6; then bits(t) - bits(C) = 64 h exactly,
   h = t - C and lo = x - h are exact, |lo| <= 2^-7, and x * 2^24 = (64 h) * 2^18 + lo * 2^24.
   Sums of 64 such lo values stay exact in fp32 (multiples of 2^-24 of magnitude <= 1/2).
2. Rounding to INT8 codes.  For |y| < 127.5, the low byte of bits(fl(y + 1.5 * 2^23)) is
   round_half_even(y) in two's complement.

These are statements about the method the kernels use, checked on the CPU; the kernels
themselves are checked against the oracle on the GPU.
"""
import numpy as np

C_SPLIT = np.float32(196608.0)      # 1.5 * 2^17
C_SPLIT_BITS = 0x48400000
C_ROUND = np.float32(12582912.0)    # 1.5 * 2^23


def _finite_fp16_as_fp32():
    h = np.arange(1 << 16, dtype=np.uint32).astype(np.uint16).view(np.float16)
    return h[np.isfinite(h)].astype(np.float32)


def test_split_is_exact_for_every_finite_fp16():
    assert np.float32(C_SPLIT).view(np.uint32) == C_SPLIT_BITS
    x = _finite_fp16_as_fp32()
    t = (x + C_SPLIT).astype(np.float32)
    h = (t - C_SPLIT).astype(np.float32)
    lo = (x - h).astype(np.float32)
    h64 = t.view(np.int32).astype(np.int64) - C_SPLIT_BITS
    exact = (x.astype(np.float64) * 2.0 ** 24).astype(np.int64)  # fp16 * 2^24 is an integer
    assert np.all(h.astype(np.float64) * 64.0 == h64)
    assert np.all(h64 * 2 ** 18 + (lo.astype(np.float64) * 2.0 ** 24).astype(np.int64) == exact)
    assert np.abs(lo).max() <= 2.0 ** -7
    assert np.abs(h64).max() < 2 ** 22  # 64 of them stay below 2^28 in int32


def test_64_token_partial_sums_of_lo_stay_exact():
    x = _finite_fp16_as_fp32()
    lo = (x - ((x + C_SPLIT).astype(np.float32) - C_SPLIT).astype(np.float32)).astype(np.float32)
    rng = np.random.default_rng(0)
    worst = np.sort(np.abs(lo))[::-1][:64]  # the largest magnitudes, all of one sign
    samples = [worst, -worst] + [lo[rng.integers(0, lo.size, 64)] for _ in range(500)]
    for v in samples:
        acc = np.float32(0.0)
        for e in v:
            acc = np.float32(acc + e)
        assert float(acc) == float(np.sum(v.astype(np.float64)))


def test_magic_add_rounds_half_to_even():
    grid = np.linspace(-127.49, 127.49, 1_000_001, dtype=np.float32)
    halves = (np.arange(-127, 127) + np.float32(0.5)).astype(np.float32)
    near = np.concatenate([np.nextafter(halves, np.float32(-200)), np.nextafter(halves, np.float32(200))])
    y = np.concatenate([grid, halves, near]).astype(np.float32)
    y = y[np.abs(y) < 127.5]
    code = ((y + C_ROUND).astype(np.float32).view(np.uint32) & 0xFF).astype(np.uint8).view(np.int8)
    assert np.array_equal(code.astype(np.int64), np.rint(y).astype(np.int64))


def test_product_with_the_inverse_scale_stays_below_127_5():
    # |x| <= a and inv = fl(127 / a) give |fl(x * inv)| <= 127 (1 + 2^-24)^2 < 127.5, so the
    # kernels need no clamp; checked here for random and adversarial absmax values
    rng = np.random.default_rng(1)
    a = np.concatenate([rng.uniform(1e-6, 7e4, 200_000).astype(np.float32),
                        np.float32(2.0) ** np.arange(-24, 17, dtype=np.float32)])
    inv = (np.float32(127.0) / a).astype(np.float32)
    y = (a * inv).astype(np.float32)
    assert np.all(np.abs(y) < 127.5)
    assert np.all(np.rint(y) == 127)
