"""The rotary kernel's exact-arithmetic steps, replayed on the host.

The CUDA rotation (rotary_append.cu and the fused projection's epilogue) uses
bit-level steps to round exactly as the oracle does:

1. A bf16 word becomes a double equal to 2^-896 times its value, by moving
   its 8 exponent bits to the bottom of the double's 11-bit field. The table
   carries the matching 2^896, so products come out unscaled and exact.
2. A per-word test flags infinities and NaNs, which take the plain path.
3. Narrowing to bf16: truncate the double to float, OR in a sticky bit from
   the 29 dropped significand bits (round to odd), then round the float to
   bf16 to nearest even. The rotary kernel's fast path instead narrows with
   the one-instruction conversion cvt.rn.bf16.f64; the round-to-odd form
   stays for the plain path and the projection's epilogue, and is the
   statement replayed here (results below float's normal range are checked
   against the oracle's rounding on that path).

These tests replay those steps with numpy integer operations, exhaustively
over all 65536 bf16 patterns where that is possible. They compare the result
with plain arithmetic and with the oracle's rounding. They check the method,
not the compiled kernel; the GPU parity tests check the kernel's words
bit-exactly against the oracle.
"""
import numpy as np

from oracle.bf16 import bf16_bits_to_f64, f64_to_bf16_bits

ALL = np.arange(1 << 16, dtype=np.uint32)
FINITE = ALL[(ALL & 0x7F80) != 0x7F80]


def _hi_to_double(hi32: np.ndarray) -> np.ndarray:
    return (hi32.astype(np.uint64) << np.uint64(32)).view(np.float64)


def scaled_lo(w: np.ndarray) -> np.ndarray:
    """The low bf16 of a 32-bit word as 2^-896 times its value."""
    hi = ((((w << 16).astype(np.uint32)).view(np.int32) >> 3).view(np.uint32)) & np.uint32(0x8FFFFFFF)
    return _hi_to_double(hi)


def scaled_hi(w: np.ndarray) -> np.ndarray:
    """The high bf16 of a 32-bit word as 2^-896 times its value."""
    hi = ((w.astype(np.uint32).view(np.int32) >> 3).view(np.uint32)) & np.uint32(0x8FFFE000)
    return _hi_to_double(hi)


def special_bits(w: np.ndarray) -> np.ndarray:
    return ((w & np.uint32(0x7F807F80)) + np.uint32(0x00800080)) & np.uint32(0x80008000)


def trunc_to_float(y: np.ndarray) -> np.ndarray:
    """Round toward zero, double -> float (FLT_MAX instead of infinity)."""
    with np.errstate(over="ignore"):
        f = y.astype(np.float32)
        away = np.abs(f.astype(np.float64)) > np.abs(y)
        f = np.where(away, np.nextafter(f, np.float32(0)), f).astype(np.float32)
    return np.where(np.isinf(f), np.copysign(np.finfo(np.float32).max, y), f).astype(np.float32)


def narrow(y: np.ndarray):
    """The fast narrowing: (bf16 words, whether the fast path applies)."""
    lo = (y.view(np.uint64) & np.uint64(0xFFFFFFFF)).astype(np.uint32)
    fb = trunc_to_float(y).view(np.uint32) | ((lo << np.uint32(3)) != 0).astype(np.uint32)
    f = fb.view(np.float32)
    fast = np.abs(f) >= np.finfo(np.float32).tiny
    b = ((fb.astype(np.uint64) + 0x7FFF + ((fb >> np.uint32(16)) & np.uint32(1))) >> np.uint64(16))
    return b.astype(np.uint16), fast


def test_scaled_widening_is_exact_for_every_finite_bf16():
    want = bf16_bits_to_f64(FINITE.astype(np.uint16)) * 2.0 ** -896
    assert np.array_equal(scaled_lo(FINITE), want)
    assert np.array_equal(scaled_hi(FINITE << 16), want)
    # the other half of the word does not leak in
    assert np.array_equal(scaled_lo(FINITE | np.uint32(0xABCD0000)), want)
    assert np.array_equal(scaled_hi((FINITE << 16) | np.uint32(0x1234)), want)


def test_special_bits_flag_exactly_the_infinities_and_nans():
    is_special = (ALL & 0x7F80) == 0x7F80
    assert np.array_equal(special_bits(ALL) != 0, is_special)
    assert np.array_equal(special_bits(ALL << 16) != 0, is_special)
    # both halves at once, without crosstalk
    rng = np.random.default_rng(3)
    a, b = rng.integers(0, 1 << 16, 200000, dtype=np.uint32), rng.integers(0, 1 << 16, 200000, dtype=np.uint32)
    s = special_bits(a | (b << 16))
    assert np.array_equal((s & 0x8000) != 0, (a & 0x7F80) == 0x7F80)
    assert np.array_equal((s & 0x80000000) != 0, (b & 0x7F80) == 0x7F80)


def test_scaled_products_are_exact_and_unscaled():
    """x * 2^-896 (from the widening) times c * 2^896 (the table) equals
    x * c exactly, for every finite bf16 x and float c of the rotation's
    range (|c| <= 1, with the subnormal floats the table can hold)."""
    rng = np.random.default_rng(4)
    x = bf16_bits_to_f64(FINITE.astype(np.uint16))
    for c in (np.cos(rng.uniform(0, 7, 8)).astype(np.float32), np.float32([1.0, -1.0, 1e-30, 1.4e-45])):
        for cv in c.astype(np.float64):
            assert np.array_equal(scaled_lo(FINITE) * (cv * 2.0 ** 896), x * cv)


def test_round_to_odd_narrowing_equals_direct_rounding():
    rng = np.random.default_rng(5)
    n = 400000
    mids = bf16_bits_to_f64(rng.integers(0x0080, 0x7F7F, n).astype(np.uint16)) * (1 + 2.0 ** -9)
    cases = [
        rng.standard_normal(n),
        rng.standard_normal(n) * 3e38,                                       # overflow edge
        3.3895313892515355e38 * (1 + rng.uniform(-2.0 ** -8, 2.0 ** -8, n)),  # around bf16's max
        rng.standard_normal(n) * 1e-36,                                      # near float's minimum
        mids, np.nextafter(mids, np.inf), np.nextafter(mids, -np.inf),       # bf16 midpoints
        -mids, np.nextafter(-mids, -np.inf),
    ]
    for y in cases:
        got, fast = narrow(y)
        with np.errstate(over="ignore"):
            want = f64_to_bf16_bits(y)
        assert fast.any()
        assert np.array_equal(got[fast], want[fast])


def test_rotated_words_through_the_fast_path_match_the_oracle():
    """Whole rotations: random bf16 pairs and table values, the kernel's
    scaled products with one FMA-style rounding (products exact, sum rounded
    once: plain double arithmetic here), narrowed the fast way where it
    applies, against rounding the exact double result."""
    rng = np.random.default_rng(6)
    n = 300000
    w1 = rng.integers(0, 1 << 16, n, dtype=np.uint32)
    w2 = rng.integers(0, 1 << 16, n, dtype=np.uint32)
    keep = ((w1 & 0x7F80) != 0x7F80) & ((w2 & 0x7F80) != 0x7F80)
    w1, w2 = w1[keep], w2[keep]
    a = rng.uniform(0, 2 * np.pi, w1.size)
    c = np.cos(a).astype(np.float32).astype(np.float64)
    s = np.sin(a).astype(np.float32).astype(np.float64)
    x1, x2 = scaled_lo(w1), scaled_lo(w2)
    y1 = x1 * (c * 2.0 ** 896) - x2 * (s * 2.0 ** 896)
    want = f64_to_bf16_bits(bf16_bits_to_f64(w1.astype(np.uint16)) * c - bf16_bits_to_f64(w2.astype(np.uint16)) * s)
    got, fast = narrow(y1)
    assert fast.mean() > 0.5
    assert np.array_equal(got[fast], want[fast])
