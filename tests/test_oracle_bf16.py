"""Pins for the oracle's float64 -> bf16 rounding: brute-force nearest search
over every finite bf16 value, and torch's float32 -> bf16 rounding on values
that are exactly float32 (there a direct rounding and torch's must agree)."""
import numpy as np
import torch

from oracle import bf16_bits_to_f64, f64_to_bf16_bits


def _all_finite_bf16():
    pos = np.arange(0x0000, 0x7F80, dtype=np.uint32)           # +0 .. max finite
    bits = np.concatenate([pos[::-1] | 0x8000, pos]).astype(np.uint16)
    vals = (bits.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    order = np.argsort(vals, kind="stable")
    return vals[order], bits[order]


VALS, BITS = _all_finite_bf16()


def brute_nearest_bf16(x):
    """Nearest finite bf16 to each float64 (ties to the even pattern), by
    search over the full sorted table; inputs stay within the finite range."""
    x = np.asarray(x, dtype=np.float64).reshape(-1)
    i = np.clip(np.searchsorted(VALS, x), 1, len(VALS) - 1)
    lo_v, hi_v = VALS[i - 1], VALS[i]
    lo_b, hi_b = BITS[i - 1], BITS[i]
    dlo, dhi = x - lo_v, hi_v - x
    pick_hi = (dhi < dlo) | ((dhi == dlo) & ((hi_b & 1) == 0))
    out = np.where(pick_hi, hi_b, lo_b)
    # signed zero: keep the sign of x (brute table holds -0 and +0 at the same value)
    zero = out & 0x7FFF == 0
    out = np.where(zero, np.where(np.signbit(x), 0x8000, 0x0000), out)
    return out.astype(np.uint16)


def test_widening_is_exact_for_every_pattern():
    b = np.arange(0, 1 << 16, dtype=np.uint32).astype(np.uint16)
    f = bf16_bits_to_f64(b)
    finite = np.isfinite(f)
    back = f64_to_bf16_bits(f[finite])
    assert np.array_equal(back, b[finite])


def test_random_doubles_match_brute_force():
    rng = np.random.default_rng(11)
    x = np.concatenate([
        rng.standard_normal(200_000) * 3.0,
        rng.standard_normal(50_000) * 1e-39,          # bf16 subnormal range
        rng.standard_normal(50_000) * 1e30,
        np.ldexp(rng.uniform(0.5, 1.0, 20_000), rng.integers(-140, 120, 20_000)),
    ])
    assert np.array_equal(f64_to_bf16_bits(x), brute_nearest_bf16(x))


def test_exact_midpoints_round_to_even_and_off_midpoints_do_not():
    rng = np.random.default_rng(12)
    b = rng.integers(0x0080, 0x7F00, 20_000).astype(np.uint16)     # normal, positive
    lo = bf16_bits_to_f64(b)
    hi = bf16_bits_to_f64(b + np.uint16(1))
    mid = (lo + hi) / 2.0                                           # exact in float64
    got = f64_to_bf16_bits(mid)
    want = np.where(b & 1, b + np.uint16(1), b).astype(np.uint16)
    assert np.array_equal(got, want)
    # a hair above the midpoint (not representable in float32) must round up:
    # a conversion through float32 would first land on the midpoint and
    # round to even, i.e. down for even b.
    above = mid + (hi - lo) * 2.0 ** -30
    assert np.array_equal(f64_to_bf16_bits(above), b + np.uint16(1))
    assert np.array_equal(f64_to_bf16_bits(-above), (b + np.uint16(1)) | np.uint16(0x8000))


def test_float32_inputs_match_torch_rounding():
    rng = np.random.default_rng(13)
    x32 = np.concatenate([
        rng.standard_normal(100_000).astype(np.float32),
        (rng.standard_normal(10_000) * 1e-39).astype(np.float32),
        rng.integers(0, 1 << 31, 50_000, dtype=np.uint32).astype(np.uint32).view(np.float32),
    ])
    x32 = x32[np.isfinite(x32) & (np.abs(x32) < 3.3e38)]
    t = torch.from_numpy(x32.copy()).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(f64_to_bf16_bits(x32.astype(np.float64)), t)


def test_specials():
    x = np.array([np.nan, np.inf, -np.inf, 0.0, -0.0, 1e300, -1e300])
    b = f64_to_bf16_bits(x)
    assert b[0] & 0x7F80 == 0x7F80 and b[0] & 0x7F
    assert list(b[1:]) == [0x7F80, 0xFF80, 0x0000, 0x8000, 0x7F80, 0xFF80]
