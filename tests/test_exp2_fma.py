"""The query-tile kernel's FMA-pipe exponential (ex2_fma2 in attn_tc.cu),
replayed on the host step by step in float32 with its own coefficients:

- Cody-Waite range reduction: j = rint(x) by adding 1.5 * 2^23 (the low
  mantissa bits of the sum then hold j), f = x - j in [-1/2, 1/2];
- a degree-5 polynomial for 2^f in Horner form with fused multiply-adds;
- 2^j placed by adding (sum bits) << 23 to the polynomial's bits.

Checked against 2^x in float64: relative error within 2^-21 (the order of
ex2.approx's own error) wherever the result is a normal float; for the
clamped bottom of the range (x <= -126, masked keys at -inf) a non-negative
value below 2^-125 that is never NaN; -inf rounds to bf16 zero. The
coefficients are checked against a fresh fit (exp2_poly_fit.py)."""
import os
import re

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "ragged_paged_kv_b200", "csrc", "attn_tc.cu")


def kernel_coefficients():
    txt = open(SRC).read()
    found = dict(re.findall(r"kExp2C(\d) = (0x[0-9a-fA-Fp.+-]+)f", txt))
    return [np.float32(float.fromhex(found[str(i)])) for i in range(6)]


def f32(x):
    return np.asarray(x, dtype=np.float32)


def fma32(a, b, c):
    # the product of two float32 values is exact in float64; one rounding
    # of the sum to float64, then to float32
    return (a.astype(np.float64) * b.astype(np.float64) + c.astype(np.float64)).astype(np.float32)


def ex2_fma(x):
    C = kernel_coefficients()
    x = np.maximum(f32(x), np.float32(-127.0))
    magic = np.float32(12582912.0)
    t = (x + magic).astype(np.float32)
    j = (t - magic).astype(np.float32)
    f = fma32(j, f32(-1.0), x)
    p = fma32(np.full_like(f, C[5]), f, np.full_like(f, C[4]))
    for c in (C[3], C[2], C[1], C[0]):
        p = fma32(p, f, np.full_like(f, c))
    bits = (p.view(np.uint32) + (t.view(np.uint32) << np.uint32(23))).astype(np.uint32)
    return bits.view(np.float32)


def test_relative_error_on_the_normal_range():
    rng = np.random.default_rng(3)
    x = np.concatenate([rng.uniform(-126.0, 9.0, 2_000_000),
                        np.arange(-126, 10, dtype=np.float64) + 0.5,        # rint ties
                        np.arange(-126, 10, dtype=np.float64),
                        np.nextafter(np.arange(-125, 10, dtype=np.float64) + 0.5, 0)])
    x = f32(x)
    y = ex2_fma(x).astype(np.float64)
    ref = np.exp2(x.astype(np.float64))
    rel = np.abs(y / ref - 1.0)
    assert np.isfinite(y).all()
    assert rel.max() <= 2.0 ** -21, rel.max()


def test_bottom_of_the_range_is_small_nonnegative_and_never_nan():
    x = f32(np.concatenate([[-np.inf, -1e30, -300.0, -127.0, -126.75, -126.5, -126.25],
                            np.linspace(-140.0, -126.0, 10001)]))
    y = ex2_fma(x)
    assert not np.isnan(y).any()
    assert (y >= 0).all() and (y < 2.0 ** -125).all()
    # the masked keys: rounds to bf16 zero
    from oracle.bf16 import f64_to_bf16_bits
    assert f64_to_bf16_bits(ex2_fma(f32([-np.inf])).astype(np.float64))[0] == 0


def test_coefficients_match_a_fresh_fit():
    import importlib.util
    spec = importlib.util.spec_from_file_location(
        "fit", os.path.join(ROOT, "ragged_paged_kv_b200", "csrc", "exp2_poly_fit.py"))
    fit = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(fit)
    c = fit.remez_relative(5).astype(np.float32)
    assert np.array_equal(c, np.array(kernel_coefficients(), dtype=np.float32))
