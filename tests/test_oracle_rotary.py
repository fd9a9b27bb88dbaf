"""Pins for the oracle's rotary step: identity at position 0, the complex
rotation it must equal, HuggingFace's rotate-half implementation, the
relative-position property that defines rotary, norm preservation and the
frequency closed form."""
import math

import numpy as np
import torch

from oracle import bf16_bits_to_f64, inv_freq, rope_table, rotate_half
from ragged_paged_kv_b200.workloads import f32_to_bf16_bits
from tests.test_oracle_bf16 import brute_nearest_bf16


def _x(n, H, d, seed):
    rng = np.random.default_rng(seed)
    return f32_to_bf16_bits(rng.standard_normal((n, H, d), dtype=np.float32))


def test_inv_freq_closed_form():
    f = inv_freq(10000.0, 128)
    assert f[0] == 1.0
    assert math.isclose(f[32], 0.01, rel_tol=1e-15)                # 10000**(-64/128)
    assert math.isclose(f[63], 10000.0 ** (-126 / 128), rel_tol=1e-15)
    assert all(a > b for a, b in zip(f, f[1:]))


def test_position_zero_is_identity_bit_exact():
    x = _x(5, 3, 64, 1)
    y = rotate_half(x, np.zeros(5, dtype=np.int64), 10000.0)
    assert np.array_equal(x, y)


def test_table_matches_numpy_within_one_float32_ulp():
    pos = np.arange(0, 40000, 97)
    c, s = rope_table(10000.0, 128, pos)
    f = np.array(inv_freq(10000.0, 128))
    a = pos[:, None].astype(np.float64) * f[None, :]
    for ours, ref in ((c, np.cos(a)), (s, np.sin(a))):
        ref32 = ref.astype(np.float32)
        d = np.abs(ours.view(np.int32).astype(np.int64) - ref32.view(np.int32).astype(np.int64))
        assert d.max() <= 1
        assert (d == 0).mean() > 0.999


def test_equals_complex_rotation_rounded_once():
    """y_i + i*y_{i+d/2} = (x_i + i*x_{i+d/2}) * (c + i*s), rounded to bf16."""
    n, H, d = 64, 4, 64
    x = _x(n, H, d, 2)
    pos = np.random.default_rng(3).integers(0, 50000, n)
    c, s = rope_table(10000.0, d, pos)
    xf = bf16_bits_to_f64(x)
    z = (xf[..., :d // 2] + 1j * xf[..., d // 2:]) * (c.astype(np.float64) + 1j * s.astype(np.float64))[:, None, :]
    want = np.concatenate([brute_nearest_bf16(z.real).reshape(z.shape),
                           brute_nearest_bf16(z.imag).reshape(z.shape)], axis=-1)
    assert np.array_equal(rotate_half(x, pos, 10000.0), want)


def test_matches_huggingface_rotate_half():
    from transformers.models.llama.modeling_llama import apply_rotary_pos_emb
    n, Hq, Hkv, d = 48, 4, 2, 128
    q, k = _x(n, Hq, d, 4), _x(n, Hkv, d, 5)
    pos = np.random.default_rng(6).integers(0, 33000, n)
    c, s = rope_table(10000.0, d, pos)
    cos = torch.from_numpy(np.concatenate([c, c], axis=1).astype(np.float64))[None]  # [1, n, d]
    sin = torch.from_numpy(np.concatenate([s, s], axis=1).astype(np.float64))[None]
    qt = torch.from_numpy(bf16_bits_to_f64(q)).permute(1, 0, 2)[None]                # [1, H, n, d]
    kt = torch.from_numpy(bf16_bits_to_f64(k)).permute(1, 0, 2)[None]
    qh, kh = apply_rotary_pos_emb(qt, kt, cos, sin)
    for ours, ref in ((rotate_half(q, pos, 10000.0), qh), (rotate_half(k, pos, 10000.0), kh)):
        ref = ref[0].permute(1, 0, 2).numpy()
        assert np.array_equal(ours, brute_nearest_bf16(ref).reshape(ref.shape))


def test_scores_depend_only_on_relative_position():
    """Unrounded rotary: <R(p) q, R(k) k> == <R(p+D) q, R(k+D) k>."""
    d = 128
    q = bf16_bits_to_f64(_x(1, 1, d, 7))
    k = bf16_bits_to_f64(_x(1, 1, d, 8))
    for p, kp, D in ((5, 3, 1000), (30000, 17, 2345), (100, 100, 31)):
        a = (rotate_half(q, [p], 1e4, exact=True) * rotate_half(k, [kp], 1e4, exact=True)).sum()
        b = (rotate_half(q, [p + D], 1e4, exact=True) * rotate_half(k, [kp + D], 1e4, exact=True)).sum()
        assert abs(a - b) <= 1e-10 * max(1.0, abs(a))


def test_unrounded_rotation_preserves_pair_norms():
    x = bf16_bits_to_f64(_x(16, 2, 64, 9))
    pos = np.arange(0, 16 * 777, 777)
    y = rotate_half(x, pos, 1e4, exact=True)
    nx = x[..., :32] ** 2 + x[..., 32:] ** 2
    ny = y[..., :32] ** 2 + y[..., 32:] ** 2
    assert np.allclose(nx, ny, rtol=1e-14, atol=1e-300)
