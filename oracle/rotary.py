"""Rotary position embedding, oracle side (test infrastructure only).

The pages name the HuggingFace LLaMA / LLaMA-2 and Mistral families as the
supported models ("DeepSpeed-FastGen — paper by Holmes et al. (2024)", Key
points). They print no rotary formula, so this follows the plainest reading
consistent with those families:

  * pairing is rotate-half: element i is paired with element i + d/2;
  * frequency i (0 <= i < d/2) is inv_freq_i = 1 / theta**(2i/d), in double;
  * for absolute position p the angle is a = p * inv_freq_i (double); its cosine
    and sine come from the C library's double cos/sin and are rounded once to
    float32 (the table a bf16 model keeps);
  * the rotation itself is done in double: each product of a bf16 value and a
    float32 table entry is exact in double, the sum rounds once, and the
    result is rounded directly to bf16 (ties to even):
        y[i]       = bf16(x[i] * c - x[i+d/2] * s)
        y[i + d/2] = bf16(x[i+d/2] * c + x[i] * s)

Scalar ``math.cos`` / ``math.sin`` / ``**`` are used on purpose: they are the
platform C library's double routines, not numpy's vectorised ones.
"""
import math

import numpy as np

from .bf16 import bf16_bits_to_f64, f64_to_bf16_bits


def inv_freq(theta: float, head_dim: int) -> list:
    return [1.0 / (float(theta) ** ((2.0 * i) / float(head_dim))) for i in range(head_dim // 2)]


def rope_table(theta: float, head_dim: int, positions, exact: bool = False):
    """cos/sin table [n_pos, d/2] for the given absolute positions.

    float32 by default; ``exact=True`` keeps float64 (used only by the
    relative-position invariance pin)."""
    f = inv_freq(theta, head_dim)
    positions = [int(p) for p in np.asarray(positions).reshape(-1)]
    uniq = sorted(set(positions))
    rows_c, rows_s = {}, {}
    for p in uniq:
        a = [float(p) * fi for fi in f]
        rows_c[p] = [math.cos(t) for t in a]
        rows_s[p] = [math.sin(t) for t in a]
    dt = np.float64 if exact else np.float32
    c = np.array([rows_c[p] for p in positions], dtype=np.float64).astype(dt)
    s = np.array([rows_s[p] for p in positions], dtype=np.float64).astype(dt)
    return c, s


def rotate_half(x_bits, positions, theta: float, exact: bool = False):
    """Rotate bf16 vectors x [n, H, d] at per-row absolute positions [n].

    Returns bf16 bits (default) or, with ``exact=True``, the unrounded float64
    rotation with an unrounded float64 table."""
    x_bits = np.asarray(x_bits)
    x = bf16_bits_to_f64(x_bits) if x_bits.dtype == np.uint16 else x_bits.astype(np.float64)
    n, H, d = x.shape
    h = d // 2
    c, s = rope_table(theta, d, positions, exact=exact)
    c = c.astype(np.float64)[:, None, :]          # [n, 1, d/2]
    s = s.astype(np.float64)[:, None, :]
    x1, x2 = x[..., :h], x[..., h:]
    y = np.empty_like(x)
    y[..., :h] = x1 * c - x2 * s
    y[..., h:] = x2 * c + x1 * s
    return y if exact else f64_to_bf16_bits(y)
