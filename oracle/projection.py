"""The Q/K/V projection in front of the hot path and the output projection
behind it, oracle side (test infrastructure only).

The pages run whole transformer models (LLaMA, Mistral, OPT: research-library
card "DeepSpeed-FastGen — paper by Holmes et al. (2024)", Key points); each
layer's attention step starts from q, k and v produced by a linear layer from
the hidden states. The plainest reading, with bf16 activations and weights:
qkv = x W^T summed exactly and rounded once to bf16 (ties to even), as a
linear layer with bf16 output returns it. (A float64 sum is not enough on its
own: its rounding error, though far below a bf16 unit, can move a sum that
lies next to a bf16 rounding boundary across it, and where that happens
depends on the order the BLAS library sums in.) W has the layout of a linear layer's weight: [(Hq + 2 Hkv) d,
hidden], the q heads' rows first, then k, then v. The output projection is
the same linear layer applied to the attention output viewed as rows of
Hq d values: y = o W_o^T, W_o of shape [out_features, Hq d]."""
import math

import numpy as np

from .bf16 import bf16_bits_to_f64, f64_to_bf16_bits

_U = 2.0 ** -53  # unit roundoff of float64


def is_bf16_midpoint(v) -> np.ndarray:
    """True where float64 v lies exactly halfway between two neighbouring
    bf16 values (the boundary above the largest finite bf16, where rounding
    turns to infinity, included). The bf16 values next to |v| = m 2^e
    (0.5 <= m < 1) are multiples of the quantum 2^(e-8), or of 2^-133 below
    the normal range; a midpoint is an odd multiple of half a quantum."""
    v = np.abs(np.asarray(v, dtype=np.float64))
    fin = np.isfinite(v) & (v > 0)
    _, e = np.frexp(np.where(fin, v, 1.0))
    k = np.where(e - 1 >= -126, 9 - e, 134)
    y = np.ldexp(np.where(fin, v, 0.0), k)
    return fin & (y == np.floor(y)) & (np.fmod(y, 2.0) == 1.0)


def round_exact_sum(terms) -> np.uint16:
    """bf16 bits of the exact sum of `terms` (float64 values, each exact),
    rounded once to the nearest bf16, ties to even. math.fsum returns the
    float64 value nearest the exact sum; its bf16 rounding is the exact sum's
    unless it sits exactly on a bf16 midpoint (every midpoint is a float64
    value, so the exact sum and its nearest float64 lie on the same side of
    any other one). There the sign of the remainder, exact sum minus that
    value (fsum again: a nonzero exact value never rounds to zero or changes
    sign), says which way the exact sum lies, and one float64 step off the
    midpoint in that direction rounds to the right bf16; a zero remainder is
    a true tie."""
    terms = [float(t) for t in terms]
    r = math.fsum(terms)
    if is_bf16_midpoint(r):
        rem = math.fsum(terms + [-r])
        if rem != 0.0:
            r = float(np.nextafter(r, np.inf if rem > 0 else -np.inf))
    return f64_to_bf16_bits(np.float64(r))[()]


def linear(x_bits, w_bits):
    """A linear layer with bf16 input, weight and output: x_bits [T, K] and
    w_bits [N, K] as bf16 words (finite values); returns the bf16 words of
    x W^T [T, N], each the exact sum of its K products rounded once to bf16
    (ties to even).

    Every product of two bf16 values is exact in float64 (two 8-bit
    significands), so a float64 sum of them in any order is within
    gamma_K * sum |x_i w_i| of the exact sum (gamma_K = K u / (1 - K u), u the
    float64 unit roundoff). Where the float64 result r, and r moved by twice
    that bound both ways (four times gamma_K times the float64 sum of
    magnitudes, which is itself within gamma_K of the true one), all round to
    the same bf16 and none of the three is a bf16 midpoint, no rounding
    boundary lies between r and the exact sum, and r's rounding is the exact
    sum's. Every other output is summed exactly (round_exact_sum)."""
    x = bf16_bits_to_f64(np.asarray(x_bits, dtype=np.uint16))
    w = bf16_bits_to_f64(np.asarray(w_bits, dtype=np.uint16))
    K = x.shape[1]
    r = x @ w.T
    g = K * _U / (1.0 - K * _U)
    bound = 4.0 * g * (np.abs(x) @ np.abs(w).T)
    lo, hi = r - bound, r + bound
    out = f64_to_bf16_bits(r)
    sure = ((f64_to_bf16_bits(lo) == out) & (f64_to_bf16_bits(hi) == out) &
            ~is_bf16_midpoint(lo) & ~is_bf16_midpoint(r) & ~is_bf16_midpoint(hi))
    for t, j in zip(*np.nonzero(~sure)):
        out[t, j] = round_exact_sum(x[t] * w[j])
    return out


def qkv_projection(x_bits, w_bits, n_q_heads, n_kv_heads, head_dim):
    """x_bits [T, hidden] and w_bits [(Hq + 2 Hkv) d, hidden] as bf16 words.
    Returns (q, k, v) bf16 words shaped [T, Hq, d], [T, Hkv, d], [T, Hkv, d]."""
    y = linear(x_bits, w_bits)
    T = y.shape[0]
    hq, hkv, d = n_q_heads, n_kv_heads, head_dim
    q = y[:, :hq * d].reshape(T, hq, d)
    k = y[:, hq * d:(hq + hkv) * d].reshape(T, hkv, d)
    v = y[:, (hq + hkv) * d:].reshape(T, hkv, d)
    return q, k, v
