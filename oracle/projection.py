"""The Q/K/V projection in front of the hot path and the output projection
behind it, oracle side (test infrastructure only).

The pages run whole transformer models (LLaMA, Mistral, OPT: research-library
card "DeepSpeed-FastGen — paper by Holmes et al. (2024)", Key points); each
layer's attention step starts from q, k and v produced by a linear layer from
the hidden states. The plainest reading, with bf16 activations and weights:
qkv = x W^T computed exactly (float64 here: every product of two bf16 values
is exact, and a 4096-term sum of them loses far less than a bf16 unit) and
rounded once to bf16 (ties to even), as a linear layer with bf16 output
returns it. W has the layout of a linear layer's weight: [(Hq + 2 Hkv) d,
hidden], the q heads' rows first, then k, then v. The output projection is
the same linear layer applied to the attention output viewed as rows of
Hq d values: y = o W_o^T, W_o of shape [out_features, Hq d]."""
import numpy as np

from .bf16 import bf16_bits_to_f64, f64_to_bf16_bits


def linear(x_bits, w_bits):
    """A linear layer with bf16 input, weight and output: x_bits [T, K] and
    w_bits [N, K] as bf16 words; returns the bf16 words of x W^T [T, N], each
    sum taken in float64 and rounded once to bf16 (ties to even)."""
    x = bf16_bits_to_f64(np.asarray(x_bits, dtype=np.uint16))
    w = bf16_bits_to_f64(np.asarray(w_bits, dtype=np.uint16))
    return f64_to_bf16_bits(x @ w.T)


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
