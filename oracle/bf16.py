"""bf16 <-> float64 conversions for the oracle (test infrastructure only).

bf16 is the storage type of the model's activations and of the KV cache (the
pages name bf16-era HuggingFace LLaMA / Mistral models; the precision of each
step is a stated reading, see rotary.py). Rounding here is one direct rounding
from float64 to the nearest bf16 value, ties to even, with bf16's subnormals
(quantum 2**-133), never through float32.
"""
import numpy as np

_BF16_MAX_EXP = 127          # largest unbiased exponent of a finite bf16
_BF16_MIN_NORMAL_EXP = -126  # smallest unbiased exponent of a normal bf16


def bf16_bits_to_f64(bits) -> np.ndarray:
    """Exact widening: bf16 bit pattern -> float64 value."""
    b = np.asarray(bits, dtype=np.uint16).astype(np.uint32) << np.uint32(16)
    with np.errstate(invalid="ignore"):      # NaN patterns widen to NaN
        return b.view(np.float32).astype(np.float64)


def f64_to_bf16_bits(x) -> np.ndarray:
    """Round float64 values to the nearest bf16 (ties to even); return bits.

    Method: write |x| = m * 2**e with 0.5 <= m < 1 (frexp, exact). A bf16 with
    that exponent has 8 significant bits, so its quantum is 2**(e-8); below the
    normal range the quantum is fixed at 2**-133. Scaling by a power of two is
    exact, so rint (ties to even) of x / quantum is the correctly rounded
    integer multiple; the product is then exactly representable in float32 and
    its upper 16 bits are the bf16 pattern.
    """
    x = np.asarray(x, dtype=np.float64)
    out = np.empty(x.shape, dtype=np.uint16)
    flat_x = x.reshape(-1)
    flat_o = out.reshape(-1)

    nan = np.isnan(flat_x)
    fin = np.isfinite(flat_x)
    _, e = np.frexp(flat_x)                       # e is exponent with 0.5<=|m|<1
    # unbiased exponent of the leading bit is e-1; bf16 normal needs e-1 >= -126
    q_exp = np.where(e - 1 >= _BF16_MIN_NORMAL_EXP, e - 8, -133)
    q = np.rint(np.ldexp(flat_x, -q_exp))          # exact scaling, RNE to integer
    r = np.ldexp(q, q_exp)                         # the rounded value, exact
    # overflow: a rounded magnitude of 2**128 or more is infinite in bf16
    over = fin & (np.abs(r) >= 2.0 ** (_BF16_MAX_EXP + 1))
    r = np.where(over, np.copysign(np.inf, flat_x), r)
    r = np.where(fin, r, flat_x)
    r32 = r.astype(np.float32)                     # exact for every finite r here
    bits = (r32.view(np.uint32) >> np.uint32(16)).astype(np.uint16)
    bits = np.where(nan, np.uint16(0x7FC0), bits)
    flat_o[:] = bits
    return out
