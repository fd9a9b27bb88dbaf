"""Ragged causal attention over a gathered context, oracle side (test
infrastructure only).

Each new token attends to every cached token of its own sequence up to and
including itself ("DeepSpeed-FastGen — paper by Holmes et al. (2024)", Summary:
a pass mixes prompt chunks, whose tokens see the earlier chunks already in the
cache, with generation tokens, which see their whole context). Readings where
the pages are silent:

  * scores z_k = scale * <q, k_k> with scale = 1/sqrt(d) (a call argument);
  * grouped-query heads: q head h reads kv head h // (Hq / Hkv);
  * sliding window W > 0 (Mistral, named under Key points): key position k is
    admitted for a query at position p iff p - W < k <= p; W = 0 means none;
  * the result is the exact softmax-weighted mean in float64:
        O = sum_k exp(z_k - m) V_k / sum_k exp(z_k - m),  m = max_k z_k.

The context is gathered into a contiguous float64 array per (sequence, kv head)
before any arithmetic; query rows are taken in blocks of at most 1024 only to
bound memory (rows are independent).
"""
import numpy as np

from .bf16 import bf16_bits_to_f64
from .paged_cache import PagedCache

ROW_BLOCK = 1024


def attend_contiguous(q, positions, K, V, scale, window=0):
    """q [n, d] float64 at absolute positions [n]; K, V [L, d] float64 hold
    positions 0..L-1. Returns O [n, d] float64."""
    q = np.asarray(q, dtype=np.float64)
    positions = np.asarray(positions, dtype=np.int64)
    out = np.empty((q.shape[0], V.shape[1]), dtype=np.float64)
    for r0 in range(0, q.shape[0], ROW_BLOCK):
        pr = positions[r0:r0 + ROW_BLOCK]
        lo = np.maximum(0, pr - window + 1) if window > 0 else np.zeros_like(pr)
        k0, k1 = int(lo.min()), int(pr.max()) + 1
        keys = np.arange(k0, k1)
        z = scale * (q[r0:r0 + ROW_BLOCK] @ K[k0:k1].T)
        ok = (keys[None, :] >= lo[:, None]) & (keys[None, :] <= pr[:, None])
        z = np.where(ok, z, -np.inf)
        m = z.max(axis=1, keepdims=True)
        w = np.exp(z - m)
        out[r0:r0 + ROW_BLOCK] = (w @ V[k0:k1]) / w.sum(axis=1, keepdims=True)
    return out


def ragged_attention(cache: PagedCache, block_tables, q_lens, ctx_lens, q_rot_bits,
                     scale, window=0, tokens=None):
    """Attention output for a ragged batch, float64 [T, Hq, d].

    ``tokens``: optional sorted batch-row indices to compute (others are NaN);
    used to sample very large batches."""
    q_all = np.asarray(q_rot_bits)
    T, Hq, d = q_all.shape
    Hkv = cache.n_kv_heads
    g = Hq // Hkv
    out = np.full((T, Hq, d), np.nan, dtype=np.float64)
    want = np.ones(T, dtype=bool) if tokens is None else np.isin(np.arange(T), tokens)
    start = 0
    for s in range(len(q_lens)):
        qs, cs = int(q_lens[s]), int(ctx_lens[s])
        rows = np.arange(start, start + qs)
        start += qs
        rows = rows[want[rows]]
        if len(rows) == 0:
            continue
        pos = cs + (rows - (start - qs))
        L = int(pos.max()) + 1
        Kw, Vw = cache.gather(block_tables[s], L)
        for hk in range(Hkv):
            K = bf16_bits_to_f64(Kw[:, hk, :])
            V = bf16_bits_to_f64(Vw[:, hk, :])
            for h in range(hk * g, (hk + 1) * g):
                q = bf16_bits_to_f64(q_all[rows, h, :])
                out[rows, h, :] = attend_contiguous(q, pos, K, V, scale, window)
    return out
