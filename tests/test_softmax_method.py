"""The attention kernels' numerical method, replayed on the host in float32.

The method: scores in fp32; an online softmax over 64-key tiles in log2
units whose running maximum moves only when a tile raises it by more than 8
(2^8); P rounded to bf16 for the P.V product while the row sum keeps the
fp32 values; optional split-KV pieces merged by a log-sum-exp combine; the
output rounded to bf16. These tests replay it with numpy and compare against
the exact float64 softmax (the oracle's definition), to show that the
parity tolerances hold for the method itself:
- max-abs 2e-2 and relative L2 5e-3 on N(0,1) data;
- 2e-2 + 2^-8 |O| + 2^-7 A on peaked scores, with A = sum p|V| / sum p;
- splitting and combining moves the result by no more than the bf16
  rounding of P does: each piece rounds its weights against its own running
  maximum, so the rounding errors differ, bounded by 2^-8 A.
"""
import numpy as np

from oracle.bf16 import bf16_bits_to_f64, f64_to_bf16_bits

LOG2E = 1.4426950408889634


def bf16(x):
    return bf16_bits_to_f64(f64_to_bf16_bits(np.asarray(x, dtype=np.float64)))


def exact(q, K, V, scale):
    z = (q @ K.T) * scale
    w = np.exp(z - z.max(axis=-1, keepdims=True))
    return (w @ V) / w.sum(axis=-1, keepdims=True), (w @ np.abs(V)) / w.sum(axis=-1, keepdims=True)


def online(q, K, V, scale, tile=64, threshold=8.0):
    """One split: returns (O unnormalised, m, l) per row, fp32, log2 units."""
    q32, K32, V32 = q.astype(np.float32), K.astype(np.float32), V.astype(np.float32)
    rows = q.shape[0]
    m = np.full(rows, -np.inf, np.float32)
    l = np.zeros(rows, np.float32)
    O = np.zeros((rows, V.shape[1]), np.float32)
    sl2 = np.float32(scale * LOG2E)
    for k0 in range(0, K.shape[0], tile):
        s = (q32 @ K32[k0:k0 + tile].T).astype(np.float32)
        mt = s.max(axis=1) * sl2
        move = mt > m + np.float32(threshold)
        alpha = np.where(move, np.where(np.isinf(m), np.float32(0), np.exp2(m - mt)), np.float32(1))
        m = np.where(move, mt, m).astype(np.float32)
        O *= alpha[:, None]
        l *= alpha
        p = np.exp2(s * sl2 - m[:, None]).astype(np.float32)
        l += p.sum(axis=1, dtype=np.float32)
        O += (bf16(p).astype(np.float32) @ V32[k0:k0 + tile]).astype(np.float32)
    return O, m, l


def combine(parts):
    M = np.max([m for _, m, _ in parts], axis=0)
    O = sum(o * np.exp2(m - M)[:, None] for o, m, _ in parts)
    L = sum(l * np.exp2(m - M) for _, m, l in parts)
    return O / L[:, None]


def case(rng, rows, keys, d, q_scale):
    q = bf16(rng.standard_normal((rows, d)) * q_scale)
    K = bf16(rng.standard_normal((keys, d)))
    V = bf16(rng.standard_normal((keys, d)))
    return q, K, V, 1.0 / np.sqrt(d)


def test_normal_scores_meet_the_parity_tolerance():
    rng = np.random.default_rng(21)
    for d, keys in ((128, 4000), (64, 1500)):
        q, K, V, scale = case(rng, 64, keys, d, 1.0)
        ref, _ = exact(q, K, V, scale)
        O, m, l = online(q, K, V, scale)
        got = bf16(O / l[:, None])
        err = np.abs(got - ref)
        assert err.max() <= 2e-2
        assert np.linalg.norm(got - ref) / np.linalg.norm(ref) <= 5e-3


def test_peaked_scores_meet_the_derived_bound():
    rng = np.random.default_rng(22)
    for d, keys in ((128, 3000), (64, 3000)):
        q, K, V, scale = case(rng, 64, keys, d, 16.0)
        ref, mass = exact(q, K, V, scale)
        O, m, l = online(q, K, V, scale)
        got = bf16(O / l[:, None])
        bound = 2e-2 + 2.0 ** -8 * np.abs(ref) + 2.0 ** -7 * mass
        assert np.all(np.abs(got - ref) <= bound)
        assert np.linalg.norm(got - ref) / np.linalg.norm(ref) <= 5e-3
        # the rescale really ran: the running maximum moved after the first tile
        _, m1, _ = online(q, K[:64], V[:64], scale)
        assert np.any(m > m1 + 8)


def test_split_and_combine_stays_within_the_weight_rounding():
    rng = np.random.default_rng(23)
    for q_scale in (1.0, 16.0):
        q, K, V, scale = case(rng, 16, 5000, 128, q_scale)
        _, mass = exact(q, K, V, scale)
        O, m, l = online(q, K, V, scale)
        one = O / l[:, None]
        for cut in (1024, 2048, 4096):
            parts = [online(q, K[:cut], V[:cut], scale), online(q, K[cut:], V[cut:], scale)]
            both = combine(parts)
            assert np.all(np.abs(both - one) <= 2.0 ** -8 * mass + 1e-6)
