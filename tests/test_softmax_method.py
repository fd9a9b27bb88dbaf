"""The attention kernels' numerical method, replayed on the host in float32.

The method: scores in fp32; an online softmax over 64-key tiles in log2
units whose running maximum moves only when a tile raises it by more than 8
(2^8); P rounded to bf16 for the P.V product while the row sum keeps the
fp32 values; optional split-KV pieces merged by a log-sum-exp combine; the
output rounded to bf16. These tests replay it with numpy and compare against
the exact float64 softmax (the oracle's definition), to show that the
parity tolerances hold for the method itself:
- max-abs 2e-2 and relative L2 5e-3 on N(0,1) data;
- on peaked scores, the bound derived from the method's two roundings to
  bf16 (unit roundoff 2^-8: 8 significant bits, ties to even):
      |bf16(O_k) - O| <= 2^-8 |O| + 2^-8 (1 + 2^-8) A + e,
  where O_k = sum bf16(p) V / sum p is the kernel's unrounded output (each
  weight off by at most 2^-8 of itself, so O_k is within 2^-8 A of O, with
  A = sum p|V| / sum p), the output rounding adds at most 2^-8 |O_k|, and e
  collects the fp32 effects (scores, ex2.approx, sums), covered by the fixed
  2e-2;
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


def peaked_bound(ref, mass):
    """The derived per-output bound (module docstring), with the fixed 2e-2
    standing for the fp32 effects."""
    return 2e-2 + 2.0 ** -8 * np.abs(ref) + 2.0 ** -8 * (1 + 2.0 ** -8) * mass


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
        bound = peaked_bound(ref, mass)
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


def test_replay_of_the_peaked_grouped_query_case():
    """The GPU parity case with peaked scores at 8/2 heads, d = 64 (queries
    times 16): its 300-token prompt chunk at context 0 runs on the query-tile
    kernel, the method replayed here. On the same data (the oracle's rotated
    queries and cache, every chunk row and head) the method itself exceeds
    the fixed 2e-2 on an output above 4 in magnitude, where rounding to bf16
    alone can move a value by 2^-6, and every output stays within the derived
    bound: an error of that size is the method's, not a kernel defect."""
    from oracle import PagedCache
    from oracle.forward import splitfuse_pass
    from ragged_paged_kv_b200 import fixtures
    from ragged_paged_kv_b200 import workloads as W
    w = W._make("peaked_gqa_d64", 8, 2, 64, 16, [0, 1, 2, 3], [300, 1, 1, 17], [0, 3000, 700, 500],
                seed=41, budget=319)
    q0, k, v = w.qkv()
    q = f64_to_bf16_bits(bf16_bits_to_f64(q0) * 16.0)
    pc = PagedCache(w.n_blocks, w.n_kv_heads, w.block_size, w.head_dim, fill=fixtures.SENTINEL)
    for s_ in range(w.n_seqs):
        ids, blocks = fixtures.context_blocks(w, s_)
        for i, b in enumerate(ids):
            pc.blocks[int(b)] = blocks[i].copy()
    q_rot, _, ref = splitfuse_pass(pc, w.block_tables, w.q_lens, w.ctx_lens, q, k, v, w.rope_theta,
                                   w.softmax_scale, 0)
    K, V = (bf16_bits_to_f64(a) for a in pc.gather(w.block_tables[0], int(w.q_lens[0])))
    g = w.n_q_heads // w.n_kv_heads
    errs, over = [], 0
    for t in range(int(w.q_lens[0])):
        for h in range(w.n_q_heads):
            qv = bf16_bits_to_f64(q_rot[t, h])[None, :]
            Kh, Vh = K[:t + 1, h // g], V[:t + 1, h // g]
            O, m, l = online(qv, Kh, Vh, w.softmax_scale)
            got = bf16(O / l[:, None])[0]
            _, mass = exact(qv, Kh, Vh, w.softmax_scale)
            err = np.abs(got - ref[t, h])
            assert np.all(err <= peaked_bound(ref[t, h], mass[0])), (t, h)
            over += int(np.sum((err > 2e-2) & (np.abs(ref[t, h]) > 4)))
            errs.append(err.max())
    assert over >= 1 and max(errs) > 2e-2
