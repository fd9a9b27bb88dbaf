"""Pins for the oracle's paged append and ragged attention: brute-force dense
attention (torch SDPA in float64 with an explicit mask), closed forms (uniform
keys, single admitted key), and invariants (block permutation, chunking,
window >= length, grouped-query replication)."""
import numpy as np
import pytest
import torch

from oracle import (PagedCache, append_kv, attend_contiguous, bf16_bits_to_f64, f64_to_bf16_bits,
                    ragged_attention, token_positions)
from oracle.forward import splitfuse_pass
from ragged_paged_kv_b200 import workloads as W
from ragged_paged_kv_b200.workloads import f32_to_bf16_bits


def _bits(rng, shape):
    return f32_to_bf16_bits(rng.standard_normal(shape, dtype=np.float32))


def _sdpa_reference(q_lens, ctx_lens, Kc, Vc, Q, Hq, Hkv, window, scale):
    """Dense per-sequence attention with an explicit L x L boolean mask,
    float64, through torch's scaled_dot_product_attention."""
    out = []
    start = 0
    g = Hq // Hkv
    for s, (qs, cs) in enumerate(zip(q_lens, ctx_lens)):
        L = cs + qs
        qpos = torch.arange(cs, L)
        kpos = torch.arange(L)
        mask = kpos[None, :] <= qpos[:, None]
        if window > 0:
            mask &= kpos[None, :] > qpos[:, None] - window
        q = torch.from_numpy(bf16_bits_to_f64(Q[start:start + qs])).permute(1, 0, 2)    # [Hq, qs, d]
        k = torch.from_numpy(bf16_bits_to_f64(Kc[s][:L])).permute(1, 0, 2).repeat_interleave(g, 0)
        v = torch.from_numpy(bf16_bits_to_f64(Vc[s][:L])).permute(1, 0, 2).repeat_interleave(g, 0)
        o = torch.nn.functional.scaled_dot_product_attention(q[None], k[None], v[None],
                                                             attn_mask=mask[None, None], scale=scale)
        out.append(o[0].permute(1, 0, 2).numpy())
        start += qs
    return np.concatenate(out, axis=0)


@pytest.mark.parametrize("d,Hq,Hkv,window", [(16, 2, 2, 0), (64, 4, 4, 0), (64, 4, 2, 0),
                                             (16, 4, 1, 5), (64, 2, 2, 1)])
def test_brute_force_dense_attention(d, Hq, Hkv, window):
    rng = np.random.default_rng(d * 100 + Hq * 10 + Hkv + window)
    q_lens, ctx_lens = [9, 1, 1, 20], [0, 37, 5, 44]
    B, nblk = 16, 32
    perm = rng.permutation(nblk)
    bt = np.full((4, 4), -1, np.int32)
    o = 0
    for s in range(4):
        n = -(-(q_lens[s] + ctx_lens[s]) // B)
        bt[s, :n] = perm[o:o + n]
        o += n
    cache = PagedCache(nblk, Hkv, B, d)
    Kc = [_bits(rng, (q + c, Hkv, d)) for q, c in zip(q_lens, ctx_lens)]
    Vc = [_bits(rng, (q + c, Hkv, d)) for q, c in zip(q_lens, ctx_lens)]
    for s in range(4):
        cache.write_positions(bt[s], np.arange(ctx_lens[s]), Kc[s][:ctx_lens[s]], Vc[s][:ctx_lens[s]])
    k_new = np.concatenate([Kc[s][ctx_lens[s]:] for s in range(4)])
    v_new = np.concatenate([Vc[s][ctx_lens[s]:] for s in range(4)])
    append_kv(cache, bt, q_lens, ctx_lens, k_new, v_new)
    T = sum(q_lens)
    Q = _bits(rng, (T, Hq, d))
    scale = 1 / np.sqrt(d)
    ours = ragged_attention(cache, bt, q_lens, ctx_lens, Q, scale, window)
    ref = _sdpa_reference(q_lens, ctx_lens, Kc, Vc, Q, Hq, Hkv, window, scale)
    assert np.abs(ours - ref).max() <= 1e-12


def test_append_is_a_bit_copy_and_leaves_other_slots():
    rng = np.random.default_rng(1)
    q_lens, ctx_lens = np.array([5, 1, 17]), np.array([0, 33, 14])
    B, Hkv, d, nblk = 16, 2, 16, 40
    bt = np.array([[7, -1, -1], [3, 30, 12], [0, 21, -1]], np.int32)
    cache = PagedCache(nblk, Hkv, B, d, fill=0xABCD)
    T = int(q_lens.sum())
    k, v = _bits(rng, (T, Hkv, d)), _bits(rng, (T, Hkv, d))
    append_kv(cache, bt, q_lens, ctx_lens, k, v)
    seq, pos = token_positions(q_lens, ctx_lens)
    written = set()
    for t in range(T):
        blk, slot = bt[seq[t], pos[t] // B], pos[t] % B
        assert np.array_equal(cache.block(blk)[0, :, slot], k[t])
        assert np.array_equal(cache.block(blk)[1, :, slot], v[t])
        written.add((blk, slot))
    for blk in range(nblk):
        for slot in range(B):
            if (blk, slot) not in written:
                assert (cache.block(blk)[:, :, slot] == 0xABCD).all()


def test_uniform_keys_give_mean_of_admitted_values():
    rng = np.random.default_rng(2)
    L, d = 50, 32
    K = np.tile(rng.standard_normal((1, d)), (L, 1))
    V = rng.standard_normal((L, d))
    pos = np.array([0, 7, 49, 30])
    q = rng.standard_normal((4, d))
    for window in (0, 8):
        o = attend_contiguous(q, pos, K, V, 0.125, window)
        for i, p in enumerate(pos):
            lo = max(0, p - window + 1) if window else 0
            assert np.allclose(o[i], V[lo:p + 1].mean(axis=0), rtol=0, atol=1e-14)


def test_single_admitted_key_returns_its_value():
    rng = np.random.default_rng(3)
    K, V = rng.standard_normal((20, 16)), rng.standard_normal((20, 16))
    q = rng.standard_normal((3, 16))
    o = attend_contiguous(q[:1], [0], K, V, 1.0)                  # position 0
    assert np.array_equal(o[0], V[0])
    o = attend_contiguous(q, [4, 11, 19], K, V, 1.0, window=1)    # window of one
    assert np.array_equal(o, V[[4, 11, 19]])


def _run(w, cache=None, write_ctx=True):
    cache = cache or PagedCache(w.n_blocks, w.n_kv_heads, w.block_size, w.head_dim)
    if write_ctx:
        for s, kc, vc in w.contexts():
            cache.write_positions(w.block_tables[s], np.arange(kc.shape[0]), kc, vc)
    q, k, v = w.qkv()
    _, _, o = splitfuse_pass(cache, w.block_tables, w.q_lens, w.ctx_lens, q, k, v,
                             w.rope_theta, w.softmax_scale, w.sliding_window)
    return cache, o


def test_block_permutation_leaves_output_bit_identical():
    w = W.config1()
    _, o1 = _run(w)
    _, o2 = _run(w.with_permuted_blocks(99))
    assert not np.array_equal(w.block_tables, w.with_permuted_blocks(99).block_tables)
    assert np.array_equal(o1, o2)


def test_chunked_prefill_equals_one_shot():
    one = W.prompt_chunks(4, 2, 64, 16, 200, 200, seed=21)
    many = W.prompt_chunks(4, 2, 64, 16, 200, 48, seed=21)
    c1, o1 = _run(one[0], write_ctx=False)
    c2 = None
    outs = []
    for w in many:
        c2, o = _run(w, c2, write_ctx=False)
        outs.append(o)
    o2 = np.concatenate(outs)
    assert set(c1.blocks) == set(c2.blocks)
    for b in c1.blocks:
        assert np.array_equal(c1.blocks[b], c2.blocks[b])
    assert np.abs(o1 - o2).max() <= 1e-12


def test_window_at_least_length_equals_no_window():
    w = W.config1()
    _, o0 = _run(w)
    w2 = W.config1()
    w2.sliding_window = 64
    _, o1 = _run(w2)
    assert np.array_equal(o0, o1)


def test_gqa_equals_mha_with_replicated_kv():
    rng = np.random.default_rng(5)
    Hq, Hkv, d, B = 4, 2, 16, 16
    q_lens, ctx_lens = np.array([6, 1]), np.array([3, 20])
    bt = np.array([[0, -1], [1, 2]], np.int32)
    T = 7
    k, v = _bits(rng, (T, Hkv, d)), _bits(rng, (T, Hkv, d))
    Q = _bits(rng, (T, Hq, d))
    kc, vc = _bits(rng, (20, Hkv, d)), _bits(rng, (20, Hkv, d))
    g = PagedCache(4, Hkv, B, d)
    m = PagedCache(4, Hq, B, d)
    g.write_positions(bt[0], np.arange(3), kc[:3], vc[:3])
    g.write_positions(bt[1], np.arange(20), kc, vc)
    m.write_positions(bt[0], np.arange(3), np.repeat(kc[:3], 2, 1), np.repeat(vc[:3], 2, 1))
    m.write_positions(bt[1], np.arange(20), np.repeat(kc, 2, 1), np.repeat(vc, 2, 1))
    append_kv(g, bt, q_lens, ctx_lens, k, v)
    append_kv(m, bt, q_lens, ctx_lens, np.repeat(k, 2, 1), np.repeat(v, 2, 1))
    og = ragged_attention(g, bt, q_lens, ctx_lens, Q, 0.25)
    om = ragged_attention(m, bt, q_lens, ctx_lens, Q, 0.25)
    assert np.array_equal(og, om)


def test_sampled_rows_equal_full_rows():
    w = W.config1()
    c, o = _run(w)
    c2, _ = _run(w, write_ctx=True)
    q, _, _ = w.qkv()
    from oracle import rotate_half
    _, pos = token_positions(w.q_lens, w.ctx_lens)
    qr = rotate_half(q, pos, w.rope_theta)
    tok = np.array([0, 39, 40, 41, 63])
    s = ragged_attention(c, w.block_tables, w.q_lens, w.ctx_lens, qr, w.softmax_scale, 0, tok)
    assert np.abs(s[tok] - o[tok]).max() <= 1e-12
    assert np.isnan(s[1]).all()


def test_pass_without_rotary_appends_the_bits_and_attends_with_q_itself():
    """The no-rotary pass (learned-position families): the cache receives K and
    V bit for bit, Q is not changed, and the attention equals brute force on
    the unrotated Q and K."""
    from oracle.forward import splitfuse_pass
    from ragged_paged_kv_b200 import workloads as W
    w = W.config1()
    pc = PagedCache(w.n_blocks, w.n_kv_heads, w.block_size, w.head_dim, fill=0)
    for s, kc, vc in w.contexts():
        pc.write_positions(w.block_tables[s], np.arange(kc.shape[0]), kc, vc)
    q, k, v = w.qkv()
    q_rot, k_rot, out = splitfuse_pass(pc, w.block_tables, w.q_lens, w.ctx_lens, q, k, v, w.rope_theta,
                                       w.softmax_scale, rotary=False)
    assert np.array_equal(q_rot, q) and np.array_equal(k_rot, k)
    cu = np.concatenate([[0], np.cumsum(w.q_lens)])
    for s in range(w.n_seqs):
        L = int(w.ctx_lens[s] + w.q_lens[s])
        Kc, Vc = pc.gather(w.block_tables[s], L)
        assert np.array_equal(Kc[w.ctx_lens[s]:], k[cu[s]:cu[s + 1]])
        assert np.array_equal(Vc[w.ctx_lens[s]:], v[cu[s]:cu[s + 1]])
        # brute force: explicit causal softmax over the gathered context
        Kf, Vf = bf16_bits_to_f64(Kc), bf16_bits_to_f64(Vc)
        for j in range(int(w.q_lens[s])):
            p = int(w.ctx_lens[s]) + j
            for h in range(w.n_q_heads):
                hk = h // (w.n_q_heads // w.n_kv_heads)
                z = w.softmax_scale * (Kf[:p + 1, hk] @ bf16_bits_to_f64(q[cu[s] + j, h]))
                e = np.exp(z - z.max())
                ref = (e[:, None] * Vf[:p + 1, hk]).sum(0) / e.sum()
                assert np.allclose(out[cu[s] + j, h], ref, rtol=0, atol=1e-12)


def test_linear_against_term_by_term_sums():
    """The output-projection oracle (a linear layer, y = o W^T) on a tiny case
    against sums written out term by term (math.fsum, exact) and a
    brute-force nearest-bf16 rounding; a transposed weight or a dropped term
    changes the words."""
    import math
    from oracle import linear
    from oracle.bf16 import bf16_bits_to_f64 as widen
    rng = np.random.default_rng(6)
    T, K, N = 4, 128, 3
    x = f32_to_bf16_bits(rng.standard_normal((T, K)).astype(np.float32))
    w = f32_to_bf16_bits((rng.standard_normal((N, K)) / 8).astype(np.float32))
    y = linear(x, w)
    assert y.shape == (T, N)
    allv = np.arange(1 << 16, dtype=np.uint32).astype(np.uint16)
    fin = allv[np.isfinite(widen(allv))]
    grid = widen(fin)
    xs, ws = widen(x), widen(w)
    for t in range(T):
        for j in range(N):
            exact = math.fsum(float(xs[t, i]) * float(ws[j, i]) for i in range(K))
            dist = np.abs(grid - exact)
            best = fin[dist == dist.min()]
            want = best[0] if len(best) == 1 else best[(best & 1) == 0][0]
            assert y[t, j] == want, (t, j)


def test_linear_rounds_the_exact_sum_once():
    """A sum whose exact value lies just above a bf16 midpoint: 1 + 2^-8 +
    2^-40 must round up to 1 + 2^-7. A float32 sum first lands on the
    midpoint 1 + 2^-8, and then rounds to even, down to 1. The mirror case
    with the last term negative rounds down. Every input is a bf16 value."""
    from oracle import linear
    x = f32_to_bf16_bits(np.array([[1.0, 1.0, 1.0]], dtype=np.float32))
    for tail, want in ((2.0 ** -40, 1.0 + 2.0 ** -7), (-(2.0 ** -40), 1.0)):
        w = f32_to_bf16_bits(np.array([[1.0, 2.0 ** -8, tail]], dtype=np.float32))
        assert bf16_bits_to_f64(linear(x, w))[0, 0] == want
        assert bf16_bits_to_f64(linear(x, w ^ np.uint16(0x8000)))[0, 0] == -want


def _tail_case(head, tail_sign):
    """x = 4096 ones; w = two head terms, then 4094 copies of +-2^-61 (all
    bf16 values)."""
    x = f32_to_bf16_bits(np.ones((1, 4096), dtype=np.float32))
    w = np.full((1, 4096), tail_sign * 2.0 ** -61, dtype=np.float32)
    w[0, :2] = head
    return x, f32_to_bf16_bits(w)


def test_linear_sums_4096_terms_exactly():
    """Two 4096-term sums that lie next to a bf16 midpoint, one on each side.
    1 + 2^-8 + 4094 * 2^-61 is just above the midpoint of 1 and 1 + 2^-7 and
    must round up; 1 + 3 * 2^-8 - 4094 * 2^-61 is just below the midpoint of
    1 + 2^-7 and 1 + 2^-6 and must round down: both give 1 + 2^-7. A float64
    sum taken left to right drops every 2^-61 term (each is under half a
    float64 unit of the running sum), lands on the midpoint, and rounds to
    even: the wrong word both times."""
    from oracle import linear
    for head, sign in (((1.0, 2.0 ** -8), 1.0), ((1.0, 3 * 2.0 ** -8), -1.0)):
        x, w = _tail_case(head, sign)
        assert bf16_bits_to_f64(linear(x, w))[0, 0] == 1.0 + 2.0 ** -7
        seq = 0.0
        for a, b in zip(bf16_bits_to_f64(x)[0], bf16_bits_to_f64(w)[0]):
            seq += float(a) * float(b)
        assert bf16_bits_to_f64(f64_to_bf16_bits(np.float64(seq)))[()] != 1.0 + 2.0 ** -7


def _nearest_bf16_exact(S):
    """Brute force on exact rationals: the bf16 word nearest the Fraction S
    (finite, inside the bf16 range), ties to the even pattern. The candidates
    are the three words around float(S)'s rounding."""
    from fractions import Fraction
    b = int(f64_to_bf16_bits(np.float64(float(S)))[()])
    cands = []
    for c in (b - 1, b, b + 1):
        c &= 0xFFFF
        v = float(bf16_bits_to_f64(np.uint16(c))[()])
        if np.isfinite(v):
            cands.append((abs(Fraction(v) - S), c & 1, c))
    cands.sort()
    best = [c for c in cands if c[0] == cands[0][0]]
    return min(best, key=lambda c: c[1])[2] if len(best) > 1 else best[0][2]


def test_round_exact_sum_against_rationals():
    """round_exact_sum (the oracle's exact path) against sums of Fractions:
    N(0,1) products, sums built to sit on a bf16 midpoint exactly (a true
    tie) and within 2^-60 of one on either side, K from 2 to 4096."""
    from fractions import Fraction
    from oracle.projection import round_exact_sum
    rng = np.random.default_rng(11)
    cases = []
    for K in (2, 17, 300, 4096):
        a = bf16_bits_to_f64(f32_to_bf16_bits(rng.standard_normal(K).astype(np.float32)))
        b = bf16_bits_to_f64(f32_to_bf16_bits(rng.standard_normal(K).astype(np.float32)))
        cases.append(a * b)
    for mid in (1.0 + 2.0 ** -8, -(3.0 + 2.0 ** -6), 2.0 ** -20 * (1 + 2.0 ** -8)):
        for eps in (0.0, 2.0 ** -60, -(2.0 ** -60)):
            t = [mid * 0.5, mid * 0.25, mid * 0.25] + [eps / 1024] * 1024 + [0.0] * 7
            cases.append(np.array(t))
    for terms in cases:
        S = sum((Fraction(float(t)) for t in terms), Fraction(0))
        assert int(round_exact_sum(terms)) == _nearest_bf16_exact(S)


def test_linear_bound_path_agrees_with_exact_sums():
    """The float64 path of linear (used where its error bound proves the
    rounding) against the exact path for every output of a K = 4096 case."""
    from oracle import linear
    from oracle.projection import round_exact_sum
    rng = np.random.default_rng(12)
    x = f32_to_bf16_bits(rng.standard_normal((3, 4096)).astype(np.float32))
    w = f32_to_bf16_bits((rng.standard_normal((24, 4096)) / 64).astype(np.float32))
    y = linear(x, w)
    xs, ws = bf16_bits_to_f64(x), bf16_bits_to_f64(w)
    for t in range(3):
        for j in range(24):
            assert y[t, j] == round_exact_sum(xs[t] * ws[j]), (t, j)


def test_qkv_projection_against_term_by_term_sums():
    """The projection oracle on a tiny case against sums written out term by
    term (math.fsum, exact) and a brute-force nearest-bf16 rounding."""
    import math
    from oracle import qkv_projection
    from oracle.bf16 import bf16_bits_to_f64 as widen
    rng = np.random.default_rng(5)
    T, hidden, hq, hkv, d = 3, 64, 2, 1, 4
    x = f32_to_bf16_bits(rng.standard_normal((T, hidden)).astype(np.float32))
    w = f32_to_bf16_bits((rng.standard_normal(((hq + 2 * hkv) * d, hidden)) / 8).astype(np.float32))
    q, k, v = qkv_projection(x, w, hq, hkv, d)
    assert q.shape == (T, hq, d) and k.shape == (T, hkv, d) and v.shape == (T, hkv, d)
    allv = np.arange(1 << 16, dtype=np.uint32).astype(np.uint16)
    fin = allv[np.isfinite(widen(allv))]
    grid = widen(fin)
    xs, ws = widen(x), widen(w)
    out = np.concatenate([q.reshape(T, -1), k.reshape(T, -1), v.reshape(T, -1)], axis=1)
    for t in range(T):
        for j in range(ws.shape[0]):
            exact = math.fsum(float(xs[t, i]) * float(ws[j, i]) for i in range(hidden))
            dist = np.abs(grid - exact)
            best = fin[dist == dist.min()]
            # ties go to the even pattern
            want = best[0] if len(best) == 1 else best[(best & 1) == 0][0]
            assert out[t, j] == want, (t, j)
