"""Input-generator checks: determinism, the fixed-budget invariant, token
conservation of the SplitFuse batch composer under both chunking policies,
the equal-split policy's even passes, and position-keyed generation (so a
chunked prompt sees the same numbers as the one-shot prompt)."""
import numpy as np
import pytest

from ragged_paged_kv_b200 import workloads as W


@pytest.mark.parametrize("n", [1, 2, 3, 4, 5])
def test_budget_is_filled_exactly(n):
    w = W.CONFIGS[n]()
    assert w.n_tokens == w.budget
    assert (w.q_lens >= 1).all() and (w.ctx_lens >= 0).all()
    for s in range(w.n_seqs):
        nb = w.blocks_used(s)
        assert (w.block_tables[s, :nb] >= 0).all()
        assert (w.block_tables[s, :nb] < w.n_blocks).all()
    used = np.concatenate([w.block_tables[s, :w.blocks_used(s)] for s in range(w.n_seqs)])
    assert len(np.unique(used)) == len(used)


def test_config_shapes():
    assert (W.config1().n_seqs, W.config3().n_seqs, W.config4().n_seqs, W.config5().n_seqs) == (4, 256, 516, 65)
    w4 = W.config4()
    assert (w4.n_q_heads, w4.n_kv_heads, w4.sliding_window) == (32, 8, 4096)
    assert w4.q_lens[0] == 2048 and w4.ctx_lens[0] == 14336
    w5 = W.config5()
    assert (w5.n_q_heads, w5.n_kv_heads) == (64, 8) and w5.ctx_lens[0] == 30720


def test_generation_is_deterministic():
    a, b = W.config2(), W.config2()
    assert np.array_equal(a.q_lens, b.q_lens) and np.array_equal(a.block_tables, b.block_tables)
    a1, b1 = W.config1().qkv(), W.config1().qkv()
    for x, y in zip(a1, b1):
        assert np.array_equal(x, y)


@pytest.mark.parametrize("policy", W.POLICIES)
def test_splitfuse_composer_conserves_tokens(policy):
    seen = {}
    for it, batch in W.splitfuse_schedule(seed=7, budget=512, n_active=8, n_total=40,
                                          prompt_mean=900.0, out_mean=12.0, policy=policy):
        assert sum(b[1] for b in batch) <= 512
        for rid, q, c in batch:
            seen.setdefault(rid, {}).setdefault("events", []).append((it, q, c))
    # replay: prompt chunks start where the previous stopped, decodes follow
    lens_rng = np.random.default_rng(np.random.SeedSequence(7, spawn_key=(W._KIND_LENS,)))
    P = np.maximum(1, np.rint(lens_rng.normal(900.0, 270.0, 40))).astype(int)
    G = np.maximum(1, np.rint(lens_rng.normal(12.0, 3.6, 40))).astype(int)
    assert len(seen) == 40
    for rid, st in seen.items():
        done = 0
        ev = st["events"]
        i = 0
        while done < P[rid]:
            it, q, c = ev[i]
            assert c == done
            done += q
            i += 1
        assert done == P[rid]
        decodes = ev[i:]
        assert len(decodes) == G[rid] - 1
        for k, (it, q, c) in enumerate(decodes):
            assert q == 1 and c == P[rid] + k


def test_snapshot_is_full_and_late_enough():
    it, batch = W.splitfuse_snapshot(2, 2048, 50)
    assert it >= 50 and sum(b[1] for b in batch) == 2048
    # and it is the first such iteration (reading c8)
    for it2, batch2 in W.splitfuse_schedule(seed=2, budget=2048):
        if it2 >= it:
            break
        assert it2 < 50 or sum(b[1] for b in batch2) < 2048


def test_positions_not_chunking_define_token_data():
    one = W.prompt_chunks(8, 2, 64, 16, 300, 300, seed=3)[0]
    many = W.prompt_chunks(8, 2, 64, 16, 300, 70, seed=3)
    q1, k1, v1 = one.qkv()
    parts = [w.qkv() for w in many]
    for i, x in enumerate((q1, k1, v1)):
        assert np.array_equal(x, np.concatenate([p[i] for p in parts]))


def test_context_slices_are_consistent():
    w = W.config1()
    k, v = w.context(1)
    k2, v2 = w.context(1, 10, 30)
    assert np.array_equal(k[10:30], k2) and np.array_equal(v[10:30], v2)


def _passes(policy, prompts, budget, outputs=None):
    n = len(prompts)
    return [sum(b[1] for b in batch) for _, batch in
            W.splitfuse_schedule(seed=0, budget=budget, n_active=n, n_total=n, policy=policy,
                                 prompts=prompts, outputs=outputs or [1] * n)]


def test_equal_split_spreads_one_long_prompt_evenly():
    # 5000 prompt tokens at budget 2048 need three passes: greedy fills two
    # and leaves 904 for the third; the even split gives 1667 + 1667 + 1666
    assert _passes("greedy", [5000], 2048) == [2048, 2048, 904]
    assert _passes("equal_split", [5000], 2048) == [1667, 1667, 1666]
    # a prompt that fits is taken whole by both
    assert _passes("equal_split", [700], 2048) == _passes("greedy", [700], 2048) == [700]


def test_equal_split_divides_a_pool_of_prompts_evenly():
    # pool 3000 + 1500 = 4500 tokens over three passes of 1500 (arrival order
    # within each pass); greedy gives 2048, 2048, 404
    assert _passes("equal_split", [3000, 1500], 2048) == [1500, 1500, 1500]
    assert _passes("greedy", [3000, 1500], 2048) == [2048, 2048, 404]


def test_equal_split_passes_differ_by_at_most_one_token():
    # all requests active from the start, one output token each (no decodes):
    # the pool only shrinks, and the passes are the even split of the pool
    # over the fewest passes that hold it
    rng = np.random.default_rng(5)
    for _ in range(200):
        n = int(rng.integers(1, 6))
        prompts = rng.integers(1, 6000, n).tolist()
        budget = int(rng.integers(16, 4096))
        p = _passes("equal_split", prompts, budget)
        total = sum(prompts)
        assert sum(p) == total and max(p) <= budget
        assert len(p) == -(-total // budget)
        assert max(p) - min(p) <= 1, (prompts, budget, p)


def test_equal_split_is_deterministic_and_never_exceeds_the_budget():
    a = list(W.splitfuse_schedule(seed=3, budget=2048, policy="equal_split"))
    b = list(W.splitfuse_schedule(seed=3, budget=2048, policy="equal_split"))
    assert a == b
    assert all(sum(x[1] for x in batch) <= 2048 for _, batch in a)
    with pytest.raises(ValueError):
        next(W.splitfuse_schedule(seed=3, policy="largest_first"))
