"""fg_ragged_batch_put's checks against a plain statement of its rules, on
random batches (host only).

The rules, as include/fg.h states them:
- every used block id lies in [0, n_blocks);
- no block appears twice in one sequence's table;
- no cache slot is written by two sequences;
- no new token is written into a slot that another sequence of the batch
  uses;
- sequence ids are distinct.
Each random batch carries at most one kind of violation. A batch the rules
accept must pass validation: on a machine without a GPU the put then stops
at its first device call with FG_ERR_CUDA. A batch the rules reject must
fail with that rule's status.
"""
import ctypes

import numpy as np
import pytest

from ragged_paged_kv_b200 import fg

B, N_BLOCKS, HKV, D = 16, 48, 2, 64
FAKE_DEV = 0x7F0000000000


def expected_status(ids, ql, cl, bt):
    if len(set(ids)) != len(ids):
        return "FG_ERR_ALIAS"
    uses = {}  # block -> [(seq, used, first written)]
    for s, (q, c) in enumerate(zip(ql, cl)):
        L = c + q
        nb = -(-L // B)
        row = bt[s][:nb]
        if any(b < 0 or b >= N_BLOCKS for b in row):
            return "FG_ERR_OUT_OF_RANGE"
        for i, blk in enumerate(row):
            used = min(B, L - i * B)
            w0 = min(max(c, i * B) - i * B, used)
            uses.setdefault(blk, []).append((s, used, w0))
    for lst in uses.values():
        for a in range(len(lst)):
            for b in range(a + 1, len(lst)):
                (s1, u1, w1), (s2, u2, w2) = lst[a], lst[b]
                if s1 == s2:
                    return "FG_ERR_ALIAS"
                if (w1 < u1 and w1 < u2) or (w2 < u2 and w2 < u1):
                    return "FG_ERR_ALIAS"
    return None


def random_batch(rng, kind):
    S = int(rng.integers(2, 6))
    ids = list(range(100, 100 + S))
    ql = [int(x) for x in rng.integers(1, 20, S)]
    cl = [int(x) for x in rng.integers(0, 40, S)]
    free = list(rng.permutation(N_BLOCKS))
    bt = []
    for q, c in zip(ql, cl):
        nb = -(-(q + c) // B)
        bt.append([int(free.pop()) for _ in range(nb)] + [-1] * (8 - nb))
    if kind == "dup_id":
        ids[1] = ids[0]
    elif kind == "range":
        s = int(rng.integers(0, S))
        bt[s][int(rng.integers(0, -(-(ql[s] + cl[s]) // B)))] = int(rng.choice([-3, N_BLOCKS, N_BLOCKS + 7]))
    elif kind == "share":
        # two sequences share a block: legal only when neither writes a slot the other uses
        s1, s2 = rng.choice(S, 2, replace=False)
        i1 = int(rng.integers(0, -(-(ql[s1] + cl[s1]) // B)))
        i2 = int(rng.integers(0, -(-(ql[s2] + cl[s2]) // B)))
        bt[s2][i2] = bt[s1][i1]
    elif kind == "prefix":
        # a shared read-only prefix: both sequences only read their first block
        s1, s2 = 0, 1
        cl[s1] = max(cl[s1], B + int(rng.integers(0, 10)))
        cl[s2] = max(cl[s2], B + int(rng.integers(0, 10)))
        bt[s1] = [int(free.pop()) for _ in range(-(-(ql[s1] + cl[s1]) // B))]
        bt[s2] = [int(free.pop()) for _ in range(-(-(ql[s2] + cl[s2]) // B))]
        bt[s2][0] = bt[s1][0]
        bt[s1] += [-1] * (8 - len(bt[s1]))
        bt[s2] += [-1] * (8 - len(bt[s2]))
    elif kind == "twice":
        s = int(np.argmax([-(-(q + c) // B) for q, c in zip(ql, cl)]))
        nb = -(-(ql[s] + cl[s]) // B)
        if nb >= 2:
            bt[s][1] = bt[s][0]
    return ids, ql, cl, bt


@pytest.mark.parametrize("kind", ["clean", "dup_id", "range", "share", "prefix", "twice"])
def test_put_checks_match_the_rules(kind, has_gpu):
    if has_gpu:
        pytest.skip("an accepted batch would reach the device; this test needs the no-GPU stop")
    rng = np.random.default_rng(["clean", "dup_id", "range", "share", "prefix", "twice"].index(kind))
    L = fg.lib()
    h = ctypes.c_void_p()
    assert L.fg_kv_cache_create_external(B, N_BLOCKS, HKV, D, ctypes.c_void_p(FAKE_DEV),
                                         N_BLOCKS * 2 * HKV * B * D * 2, ctypes.byref(h)) == 0
    b = fg.RaggedBatch(max_tokens=256, max_seqs=8, max_blocks_per_seq=8)

    class _C:
        handle = h
    seen = set()
    for _ in range(150):
        ids, ql, cl, bt = random_batch(rng, kind)
        want = expected_status(ids, ql, cl, bt)
        seen.add(want)
        try:
            b.put(_C(), ids, ql, cl, np.asarray(bt, np.int32), stream=0)
            got = "FG_OK"
        except fg.FgError as e:
            got = e.name
        assert got == (want or "FG_ERR_CUDA"), (ids, ql, cl, bt, want, got)
    L.fg_kv_cache_destroy(h)
    if kind == "share":
        assert None in seen and "FG_ERR_ALIAS" in seen  # both legal and illegal sharing came up
