"""The attention work plan, checked on the host (no GPU).

fg_plan_describe returns the plan fg_ragged_attention would launch for a batch
of given lengths. These tests check it against a plain statement of what a
correct plan is. Every (sequence, kv head, new token) must be served by units
whose key ranges, cut at most into pieces, exactly cover the keys that token
may see: from max(0, p - W + 1), or 0 without a window, to its own position
p. Each sequence must go to the kernel its shape selects. Split pieces must
own disjoint partial rows, which their combine group lists in key order.
Each list must be ordered longest first; the query-tile list by a coarse
length (the stage count with all but its top four bits cleared) and, among
equal coarse lengths, by (kv head, first key, sequence), so that units that
read the same K/V run together.
"""
import numpy as np
import pytest

from ragged_paged_kv_b200 import fg
from ragged_paged_kv_b200 import workloads as W

SEQ, HEAD, TOK0, NTOK, KB, KE, PART, NROWS = range(8)


def expected_kernel(q, g, d, use_tc):
    if use_tc and q == 1 and d == 128 and g <= 16:
        return "dtc"
    if q == 1 and g == 1:
        return "decode"
    return "tc" if use_tc else "general"


def max_tile_tokens(kind, g):
    return {"dtc": 1, "decode": 1, "tc": 256 // g, "general": max(1, 16 // g)}[kind]


def stages(u):
    kb = int(u[KB])
    return min(4095, (int(u[KE]) - (kb - kb % 64) + 63) >> 6)


def coarse(n):
    """n with all but its four leading bits cleared."""
    b = max(0, int(n).bit_length() - 4)
    return (int(n) >> b) << b


def check_plan(q_lens, ctx_lens, hkv, g, d, window, use_tc, slots=148):
    p = fg.describe_plan(q_lens, ctx_lens, hkv, g, d, window, use_tc, slots)
    kinds = ("general", "decode", "tc", "dtc")
    # every unit of a sequence is in the list its shape selects
    owner = {}
    for kind in kinds:
        for u in p[kind]:
            owner.setdefault(int(u[SEQ]), set()).add(kind)
    for s, q in enumerate(q_lens):
        assert owner.get(s) == {expected_kernel(int(q), g, d, use_tc)}, (s, owner.get(s))
    # longest first within each persistent kernel's list
    for kind in ("decode", "dtc"):
        st = [stages(u) for u in p[kind]]
        assert all(a >= b for a, b in zip(st, st[1:])), kind
    keys = [(-coarse(stages(u)), int(u[HEAD]), int(u[KB]), int(u[SEQ])) for u in p["tc"]]
    assert keys == sorted(keys), "tc order"
    # group the pieces by (seq, head, tile)
    tiles = {}
    for kind in kinds:
        for u in p[kind]:
            assert u[NROWS] == u[NTOK] * g
            assert 1 <= u[NTOK] <= max_tile_tokens(kind, g)
            assert 0 <= u[HEAD] < hkv
            assert u[KB] < u[KE]
            tiles.setdefault((int(u[SEQ]), int(u[HEAD]), int(u[TOK0]), int(u[NTOK])), []).append(u)
    combine = {(int(c[0]), int(c[1]), int(c[2]), int(c[3])): c for c in p["combine"]}
    assert len(combine) == len(p["combine"])
    part_rows = []
    for s, (q, c) in enumerate(zip(q_lens, ctx_lens)):
        q, c = int(q), int(c)
        for h in range(hkv):
            mine = sorted(k for k in tiles if k[0] == s and k[1] == h)
            # the tiles partition the sequence's new tokens
            t = 0
            for (_, _, t0, nt) in mine:
                assert t0 == t
                t += nt
            assert t == q, (s, h)
            for key in mine:
                t0, nt = key[2], key[3]
                p0, p1 = c + t0, c + t0 + nt - 1
                kb = max(0, p0 - window + 1) if window > 0 else 0
                pieces = sorted(tiles[key], key=lambda u: int(u[KB]))
                # the pieces cut the tile's key range [kb, p1] into runs
                lo = kb
                for u in pieces:
                    assert u[KB] == lo
                    lo = int(u[KE])
                assert lo == p1 + 1, (s, h, t0)
                R = nt * g
                if len(pieces) == 1:
                    assert pieces[0][PART] == -1 and key not in combine
                else:
                    cg = combine[key]
                    assert cg[5] == len(pieces) and cg[6] == R
                    for i, u in enumerate(pieces):
                        assert u[PART] == cg[4] + i * R
                        part_rows.append((int(u[PART]), int(u[PART]) + R))
    # partial rows: disjoint, and together exactly the rows the plan reserves
    part_rows.sort()
    assert all(a[1] <= b[0] for a, b in zip(part_rows, part_rows[1:]))
    assert sum(b - a for a, b in part_rows) == p["part_rows"]
    if part_rows:
        assert part_rows[-1][1] <= p["part_rows"]
    assert p["max_combine_rows"] == max([int(c[6]) for c in p["combine"]], default=0)
    return p


@pytest.mark.parametrize("n", [1, 2, 3, 4, 5])
@pytest.mark.parametrize("use_tc", [True, False])
def test_plans_of_the_measured_batches(n, use_tc):
    w = W.CONFIGS[n]()
    g = w.n_q_heads // w.n_kv_heads
    if not use_tc and g > 16:
        pytest.skip("groups above 16 need the tensor-core path")
    check_plan(w.q_lens, w.ctx_lens, w.n_kv_heads, g, w.head_dim, w.sliding_window, use_tc)


def test_random_batches():
    rng = np.random.default_rng(12)
    for case in range(60):
        S = int(rng.integers(1, 40))
        q = np.where(rng.random(S) < 0.5, 1, rng.integers(1, 1200, S))
        c = rng.integers(0, 20000, S)
        d = int(rng.choice([64, 128]))
        g = int(rng.choice([1, 2, 3, 4, 8, 16]))
        hkv = int(rng.integers(1, 9))
        window = int(rng.choice([0, 0, 1, 17, 700, 4096]))
        use_tc = bool(rng.random() < 0.7) and (g & (g - 1)) == 0
        slots = int(rng.choice([1, 8, 148]))
        check_plan(q, c, hkv, g, d, window, use_tc, slots)


def test_one_long_prompt_is_split_for_the_persistent_grid():
    """128 new tokens at context 30720 with 8 kv heads of 8 q heads each are
    4 tiles of 32 tokens per kv head: 32 long query tiles for 148 CTAs. The
    planner cuts each into pieces of at least 4096 keys (here 8), merged by
    the combine kernel."""
    p = check_plan([128], [30720], 8, 8, 128, 0, True)
    assert len(p["combine"]) == 32 and np.all(p["combine"][:, 5] == 8)
    for cg in p["combine"]:
        pieces = [u for u in p["tc"] if (u[HEAD], u[TOK0]) == (cg[1], cg[2])]
        pieces.sort(key=lambda u: int(u[KB]))
        assert len(pieces) == 8
        assert all(u[KE] - u[KB] >= 4096 for u in pieces[:-1])


def test_only_the_longest_tiles_are_split_to_the_balance_target():
    """The long-prompt batch (2048 new tokens at context 30720, 64/8 heads):
    64 token tiles x 8 kv heads = 512 dense tiles for 148 CTA slots, whose
    target is 4 units per slot (592). The planner cuts only the 10 longest
    token tiles (the chunk's last, with the most keys) in two, for 592 units,
    instead of every tile."""
    w = W.config5()
    p = check_plan(w.q_lens, w.ctx_lens, 8, 8, 128, 0, True)
    tc = p["tc"]
    assert len(tc) == 592
    pieces = {}
    for u in tc:
        if int(u[SEQ]) == 0:
            pieces.setdefault((int(u[HEAD]), int(u[TOK0])), []).append(u)
    split = sorted({t0 for (h, t0), us in pieces.items() if len(us) > 1})
    assert split == [2016 - 32 * i for i in range(10)][::-1]
    assert all(len(us) == 2 for (h, t0), us in pieces.items() if t0 in split)
    assert len(pieces) == 64 * 8


def test_bad_arguments_are_rejected():
    with pytest.raises(fg.FgError):
        fg.describe_plan([0], [5], 1, 1, 128)
    with pytest.raises(fg.FgError):
        fg.describe_plan([1], [-1], 1, 1, 128)
    with pytest.raises(fg.FgError):
        fg.describe_plan([1], [5], 1, 1, 96)
