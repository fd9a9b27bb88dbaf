"""bench.py's host-side pieces, on the CPU: the algorithmic work the roofline
divides by (against a brute-force count), the workload config both arms
print, the serving simulation's block free list, and the token-sweep
batches."""
import contextlib
import io
import json
import os
import sys
import types

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import bench  # noqa: E402
from ragged_paged_kv_b200 import workloads as W  # noqa: E402


@pytest.mark.parametrize("window", [0, 4, 100])
def test_algorithmic_work_against_a_brute_force_count(window):
    w = W._make("work", 8, 2, 64, 16, [0, 1, 2, 3], [5, 1, 3, 1], [0, 10, 20, 0], seed=1, budget=10,
                window=window)
    Hq, Hkv, d = w.n_q_heads, w.n_kv_heads, w.head_dim
    pairs = kv_rows = 0
    for q, c in zip(w.q_lens, w.ctx_lens):
        seen = set()
        for j in range(int(q)):
            p = int(c) + j
            for k in range(p + 1):
                if window == 0 or p - k < window:
                    pairs += 1
                    seen.add(k)
        kv_rows += max(seen) - min(seen) + 1  # the tile's key range: first token's lo .. last token
    T = w.n_tokens
    got = bench.algorithmic_work(w)
    assert got["pairs"] == pairs
    assert got["flops"] == 4 * d * Hq * pairs
    assert got["attn_bytes"] == kv_rows * Hkv * d * 4 + T * Hq * d * 4
    assert got["append_bytes"] == T * Hkv * d * 8 + T * Hq * d * 4
    assert got["decode_flops"] + got["tc_flops"] == got["flops"]


def test_both_arms_print_the_same_workload_config():
    w = W.config1()
    args = types.SimpleNamespace(steps=1, warmup=3, gpus=1)
    buf = io.StringIO()
    with contextlib.redirect_stdout(buf):
        assert bench.run_reference(args, w, 0, 1) == 0
    line = json.loads(buf.getvalue().strip().splitlines()[-1])
    assert line["impl"] == "reference" and line["config"] == bench.workload_config(w, 1)
    assert line["metric"] == bench.METRIC and line["unit"] == "tokens/s" and line["higher_is_better"]


def test_block_free_list_gives_out_distinct_blocks_and_takes_them_back():
    a = bench.BlockAllocator(10, 16, seed=3)
    x = a.ensure(0, 40)           # 3 blocks
    y = a.ensure(1, 16)           # 1 block
    assert len(x) == 3 and len(y) == 1 and not set(x) & set(y)
    assert a.ensure(0, 48) == x   # still 3 blocks
    assert len(a.ensure(0, 49)) == 4
    a.release(0)
    assert len(a.free) == 9
    with pytest.raises(RuntimeError):
        a.ensure(2, 16 * 10)


@pytest.mark.parametrize("n", [64, 2048, 8192])
def test_sweep_batches_fill_their_token_count(n):
    w = bench.sweep_workload(n)
    assert w.n_tokens == n == w.budget
    assert int((w.q_lens == 1).sum()) >= 32
    assert (w.n_q_heads, w.n_kv_heads, w.head_dim, w.block_size) == (32, 32, 128, 64)
