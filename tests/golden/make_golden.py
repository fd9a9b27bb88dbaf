"""Writes tests/golden/oracle_regression.json from the oracle alone.

The pages print no worked example (no tensors, no numbers to reproduce), so
these fixtures are not independent pins: they record what the oracle and the
seeded input generator produce today, so that an unintended change to either
shows up as a failing test (tests/test_golden.py). The oracle's independent
pins are the tests in tests/test_oracle_*.py. Regenerate only with a change
whose commit message names the passage, or the reading of it, that justifies
the new values:

    python tests/golden/make_golden.py
"""
import hashlib
import json
import os
import sys

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, os.path.dirname(os.path.dirname(HERE)))

from oracle import PagedCache, rope_table  # noqa: E402
from oracle.forward import splitfuse_pass  # noqa: E402
from ragged_paged_kv_b200 import workloads as W  # noqa: E402

SENTINEL = 0x7FC1  # what untouched slots hold in the oracle's cache


def sha(a) -> str:
    return hashlib.sha256(np.ascontiguousarray(a).tobytes()).hexdigest()


def tiny_pass():
    """The tiny workload (4 sequences, 4/4 heads, d = 64, B = 16): context
    written into its slots, then one full pass of rotary, append and
    attention."""
    w = W.config1()
    pc = PagedCache(w.n_blocks, w.n_kv_heads, w.block_size, w.head_dim, fill=SENTINEL)
    for s in range(w.n_seqs):
        c = int(w.ctx_lens[s])
        if c:
            k, v = w.context(s)
            pc.write_positions(w.block_tables[s], np.arange(c), k, v)
    q, k, v = w.qkv()
    q_rot, _, out = splitfuse_pass(pc, w.block_tables, w.q_lens, w.ctx_lens, q, k, v, w.rope_theta,
                                   w.softmax_scale, w.sliding_window)
    used = sorted({int(b) for s in range(w.n_seqs) for b in w.block_tables[s, :w.blocks_used(s)]})
    cache = np.stack([pc.block(b) for b in used])
    picks = [(0, 0, 0), (0, 3, 63), (39, 1, 17), (40, 2, 5), (41, 0, 40), (63, 3, 31)]
    return {
        "q_rot_sha256": sha(q_rot),
        "cache_blocks_sha256": sha(cache),
        "cache_block_ids": used,
        "out_samples": [[t, h, e, repr(float(out[t, h, e]))] for t, h, e in picks],
        "out_sum": repr(float(np.sum(out))),
    }


def headline_snapshot():
    """The headline batch (reading c8: the first SplitFuse iteration at or
    after 50 that fills the 2048-token budget exactly)."""
    w = W.config2()
    return {"note": w.note, "q_lens": [int(x) for x in w.q_lens], "ctx_lens": [int(x) for x in w.ctx_lens]}


def rope_rows():
    """cos/sin float32 bits of the rotary table at a few positions (reading c2)."""
    pos = np.array([0, 1, 2017, 32767])
    c, s = rope_table(10000.0, 128, pos)
    return {"positions": pos.tolist(), "cos_bits_sha256": sha(c.view(np.uint32)),
            "sin_bits_sha256": sha(s.view(np.uint32))}


def main():
    data = {"tiny_pass": tiny_pass(), "headline_snapshot": headline_snapshot(), "rope_rows": rope_rows()}
    with open(os.path.join(HERE, "oracle_regression.json"), "w") as f:
        json.dump(data, f, indent=1)
        f.write("\n")


if __name__ == "__main__":
    main()
