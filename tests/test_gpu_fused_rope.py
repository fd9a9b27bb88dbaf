"""The one-call pass with the query rotation moved into the query-tile
kernel's load of Q (fg_rotary_kv_attention), against the two calls it stands
for (fg_rotary_kv_append, then fg_ragged_attention).

Both run the same plan and the same kernels, and the query-tile kernel
rotates its Q rows in shared memory with the same exact arithmetic and table
as the rotary kernel, so every word of the output and of the cache must be
the same. q_rot must hold the rotated rows of the tokens the decode kernels
serve (bit-identical to the two-call path's) and keep its prior contents on
the rows the query-tile kernel rotates itself; q is left as it was. Checked
on the configurations' shapes and on the shape sweep of the parity tests
(block sizes 16 to 128, d = 64 and 128, MHA, grouped and non-power-of-two
groups, windows, a group past the grouped decode kernel's)."""
import gc

import numpy as np
import pytest
import torch

from ragged_paged_kv_b200 import fg, fixtures
from ragged_paged_kv_b200 import workloads as W
from ragged_paged_kv_b200.fixtures import to_bits

pytestmark = pytest.mark.gpu

QROT_FILL = 0x7FA1  # a NaN pattern the rotation cannot produce from finite inputs


def _pass(w, fused):
    cache = fg.KVCache(w.block_size, w.n_blocks, w.n_kv_heads, w.head_dim)
    fixtures.fill(cache.tensor)
    fixtures.write_context(w, cache.tensor, keep=(), others="pool")
    batch = fg.RaggedBatch(w.n_tokens, w.n_seqs, w.block_tables.shape[1])
    batch.put(cache, w.seq_ids, w.q_lens, w.ctx_lens, w.block_tables)
    q, k, v = fixtures.qkv_device(w)
    q_before = to_bits(q)
    q_rot = torch.empty_like(q)
    q_rot.view(torch.int16).fill_(QROT_FILL)
    out = torch.empty_like(q)
    if fused:
        fg.rotary_kv_attention(cache, batch, q, k, v, q_rot, out, w.n_q_heads, w.rope_theta, w.softmax_scale,
                               w.sliding_window)
    else:
        fg.forward(cache, batch, q, k, v, q_rot, out, w.n_q_heads, w.rope_theta, w.softmax_scale,
                   w.sliding_window)
    torch.cuda.synchronize()
    batch.device_status()
    ids = np.unique(np.concatenate([w.block_tables[s, :w.blocks_used(s)] for s in range(w.n_seqs)]))
    blocks = to_bits(cache.tensor[torch.from_numpy(ids.astype(np.int64)).cuda()])
    res = {"out": to_bits(out), "q_rot": to_bits(q_rot), "blocks": blocks, "q_same": np.array_equal(to_bits(q), q_before)}
    cache.close()
    batch.close()
    del q, k, v, q_rot, out
    gc.collect()
    torch.cuda.empty_cache()
    return res


def _tc_rows(w):
    """Token rows whose sequence the query-tile kernel serves (for a group
    size it takes; none otherwise)."""
    g = w.n_q_heads // w.n_kv_heads
    if g & (g - 1):
        return np.zeros(w.n_tokens, bool)
    p = fg.describe_plan(w.q_lens, w.ctx_lens, w.n_kv_heads, g, w.head_dim, w.sliding_window, True, 148)
    seqs = {int(u[0]) for u in p["tc"]}
    rows = np.zeros(w.n_tokens, bool)
    cu = w.cu_q
    for s in seqs:
        rows[int(cu[s]):int(cu[s + 1])] = True
    return rows


def _check(w):
    a = _pass(w, fused=False)
    b = _pass(w, fused=True)
    assert np.array_equal(a["out"], b["out"]), f"{w.name}: outputs differ"
    assert np.array_equal(a["blocks"], b["blocks"]), f"{w.name}: cache blocks differ"
    assert b["q_same"], f"{w.name}: q was modified"
    tc = _tc_rows(w)
    assert np.array_equal(a["q_rot"][~tc], b["q_rot"][~tc]), f"{w.name}: q_rot of decode-served rows differs"
    assert (b["q_rot"][tc].view(np.uint16) == QROT_FILL).all(), f"{w.name}: q_rot rows of the query tiles written"
    return tc


@pytest.mark.parametrize("which", ["config1", "config2", "config4", "config5"])
def test_fused_pass_equals_two_calls(which):
    w = getattr(W, which)()
    tc = _check(w)
    assert tc.any(), f"{w.name}: no query-tile rows, the rotation-at-load path did not run"


@pytest.mark.parametrize("B,d,Hq,Hkv,window", [
    (16, 64, 4, 4, 0), (32, 128, 8, 2, 0), (64, 128, 8, 1, 0), (128, 64, 6, 3, 0),
    (16, 128, 16, 2, 37), (64, 64, 4, 4, 300), (128, 128, 32, 8, 0), (32, 64, 16, 16, 1),
    (64, 128, 12, 4, 0), (32, 64, 10, 2, 50), (64, 128, 32, 2, 0), (64, 128, 64, 2, 0)])
def test_fused_pass_shape_sweep(B, d, Hq, Hkv, window):
    rng = np.random.default_rng(B * 7 + d + Hq * 3 + Hkv + window)
    q_lens = [1, 1, 3, 130, 17, 1, 257]
    ctx_lens = [0, 700, 64, 0, 1111, 2049, 90]
    w = W._make(f"sweep_B{B}_d{d}_g{Hq // Hkv}_w{window}", Hq, Hkv, d, B, list(range(7)),
                q_lens, ctx_lens, seed=int(rng.integers(1 << 30)), budget=sum(q_lens), window=window)
    _check(w)


def test_fused_pass_rejects_bad_arguments():
    """After a valid put: q_rot equal to q, a non-positive rope_theta or
    softmax_scale, a negative window and a misaligned pointer are rejected
    before any launch, and the cache is untouched."""
    w = W.config1()
    cache = fg.KVCache(w.block_size, w.n_blocks, w.n_kv_heads, w.head_dim)
    fixtures.fill(cache.tensor)
    before = to_bits(cache.tensor)
    batch = fg.RaggedBatch(w.n_tokens, w.n_seqs, w.block_tables.shape[1])
    batch.put(cache, w.seq_ids, w.q_lens, w.ctx_lens, w.block_tables)
    q, k, v = fixtures.qkv_device(w)
    q_rot, out = torch.empty_like(q), torch.empty_like(q)
    bad = [dict(q_rot=q), dict(rope_theta=0.0), dict(softmax_scale=0.0), dict(sliding_window=-1),
           dict(out=out.view(-1)[1:])]
    for b in bad:
        args = dict(q_rot=q_rot, out=out, rope_theta=w.rope_theta, softmax_scale=w.softmax_scale, sliding_window=0)
        args.update(b)
        with pytest.raises(fg.FgError) as e:
            fg.rotary_kv_attention(cache, batch, q, k, v, args["q_rot"], args["out"], w.n_q_heads,
                                   args["rope_theta"], args["softmax_scale"], args["sliding_window"])
        assert e.value.name == "FG_ERR_INVALID_ARG", (b, e.value.name)
    torch.cuda.synchronize()
    assert np.array_equal(to_bits(cache.tensor), before)
    cache.close()
    batch.close()
