"""fg_ragged_attention_noalloc: the attention pass for callers that cannot
allocate device memory (a server that reserved all of HBM for its KV pool, an
allocation policy that forbids cudaMalloc inside a step). It runs on the
library's fixed device arrays instead of a per-batch workspace.

The checks call it through the C ABI twice in a row on the same inputs and
require each result to equal fg_ragged_attention's bit for bit: both entry
points run one launch sequence with the same work plan and kernels, and only
the addresses of the workspace and plan differ, so a wrong offset into the
fixed arrays or a stale value left there by the previous call shows up as a
differing word. (The parity tolerance used everywhere else, max-abs 2e-2 and
relative L2 5e-3 against fg_ragged_attention, is reported in the failure
message.) They also check that a pass too big for the fixed arrays is
refused before any launch. The file is named
to be collected last; it also passes on its own in a fresh process."""
import ctypes

import numpy as np
import pytest
import torch

from ragged_paged_kv_b200 import fg, fixtures
from ragged_paged_kv_b200 import workloads as W
from ragged_paged_kv_b200.fixtures import to_bits

pytestmark = pytest.mark.gpu

MAX_ABS, REL_L2 = 2e-2, 5e-3


def _bf16(bits):
    return (bits.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def _same_bits(a, b):
    """Bit identity, with the parity-tolerance figures in the message."""
    if np.array_equal(a, b):
        return
    x, y = _bf16(a), _bf16(b)
    rel = np.linalg.norm(x - y) / max(np.linalg.norm(y), 1e-30)
    raise AssertionError(f"{int((a != b).sum())} of {a.size} words differ; max-abs "
                         f"{np.nanmax(np.abs(x - y)):.3e} (tolerance {MAX_ABS}), rel-L2 {rel:.3e} "
                         f"(tolerance {REL_L2})")


def _noalloc(cache, batch, q_rot, out, w):
    st = fg.lib().fg_ragged_attention_noalloc(
        cache.handle, batch.handle, ctypes.c_void_p(q_rot.data_ptr()), ctypes.c_void_p(out.data_ptr()),
        w.n_q_heads, ctypes.c_float(w.softmax_scale), w.sliding_window,
        ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert st == 0, fg.lib().fg_last_error().decode()


@pytest.mark.parametrize("make", [
    W.config2,
    lambda: W._make("gqa_window_splits", 32, 8, 128, 64, list(range(6)), [300, 1, 1, 1, 64, 1],
                    [900, 9000, 2500, 6000, 0, 130], seed=9, budget=368, window=4096),
], ids=["llama7b_splitfuse", "gqa_window_splits"])
def test_noalloc_matches_fg_ragged_attention_twice(make):
    w = make()
    cache = fg.KVCache(w.block_size, w.n_blocks, w.n_kv_heads, w.head_dim)
    fixtures.fill(cache.tensor)
    fixtures.write_context(w, cache.tensor)
    batch = fg.RaggedBatch(w.n_tokens, w.n_seqs, w.block_tables.shape[1])
    batch.put(cache, w.seq_ids, w.q_lens, w.ctx_lens, w.block_tables)
    q, k, v = fixtures.qkv_device(w)
    q_rot = torch.empty_like(q)
    fg.rotary_kv_append(cache, batch, q, k, v, q_rot, w.n_q_heads, w.rope_theta)
    ref = torch.empty_like(q)
    fg.ragged_attention(cache, batch, q_rot, ref, w.n_q_heads, w.softmax_scale, w.sliding_window)
    outs = []
    for _ in range(2):
        o = torch.full_like(q, float("nan"))
        _noalloc(cache, batch, q_rot, o, w)
        torch.cuda.synchronize()
        outs.append(to_bits(o))
    batch.device_status()
    r = to_bits(ref)
    assert np.isfinite(_bf16(r)).all()
    for o in outs:
        _same_bits(o, r)
    cache.close()
    batch.close()


def test_noalloc_refuses_a_pass_larger_than_its_arrays():
    # 32 one-token decodes over 32767 cached tokens, 64 heads of 64 dims: the
    # split partials need 32 * 64 * 64 rows * 66 floats, more than 8 Mi floats.
    # The sequences share their read-only prefix blocks; each writes only its
    # own last block, so the batch itself is valid.
    B, Hq, d, S = 128, 64, 64, 32
    shared = np.arange(255, dtype=np.int32)
    bt = np.stack([np.concatenate([shared, [255 + s]]) for s in range(S)]).astype(np.int32)
    cache = fg.KVCache(B, 255 + S, Hq, d)
    batch = fg.RaggedBatch(S, S, 256)
    batch.put(cache, np.arange(S), np.ones(S, np.int32), np.full(S, 32767, np.int32), bt)
    q = torch.zeros((S, Hq, d), dtype=torch.bfloat16, device="cuda")
    out = torch.zeros_like(q)
    st = fg.lib().fg_ragged_attention_noalloc(cache.handle, batch.handle, ctypes.c_void_p(q.data_ptr()),
                                              ctypes.c_void_p(out.data_ptr()), Hq, ctypes.c_float(0.125),
                                              0, ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert fg.STATUS[st] == "FG_ERR_CAPACITY", fg.lib().fg_last_error().decode()
    torch.cuda.synchronize()
    assert (to_bits(out) == 0).all()
    cache.close()
    batch.close()
