"""Failure detection on the GPU without a fault: a bounded device wait on a
barrier that nothing completes must give up and report FG_ERR_TIMEOUT, and
the context must stay usable for a normal pass afterwards."""
import ctypes

import numpy as np
import pytest
import torch

from ragged_paged_kv_b200 import fg, fixtures
from ragged_paged_kv_b200 import workloads as W

pytestmark = pytest.mark.gpu


def test_bounded_wait_gives_up_and_reports_timeout():
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    for limit in (1 << 16, 1 << 22):
        st = fg.lib().fg_selftest_bounded_wait(limit, stream)
        assert fg.STATUS[st] == "FG_ERR_TIMEOUT", fg.lib().fg_last_error().decode()
    # the context is intact: a normal pass still runs and reports no device error
    w = W.config1()
    cache = fg.KVCache(w.block_size, w.n_blocks, w.n_kv_heads, w.head_dim)
    fixtures.fill(cache.tensor)
    fixtures.write_context(w, cache.tensor)
    batch = fg.RaggedBatch(w.n_tokens, w.n_seqs, w.block_tables.shape[1])
    batch.put(cache, w.seq_ids, w.q_lens, w.ctx_lens, w.block_tables)
    q, k, v = fixtures.qkv_device(w)
    q_rot, out = torch.empty_like(q), torch.empty_like(q)
    fg.forward(cache, batch, q, k, v, q_rot, out, w.n_q_heads, w.rope_theta, w.softmax_scale)
    torch.cuda.synchronize()
    batch.device_status()
    assert torch.isfinite(out.float()).all()


def test_invalid_limit_is_rejected_before_launch():
    st = fg.lib().fg_selftest_bounded_wait(-1, ctypes.c_void_p(0))
    assert fg.STATUS[st] == "FG_ERR_INVALID_ARG"
