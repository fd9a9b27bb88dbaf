"""C-ABI checks that need no GPU: the library loads, exports every symbol
include/fg.h declares, and rejects bad arguments before any device work;
its host rotary table equals the oracle's bit for bit."""
import ctypes
import subprocess

import numpy as np
import pytest

from ragged_paged_kv_b200 import fg

FAKE_DEV = 0x7F0000000000   # 16-byte aligned; never dereferenced by failing calls


def test_library_exports_every_declared_symbol():
    L = fg.lib()
    names = fg.header_symbols()
    assert len(names) >= 14
    for n in names:
        assert hasattr(L, n), n
    out = subprocess.run(["nm", "-D", "--defined-only", fg.LIB_PATH], capture_output=True, text=True).stdout
    exported = {line.split()[-1] for line in out.splitlines() if " T " in line}
    assert set(names) <= exported


def test_status_strings():
    L = fg.lib()
    for code, name in fg.STATUS.items():
        assert L.fg_status_string(code).decode() == name


def _fake_cache(B=16, nblk=64, hkv=2, d=64):
    return fg.KVCache.__new__(fg.KVCache), (B, nblk, hkv, d)


def _external(B=16, nblk=64, hkv=2, d=64):
    h = ctypes.c_void_p()
    st = fg.lib().fg_kv_cache_create_external(B, nblk, hkv, d, ctypes.c_void_p(FAKE_DEV),
                                              nblk * 2 * hkv * B * d * 2, ctypes.byref(h))
    assert st == 0, fg.lib().fg_last_error()
    return h


@pytest.mark.parametrize("B,d,status", [(17, 64, "FG_ERR_UNSUPPORTED"), (16, 96, "FG_ERR_UNSUPPORTED"),
                                        (256, 128, "FG_ERR_UNSUPPORTED")])
def test_unsupported_cache_shapes(B, d, status):
    h = ctypes.c_void_p()
    st = fg.lib().fg_kv_cache_create(B, 8, 2, d, ctypes.byref(h))
    assert fg.STATUS[st] == status and not h.value


def test_external_cache_too_small_is_capacity():
    h = ctypes.c_void_p()
    st = fg.lib().fg_kv_cache_create_external(16, 8, 2, 64, ctypes.c_void_p(FAKE_DEV), 100, ctypes.byref(h))
    assert fg.STATUS[st] == "FG_ERR_CAPACITY"


class _Cache:
    def __init__(self, h):
        self.handle = h


def _put(batch, cache_h, ids, ql, cl, bt):
    batch.put(_Cache(cache_h), ids, ql, cl, np.asarray(bt, np.int32), stream=0)


@pytest.mark.parametrize("case,ids,ql,cl,bt,status", [
    ("q_len 0", [0], [0], [5], [[1]], "FG_ERR_INVALID_ARG"),
    ("negative ctx", [0], [1], [-1], [[1]], "FG_ERR_INVALID_ARG"),
    ("too many tokens", [0, 1], [40, 30], [0, 0], [[1, 2, 3], [4, 5, 6]], "FG_ERR_CAPACITY"),
    ("too many blocks", [0], [1], [16 * 8], [[0, 1, 2, 3, 4, 5, 6, 7, 8]], "FG_ERR_CAPACITY"),
    ("table too narrow", [0], [20], [0], [[1]], "FG_ERR_INVALID_ARG"),
    ("block id out of range", [0], [3], [0], [[64]], "FG_ERR_OUT_OF_RANGE"),
    ("negative block id", [0], [3], [0], [[-1]], "FG_ERR_OUT_OF_RANGE"),
    ("duplicate seq ids", [7, 7], [1, 1], [0, 0], [[1], [2]], "FG_ERR_ALIAS"),
    ("block twice in a table", [0], [1], [20], [[3, 3]], "FG_ERR_ALIAS"),
    ("two writers, one block", [0, 1], [2, 2], [0, 4], [[5], [5]], "FG_ERR_ALIAS"),
    ("write into a block another reads", [0, 1], [1, 1], [20, 3], [[5, 6], [6, -1]], "FG_ERR_ALIAS"),
])
def test_put_validation_fails_before_device_work(case, ids, ql, cl, bt, status):
    h = _external()
    b = fg.RaggedBatch(max_tokens=64, max_seqs=4, max_blocks_per_seq=8)
    with pytest.raises(fg.FgError) as e:
        _put(b, h, ids, ql, cl, bt)
    assert e.value.name == status, (case, str(e.value))
    fg.lib().fg_kv_cache_destroy(h)


def test_put_capacity_of_sequences():
    h = _external()
    b = fg.RaggedBatch(max_tokens=64, max_seqs=2, max_blocks_per_seq=8)
    with pytest.raises(fg.FgError) as e:
        _put(b, h, [0, 1, 2], [1, 1, 1], [0, 0, 0], [[1], [2], [3]])
    assert e.value.name == "FG_ERR_CAPACITY"


def test_shared_read_only_prefix_is_not_an_alias(has_gpu):
    """Two sequences reading one full prefix block and writing elsewhere is legal."""
    h = _external()
    b = fg.RaggedBatch(max_tokens=64, max_seqs=4, max_blocks_per_seq=8)
    try:
        _put(b, h, [0, 1], [1, 1], [16, 16], [[3, 4], [3, 5]])
    except fg.FgError as e:
        assert not has_gpu and e.name == "FG_ERR_CUDA"   # validation passed, no device here


def test_attention_before_put_is_rejected():
    h = _external()
    b = fg.RaggedBatch(max_tokens=8, max_seqs=2, max_blocks_per_seq=2)
    st = fg.lib().fg_ragged_attention(h, b.handle, ctypes.c_void_p(FAKE_DEV), ctypes.c_void_p(FAKE_DEV),
                                      2, 0.125, 0, ctypes.c_void_p(0))
    assert fg.STATUS[st] == "FG_ERR_INVALID_ARG"


def test_host_rotary_table_equals_oracle_bitwise():
    from oracle import rope_table
    for theta, d, p0, n in ((10000.0, 128, 0, 300), (10000.0, 64, 32000, 200), (500000.0, 128, 7, 50)):
        c, s = fg.rotary_table(theta, d, p0, n)
        oc, os_ = rope_table(theta, d, np.arange(p0, p0 + n))
        assert np.array_equal(c.view(np.uint32), oc.view(np.uint32))
        assert np.array_equal(s.view(np.uint32), os_.view(np.uint32))


@pytest.mark.parametrize("k_in,n_out,status", [(4096, 4096, "FG_ERR_INVALID_ARG"),   # no put yet
                                               (100, 4096, "FG_ERR_UNSUPPORTED"),
                                               (4096, 96, "FG_ERR_UNSUPPORTED"),
                                               (0, 64, "FG_ERR_UNSUPPORTED")])
def test_output_projection_rejects_bad_arguments(k_in, n_out, status):
    b = fg.RaggedBatch(max_tokens=8, max_seqs=2, max_blocks_per_seq=2)
    d = ctypes.c_void_p(FAKE_DEV)
    st = fg.lib().fg_output_projection(b.handle, d, d, k_in, n_out, d, ctypes.c_void_p(0))
    assert fg.STATUS[st] == status
    st = fg.lib().fg_output_projection(None, d, d, 4096, 4096, d, ctypes.c_void_p(0))
    assert fg.STATUS[st] == "FG_ERR_INVALID_ARG"


def test_prepare_rotary_rejects_bad_arguments():
    h = _external()
    L = fg.lib()
    assert fg.STATUS[L.fg_kv_cache_prepare_rotary(h, 0.0, 100)] == "FG_ERR_INVALID_ARG"
    assert fg.STATUS[L.fg_kv_cache_prepare_rotary(h, 10000.0, -1)] == "FG_ERR_INVALID_ARG"
    assert fg.STATUS[L.fg_kv_cache_prepare_rotary(None, 10000.0, 100)] == "FG_ERR_INVALID_ARG"
    L.fg_kv_cache_destroy(h)


def test_one_call_pass_rejects_bad_arguments():
    """fg_rotary_kv_attention checks its handles and arguments before any
    device work: a batch not put against this cache, NULL handles, a
    non-positive rope_theta or softmax_scale, a negative window."""
    h = _external()
    b = fg.RaggedBatch(max_tokens=8, max_seqs=2, max_blocks_per_seq=2)
    L = fg.lib()
    d = ctypes.c_void_p(FAKE_DEV)
    z = ctypes.c_void_p(0)

    def call(cache, batch, theta=10000.0, scale=0.125, window=0, heads=2):
        return fg.STATUS[L.fg_rotary_kv_attention(cache, batch, d, d, d, d, d, heads, theta, scale, window, z)]

    assert call(h, b.handle) == "FG_ERR_INVALID_ARG"     # no put against this cache yet
    assert call(None, b.handle) == "FG_ERR_INVALID_ARG"
    assert call(h, None) == "FG_ERR_INVALID_ARG"
    L.fg_kv_cache_destroy(h)
