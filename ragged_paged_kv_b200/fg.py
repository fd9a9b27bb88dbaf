"""Python binding of libfg (ctypes). Argument marshalling only: every step of
the path runs in the library's CUDA kernels; PyTorch supplies device memory
and streams. If libfg.so is missing this module raises at import of the
library (there is no fallback of any kind)."""
from __future__ import annotations

import ctypes
import os
import re

import numpy as np

_PKG = os.path.dirname(os.path.abspath(__file__))
# RAGGED_PAGED_KV_LIB=<name> loads libfg_<name>.so from the package instead
# of libfg.so: "trace" is the instrumented build (the same kernels plus cycle
# accounting in the query-tile kernel, python -m ragged_paged_kv_b200.build
# --trace)
_VARIANT = os.environ.get("RAGGED_PAGED_KV_LIB", "")
LIB_PATH = os.path.join(_PKG, f"libfg_{_VARIANT}.so" if _VARIANT else "libfg.so")
HEADER_PATH = os.path.join(os.path.dirname(_PKG), "include", "fg.h")

STATUS = {0: "FG_OK", 1: "FG_ERR_INVALID_ARG", 2: "FG_ERR_OUT_OF_RANGE", 3: "FG_ERR_ALIAS",
          4: "FG_ERR_CAPACITY", 5: "FG_ERR_UNSUPPORTED", 6: "FG_ERR_CUDA",
          7: "FG_ERR_DEVICE_CHECK", 8: "FG_ERR_TIMEOUT"}
_c_int32_p = ctypes.POINTER(ctypes.c_int32)
_c_float_p = ctypes.POINTER(ctypes.c_float)

_lib = None


class FgError(RuntimeError):
    def __init__(self, status: int, where: str, detail: str):
        self.status = status
        self.name = STATUS.get(status, str(status))
        super().__init__(f"{where}: {self.name}: {detail}")


def lib() -> ctypes.CDLL:
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise RuntimeError(f"{LIB_PATH} is not built; run `python -m ragged_paged_kv_b200.build`")
    L = ctypes.CDLL(LIB_PATH)
    V, P, I32, I64, F, D, SZ = (ctypes.c_void_p, ctypes.POINTER(ctypes.c_void_p), ctypes.c_int32,
                                ctypes.c_int64, ctypes.c_float, ctypes.c_double, ctypes.c_size_t)
    sig = {
        "fg_kv_cache_create": [I32, I32, I32, I32, P],
        "fg_kv_cache_create_external": [I32, I32, I32, I32, V, SZ, P],
        "fg_kv_cache_layout": [V, P, ctypes.POINTER(I64)],
        "fg_kv_cache_destroy": [V],
        "fg_ragged_batch_create": [I32, I32, I32, P],
        "fg_ragged_batch_put": [V, V, I32, _c_int32_p, _c_int32_p, _c_int32_p, _c_int32_p, I32, V],
        "fg_ragged_batch_shape": [V, _c_int32_p, _c_int32_p],
        "fg_ragged_batch_destroy": [V],
        "fg_rotary_kv_append": [V, V, V, V, V, V, I32, D, V],
        "fg_kv_append": [V, V, V, V, V],
        "fg_qkv_rotary_kv_append": [V, V, V, V, I32, V, I32, D, V],
        "fg_output_projection": [V, V, V, I32, I32, V, V],
        "fg_kv_cache_prepare_rotary": [V, D, I32],
        "fg_ragged_attention": [V, V, V, V, I32, F, I32, V],
        "fg_rotary_kv_attention": [V, V, V, V, V, V, V, I32, D, F, I32, V],
        "fg_ragged_attention_noalloc": [V, V, V, V, I32, F, I32, V],
        "fg_device_status": [V, V],
        "fg_attention_plan_info": [V, _c_int32_p],
        "fg_ragged_batch_set_timing": [V, I32],
        "fg_ragged_batch_set_overlap": [V, I32],
        "fg_host_profile_us": [V, ctypes.POINTER(ctypes.c_double), I32],
        "fg_selftest_bounded_wait": [I64, V],
        "fg_attention_kernel_ms": [V, _c_float_p],
        "fg_rotary_table": [D, I32, I32, I32, _c_float_p, _c_float_p],
        "fg_plan_describe": [_c_int32_p, _c_int32_p, I32, I32, I32, I32, I32, I32, I32, V, SZ,
                             ctypes.POINTER(I64)],
    }
    for name, args in sig.items():
        fn = getattr(L, name)
        fn.argtypes = args
        fn.restype = ctypes.c_int
    L.fg_status_string.argtypes = [ctypes.c_int]
    L.fg_status_string.restype = ctypes.c_char_p
    L.fg_last_error.argtypes = []
    L.fg_last_error.restype = ctypes.c_char_p
    if hasattr(L, "fg_phase_trace_read"):  # the trace build only
        L.fg_phase_trace_read.argtypes = [ctypes.POINTER(ctypes.c_ulonglong), ctypes.c_int, ctypes.c_int]
        L.fg_phase_trace_read.restype = ctypes.c_int
    _lib = L
    return L


def _check(st: int, where: str):
    if st != 0:
        raise FgError(st, where, lib().fg_last_error().decode())


def header_symbols() -> list[str]:
    """Function names declared in include/fg.h."""
    txt = open(HEADER_PATH).read()
    txt = re.sub(r"/\*.*?\*/", "", txt, flags=re.S)
    return sorted(set(re.findall(r"\b(fg_[a-z0-9_]+)\s*\(", txt)))


def _stream_ptr(stream) -> ctypes.c_void_p:
    if stream is None:
        import torch
        stream = torch.cuda.current_stream()
    if hasattr(stream, "cuda_stream"):
        stream = stream.cuda_stream
    return ctypes.c_void_p(int(stream))


def _dev_ptr(t, name: str) -> ctypes.c_void_p:
    import torch
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch tensor")
    if not t.is_cuda:
        raise ValueError(f"{name} must live on a CUDA device")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if t.element_size() != 2:
        raise ValueError(f"{name} must hold 16-bit (bf16) elements")
    return ctypes.c_void_p(t.data_ptr())


def _i32(a, name: str) -> np.ndarray:
    a = np.ascontiguousarray(np.asarray(a, dtype=np.int32))
    return a


def _i32p(a: np.ndarray):
    return a.ctypes.data_as(_c_int32_p)


# ----------------------------------------------------------------------------
class KVCache:
    """Blocked KV cache [n_blocks][2][n_kv_heads][block_size][head_dim] bf16.

    By default the pool is a torch tensor (``self.tensor``, viewed as that 5-d
    shape) registered through fg_kv_cache_create_external, so tests and tools
    can read and write it; ``owned=True`` lets the library cudaMalloc it."""

    def __init__(self, block_size: int, n_blocks: int, n_kv_heads: int, head_dim: int, *,
                 tensor=None, owned: bool = False, device=None):
        import torch
        self.block_size, self.n_blocks = int(block_size), int(n_blocks)
        self.n_kv_heads, self.head_dim = int(n_kv_heads), int(head_dim)
        self._h = ctypes.c_void_p()
        self.tensor = None
        if owned:
            _check(lib().fg_kv_cache_create(self.block_size, self.n_blocks, self.n_kv_heads,
                                            self.head_dim, ctypes.byref(self._h)),
                   "fg_kv_cache_create")
            return
        shape = (self.n_blocks, 2, self.n_kv_heads, self.block_size, self.head_dim)
        if tensor is None:
            tensor = torch.empty(shape, dtype=torch.bfloat16, device=device or "cuda")
        if tuple(tensor.shape) != shape:
            raise ValueError(f"cache tensor shape {tuple(tensor.shape)} != {shape}")
        self.tensor = tensor
        _check(lib().fg_kv_cache_create_external(self.block_size, self.n_blocks, self.n_kv_heads,
                                                 self.head_dim, _dev_ptr(tensor, "cache"),
                                                 tensor.numel() * 2, ctypes.byref(self._h)),
               "fg_kv_cache_create_external")

    @property
    def handle(self):
        return self._h

    def layout(self):
        base = ctypes.c_void_p()
        strides = (ctypes.c_int64 * 5)()
        _check(lib().fg_kv_cache_layout(self._h, ctypes.byref(base), strides), "fg_kv_cache_layout")
        return base.value, list(strides)

    def prepare_rotary(self, rope_theta: float, max_position: int):
        """Build the rotary table for positions 0 .. max_position up front
        (see fg_kv_cache_prepare_rotary)."""
        _check(lib().fg_kv_cache_prepare_rotary(self._h, float(rope_theta), int(max_position)),
               "fg_kv_cache_prepare_rotary")

    def close(self):
        if self._h:
            lib().fg_kv_cache_destroy(self._h)
            self._h = ctypes.c_void_p()

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


class RaggedBatch:
    """Holder of one pass's batch metadata (fg_ragged_batch)."""

    def __init__(self, max_tokens: int, max_seqs: int, max_blocks_per_seq: int):
        self._h = ctypes.c_void_p()
        self.max_tokens, self.max_seqs, self.max_blocks_per_seq = max_tokens, max_seqs, max_blocks_per_seq
        _check(lib().fg_ragged_batch_create(int(max_tokens), int(max_seqs), int(max_blocks_per_seq),
                                            ctypes.byref(self._h)), "fg_ragged_batch_create")

    @property
    def handle(self):
        return self._h

    def put(self, cache: KVCache, seq_ids, q_lens, ctx_lens, block_tables, stream=None):
        ids, ql, cl = _i32(seq_ids, "seq_ids"), _i32(q_lens, "q_lens"), _i32(ctx_lens, "ctx_lens")
        bt = _i32(block_tables, "block_tables")
        if bt.ndim != 2:
            raise ValueError("block_tables must be 2-d [n_seqs, stride]")
        n = len(ql)
        if not (len(ids) == len(cl) == n == bt.shape[0]):
            raise ValueError("seq_ids, q_lens, ctx_lens and block_tables rows must agree")
        st = _stream_ptr(stream) if n else ctypes.c_void_p(0)
        _check(lib().fg_ragged_batch_put(self._h, cache.handle, n, _i32p(ids), _i32p(ql), _i32p(cl),
                                         _i32p(bt), int(bt.shape[1]) if n else 1, st),
               "fg_ragged_batch_put")

    def shape(self):
        t, s = ctypes.c_int32(), ctypes.c_int32()
        _check(lib().fg_ragged_batch_shape(self._h, ctypes.byref(t), ctypes.byref(s)), "fg_ragged_batch_shape")
        return t.value, s.value

    def plan_info(self) -> dict:
        a = (ctypes.c_int32 * 8)()
        _check(lib().fg_attention_plan_info(self._h, ctypes.cast(a, _c_int32_p)), "fg_attention_plan_info")
        keys = ("general_units", "decode_units", "tensor_units", "combine_groups", "partial_rows",
                "launches")
        return dict(zip(keys, list(a)[:6]))

    def host_profile_us(self, reset: bool = False) -> dict:
        a = (ctypes.c_double * 8)()
        _check(lib().fg_host_profile_us(self._h, a, 1 if reset else 0), "fg_host_profile_us")
        keys = ("put", "put_validate", "put_stage_wait", "attention", "plan", "plan_stage_wait",
                "tensor_maps", "launches")
        return dict(zip(keys, list(a)))

    def set_overlap(self, enable: bool = True):
        _check(lib().fg_ragged_batch_set_overlap(self._h, 1 if enable else 0), "fg_ragged_batch_set_overlap")

    def set_timing(self, enable: bool = True):
        _check(lib().fg_ragged_batch_set_timing(self._h, 1 if enable else 0), "fg_ragged_batch_set_timing")

    def kernel_ms(self) -> dict:
        """Durations (ms) of the last attention call's kernels (timing must be on)."""
        a = (ctypes.c_float * 4)()
        _check(lib().fg_attention_kernel_ms(self._h, ctypes.cast(a, _c_float_p)), "fg_attention_kernel_ms")
        return dict(zip(("decode", "tc", "general", "combine"), list(a)))

    def device_status(self, stream=None):
        _check(lib().fg_device_status(self._h, _stream_ptr(stream)), "fg_device_status")

    def close(self):
        if self._h:
            lib().fg_ragged_batch_destroy(self._h)
            self._h = ctypes.c_void_p()

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


def rotary_kv_append(cache: KVCache, batch: RaggedBatch, q, k, v, q_rot, n_q_heads: int,
                     rope_theta: float, stream=None):
    _check(lib().fg_rotary_kv_append(cache.handle, batch.handle, _dev_ptr(q, "q"), _dev_ptr(k, "k"),
                                     _dev_ptr(v, "v"), _dev_ptr(q_rot, "q_rot"), int(n_q_heads),
                                     float(rope_theta), _stream_ptr(stream)),
           "fg_rotary_kv_append")


def qkv_rotary_kv_append(cache: KVCache, batch: RaggedBatch, x, w_qkv, q_rot, n_q_heads: int,
                         rope_theta: float, stream=None):
    """The Q/K/V projection x w_qkv^T fused with rotary + append (see
    fg_qkv_rotary_kv_append): x [T, hidden], w_qkv [(Hq + 2 Hkv) d, hidden]."""
    if x.dim() != 2 or w_qkv.dim() != 2 or x.shape[1] != w_qkv.shape[1]:
        raise ValueError("x must be [T, hidden] and w_qkv [(Hq + 2 Hkv) d, hidden]")
    _check(lib().fg_qkv_rotary_kv_append(cache.handle, batch.handle, _dev_ptr(x, "x"), _dev_ptr(w_qkv, "w_qkv"),
                                         int(x.shape[1]), _dev_ptr(q_rot, "q_rot"), int(n_q_heads),
                                         float(rope_theta), _stream_ptr(stream)),
           "fg_qkv_rotary_kv_append")


def output_projection(batch: RaggedBatch, attn_out, w_o, y, stream=None):
    """The layer's output projection y = attn_out w_o^T (see
    fg_output_projection): attn_out [T, in] (or [T, Hq, d]), w_o [out, in],
    y [T, out], all bf16 on the device."""
    x = attn_out.reshape(attn_out.shape[0], -1) if attn_out.dim() == 3 else attn_out
    if x.dim() != 2 or w_o.dim() != 2 or x.shape[1] != w_o.shape[1] or tuple(y.shape) != (x.shape[0], w_o.shape[0]):
        raise ValueError("attn_out must be [T, in], w_o [out, in] and y [T, out]")
    _check(lib().fg_output_projection(batch.handle, _dev_ptr(x, "attn_out"), _dev_ptr(w_o, "w_o"),
                                      int(w_o.shape[1]), int(w_o.shape[0]), _dev_ptr(y, "y"),
                                      _stream_ptr(stream)), "fg_output_projection")


def kv_append(cache: KVCache, batch: RaggedBatch, k, v, stream=None):
    """Append without rotary (learned-position families such as OPT): K and V
    go into the cache unchanged; pass q itself as q_rot to the attention."""
    _check(lib().fg_kv_append(cache.handle, batch.handle, _dev_ptr(k, "k"), _dev_ptr(v, "v"),
                              _stream_ptr(stream)), "fg_kv_append")


def ragged_attention(cache: KVCache, batch: RaggedBatch, q_rot, out, n_q_heads: int,
                     softmax_scale: float, sliding_window: int = 0, stream=None):
    _check(lib().fg_ragged_attention(cache.handle, batch.handle, _dev_ptr(q_rot, "q_rot"),
                                     _dev_ptr(out, "out"), int(n_q_heads), float(softmax_scale),
                                     int(sliding_window), _stream_ptr(stream)),
           "fg_ragged_attention")


def rotary_kv_attention(cache: KVCache, batch: RaggedBatch, q, k, v, q_rot, out, n_q_heads: int,
                        rope_theta: float, softmax_scale: float, sliding_window: int = 0, stream=None):
    """fg_rotary_kv_attention: rotary + append + attention in one call, the
    query-tile kernel rotating its Q rows as it loads them (q_rot receives
    only the decode tokens' rows; out and the cache equal the two-call path's)."""
    _check(lib().fg_rotary_kv_attention(cache.handle, batch.handle, _dev_ptr(q, "q"), _dev_ptr(k, "k"),
                                        _dev_ptr(v, "v"), _dev_ptr(q_rot, "q_rot"), _dev_ptr(out, "out"),
                                        int(n_q_heads), float(rope_theta), float(softmax_scale),
                                        int(sliding_window), _stream_ptr(stream)),
           "fg_rotary_kv_attention")


def ragged_attention_noalloc(cache: KVCache, batch: RaggedBatch, q_rot, out, n_q_heads: int,
                             softmax_scale: float, sliding_window: int = 0, stream=None):
    """fg_ragged_attention_noalloc: the attention pass for callers that cannot
    allocate; uses the library's fixed device arrays (see include/fg.h)."""
    _check(lib().fg_ragged_attention_noalloc(cache.handle, batch.handle, _dev_ptr(q_rot, "q_rot"),
                                             _dev_ptr(out, "out"), int(n_q_heads), float(softmax_scale),
                                             int(sliding_window), _stream_ptr(stream)),
           "fg_ragged_attention_noalloc")


def rotary_table(rope_theta: float, head_dim: int, pos_begin: int, n_pos: int):
    """Host float32 cos/sin tables [n_pos, head_dim/2] exactly as libfg builds them."""
    c = np.empty((n_pos, head_dim // 2), np.float32)
    s = np.empty((n_pos, head_dim // 2), np.float32)
    _check(lib().fg_rotary_table(float(rope_theta), int(head_dim), int(pos_begin), int(n_pos),
                                 c.ctypes.data_as(_c_float_p), s.ctypes.data_as(_c_float_p)),
           "fg_rotary_table")
    return c, s


def describe_plan(q_lens, ctx_lens, n_kv_heads: int, group: int, head_dim: int, window: int = 0,
                  use_tc: bool = True, slots: int = 148):
    """The attention work plan for these lengths, built on the host (see
    fg_plan_describe): a dict of int32 arrays [n, 8] for "general",
    "decode", "tc", "dtc" (units) and "combine" (groups), plus "part_rows"
    and "max_combine_rows"."""
    ql, cl = _i32(q_lens, "q_lens"), _i32(ctx_lens, "ctx_lens")
    if ql.shape != cl.shape or ql.ndim != 1:
        raise ValueError("q_lens and ctx_lens must be 1-d arrays of the same length")
    counts = (ctypes.c_int64 * 12)()
    args = (ql.ctypes.data_as(_c_int32_p), cl.ctypes.data_as(_c_int32_p), int(ql.size), int(n_kv_heads),
            int(group), int(head_dim), int(window), int(bool(use_tc)), int(slots))
    _check(lib().fg_plan_describe(*args, None, 0, counts), "fg_plan_describe")
    buf = np.zeros(max(int(counts[11]), 4) // 4, dtype=np.int32)
    _check(lib().fg_plan_describe(*args, buf.ctypes.data_as(ctypes.c_void_p), buf.nbytes, counts),
           "fg_plan_describe")
    offs = [0, counts[7], counts[8], counts[9], counts[10]]
    out = {}
    for i, name in enumerate(("general", "decode", "tc", "dtc", "combine")):
        n = int(counts[i])
        out[name] = buf[offs[i] // 4: offs[i] // 4 + 8 * n].reshape(n, 8).copy()
    out["part_rows"], out["max_combine_rows"] = int(counts[5]), int(counts[6])
    return out


def forward(cache: KVCache, batch: RaggedBatch, q, k, v, q_rot, out, n_q_heads: int,
            rope_theta: float, softmax_scale: float, sliding_window: int = 0, stream=None):
    """One pass on device tensors: rotary + append, then ragged attention."""
    rotary_kv_append(cache, batch, q, k, v, q_rot, n_q_heads, rope_theta, stream)
    ragged_attention(cache, batch, q_rot, out, n_q_heads, softmax_scale, sliding_window, stream)


def forward_host(cache: KVCache, batch: RaggedBatch, host_in: dict, dev: dict, host_out,
                 n_q_heads: int, rope_theta: float, softmax_scale: float,
                 sliding_window: int = 0, stream=None):
    """One pass from host buffers: pinned host q/k/v (``host_in``) are copied to
    the device tensors in ``dev`` ('q', 'k', 'v', 'q_rot', 'out'), the pass runs,
    and the output is copied back into pinned ``host_out``; all on ``stream``."""
    import torch
    s = stream or torch.cuda.current_stream()
    with torch.cuda.stream(s):
        for name in ("q", "k", "v"):
            dev[name].copy_(host_in[name], non_blocking=True)
        forward(cache, batch, dev["q"], dev["k"], dev["v"], dev["q_rot"], dev["out"], n_q_heads,
                rope_theta, softmax_scale, sliding_window, s)
        host_out.copy_(dev["out"], non_blocking=True)


class HostPipeline:
    """Passes from pinned host memory with the copies overlapped across passes.

    Each pass copies its q, k, v from pinned host memory to the device, runs
    rotary + append and the ragged attention (fg_rotary_kv_append,
    fg_ragged_attention), and copies the output back to pinned host memory.
    The host-to-device copy of pass i + 1 runs on an upload stream and the
    device-to-host copy of pass i - 1 on a download stream while pass i
    computes on the compute stream (PCIe carries both directions at once);
    two device buffer sets are used in turn, and events order each copy
    after the pass that last used its buffers. submit() only enqueues; a
    pass's host buffers must stay untouched until wait() for it returns.
    The batch metadata of each pass is put on the compute stream, so one
    batch handle serves every pass (its uploads are double-buffered)."""

    def __init__(self, cache: "KVCache", max_tokens: int, n_q_heads: int, device=None):
        import torch
        dev = device if device is not None else torch.device("cuda", torch.cuda.current_device())
        d, hkv = cache.head_dim, cache.n_kv_heads
        mk = lambda h: torch.empty((max_tokens, h, d), dtype=torch.bfloat16, device=dev)
        self.cache, self.n_q_heads, self.max_tokens = cache, int(n_q_heads), int(max_tokens)
        self.bufs = [{"q": mk(n_q_heads), "k": mk(hkv), "v": mk(hkv), "q_rot": mk(n_q_heads),
                      "out": mk(n_q_heads)} for _ in range(2)]
        self.up, self.comp, self.down = (torch.cuda.Stream(device=dev) for _ in range(3))
        ev = lambda: [torch.cuda.Event() for _ in range(2)]
        # inputs uploaded; inputs consumed (append done); output ready; output downloaded
        self.ev_up, self.ev_in_free, self.ev_done, self.ev_out_free = ev(), ev(), ev(), ev()
        self.n = 0

    def submit(self, batch: "RaggedBatch", seq_ids, q_lens, ctx_lens, block_tables, host_q, host_k,
               host_v, host_out, rope_theta: float, softmax_scale: float, sliding_window: int = 0) -> int:
        """Enqueue one pass; returns its index (for wait())."""
        import torch
        T = int(np.asarray(q_lens, dtype=np.int64).sum())
        if T > self.max_tokens:
            raise ValueError(f"{T} tokens > max_tokens {self.max_tokens}")
        for name, t in (("host_q", host_q), ("host_k", host_k), ("host_v", host_v), ("host_out", host_out)):
            if t.is_cuda or not t.is_pinned() or t.shape[0] != T:
                raise ValueError(f"{name} must be pinned host memory with {T} rows")
        j = self.n % 2
        b = self.bufs[j]
        if self.n >= 2:
            self.up.wait_event(self.ev_in_free[j])
        with torch.cuda.stream(self.up):
            b["q"][:T].copy_(host_q, non_blocking=True)
            b["k"][:T].copy_(host_k, non_blocking=True)
            b["v"][:T].copy_(host_v, non_blocking=True)
            self.ev_up[j].record(self.up)
        self.comp.wait_event(self.ev_up[j])
        if self.n >= 2:
            self.comp.wait_event(self.ev_out_free[j])
        batch.put(self.cache, seq_ids, q_lens, ctx_lens, block_tables, self.comp)
        rotary_kv_append(self.cache, batch, b["q"][:T], b["k"][:T], b["v"][:T], b["q_rot"][:T],
                         self.n_q_heads, rope_theta, self.comp)
        self.ev_in_free[j].record(self.comp)
        ragged_attention(self.cache, batch, b["q_rot"][:T], b["out"][:T], self.n_q_heads, softmax_scale,
                         sliding_window, self.comp)
        self.ev_done[j].record(self.comp)
        self.down.wait_event(self.ev_done[j])
        with torch.cuda.stream(self.down):
            host_out.copy_(b["out"][:T], non_blocking=True)
            self.ev_out_free[j].record(self.down)
        self.n += 1
        return self.n - 1

    def wait(self, i: int):
        """Block until pass i's output is in host memory (the last two
        passes can be waited for)."""
        if not (self.n - 2 <= i < self.n):
            raise ValueError(f"pass {i} is not one of the last two of {self.n}")
        self.ev_out_free[i % 2].synchronize()

    def drain(self):
        self.down.synchronize()
        self.comp.synchronize()
        self.up.synchronize()
