"""Device staging of synthetic workloads for tests and the benchmark.

Not part of the forward path: it copies generated inputs to the GPU and
writes a workload's prior (already cached) context straight into the cache
tensor, block by block, before a pass runs. Slots a sequence has not filled
yet keep a sentinel pattern so that tests can see any stray write.
"""
from __future__ import annotations

import numpy as np

from .workloads import Workload

SENTINEL = 0xFFFF   # a bf16 NaN pattern: never produced by rounding a finite value


def context_blocks(w: Workload, s: int, sentinel: int = SENTINEL):
    """Physical block ids and their full contents [n, 2, Hkv, B, d] (bf16 bits)
    for the blocks holding sequence s's prior context."""
    c = int(w.ctx_lens[s])
    B = w.block_size
    nb = -(-c // B)
    if nb == 0:
        return np.empty(0, np.int64), None
    k, v = w.context(s)
    blocks = np.full((nb, 2, w.n_kv_heads, B, w.head_dim), sentinel, dtype=np.uint16)
    pad = nb * B - c
    kk = np.concatenate([k, np.full((pad,) + k.shape[1:], sentinel, np.uint16)]) if pad else k
    vv = np.concatenate([v, np.full((pad,) + v.shape[1:], sentinel, np.uint16)]) if pad else v
    blocks[:, 0] = kk.reshape(nb, B, w.n_kv_heads, w.head_dim).transpose(0, 2, 1, 3)
    blocks[:, 1] = vv.reshape(nb, B, w.n_kv_heads, w.head_dim).transpose(0, 2, 1, 3)
    return w.block_tables[s, :nb].astype(np.int64), blocks


def write_context(w: Workload, cache_tensor, keep=(), sentinel: int = SENTINEL, others: str = "random"):
    """Write every sequence's prior context into ``cache_tensor`` (a torch bf16
    tensor shaped [n_blocks, 2, Hkv, B, d]). Returns {s: (ids, blocks)} for the
    sequences in ``keep`` (host copies for an oracle).

    ``others="pool"`` fills the sequences outside ``keep`` from a small pool of
    seeded N(0,1) blocks instead of their own draws (same sizes and
    distribution, far less host work; for very large pools)."""
    import torch
    from concurrent.futures import ThreadPoolExecutor
    kept = {}
    keep = set(keep)
    seqs = [s for s in range(w.n_seqs) if int(w.ctx_lens[s]) > 0]
    own = seqs if others == "random" else [s for s in seqs if s in keep]
    dev = cache_tensor.device
    flat = cache_tensor.view(torch.int16)
    with ThreadPoolExecutor(max_workers=8) as ex:
        for s, (ids, blocks) in zip(own, ex.map(lambda s: context_blocks(w, s, sentinel), own)):
            t = torch.from_numpy(blocks.view(np.int16)).to(dev, non_blocking=False)
            flat[torch.from_numpy(ids).to(dev)] = t
            if s in keep:
                kept[s] = (ids, blocks)
    if others != "random":
        rest = [s for s in seqs if s not in keep]
        if rest:
            n_pool = 64
            rng = np.random.default_rng(np.random.SeedSequence(w.seed, spawn_key=(99,)))
            from .workloads import f32_to_bf16_bits
            pool = f32_to_bf16_bits(rng.standard_normal((n_pool,) + tuple(cache_tensor.shape[1:]),
                                                        dtype=np.float32))
            pool_t = torch.from_numpy(pool.view(np.int16)).to(dev)
            ids = np.concatenate([w.block_tables[s, :-(-int(w.ctx_lens[s]) // w.block_size)] for s in rest])
            ids_t = torch.from_numpy(ids.astype(np.int64)).to(dev)
            for i in range(0, len(ids), 4096):
                part = ids_t[i:i + 4096]
                flat[part] = pool_t[part % n_pool]
    return kept


def fill(cache_tensor, sentinel: int = SENTINEL):
    import torch
    cache_tensor.view(torch.int16).fill_(np.int16(np.uint16(sentinel).view(np.int16)))


def qkv_device(w: Workload, device="cuda"):
    import torch
    q, k, v = w.qkv()
    return tuple(torch.from_numpy(x.view(np.int16)).to(device).view(torch.bfloat16) for x in (q, k, v))


def to_bits(t) -> np.ndarray:
    """A bf16 torch tensor as numpy uint16 bits (host)."""
    import torch
    return t.detach().contiguous().view(torch.int16).cpu().numpy().view(np.uint16)
