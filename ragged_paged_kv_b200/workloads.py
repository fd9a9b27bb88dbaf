"""Seeded synthetic ragged batches for the Dynamic SplitFuse attention path.

This module is an input generator only. It draws bf16 tensors and composes
ragged batches (which sequences, how many new tokens each, how much cached
context each has, which physical KV blocks each owns). It does none of the
path's arithmetic: no rotary, no cache addressing, no attention.

Sources for the shapes and distributions ("DeepSpeed-FastGen" research-library
card, Summary and Key points; the reading-notes page, method line):
  * every forward pass carries a fixed token budget, long prompts are cut into
    chunks, decode tokens and short prompts fill the rest;
  * benchmark clients send 512 requests, prompt length ~ N(2600, 30%) and
    output length ~ N(60, 30%) (read as sd = 0.3 * mean);
  * the KV cache is blocked (paged), each sequence addressing its blocks
    through a per-sequence table.

Determinism: every random draw comes from ``numpy.random.SeedSequence`` keyed
by (config seed, stream kind, request id, 64-position chunk). A token's Q/K/V
(and a cached position's prior K/V) therefore depend only on (request,
absolute position), never on how the batch was chunked, so a prompt processed
in N chunks sees exactly the same numbers as the same prompt in one shot.
"""
from __future__ import annotations

import math
import os
from concurrent.futures import ThreadPoolExecutor
from dataclasses import dataclass, field, replace

import numpy as np

CHUNK = 64                      # positions per seeded generation chunk
_KIND_QKV, _KIND_CTX, _KIND_PERM, _KIND_SCHED, _KIND_LENS = 1, 2, 3, 4, 5


# ----------------------------------------------------------------------------
# bf16 sampling
# ----------------------------------------------------------------------------
def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round float32 values to bf16 (round-half-even) and return the raw bits.

    Used only to turn float32 normal draws into bf16 inputs. Inputs are finite.
    """
    b = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    r = (b + np.uint32(0x7FFF) + ((b >> np.uint32(16)) & np.uint32(1))) >> np.uint32(16)
    return r.astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    return (np.asarray(b, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


def _normal_bf16(seed: int, key: tuple, shape) -> np.ndarray:
    rng = np.random.default_rng(np.random.SeedSequence(seed, spawn_key=key))
    return f32_to_bf16_bits(rng.standard_normal(shape, dtype=np.float32))


def _chunked(seed, kind, req, pos_begin, pos_end, width, n_arrays):
    """Draw ``n_arrays`` bf16 arrays of shape [pos_end-pos_begin, width] for a
    request's absolute positions, assembled from 64-position seeded chunks."""
    n = pos_end - pos_begin
    outs = [np.empty((n, width), dtype=np.uint16) for _ in range(n_arrays)]
    if n <= 0:
        return outs
    c0, c1 = pos_begin // CHUNK, (pos_end - 1) // CHUNK
    for c in range(c0, c1 + 1):
        blk = _normal_bf16(seed, (kind, int(req), c), (n_arrays, CHUNK, width))
        lo = max(pos_begin, c * CHUNK)
        hi = min(pos_end, (c + 1) * CHUNK)
        for a in range(n_arrays):
            outs[a][lo - pos_begin:hi - pos_begin] = blk[a, lo - c * CHUNK:hi - c * CHUNK]
    return outs


def _pool():
    return ThreadPoolExecutor(max_workers=max(1, min(32, len(os.sched_getaffinity(0)))))


# ----------------------------------------------------------------------------
# Workload description
# ----------------------------------------------------------------------------
@dataclass
class Workload:
    """One ragged batch plus the model shape it runs at.

    Token rows are packed in ``seq_ids`` order; sequence s owns rows
    ``cu_q[s] .. cu_q[s+1]-1`` holding its new tokens at absolute positions
    ``ctx_lens[s] .. ctx_lens[s]+q_lens[s]-1``.
    """
    name: str
    n_q_heads: int
    n_kv_heads: int
    head_dim: int
    block_size: int
    n_blocks: int
    rope_theta: float
    sliding_window: int
    seq_ids: np.ndarray
    q_lens: np.ndarray
    ctx_lens: np.ndarray
    block_tables: np.ndarray      # int32 [S, max_blocks_per_seq], -1 padded
    seed: int
    budget: int
    note: str = ""
    _cache: dict = field(default_factory=dict, repr=False)

    # -- sizes --------------------------------------------------------------
    @property
    def n_seqs(self) -> int:
        return int(len(self.q_lens))

    @property
    def n_tokens(self) -> int:
        return int(self.q_lens.sum())

    @property
    def cu_q(self) -> np.ndarray:
        return np.concatenate([[0], np.cumsum(self.q_lens)]).astype(np.int64)

    @property
    def softmax_scale(self) -> float:
        return 1.0 / math.sqrt(self.head_dim)

    @property
    def block_bytes(self) -> int:
        return 2 * self.n_kv_heads * self.block_size * self.head_dim * 2

    def blocks_used(self, s: int) -> int:
        L = int(self.ctx_lens[s] + self.q_lens[s])
        return -(-L // self.block_size)

    # -- tensors ------------------------------------------------------------
    def qkv(self):
        """bf16 bits of the new tokens: q [T,Hq,d], k [T,Hkv,d], v [T,Hkv,d]."""
        if "qkv" in self._cache:
            return self._cache["qkv"]
        Hq, Hkv, d = self.n_q_heads, self.n_kv_heads, self.head_dim
        width = (Hq + 2 * Hkv) * d

        def one(s):
            c = int(self.ctx_lens[s])
            (x,) = _chunked(self.seed, _KIND_QKV, self.seq_ids[s], c, c + int(self.q_lens[s]), width, 1)
            return x

        with _pool() as ex:
            parts = list(ex.map(one, range(self.n_seqs)))
        x = np.concatenate(parts, axis=0) if parts else np.empty((0, width), np.uint16)
        T = x.shape[0]
        q = np.ascontiguousarray(x[:, :Hq * d].reshape(T, Hq, d))
        k = np.ascontiguousarray(x[:, Hq * d:(Hq + Hkv) * d].reshape(T, Hkv, d))
        v = np.ascontiguousarray(x[:, (Hq + Hkv) * d:].reshape(T, Hkv, d))
        self._cache["qkv"] = (q, k, v)
        return q, k, v

    def context(self, s: int, pos_begin: int = 0, pos_end: int | None = None):
        """Prior cached K (already rotated) and V of sequence s at positions
        [pos_begin, pos_end) (default: the whole prior context), bf16 bits
        shaped [n, Hkv, d]."""
        c = int(self.ctx_lens[s])
        pos_end = c if pos_end is None else min(pos_end, c)
        width = self.n_kv_heads * self.head_dim
        k, v = _chunked(self.seed, _KIND_CTX, self.seq_ids[s], pos_begin, pos_end, width, 2)
        n = k.shape[0]
        return (k.reshape(n, self.n_kv_heads, self.head_dim),
                v.reshape(n, self.n_kv_heads, self.head_dim))

    def contexts(self, seqs=None):
        """Iterate (s, k_ctx, v_ctx) over sequences, generated by a thread pool."""
        seqs = range(self.n_seqs) if seqs is None else seqs
        seqs = [s for s in seqs if int(self.ctx_lens[s]) > 0]
        with _pool() as ex:
            for s, kv in zip(seqs, ex.map(self.context, seqs)):
                yield s, kv[0], kv[1]

    # -- variants -----------------------------------------------------------
    def with_permuted_blocks(self, perm_seed: int) -> "Workload":
        """Same tokens, same logical layout, different physical block ids."""
        bt = _assign_blocks(self.q_lens + self.ctx_lens, self.block_size, self.n_blocks,
                            self.seed * 1000003 + perm_seed)
        w = replace(self, block_tables=bt, _cache={})
        if "qkv" in self._cache:
            w._cache["qkv"] = self._cache["qkv"]
        return w

    def summary(self) -> dict:
        return {"name": self.name, "tokens": self.n_tokens, "seqs": self.n_seqs,
                "q_heads": self.n_q_heads, "kv_heads": self.n_kv_heads,
                "head_dim": self.head_dim, "block_size": self.block_size,
                "n_blocks": self.n_blocks, "sliding_window": self.sliding_window,
                "note": self.note}


def _assign_blocks(lengths, block_size, n_blocks, seed) -> np.ndarray:
    """Give each sequence ceil(L/B) distinct physical blocks, drawn in order
    from a seeded permutation of the whole pool."""
    need = [-(-int(L) // block_size) for L in lengths]
    total = sum(need)
    if total > n_blocks:
        raise ValueError(f"pool of {n_blocks} blocks cannot hold {total}")
    rng = np.random.default_rng(np.random.SeedSequence(seed, spawn_key=(_KIND_PERM,)))
    if n_blocks <= 4 * total + 65536:
        ids = rng.permutation(n_blocks)[:total]
    else:  # large pool: distinct uniform draws without materialising it all
        ids = rng.choice(n_blocks, size=total, replace=False)
    width = max(need) if need else 1
    bt = np.full((len(need), width), -1, dtype=np.int32)
    o = 0
    for s, n in enumerate(need):
        bt[s, :n] = ids[o:o + n]
        o += n
    return bt


def _make(name, Hq, Hkv, d, B, seq_ids, q_lens, ctx_lens, seed, budget, *, n_blocks=None,
          theta=10000.0, window=0, note="") -> Workload:
    q_lens = np.asarray(q_lens, dtype=np.int32)
    ctx_lens = np.asarray(ctx_lens, dtype=np.int32)
    need = int(sum(-(-int(L) // B) for L in q_lens + ctx_lens))
    if n_blocks is None:
        n_blocks = max(4 * need, 4096)
    bt = _assign_blocks(q_lens + ctx_lens, B, n_blocks, seed)
    return Workload(name=name, n_q_heads=Hq, n_kv_heads=Hkv, head_dim=d, block_size=B,
                    n_blocks=int(n_blocks), rope_theta=theta, sliding_window=window,
                    seq_ids=np.asarray(seq_ids, dtype=np.int32), q_lens=q_lens,
                    ctx_lens=ctx_lens, block_tables=bt, seed=seed, budget=budget, note=note)


# ----------------------------------------------------------------------------
# Dynamic SplitFuse batch composition (closed-loop synthetic clients)
# ----------------------------------------------------------------------------
@dataclass
class _Req:
    rid: int
    prompt: int
    out: int
    done: int = 0      # prompt tokens already in the cache
    gen: int = 0       # tokens generated so far


POLICIES = ("greedy", "equal_split")


def splitfuse_schedule(seed: int, budget: int = 2048, n_active: int = 32, n_total: int = 512,
                       prompt_mean: float = 2600.0, out_mean: float = 60.0, rel_sd: float = 0.3,
                       events: list | None = None, policy: str = "greedy", prompts=None, outputs=None):
    """Yield (iteration, [(rid, q_len, ctx_len), ...]) for a closed loop of
    synthetic clients under a fixed token budget.

    Rules of each iteration:
      1. every request already generating contributes one decode token, its
         context being the prompt plus the tokens generated before it;
      2. the rest of the budget goes to requests still in their prompt, in
         arrival order, each taking min(prompt tokens left, share left),
         where the share depends on ``policy``:
           "greedy"       the whole rest of the budget (every pass is filled
                          while prompt tokens are pending);
           "equal_split"  the pending prompt tokens (the pool) divided evenly
                          over the passes they need at this rest r: with
                          n = ceil(pool / r) passes, ceil(pool / n) tokens
                          (the card's concavity argument: throughput is
                          concave in tokens per pass, so splitting a pool of
                          tokens evenly across passes is optimal; "Interesting
                          ideas" of the DeepSpeed-FastGen research-library
                          card);
      3. a request whose prompt completes in this iteration has produced its
         first output token; a generating request produces one more;
      4. a request that has produced its G-th token leaves at the end of the
         iteration and the next arrival takes its place.
    Prompt length P = max(1, round(N(2600, 780))), output length
    G = max(1, round(N(60, 18))); ``prompts`` / ``outputs`` (sequences of
    n_total ints) replace the draws.
    If `events` is a list, each iteration appends (iteration, produced,
    joined, left) to it after the batch has been consumed: the (rid,
    is_first_token) pairs of the tokens the iteration produced, the requests
    that became active for the next iteration and those that finished.
    """
    if policy not in POLICIES:
        raise ValueError(f"policy {policy!r} not in {POLICIES}")
    rng = np.random.default_rng(np.random.SeedSequence(seed, spawn_key=(_KIND_LENS,)))
    P = np.maximum(1, np.rint(rng.normal(prompt_mean, rel_sd * prompt_mean, n_total))).astype(int)
    G = np.maximum(1, np.rint(rng.normal(out_mean, rel_sd * out_mean, n_total))).astype(int)
    if prompts is not None:
        P = np.asarray(prompts, dtype=int)
    if outputs is not None:
        G = np.asarray(outputs, dtype=int)
    if len(P) < n_total or len(G) < n_total or (P < 1).any() or (G < 1).any():
        raise ValueError("need n_total prompt and output lengths, each >= 1")
    nxt = 0
    active: list[_Req] = []
    while len(active) < n_active and nxt < n_total:
        active.append(_Req(nxt, int(P[nxt]), int(G[nxt])))
        nxt += 1
    it = 0
    while active:
        batch = []
        left = budget
        for r in active:
            if r.done == r.prompt and left > 0:
                batch.append((r.rid, 1, r.prompt + r.gen - 1))
                left -= 1
        share = left
        if policy == "equal_split" and left > 0:
            pool = sum(r.prompt - r.done for r in active if r.done < r.prompt)
            if pool > left:
                n_pass = -(-pool // left)
                share = -(-pool // n_pass)
        for r in active:
            if r.done < r.prompt and share > 0:
                c = min(r.prompt - r.done, share)
                batch.append((r.rid, c, r.done))
                share -= c
        yield it, batch
        by_id = {b[0]: b for b in batch}
        still = []
        produced = []
        for r in active:
            b = by_id.get(r.rid)
            if b is not None:
                if r.done < r.prompt:
                    r.done += b[1]
                    if r.done == r.prompt:
                        r.gen = 1
                        produced.append((r.rid, True))
                else:
                    r.gen += 1
                    produced.append((r.rid, False))
            if r.done == r.prompt and r.gen >= r.out:
                continue
            still.append(r)
        left_ids = [r.rid for r in active if r not in still]
        active = still
        joined = []
        while len(active) < n_active and nxt < n_total:
            active.append(_Req(nxt, int(P[nxt]), int(G[nxt])))
            joined.append(nxt)
            nxt += 1
        if events is not None:
            events.append((it, produced, joined, left_ids))
        it += 1


def splitfuse_snapshot(seed: int, budget: int = 2048, at_least: int = 50):
    """First iteration >= ``at_least`` whose batch fills the budget exactly."""
    for it, batch in splitfuse_schedule(seed, budget):
        if it >= at_least and sum(b[1] for b in batch) == budget:
            return it, batch
    raise RuntimeError("schedule ended before a full batch appeared")


# ----------------------------------------------------------------------------
# The five configurations
# ----------------------------------------------------------------------------
def config1(seed: int = 1) -> Workload:
    """Tiny ragged batch: 4/4 heads, d=64, B=16, 64 blocks; (q, ctx) =
    (40,0), (1,37), (1,5), (22,10)."""
    return _make("tiny", 4, 4, 64, 16, [0, 1, 2, 3], [40, 1, 1, 22], [0, 37, 5, 10],
                 seed, 64, n_blocks=64, note="prefill 40 + decode ctx37 + decode ctx5 + chunk 22 at ctx10")


def config2(seed: int = 2) -> Workload:
    """Llama-2-7B shape (32/32 heads, d=128, B=64): SplitFuse snapshot of a
    budget-2048 closed loop, first full iteration at or after 50."""
    it, batch = splitfuse_snapshot(seed, 2048, 50)
    rid = [b[0] for b in batch]
    q = [b[1] for b in batch]
    c = [b[2] for b in batch]
    nd = sum(1 for x in q if x == 1)
    return _make("llama7b_splitfuse", 32, 32, 128, 64, rid, q, c, seed, 2048,
                 note=f"iteration {it}: {nd} decodes + {len(q) - nd} prompt chunk(s)")


def config3(seed: int = 3, n_blocks: int | None = None) -> Workload:
    """Decode-heavy: 256 decodes, ctx ~ U[512, 4096], Llama-2-7B shape,
    blocks drawn from a large permuted pool (180 GB-sized on a B200)."""
    rng = np.random.default_rng(np.random.SeedSequence(seed, spawn_key=(_KIND_SCHED,)))
    ctx = rng.integers(512, 4096, size=256, endpoint=True)
    if n_blocks is None:
        n_blocks = 180 * 10**9 // (2 * 32 * 64 * 128 * 2)
    return _make("decode_heavy", 32, 32, 128, 64, list(range(256)), [1] * 256, ctx, seed, 256,
                 n_blocks=n_blocks, note=f"pool {n_blocks} blocks")


def config4(seed: int = 4) -> Workload:
    """Mistral-7B GQA (32/8, d=128, window 4096, B=64), budget 4096: last
    2048-token chunk of a 16384 prompt + 3 x 512-token chunks of 3000-token
    prompts + 512 decodes with ctx ~ U[1024, 8192]."""
    rng = np.random.default_rng(np.random.SeedSequence(seed, spawn_key=(_KIND_SCHED,)))
    ks = rng.integers(0, 4, size=3, endpoint=True)
    dctx = rng.integers(1024, 8192, size=512, endpoint=True)
    q = [2048] + [512] * 3 + [1] * 512
    c = [14336] + [512 * int(k) for k in ks] + [int(x) for x in dctx]
    return _make("mistral_gqa_window", 32, 8, 128, 64, list(range(len(q))), q, c, seed, 4096,
                 window=4096, note=f"3000-token prompts at ctx {[512 * int(k) for k in ks]}")


def config5(seed: int = 5) -> Workload:
    """Llama-2-70B GQA (64/8, d=128, B=64), budget 2112: last 2048-token
    chunk of a 32768 prompt (ctx 30720) + 64 decodes at ctx ~ U[2048, 32768]."""
    rng = np.random.default_rng(np.random.SeedSequence(seed, spawn_key=(_KIND_SCHED,)))
    dctx = rng.integers(2048, 32768, size=64, endpoint=True)
    q = [2048] + [1] * 64
    c = [30720] + [int(x) for x in dctx]
    return _make("llama70b_long_prompt", 64, 8, 128, 64, list(range(65)), q, c, seed, 2112)


def prompt_chunks(Hq, Hkv, d, B, prompt: int, chunk: int, seed: int, *, n_blocks=None,
                  window=0, rid: int = 0) -> list[Workload]:
    """A single prompt of ``prompt`` tokens split into consecutive chunks of
    ``chunk`` (chunk == prompt gives the one-shot prefill). All chunks share one
    block table, so appending them in order builds the same cache as one shot."""
    if n_blocks is None:
        n_blocks = max(4 * -(-prompt // B), 4096)
    bt = _assign_blocks(np.array([prompt]), B, n_blocks, seed)
    out = []
    for c0 in range(0, prompt, chunk):
        n = min(chunk, prompt - c0)
        L = c0 + n
        nb = -(-L // B)
        t = bt[:, :nb].copy()
        out.append(Workload(name=f"prompt{prompt}_chunk{c0}", n_q_heads=Hq, n_kv_heads=Hkv,
                            head_dim=d, block_size=B, n_blocks=int(n_blocks), rope_theta=10000.0,
                            sliding_window=window, seq_ids=np.array([rid], np.int32),
                            q_lens=np.array([n], np.int32), ctx_lens=np.array([c0], np.int32),
                            block_tables=t, seed=seed, budget=n))
    return out


CONFIGS = {1: config1, 2: config2, 3: config3, 4: config4, 5: config5}
