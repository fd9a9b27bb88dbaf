"""Blocked (paged) KV cache model, oracle side (test infrastructure only).

The pages say FastGen keeps the KV cache in fixed-size blocks, as
PagedAttention does ("DeepSpeed-FastGen — paper by Holmes et al. (2024)", Key
points), and that a forward pass holds a ragged mix of prompt chunks and
decode tokens (Summary). They give no layout; the reading used here:

  * physical storage is [n_blocks][2 (K, V)][n_kv_heads][block_size][head_dim]
    of bf16 words;
  * sequence s owns the blocks listed in its block table, in logical order:
    its token at absolute position p lives in block bt_s[p // B], slot p % B;
  * a batch row j of sequence s (0 <= j < q_s) is the token at position
    ctx_s + j, rows of the batch are packed sequence after sequence.

The model is sparse (a dict of touched blocks) so that pools of any size cost
only what a test writes.
"""
import numpy as np


class PagedCache:
    def __init__(self, n_blocks, n_kv_heads, block_size, head_dim, fill=0xFFFF):
        self.n_blocks = int(n_blocks)
        self.n_kv_heads = int(n_kv_heads)
        self.block_size = int(block_size)
        self.head_dim = int(head_dim)
        self.fill = np.uint16(fill)
        self.blocks = {}

    def block(self, b: int) -> np.ndarray:
        b = int(b)
        if not 0 <= b < self.n_blocks:
            raise IndexError(f"block id {b} outside [0, {self.n_blocks})")
        if b not in self.blocks:
            self.blocks[b] = np.full((2, self.n_kv_heads, self.block_size, self.head_dim),
                                     self.fill, dtype=np.uint16)
        return self.blocks[b]

    def write_positions(self, bt_row, positions, k_bits, v_bits):
        """Store K [n, Hkv, d] and V at the given absolute positions."""
        B = self.block_size
        for i, p in enumerate(np.asarray(positions).reshape(-1)):
            blk = self.block(bt_row[int(p) // B])
            blk[0, :, int(p) % B, :] = k_bits[i]
            blk[1, :, int(p) % B, :] = v_bits[i]

    def gather(self, bt_row, length: int):
        """Contiguous K, V [length, Hkv, d] of one sequence (bf16 words)."""
        B = self.block_size
        nb = -(-int(length) // B)
        K = np.empty((nb * B, self.n_kv_heads, self.head_dim), dtype=np.uint16)
        V = np.empty_like(K)
        for i in range(nb):
            blk = self.block(bt_row[i])
            K[i * B:(i + 1) * B] = blk[0].transpose(1, 0, 2)
            V[i * B:(i + 1) * B] = blk[1].transpose(1, 0, 2)
        return K[:length], V[:length]


def token_positions(q_lens, ctx_lens):
    """Per batch row: (sequence index, absolute position)."""
    seq = np.repeat(np.arange(len(q_lens)), np.asarray(q_lens))
    starts = np.concatenate([[0], np.cumsum(q_lens)[:-1]]).astype(np.int64)
    j = np.arange(int(np.sum(q_lens))) - starts[seq]
    pos = np.asarray(ctx_lens, dtype=np.int64)[seq] + j
    return seq, pos


def append_kv(cache: PagedCache, block_tables, q_lens, ctx_lens, k_rot_bits, v_bits):
    """Write every new token's rotated K and its V into its cache slot
    (a bit copy); all other slots keep their previous bits."""
    seq, pos = token_positions(q_lens, ctx_lens)
    for s in range(len(q_lens)):
        rows = np.nonzero(seq == s)[0]
        if len(rows):
            cache.write_positions(block_tables[s], pos[rows], k_rot_bits[rows], v_bits[rows])
