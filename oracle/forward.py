"""One SplitFuse forward pass of the attention path, oracle side (test
infrastructure only): rotary on Q and K, append K_rot / V into the paged
cache, ragged causal attention with the rotated Q. The order follows the
pages' description of a forward pass over a fixed-budget ragged batch
("DeepSpeed-FastGen — paper by Holmes et al. (2024)", Summary)."""
from .attention import ragged_attention
from .paged_cache import PagedCache, append_kv, token_positions
from .rotary import rotate_half


def splitfuse_pass(cache: PagedCache, block_tables, q_lens, ctx_lens, q_bits, k_bits, v_bits,
                   theta, scale, window=0, tokens=None, rotary=True):
    """Returns (q_rot bits [T,Hq,d], k_rot bits [T,Hkv,d], O float64 [T,Hq,d]).
    Mutates ``cache`` by the append. rotary=False is the pass of a family
    without rotary embedding (OPT, named beside LLaMA and Mistral in the
    card's Key points; its positions are learned and added before the Q/K/V
    projections): Q and K are used as they are."""
    _, pos = token_positions(q_lens, ctx_lens)
    if rotary:
        q_rot = rotate_half(q_bits, pos, theta)
        k_rot = rotate_half(k_bits, pos, theta)
    else:
        q_rot, k_rot = q_bits.copy(), k_bits.copy()
    append_kv(cache, block_tables, q_lens, ctx_lens, k_rot, v_bits)
    out = ragged_attention(cache, block_tables, q_lens, ctx_lens, q_rot, scale, window, tokens)
    return q_rot, k_rot, out
