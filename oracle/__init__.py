"""Float64 CPU oracle for the ragged paged-KV attention path.

TEST INFRASTRUCTURE ONLY. Nothing in the product path may import, call or
execute this package: only the tests, the smoke check and the benchmark's
CPU-baseline / reference arm use it. It shares no code with the CUDA library
(no kernels, headers, tables or helpers); both sides only consume the same
seeded inputs.

What it computes (DeepSpeed-FastGen, as summarised on the research-library
card "DeepSpeed-FastGen — paper by Holmes et al. (2024)", Summary and Key
points): for one Dynamic SplitFuse forward pass over a ragged batch of prompt
chunks and decode tokens,
  1. rotary position embedding of Q and K at each token's absolute position
     (the LLaMA / Mistral families named under Key points use rotate-half
     rotary; the pages give no formula, the reading is stated in rotary.py);
  2. append of the new K and V into a blocked ("paged", as in PagedAttention,
     Key points) KV cache through per-sequence block tables;
  3. causal softmax attention of every new token over its sequence's whole
     cached context, gathered into a contiguous array first.

Parity status: every function here is pinned by the CPU tests in
tests/test_oracle_*.py against brute force, closed forms, library special
cases or invariants. The SplitFuse batch composer is an input generator, not
part of the oracle.
"""
from .bf16 import bf16_bits_to_f64, f64_to_bf16_bits
from .rotary import inv_freq, rope_table, rotate_half
from .paged_cache import PagedCache, append_kv, token_positions
from .attention import attend_contiguous, ragged_attention
from .projection import linear, qkv_projection

__all__ = [
    "bf16_bits_to_f64", "f64_to_bf16_bits", "inv_freq", "rope_table", "rotate_half",
    "PagedCache", "append_kv", "token_positions", "attend_contiguous", "ragged_attention",
]
