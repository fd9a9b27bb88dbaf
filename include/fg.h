/*
 * fg.h - C ABI of the B200 ragged paged-KV attention library (libfg).
 *
 * One Dynamic SplitFuse forward pass of attention: a ragged batch of prompt
 * chunks and single-token decodes, at most a fixed token budget ("DeepSpeed-
 * FastGen — paper by Holmes et al. (2024)", Summary: every forward pass is
 * kept at a fixed token count; long prompts are cut into chunks spread over
 * several iterations; short prompts and generation tokens fill the rest). For
 * that batch the library
 *   1. rotates Q and K with rotary position embedding,
 *   2. appends the new K and V into a blocked (paged) KV cache through
 *      per-sequence block tables (same page, Key points: the KV cache is
 *      blocked as in PagedAttention),
 *   3. runs one ragged causal attention of every new token over its
 *      sequence's cached context.
 * Around those steps it also provides the layer's Q/K/V projection fused
 * with steps 1 and 2 (fg_qkv_rotary_kv_append) and its output projection
 * (fg_output_projection), both on the tensor cores.
 *
 * Conventions shared by every call
 *   - Types: all tensors are bf16 (16-bit words), row-major, densely packed.
 *     T = tokens in the batch, Hq / Hkv = query / key-value heads,
 *     d = head_dim, B = block_size.
 *   - Pointers marked "device" must point to memory of the current CUDA
 *     device; "host" pointers are ordinary CPU memory that the call only
 *     reads during the call (nothing is retained).
 *   - `stream` is a cudaStream_t passed as void* (NULL = legacy default
 *     stream). Device work is asynchronous on it; calls that touch the same
 *     cache / batch must be issued on one stream, in the order
 *     put -> rotary_kv_append -> ragged_attention.
 *   - Every call returns an fg_status and never aborts the process. On
 *     failure nothing was launched and no output was written;
 *     fg_last_error() gives a thread-local, human-readable reason.
 *   - Handles are owned by the caller and released by the matching
 *     *_destroy. A handle may be used by one host thread at a time.
 */
#ifndef FG_H_
#define FG_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum fg_status {
  FG_OK = 0,
  FG_ERR_INVALID_ARG = 1,   /* null pointer, negative size, bad handle          */
  FG_ERR_OUT_OF_RANGE = 2,  /* a block id outside [0, n_blocks)                 */
  FG_ERR_ALIAS = 3,         /* two writes to one cache slot, duplicate seq ids  */
  FG_ERR_CAPACITY = 4,      /* batch larger than the handle was created for     */
  FG_ERR_UNSUPPORTED = 5,   /* head_dim / block_size / head ratio not built     */
  FG_ERR_CUDA = 6,          /* a CUDA runtime call failed (no device, OOM ...)  */
  FG_ERR_DEVICE_CHECK = 7,  /* a kernel found an out-of-range index and skipped */
  FG_ERR_TIMEOUT = 8        /* a bounded device wait gave up                    */
} fg_status;

typedef struct fg_kv_cache fg_kv_cache;         /* opaque */
typedef struct fg_ragged_batch fg_ragged_batch; /* opaque */

/* ------------------------------------------------------------------------ */
/* Paged KV cache (Key points: blocked KV cache as in PagedAttention)        */
/* ------------------------------------------------------------------------ */

/* Allocate a cache of n_blocks blocks on the current device with cudaMalloc.
 * Layout (bf16 words): [n_blocks][2 (0 = K, 1 = V)][n_kv_heads][block_size]
 * [head_dim]; one (block, K|V, head) tile is block_size*head_dim contiguous
 * words. Contents are left uninitialised. Supported: head_dim in {64, 128},
 * block_size in {16, 32, 64, 128}, n_kv_heads in [1, 256], n_blocks >= 1,
 * else FG_ERR_UNSUPPORTED / FG_ERR_INVALID_ARG. Offsets are 64-bit, so a pool
 * may fill the whole of a 180 GB device. */
fg_status fg_kv_cache_create(int32_t block_size, int32_t n_blocks, int32_t n_kv_heads,
                             int32_t head_dim, fg_kv_cache** out);

/* Same, over caller-owned device memory (e.g. a torch tensor) of `bytes`
 * bytes at `dev_ptr` (16-byte aligned, at least the size above). The
 * memory is borrowed: it must outlive the handle and is never freed here. */
fg_status fg_kv_cache_create_external(int32_t block_size, int32_t n_blocks, int32_t n_kv_heads,
                                      int32_t head_dim, void* dev_ptr, size_t bytes,
                                      fg_kv_cache** out);

/* Base device pointer and element strides of the 5-d layout above
 * (strides_elems[0] = block, [1] = K|V, [2] = head, [3] = slot, [4] = dim). */
fg_status fg_kv_cache_layout(const fg_kv_cache* cache, void** base, int64_t strides_elems[5]);

/* Builds the rotary cos/sin table for positions 0 .. max_position (at least;
 * the table is sized in powers of two, 4096 positions or more) and the given
 * rope_theta, on the host, and uploads it: the work the first rotary call
 * for a position range does otherwise. A server calls it once at start-up
 * with its longest context, so that no pass pays for it. Synchronous and
 * allocating; a table that already covers the range is kept. */
fg_status fg_kv_cache_prepare_rotary(fg_kv_cache* cache, double rope_theta, int32_t max_position);

/* Releases the handle and (for fg_kv_cache_create) the pool. Waits for the
 * device first. NULL is accepted. */
fg_status fg_kv_cache_destroy(fg_kv_cache* cache);

/* ------------------------------------------------------------------------ */
/* Ragged batch (Summary: a fixed budget filled with prompt chunks and       */
/* generation tokens)                                                        */
/* ------------------------------------------------------------------------ */

/* A reusable holder for one batch's metadata, sized for at most max_tokens
 * new tokens, max_seqs sequences and max_blocks_per_seq blocks per sequence.
 * Device buffers are allocated on the first successful put. */
fg_status fg_ragged_batch_create(int32_t max_tokens, int32_t max_seqs, int32_t max_blocks_per_seq,
                                 fg_ragged_batch** out);

/* Describe the next forward pass. Host arrays, all of length n_seqs:
 *   seq_ids   caller's sequence ids (distinct; used only for validation),
 *   q_lens    new tokens of each sequence (>= 1): prompt-chunk length or 1,
 *   ctx_lens  tokens already in the cache before this pass (>= 0);
 * block_tables: host int32 [n_seqs][block_table_stride]; row s lists the
 * physical blocks of sequence s in logical order and must hold at least
 * ceil((ctx_lens[s] + q_lens[s]) / block_size) valid ids; entries past that
 * are ignored. Token rows of q/k/v/out are packed in this sequence order,
 * sequence s's new tokens sitting at absolute positions ctx_lens[s] ..
 * ctx_lens[s] + q_lens[s] - 1. n_seqs == 0 describes an empty pass.
 * Checks, all before any device work: sizes within the handle's capacity
 * (FG_ERR_CAPACITY), q_lens >= 1 and ctx_lens >= 0 (FG_ERR_INVALID_ARG),
 * used block ids inside the cache (FG_ERR_OUT_OF_RANGE), no cache slot
 * written twice, no block repeated within one table, no new token written
 * into a slot that another sequence of the batch reads, distinct seq_ids
 * (FG_ERR_ALIAS). The packed metadata is copied to the device
 * asynchronously from a pinned staging buffer, into one half of a double
 * buffer, on a copy stream of the handle's own; `stream` waits for that copy,
 * so work queued on it after the put sees the new pass. The copy itself waits
 * only for the work queued on `stream` before the previous put (the last
 * work that read the same half), so it runs while the device still works on
 * the previous pass. Keep every call that uses a pass on the stream of its
 * put, or order other streams after it. A put on the same handle may wait on
 * the host for the copy of the put two before it. */
fg_status fg_ragged_batch_put(fg_ragged_batch* batch, const fg_kv_cache* cache, int32_t n_seqs,
                              const int32_t* seq_ids, const int32_t* q_lens,
                              const int32_t* ctx_lens, const int32_t* block_tables,
                              int32_t block_table_stride, void* stream);

/* Tokens and sequences of the last successful put. */
fg_status fg_ragged_batch_shape(const fg_ragged_batch* batch, int32_t* n_tokens, int32_t* n_seqs);

fg_status fg_ragged_batch_destroy(fg_ragged_batch* batch);

/* ------------------------------------------------------------------------ */
/* Step 1 + 2: rotary on Q/K, append K_rot and V into the cache              */
/* ------------------------------------------------------------------------ */

/* q: device [T][n_q_heads][d], k and v: device [T][Hkv][d], q_rot: device
 * [T][n_q_heads][d] (may equal q for in-place). For token at position p and
 * frequency i < d/2: inv_freq_i = 1 / rope_theta^(2i/d), a = p * inv_freq_i
 * in double; c, s = cos(a), sin(a) by the host C library in double, rounded
 * once to float; pairs (i, i + d/2) are rotated in double,
 *   y_i = x_i c - x_{i+d/2} s,   y_{i+d/2} = x_{i+d/2} c + x_i s,
 * and each result is rounded once to bf16 (ties to even). The pages name the
 * HuggingFace LLaMA / Mistral families (Key points), which use this
 * rotate-half pairing. K_rot and V are bit-copied to slot p % B of block
 * block_table[s][p / B]; no other cache word changes. n_q_heads must be a
 * multiple of the cache's n_kv_heads. The first call for a (rope_theta,
 * position range) builds or grows the cos/sin table on the host and uploads
 * it (synchronous, allocating); later calls reuse it. */
fg_status fg_rotary_kv_append(fg_kv_cache* cache, const fg_ragged_batch* batch, const void* q,
                              const void* k, const void* v, void* q_rot, int32_t n_q_heads,
                              double rope_theta, void* stream);

/* The Q/K/V projection fused with steps 1 and 2 (the GEMM that produces q,
 * k and v for this hot path, kept on the device): qkv = x w_qkv^T with x
 * device [T][hidden] bf16 (T = the batch's tokens) and w_qkv device
 * [(n_q_heads + 2 Hkv) d][hidden] bf16 (rows: the q heads, then k, then v,
 * d rows each; the layout of a linear layer's weight), fp32 accumulation;
 * each output is rounded once to bf16, as a projection with bf16 output
 * would, then q and k are rotated and stored exactly as
 * fg_rotary_kv_append does (q_rot device [T][n_q_heads][d]; K_rot and V
 * bit-copied into slot p % B of block block_table[s][p / B]). hidden must be
 * a positive multiple of 64; x, w_qkv and q_rot 16-byte aligned. The result
 * equals the projection followed by fg_rotary_kv_append up to the
 * projection's own rounding (fp32 sums in another order can round a value to
 * the neighbouring bf16). Asynchronous on `stream`; the first call for a
 * rope_theta and position range builds the cos/sin table (synchronous). */
fg_status fg_qkv_rotary_kv_append(fg_kv_cache* cache, const fg_ragged_batch* batch, const void* x,
                                  const void* w_qkv, int32_t hidden, void* q_rot, int32_t n_q_heads,
                                  double rope_theta, void* stream);

/* Step 2 alone, for model families without rotary position embedding: the
 * pages name OPT beside LLaMA and Mistral (Key points), and OPT adds learned
 * absolute position embeddings to the hidden states before the Q/K/V
 * projections, so its K and V enter the cache as they are. k and v: device
 * [T][Hkv][d], 16-byte aligned; both are bit-copied to slot p % B of block
 * block_table[s][p / B] (no other cache word changes), and the attention
 * then takes the queries themselves as q_rot. Asynchronous on `stream`;
 * errors as fg_rotary_kv_append (FG_ERR_INVALID_ARG for NULL or misaligned
 * tensors, a batch whose cache is not `cache`). */
fg_status fg_kv_append(fg_kv_cache* cache, const fg_ragged_batch* batch, const void* k, const void* v,
                       void* stream);

/* ------------------------------------------------------------------------ */
/* Step 3: one ragged causal attention over every sequence's cached context  */
/* ------------------------------------------------------------------------ */

/* q_rot: device [T][n_q_heads][d] (rotated queries); out: device
 * [T][n_q_heads][d]. Query head h reads kv head h / (n_q_heads / Hkv). The
 * token at position p attends to the cached positions k with
 * max(0, p - sliding_window + 1) <= k <= p (sliding_window = 0: no window),
 *   out = sum_k exp(z_k - m) V_k / sum_k exp(z_k - m),
 *   z_k = softmax_scale * <q, K_k>,  m = max_k z_k,
 * with bf16 operands, fp32 accumulation and fp32 softmax. Must follow the
 * append of the same batch (fg_rotary_kv_append, fg_kv_append or
 * fg_qkv_rotary_kv_append) on the same stream (a token sees its own K/V).
 * Long contexts are split across thread blocks and merged by a log-sum-exp
 * combine. The split workspace and the work-plan buffer are owned by the
 * batch handle and grown with stream-ordered allocation (cudaMallocAsync on
 * `stream`) when a pass needs more; the host builds the plan and uploads it
 * through pinned staging each time the batch or (n_q_heads, window) changes,
 * into one half of a double buffer on the handle's copy stream, the way
 * fg_ragged_batch_put uploads the metadata (`stream` waits for the copy, the
 * copy for the work queued on `stream` before the previous upload). */
fg_status fg_ragged_attention(const fg_kv_cache* cache, fg_ragged_batch* batch, const void* q_rot,
                              void* out, int32_t n_q_heads, float softmax_scale,
                              int32_t sliding_window, void* stream);

/* Steps 1 to 3 in one call: fg_rotary_kv_append followed by
 * fg_ragged_attention, with the rotation of the queries that the query-tile
 * (prefill) kernel serves moved into that kernel's load of Q. Those Q rows
 * are read unrotated from q and rotated in shared memory with the same exact
 * arithmetic and table, so the rotated Q never makes a round trip through
 * HBM (the rotation of "DeepSpeed-FastGen — paper by Holmes et al. (2024)",
 * Key points, as in fg_rotary_kv_append; the attention as in
 * fg_ragged_attention). q: device [T][n_q_heads][d], not modified; k, v:
 * device [T][Hkv][d]; q_rot: device [T][n_q_heads][d], receives the rotated
 * rows of the tokens served by the decode kernels only (the other rows are
 * left as they were); out: device [T][n_q_heads][d]. Every word of out and
 * of the cache equals that of the two calls in sequence. All pointers
 * 16-byte aligned, q_rot distinct from q. Where the query-tile kernel does
 * not serve the batch (a group size it does not take), the call runs the
 * two steps unchanged. Errors, allocation and ordering as the two calls;
 * asynchronous on `stream`. */
fg_status fg_rotary_kv_attention(fg_kv_cache* cache, fg_ragged_batch* batch, const void* q, const void* k,
                                 const void* v, void* q_rot, void* out, int32_t n_q_heads,
                                 double rope_theta, float softmax_scale, int32_t sliding_window,
                                 void* stream);

/* The same pass as fg_ragged_attention, for callers that must not allocate.
 * The pages have no counterpart: this is a library convenience. Some callers
 * cannot call cudaMalloc (or cudaMallocAsync / cudaFree, or a framework
 * allocator) when the pass runs: a server that reserved all of HBM for the KV
 * pool up front, code under an allocation policy that forbids device
 * allocation inside a step, or a host framework that owns device memory
 * itself. This entry point allocates nothing, on the device or pinned on the
 * host. Its split-KV workspace and its work plan live in two fixed arrays in
 * the library's device image (8 Mi floats = 32 MiB and 4 MiB), which every
 * GPU that loads the library holds until the process exits.
 *   - Limits: a pass whose split partials need more than 8 Mi floats
 *     (partial rows * (head_dim + 2)) or whose work plan exceeds 4 MiB
 *     returns FG_ERR_CAPACITY before any launch.
 *   - First use on a device: the call looks up the arrays' device addresses
 *     (cudaGetSymbolAddress, with that device current). Make that first call
 *     before any stream capture.
 *   - The plan is sent with a copy from ordinary (pageable) host memory, so
 *     the call may wait for work already queued on `stream`.
 *   - The arrays are shared by every call in the process and keep the last
 *     call's contents; nothing in them needs to start at zero (each call
 *     writes every value it reads). Calls whose device work overlaps (two
 *     streams, or two threads) race on the arrays: serialise them.
 * Arguments, layouts and errors are those of fg_ragged_attention. */
fg_status fg_ragged_attention_noalloc(const fg_kv_cache* cache, fg_ragged_batch* batch,
                                      const void* q_rot, void* out, int32_t n_q_heads,
                                      float softmax_scale, int32_t sliding_window, void* stream);

/* ------------------------------------------------------------------------ */
/* After step 3: the layer's output projection                               */
/* ------------------------------------------------------------------------ */

/* y = attn_out w_o^T for the batch's T tokens: attn_out device
 * [T][in_features] bf16 (the attention output [T][n_q_heads][d] viewed as
 * rows of n_q_heads * d), w_o device [out_features][in_features] bf16 (the
 * layout of a linear layer's weight), y device [T][out_features] bf16. Each
 * output is the fp32-accumulated sum rounded once to bf16 (ties to even), as
 * a linear layer with bf16 output returns it; fp32 sums in another order can
 * round a value to the neighbouring bf16 of the exact sum's rounding. The
 * pages run whole transformer layers (Key points); this is the GEMM that
 * follows the attention in each of them. in_features and out_features must
 * be positive multiples of 64 (FG_ERR_UNSUPPORTED); the pointers 16-byte
 * aligned (FG_ERR_INVALID_ARG). The batch must hold a valid put (its T is
 * used; nothing else). Asynchronous on `stream`; allocates nothing. */
fg_status fg_output_projection(const fg_ragged_batch* batch, const void* attn_out, const void* w_o,
                               int32_t in_features, int32_t out_features, void* y, void* stream);

/* Work plan of the batch's last fg_ragged_attention call, for profiling:
 * info[0] = general-path units, info[1] = split-KV decode units,
 * info[2] = tensor-core units, info[3] = combine groups, info[4] = partial
 * rows in the split workspace, info[5] = kernels launched by that call,
 * info[6..7] = 0. */
fg_status fg_attention_plan_info(const fg_ragged_batch* batch, int32_t info[8]);

/* The work plan fg_ragged_attention would use for a batch of these lengths,
 * built on the host alone (no device, no handle), for tests and tooling.
 * q_lens / ctx_lens: host arrays of n_seqs entries (q >= 1, ctx >= 0);
 * group = n_q_heads / n_kv_heads; head_dim 64 or 128; window 0 = none;
 * use_tc != 0: the tensor-core kernels serve the batch (group a power of two
 * <= 128, as fg_ragged_attention decides when the cache's tensor map can be
 * built); slots: CTAs of the persistent query-tile kernel (the SM count).
 * counts[0..6] = general, decode, query-tile and keys-as-rows decode units,
 * combine groups, partial rows, largest combine row count; counts[7..10] =
 * byte offsets of the decode, query-tile, keys-as-rows and combine lists in
 * the packed plan (the general list starts at 0); counts[11] = packed bytes.
 * With out != NULL and out_bytes >= counts[11] the packed plan is copied to
 * out: lists of 32-byte units (int32 seq, kv_head, tok_begin, n_tok,
 * key_begin, key_end, part, n_rows; part -1 = final output, else the first
 * partial row) and 32-byte combine groups (int32 seq, kv_head, tok_begin,
 * n_tok, part_base, n_splits, n_rows, pad); FG_ERR_CAPACITY when out_bytes
 * is too small. */
fg_status fg_plan_describe(const int32_t* q_lens, const int32_t* ctx_lens, int32_t n_seqs, int32_t n_kv_heads,
                           int32_t group, int32_t head_dim, int32_t window, int32_t use_tc, int32_t slots,
                           void* out, size_t out_bytes, int64_t counts[12]);

/* Kernel timing for profiling. With `enable` != 0, each later
 * fg_ragged_attention call on this batch records CUDA events around its
 * kernels, on the streams they run on; fg_attention_kernel_ms then waits for
 * the last call's events and returns the duration in milliseconds of
 * ms[0] = MHA split-KV decode kernel, ms[1] = tensor-core kernel,
 * ms[2] = general-path kernel, ms[3] = combine kernel (0 where a kernel did
 * not run). Off by default. */
fg_status fg_ragged_batch_set_timing(fg_ragged_batch* batch, int32_t enable);
fg_status fg_attention_kernel_ms(fg_ragged_batch* batch, float ms[4]);

/* Host time spent inside this batch's calls, in microseconds, accumulated
 * since the last reset: out[0] fg_ragged_batch_put in total, out[1] its
 * validation, out[2] its wait for a free staging buffer, out[3]
 * fg_ragged_attention in total, out[4] work planning, out[5] the wait for a
 * free plan staging buffer, out[6] tensor-map encoding, out[7] kernel
 * launches. reset != 0 zeroes the counters after reading them. */
fg_status fg_host_profile_us(fg_ragged_batch* batch, double out[8], int32_t reset);

/* Scheduling of one attention call that has both one-token decodes (d = 128,
 * on the tensor-core decode kernel) and prompt-chunk query tiles.
 * enable == 0 (default): the query-tile kernel, then the decode kernel (its
 * CTAs take SMs as the query-tile CTAs leave), then the combine, on the
 * caller's stream. enable != 0: the two kernels run side by side, the query
 * tiles on a second, high-priority stream: a cost model picks K, the
 * query-tile kernel takes the SMs with id < K and the decode kernel the
 * rest, and decode CTAs move onto the first K SMs once every query tile has
 * been claimed; when the model predicts no gain the call runs as with
 * enable == 0. On a B200 the default is faster on the measured batches (the
 * decode kernel needs nearly every SM to reach HBM speed). Results are
 * identical either way. */
fg_status fg_ragged_batch_set_overlap(fg_ragged_batch* batch, int32_t enable);

/* Reads (and clears) the batch's device error word after synchronising
 * `stream`: FG_OK, or FG_ERR_DEVICE_CHECK if a kernel met an index outside
 * its buffers (the access was skipped), or FG_ERR_TIMEOUT. */
fg_status fg_device_status(fg_ragged_batch* batch, void* stream);

/* Self-test of the bounded waits the kernels use instead of unbounded spins:
 * launches one CTA that waits, with a limit of `limit_cycles` SM clocks, on
 * an mbarrier nothing will ever complete, then reads the status the CTA
 * wrote. Returns FG_ERR_TIMEOUT when the wait gave up as designed (the
 * expected result), FG_ERR_DEVICE_CHECK if it did not, FG_ERR_CUDA on a
 * runtime error. Synchronises `stream`. No device fault is involved. */
fg_status fg_selftest_bounded_wait(int64_t limit_cycles, void* stream);

/* ------------------------------------------------------------------------ */
/* Host-only helpers                                                          */
/* ------------------------------------------------------------------------ */

/* The float cos/sin table rotary uses, for positions pos_begin ..
 * pos_begin + n_pos - 1: cos_out/sin_out are host float [n_pos][head_dim/2].
 * No device needed. */
fg_status fg_rotary_table(double rope_theta, int32_t head_dim, int32_t pos_begin, int32_t n_pos,
                          float* cos_out, float* sin_out);

const char* fg_status_string(fg_status status);
const char* fg_last_error(void);

#ifdef __cplusplus
}
#endif
#endif /* FG_H_ */
