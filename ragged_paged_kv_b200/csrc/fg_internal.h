// Internal declarations shared by the host library and the CUDA kernels.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <atomic>
#include <cstdint>

namespace fg {

// One-time launch set-up (cudaFuncSetAttribute and the like) per device:
// such attributes apply to the device that is current when they are set, so
// a process that drives several GPUs must set them on each. run(f) calls f
// with the device current unless it already succeeded there; an ordinal
// beyond the table runs f every time.
struct PerDeviceOnce {
  static constexpr int kMaxDevices = 64;
  std::atomic<bool> done[kMaxDevices];
  template <class F>
  cudaError_t run(F&& f) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= kMaxDevices) return f();
    if (done[dev].load(std::memory_order_acquire)) return cudaSuccess;
    e = f();
    if (e == cudaSuccess) done[dev].store(true, std::memory_order_release);
    return e;
  }
};

// Device error word bits (read back by fg_device_status).
enum : int32_t { kErrBadBlock = 1, kErrBadIndex = 2, kErrTimeout = 4 };

// One attention work unit: the query rows of `n_tok` consecutive new tokens
// of sequence `seq` (all q heads of kv head `kv_head`), against the cached
// key positions [key_begin, key_end). Query row r of the unit is token
// tok_begin + r / g, q head kv_head * g + r % g.
struct WorkItem {
  int32_t seq;
  int32_t kv_head;
  int32_t tok_begin;  // index within the sequence's new tokens
  int32_t n_tok;
  int32_t key_begin;  // absolute position, inclusive
  int32_t key_end;    // absolute position, exclusive
  int32_t part;       // -1: write the normalised bf16 output; else first partial row
  int32_t n_rows;     // n_tok * g
};

// Rows whose key range was split: `n_splits` partials of n_rows rows each,
// split i's row r at partial row part_base + i * n_rows + r.
struct CombineItem {
  int32_t seq;
  int32_t kv_head;
  int32_t tok_begin;
  int32_t n_tok;
  int32_t part_base;
  int32_t n_splits;
  int32_t n_rows;
  int32_t pad;
};

struct CacheView {
  __nv_bfloat16* base;
  int32_t n_blocks;
  int32_t n_kv_heads;
  int32_t block_size;
  int32_t head_dim;
};

struct BatchView {
  const int32_t* cu_q;     // [S + 1] first batch row of each sequence
  const int32_t* ctx;      // [S] cached tokens before this pass
  const int32_t* bt_off;   // [S + 1] CSR offsets into bt
  const int32_t* bt;       // physical block ids, logical order per sequence
  const int32_t* tok_seq;  // [T] sequence index of each batch row
  const int32_t* tok_pos;  // [T] absolute position of each batch row (ctx + index in its sequence)
  const int32_t* tok_blk;  // [T] physical block holding that position's cache slot
  int32_t n_seqs;
  int32_t n_tokens;
  int32_t* err;            // device error word
};

// Offset in bf16 words of (block, kv, head, slot, dim 0) in the cache.
__host__ __device__ inline int64_t cache_offset(const CacheView& c, int64_t blk, int kv, int head,
                                                int slot) {
  return (((blk * 2 + kv) * c.n_kv_heads + head) * (int64_t)c.block_size + slot) *
         (int64_t)c.head_dim;
}

cudaError_t launch_rotary_append(const CacheView& cache, const BatchView& batch,
                                 const __nv_bfloat16* q, const __nv_bfloat16* k,
                                 const __nv_bfloat16* v, __nv_bfloat16* q_rot, const double2* rope,
                                 int n_q_heads, bool rotate, cudaStream_t stream, int skip_tc_q = 0);

cudaError_t launch_attention_general(const CacheView& cache, const BatchView& batch,
                                     const WorkItem* items, int n_items,
                                     const __nv_bfloat16* q_rot, __nv_bfloat16* out,
                                     float* part_o, float* part_ml, int n_q_heads, int g,
                                     float scale_log2, int window, cudaStream_t stream);

cudaError_t launch_attention_decode(const CacheView& cache, const BatchView& batch,
                                    const WorkItem* items, int n_items,
                                    const __nv_bfloat16* q_rot, __nv_bfloat16* out, float* part_o,
                                    float* part_ml, int n_q_heads, float scale_log2,
                                    cudaStream_t stream);

// tm_q / tm_kv point to CUtensorMap objects (host memory, passed by value).
// The persistent tensor-core kernels take their units from *counter, which
// must be zero when the kernel starts. With rope != nullptr the query-tile
// kernel reads Q unrotated (tm_q over q) and rotates it in shared memory
// with that table (the rotary kernel's table, times 2^896).
cudaError_t launch_attention_tc(const void* tm_q, const void* tm_kv, const CacheView& cache,
                                const BatchView& batch, const WorkItem* items, int n_items,
                                __nv_bfloat16* out, float* part_o, float* part_ml, int n_q_heads,
                                int g, float scale_log2, int window, int grid, int sm_end,
                                int* counter, cudaStream_t stream, const double2* rope = nullptr);

// Grouped (or MHA) one-token decode on tensor cores, keys as MMA rows;
// tm_q1 views q_rot with boxes of 64 dims x g heads x 1 token. d = 128.
cudaError_t launch_attention_decode_tc(const void* tm_q1, const void* tm_kv, const CacheView& cache,
                                       const BatchView& batch, const WorkItem* items, int n_items,
                                       __nv_bfloat16* out, float* part_o, float* part_ml, int n_q_heads,
                                       int g, float scale_log2, int grid, int* counter,
                                       int sm_tc_end, const int* tc_counter, int n_tc, bool pdl,
                                       cudaStream_t stream);

// persistent: the 128 x 256 tile form (one CTA per SM, two TMEM
// accumulators; the output width (n_q_heads + 2 Hkv) d a multiple of 256,
// tm_w with 64 x 256 boxes); otherwise one 128-token x d tile per CTA
// (tm_w with 64 x d boxes). tm_x has 64 x 128 boxes.
cudaError_t launch_qkv_rotary_append(const void* tm_x, const void* tm_w, const CacheView& cache,
                                     const BatchView& batch, __nv_bfloat16* q_rot, const double2* rope,
                                     int n_q_heads, int hidden, cudaStream_t stream, bool persistent);

// y[T][n_out] = x[T][k_len] w[n_out][k_len]^T in bf16 with fp32 accumulation
// (the layer's output projection); T = batch.n_tokens, n_tile (64 or 128)
// output features per CTA, or 256: the persistent 128 x 256 tile form;
// tm_x / tm_w 2-D maps with 64 x 128 and 64 x n_tile boxes.
cudaError_t launch_linear_bf16(const void* tm_x, const void* tm_w, const BatchView& batch, __nv_bfloat16* y,
                               int k_len, int n_out, int n_tile, cudaStream_t stream);

cudaError_t launch_combine(const BatchView& batch, const CombineItem* items, int n_items,
                           int max_rows, const float* part_o, const float* part_ml,
                           __nv_bfloat16* out, int n_q_heads, int g, int head_dim, bool pdl,
                           cudaStream_t stream);

}  // namespace fg
