// Host side of libfg: handles, argument validation, batch metadata packing,
// the rotary cos/sin table, work planning and kernel launch sequencing.
//
// Everything the kernels need about a ragged batch is packed by
// fg_ragged_batch_put into one int32 buffer and sent with a single
// asynchronous host-to-device copy; fg_ragged_attention plans its work units
// on the host (integer work only) and sends them the same way.
#include <algorithm>
#include <chrono>
#include <climits>
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <string>
#include <vector>

#include <cuda.h>
#include <cudaTypedefs.h>

#include "../../include/fg.h"
#include "fg_internal.h"
#include "fg_plan.h"

using fg::BatchView;
using fg::CacheView;
using fg::CombineItem;
using fg::WorkItem;

namespace {

thread_local std::string g_last_error;

fg_status fail(fg_status st, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof(buf), fmt, ap);
  va_end(ap);
  g_last_error = buf;
  return st;
}

fg_status cuda_fail(cudaError_t e, const char* what) {
  return fail(FG_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

#define FG_CUDA(call)                                   \
  do {                                                  \
    cudaError_t e_ = (call);                            \
    if (e_ != cudaSuccess) return cuda_fail(e_, #call); \
  } while (0)

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

double now_us() {
  return std::chrono::duration<double, std::micro>(std::chrono::steady_clock::now().time_since_epoch())
      .count();
}

// A pinned host staging area with two halves used in turn; before a half is
// rewritten the host waits for the copy that last read it.
struct Staging {
  void* host[2] = {nullptr, nullptr};
  size_t bytes = 0;
  cudaEvent_t done[2] = {nullptr, nullptr};
  bool pending[2] = {false, false};
  int next = 0;

  fg_status reserve(size_t need) {
    if (need <= bytes) return FG_OK;
    for (int i = 0; i < 2; ++i) {
      if (pending[i]) FG_CUDA(cudaEventSynchronize(done[i]));
      pending[i] = false;
      if (host[i]) cudaFreeHost(host[i]);
      host[i] = nullptr;
    }
    size_t cap = std::max<size_t>(need, 4096);
    for (int i = 0; i < 2; ++i) {
      FG_CUDA(cudaHostAlloc(&host[i], cap, cudaHostAllocDefault));
      if (!done[i]) FG_CUDA(cudaEventCreateWithFlags(&done[i], cudaEventDisableTiming));
    }
    bytes = cap;
    return FG_OK;
  }
  // Returns a half that is free to write.
  fg_status acquire(void** out, int* idx) {
    const int i = next;
    if (pending[i]) FG_CUDA(cudaEventSynchronize(done[i]));
    pending[i] = false;
    *out = host[i];
    *idx = i;
    next ^= 1;
    return FG_OK;
  }
  fg_status copy(int i, void* dst, size_t n, cudaStream_t st) {
    if (n) FG_CUDA(cudaMemcpyAsync(dst, host[i], n, cudaMemcpyHostToDevice, st));
    FG_CUDA(cudaEventRecord(done[i], st));
    pending[i] = true;
    return FG_OK;
  }
  void release() {
    for (int i = 0; i < 2; ++i) {
      if (pending[i]) cudaEventSynchronize(done[i]);
      if (host[i]) cudaFreeHost(host[i]);
      if (done[i]) cudaEventDestroy(done[i]);
      host[i] = nullptr;
      done[i] = nullptr;
    }
  }
};

// A device buffer with two halves used in turn by successive uploads, so
// that the upload of the next pass's data (on the handle's copy stream) runs
// while the device still works on the current pass. rel[i] marks, on the
// caller's stream, the end of the work queued while half i was current;
// ready[i] the end of the copy into it, which the caller's stream waits for.
struct DevDouble {
  void* buf[2] = {nullptr, nullptr};
  size_t cap[2] = {0, 0};
  cudaEvent_t rel[2] = {nullptr, nullptr};
  cudaEvent_t ready[2] = {nullptr, nullptr};
  bool rel_set[2] = {false, false};
  int cur = -1;

  // Makes the other half current-to-be: sized for `need` bytes (grown on
  // `strm` with stream-ordered allocation, or with cudaMalloc when `sync`),
  // and `copy` ordered after the last use of it. Returns its index.
  fg_status begin(size_t need, bool sync, cudaStream_t strm, cudaStream_t copy, int* out) {
    for (int i = 0; i < 2; ++i) {
      if (!rel[i]) FG_CUDA(cudaEventCreateWithFlags(&rel[i], cudaEventDisableTiming));
      if (!ready[i]) FG_CUDA(cudaEventCreateWithFlags(&ready[i], cudaEventDisableTiming));
    }
    if (cur >= 0) {
      FG_CUDA(cudaEventRecord(rel[cur], strm));
      rel_set[cur] = true;
    }
    const int i = cur < 0 ? 0 : cur ^ 1;
    if (need > cap[i]) {
      const size_t c = sync ? need : std::max<size_t>(need + need / 2, 1 << 16);
      if (sync) {
        if (buf[i]) FG_CUDA(cudaFree(buf[i]));
        buf[i] = nullptr;
        FG_CUDA(cudaMalloc(&buf[i], c));
      } else {
        if (buf[i]) FG_CUDA(cudaFreeAsync(buf[i], strm));
        buf[i] = nullptr;
        FG_CUDA(cudaMallocAsync(&buf[i], c, strm));
        FG_CUDA(cudaEventRecord(rel[i], strm));
        rel_set[i] = true;
      }
      cap[i] = c;
    }
    if (rel_set[i]) FG_CUDA(cudaStreamWaitEvent(copy, rel[i], 0));
    *out = i;
    return FG_OK;
  }
  // The copy into half i is queued on `copy`: make it current and order
  // `strm` after the copy.
  fg_status commit(int i, cudaStream_t strm, cudaStream_t copy) {
    FG_CUDA(cudaEventRecord(ready[i], copy));
    FG_CUDA(cudaStreamWaitEvent(strm, ready[i], 0));
    cur = i;
    return FG_OK;
  }
  void* current() const { return cur < 0 ? nullptr : buf[cur]; }
  // Call with the device idle.
  void release() {
    for (int i = 0; i < 2; ++i) {
      if (buf[i]) cudaFree(buf[i]);
      if (rel[i]) cudaEventDestroy(rel[i]);
      if (ready[i]) cudaEventDestroy(ready[i]);
      buf[i] = nullptr;
      rel[i] = ready[i] = nullptr;
      cap[i] = 0;
    }
    cur = -1;
  }
};

}  // namespace

struct fg_kv_cache {
  int32_t block_size = 0, n_blocks = 0, n_kv_heads = 0, head_dim = 0;
  void* base = nullptr;
  size_t bytes = 0;
  bool owned = false;
  int device = 0;
  // rotary table [rope_npos][head_dim / 2] of (cos, sin): the float-rounded
  // values, widened to double and scaled by 2^896; within a position row,
  // pair i = 8 g + e sits at entry e * (head_dim / 16) + g (the order the
  // kernel's threads read it in)
  double rope_theta = 0.0;
  int32_t rope_npos = 0;
  double2* rope = nullptr;
  // TMA view of the pool: 2-D (head_dim, every slot row), 64 x min(B, 64) boxes
  alignas(64) CUtensorMap tm_kv;
  int tm_kv_state = 0;  // 0 = not built, 1 = built, -1 = unavailable
};

struct fg_ragged_batch {
  int32_t max_tokens = 0, max_seqs = 0, max_blocks_per_seq = 0;
  int device = -1;
  // device metadata (two halves, see DevDouble) + error word; the uploads of
  // metadata and plan run on `copy`
  DevDouble meta;
  size_t dmeta_words = 0;
  int32_t* derr = nullptr;
  cudaStream_t copy = nullptr;
  // The persistent kernels' next-unit counters sit in the 256 bytes after
  // the plan in the plan buffer; an upload of a new plan zeroes them too
  // (ctr_fresh), otherwise a memset does before the kernels run.
  bool ctr_fresh = false;
  Staging meta_stage;
  // last put
  const fg_kv_cache* cache = nullptr;
  uint64_t put_gen = 0;
  int32_t n_seqs = 0, n_tokens = 0, max_pos = -1;
  std::vector<int32_t> q_lens, ctx_lens;
  BatchView view{};
  // alias-check scratch, indexed by block id
  std::vector<uint64_t> stamp;
  std::vector<int32_t> head;
  // attention plan
  fg::Plan plan;
  uint64_t plan_key[4] = {~0ull, 0, 0, 0};
  DevDouble dplan;
  Staging plan_stage;
  int32_t last_launches = 0;
  // second stream: tensor-core tiles run beside the decode kernel
  cudaStream_t aux = nullptr;
  cudaEvent_t fork = nullptr, join = nullptr;
  // optional kernel timing: begin/end events of decode, tc, general, combine
  bool overlap = false;
  bool timing = false;
  cudaEvent_t tev[8] = {};
  bool tran[4] = {};
  // host-time profile (microseconds, accumulated): put, validation, put
  // staging wait, attention, planning, plan staging wait, tensor maps, calls
  double hprof[8] = {};
  // split-KV partials
  float* ws = nullptr;
  size_t ws_bytes = 0;
};

// ---------------------------------------------------------------------------
// rotary table
// ---------------------------------------------------------------------------
static void build_rope_rows(double theta, int d, int p0, int n, float* c, float* s, int ld) {
  const int half = d / 2;
  std::vector<double> inv(half);
  for (int i = 0; i < half; ++i) inv[i] = 1.0 / std::pow(theta, (2.0 * i) / (double)d);
  for (int r = 0; r < n; ++r) {
    const double p = (double)(p0 + r);
    for (int i = 0; i < half; ++i) {
      const double a = p * inv[i];
      c[(size_t)r * ld + i] = (float)std::cos(a);
      s[(size_t)r * ld + i] = (float)std::sin(a);
    }
  }
}

extern "C" fg_status fg_rotary_table(double rope_theta, int32_t head_dim, int32_t pos_begin,
                                     int32_t n_pos, float* cos_out, float* sin_out) {
  if (!(rope_theta > 0.0) || head_dim <= 0 || (head_dim & 1) || pos_begin < 0 || n_pos < 0 ||
      (n_pos > 0 && (!cos_out || !sin_out)))
    return fail(FG_ERR_INVALID_ARG, "fg_rotary_table: bad argument");
  build_rope_rows(rope_theta, head_dim, pos_begin, n_pos, cos_out, sin_out, head_dim / 2);
  return FG_OK;
}

static fg_status ensure_rope(fg_kv_cache* c, double theta, int32_t max_pos) {
  if (c->rope && c->rope_theta == theta && max_pos < c->rope_npos) return FG_OK;
  int64_t need = (int64_t)max_pos + 1;
  int64_t cap = 4096;
  while (cap < need) cap *= 2;
  const int half = c->head_dim / 2;
  std::vector<float> cs((size_t)cap * half), sn((size_t)cap * half);
  build_rope_rows(theta, c->head_dim, 0, (int)cap, cs.data(), sn.data(), half);
  std::vector<double2> tab((size_t)cap * half);
  // stored times 2^896 (exact): the kernel widens bf16 inputs to doubles
  // that are 2^-896 times their value, and the two scalings cancel in
  // every product
  const int groups = half / 8;
  for (int64_t p = 0; p < cap; ++p)
    for (int i = 0; i < half; ++i) {
      const size_t src = (size_t)p * half + i;
      tab[(size_t)p * half + (i % 8) * groups + i / 8] =
          make_double2(std::ldexp((double)cs[src], 896), std::ldexp((double)sn[src], 896));
    }
  double2* dnew = nullptr;
  FG_CUDA(cudaMalloc(&dnew, tab.size() * sizeof(double2)));
  cudaError_t e = cudaMemcpy(dnew, tab.data(), tab.size() * sizeof(double2), cudaMemcpyHostToDevice);
  if (e != cudaSuccess) {
    cudaFree(dnew);
    return cuda_fail(e, "rotary table upload");
  }
  if (c->rope) {
    FG_CUDA(cudaDeviceSynchronize());  // earlier launches may still read the old table
    cudaFree(c->rope);
  }
  c->rope = dnew;
  c->rope_npos = (int32_t)cap;
  c->rope_theta = theta;
  return FG_OK;
}

// ---------------------------------------------------------------------------
// cache
// ---------------------------------------------------------------------------
static fg_status check_cache_shape(int32_t B, int32_t nb, int32_t hkv, int32_t d) {
  if (nb < 1 || hkv < 1) return fail(FG_ERR_INVALID_ARG, "n_blocks and n_kv_heads must be >= 1");
  if (hkv > 256) return fail(FG_ERR_UNSUPPORTED, "n_kv_heads %d > 256", hkv);
  if (d != 64 && d != 128) return fail(FG_ERR_UNSUPPORTED, "head_dim %d not in {64, 128}", d);
  if (B != 16 && B != 32 && B != 64 && B != 128)
    return fail(FG_ERR_UNSUPPORTED, "block_size %d not in {16, 32, 64, 128}", B);
  return FG_OK;
}

static size_t cache_bytes(int32_t B, int32_t nb, int32_t hkv, int32_t d) {
  return (size_t)nb * 2 * (size_t)hkv * (size_t)B * (size_t)d * 2;
}

extern "C" fg_status fg_kv_cache_create(int32_t block_size, int32_t n_blocks, int32_t n_kv_heads,
                                        int32_t head_dim, fg_kv_cache** out) {
  if (!out) return fail(FG_ERR_INVALID_ARG, "out is NULL");
  *out = nullptr;
  fg_status st = check_cache_shape(block_size, n_blocks, n_kv_heads, head_dim);
  if (st) return st;
  auto* c = new fg_kv_cache;
  c->block_size = block_size;
  c->n_blocks = n_blocks;
  c->n_kv_heads = n_kv_heads;
  c->head_dim = head_dim;
  c->bytes = cache_bytes(block_size, n_blocks, n_kv_heads, head_dim);
  c->owned = true;
  cudaError_t e = cudaGetDevice(&c->device);
  if (e == cudaSuccess) e = cudaMalloc(&c->base, c->bytes);
  if (e != cudaSuccess) {
    delete c;
    return cuda_fail(e, "fg_kv_cache_create: cudaMalloc of the block pool");
  }
  *out = c;
  return FG_OK;
}

extern "C" fg_status fg_kv_cache_create_external(int32_t block_size, int32_t n_blocks,
                                                 int32_t n_kv_heads, int32_t head_dim,
                                                 void* dev_ptr, size_t bytes, fg_kv_cache** out) {
  if (!out) return fail(FG_ERR_INVALID_ARG, "out is NULL");
  *out = nullptr;
  fg_status st = check_cache_shape(block_size, n_blocks, n_kv_heads, head_dim);
  if (st) return st;
  if (!dev_ptr || !aligned16(dev_ptr))
    return fail(FG_ERR_INVALID_ARG, "dev_ptr must be a 16-byte aligned device pointer");
  const size_t need = cache_bytes(block_size, n_blocks, n_kv_heads, head_dim);
  if (bytes < need)
    return fail(FG_ERR_CAPACITY, "external cache has %zu bytes, layout needs %zu", bytes, need);
  auto* c = new fg_kv_cache;
  c->block_size = block_size;
  c->n_blocks = n_blocks;
  c->n_kv_heads = n_kv_heads;
  c->head_dim = head_dim;
  c->bytes = need;
  c->base = dev_ptr;
  c->owned = false;
  if (cudaGetDevice(&c->device) != cudaSuccess) c->device = -1;
  *out = c;
  return FG_OK;
}

extern "C" fg_status fg_kv_cache_layout(const fg_kv_cache* c, void** base, int64_t strides[5]) {
  if (!c || !base || !strides) return fail(FG_ERR_INVALID_ARG, "NULL argument");
  *base = c->base;
  strides[4] = 1;
  strides[3] = c->head_dim;
  strides[2] = (int64_t)c->block_size * c->head_dim;
  strides[1] = strides[2] * c->n_kv_heads;
  strides[0] = strides[1] * 2;
  return FG_OK;
}

extern "C" fg_status fg_kv_cache_prepare_rotary(fg_kv_cache* c, double rope_theta, int32_t max_position) {
  if (!c) return fail(FG_ERR_INVALID_ARG, "cache is NULL");
  if (!(rope_theta > 0.0)) return fail(FG_ERR_INVALID_ARG, "rope_theta must be > 0");
  if (max_position < 0) return fail(FG_ERR_INVALID_ARG, "max_position %d < 0", max_position);
  return ensure_rope(c, rope_theta, max_position);
}

extern "C" fg_status fg_kv_cache_destroy(fg_kv_cache* c) {
  if (!c) return FG_OK;
  if (c->owned || c->rope) cudaDeviceSynchronize();
  if (c->owned && c->base) cudaFree(c->base);
  if (c->rope) cudaFree(c->rope);
  delete c;
  return FG_OK;
}

// ---------------------------------------------------------------------------
// ragged batch
// ---------------------------------------------------------------------------
extern "C" fg_status fg_ragged_batch_create(int32_t max_tokens, int32_t max_seqs,
                                            int32_t max_blocks_per_seq, fg_ragged_batch** out) {
  if (!out) return fail(FG_ERR_INVALID_ARG, "out is NULL");
  *out = nullptr;
  if (max_tokens < 1 || max_seqs < 1 || max_blocks_per_seq < 1)
    return fail(FG_ERR_INVALID_ARG, "capacities must be >= 1");
  if ((int64_t)max_seqs * max_blocks_per_seq > (int64_t)1 << 30)
    return fail(FG_ERR_CAPACITY, "max_seqs * max_blocks_per_seq too large");
  auto* b = new fg_ragged_batch;
  b->max_tokens = max_tokens;
  b->max_seqs = max_seqs;
  b->max_blocks_per_seq = max_blocks_per_seq;
  *out = b;
  return FG_OK;
}

extern "C" fg_status fg_ragged_batch_destroy(fg_ragged_batch* b) {
  if (!b) return FG_OK;
  if (b->derr || b->dplan.cur >= 0 || b->ws) cudaDeviceSynchronize();
  b->meta_stage.release();
  b->plan_stage.release();
  b->meta.release();
  b->dplan.release();
  if (b->derr) cudaFree(b->derr);
  if (b->ws) cudaFree(b->ws);
  if (b->copy) cudaStreamDestroy(b->copy);
  for (cudaEvent_t e : b->tev)
    if (e) cudaEventDestroy(e);
  if (b->aux) cudaStreamDestroy(b->aux);
  if (b->fork) cudaEventDestroy(b->fork);
  if (b->join) cudaEventDestroy(b->join);
  delete b;
  return FG_OK;
}

extern "C" fg_status fg_ragged_batch_shape(const fg_ragged_batch* b, int32_t* n_tokens,
                                           int32_t* n_seqs) {
  if (!b) return fail(FG_ERR_INVALID_ARG, "batch is NULL");
  if (n_tokens) *n_tokens = b->n_tokens;
  if (n_seqs) *n_seqs = b->n_seqs;
  return FG_OK;
}

namespace {

// Every check of fg_ragged_batch_put that needs no device.
fg_status validate_batch(fg_ragged_batch* b, const fg_kv_cache* c, int32_t S, const int32_t* ids,
                         const int32_t* ql, const int32_t* cl, const int32_t* bt, int32_t stride,
                         int64_t* T_out, int64_t* nblk_out, int32_t* maxpos_out) {
  if (S < 0) return fail(FG_ERR_INVALID_ARG, "n_seqs %d < 0", S);
  if (S > b->max_seqs) return fail(FG_ERR_CAPACITY, "n_seqs %d > max_seqs %d", S, b->max_seqs);
  if (S > 0 && (!ids || !ql || !cl || !bt))
    return fail(FG_ERR_INVALID_ARG, "NULL host array");
  if (S > 0 && stride < 1) return fail(FG_ERR_INVALID_ARG, "block_table_stride %d < 1", stride);
  const int64_t B = c->block_size;
  int64_t T = 0, nblk = 0;
  int32_t maxpos = -1;
  for (int32_t s = 0; s < S; ++s) {
    if (ql[s] < 1) return fail(FG_ERR_INVALID_ARG, "q_lens[%d] = %d < 1", s, ql[s]);
    if (cl[s] < 0) return fail(FG_ERR_INVALID_ARG, "ctx_lens[%d] = %d < 0", s, cl[s]);
    const int64_t L = (int64_t)cl[s] + ql[s];
    if (L > (int64_t)1 << 30) return fail(FG_ERR_CAPACITY, "sequence %d length %lld too long", s, (long long)L);
    const int64_t nb = (L + B - 1) / B;
    if (nb > b->max_blocks_per_seq)
      return fail(FG_ERR_CAPACITY, "sequence %d needs %lld blocks > max_blocks_per_seq %d", s,
                  (long long)nb, b->max_blocks_per_seq);
    if (nb > stride)
      return fail(FG_ERR_INVALID_ARG, "sequence %d needs %lld blocks > block_table_stride %d", s,
                  (long long)nb, stride);
    T += ql[s];
    nblk += nb;
    maxpos = std::max<int32_t>(maxpos, (int32_t)(L - 1));
  }
  if (T > b->max_tokens)
    return fail(FG_ERR_CAPACITY, "%lld tokens > max_tokens %d", (long long)T, b->max_tokens);
  // distinct sequence ids
  {
    std::vector<int32_t> sid(ids, ids + S);
    std::sort(sid.begin(), sid.end());
    for (int32_t i = 1; i < S; ++i)
      if (sid[i] == sid[i - 1]) return fail(FG_ERR_ALIAS, "duplicate seq_id %d", sid[i]);
  }
  // block ids in range; per block, the sequences that use it must not collide:
  // a sequence writing slots [w, used) of a block conflicts with any other
  // sequence touching slots below `used` at or above w.
  struct Use { int32_t seq, used, wlo, next; };
  std::vector<Use> uses;
  uses.reserve((size_t)nblk);
  if (b->stamp.size() != (size_t)c->n_blocks) {
    b->stamp.assign((size_t)c->n_blocks, 0);
    b->head.assign((size_t)c->n_blocks, -1);
  }
  const uint64_t gen = ++b->put_gen;
  for (int32_t s = 0; s < S; ++s) {
    const int64_t L = (int64_t)cl[s] + ql[s];
    const int64_t nb = (L + B - 1) / B;
    for (int64_t i = 0; i < nb; ++i) {
      const int32_t blk = bt[(int64_t)s * stride + i];
      if (blk < 0 || blk >= c->n_blocks)
        return fail(FG_ERR_OUT_OF_RANGE, "block_tables[%d][%lld] = %d outside [0, %d)", s,
                    (long long)i, blk, c->n_blocks);
      const int32_t used = (int32_t)std::min<int64_t>(B, L - i * B);
      const int64_t w0 = std::max<int64_t>(cl[s], i * B) - i * B;  // first written slot
      const int32_t wlo = (int32_t)std::min<int64_t>(w0, used);     // == used: no write
      Use u{s, used, wlo, -1};
      if (b->stamp[blk] == gen) {
        for (int32_t e = b->head[blk]; e >= 0; e = uses[e].next) {
          const Use& o = uses[e];
          if (o.seq == s)
            return fail(FG_ERR_ALIAS, "block %d appears twice in the table of sequence %d", blk, s);
          if ((u.wlo < u.used && o.used > u.wlo) || (o.wlo < o.used && u.used > o.wlo))
            return fail(FG_ERR_ALIAS, "block %d: sequence %d and %d collide on written slots", blk,
                        o.seq, s);
        }
        u.next = b->head[blk];
      } else {
        b->stamp[blk] = gen;
      }
      b->head[blk] = (int32_t)uses.size();
      uses.push_back(u);
    }
  }
  *T_out = T;
  *nblk_out = nblk;
  *maxpos_out = maxpos;
  return FG_OK;
}

}  // namespace

extern "C" fg_status fg_ragged_batch_put(fg_ragged_batch* b, const fg_kv_cache* c, int32_t S,
                                         const int32_t* ids, const int32_t* ql, const int32_t* cl,
                                         const int32_t* bt, int32_t stride, void* stream) {
  if (!b || !c) return fail(FG_ERR_INVALID_ARG, "NULL handle");
  const double t_in = now_us();
  int64_t T = 0, nblk = 0;
  int32_t maxpos = -1;
  fg_status st = validate_batch(b, c, S, ids, ql, cl, bt, stride, &T, &nblk, &maxpos);
  b->hprof[1] += now_us() - t_in;
  if (st) {
    b->cache = nullptr;  // the previous batch is no longer valid either
    return st;
  }
  cudaStream_t strm = static_cast<cudaStream_t>(stream);
  if (!b->derr) {
    b->dmeta_words = 3 * (size_t)b->max_seqs + 2 + 3 * (size_t)b->max_tokens +
                     (size_t)b->max_seqs * b->max_blocks_per_seq;
    FG_CUDA(cudaGetDevice(&b->device));
    if (!b->copy) {
      int lo = 0, hi = 0;
      FG_CUDA(cudaDeviceGetStreamPriorityRange(&lo, &hi));
      FG_CUDA(cudaStreamCreateWithPriority(&b->copy, cudaStreamNonBlocking, hi));
    }
    st = b->meta_stage.reserve(b->dmeta_words * 4);
    if (st) return st;
    FG_CUDA(cudaMalloc(&b->derr, 4));
    FG_CUDA(cudaMemset(b->derr, 0, 4));
  }
  // the half of the device buffer this pass uses; its copy waits for the
  // work queued on `stream` before the previous put (the last pass that read it)
  int half = 0;
  st = b->meta.begin(b->dmeta_words * 4, true, strm, b->copy, &half);
  if (st) return st;
  // pack: cu_q[S+1] ctx[S] bt_off[S+1] tok_seq[T] tok_pos[T] tok_blk[T] bt[nblk]
  // (each row's position and block resolved here, so the append's producer
  // reads them with one load instead of a chain of dependent ones)
  const size_t words = 3 * (size_t)S + 2 + 3 * (size_t)T + (size_t)nblk;
  void* hp = nullptr;
  int slot = 0;
  const double t_w = now_us();
  st = b->meta_stage.acquire(&hp, &slot);
  b->hprof[2] += now_us() - t_w;
  if (st) return st;
  int32_t* h = static_cast<int32_t*>(hp);
  int32_t* cu = h;
  int32_t* cx = cu + S + 1;
  int32_t* bo = cx + S;
  int32_t* ts = bo + S + 1;
  int32_t* tp = ts + T;
  int32_t* tb = tp + T;
  int32_t* bb = tb + T;
  cu[0] = 0;
  bo[0] = 0;
  const int64_t B = c->block_size;
  for (int32_t s = 0; s < S; ++s) {
    cu[s + 1] = cu[s] + ql[s];
    cx[s] = cl[s];
    const int64_t nb = ((int64_t)cl[s] + ql[s] + B - 1) / B;
    bo[s + 1] = bo[s] + (int32_t)nb;
    std::memcpy(bb + bo[s], bt + (int64_t)s * stride, (size_t)nb * 4);
    const int32_t* row = bt + (int64_t)s * stride;
    for (int32_t j = 0; j < ql[s]; ++j) {
      const int32_t pos = cl[s] + j;
      ts[cu[s] + j] = s;
      tp[cu[s] + j] = pos;
      tb[cu[s] + j] = row[pos / B];
    }
  }
  int32_t* d = static_cast<int32_t*>(b->meta.buf[half]);
  st = b->meta_stage.copy(slot, d, words * 4, b->copy);
  if (st) return st;
  st = b->meta.commit(half, strm, b->copy);
  if (st) return st;
  b->hprof[0] += now_us() - t_in;
  b->view.cu_q = d;
  b->view.ctx = d + S + 1;
  b->view.bt_off = d + 2 * S + 1;
  b->view.tok_seq = d + 3 * S + 2;
  b->view.tok_pos = d + 3 * S + 2 + T;
  b->view.tok_blk = d + 3 * S + 2 + 2 * T;
  b->view.bt = d + 3 * S + 2 + 3 * T;
  b->view.n_seqs = S;
  b->view.n_tokens = (int32_t)T;
  b->view.err = b->derr;
  b->q_lens.assign(ql, ql + S);
  b->ctx_lens.assign(cl, cl + S);
  b->n_seqs = S;
  b->n_tokens = (int32_t)T;
  b->max_pos = maxpos;
  b->cache = c;
  return FG_OK;
}

// ---------------------------------------------------------------------------
// forward steps
// ---------------------------------------------------------------------------
static CacheView cache_view(const fg_kv_cache* c) {
  CacheView v;
  v.base = static_cast<__nv_bfloat16*>(c->base);
  v.n_blocks = c->n_blocks;
  v.n_kv_heads = c->n_kv_heads;
  v.block_size = c->block_size;
  v.head_dim = c->head_dim;
  return v;
}

static fg_status check_pass(const fg_kv_cache* c, const fg_ragged_batch* b, int32_t hq) {
  if (!c || !b) return fail(FG_ERR_INVALID_ARG, "NULL handle");
  if (b->cache != c)
    return fail(FG_ERR_INVALID_ARG, "batch was not put against this cache (or its last put failed)");
  if (hq < 1 || hq % c->n_kv_heads)
    return fail(FG_ERR_UNSUPPORTED, "n_q_heads %d is not a multiple of n_kv_heads %d", hq,
                c->n_kv_heads);
  int dev = -1;
  if (cudaGetDevice(&dev) == cudaSuccess && b->device >= 0 && dev != b->device)
    return fail(FG_ERR_INVALID_ARG, "current device %d is not the batch's device %d", dev, b->device);
  return FG_OK;
}

extern "C" fg_status fg_rotary_kv_append(fg_kv_cache* c, const fg_ragged_batch* b, const void* q,
                                         const void* k, const void* v, void* q_rot,
                                         int32_t n_q_heads, double rope_theta, void* stream) {
  fg_status st = check_pass(c, b, n_q_heads);
  if (st) return st;
  if (!(rope_theta > 0.0)) return fail(FG_ERR_INVALID_ARG, "rope_theta must be > 0");
  if (b->n_tokens == 0) return FG_OK;
  if (!q || !k || !v || !q_rot) return fail(FG_ERR_INVALID_ARG, "NULL tensor pointer");
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(q_rot))
    return fail(FG_ERR_INVALID_ARG, "q, k, v and q_rot must be 16-byte aligned");
  st = ensure_rope(c, rope_theta, b->max_pos);
  if (st) return st;
  cudaError_t e = fg::launch_rotary_append(
      cache_view(c), b->view, static_cast<const __nv_bfloat16*>(q),
      static_cast<const __nv_bfloat16*>(k), static_cast<const __nv_bfloat16*>(v),
      static_cast<__nv_bfloat16*>(q_rot), c->rope, n_q_heads, true, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "rotary_append launch");
  return FG_OK;
}

extern "C" fg_status fg_kv_append(fg_kv_cache* c, const fg_ragged_batch* b, const void* k, const void* v,
                                  void* stream) {
  fg_status st = check_pass(c, b, c ? c->n_kv_heads : 1);
  if (st) return st;
  if (b->n_tokens == 0) return FG_OK;
  if (!k || !v) return fail(FG_ERR_INVALID_ARG, "NULL tensor pointer");
  if (!aligned16(k) || !aligned16(v)) return fail(FG_ERR_INVALID_ARG, "k and v must be 16-byte aligned");
  cudaError_t e = fg::launch_rotary_append(cache_view(c), b->view, nullptr, static_cast<const __nv_bfloat16*>(k),
                                           static_cast<const __nv_bfloat16*>(v), nullptr, nullptr, 0, false,
                                           static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "kv_append launch");
  return FG_OK;
}

namespace {

// cuTensorMapEncodeTiled through the runtime's driver entry point (no link
// against libcuda). nullptr if the driver does not provide it.
PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static bool tried = false;
  if (!tried) {
    tried = true;
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q{};
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  }
  return fn;
}

// The pool as a 2-D bf16 tensor: inner dim head_dim, outer dim every slot row
// ((block * 2 + kv) * Hkv + head) * B + slot; boxes of 64 dims x min(B, 64)
// rows, 128-byte swizzle (the layout the tensor-core operands use).
bool ensure_kv_map(fg_kv_cache* c) {
  if (c->tm_kv_state) return c->tm_kv_state > 0;
  c->tm_kv_state = -1;
  auto enc = tensor_map_encoder();
  const uint64_t rows = (uint64_t)c->n_blocks * 2 * c->n_kv_heads * c->block_size;
  if (!enc || rows >= (1ull << 31)) return false;
  cuuint64_t dims[2] = {(cuuint64_t)c->head_dim, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)c->head_dim * 2};
  cuuint32_t box[2] = {64, (cuuint32_t)std::min(c->block_size, 64)};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = enc(&c->tm_kv, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, c->base, dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return false;
  c->tm_kv_state = 1;
  return true;
}

// q_rot as a 3-D bf16 tensor (head_dim, n_q_heads, tokens); a box of
// 64 dims x g heads x 128/g tokens lands as 128 rows (token-major, head-minor)
// of 128 bytes, the A-operand layout of a query tile.
// tokens_per_box = 1 gives the decode kernel's view: g rows of one token.
bool make_q_map(CUtensorMap* m, const void* q_rot, int T, int Hq, int d, int g,
                int tokens_per_box = 0) {
  auto enc = tensor_map_encoder();
  if (!enc) return false;
  cuuint64_t dims[3] = {(cuuint64_t)d, (cuuint64_t)Hq, (cuuint64_t)T};
  cuuint64_t strides[2] = {(cuuint64_t)d * 2, (cuuint64_t)Hq * d * 2};
  cuuint32_t box[3] = {64, (cuuint32_t)g,
                       (cuuint32_t)(tokens_per_box > 0 ? tokens_per_box : fg::kTcRows / g)};
  cuuint32_t estr[3] = {1, 1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(q_rot), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

int sm_count() {
  static int n[64] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 148;
  if (!n[dev] && cudaDeviceGetAttribute(&n[dev], cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
    n[dev] = 148;
  return n[dev];
}

// Side-by-side mode: the query-tile kernel (compute bound) takes the SMs with
// id < K and the tensor-core decode kernel (HBM bound) the rest; decode CTAs
// also move onto the first K SMs once every query tile has been claimed.
// K comes from a small cost model: a 128-row x 64-key tile takes about
// kTileSmUs SM-microseconds (two CTAs per SM), and decode streams about
// kDecodeSmBytesPerUs per SM up to kHbmBytesPerUs in total (measured on B200).
// Returns 0 when running the two kernels one after the other is predicted to
// be as fast.
constexpr double kTileSmUs = 0.75;
constexpr double kDecodeSmBytesPerUs = 52.0e3;
constexpr double kHbmBytesPerUs = 6.4e6;

int tc_share(const fg::Plan& P, int head_dim, int n_sm) {
  if (P.n_tc == 0 || P.n_dtc == 0 || n_sm < 8) return 0;
  double tiles = 0.0, bytes = 0.0;
  for (const WorkItem& w : P.tc)
    tiles += ((w.key_end - (w.key_begin - (w.key_begin & 63)) + 63) / 64) * (w.n_rows > fg::kTcRows ? 2 : 1);
  for (const WorkItem& w : P.dtc) bytes += (double)(w.key_end - w.key_begin) * head_dim * 4.0;
  const double w_tc = tiles * kTileSmUs;
  auto dec = [&](int sms) { return bytes / std::min(kHbmBytesPerUs, sms * kDecodeSmBytesPerUs); };
  const double t_seq = w_tc / n_sm + dec(n_sm);
  int best = 0;
  double t_best = 0.97 * t_seq;
  for (int k = 1; k < n_sm; ++k) {
    const double t = std::max(w_tc / k, dec(n_sm - k));
    if (t < t_best) {
      t_best = t;
      best = k;
    }
  }
  return best;
}

fg_status ensure_aux_stream(fg_ragged_batch* b) {
  if (b->aux) return FG_OK;
  int lo = 0, hi = 0;
  FG_CUDA(cudaDeviceGetStreamPriorityRange(&lo, &hi));
  FG_CUDA(cudaStreamCreateWithPriority(&b->aux, cudaStreamNonBlocking, hi));
  FG_CUDA(cudaEventCreateWithFlags(&b->fork, cudaEventDisableTiming));
  FG_CUDA(cudaEventCreateWithFlags(&b->join, cudaEventDisableTiming));
  return FG_OK;
}

bool tc_eligible(fg_kv_cache* c, int g) {
  const bool pow2 = g >= 1 && g <= fg::kTcRows && (g & (g - 1)) == 0;
  return pow2 && ensure_kv_map(c);
}

// Upload the plan for (g, window) unless the batch's current plan already is.
fg_status prepare_plan(fg_ragged_batch* b, const fg_kv_cache* c, int32_t g, int32_t window,
                       bool use_tc, cudaStream_t strm) {
  const uint64_t key[4] = {b->put_gen, (uint64_t)g, (uint64_t)(uint32_t)window,
                           (uint64_t)c->head_dim | ((uint64_t)use_tc << 32)};
  if (std::equal(key, key + 4, b->plan_key) && b->dplan.current()) return FG_OK;
  const double t_p = now_us();
  fg::build_plan(b->q_lens, b->ctx_lens, c->n_kv_heads, g, c->head_dim, window, use_tc,
                 sm_count(), &b->plan);
  b->hprof[4] += now_us() - t_p;
  const size_t bytes = b->plan.bytes() + 256;  // plan, then the unit counters
  // the other half of the plan buffer, once the last pass that used it is done
  int half = 0;
  fg_status st = b->dplan.begin(bytes, false, strm, b->copy, &half);
  if (st) return st;
  st = b->plan_stage.reserve(b->dplan.cap[half]);
  if (st) return st;
  void* hp = nullptr;
  int slot = 0;
  const double t_w = now_us();
  st = b->plan_stage.acquire(&hp, &slot);
  b->hprof[5] += now_us() - t_w;
  if (st) return st;
  b->plan.pack(hp);
  std::memset(static_cast<char*>(hp) + b->plan.bytes(), 0, 256);
  st = b->plan_stage.copy(slot, b->dplan.buf[half], bytes, b->copy);
  if (st) return st;
  st = b->dplan.commit(half, strm, b->copy);
  if (st) return st;
  b->ctr_fresh = true;
  std::copy(key, key + 4, b->plan_key);
  return FG_OK;
}

fg_status ensure_workspace(fg_ragged_batch* b, size_t floats, cudaStream_t strm) {
  const size_t bytes = floats * 4;
  if (bytes <= b->ws_bytes) return FG_OK;
  if (b->ws) FG_CUDA(cudaFreeAsync(b->ws, strm));
  b->ws = nullptr;
  const size_t cap = std::max<size_t>(bytes + bytes / 4, 1 << 20);
  FG_CUDA(cudaMallocAsync(&b->ws, cap, strm));
  b->ws_bytes = cap;
  return FG_OK;
}

}  // namespace

// Where an attention pass keeps its split workspace and its work plan when
// the caller supplies them (the allocation-free entry point): `ws` holds
// ws_floats floats, `plan_dev` plan_bytes bytes whose last 256 bytes hold the
// persistent kernels' unit counters.
struct FixedPassStorage {
  float* ws;
  size_t ws_floats;
  void* plan_dev;
  size_t plan_bytes;
};

fg_status fg_attention_launch(const fg_kv_cache* c, fg_ragged_batch* b, const void* q_rot, void* out,
                              int32_t n_q_heads, float softmax_scale, int32_t window, cudaStream_t strm,
                              const FixedPassStorage* fixed, const void* q_tc = nullptr);

extern "C" fg_status fg_ragged_attention(const fg_kv_cache* c, fg_ragged_batch* b,
                                         const void* q_rot, void* out, int32_t n_q_heads,
                                         float softmax_scale, int32_t sliding_window,
                                         void* stream) {
  return fg_attention_launch(c, b, q_rot, out, n_q_heads, softmax_scale, sliding_window,
                             static_cast<cudaStream_t>(stream), nullptr);
}

// Rotary + append + attention in one call, with the rotation of the Q rows
// the query-tile kernel serves moved into that kernel's Q load: the rotary
// kernel leaves those rows of q_rot unwritten (and does not read them from
// q), and the query-tile kernel reads them unrotated from q and rotates them
// in shared memory with the same exact arithmetic. Every output and cache
// word equals that of fg_rotary_kv_append followed by fg_ragged_attention.
extern "C" fg_status fg_rotary_kv_attention(fg_kv_cache* c, fg_ragged_batch* b, const void* q,
                                            const void* k, const void* v, void* q_rot, void* out,
                                            int32_t n_q_heads, double rope_theta, float softmax_scale,
                                            int32_t sliding_window, void* stream) {
  fg_status st = check_pass(c, b, n_q_heads);
  if (st) return st;
  if (!(rope_theta > 0.0)) return fail(FG_ERR_INVALID_ARG, "rope_theta must be > 0");
  if (!(softmax_scale > 0.f) || !std::isfinite(softmax_scale))
    return fail(FG_ERR_INVALID_ARG, "softmax_scale must be finite and > 0");
  if (sliding_window < 0) return fail(FG_ERR_INVALID_ARG, "sliding_window %d < 0", sliding_window);
  if (b->n_tokens == 0) return FG_OK;
  if (!q || !k || !v || !q_rot || !out) return fail(FG_ERR_INVALID_ARG, "NULL tensor pointer");
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(q_rot) || !aligned16(out))
    return fail(FG_ERR_INVALID_ARG, "q, k, v, q_rot and out must be 16-byte aligned");
  if (q == q_rot) return fail(FG_ERR_INVALID_ARG, "q_rot must be distinct from q");
  const int32_t g = n_q_heads / c->n_kv_heads;
  const bool fuse = tc_eligible(c, g);
  st = ensure_rope(c, rope_theta, b->max_pos);
  if (st) return st;
  const cudaStream_t strm = static_cast<cudaStream_t>(stream);
  cudaError_t e = fg::launch_rotary_append(
      cache_view(c), b->view, static_cast<const __nv_bfloat16*>(q), static_cast<const __nv_bfloat16*>(k),
      static_cast<const __nv_bfloat16*>(v), static_cast<__nv_bfloat16*>(q_rot), c->rope, n_q_heads, true, strm,
      fuse ? fg::kDtcMaxGroup : 0);
  if (e != cudaSuccess) return cuda_fail(e, "rotary_append launch");
  return fg_attention_launch(c, b, q_rot, out, n_q_heads, softmax_scale, sliding_window, strm, nullptr,
                             fuse ? q : nullptr);
}

// The one launch sequence of both attention entry points. With fixed ==
// nullptr the batch's own workspace and double-buffered plan are used (grown
// with stream-ordered allocation, the plan uploaded from pinned staging on
// the copy stream and cached per batch and shape). Otherwise the plan is
// built into thread-local host memory, sent into fixed->plan_dev with a
// plain copy on `strm`, and the workspace is fixed->ws: nothing is allocated,
// and the batch's own plan cache and workspace are left alone. Only the
// storage differs; the kernels, their order and their arguments are the same.
fg_status fg_attention_launch(const fg_kv_cache* c, fg_ragged_batch* b, const void* q_rot, void* out,
                              int32_t n_q_heads, float softmax_scale, int32_t window, cudaStream_t strm,
                              const FixedPassStorage* fixed, const void* q_tc) {
  fg_status st = check_pass(c, b, n_q_heads);
  if (st) return st;
  if (!(softmax_scale > 0.f) || !std::isfinite(softmax_scale))
    return fail(FG_ERR_INVALID_ARG, "softmax_scale must be finite and > 0");
  if (window < 0) return fail(FG_ERR_INVALID_ARG, "sliding_window %d < 0", window);
  if (b->n_tokens == 0) return FG_OK;
  if (!q_rot || !out) return fail(FG_ERR_INVALID_ARG, "NULL tensor pointer");
  if (!aligned16(q_rot) || !aligned16(out))
    return fail(FG_ERR_INVALID_ARG, "q_rot and out must be 16-byte aligned");
  const int32_t g = n_q_heads / c->n_kv_heads;
  const bool use_tc = tc_eligible(const_cast<fg_kv_cache*>(c), g);
  if (!use_tc && g > fg::kMaxGroup)
    return fail(FG_ERR_UNSUPPORTED, "n_q_heads / n_kv_heads = %d > %d", g, fg::kMaxGroup);
  const double t_a = now_us();
  // q_tc: the query-tile kernel reads Q unrotated from there and rotates it
  // as it loads it (its rows of q_rot are then not needed)
  if (q_tc && !use_tc) return fail(FG_ERR_INVALID_ARG, "rotary-at-load needs the query-tile kernel");
  CUtensorMap tm_q, tm_q1;
  if (use_tc && (!make_q_map(&tm_q, q_tc ? q_tc : q_rot, b->n_tokens, n_q_heads, c->head_dim, g) ||
                 !make_q_map(&tm_q1, q_rot, b->n_tokens, n_q_heads, c->head_dim, g, 1)))
    return fail(FG_ERR_CUDA, "cuTensorMapEncodeTiled failed for q_rot");
  b->hprof[6] += now_us() - t_a;
  const fg::Plan* plan = &b->plan;
  const char* base = nullptr;
  int* ctr = nullptr;  // the persistent kernels' unit counters (zero at launch)
  float* ws = nullptr;
  if (!fixed) {
    st = prepare_plan(b, c, g, window, use_tc, strm);
    if (st) return st;
    base = static_cast<const char*>(b->dplan.current());
    ctr = reinterpret_cast<int*>(static_cast<char*>(b->dplan.current()) + plan->bytes());
    st = ensure_workspace(b, (size_t)plan->part_rows * (c->head_dim + 2), strm);
    if (st) return st;
    ws = b->ws;
  } else {
    thread_local fg::Plan P_fixed;
    thread_local std::vector<unsigned char> packed;
    fg::build_plan(b->q_lens, b->ctx_lens, c->n_kv_heads, g, c->head_dim, window, use_tc, sm_count(), &P_fixed);
    plan = &P_fixed;
    if (P_fixed.bytes() + 256 > fixed->plan_bytes)
      return fail(FG_ERR_CAPACITY, "pass needs a %zu-byte work plan, the fixed area holds %zu", P_fixed.bytes(),
                  fixed->plan_bytes - 256);
    const size_t need = (size_t)P_fixed.part_rows * (c->head_dim + 2);
    if (need > fixed->ws_floats)
      return fail(FG_ERR_CAPACITY, "pass needs %zu split-workspace floats, the fixed area holds %zu", need,
                  fixed->ws_floats);
    packed.resize(P_fixed.bytes());
    P_fixed.pack(packed.data());
    if (!packed.empty())
      FG_CUDA(cudaMemcpyAsync(fixed->plan_dev, packed.data(), packed.size(), cudaMemcpyHostToDevice, strm));
    base = static_cast<const char*>(fixed->plan_dev);
    ctr = reinterpret_cast<int*>(static_cast<char*>(fixed->plan_dev) + fixed->plan_bytes - 256);
    ws = fixed->ws;
  }
  const fg::Plan& P = *plan;
  const double t_l = now_us();
  float* part_o = ws;
  float* part_ml = ws ? ws + (size_t)P.part_rows * c->head_dim : nullptr;
  const float scale_log2 = softmax_scale * 1.4426950408889634f;
  b->last_launches = (P.n_general > 0) + (P.n_decode > 0) + (P.n_tc > 0) + (P.n_dtc > 0) +
                     (P.n_combine > 0);
  const CacheView cv = cache_view(c);
  const auto* qr = static_cast<const __nv_bfloat16*>(q_rot);
  auto* o = static_cast<__nv_bfloat16*>(out);
  // optional timing events around each kernel, on its own stream
  auto mark = [&](int k, int end, cudaStream_t st_) -> fg_status {
    if (!b->timing) return FG_OK;
    FG_CUDA(cudaEventRecord(b->tev[2 * k + end], st_));
    b->tran[k] = true;
    return FG_OK;
  };
  if (b->timing)
    for (bool& r : b->tran) r = false;
  if (P.n_general && (st = mark(2, 0, strm))) return st;
  cudaError_t e = fg::launch_attention_general(
      cv, b->view, reinterpret_cast<const WorkItem*>(base + P.off_general), P.n_general, qr, o,
      part_o, part_ml, n_q_heads, g, scale_log2, window, strm);
  if (e != cudaSuccess) return cuda_fail(e, "attention launch");
  if (P.n_general && (st = mark(2, 1, strm))) return st;
  // tensor-core tiles and MHA decode units touch disjoint outputs and
  // partial rows: run them side by side (tc on a high-priority second
  // stream forked from and joined back into the caller's stream)
  const int tc_sms = b->overlap && !fixed ? tc_share(P, c->head_dim, sm_count()) : 0;
  const bool both = tc_sms > 0;
  cudaStream_t tc_stream = strm;
  if (both) {
    st = ensure_aux_stream(b);
    if (st) return st;
    tc_stream = b->aux;
  }
  // the persistent kernels' unit counters start at zero (a fresh upload of
  // the batch's own plan zeroed them already)
  if ((P.n_tc || P.n_dtc) && (fixed || !b->ctr_fresh)) FG_CUDA(cudaMemsetAsync(ctr, 0, 8, strm));
  if (!fixed) b->ctr_fresh = false;
  // programmatic dependent launch along the chain query tiles -> decode ->
  // combine when the kernels follow each other on one stream with nothing
  // in between (the decode kernel waits for the query-tile grid before its
  // CTAs end, so the combine behind it sees both)
  const bool pdl = !both && !b->timing;
  if (both) {
    FG_CUDA(cudaEventRecord(b->fork, strm));
    FG_CUDA(cudaStreamWaitEvent(b->aux, b->fork, 0));
  }
  if (P.n_tc) {
    if ((st = mark(1, 0, tc_stream))) return st;
    e = fg::launch_attention_tc(&tm_q, &c->tm_kv, cv, b->view,
                                reinterpret_cast<const WorkItem*>(base + P.off_tc), P.n_tc, o, part_o,
                                part_ml, n_q_heads, g, scale_log2, window, sm_count(),
                                both ? tc_sms : INT32_MAX, ctr, tc_stream, q_tc ? c->rope : nullptr);
    if (e != cudaSuccess) return cuda_fail(e, "tensor-core attention launch");
    if ((st = mark(1, 1, tc_stream))) return st;
  }
  if (P.n_decode && (st = mark(0, 0, strm))) return st;
  e = fg::launch_attention_decode(cv, b->view,
                                  reinterpret_cast<const WorkItem*>(base + P.off_decode), P.n_decode,
                                  qr, o, part_o, part_ml, n_q_heads, scale_log2, strm);
  if (e != cudaSuccess) return cuda_fail(e, "decode attention launch");
  if (P.n_decode && (st = mark(0, 1, strm))) return st;
  if (P.n_dtc) {
    if ((st = mark(0, 0, strm))) return st;
    e = fg::launch_attention_decode_tc(&tm_q1, &c->tm_kv, cv, b->view,
                                       reinterpret_cast<const WorkItem*>(base + P.off_dtc), P.n_dtc, o,
                                       part_o, part_ml, n_q_heads, g, scale_log2,
                                       sm_count() * (both ? 4 : 2), ctr + 1, both ? tc_sms : 0,
                                       ctr, P.n_tc, pdl && P.n_tc > 0, strm);
    if (e != cudaSuccess) return cuda_fail(e, "tensor-core decode launch");
    if ((st = mark(0, 1, strm))) return st;
  }
  if (both) {
    FG_CUDA(cudaEventRecord(b->join, b->aux));
    FG_CUDA(cudaStreamWaitEvent(strm, b->join, 0));
  }
  if (P.n_combine && (st = mark(3, 0, strm))) return st;
  e = fg::launch_combine(b->view, reinterpret_cast<const CombineItem*>(base + P.off_combine),
                         P.n_combine, P.max_combine_rows, part_o, part_ml, o, n_q_heads, g,
                         c->head_dim, pdl && P.n_dtc > 0, strm);
  if (e != cudaSuccess) return cuda_fail(e, "combine launch");
  if (P.n_combine && (st = mark(3, 1, strm))) return st;
  const double t_end = now_us();
  b->hprof[7] += t_end - t_l;
  b->hprof[3] += t_end - t_a;
  return FG_OK;
}

extern "C" fg_status fg_host_profile_us(fg_ragged_batch* b, double out[8], int32_t reset) {
  if (!b || !out) return fail(FG_ERR_INVALID_ARG, "NULL argument");
  for (int i = 0; i < 8; ++i) {
    out[i] = b->hprof[i];
    if (reset) b->hprof[i] = 0.0;
  }
  return FG_OK;
}

extern "C" fg_status fg_ragged_batch_set_overlap(fg_ragged_batch* b, int32_t enable) {
  if (!b) return fail(FG_ERR_INVALID_ARG, "batch is NULL");
  b->overlap = enable != 0;
  return FG_OK;
}

extern "C" fg_status fg_ragged_batch_set_timing(fg_ragged_batch* b, int32_t enable) {
  if (!b) return fail(FG_ERR_INVALID_ARG, "batch is NULL");
  if (enable)
    for (cudaEvent_t& e : b->tev)
      if (!e) FG_CUDA(cudaEventCreate(&e));
  b->timing = enable != 0;
  return FG_OK;
}

extern "C" fg_status fg_attention_kernel_ms(fg_ragged_batch* b, float ms[4]) {
  if (!b || !ms) return fail(FG_ERR_INVALID_ARG, "NULL argument");
  for (int k = 0; k < 4; ++k) {
    ms[k] = 0.f;
    if (!b->timing || !b->tran[k]) continue;
    FG_CUDA(cudaEventSynchronize(b->tev[2 * k + 1]));
    FG_CUDA(cudaEventElapsedTime(&ms[k], b->tev[2 * k], b->tev[2 * k + 1]));
  }
  return FG_OK;
}

extern "C" fg_status fg_attention_plan_info(const fg_ragged_batch* b, int32_t info[8]) {
  if (!b || !info) return fail(FG_ERR_INVALID_ARG, "NULL argument");
  const fg::Plan& P = b->plan;
  info[0] = P.n_general;
  info[1] = P.n_decode + P.n_dtc;
  info[2] = P.n_tc;
  info[3] = P.n_combine;
  info[4] = P.part_rows;
  info[5] = b->last_launches;
  info[6] = info[7] = 0;
  return FG_OK;
}

extern "C" fg_status fg_plan_describe(const int32_t* q_lens, const int32_t* ctx_lens, int32_t n_seqs,
                                     int32_t n_kv_heads, int32_t group, int32_t head_dim, int32_t window,
                                     int32_t use_tc, int32_t slots, void* out, size_t out_bytes,
                                     int64_t counts[12]) {
  if (n_seqs < 0 || (n_seqs > 0 && (!q_lens || !ctx_lens)) || !counts)
    return fail(FG_ERR_INVALID_ARG, "fg_plan_describe: bad argument");
  if (n_kv_heads < 1 || group < 1 || (head_dim != 64 && head_dim != 128) || window < 0 || slots < 1)
    return fail(FG_ERR_INVALID_ARG, "fg_plan_describe: bad shape");
  for (int32_t s = 0; s < n_seqs; ++s)
    if (q_lens[s] < 1 || ctx_lens[s] < 0) return fail(FG_ERR_INVALID_ARG, "fg_plan_describe: bad lengths");
  std::vector<int32_t> ql(q_lens, q_lens + n_seqs), cl(ctx_lens, ctx_lens + n_seqs);
  fg::Plan P;
  fg::build_plan(ql, cl, n_kv_heads, group, head_dim, window, use_tc != 0, slots, &P);
  counts[0] = P.n_general;
  counts[1] = P.n_decode;
  counts[2] = P.n_tc;
  counts[3] = P.n_dtc;
  counts[4] = P.n_combine;
  counts[5] = P.part_rows;
  counts[6] = P.max_combine_rows;
  counts[7] = (int64_t)P.off_decode;
  counts[8] = (int64_t)P.off_tc;
  counts[9] = (int64_t)P.off_dtc;
  counts[10] = (int64_t)P.off_combine;
  counts[11] = (int64_t)P.bytes();
  if (out) {
    if (out_bytes < P.bytes()) return fail(FG_ERR_CAPACITY, "plan needs %zu bytes", P.bytes());
    P.pack(out);
  }
  return FG_OK;
}

extern "C" fg_status fg_device_status(fg_ragged_batch* b, void* stream) {
  if (!b) return fail(FG_ERR_INVALID_ARG, "batch is NULL");
  if (!b->derr) return FG_OK;
  cudaStream_t strm = static_cast<cudaStream_t>(stream);
  int32_t w = 0;
  FG_CUDA(cudaMemcpyAsync(&w, b->derr, 4, cudaMemcpyDeviceToHost, strm));
  FG_CUDA(cudaStreamSynchronize(strm));
  FG_CUDA(cudaMemsetAsync(b->derr, 0, 4, strm));
  FG_CUDA(cudaStreamSynchronize(strm));
  if (w & fg::kErrTimeout) return fail(FG_ERR_TIMEOUT, "a bounded device wait gave up (word 0x%x)", w);
  if (w) return fail(FG_ERR_DEVICE_CHECK, "a kernel skipped an out-of-range access (word 0x%x)", w);
  return FG_OK;
}

extern "C" const char* fg_status_string(fg_status s) {
  switch (s) {
    case FG_OK: return "FG_OK";
    case FG_ERR_INVALID_ARG: return "FG_ERR_INVALID_ARG";
    case FG_ERR_OUT_OF_RANGE: return "FG_ERR_OUT_OF_RANGE";
    case FG_ERR_ALIAS: return "FG_ERR_ALIAS";
    case FG_ERR_CAPACITY: return "FG_ERR_CAPACITY";
    case FG_ERR_UNSUPPORTED: return "FG_ERR_UNSUPPORTED";
    case FG_ERR_CUDA: return "FG_ERR_CUDA";
    case FG_ERR_DEVICE_CHECK: return "FG_ERR_DEVICE_CHECK";
    case FG_ERR_TIMEOUT: return "FG_ERR_TIMEOUT";
  }
  return "FG_ERR_UNKNOWN";
}

extern "C" const char* fg_last_error(void) { return g_last_error.c_str(); }

// The allocation-free entry point's launch (its storage is in attn_noalloc.cu).
fg_status fg_attention_launch_fixed(const fg_kv_cache* c, fg_ragged_batch* b, const void* q_rot,
                                    void* out, int32_t n_q_heads, float softmax_scale,
                                    int32_t window, cudaStream_t strm, float* ws,
                                    size_t ws_floats, void* plan_dev, size_t plan_bytes) {
  const FixedPassStorage fixed{ws, ws_floats, plan_dev, plan_bytes};
  return fg_attention_launch(c, b, q_rot, out, n_q_heads, softmax_scale, window, strm, &fixed);
}

// 2-D bf16 view (inner dim `inner`, outer dim `outer`, row stride inner * 2 B)
// with boxes of 64 x box_rows, 128-byte swizzle: the K-major operand layout
// of the projection's MMAs.
static bool make_rows_map(CUtensorMap* m, const void* base, uint64_t inner, uint64_t outer, uint32_t box_rows) {
  auto enc = tensor_map_encoder();
  if (!enc) return false;
  cuuint64_t dims[2] = {(cuuint64_t)inner, (cuuint64_t)outer};
  cuuint64_t strides[1] = {(cuuint64_t)inner * 2};
  cuuint32_t box[2] = {64, box_rows};
  cuuint32_t estr[2] = {1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

extern "C" fg_status fg_qkv_rotary_kv_append(fg_kv_cache* c, const fg_ragged_batch* b, const void* x,
                                             const void* w_qkv, int32_t hidden, void* q_rot, int32_t n_q_heads,
                                             double rope_theta, void* stream) {
  fg_status st = check_pass(c, b, n_q_heads);
  if (st) return st;
  if (!(rope_theta > 0.0)) return fail(FG_ERR_INVALID_ARG, "rope_theta must be > 0");
  if (hidden < 64 || hidden % 64) return fail(FG_ERR_UNSUPPORTED, "hidden %d is not a positive multiple of 64", hidden);
  if (b->n_tokens == 0) return FG_OK;
  if (!x || !w_qkv || !q_rot) return fail(FG_ERR_INVALID_ARG, "NULL tensor pointer");
  if (!aligned16(x) || !aligned16(w_qkv) || !aligned16(q_rot))
    return fail(FG_ERR_INVALID_ARG, "x, w_qkv and q_rot must be 16-byte aligned");
  st = ensure_rope(c, rope_theta, b->max_pos);
  if (st) return st;
  const int d = c->head_dim;
  const uint64_t n_out = (uint64_t)(n_q_heads + 2 * c->n_kv_heads) * d;
  // the persistent 128 x 256 tile form when the output width allows it
  const bool persistent = n_out % 256 == 0;
  CUtensorMap tm_x, tm_w;
  if (!make_rows_map(&tm_x, x, (uint64_t)hidden, (uint64_t)b->n_tokens, 128) ||
      !make_rows_map(&tm_w, w_qkv, (uint64_t)hidden, n_out, persistent ? 256u : (uint32_t)d))
    return fail(FG_ERR_CUDA, "cuTensorMapEncodeTiled failed for x or w_qkv");
  cudaError_t e = fg::launch_qkv_rotary_append(&tm_x, &tm_w, cache_view(c), b->view,
                                               static_cast<__nv_bfloat16*>(q_rot), c->rope, n_q_heads, hidden,
                                               static_cast<cudaStream_t>(stream), persistent);
  if (e != cudaSuccess) return cuda_fail(e, "qkv_rotary_append launch");
  return FG_OK;
}

extern "C" fg_status fg_output_projection(const fg_ragged_batch* b, const void* attn_out, const void* w_o,
                                          int32_t in_features, int32_t out_features, void* y, void* stream) {
  if (!b) return fail(FG_ERR_INVALID_ARG, "batch is NULL");
  if (in_features < 64 || in_features % 64)
    return fail(FG_ERR_UNSUPPORTED, "in_features %d is not a positive multiple of 64", in_features);
  if (out_features < 64 || out_features % 64)
    return fail(FG_ERR_UNSUPPORTED, "out_features %d is not a positive multiple of 64", out_features);
  if (!b->cache) return fail(FG_ERR_INVALID_ARG, "batch has no valid put");
  int dev = -1;
  if (cudaGetDevice(&dev) == cudaSuccess && b->device >= 0 && dev != b->device)
    return fail(FG_ERR_INVALID_ARG, "current device %d is not the batch's device %d", dev, b->device);
  if (b->n_tokens == 0) return FG_OK;
  if (!attn_out || !w_o || !y) return fail(FG_ERR_INVALID_ARG, "NULL tensor pointer");
  if (!aligned16(attn_out) || !aligned16(w_o) || !aligned16(y))
    return fail(FG_ERR_INVALID_ARG, "attn_out, w_o and y must be 16-byte aligned");
  const uint32_t n_tile = out_features % 256 == 0 ? 256 : out_features % 128 == 0 ? 128 : 64;
  CUtensorMap tm_x, tm_w;
  if (!make_rows_map(&tm_x, attn_out, (uint64_t)in_features, (uint64_t)b->n_tokens, 128) ||
      !make_rows_map(&tm_w, w_o, (uint64_t)in_features, (uint64_t)out_features, n_tile))
    return fail(FG_ERR_CUDA, "cuTensorMapEncodeTiled failed for attn_out or w_o");
  cudaError_t e = fg::launch_linear_bf16(&tm_x, &tm_w, b->view, static_cast<__nv_bfloat16*>(y), in_features,
                                         out_features, (int)n_tile, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "output projection launch");
  return FG_OK;
}

// Sets the thread-local error text (for entry points defined in other files).
fg_status fg_set_error(fg_status st, const char* msg) { return fail(st, "%s", msg); }
