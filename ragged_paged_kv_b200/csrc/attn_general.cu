// Ragged paged attention, general CUDA-core path.
//
// Serves any work unit (up to 16 query rows of one sequence and kv head, any
// key range), so it is the path for shapes the specialised kernels do not
// cover. One CTA per unit; keys are walked in 64-key stages gathered from the
// block table into shared memory with 16-byte loads; scores, online softmax
// (running max and sum per row, rescaling the accumulators when the max
// grows) and the P.V product run on CUDA cores in fp32.
#include <cfloat>

#include "fg_internal.h"
#include "sm100_ptx.cuh"

namespace fg {
namespace {

constexpr int kRows = 16;
constexpr int kStage = 64;
constexpr int kThreads = 128;

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}
__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

template <int D>
__global__ void __launch_bounds__(kThreads) attn_general_kernel(
    CacheView cache, BatchView batch, const WorkItem* __restrict__ items,
    const __nv_bfloat16* __restrict__ q_rot, __nv_bfloat16* __restrict__ out,
    float* __restrict__ part_o, float* __restrict__ part_ml, int Hq, int g, float scale_log2,
    int window) {
  constexpr int KP = D + 8;                    // padded K row: conflict-free 16 B reads
  constexpr int RPT = kRows * D / kThreads;    // accumulator rows per thread
  constexpr int RSTEP = kThreads / D;          // row stride between a thread's rows
  __shared__ __align__(16) float qs[kRows][D];
  __shared__ __align__(16) __nv_bfloat16 ks[kStage][KP];
  __shared__ __align__(16) __nv_bfloat16 vs[kStage][D];
  __shared__ float ps[kRows][kStage];
  __shared__ float row_m[kRows], row_l[kRows], row_a[kRows];
  __shared__ int row_p[kRows];

  const WorkItem it = items[blockIdx.x];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int s = it.seq;
  const int R = it.n_rows;
  const int ctx = batch.ctx[s];
  const int row0 = batch.cu_q[s] + it.tok_begin;
  const int32_t* bt = batch.bt + batch.bt_off[s];
  const int Hkv = cache.n_kv_heads;

  for (int idx = tid; idx < kRows * D; idx += kThreads) {
    const int r = idx / D, dd = idx - r * D;
    float x = 0.f;
    if (r < R) {
      const int j = r / g, h = it.kv_head * g + (r - j * g);
      x = __bfloat162float(q_rot[((int64_t)(row0 + j) * Hq + h) * D + dd]) * scale_log2;
    }
    qs[r][dd] = x;
  }
  if (tid < kRows) {
    row_m[tid] = -INFINITY;
    row_l[tid] = 0.f;
    row_p[tid] = ctx + it.tok_begin + tid / g;
  }
  float acc[RPT];
#pragma unroll
  for (int i = 0; i < RPT; ++i) acc[i] = 0.f;
  const int dim = tid % D;
  const int rbase = tid / D;

  const int kb = it.key_begin, ke = it.key_end;
  for (int st = kb - (kb % kStage); st < ke; st += kStage) {
    __syncthreads();
    constexpr int CH = D / 8;
    for (int c = tid; c < kStage * CH; c += kThreads) {
      const int kk = c / CH, c8 = (c - kk * CH) * 8;
      const int kp = st + kk;
      uint4 kx = make_uint4(0, 0, 0, 0), vx = kx;
      if (kp >= kb && kp < ke) {
        const int lb = kp / cache.block_size;
        const int32_t blk = bt[lb];
        if (blk >= 0 && blk < cache.n_blocks) {
          const int slot = kp - lb * cache.block_size;
          kx = *reinterpret_cast<const uint4*>(cache.base + cache_offset(cache, blk, 0, it.kv_head, slot) + c8);
          vx = *reinterpret_cast<const uint4*>(cache.base + cache_offset(cache, blk, 1, it.kv_head, slot) + c8);
        } else if (c8 == 0) {
          atomicOr(batch.err, kErrBadBlock);
        }
      }
      *reinterpret_cast<uint4*>(&ks[kk][c8]) = kx;
      *reinterpret_cast<uint4*>(&vs[kk][c8]) = vx;
    }
    __syncthreads();
    // scores: thread -> key tid % 64, rows tid / 64 + 2 i
    {
      const int kk = tid % kStage;
      const int kp = st + kk;
      for (int r = tid / kStage; r < kRows; r += kThreads / kStage) {
        float dot = 0.f;
        if (r < R) {
#pragma unroll 4
          for (int c8 = 0; c8 < D; c8 += 8) {
            const uint4 kx = *reinterpret_cast<const uint4*>(&ks[kk][c8]);
            const float4 qa = *reinterpret_cast<const float4*>(&qs[r][c8]);
            const float4 qb = *reinterpret_cast<const float4*>(&qs[r][c8 + 4]);
            const __nv_bfloat162* k2 = reinterpret_cast<const __nv_bfloat162*>(&kx);
            float2 f0 = __bfloat1622float2(k2[0]), f1 = __bfloat1622float2(k2[1]);
            float2 f2 = __bfloat1622float2(k2[2]), f3 = __bfloat1622float2(k2[3]);
            dot = fmaf(qa.x, f0.x, dot); dot = fmaf(qa.y, f0.y, dot);
            dot = fmaf(qa.z, f1.x, dot); dot = fmaf(qa.w, f1.y, dot);
            dot = fmaf(qb.x, f2.x, dot); dot = fmaf(qb.y, f2.y, dot);
            dot = fmaf(qb.z, f3.x, dot); dot = fmaf(qb.w, f3.y, dot);
          }
        }
        const int p = row_p[r];
        const bool ok = r < R && kp >= kb && kp < ke && kp <= p && (window <= 0 || kp > p - window);
        ps[r][kk] = ok ? dot : -INFINITY;
      }
    }
    __syncthreads();
    // online softmax, one warp per row
    for (int r = warp; r < R; r += kThreads / 32) {
      const float v0 = ps[r][lane], v1 = ps[r][lane + 32];
      const float mx = warp_max(fmaxf(v0, v1));
      const float m_old = row_m[r];
      const float m_new = fmaxf(m_old, mx);
      float p0 = 0.f, p1 = 0.f, alpha = 1.f;
      if (m_new != -INFINITY) {
        p0 = exp2f(v0 - m_new);
        p1 = exp2f(v1 - m_new);
        alpha = exp2f(m_old - m_new);
      }
      const float sum = warp_sum(p0 + p1);
      ps[r][lane] = p0;
      ps[r][lane + 32] = p1;
      if (lane == 0) {
        row_l[r] = row_l[r] * alpha + sum;
        row_m[r] = m_new;
        row_a[r] = alpha;
      }
    }
    __syncthreads();
#pragma unroll
    for (int i = 0; i < RPT; ++i) {
      const int r = rbase + i * RSTEP;
      acc[i] *= (r < R) ? row_a[r] : 1.f;
    }
    for (int kk = 0; kk < kStage; ++kk) {
      const float vv = __bfloat162float(vs[kk][dim]);
#pragma unroll
      for (int i = 0; i < RPT; ++i) acc[i] = fmaf(ps[rbase + i * RSTEP][kk], vv, acc[i]);
    }
  }
  __syncthreads();
#pragma unroll
  for (int i = 0; i < RPT; ++i) {
    const int r = rbase + i * RSTEP;
    if (r >= R) continue;
    if (it.part < 0) {
      const int j = r / g, h = it.kv_head * g + (r - j * g);
      const float l = row_l[r];
      const float o = l > 0.f ? acc[i] / l : 0.f;
      out[((int64_t)(row0 + j) * Hq + h) * D + dim] = __float2bfloat16_rn(o);
    } else {
      part_o[(int64_t)(it.part + r) * D + dim] = acc[i];
      if (dim == 0) {
        part_ml[(int64_t)(it.part + r) * 2] = row_m[r];
        part_ml[(int64_t)(it.part + r) * 2 + 1] = row_l[r];
      }
    }
  }
  (void)Hkv;
}

// Merge split partials: O = sum_i 2^(m_i - M) O_i / sum_i 2^(m_i - M) l_i.
template <int D>
__global__ void __launch_bounds__(128) combine_kernel(BatchView batch,
                                                      const CombineItem* __restrict__ items,
                                                      const float* __restrict__ part_o,
                                                      const float* __restrict__ part_ml,
                                                      __nv_bfloat16* __restrict__ out, int Hq,
                                                      int g) {
  // launched behind the kernel that wrote the partials: wait for it (and
  // everything before it) to finish before reading them
  ptx::grid_dependency_wait();
  const CombineItem it = items[blockIdx.x];
  const int r = blockIdx.y * (blockDim.x >> 5) + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (r >= it.n_rows) return;
  // one pass of running log-sum-exp merges; four splits' loads in flight at once
  constexpr int PER = D / 32;
  float M = -INFINITY, L = 0.f, o[PER];
#pragma unroll
  for (int e = 0; e < PER; ++e) o[e] = 0.f;
#pragma unroll 4
  for (int i = 0; i < it.n_splits; ++i) {
    const int64_t pr = it.part_base + (int64_t)i * it.n_rows + r;
    const float m = part_ml[pr * 2], l = part_ml[pr * 2 + 1];
    float x[PER];
#pragma unroll
    for (int e = 0; e < PER; ++e) x[e] = part_o[pr * D + lane + 32 * e];
    if (m != -INFINITY) {
      const float Mn = fmaxf(M, m);
      const float s_old = M == -INFINITY ? 0.f : exp2f(M - Mn), s_new = exp2f(m - Mn);
      L = fmaf(L, s_old, l * s_new);
#pragma unroll
      for (int e = 0; e < PER; ++e) o[e] = fmaf(o[e], s_old, x[e] * s_new);
      M = Mn;
    }
  }
  const int j = r / g, h = it.kv_head * g + (r - j * g);
  const int64_t row = batch.cu_q[it.seq] + it.tok_begin + j;
  const float inv = L > 0.f ? 1.f / L : 0.f;
#pragma unroll
  for (int e = 0; e < PER; ++e)
    out[(row * Hq + h) * D + lane + 32 * e] = __float2bfloat16_rn(o[e] * inv);
}

}  // namespace

cudaError_t launch_attention_general(const CacheView& cache, const BatchView& batch,
                                     const WorkItem* items, int n_items,
                                     const __nv_bfloat16* q_rot, __nv_bfloat16* out,
                                     float* part_o, float* part_ml, int n_q_heads, int g,
                                     float scale_log2, int window, cudaStream_t stream) {
  if (n_items == 0) return cudaSuccess;
  if (cache.head_dim == 128)
    attn_general_kernel<128><<<n_items, kThreads, 0, stream>>>(cache, batch, items, q_rot, out, part_o,
                                                               part_ml, n_q_heads, g, scale_log2, window);
  else
    attn_general_kernel<64><<<n_items, kThreads, 0, stream>>>(cache, batch, items, q_rot, out, part_o,
                                                              part_ml, n_q_heads, g, scale_log2, window);
  return cudaGetLastError();
}

cudaError_t launch_combine(const BatchView& batch, const CombineItem* items, int n_items,
                           int max_rows, const float* part_o, const float* part_ml,
                           __nv_bfloat16* out, int n_q_heads, int g, int head_dim, bool pdl,
                           cudaStream_t stream) {
  if (n_items == 0) return cudaSuccess;
  // one warp per row, up to four rows per CTA
  const int warps = max_rows < 4 ? (max_rows < 1 ? 1 : max_rows) : 4;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(n_items, (max_rows + warps - 1) / warps);
  cfg.blockDim = dim3(32 * warps);
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl ? 1 : 0;
  if (head_dim == 128)
    return cudaLaunchKernelEx(&cfg, combine_kernel<128>, batch, items, part_o, part_ml, out, n_q_heads, g);
  return cudaLaunchKernelEx(&cfg, combine_kernel<64>, batch, items, part_o, part_ml, out, n_q_heads, g);
}

}  // namespace fg
