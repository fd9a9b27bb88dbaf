// Split-KV decode attention for one-token queries with one query head per kv
// head (MHA decode). This is where decode-heavy batches spend their time, and
// it is bound by HBM bandwidth: every cached K and V row is read once.
//
// One CTA per work unit = (sequence, head, 64-aligned key range). Warp 0 is
// the producer: one lane streams the unit's 64-key stages with 1-D bulk copies
// (cp.async.bulk, the TMA's linear mode) straight from the paged cache - a
// (block, head) K or V tile is contiguous, so a 64-key stage is one 16 KB copy
// per operand at block_size >= 64 - into a ring of shared-memory stages
// guarded by mbarriers (full: transaction bytes; empty: consumer arrivals).
// Warps 1..4 consume: each takes 16 keys of a stage, computes the 16 dot
// products with 16-byte shared loads and a multi-value butterfly reduction,
// keeps a private online softmax (running max / sum in registers, rescaling
// its accumulators when the max grows), and accumulates P.V with each lane
// owning d/32 output dims. The four warp states are merged in shared memory
// at the end. Waits are bounded; a wait that gives up records kErrTimeout.
#include <cfloat>

#include "fg_internal.h"
#include "sm100_ptx.cuh"

namespace fg {
namespace {

constexpr long long kWaitLimit = 1LL << 31;  // SM cycles, ~1 s

template <int D>
struct DecodeCfg {
  static constexpr int kStageKeys = 64;
  static constexpr int kStages = D == 128 ? 3 : 4;
  static constexpr int kConsumers = 4;
  static constexpr int kThreads = 32 * (kConsumers + 1);
  static constexpr int kKeysPerWarp = kStageKeys / kConsumers;  // 16
  static constexpr int kLanesPerKey = D / 8;                     // 16-byte chunks per row
  static constexpr int kKeysPerIter = 32 / kLanesPerKey;
  static constexpr int kIters = kKeysPerWarp / kKeysPerIter;     // == kLanesPerKey / 2
  static constexpr int kDimsPerLane = D / 32;
  static constexpr int kTileBytes = kStageKeys * D * 2;
  static constexpr int kStageBytes = 2 * kTileBytes;
  static constexpr int kBarBytes = 2 * kStages * 8;
  static constexpr int kMergeBytes = kConsumers * (D + 2) * 4;
  static constexpr int kSmem = 128 + kStages * kStageBytes + kBarBytes + kMergeBytes;
  static_assert(kIters * 2 == kLanesPerKey, "lane/key mapping assumes iters = lanes_per_key / 2");
};

// Sum v[0..CNT) across the lanes of an M*2-lane group, halving the number of
// values held per lane at each step; ends with every lane holding one full
// sum (lanes l and l^1 hold the same one).
template <int CNT, int M>
__device__ __forceinline__ void butterfly(float (&v)[8], int lane) {
  if constexpr (M >= 1) {
    if constexpr (CNT > 1) {
      const bool up = (lane & M) != 0;
#pragma unroll
      for (int i = 0; i < CNT / 2; ++i) {
        const float send = up ? v[i] : v[i + CNT / 2];
        const float keep = up ? v[i + CNT / 2] : v[i];
        v[i] = keep + __shfl_xor_sync(0xffffffffu, send, M);
      }
      butterfly<CNT / 2, M / 2>(v, lane);
    } else {
      v[0] += __shfl_xor_sync(0xffffffffu, v[0], M);
      butterfly<1, M / 2>(v, lane);
    }
  }
}

__device__ __forceinline__ float bf_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf_hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

template <int D>
__global__ void __launch_bounds__(DecodeCfg<D>::kThreads) attn_decode_kernel(
    CacheView cache, BatchView batch, const WorkItem* __restrict__ items,
    const __nv_bfloat16* __restrict__ q_rot, __nv_bfloat16* __restrict__ out,
    float* __restrict__ part_o, float* __restrict__ part_ml, int Hq, float scale_log2) {
  using C = DecodeCfg<D>;
  extern __shared__ __align__(128) unsigned char smem_raw[];
  unsigned char* smem = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 127) & ~uintptr_t(127));
  unsigned char* stages = smem;
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + C::kStages * C::kStageBytes);
  uint64_t* empty = full + C::kStages;
  float* merge = reinterpret_cast<float*>(empty + C::kStages);

  const WorkItem it = items[blockIdx.x];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int s = it.seq, h = it.kv_head;
  const int kb = it.key_begin, ke = it.key_end;
  const int kb_al = kb - (kb & (C::kStageKeys - 1));
  const int n_st = (ke - kb_al + C::kStageKeys - 1) / C::kStageKeys;

  if (threadIdx.x == 0) {
    for (int i = 0; i < C::kStages; ++i) {
      ptx::mbar_init(&full[i], 1);
      ptx::mbar_init(&empty[i], C::kConsumers);
    }
    ptx::fence_mbar_init();
  }
  __syncthreads();

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      const int32_t* bt = batch.bt + batch.bt_off[s];
      const int nb = batch.bt_off[s + 1] - batch.bt_off[s];
      const int B = cache.block_size;
      bool ok = true;
      for (int st = 0; st < n_st && ok; ++st) {
        const int slot = st % C::kStages;
        if (st >= C::kStages &&
            !ptx::mbar_wait_bounded(&empty[slot], ((st / C::kStages) - 1) & 1, kWaitLimit)) {
          atomicOr(batch.err, kErrTimeout);
          ok = false;
          break;
        }
        const int p0 = kb_al + st * C::kStageKeys;
        // count the bytes first: expect_tx must cover exactly what is issued
        uint32_t bytes = 0;
        for (int pos = p0; pos < p0 + C::kStageKeys;) {
          const int lb = pos / B, off = pos - lb * B;
          const int n = min(B - off, p0 + C::kStageKeys - pos);
          if (lb < nb) {
            const int32_t blk = bt[lb];
            if (blk >= 0 && blk < cache.n_blocks) bytes += 2u * n * D * 2;
          }
          pos += n;
        }
        ptx::mbar_arrive_expect_tx(&full[slot], bytes);
        unsigned char* kdst = stages + slot * C::kStageBytes;
        unsigned char* vdst = kdst + C::kTileBytes;
        for (int pos = p0; pos < p0 + C::kStageKeys;) {
          const int lb = pos / B, off = pos - lb * B;
          const int n = min(B - off, p0 + C::kStageKeys - pos);
          if (lb < nb) {
            const int32_t blk = bt[lb];
            if (blk >= 0 && blk < cache.n_blocks) {
              const uint32_t nbytes = n * D * 2;
              const int row = pos - p0;
              ptx::bulk_g2s(kdst + row * D * 2, cache.base + cache_offset(cache, blk, 0, h, off), nbytes,
                            &full[slot]);
              ptx::bulk_g2s(vdst + row * D * 2, cache.base + cache_offset(cache, blk, 1, h, off), nbytes,
                            &full[slot]);
            } else {
              atomicOr(batch.err, kErrBadBlock);
            }
          }
          pos += n;
        }
      }
      // do not leave while copies may still land in this CTA's shared memory
      for (int st = max(0, n_st - C::kStages); st < n_st && ok; ++st)
        if (!ptx::mbar_wait_bounded(&full[st % C::kStages], (st / C::kStages) & 1, kWaitLimit)) {
          atomicOr(batch.err, kErrTimeout);
          break;
        }
    }
    return;
  }

  // -------------------------------------------------------------- consumers
  const int cw = warp - 1;
  const int row = batch.cu_q[s] + it.tok_begin;
  // q chunk of this lane (the 16-byte chunk it multiplies), pre-scaled by
  // softmax_scale * log2(e) so scores are in base-2 units
  const int chunk = lane % C::kLanesPerKey;
  float qf[8];
  {
    const uint4 qv = *reinterpret_cast<const uint4*>(q_rot + ((int64_t)row * Hq + h) * D + chunk * 8);
    const uint32_t w[4] = {qv.x, qv.y, qv.z, qv.w};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      qf[2 * e] = bf_lo(w[e]) * scale_log2;
      qf[2 * e + 1] = bf_hi(w[e]) * scale_log2;
    }
  }
  float m = -INFINITY, l = 0.f;
  float acc[C::kDimsPerLane];
#pragma unroll
  for (int j = 0; j < C::kDimsPerLane; ++j) acc[j] = 0.f;
  const int my_key = ((lane >> 1) & (C::kIters - 1)) * C::kKeysPerIter + lane / C::kLanesPerKey;
  bool alive = true;

  for (int st = 0; st < n_st; ++st) {
    const int slot = st % C::kStages;
    if (!ptx::mbar_wait_bounded(&full[slot], (st / C::kStages) & 1, kWaitLimit)) {
      if (lane == 0) atomicOr(batch.err, kErrTimeout);
      alive = false;
      break;
    }
    const unsigned char* ks = stages + slot * C::kStageBytes + cw * C::kKeysPerWarp * D * 2;
    const unsigned char* vs = ks + C::kTileBytes;
    float v[8];
#pragma unroll
    for (int i = 0; i < C::kIters; ++i) {
      const int key = i * C::kKeysPerIter + lane / C::kLanesPerKey;
      const uint4 kv = *reinterpret_cast<const uint4*>(ks + key * D * 2 + chunk * 16);
      const uint32_t w[4] = {kv.x, kv.y, kv.z, kv.w};
      float d0 = 0.f, d1 = 0.f;
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        d0 = fmaf(qf[2 * e], bf_lo(w[e]), d0);
        d1 = fmaf(qf[2 * e + 1], bf_hi(w[e]), d1);
      }
      v[i] = d0 + d1;
    }
    butterfly<C::kIters, C::kLanesPerKey / 2>(v, lane);
    const int kp = kb_al + st * C::kStageKeys + cw * C::kKeysPerWarp + my_key;
    const float sc = (kp >= kb && kp < ke) ? v[0] : -INFINITY;
    float mt = sc;
#pragma unroll
    for (int o = 16; o >= 2; o >>= 1) mt = fmaxf(mt, __shfl_xor_sync(0xffffffffu, mt, o));
    const float m_new = fmaxf(m, mt);
    float p = 0.f, alpha = 1.f;
    if (m_new != -INFINITY) {
      p = exp2f(sc - m_new);
      alpha = exp2f(m - m_new);
    }
    float ps = p;
#pragma unroll
    for (int o = 16; o >= 2; o >>= 1) ps += __shfl_xor_sync(0xffffffffu, ps, o);
    l = l * alpha + ps;
    m = m_new;
#pragma unroll
    for (int j = 0; j < C::kDimsPerLane; ++j) acc[j] *= alpha;
#pragma unroll
    for (int k = 0; k < C::kKeysPerWarp; ++k) {
      const int src = (k % C::kKeysPerIter) * C::kLanesPerKey + ((k / C::kKeysPerIter) << 1);
      const float pk = __shfl_sync(0xffffffffu, p, src);
      if (pk != 0.f) {
        if constexpr (C::kDimsPerLane == 4) {
          const uint2 vv = *reinterpret_cast<const uint2*>(vs + k * D * 2 + lane * 8);
          acc[0] = fmaf(pk, bf_lo(vv.x), acc[0]);
          acc[1] = fmaf(pk, bf_hi(vv.x), acc[1]);
          acc[2] = fmaf(pk, bf_lo(vv.y), acc[2]);
          acc[3] = fmaf(pk, bf_hi(vv.y), acc[3]);
        } else {
          const uint32_t vv = *reinterpret_cast<const uint32_t*>(vs + k * D * 2 + lane * 4);
          acc[0] = fmaf(pk, bf_lo(vv), acc[0]);
          acc[1] = fmaf(pk, bf_hi(vv), acc[1]);
        }
      }
    }
    __syncwarp();
    if (lane == 0) ptx::mbar_arrive(&empty[slot]);
  }

  // merge the four warp states
  float* mw = merge;                       // [kConsumers] max
  float* lw = merge + C::kConsumers;       // [kConsumers] sum
  float* aw = merge + 2 * C::kConsumers;   // [kConsumers][D]
  if (lane == 0) {
    mw[cw] = alive ? m : -INFINITY;
    lw[cw] = alive ? l : 0.f;
  }
#pragma unroll
  for (int j = 0; j < C::kDimsPerLane; ++j) aw[cw * D + lane * C::kDimsPerLane + j] = acc[j];
  asm volatile("bar.sync 1, %0;" ::"n"(C::kConsumers * 32));
  const int t = threadIdx.x - 32;
  if (t < D) {
    float M = -INFINITY;
#pragma unroll
    for (int i = 0; i < C::kConsumers; ++i) M = fmaxf(M, mw[i]);
    float L = 0.f, o = 0.f;
#pragma unroll
    for (int i = 0; i < C::kConsumers; ++i) {
      const float wgt = mw[i] == -INFINITY ? 0.f : exp2f(mw[i] - M);
      L = fmaf(wgt, lw[i], L);
      o = fmaf(wgt, aw[i * D + t], o);
    }
    if (it.part < 0) {
      out[((int64_t)row * Hq + h) * D + t] = __float2bfloat16_rn(L > 0.f ? o / L : 0.f);
    } else {
      part_o[(int64_t)it.part * D + t] = o;
      if (t == 0) {
        part_ml[(int64_t)it.part * 2] = M;
        part_ml[(int64_t)it.part * 2 + 1] = L;
      }
    }
  }
}

template <int D>
cudaError_t launch_decode_d(const CacheView& cache, const BatchView& batch, const WorkItem* items,
                            int n_items, const __nv_bfloat16* q_rot, __nv_bfloat16* out,
                            float* part_o, float* part_ml, int Hq, float scale_log2,
                            cudaStream_t stream) {
  using C = DecodeCfg<D>;
  // per device: the attributes apply to the current device only
  static PerDeviceOnce configured;
  cudaError_t e0 = configured.run([] {
    cudaError_t e = cudaFuncSetAttribute(attn_decode_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmem);
    // the largest shared-memory carveout, so CTAs of different kernels can
    // share an SM
    if (e == cudaSuccess)
      e = cudaFuncSetAttribute(attn_decode_kernel<D>, cudaFuncAttributePreferredSharedMemoryCarveout,
                               cudaSharedmemCarveoutMaxShared);
    return e;
  });
  if (e0 != cudaSuccess) return e0;
  attn_decode_kernel<D><<<n_items, C::kThreads, C::kSmem, stream>>>(cache, batch, items, q_rot, out,
                                                                    part_o, part_ml, Hq, scale_log2);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_attention_decode(const CacheView& cache, const BatchView& batch,
                                    const WorkItem* items, int n_items,
                                    const __nv_bfloat16* q_rot, __nv_bfloat16* out, float* part_o,
                                    float* part_ml, int n_q_heads, float scale_log2,
                                    cudaStream_t stream) {
  if (n_items == 0) return cudaSuccess;
  if (cache.head_dim == 128)
    return launch_decode_d<128>(cache, batch, items, n_items, q_rot, out, part_o, part_ml, n_q_heads,
                                scale_log2, stream);
  return launch_decode_d<64>(cache, batch, items, n_items, q_rot, out, part_o, part_ml, n_q_heads,
                             scale_log2, stream);
}

}  // namespace fg
