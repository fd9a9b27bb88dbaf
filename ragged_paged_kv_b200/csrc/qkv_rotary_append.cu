// The Q/K/V projection fused with steps 1 and 2: qkv = x W^T on the tensor
// cores (tcgen05, fp32 accumulation in TMEM), and in the epilogue every
// output row is rounded to bf16 (as a projection with bf16 output would), Q
// and K rotated exactly as fg_rotary_kv_append does, Q written to q_rot and
// K, V written into their cache slots. The projected Q/K/V never make a round
// trip through HBM.
//
// A CTA computes one tile: 128 tokens x one head (d output features), so the
// epilogue thread that owns a token holds the head's whole row, both halves
// of every rotary pair. Roles: warp 0 (one thread) streams 64-wide K slices
// of x and W with 2-D TMA boxes (128-byte swizzle) into a 3-stage ring, warp
// 1 (one thread) issues the MMAs, warps 2-5 (TMEM lanes 32 (w % 4) ..) run
// the epilogue. Every wait is bounded.
//
// The same kernel with LINEAR = true is the layer's output projection
// y = o W_o^T (o the attention output viewed as [T, Hq d]): a CTA computes
// 128 tokens x D output features, and the epilogue rounds them to bf16 and
// stores them into y.
#include <cuda.h>

#include <cfloat>

#include "fg_internal.h"
#include "sm100_ptx.cuh"

namespace fg {
namespace {

constexpr long long kWaitLimit = 1LL << 31;

template <int D>
struct QkvCfg {
  static constexpr int BM = 128;  // tokens per tile
  static constexpr int BK = 64;   // hidden features per stage (one 128-byte row)
  static constexpr int ST = 3;
  static constexpr int kABytes = BM * BK * 2;
  static constexpr int kBBytes = D * BK * 2;
  static constexpr int kStage = kABytes + kBBytes;
  static constexpr int kOffBar = ST * kStage;
  static constexpr int kNumBars = 2 * ST + 1;  // full[ST], empty[ST], acc_full
  static constexpr int kSmem = kOffBar + kNumBars * 8 + 16;
  static constexpr int kThreads = 192;
  static constexpr uint32_t kTmemCols = D < 32 ? 32 : D;
};

struct QkvArgs {
  CacheView cache;
  BatchView batch;
  __nv_bfloat16* q_rot;
  const double2* rope;  // the rotary table, see below
  int Hq;
  int hidden;           // the contraction length
  __nv_bfloat16* y;     // LINEAR: output [T][n_out]
  int n_out;
};

// float64 -> bf16 with one rounding. Finite values: one PTX conversion
// (cvt.rn.bf16.f64, round to nearest even). Others: truncate to float and
// force the last bit on when anything was dropped (round to odd), then
// round to nearest even, which also rounds once.
__device__ __forceinline__ unsigned short f64_to_bf16(double x) {
  if (isfinite(x)) {
    unsigned short r;
    asm("cvt.rn.bf16.f64 %0, %1;" : "=h"(r) : "d"(x));
    return r;
  }
  float f = __double2float_rz(x);
  if ((double)f != x) f = __uint_as_float(__float_as_uint(f) | 1u);
  return __bfloat16_as_ushort(__float2bfloat16_rn(f));
}

__device__ __forceinline__ bool wait_or_flag(uint64_t* bar, uint32_t parity, int32_t* err, bool& ok) {
  if (!ok) return false;
  if (!ptx::mbar_wait_bounded(bar, parity, kWaitLimit)) {
    atomicOr(err, kErrTimeout);
    ok = false;
  }
  return ok;
}

// The epilogue of one accumulator row (token t) of one head of the
// projection (LINEAR: one D-wide column block of y): round to bf16, and for
// the Q/K/V projection rotate q and k and store q_rot or the cache slots.
template <int D, bool LINEAR>
__device__ __forceinline__ void epilogue_row(const QkvArgs& a, uint32_t (&acc)[D], int t, int head) {
  constexpr int HALF = D / 2;
  constexpr int GROUPS = HALF / 8;
  int32_t* err = a.batch.err;
  if (LINEAR && t < a.batch.n_tokens) {
    // round to bf16, pack pairs, and store the row's D features (32-byte
    // stores when y and its row pitch allow)
    __nv_bfloat16* dst = a.y + (int64_t)t * a.n_out + head * D;
    const bool wide = ((reinterpret_cast<uintptr_t>(a.y) | ((uintptr_t)a.n_out * 2)) & 31u) == 0;
#pragma unroll
    for (int q8 = 0; q8 < D / 16; ++q8) {
      uint32_t w[8];
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        __nv_bfloat162 pr = __floats2bfloat162_rn(__uint_as_float(acc[q8 * 16 + 2 * e]),
                                                  __uint_as_float(acc[q8 * 16 + 2 * e + 1]));
        w[e] = *reinterpret_cast<uint32_t*>(&pr);
      }
      if (wide) {
        ptx::st_global_v8(dst + q8 * 16, w);
      } else {
        uint4* d4 = reinterpret_cast<uint4*>(dst + q8 * 16);
        d4[0] = make_uint4(w[0], w[1], w[2], w[3]);
        d4[1] = make_uint4(w[4], w[5], w[6], w[7]);
      }
    }
  } else if (!LINEAR && t < a.batch.n_tokens) {
    // the projection's bf16 output, in place (bits in the low half)
#pragma unroll
    for (int e = 0; e < D; ++e) acc[e] = __bfloat16_as_ushort(__float2bfloat16_rn(__uint_as_float(acc[e])));
    const int Hkv = a.cache.n_kv_heads;
    const int p = a.batch.tok_pos[t];
    __nv_bfloat16* dst = nullptr;
    if (head < a.Hq) {
      dst = a.q_rot + ((int64_t)t * a.Hq + head) * D;
    } else {
      const int lb = p / a.cache.block_size;
      const int32_t blk = a.batch.tok_blk[t];
      if (blk >= 0 && blk < a.cache.n_blocks) {
        const int kv = head < a.Hq + Hkv ? 0 : 1;
        dst = a.cache.base +
              cache_offset(a.cache, blk, kv, head - a.Hq - kv * Hkv, p - lb * a.cache.block_size);
      } else {
        atomicOr(err, kErrBadBlock);
      }
    }
    if (head < a.Hq + Hkv) {
      // rotate-half in double, one rounding to bf16; the table row of
      // position p holds pair i = 8 g + e at entry e * GROUPS + g, times
      // 2^896
      const double2* rrow = a.rope + (int64_t)p * HALF;
#pragma unroll
      for (int i = 0; i < HALF; ++i) {
        const double2 cs = rrow[(i & 7) * GROUPS + (i >> 3)];
        const double c = cs.x * 0x1p-896, sn = cs.y * 0x1p-896;
        const double x1 = (double)__uint_as_float(acc[i] << 16);
        const double x2 = (double)__uint_as_float(acc[i + HALF] << 16);
        acc[i] = f64_to_bf16(__dsub_rn(__dmul_rn(x1, c), __dmul_rn(x2, sn)));
        acc[i + HALF] = f64_to_bf16(__dadd_rn(__dmul_rn(x2, c), __dmul_rn(x1, sn)));
      }
    }
    if (dst) {
      uint4* d4 = reinterpret_cast<uint4*>(dst);
#pragma unroll
      for (int q = 0; q < D / 8; ++q)
        d4[q] = make_uint4(acc[8 * q] | (acc[8 * q + 1] << 16), acc[8 * q + 2] | (acc[8 * q + 3] << 16),
                           acc[8 * q + 4] | (acc[8 * q + 5] << 16), acc[8 * q + 6] | (acc[8 * q + 7] << 16));
    }
  }
}

template <int D, bool LINEAR>
__global__ void __launch_bounds__(192, 2) qkv_rotary_append_kernel(const __grid_constant__ CUtensorMap tm_x,
                                                                  const __grid_constant__ CUtensorMap tm_w,
                                                                  QkvArgs a) {
  using C = QkvCfg<D>;
  extern __shared__ __align__(1024) unsigned char smem[];
  if (ptx::smem_u32(smem) & 1023u) {
    if (threadIdx.x == 0) atomicOr(a.batch.err, kErrBadIndex);
    return;
  }
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + C::kOffBar);
  uint64_t* empty = full + C::ST;
  uint64_t* acc_full = empty + C::ST;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(acc_full + 1);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int t0 = blockIdx.x * C::BM;  // first token of the tile
  const int head = blockIdx.y;        // in the q | k | v head list
  const int n_k = a.hidden / C::BK;
  int32_t* err = a.batch.err;
  if (threadIdx.x == 0) {
    for (int i = 0; i < C::ST; ++i) {
      ptx::mbar_init(&full[i], 1);
      ptx::mbar_init(&empty[i], 1);
    }
    ptx::mbar_init(acc_full, 1);
    ptx::fence_mbar_init();
  }
  if (warp == 1) {
    ptx::tmem_alloc(tmem_slot, C::kTmemCols);
    ptx::tmem_relinquish();
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  bool ok = true;

  if (warp == 0) {
    // ------------------------------------------------------------- loads
    if (lane == 0) {
      for (int i = 0; i < n_k && ok; ++i) {
        const int st = i % C::ST;
        if (i >= C::ST && !wait_or_flag(&empty[st], ((i / C::ST) - 1) & 1, err, ok)) break;
        ptx::mbar_arrive_expect_tx(&full[st], C::kStage);
        unsigned char* s = smem + st * C::kStage;
        ptx::tma_load_2d(s, &tm_x, i * C::BK, t0, &full[st]);  // rows past T read as zeros
        ptx::tma_load_2d(s + C::kABytes, &tm_w, i * C::BK, head * D, &full[st]);
      }
      for (int i = max(0, n_k - C::ST); i < n_k && ok; ++i)
        wait_or_flag(&full[i % C::ST], (i / C::ST) & 1, err, ok);
    }
  } else if (warp == 1) {
    // --------------------------------------------------------------- MMA
    if (lane == 0) {
      constexpr uint32_t idesc = ptx::idesc_bf16_f32(C::BM, D, 0, 0);
      const uint32_t base = ptx::smem_u32(smem);
      for (int i = 0; i < n_k && ok; ++i) {
        const int st = i % C::ST;
        if (!wait_or_flag(&full[st], (i / C::ST) & 1, err, ok)) break;
        ptx::tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < C::BK / 16; ++kk) {
          const uint64_t ad = ptx::smem_desc_sw128(base + st * C::kStage + kk * 32, 16, 1024);
          const uint64_t bd = ptx::smem_desc_sw128(base + st * C::kStage + C::kABytes + kk * 32, 16, 1024);
          ptx::mma_bf16(tmem, ad, bd, idesc, (i > 0 || kk > 0) ? 1u : 0u);
        }
        ptx::mma_commit(&empty[st]);
      }
      ptx::mma_commit(acc_full);
    }
  } else {
    // ---------------------------------------------------------- epilogue
    const int r = (warp & 3) * 32 + lane;  // token row == TMEM lane
    const uint32_t lane_base = (uint32_t)((warp & 3) * 32) << 16;
    const int t = t0 + r;
    const bool live = (warp & 3) * 32 + t0 < a.batch.n_tokens;
    if (wait_or_flag(acc_full, 0, err, ok) && live) {
      ptx::tc_fence_after();
      uint32_t acc[D];
#pragma unroll
      for (int c = 0; c < D / 32; ++c)
        ptx::tmem_ld32(tmem + lane_base + c * 32, *reinterpret_cast<uint32_t(*)[32]>(&acc[c * 32]));
      ptx::tmem_ld_wait();
      epilogue_row<D, LINEAR>(a, acc, t, head);
    }
  }
  ptx::tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    ptx::tc_fence_after();
    ptx::tmem_dealloc(tmem, C::kTmemCols);
  }
}

// The persistent form for output widths that are a multiple of 256: one CTA
// per SM walks tiles of 128 tokens x 256 outputs (tile index m fastest, so
// the CTAs running at once share a 256-row slice of W in L2). Warp 0 streams
// 64-wide K slices of x (16 KB) and W (32 KB) into a 4-stage ring, warp 1
// issues M = 128, N = 256 MMAs into one of two TMEM accumulators (256
// columns each), and warps 2-5 run the epilogue of the other: the epilogue
// of a tile overlaps the next tile's mainloop. D is the epilogue's block
// width (the head dim for the Q/K/V projection, 128 for the linear form);
// a tile holds 256 / D of them. Every wait is bounded.
struct GemmCfg {
  static constexpr int BM = 128, BN = 256, BK = 64, ST = 4;
  static constexpr int kABytes = BM * BK * 2;
  static constexpr int kBBytes = BN * BK * 2;
  static constexpr int kStage = kABytes + kBBytes;
  static constexpr int kOffBar = ST * kStage;
  static constexpr int kNumBars = 2 * ST + 4;  // full[ST], empty[ST], acc_full[2], acc_empty[2]
  static constexpr int kSmem = kOffBar + kNumBars * 8 + 16;
  static constexpr int kThreads = 192;
  static_assert(kSmem + 1024 <= 228 * 1024, "shared memory budget");
};

template <int D, bool LINEAR>
__global__ void __launch_bounds__(192, 1) gemm_persistent_kernel(const __grid_constant__ CUtensorMap tm_x,
                                                                const __grid_constant__ CUtensorMap tm_w,
                                                                QkvArgs a, int n_tiles_m, int n_tiles) {
  using C = GemmCfg;
  extern __shared__ __align__(1024) unsigned char smem[];
  if (ptx::smem_u32(smem) & 1023u) {
    if (threadIdx.x == 0) atomicOr(a.batch.err, kErrBadIndex);
    return;
  }
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + C::kOffBar);
  uint64_t* empty = full + C::ST;
  uint64_t* acc_full = empty + C::ST;
  uint64_t* acc_empty = acc_full + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(acc_empty + 2);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n_k = a.hidden / C::BK;
  int32_t* err = a.batch.err;
  if (threadIdx.x == 0) {
    for (int i = 0; i < C::ST; ++i) {
      ptx::mbar_init(&full[i], 1);
      ptx::mbar_init(&empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      ptx::mbar_init(&acc_full[i], 1);
      ptx::mbar_init(&acc_empty[i], 4);
    }
    ptx::fence_mbar_init();
  }
  if (warp == 1) {
    ptx::tmem_alloc(tmem_slot, 512);
    ptx::tmem_relinquish();
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  bool ok = true;

  if (warp == 0) {
    // ------------------------------------------------------------- loads
    if (lane == 0) {
      int it = 0;
      for (int tile = blockIdx.x; tile < n_tiles && ok; tile += gridDim.x) {
        const int m = tile % n_tiles_m, n = tile / n_tiles_m;
        for (int i = 0; i < n_k && ok; ++i, ++it) {
          const int st = it % C::ST;
          if (it >= C::ST && !wait_or_flag(&empty[st], ((it / C::ST) - 1) & 1, err, ok)) break;
          ptx::mbar_arrive_expect_tx(&full[st], C::kStage);
          unsigned char* sp = smem + st * C::kStage;
          ptx::tma_load_2d(sp, &tm_x, i * C::BK, m * C::BM, &full[st]);  // rows past T read as zeros
          ptx::tma_load_2d(sp + C::kABytes, &tm_w, i * C::BK, n * C::BN, &full[st]);
        }
      }
      // let the loads in flight land before the CTA can exit
      for (int j = max(0, it - C::ST); j < it && ok; ++j) wait_or_flag(&full[j % C::ST], (j / C::ST) & 1, err, ok);
    }
  } else if (warp == 1) {
    // --------------------------------------------------------------- MMA
    if (lane == 0) {
      constexpr uint32_t idesc = ptx::idesc_bf16_f32(C::BM, C::BN, 0, 0);
      const uint32_t base = ptx::smem_u32(smem);
      int it = 0, tl = 0;
      for (int tile = blockIdx.x; tile < n_tiles && ok; tile += gridDim.x, ++tl) {
        const int ab = tl & 1;
        // the epilogue of the tile two back must have read this accumulator
        if (tl >= 2 && !wait_or_flag(&acc_empty[ab], ((tl >> 1) - 1) & 1, err, ok)) break;
        ptx::tc_fence_after();
        for (int i = 0; i < n_k && ok; ++i, ++it) {
          const int st = it % C::ST;
          if (!wait_or_flag(&full[st], (it / C::ST) & 1, err, ok)) break;
          ptx::tc_fence_after();
#pragma unroll
          for (int kk = 0; kk < C::BK / 16; ++kk) {
            const uint64_t ad = ptx::smem_desc_sw128(base + st * C::kStage + kk * 32, 16, 1024);
            const uint64_t bd = ptx::smem_desc_sw128(base + st * C::kStage + C::kABytes + kk * 32, 16, 1024);
            ptx::mma_bf16(tmem + ab * C::BN, ad, bd, idesc, (i > 0 || kk > 0) ? 1u : 0u);
          }
          ptx::mma_commit(&empty[st]);
        }
        ptx::mma_commit(&acc_full[ab]);
      }
    }
  } else {
    // ---------------------------------------------------------- epilogue
    const int r = (warp & 3) * 32 + lane;  // token row == TMEM lane
    const uint32_t lane_base = (uint32_t)((warp & 3) * 32) << 16;
    int tl = 0;
    for (int tile = blockIdx.x; tile < n_tiles; tile += gridDim.x, ++tl) {
      const int m = tile % n_tiles_m, n = tile / n_tiles_m;
      const int ab = tl & 1;
      if (!wait_or_flag(&acc_full[ab], (tl >> 1) & 1, err, ok)) break;
      ptx::tc_fence_after();
      const int t = m * C::BM + r;
      if ((warp & 3) * 32 + m * C::BM < a.batch.n_tokens) {
#pragma unroll 1
        for (int part = 0; part < C::BN / D; ++part) {
          uint32_t acc[D];
#pragma unroll
          for (int c = 0; c < D / 32; ++c)
            ptx::tmem_ld32(tmem + lane_base + ab * C::BN + part * D + c * 32,
                           *reinterpret_cast<uint32_t(*)[32]>(&acc[c * 32]));
          ptx::tmem_ld_wait();
          epilogue_row<D, LINEAR>(a, acc, t, n * (C::BN / D) + part);
        }
      }
      // this accumulator may take the tile after next
      ptx::tc_fence_before();
      __syncwarp();
      if (lane == 0) ptx::mbar_arrive(&acc_empty[ab]);
    }
  }
  ptx::tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    ptx::tc_fence_after();
    ptx::tmem_dealloc(tmem, 512);
  }
}

template <int D, bool LINEAR>
cudaError_t launch_persistent_d(const CUtensorMap& tm_x, const CUtensorMap& tm_w, const QkvArgs& args,
                                int n_out, cudaStream_t stream) {
  using C = GemmCfg;
  static PerDeviceOnce configured;
  cudaError_t e0 = configured.run([] {
    return cudaFuncSetAttribute(gemm_persistent_kernel<D, LINEAR>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                C::kSmem);
  });
  if (e0 != cudaSuccess) return e0;
  const int n_tiles_m = (args.batch.n_tokens + C::BM - 1) / C::BM;
  const int n_tiles = n_tiles_m * (n_out / C::BN);
  int dev = 0, sms = 148;
  if (cudaGetDevice(&dev) != cudaSuccess || cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
    sms = 148;
  const int grid = n_tiles < sms ? n_tiles : sms;
  gemm_persistent_kernel<D, LINEAR><<<grid, C::kThreads, C::kSmem, stream>>>(tm_x, tm_w, args, n_tiles_m, n_tiles);
  return cudaGetLastError();
}

template <int D, bool LINEAR>
cudaError_t launch_qkv_d(const CUtensorMap& tm_x, const CUtensorMap& tm_w, const QkvArgs& args,
                         int n_heads_total, cudaStream_t stream) {
  using C = QkvCfg<D>;
  // per device: the attributes apply to the current device only
  static PerDeviceOnce configured;
  cudaError_t e0 = configured.run([] {
    cudaError_t e = cudaFuncSetAttribute(qkv_rotary_append_kernel<D, LINEAR>, cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmem);
    return e;
  });
  if (e0 != cudaSuccess) return e0;
  dim3 grid((args.batch.n_tokens + C::BM - 1) / C::BM, n_heads_total);
  qkv_rotary_append_kernel<D, LINEAR><<<grid, C::kThreads, C::kSmem, stream>>>(tm_x, tm_w, args);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_qkv_rotary_append(const void* tm_x, const void* tm_w, const CacheView& cache,
                                     const BatchView& batch, __nv_bfloat16* q_rot, const double2* rope,
                                     int n_q_heads, int hidden, cudaStream_t stream, bool persistent) {
  if (batch.n_tokens == 0) return cudaSuccess;
  QkvArgs args{cache, batch, q_rot, rope, n_q_heads, hidden, nullptr, 0};
  const int heads = n_q_heads + 2 * cache.n_kv_heads;
  const CUtensorMap& x = *static_cast<const CUtensorMap*>(tm_x);
  const CUtensorMap& w = *static_cast<const CUtensorMap*>(tm_w);
  if (persistent) {
    if (cache.head_dim == 128) return launch_persistent_d<128, false>(x, w, args, heads * 128, stream);
    return launch_persistent_d<64, false>(x, w, args, heads * 64, stream);
  }
  if (cache.head_dim == 128) return launch_qkv_d<128, false>(x, w, args, heads, stream);
  return launch_qkv_d<64, false>(x, w, args, heads, stream);
}

cudaError_t launch_linear_bf16(const void* tm_x, const void* tm_w, const BatchView& batch, __nv_bfloat16* y,
                               int k_len, int n_out, int n_tile, cudaStream_t stream) {
  if (batch.n_tokens == 0) return cudaSuccess;
  QkvArgs args{};
  args.batch = batch;
  args.hidden = k_len;
  args.y = y;
  args.n_out = n_out;
  const CUtensorMap& x = *static_cast<const CUtensorMap*>(tm_x);
  const CUtensorMap& w = *static_cast<const CUtensorMap*>(tm_w);
  if (n_tile == 256) return launch_persistent_d<128, true>(x, w, args, n_out, stream);
  if (n_tile == 128) return launch_qkv_d<128, true>(x, w, args, n_out / 128, stream);
  return launch_qkv_d<64, true>(x, w, args, n_out / 64, stream);
}

}  // namespace fg
