// Ragged paged attention on the 5th-generation tensor cores (tcgen05).
//
// A work unit is one 128-row query tile of one sequence and kv head: the
// rows are (token, q head of the group) pairs, 128/g consecutive new tokens
// times the g q heads that share the kv head, so a grouped-query tile reuses
// each K/V tile for all g heads. Prompt chunks give full tiles; a grouped
// decode token gives a g-row tile. The unit walks its key range in 128-key
// tiles:
//
//   warp 4 (TMA)      Q once (3-D box: 64 dims x g heads x 128/g tokens), then
//                     K and V tiles through the block table, one 2-D box per
//                     (block part, 64 dims), into 2-stage K and V rings;
//   warp 5 (MMA)      one thread issues S = Q K^T into a double-buffered TMEM
//                     S tile, and O += P V into a TMEM O tile;
//   warps 0-3         thread r owns query row r (TMEM lane r): reads its S
//                     row with tcgen05.ld, masks (causal, window, unit range),
//                     keeps an online softmax (a running max that is only
//                     moved - with a rescale of its O row in TMEM - when a
//                     tile raises it by more than 2^8), writes P as bf16 into
//                     the swizzled shared-memory layout the second MMA reads,
//                     and at the end normalises O and stores it.
//
// Every wait is bounded; a wait that gives up sets kErrTimeout and the CTA
// drains and returns.
#include <cuda.h>

#include <cfloat>

#include "fg_internal.h"
#include "sm100_ptx.cuh"

namespace fg {
namespace {

constexpr long long kWaitLimit = 1LL << 31;

template <int D>
struct TcCfg {
  static constexpr int BM = 128;  // query rows per tile
  static constexpr int BN = 128;  // keys per tile
  static constexpr int KST = 2, VST = 2;
  static constexpr int DH = D / 64;  // 64-dim (128-byte) boxes per row
  static constexpr int kQBytes = BM * D * 2;
  static constexpr int kKVBytes = BN * D * 2;
  static constexpr int kPBytes = BM * BN * 2;
  static constexpr int kOffQ = 0;
  static constexpr int kOffK = kOffQ + kQBytes;
  static constexpr int kOffV = kOffK + KST * kKVBytes;
  static constexpr int kOffP = kOffV + VST * kKVBytes;
  static constexpr int kOffBar = kOffP + kPBytes;
  // q_full, k_full[KST], k_empty[KST], v_full[VST], v_empty[VST], s_full[2],
  // s_free[2], p_full, pv_done
  static constexpr int kNumBars = 1 + 2 * KST + 2 * VST + 2 + 2 + 2;
  static constexpr int kSmem = 1024 + kOffBar + kNumBars * 8 + 16;
  static constexpr int kThreads = 192;
  static constexpr uint32_t kTmemCols = 512;
  static constexpr uint32_t kColS = 0;    // S buffers at columns 0 and 128
  static constexpr uint32_t kColO = 256;  // O at columns 256 .. 256 + D
};

struct TcArgs {
  CacheView cache;
  BatchView batch;
  const WorkItem* items;
  __nv_bfloat16* out;
  float* part_o;
  float* part_ml;
  int Hq;
  int g;
  float scale_log2;
  int window;
};

__device__ __forceinline__ bool wait_or_flag(uint64_t* bar, uint32_t parity, int32_t* err, bool& ok) {
  if (!ok) return false;
  if (!ptx::mbar_wait_bounded(bar, parity, kWaitLimit)) {
    atomicOr(err, kErrTimeout);
    ok = false;
  }
  return ok;
}

template <int D>
__global__ void __launch_bounds__(192, 1) attn_tc_kernel(const __grid_constant__ CUtensorMap tm_q,
                                                        const __grid_constant__ CUtensorMap tm_kv,
                                                        TcArgs a) {
  using C = TcCfg<D>;
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  unsigned char* smem = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  unsigned char* sQ = smem + C::kOffQ;
  unsigned char* sK = smem + C::kOffK;
  unsigned char* sV = smem + C::kOffV;
  unsigned char* sP = smem + C::kOffP;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::kOffBar);
  uint64_t* q_full = bars;
  uint64_t* k_full = q_full + 1;
  uint64_t* k_empty = k_full + C::KST;
  uint64_t* v_full = k_empty + C::KST;
  uint64_t* v_empty = v_full + C::VST;
  uint64_t* s_full = v_empty + C::VST;
  uint64_t* s_free = s_full + 2;
  uint64_t* p_full = s_free + 2;
  uint64_t* pv_done = p_full + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + C::kNumBars);

  const WorkItem it = a.items[blockIdx.x];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int s = it.seq, h = it.kv_head, g = a.g;
  const int ctx = a.batch.ctx[s];
  const int L = ctx + (a.batch.cu_q[s + 1] - a.batch.cu_q[s]);
  const int kb = it.key_begin, ke = it.key_end;
  const int k00 = kb - (kb & 63);
  const int n_tiles = (ke - k00 + C::BN - 1) / C::BN;
  int32_t* err = a.batch.err;

  if (threadIdx.x == 0) {
    ptx::mbar_init(q_full, 1);
    for (int i = 0; i < C::KST; ++i) {
      ptx::mbar_init(&k_full[i], 1);
      ptx::mbar_init(&k_empty[i], 1);
    }
    for (int i = 0; i < C::VST; ++i) {
      ptx::mbar_init(&v_full[i], 1);
      ptx::mbar_init(&v_empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      ptx::mbar_init(&s_full[i], 1);
      ptx::mbar_init(&s_free[i], 4);
    }
    ptx::mbar_init(p_full, 4);
    ptx::mbar_init(pv_done, 1);
    ptx::fence_mbar_init();
  }
  if (warp == 5) {
    ptx::tmem_alloc(tmem_slot, C::kTmemCols);
    ptx::tmem_relinquish();
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  bool ok = true;

  if (warp == 4) {
    // ---------------------------------------------------------------- TMA
    if (lane == 0) {
      const int row0 = a.batch.cu_q[s] + it.tok_begin;
      ptx::mbar_arrive_expect_tx(q_full, C::kQBytes);
#pragma unroll
      for (int dh = 0; dh < C::DH; ++dh)
        ptx::tma_load_3d(sQ + dh * C::BM * 128, &tm_q, dh * 64, h * g, row0, q_full);
      const int32_t* bt = a.batch.bt + a.batch.bt_off[s];
      const int nb = a.batch.bt_off[s + 1] - a.batch.bt_off[s];
      const int B = a.cache.block_size;
      const int BR = B < 64 ? B : 64;
      const int Hkv = a.cache.n_kv_heads;
      for (int i = 0; i < n_tiles && ok; ++i) {
        const int k0 = k00 + i * C::BN;
        uint32_t bytes = 0;
        for (int pos = k0; pos < k0 + C::BN; pos += BR) {
          const int lb = pos / B;
          if (lb < nb && bt[lb] >= 0 && bt[lb] < a.cache.n_blocks) bytes += BR * 128 * C::DH;
        }
        const int ks = i % C::KST, vs = i % C::VST;
        if (i >= C::KST && !wait_or_flag(&k_empty[ks], ((i / C::KST) - 1) & 1, err, ok)) break;
        ptx::mbar_arrive_expect_tx(&k_full[ks], bytes);
        for (int pos = k0; pos < k0 + C::BN; pos += BR) {
          const int lb = pos / B;
          if (lb >= nb) continue;
          const int32_t blk = bt[lb];
          if (blk < 0 || blk >= a.cache.n_blocks) {
            atomicOr(err, kErrBadBlock);
            continue;
          }
          const int row = (int)(((int64_t)blk * 2 * Hkv + h) * B + (pos - lb * B));
#pragma unroll
          for (int dh = 0; dh < C::DH; ++dh)
            ptx::tma_load_2d(sK + ks * C::kKVBytes + dh * C::BN * 128 + (pos - k0) * 128, &tm_kv, dh * 64,
                             row, &k_full[ks]);
        }
        if (i >= C::VST && !wait_or_flag(&v_empty[vs], ((i / C::VST) - 1) & 1, err, ok)) break;
        ptx::mbar_arrive_expect_tx(&v_full[vs], bytes);
        for (int pos = k0; pos < k0 + C::BN; pos += BR) {
          const int lb = pos / B;
          if (lb >= nb) continue;
          const int32_t blk = bt[lb];
          if (blk < 0 || blk >= a.cache.n_blocks) continue;
          const int row = (int)((((int64_t)blk * 2 + 1) * Hkv + h) * B + (pos - lb * B));
#pragma unroll
          for (int dh = 0; dh < C::DH; ++dh)
            ptx::tma_load_2d(sV + vs * C::kKVBytes + dh * C::BN * 128 + (pos - k0) * 128, &tm_kv, dh * 64,
                             row, &v_full[vs]);
        }
      }
      // let in-flight loads land before the CTA can exit
      for (int i = max(0, n_tiles - C::KST); i < n_tiles && ok; ++i)
        wait_or_flag(&k_full[i % C::KST], (i / C::KST) & 1, err, ok);
      for (int i = max(0, n_tiles - C::VST); i < n_tiles && ok; ++i)
        wait_or_flag(&v_full[i % C::VST], (i / C::VST) & 1, err, ok);
    }
  } else if (warp == 5) {
    // ---------------------------------------------------------------- MMA
    if (lane == 0) {
      constexpr uint32_t idesc_qk = ptx::idesc_bf16_f32(C::BM, C::BN, 0, 0);
      constexpr uint32_t idesc_pv = ptx::idesc_bf16_f32(C::BM, D, 0, 1);
      const uint32_t q_addr = ptx::smem_u32(sQ), k_addr = ptx::smem_u32(sK);
      const uint32_t v_addr = ptx::smem_u32(sV), p_addr = ptx::smem_u32(sP);
      auto issue_pv = [&](int j) {
        const int vs = j % C::VST;
        if (!wait_or_flag(&v_full[vs], (j / C::VST) & 1, err, ok)) return;
        if (!wait_or_flag(p_full, j & 1, err, ok)) return;
        ptx::tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < C::BN / 16; ++kk) {
          const uint64_t ad = ptx::smem_desc_sw128(p_addr + (kk >> 2) * C::BM * 128 + (kk & 3) * 32, 16, 1024);
          const uint64_t bd = ptx::smem_desc_sw128(v_addr + vs * C::kKVBytes + kk * 16 * 128, C::BN * 128, 1024);
          ptx::mma_bf16(tmem + C::kColO, ad, bd, idesc_pv, (j > 0 || kk > 0) ? 1u : 0u);
        }
        ptx::mma_commit(pv_done);
        ptx::mma_commit(&v_empty[vs]);
      };
      wait_or_flag(q_full, 0, err, ok);
      for (int i = 0; i < n_tiles && ok; ++i) {
        const int ks = i % C::KST, sb = i & 1;
        if (!wait_or_flag(&k_full[ks], (i / C::KST) & 1, err, ok)) break;
        if (i >= 2 && !wait_or_flag(&s_free[sb], ((i >> 1) - 1) & 1, err, ok)) break;
        ptx::tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (kk >> 2) * C::BM * 128 + (kk & 3) * 32;
          const uint64_t ad = ptx::smem_desc_sw128(q_addr + off, 16, 1024);
          const uint64_t bd = ptx::smem_desc_sw128(k_addr + ks * C::kKVBytes + (kk >> 2) * C::BN * 128 + (kk & 3) * 32,
                                                   16, 1024);
          ptx::mma_bf16(tmem + C::kColS + sb * C::BN, ad, bd, idesc_qk, kk > 0 ? 1u : 0u);
        }
        ptx::mma_commit(&s_full[sb]);
        ptx::mma_commit(&k_empty[ks]);
        if (i >= 1) issue_pv(i - 1);
      }
      if (ok && n_tiles > 0) issue_pv(n_tiles - 1);
    }
  } else {
    // ---------------------------------------------------- softmax / epilogue
    const int r = threadIdx.x;  // query row == TMEM lane
    const uint32_t lane_base = (uint32_t)(warp * 32) << 16;
    const int R = it.n_rows;
    const bool row_ok = r < R;
    const int p_r = ctx + it.tok_begin + r / g;
    int lower = 0, upper = 0;
    if (row_ok) {
      lower = max(kb, a.window > 0 ? p_r - a.window + 1 : 0);
      upper = min(ke, p_r + 1);
    }
    const bool warp_live = (warp * 32) < R;
    float m_used = -INFINITY, l = 0.f;
    for (int i = 0; i < n_tiles; ++i) {
      const int sb = i & 1;
      const int k0 = k00 + i * C::BN;
      if (!warp_live) {
        // rows of this warp are padding: release S at once, provide no P
        if (!wait_or_flag(&s_full[sb], (i >> 1) & 1, err, ok)) break;
        if (lane == 0) ptx::mbar_arrive(&s_free[sb]);
        if (i >= 1 && !wait_or_flag(pv_done, (i - 1) & 1, err, ok)) break;
        if (lane == 0) ptx::mbar_arrive(p_full);
        continue;
      }
      if (!wait_or_flag(&s_full[sb], (i >> 1) & 1, err, ok)) break;
      ptx::tc_fence_after();
      float sv[C::BN];
#pragma unroll
      for (int c = 0; c < C::BN / 32; ++c) {
        uint32_t raw[32];
        ptx::tmem_ld32(tmem + lane_base + C::kColS + sb * C::BN + c * 32, raw);
        ptx::tmem_ld_wait();
#pragma unroll
        for (int e = 0; e < 32; ++e) sv[c * 32 + e] = __uint_as_float(raw[e]);
      }
      ptx::tc_fence_before();
      __syncwarp();
      if (lane == 0) ptx::mbar_arrive(&s_free[sb]);
      // mask and tile max
      const int c_lo = lower - k0, c_hi = upper - k0;
      float mt = -INFINITY;
      if (c_lo <= 0 && c_hi >= C::BN) {
#pragma unroll
        for (int c = 0; c < C::BN; ++c) mt = fmaxf(mt, sv[c]);
      } else {
#pragma unroll
        for (int c = 0; c < C::BN; ++c) {
          sv[c] = (c >= c_lo && c < c_hi) ? sv[c] : -INFINITY;
          mt = fmaxf(mt, sv[c]);
        }
      }
      const float mts = mt == -INFINITY ? -INFINITY : mt * a.scale_log2;
      float alpha = 1.f;
      if (mts > m_used + 8.f) {  // also true the first time a row sees a key
        alpha = m_used == -INFINITY ? 0.f : exp2f(m_used - mts);
        m_used = mts;
        l *= alpha;
      }
      // wait until PV of the previous tile is done: O may then be rescaled and
      // the single P buffer rewritten
      if (i >= 1 && !wait_or_flag(pv_done, (i - 1) & 1, err, ok)) break;
      ptx::tc_fence_after();
      if (i >= 1 && __any_sync(0xffffffffu, alpha != 1.f)) {
#pragma unroll
        for (int c = 0; c < D / 32; ++c) {
          uint32_t raw[32];
          const uint32_t ta = tmem + lane_base + C::kColO + c * 32;
          ptx::tmem_ld32(ta, raw);
          ptx::tmem_ld_wait();
#pragma unroll
          for (int e = 0; e < 32; ++e) raw[e] = __float_as_uint(__uint_as_float(raw[e]) * alpha);
          ptx::tmem_st32(ta, raw);
        }
        ptx::tmem_st_wait();
      }
      // P = 2^(s*scale - m_used) as bf16 into the 128-byte-swizzled layout:
      // key c of row r sits in atom c/64, row r, chunk ((c%64)/8) ^ (r%8)
      float ls = 0.f;
      const float neg_m = m_used == -INFINITY ? 0.f : -m_used;
      const bool none = m_used == -INFINITY;
#pragma unroll
      for (int ch = 0; ch < C::BN / 8; ++ch) {
        uint32_t w[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float x0 = sv[ch * 8 + 2 * e], x1 = sv[ch * 8 + 2 * e + 1];
          const float p0 = none ? 0.f : exp2f(fmaf(x0, a.scale_log2, neg_m));
          const float p1 = none ? 0.f : exp2f(fmaf(x1, a.scale_log2, neg_m));
          ls += p0 + p1;
          __nv_bfloat162 pr = __floats2bfloat162_rn(p0, p1);
          w[e] = *reinterpret_cast<uint32_t*>(&pr);
        }
        const int atom = ch >> 3, cin = ch & 7;
        unsigned char* dst = sP + atom * C::BM * 128 + r * 128 + ((cin ^ (r & 7)) << 4);
        *reinterpret_cast<uint4*>(dst) = make_uint4(w[0], w[1], w[2], w[3]);
      }
      l += ls;
      // keys at or past the sequence end may hold anything (unwritten slots,
      // stale stage data): zero those V rows so 0 * garbage cannot reach O
      if (k0 + C::BN > L) {
        const int vs = i % C::VST;
        if (!wait_or_flag(&v_full[vs], (i / C::VST) & 1, err, ok)) break;
        const int z0 = max(0, L - k0);
        const int nz = (C::BN - z0) * 8 * C::DH;  // 16-byte chunks to clear
        const int n_live = min(C::BM, (R + 31) & ~31);  // threads of the live warps
        for (int z = threadIdx.x; z < nz; z += n_live) {
          const int dh = z / ((C::BN - z0) * 8), rem = z % ((C::BN - z0) * 8);
          const int row = z0 + rem / 8, chn = rem % 8;
          *reinterpret_cast<uint4*>(sV + vs * C::kKVBytes + dh * C::BN * 128 + row * 128 + chn * 16) =
              make_uint4(0, 0, 0, 0);
        }
      }
      ptx::fence_proxy_async_smem();
      ptx::tc_fence_before();
      __syncwarp();
      if (lane == 0) ptx::mbar_arrive(p_full);
    }
    // epilogue: wait for the last PV, normalise, store
    if (n_tiles > 0) wait_or_flag(pv_done, (n_tiles - 1) & 1, err, ok);
    ptx::tc_fence_after();
    if (ok && warp_live) {
      const int row = a.batch.cu_q[s] + it.tok_begin + r / g;
      const int qh = h * g + (r % g);
      const float inv = l > 0.f ? 1.f / l : 0.f;
#pragma unroll
      for (int c = 0; c < D / 32; ++c) {
        uint32_t raw[32];
        ptx::tmem_ld32(tmem + lane_base + C::kColO + c * 32, raw);
        ptx::tmem_ld_wait();
        if (!row_ok) continue;
        if (it.part < 0) {
          uint4* dst = reinterpret_cast<uint4*>(a.out + ((int64_t)row * a.Hq + qh) * D + c * 32);
#pragma unroll
          for (int q4 = 0; q4 < 4; ++q4) {
            uint32_t w[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              __nv_bfloat162 pr = __floats2bfloat162_rn(__uint_as_float(raw[q4 * 8 + 2 * e]) * inv,
                                                        __uint_as_float(raw[q4 * 8 + 2 * e + 1]) * inv);
              w[e] = *reinterpret_cast<uint32_t*>(&pr);
            }
            dst[q4] = make_uint4(w[0], w[1], w[2], w[3]);
          }
        } else {
          float4* dst = reinterpret_cast<float4*>(a.part_o + (int64_t)(it.part + r) * D + c * 32);
#pragma unroll
          for (int q4 = 0; q4 < 8; ++q4)
            dst[q4] = make_float4(__uint_as_float(raw[4 * q4]), __uint_as_float(raw[4 * q4 + 1]),
                                  __uint_as_float(raw[4 * q4 + 2]), __uint_as_float(raw[4 * q4 + 3]));
        }
      }
      if (row_ok && it.part >= 0) {
        a.part_ml[(int64_t)(it.part + r) * 2] = m_used;
        a.part_ml[(int64_t)(it.part + r) * 2 + 1] = l;
      }
    }
  }
  ptx::tc_fence_before();
  __syncthreads();
  if (warp == 5) {
    ptx::tc_fence_after();
    ptx::tmem_dealloc(tmem, C::kTmemCols);
  }
}

template <int D>
cudaError_t launch_tc_d(const CUtensorMap& tm_q, const CUtensorMap& tm_kv, const TcArgs& args,
                        int n_items, cudaStream_t stream) {
  using C = TcCfg<D>;
  static bool configured = false;
  if (!configured) {
    cudaError_t e = cudaFuncSetAttribute(attn_tc_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         C::kSmem);
    if (e != cudaSuccess) return e;
    configured = true;
  }
  attn_tc_kernel<D><<<n_items, C::kThreads, C::kSmem, stream>>>(tm_q, tm_kv, args);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_attention_tc(const void* tm_q, const void* tm_kv, const CacheView& cache,
                                const BatchView& batch, const WorkItem* items, int n_items,
                                __nv_bfloat16* out, float* part_o, float* part_ml, int n_q_heads,
                                int g, float scale_log2, int window, cudaStream_t stream) {
  if (n_items == 0) return cudaSuccess;
  TcArgs args{cache, batch, items, out, part_o, part_ml, n_q_heads, g, scale_log2, window};
  const CUtensorMap& q = *static_cast<const CUtensorMap*>(tm_q);
  const CUtensorMap& kv = *static_cast<const CUtensorMap*>(tm_kv);
  if (cache.head_dim == 128) return launch_tc_d<128>(q, kv, args, n_items, stream);
  return launch_tc_d<64>(q, kv, args, n_items, stream);
}

}  // namespace fg
