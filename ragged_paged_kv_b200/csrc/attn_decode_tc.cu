// Decode attention on the tensor cores, keys on the MMA's M side.
//
// A unit is one new token of one sequence with the g query heads that share
// one kv head (g <= 16, d = 128), over a range of its cached keys. For every
// 128-key stage the kernel computes the transposed scores and output:
//
//   S^T [128 keys x 16]  = K [128 keys x d] . Q^T        (A = K tile, K-major)
//   O^T [d x 16]        += V^T [d x 128 keys] . P^T      (A = V tile, MN-major)
//
// with the g query heads as the N = 16 columns (padding columns are never
// read). K and V come straight from the paged cache tiles by 2-D TMA boxes,
// so the only per-key work left on the CUDA cores is one score per (key,
// head): thread t of the softmax warpgroup owns key t of the stage (TMEM lane
// t of S^T) and, in the epilogue, output dim t (lane t of O^T). Column maxima
// over the 128 keys are reduced with shuffles plus one rendezvous of the four
// warps on an mbarrier (bounded, where bar.sync would not be); the
// running max per head moves (with a rescale of O^T in TMEM) only when a
// stage raises it by more than 2^8; per-thread partial sums are reduced once
// per unit.
//
// The kernel is persistent, two CTAs per SM (about 109 KB of shared memory
// and 64 TMEM columns each): the TMA warp takes units from a global counter
// over a longest-first list and hands them to the other roles through a
// small queue, and K and V stream through one ring of 32 KB slots (K and V
// of a stage take consecutive slots). Launched behind the query-tile kernel
// with programmatic dependent launch, its CTAs take SMs as that kernel's
// CTAs leave; it does not read that kernel's results, but waits for it
// before its own CTAs end so that the combine launched behind it sees both.
// Every wait is bounded.
#include <cuda.h>

#include <cfloat>

#include "fg_internal.h"
#include "sm100_ptx.cuh"

namespace fg {
namespace {

constexpr long long kWaitLimit = 1LL << 31;

struct DtcCfg {
  static constexpr int D = 128;
  static constexpr int BK = 128;  // keys per stage (MMA M)
  static constexpr int N = 16;    // query columns (MMA N)
  static constexpr int NSLOT = 3;
  static constexpr int kSlotBytes = BK * D * 2;  // K or V of one stage, [d half][128 keys][128 B]
  static constexpr int kQBytes = N * D * 2;      // [d half][16 rows][128 B]
  static constexpr int kPBytes = N * BK * 2;     // [key half][16 rows][128 B]
  static constexpr int kOffSlot = 0;
  static constexpr int kOffQ = kOffSlot + NSLOT * kSlotBytes;
  static constexpr int kOffP = kOffQ + kQBytes;             // two P buffers
  static constexpr int kOffRed = kOffP + 2 * kPBytes;       // [2][4 warps][16] floats
  static constexpr int kOffBar = kOffRed + 2 * 4 * N * 4;
  // q_full, q_empty, slot_full[NSLOT], slot_empty[NSLOT], s_full[2], s_free[2],
  // p_full[2], pv_done[2], o_free, red_bar
  static constexpr int kNumBars = 2 + 2 * NSLOT + 2 + 2 + 2 + 2 + 1 + 1 + 2 * UnitQueue::kDepth;
  static constexpr int kSmem = kOffBar + kNumBars * 8 + 16 + UnitQueue::kDepth * 4;
  static constexpr int kThreads = 192;
  static constexpr uint32_t kTmemCols = 64;
  static constexpr uint32_t kColS = 0;   // S^T buffers at columns 0 and 16
  static constexpr uint32_t kColO = 32;  // O^T at columns 32 .. 47
};

struct DtcArgs {
  CacheView cache;
  BatchView batch;
  const WorkItem* items;
  __nv_bfloat16* out;
  float* part_o;
  float* part_ml;
  int Hq;
  int g;
  float scale_log2;
  int n_items;
  int* counter;  // next-unit counter, zero at launch
  // When the query-tile kernel runs beside this one on SMs [0, sm_tc_end):
  // a CTA placed there while query tiles are still unclaimed leaves at once
  // (the SM belongs to that kernel); one placed there later helps here.
  int sm_tc_end;
  const int* tc_counter;
  int n_tc;
};

__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ bool wait_or_flag(uint64_t* bar, uint32_t parity, int32_t* err, bool& ok) {
  if (!ok) return false;
  if (!ptx::mbar_wait_bounded(bar, parity, kWaitLimit)) {
    atomicOr(err, kErrTimeout);
    ok = false;
  }
  return ok;
}

// 16 consecutive 32-bit TMEM columns of this warp's 32 lanes.
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, "
      "%13, %14, %15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]),
        "=r"(r[15])
      : "r"(taddr));
}
__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, "
      "%13, %14, %15, %16};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]),
      "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15])
      : "memory");
}


__global__ void __launch_bounds__(192, 2) attn_decode_tc_kernel(const __grid_constant__ CUtensorMap tm_q,
                                                               const __grid_constant__ CUtensorMap tm_kv,
                                                               DtcArgs a) {
  using C = DtcCfg;
  constexpr int D = C::D;
  extern __shared__ __align__(1024) unsigned char smem[];
  if (ptx::sm_id() < a.sm_tc_end && *(volatile const int*)a.tc_counter < a.n_tc) return;
  if (ptx::smem_u32(smem) & 1023u) {
    if (threadIdx.x == 0) atomicOr(a.batch.err, kErrBadIndex);
    return;
  }
  unsigned char* sSlot = smem + C::kOffSlot;
  unsigned char* sQ = smem + C::kOffQ;
  unsigned char* sP = smem + C::kOffP;
  float* red = reinterpret_cast<float*>(smem + C::kOffRed);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::kOffBar);
  uint64_t* q_full = bars;
  uint64_t* q_empty = q_full + 1;
  uint64_t* slot_full = q_empty + 1;
  uint64_t* slot_empty = slot_full + C::NSLOT;
  uint64_t* s_full = slot_empty + C::NSLOT;
  uint64_t* s_free = s_full + 2;
  uint64_t* p_full = s_free + 2;
  uint64_t* pv_done = p_full + 2;
  uint64_t* o_free = pv_done + 2;
  uint64_t* red_bar = o_free + 1;  // rendezvous of the four softmax warps
  uint64_t* uq_full = red_bar + 1;
  uint64_t* uq_empty = uq_full + UnitQueue::kDepth;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + C::kNumBars);
  const UnitQueue uq{reinterpret_cast<int32_t*>(tmem_slot + 4), uq_full, uq_empty, 5};

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = a.g;
  int32_t* err = a.batch.err;

  if (threadIdx.x == 0) {
    ptx::mbar_init(q_full, 1);
    ptx::mbar_init(q_empty, 1);
    for (int i = 0; i < C::NSLOT; ++i) {
      ptx::mbar_init(&slot_full[i], 1);
      ptx::mbar_init(&slot_empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      ptx::mbar_init(&s_full[i], 1);
      ptx::mbar_init(&s_free[i], 4);
      ptx::mbar_init(&p_full[i], 4);
      ptx::mbar_init(&pv_done[i], 1);
    }
    ptx::mbar_init(o_free, 4);
    ptx::mbar_init(red_bar, 4);
    uq.init();
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
      const int B = a.cache.block_size;
      const int BR = B < 64 ? B : 64;
      const int Hkv = a.cache.n_kv_heads;
      // each key's K and V is read by one unit only: evict those lines first
      const uint64_t l2_once = ptx::l2_evict_first_policy();
      int gt = 0, un = 0;
      for (;; ++un) {
        int u = -1;
        if (!uq.push_next(un, a.counter, a.n_items, kWaitLimit, &u)) {
          atomicOr(err, kErrTimeout);
          ok = false;
        }
        if (u < 0 || !ok) break;
        const WorkItem it = a.items[u];
        const int s = it.seq, h = it.kv_head;
        const int row = a.batch.cu_q[s] + it.tok_begin;
        const int k00 = it.key_begin - (it.key_begin & 63);
        const int n_st = (it.key_end - k00 + C::BK - 1) / C::BK;
        if (un >= 1 && !wait_or_flag(q_empty, (un - 1) & 1, err, ok)) break;
        ptx::mbar_arrive_expect_tx(q_full, 2 * g * 128);
        ptx::tma_load_3d(sQ, &tm_q, 0, h * g, row, q_full);
        ptx::tma_load_3d(sQ + C::N * 128, &tm_q, 64, h * g, row, q_full);
        const int32_t* bt = a.batch.bt + a.batch.bt_off[s];
        const int nb = a.batch.bt_off[s + 1] - a.batch.bt_off[s];
        for (int i = 0; i < n_st && ok; ++i, ++gt) {
          const int k0 = k00 + i * C::BK;
          uint32_t bytes = 0;
          for (int pos = k0; pos < k0 + C::BK; pos += BR) {
            const int lb = pos / B;
            if (lb < nb && bt[lb] >= 0 && bt[lb] < a.cache.n_blocks) bytes += BR * 256;
          }
          for (int kv = 0; kv < 2 && ok; ++kv) {
            const int use = 2 * gt + kv, slot = use % C::NSLOT;
            if (use >= C::NSLOT && !wait_or_flag(&slot_empty[slot], ((use / C::NSLOT) - 1) & 1, err, ok))
              break;
            ptx::mbar_arrive_expect_tx(&slot_full[slot], bytes);
            unsigned char* dst = sSlot + slot * C::kSlotBytes;
            for (int pos = k0; pos < k0 + C::BK; pos += BR) {
              const int lb = pos / B;
              if (lb >= nb) continue;
              const int32_t blk = bt[lb];
              if (blk < 0 || blk >= a.cache.n_blocks) {
                if (kv == 0) atomicOr(err, kErrBadBlock);
                continue;
              }
              const int r0 = (int)((((int64_t)blk * 2 + kv) * Hkv + h) * B + (pos - lb * B));
              ptx::tma_load_2d_hint(dst + (pos - k0) * 128, &tm_kv, 0, r0, &slot_full[slot], l2_once);
              ptx::tma_load_2d_hint(dst + C::BK * 128 + (pos - k0) * 128, &tm_kv, 64, r0, &slot_full[slot], l2_once);
            }
          }
        }
      }
      for (int use = max(0, 2 * gt - C::NSLOT); use < 2 * gt && ok; ++use)
        wait_or_flag(&slot_full[use % C::NSLOT], (use / C::NSLOT) & 1, err, ok);
      if (un >= 1) wait_or_flag(q_full, (un - 1) & 1, err, ok);
    }
  } else if (warp == 5) {
    // ---------------------------------------------------------------- MMA
    if (lane == 0) {
      constexpr uint32_t idesc_s = ptx::idesc_bf16_f32(C::BK, C::N, 0, 0);  // K . Q^T
      constexpr uint32_t idesc_o = ptx::idesc_bf16_f32(D, C::N, 1, 0);      // V^T . P^T
      const uint32_t slot_addr = ptx::smem_u32(sSlot), q_addr = ptx::smem_u32(sQ);
      const uint32_t p_addr = ptx::smem_u32(sP);
      int gt = 0, un = 0;
      auto issue_pv = [&](int t, bool first) {
        const int use = 2 * t + 1, slot = use % C::NSLOT, pb = t & 1;
        if (!wait_or_flag(&slot_full[slot], (use / C::NSLOT) & 1, err, ok)) return;
        if (!wait_or_flag(&p_full[pb], (t >> 1) & 1, err, ok)) return;
        if (first && un >= 1 && !wait_or_flag(o_free, (un - 1) & 1, err, ok)) return;
        ptx::tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < C::BK / 16; ++kk) {
          const uint64_t ad =
              ptx::smem_desc_sw128(slot_addr + slot * C::kSlotBytes + kk * 16 * 128, C::BK * 128, 1024);
          const uint64_t bd = ptx::smem_desc_sw128(
              p_addr + pb * C::kPBytes + (kk >> 2) * C::N * 128 + (kk & 3) * 32, 16, 1024);
          ptx::mma_bf16(tmem + C::kColO, ad, bd, idesc_o, (!first || kk > 0) ? 1u : 0u);
        }
        ptx::mma_commit(&pv_done[pb]);
        ptx::mma_commit(&slot_empty[slot]);
      };
      for (;; ++un) {
        int u = -1;
        if (!uq.pop(un, false, kWaitLimit, &u)) {
          atomicOr(err, kErrTimeout);
          ok = false;
        }
        if (u < 0 || !ok) break;
        const WorkItem it = a.items[u];
        const int k00 = it.key_begin - (it.key_begin & 63);
        const int n_st = (it.key_end - k00 + C::BK - 1) / C::BK;
        if (!wait_or_flag(q_full, un & 1, err, ok)) break;
        const int gt0 = gt;
        for (int i = 0; i < n_st && ok; ++i, ++gt) {
          const int use = 2 * gt, slot = use % C::NSLOT, sb = gt & 1;
          if (!wait_or_flag(&slot_full[slot], (use / C::NSLOT) & 1, err, ok)) break;
          if (gt >= 2 && !wait_or_flag(&s_free[sb], ((gt >> 1) - 1) & 1, err, ok)) break;
          ptx::tc_fence_after();
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const uint32_t off_k = (kk >> 2) * C::BK * 128 + (kk & 3) * 32;
            const uint32_t off_q = (kk >> 2) * C::N * 128 + (kk & 3) * 32;
            const uint64_t ad = ptx::smem_desc_sw128(slot_addr + slot * C::kSlotBytes + off_k, 16, 1024);
            const uint64_t bd = ptx::smem_desc_sw128(q_addr + off_q, 16, 1024);
            ptx::mma_bf16(tmem + C::kColS + sb * C::N, ad, bd, idesc_s, kk > 0 ? 1u : 0u);
          }
          ptx::mma_commit(&s_full[sb]);
          ptx::mma_commit(&slot_empty[slot]);
          if (i == n_st - 1) ptx::mma_commit(q_empty);
          if (i >= 1) issue_pv(gt - 1, i == 1);
        }
        if (ok) issue_pv(gt - 1, gt - 1 == gt0);
      }
    }
  } else {
    // ------------------------------------------- softmax over keys / epilogue
    const int t = threadIdx.x;  // key t of a stage; output dim t in the epilogue
    const uint32_t lane_base = (uint32_t)(warp * 32) << 16;
    // all four warps meet here (bounded, unlike bar.sync)
    uint32_t red_phase = 0;
    auto rendezvous = [&]() -> bool {
      __syncwarp();
      if (lane == 0) ptx::mbar_arrive(red_bar);
      return wait_or_flag(red_bar, (red_phase++) & 1, err, ok);
    };
    int gt = 0, un = 0;
    for (;; ++un) {
      int u = -1;
      if (!uq.pop(un, true, kWaitLimit, &u)) {
        if (lane == 0) atomicOr(err, kErrTimeout);
        ok = false;
      }
      if (u < 0 || !ok) break;
      const WorkItem it = a.items[u];
      const int s = it.seq;
      const int ctx = a.batch.ctx[s];
      const int L = ctx + (a.batch.cu_q[s + 1] - a.batch.cu_q[s]);
      const int kb = it.key_begin, ke = it.key_end;
      const int k00 = kb - (kb & 63);
      const int n_st = (ke - k00 + C::BK - 1) / C::BK;
      float m_used[C::N], lp[C::N];
#pragma unroll
      for (int j = 0; j < C::N; ++j) {
        m_used[j] = -INFINITY;
        lp[j] = 0.f;
      }
      for (int i = 0; i < n_st && ok; ++i, ++gt) {
        const int sb = gt & 1, pb = gt & 1;
        const int k0 = k00 + i * C::BK;
        if (!wait_or_flag(&s_full[sb], (gt >> 1) & 1, err, ok)) break;
        ptx::tc_fence_after();
        uint32_t raw[C::N];
        tmem_ld16(tmem + lane_base + C::kColS + sb * C::N, raw);
        ptx::tmem_ld_wait();
        ptx::tc_fence_before();
        __syncwarp();
        if (lane == 0) ptx::mbar_arrive(&s_free[sb]);
        const int key = k0 + t;
        const bool valid = key >= kb && key < ke;
        float sc[C::N];
        float* rd = red + (gt & 1) * 4 * C::N;
#pragma unroll
        for (int j = 0; j < C::N; ++j) {
          if (j >= g) break;
          sc[j] = valid ? __uint_as_float(raw[j]) : -INFINITY;
          float m = sc[j];
#pragma unroll
          for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
          if (lane == 0) rd[warp * C::N + j] = m;
        }
        if (!rendezvous()) break;
        float alpha[C::N];
        bool rescale = false;
#pragma unroll
        for (int j = 0; j < C::N; ++j) {
          alpha[j] = 1.f;
          if (j >= g) break;
          const float mt = fmaxf(fmaxf(rd[j], rd[C::N + j]), fmaxf(rd[2 * C::N + j], rd[3 * C::N + j]));
          const float mts = mt == -INFINITY ? -INFINITY : mt * a.scale_log2;
          if (mts > m_used[j] + 8.f) {  // identical in every thread
            alpha[j] = m_used[j] == -INFINITY ? 0.f : ex2(m_used[j] - mts);
            m_used[j] = mts;
            lp[j] *= alpha[j];
            rescale = true;
          }
        }
        // O^T may be rescaled only after the previous PV; P buffer pb only
        // after the PV two stages back
        if (gt >= 2 && !wait_or_flag(&pv_done[pb], ((gt >> 1) - 1) & 1, err, ok)) break;
        if (rescale && i >= 1) {
          if (!wait_or_flag(&pv_done[(gt - 1) & 1], ((gt - 1) >> 1) & 1, err, ok)) break;
          ptx::tc_fence_after();
          uint32_t o[C::N];
          tmem_ld16(tmem + lane_base + C::kColO, o);
          ptx::tmem_ld_wait();
#pragma unroll
          for (int j = 0; j < C::N; ++j) o[j] = __float_as_uint(__uint_as_float(o[j]) * alpha[j]);
          tmem_st16(tmem + lane_base + C::kColO, o);
          ptx::tmem_st_wait();
        }
        // P^T[j][key t] = 2^(s*scale - m_used_j) as bf16, 128-byte-swizzled
        // K-major rows of 128 keys: key half t/64, row j, chunk ((t%64)/8)^(j%8)
        unsigned char* pbase = sP + pb * C::kPBytes + (t >> 6) * C::N * 128 + (t & 7) * 2;
        const int chunk = (t & 63) >> 3;
#pragma unroll
        for (int j = 0; j < C::N; ++j) {
          if (j >= g) break;
          const float neg_m = m_used[j] == -INFINITY ? 0.f : -m_used[j];
          const float p = ex2(fmaf(sc[j], a.scale_log2, neg_m));
          lp[j] += p;
          *reinterpret_cast<__nv_bfloat16*>(pbase + j * 128 + ((chunk ^ (j & 7)) << 4)) = __float2bfloat16_rn(p);
        }
        // V rows at or past the sequence end may hold anything: zero them
        if (k0 + C::BK > L) {
          const int use = 2 * gt + 1, slot = use % C::NSLOT;
          if (!wait_or_flag(&slot_full[slot], (use / C::NSLOT) & 1, err, ok)) break;
          const int z0 = max(0, L - k0);
          const int per_half = (C::BK - z0) * 8;
          for (int z = t; z < 2 * per_half; z += 128) {
            const int dh = z / per_half, rem = z - dh * per_half;
            *reinterpret_cast<uint4*>(sSlot + slot * C::kSlotBytes + dh * C::BK * 128 + (z0 + rem / 8) * 128 +
                                      (rem % 8) * 16) = make_uint4(0, 0, 0, 0);
          }
        }
        ptx::fence_proxy_async_smem();
        ptx::tc_fence_before();
        __syncwarp();
        if (lane == 0) ptx::mbar_arrive(&p_full[pb]);
      }
      if (!ok) break;
      // epilogue: row sums over the 128 key threads, then O^T / l
      float* rd = red + (gt & 1) * 4 * C::N;  // the buffer the next stage would use
#pragma unroll
      for (int j = 0; j < C::N; ++j) {
        if (j >= g) break;
        float v = lp[j];
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
        if (lane == 0) rd[warp * C::N + j] = v;
      }
      if (!rendezvous()) break;
      const int last = gt - 1;
      if (!wait_or_flag(&pv_done[last & 1], (last >> 1) & 1, err, ok)) break;
      ptx::tc_fence_after();
      uint32_t o[C::N];
      tmem_ld16(tmem + lane_base + C::kColO, o);
      ptx::tmem_ld_wait();
      const int row = a.batch.cu_q[s] + it.tok_begin;
#pragma unroll
      for (int j = 0; j < C::N; ++j) {
        if (j >= g) break;
        const float l = rd[j] + rd[C::N + j] + rd[2 * C::N + j] + rd[3 * C::N + j];
        const float v = __uint_as_float(o[j]);
        const int qh = it.kv_head * g + j;
        if (it.part < 0) {
          a.out[((int64_t)row * a.Hq + qh) * D + t] = __float2bfloat16_rn(l > 0.f ? v / l : 0.f);
        } else {
          a.part_o[(int64_t)(it.part + j) * D + t] = v;
          if (t == 0) {
            a.part_ml[(int64_t)(it.part + j) * 2] = m_used[j];
            a.part_ml[(int64_t)(it.part + j) * 2 + 1] = l;
          }
        }
      }
      // the reduction buffer is reused two stages on; make sure all reads of
      // it are done before anyone can get there
      if (!rendezvous()) break;
      ptx::tc_fence_before();
      __syncwarp();
      if (lane == 0) ptx::mbar_arrive(o_free);
    }
  }
  ptx::tc_fence_before();
  __syncthreads();
  if (warp == 5) {
    ptx::tc_fence_after();
    ptx::tmem_dealloc(tmem, C::kTmemCols);
  }
  // Launched behind the query-tile kernel (programmatic dependent launch),
  // this grid may start before that one ends; it does not read its results,
  // but a grid launched behind this one (the combine) must be able to rely
  // on both: so no CTA ends before the preceding grid has.
  ptx::grid_dependency_wait();
}

}  // namespace

cudaError_t launch_attention_decode_tc(const void* tm_q1, const void* tm_kv, const CacheView& cache,
                                       const BatchView& batch, const WorkItem* items, int n_items,
                                       __nv_bfloat16* out, float* part_o, float* part_ml, int n_q_heads,
                                       int g, float scale_log2, int grid, int* counter,
                                       int sm_tc_end, const int* tc_counter, int n_tc, bool pdl,
                                       cudaStream_t stream) {
  if (n_items == 0) return cudaSuccess;
  // per device: the attributes apply to the current device only
  static PerDeviceOnce configured;
  cudaError_t e0 = configured.run([] {
    cudaError_t e = cudaFuncSetAttribute(attn_decode_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, DtcCfg::kSmem);
    // the largest shared-memory carveout, so CTAs of different kernels can
    // share an SM
    if (e == cudaSuccess)
      e = cudaFuncSetAttribute(attn_decode_tc_kernel, cudaFuncAttributePreferredSharedMemoryCarveout,
                               cudaSharedmemCarveoutMaxShared);
    return e;
  });
  if (e0 != cudaSuccess) return e0;
  DtcArgs args{cache, batch, items, out, part_o, part_ml, n_q_heads, g, scale_log2, n_items, counter,
               sm_tc_end, tc_counter, n_tc};
  grid = grid < 1 ? 1 : (grid > n_items ? n_items : grid);
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(DtcCfg::kThreads);
  cfg.dynamicSmemBytes = DtcCfg::kSmem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, attn_decode_tc_kernel, *static_cast<const CUtensorMap*>(tm_q1),
                            *static_cast<const CUtensorMap*>(tm_kv), args);
}

}  // namespace fg
