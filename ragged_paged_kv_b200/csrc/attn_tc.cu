// Ragged paged attention on the 5th-generation tensor cores (tcgen05).
//
// A work unit is one 128-row query tile of one sequence and kv head: the
// rows are (token, q head of the group) pairs, 128/g consecutive new tokens
// times the g q heads that share the kv head, so a grouped-query tile reuses
// each K/V tile for all g heads. The kernel is persistent: the TMA warp takes
// units one by one from a global counter over a longest-first list and hands
// them to the other warps, and every role counts tiles globally, so the rings
// and barrier phases run on across units (the next unit's K/V stream in while
// the last one's epilogue runs). A unit walks its key range in 64-key tiles:
//
//   warp 4 (TMA)      Q once (3-D box: 64 dims x g heads x 128/g tokens), then
//                     K and V tiles through the block table, one 2-D box per
//                     (block part, 64 dims), into 3-stage K and 2-stage V
//                     rings;
//   warp 5 (MMA)      one thread issues S = Q K^T into one of two TMEM S
//                     tiles, and O += P V into the TMEM O tile with P read
//                     from tensor memory;
//   warps 0-3         thread r owns query row r (TMEM lane r): reads its S
//                     row with tcgen05.ld, masks (causal, window, unit range),
//                     keeps an online softmax (a running max that is only
//                     moved - with a rescale of its O row in TMEM - when a
//                     tile raises it by more than 2^8), writes P as packed
//                     bf16 back over the S tile it came from, and at the end
//                     normalises O and stores it.
//
// Keeping P in tensor memory makes it double-buffered with S for free: the
// softmax of tile i+1 never waits for the P.V product of tile i, and the S
// product of tile i+2, which overwrites that buffer, is issued right behind
// that P.V (the tensor core runs one thread's MMAs in issue order).
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
  static constexpr int BN = 64;   // keys per tile (two CTAs fit on one SM)
  // K is needed one tile earlier than V (the S product of tile i is issued
  // right behind the P.V of tile i-2), so its ring is one stage deeper: at
  // about 2 us of load latency two stages leave the MMA waiting for K
  static constexpr int KST = 3, VST = 2;
  static constexpr int DH = D / 64;  // 64-dim (128-byte) boxes per row
  static constexpr int kQBytes = BM * D * 2;
  static constexpr int kKVBytes = BN * D * 2;
  static constexpr int kOffQ = 0;
  static constexpr int kOffK = kOffQ + kQBytes;
  static constexpr int kOffV = kOffK + KST * kKVBytes;
  static constexpr int kOffBar = kOffV + VST * kKVBytes;
  // q_full, q_empty, k_full[KST], k_empty[KST], v_full[VST], v_empty[VST],
  // s_full[2], p_full[2], pv_done[2], o_free, unit queue full/empty
  static constexpr int kNumBars = 2 + 2 * KST + 2 * VST + 2 + 2 + 2 + 1 + 2 * UnitQueue::kDepth;
  static constexpr int kSmem = kOffBar + kNumBars * 8 + 16 + UnitQueue::kDepth * 4;
  static constexpr int kThreads = 192;
  static constexpr uint32_t kTmemCols = 256;
  static constexpr uint32_t kColS = 0;       // S (then P) buffers at columns 0 and BN
  static constexpr uint32_t kColO = 2 * BN;  // O at columns 2*BN .. 2*BN + D
  static_assert(kColO + D <= kTmemCols, "TMEM budget");
  // two CTAs per SM: 228 KB of shared memory per SM, 1 KB reserved per CTA
  static_assert(2 * (kSmem + 1024) <= 228 * 1024, "two CTAs must fit on one SM");
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
  int n_items;
  int* counter;  // next-unit counter, zero at launch
  int sm_end;    // only CTAs on SMs with id < sm_end take units (the others leave at once)
};

// What every role needs to know about one unit.
struct Unit {
  int s, h, ctx, L, kb, ke, k00, n_tiles, row0, tok_begin, R, part;
};

__device__ __forceinline__ Unit load_unit(const TcArgs& a, int u, int bn) {
  const WorkItem it = a.items[u];
  Unit x;
  x.s = it.seq;
  x.h = it.kv_head;
  x.ctx = a.batch.ctx[x.s];
  x.L = x.ctx + (a.batch.cu_q[x.s + 1] - a.batch.cu_q[x.s]);
  x.kb = it.key_begin;
  x.ke = it.key_end;
  x.k00 = x.kb - (x.kb & 63);
  x.n_tiles = (x.ke - x.k00 + bn - 1) / bn;
  x.tok_begin = it.tok_begin;
  x.row0 = a.batch.cu_q[x.s] + it.tok_begin;
  x.R = it.n_rows;
  x.part = it.part;
  return x;
}

// 2^x on the special-function unit (ex2.approx.ftz: max relative error about
// 2^-22; -inf gives +0). P is rounded to bf16 afterwards.
__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
// 3-input maximum (sm_100): one instruction for two comparisons.
__device__ __forceinline__ float max3(float a, float b, float c) {
  float m;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(m) : "f"(a), "f"(b), "f"(c));
  return m;
}
// D[tmem] (+)= A[tmem] * B[smem]: A is M x K bf16 packed two per 32-bit
// column (row m in lane m), B given by a matrix descriptor.
__device__ __forceinline__ void mma_bf16_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc, uint32_t idesc,
                                            uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
      "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

__device__ __forceinline__ bool wait_or_flag(uint64_t* bar, uint32_t parity, int32_t* err, bool& ok) {
  if (!ok) return false;
  if (!ptx::mbar_wait_bounded(bar, parity, kWaitLimit)) {
    atomicOr(err, kErrTimeout);
    ok = false;
  }
  return ok;
}

template <int D>
__global__ void __launch_bounds__(192, 2) attn_tc_kernel(const __grid_constant__ CUtensorMap tm_q,
                                                        const __grid_constant__ CUtensorMap tm_kv,
                                                        TcArgs a) {
  using C = TcCfg<D>;
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  unsigned char* smem = smem_raw;
  // SMs outside the kernel's share are left to the decode kernel
  if (ptx::sm_id() >= a.sm_end) return;
  // the swizzled tiles need 1024-byte alignment of the dynamic window
  if (ptx::smem_u32(smem_raw) & 1023u) {
    if (threadIdx.x == 0) atomicOr(a.batch.err, kErrBadIndex);
    return;
  }
  unsigned char* sQ = smem + C::kOffQ;
  unsigned char* sK = smem + C::kOffK;
  unsigned char* sV = smem + C::kOffV;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::kOffBar);
  uint64_t* q_full = bars;
  uint64_t* q_empty = q_full + 1;
  uint64_t* k_full = q_empty + 1;
  uint64_t* k_empty = k_full + C::KST;
  uint64_t* v_full = k_empty + C::KST;
  uint64_t* v_empty = v_full + C::VST;
  uint64_t* s_full = v_empty + C::VST;
  uint64_t* p_full = s_full + 2;
  uint64_t* pv_done = p_full + 2;
  uint64_t* o_free = pv_done + 2;
  uint64_t* uq_full = o_free + 1;
  uint64_t* uq_empty = uq_full + UnitQueue::kDepth;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + C::kNumBars);
  // units come from a global counter through this queue (the V loader, the
  // MMA thread and the four softmax warps consume)
  const UnitQueue uq{reinterpret_cast<int32_t*>(tmem_slot + 4), uq_full, uq_empty, 6};

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = a.g;
  int32_t* err = a.batch.err;

  if (threadIdx.x == 0) {
    ptx::mbar_init(q_full, 1);
    ptx::mbar_init(q_empty, 1);
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
      ptx::mbar_init(&p_full[i], 4);
      ptx::mbar_init(&pv_done[i], 1);
    }
    ptx::mbar_init(o_free, 4);
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
    // Lane 0 takes units from the global counter and loads Q and the K
    // tiles; lane 1 follows the same units through the queue and loads the
    // V tiles. The two streams run on independent rings, so a K load is
    // never held back behind a V stage that the P.V of an earlier tile still
    // occupies.
    if (lane < 2) {
      const bool is_k = lane == 0;
      const int B = a.cache.block_size;
      const int BR = B < 64 ? B : 64;
      const int Hkv = a.cache.n_kv_heads;
      const int kv = is_k ? 0 : 1;
      const int NST = is_k ? C::KST : C::VST;
      uint64_t* full = is_k ? k_full : v_full;
      uint64_t* empty = is_k ? k_empty : v_empty;
      unsigned char* ring = is_k ? sK : sV;
      int gt = 0, un = 0;
      for (;; ++un) {
        int u = -1;
        const bool got = is_k ? uq.push_next(un, a.counter, a.n_items, kWaitLimit, &u)
                              : uq.pop(un, false, kWaitLimit, &u);
        if (!got) {
          atomicOr(err, kErrTimeout);
          ok = false;
        }
        if (u < 0 || !ok) break;
        const Unit x = load_unit(a, u, C::BN);
        if (is_k) {
          if (un >= 1 && !wait_or_flag(q_empty, (un - 1) & 1, err, ok)) break;
          ptx::mbar_arrive_expect_tx(q_full, C::kQBytes);
#pragma unroll
          for (int dh = 0; dh < C::DH; ++dh)
            ptx::tma_load_3d(sQ + dh * C::BM * 128, &tm_q, dh * 64, x.h * g, x.row0, q_full);
        }
        const int32_t* bt = a.batch.bt + a.batch.bt_off[x.s];
        const int nb = a.batch.bt_off[x.s + 1] - a.batch.bt_off[x.s];
        for (int i = 0; i < x.n_tiles && ok; ++i, ++gt) {
          const int k0 = x.k00 + i * C::BN;
          uint32_t bytes = 0;
          for (int pos = k0; pos < k0 + C::BN; pos += BR) {
            const int lb = pos / B;
            if (lb < nb && bt[lb] >= 0 && bt[lb] < a.cache.n_blocks) bytes += BR * 128 * C::DH;
          }
          const int st = gt % NST;
          if (gt >= NST && !wait_or_flag(&empty[st], ((gt / NST) - 1) & 1, err, ok)) break;
          ptx::mbar_arrive_expect_tx(&full[st], bytes);
          for (int pos = k0; pos < k0 + C::BN; pos += BR) {
            const int lb = pos / B;
            if (lb >= nb) continue;
            const int32_t blk = bt[lb];
            if (blk < 0 || blk >= a.cache.n_blocks) {
              if (is_k) atomicOr(err, kErrBadBlock);
              continue;
            }
            const int row = (int)((((int64_t)blk * 2 + kv) * Hkv + x.h) * B + (pos - lb * B));
#pragma unroll
            for (int dh = 0; dh < C::DH; ++dh)
              ptx::tma_load_2d(ring + st * C::kKVBytes + dh * C::BN * 128 + (pos - k0) * 128, &tm_kv, dh * 64,
                               row, &full[st]);
          }
        }
      }
      // every unit is claimed: a grid launched behind this one (the decode
      // kernel) may take SMs as this kernel's CTAs leave
      if (is_k) ptx::allow_dependent_launch();
      // let in-flight loads land before the CTA can exit
      for (int t = max(0, gt - NST); t < gt && ok; ++t) wait_or_flag(&full[t % NST], (t / NST) & 1, err, ok);
      if (is_k && un >= 1) wait_or_flag(q_full, (un - 1) & 1, err, ok);
    }
  } else if (warp == 5) {
    // ---------------------------------------------------------------- MMA
    if (lane == 0) {
      constexpr uint32_t idesc_qk = ptx::idesc_bf16_f32(C::BM, C::BN, 0, 0);
      constexpr uint32_t idesc_pv = ptx::idesc_bf16_f32(C::BM, D, 0, 1);
      const uint32_t q_addr = ptx::smem_u32(sQ), k_addr = ptx::smem_u32(sK);
      const uint32_t v_addr = ptx::smem_u32(sV);
      int gt = 0, un = 0;
      // O += P V for global tile t, P in the TMEM S buffer t&1 (bf16 packed,
      // 16 keys = 8 columns per MMA step); `first` starts a unit's
      // accumulation and must wait until the previous unit's epilogue has
      // read O.
      auto issue_pv = [&](int t, bool first) {
        const int vs = t % C::VST, pb = t & 1;
        if (!wait_or_flag(&v_full[vs], (t / C::VST) & 1, err, ok)) return;
        if (!wait_or_flag(&p_full[pb], (t >> 1) & 1, err, ok)) return;
        if (first && un >= 1 && !wait_or_flag(o_free, (un - 1) & 1, err, ok)) return;
        ptx::tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < C::BN / 16; ++kk) {
          const uint64_t bd = ptx::smem_desc_sw128(v_addr + vs * C::kKVBytes + kk * 16 * 128, C::BN * 128, 1024);
          mma_bf16_ts(tmem + C::kColO, tmem + C::kColS + pb * C::BN + kk * 8, bd, idesc_pv,
                      (!first || kk > 0) ? 1u : 0u);
        }
        ptx::mma_commit(&pv_done[pb]);
        ptx::mma_commit(&v_empty[vs]);
      };
      for (;; ++un) {
        int u = -1;
        if (!uq.pop(un, false, kWaitLimit, &u)) {
          atomicOr(err, kErrTimeout);
          ok = false;
        }
        if (u < 0 || !ok) break;
        const Unit x = load_unit(a, u, C::BN);
        if (!wait_or_flag(q_full, un & 1, err, ok)) break;
        const int gt0 = gt;
        for (int i = 0; i < x.n_tiles && ok; ++i, ++gt) {
          const int ks = gt % C::KST, sb = gt & 1;
          if (!wait_or_flag(&k_full[ks], (gt / C::KST) & 1, err, ok)) break;
          // S buffer sb holds P of tile gt-2, which the P.V product issued
          // just before this one reads: tcgen05.mma operations issued by one
          // thread execute in issue order, so this S product is queued
          // behind that P.V instead of waiting for its completion here
          ptx::tc_fence_after();
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const uint32_t off = (kk >> 2) * C::BM * 128 + (kk & 3) * 32;
            const uint64_t ad = ptx::smem_desc_sw128(q_addr + off, 16, 1024);
            const uint64_t bd = ptx::smem_desc_sw128(
                k_addr + ks * C::kKVBytes + (kk >> 2) * C::BN * 128 + (kk & 3) * 32, 16, 1024);
            ptx::mma_bf16(tmem + C::kColS + sb * C::BN, ad, bd, idesc_qk, kk > 0 ? 1u : 0u);
          }
          ptx::mma_commit(&s_full[sb]);
          ptx::mma_commit(&k_empty[ks]);
          if (i == x.n_tiles - 1) ptx::mma_commit(q_empty);
          if (i >= 1) issue_pv(gt - 1, i == 1);
        }
        if (ok) issue_pv(gt - 1, gt - 1 == gt0);
      }
    }
  } else {
    // ---------------------------------------------------- softmax / epilogue
    const int r = threadIdx.x;  // query row == TMEM lane
    const uint32_t lane_base = (uint32_t)(warp * 32) << 16;
    int gt = 0, un = 0;
    for (;; ++un) {
      int u = -1;
      if (!uq.pop(un, true, kWaitLimit, &u)) {
        if (lane == 0) atomicOr(err, kErrTimeout);
        ok = false;
      }
      if (u < 0 || !ok) break;
      const Unit x = load_unit(a, u, C::BN);
      const bool row_ok = r < x.R;
      const int p_r = x.ctx + x.tok_begin + r / g;
      int lower = 0, upper = 0;
      if (row_ok) {
        lower = max(x.kb, a.window > 0 ? p_r - a.window + 1 : 0);
        upper = min(x.ke, p_r + 1);
      }
      const bool warp_live = (warp * 32) < x.R;
      float m_used = -INFINITY, l = 0.f;
      for (int i = 0; i < x.n_tiles && ok; ++i, ++gt) {
        const int sb = gt & 1;
        const int k0 = x.k00 + i * C::BN;
        if (!wait_or_flag(&s_full[sb], (gt >> 1) & 1, err, ok)) break;
        if (warp_live) {
          ptx::tc_fence_after();
          uint32_t raw[C::BN];
#pragma unroll
          for (int c = 0; c < C::BN / 32; ++c)
            ptx::tmem_ld32(tmem + lane_base + C::kColS + sb * C::BN + c * 32,
                           *reinterpret_cast<uint32_t(*)[32]>(&raw[c * 32]));
          ptx::tmem_ld_wait();
          float sv[C::BN];
          // mask, then the tile max as a tree of 3-input maxima (8 independent
          // chains, so the reduction is not one 64-long dependency chain)
          const int c_lo = lower - k0, c_hi = upper - k0;
#pragma unroll
          for (int c = 0; c < C::BN; ++c) sv[c] = __uint_as_float(raw[c]);
          // most tiles need no mask; the test is a warp vote, so the selects
          // below run (for the whole warp) only on tiles that need them
          if (__any_sync(0xffffffffu, c_lo > 0 || c_hi < C::BN)) {
#pragma unroll
            for (int c = 0; c < C::BN; ++c)
              if (c < c_lo || c >= c_hi) sv[c] = -INFINITY;
          }
          float mx[8];
#pragma unroll
          for (int j = 0; j < 8; ++j) mx[j] = fmaxf(sv[j], sv[8 + j]);
#pragma unroll
          for (int c = 16; c < C::BN; c += 16)
#pragma unroll
            for (int j = 0; j < 8; ++j) mx[j] = max3(mx[j], sv[c + j], sv[c + 8 + j]);
          const float mt = max3(max3(mx[0], mx[1], mx[2]), max3(mx[3], mx[4], mx[5]), fmaxf(mx[6], mx[7]));
          const float mts = mt == -INFINITY ? -INFINITY : mt * a.scale_log2;
          float alpha = 1.f;
          if (mts > m_used + 8.f) {  // also true the first time a row sees a key
            alpha = m_used == -INFINITY ? 0.f : ex2(m_used - mts);
            m_used = mts;
            l *= alpha;
          }
          // O may be rescaled only once the P.V of the previous tile is done
          if (i >= 1 && __any_sync(0xffffffffu, alpha != 1.f)) {
            if (!wait_or_flag(&pv_done[(gt - 1) & 1], ((gt - 1) >> 1) & 1, err, ok)) break;
            ptx::tc_fence_after();
#pragma unroll
            for (int c = 0; c < D / 32; ++c) {
              uint32_t o[32];
              const uint32_t ta = tmem + lane_base + C::kColO + c * 32;
              ptx::tmem_ld32(ta, o);
              ptx::tmem_ld_wait();
              const float2 al2 = make_float2(alpha, alpha);
#pragma unroll
              for (int e = 0; e < 32; e += 2) {
                const float2 r = __fmul2_rn(make_float2(__uint_as_float(o[e]), __uint_as_float(o[e + 1])), al2);
                o[e] = __float_as_uint(r.x);
                o[e + 1] = __float_as_uint(r.y);
              }
              ptx::tmem_st32(ta, o);
            }
            ptx::tmem_st_wait();
          }
          // P = 2^(s*scale - m_used), packed two bf16 per 32-bit word, written
          // over the first BN/2 columns of this S buffer (lane r = row r).
          // Masked keys are -inf and give 0; a row with no key yet has
          // m_used = -inf, all its scores -inf, and neg_m = 0 keeps them 0.
          // the scale-and-shift and the running sums use the packed f32x2
          // FMA/add, two keys per instruction
          float2 ls[4] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f),
                          make_float2(0.f, 0.f)};
          const float neg_m = m_used == -INFINITY ? 0.f : -m_used;
          const float2 sc2 = make_float2(a.scale_log2, a.scale_log2), nm2 = make_float2(neg_m, neg_m);
          uint32_t pw[C::BN / 2];
#pragma unroll
          for (int c = 0; c < C::BN / 2; ++c) {
            const float2 x = __ffma2_rn(make_float2(sv[2 * c], sv[2 * c + 1]), sc2, nm2);
            const float2 pp = make_float2(ex2(x.x), ex2(x.y));
            ls[c & 3] = __fadd2_rn(ls[c & 3], pp);
            __nv_bfloat162 pr = __floats2bfloat162_rn(pp.x, pp.y);
            pw[c] = *reinterpret_cast<uint32_t*>(&pr);
          }
          ptx::tmem_st32(tmem + lane_base + C::kColS + sb * C::BN, pw);
          const float2 l01 = __fadd2_rn(ls[0], ls[1]), l23 = __fadd2_rn(ls[2], ls[3]);
          l += (l01.x + l01.y) + (l23.x + l23.y);
          // keys at or past the sequence end may hold anything (unwritten
          // slots, stale stage data): zero those V rows so 0 * garbage cannot
          // reach O
          if (k0 + C::BN > x.L) {
            const int vs = gt % C::VST;
            if (!wait_or_flag(&v_full[vs], (gt / C::VST) & 1, err, ok)) break;
            const int z0 = max(0, x.L - k0);
            const int per_dh = (C::BN - z0) * 8;  // 16-byte chunks per 64-dim half
            const int nz = per_dh * C::DH;
            const int n_live = min(C::BM, (x.R + 31) & ~31);  // threads of the live warps
            for (int z = threadIdx.x; z < nz; z += n_live) {
              const int dh = z / per_dh, rem = z - dh * per_dh;
              const int row = z0 + rem / 8, chn = rem % 8;
              *reinterpret_cast<uint4*>(sV + vs * C::kKVBytes + dh * C::BN * 128 + row * 128 + chn * 16) =
                  make_uint4(0, 0, 0, 0);
            }
            ptx::fence_proxy_async_smem();
          }
          ptx::tmem_st_wait();
        }
        // padding warps write no P: arriving right after their s_full wait
        // is safe, because tile gt + 2 cannot start before this phase ends
        ptx::tc_fence_before();
        __syncwarp();
        if (lane == 0) ptx::mbar_arrive(&p_full[sb]);
      }
      if (!ok) break;
      // epilogue: wait for the unit's last PV, normalise, store, free O
      const int last = gt - 1;
      if (!wait_or_flag(&pv_done[last & 1], (last >> 1) & 1, err, ok)) break;
      ptx::tc_fence_after();
      if (warp_live) {
        const int row = x.row0 + r / g;
        const int qh = x.h * g + (r % g);
        const float inv = l > 0.f ? 1.f / l : 0.f;
#pragma unroll
        for (int c = 0; c < D / 32; ++c) {
          uint32_t o[32];
          ptx::tmem_ld32(tmem + lane_base + C::kColO + c * 32, o);
          ptx::tmem_ld_wait();
          if (!row_ok) continue;
          if (x.part < 0) {
            uint4* dst = reinterpret_cast<uint4*>(a.out + ((int64_t)row * a.Hq + qh) * D + c * 32);
#pragma unroll
            for (int q4 = 0; q4 < 4; ++q4) {
              uint32_t w[4];
#pragma unroll
              for (int e = 0; e < 4; ++e) {
                __nv_bfloat162 pr = __floats2bfloat162_rn(__uint_as_float(o[q4 * 8 + 2 * e]) * inv,
                                                          __uint_as_float(o[q4 * 8 + 2 * e + 1]) * inv);
                w[e] = *reinterpret_cast<uint32_t*>(&pr);
              }
              dst[q4] = make_uint4(w[0], w[1], w[2], w[3]);
            }
          } else {
            float4* dst = reinterpret_cast<float4*>(a.part_o + (int64_t)(x.part + r) * D + c * 32);
#pragma unroll
            for (int q4 = 0; q4 < 8; ++q4)
              dst[q4] = make_float4(__uint_as_float(o[4 * q4]), __uint_as_float(o[4 * q4 + 1]),
                                    __uint_as_float(o[4 * q4 + 2]), __uint_as_float(o[4 * q4 + 3]));
          }
        }
        if (row_ok && x.part >= 0) {
          a.part_ml[(int64_t)(x.part + r) * 2] = m_used;
          a.part_ml[(int64_t)(x.part + r) * 2 + 1] = l;
        }
      }
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
}

template <int D>
cudaError_t launch_tc_d(const CUtensorMap& tm_q, const CUtensorMap& tm_kv, const TcArgs& args, int grid,
                        cudaStream_t stream) {
  using C = TcCfg<D>;
  static bool configured = false;
  if (!configured) {
    cudaError_t e =
        cudaFuncSetAttribute(attn_tc_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmem);
    if (e != cudaSuccess) return e;
    // the largest shared-memory carveout: two CTAs per SM, and a decode CTA
    // beside one when the kernels share the GPU
    e = cudaFuncSetAttribute(attn_tc_kernel<D>, cudaFuncAttributePreferredSharedMemoryCarveout,
                             cudaSharedmemCarveoutMaxShared);
    if (e != cudaSuccess) return e;
    configured = true;
  }
  attn_tc_kernel<D><<<grid, C::kThreads, C::kSmem, stream>>>(tm_q, tm_kv, args);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_attention_tc(const void* tm_q, const void* tm_kv, const CacheView& cache,
                                const BatchView& batch, const WorkItem* items, int n_items,
                                __nv_bfloat16* out, float* part_o, float* part_ml, int n_q_heads,
                                int g, float scale_log2, int window, int grid, int sm_end,
                                int* counter, cudaStream_t stream) {
  if (n_items == 0) return cudaSuccess;
  TcArgs args{cache, batch, items, out, part_o, part_ml, n_q_heads, g, scale_log2, window, n_items,
              counter, sm_end};
  grid = grid < 1 ? 1 : (grid > n_items ? n_items : grid);
  const CUtensorMap& q = *static_cast<const CUtensorMap*>(tm_q);
  const CUtensorMap& kv = *static_cast<const CUtensorMap*>(tm_kv);
  if (cache.head_dim == 128) return launch_tc_d<128>(q, kv, args, grid, stream);
  return launch_tc_d<64>(q, kv, args, grid, stream);
}

}  // namespace fg
