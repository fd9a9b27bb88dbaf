// Ragged paged attention on the 5th-generation tensor cores (tcgen05).
//
// A work unit is up to two 128-row query tiles (0 and 1) of one sequence and
// kv head that share every K/V tile: the rows are (token, q head of the
// group) pairs, up to 256/g consecutive new tokens times the g q heads that
// share the kv head, rows 0-127 in tile 0 and 128-255 in tile 1. Each K/V
// tile is loaded once per unit and serves both query tiles and all g heads.
// The kernel is persistent, one CTA per SM: the K loader takes units one by
// one from a global counter over a longest-first list and hands them to the
// other roles, and every role counts tiles globally, so the rings and barrier
// phases run on across units. A unit walks the key range of its last row in
// 64-key tiles:
//
//   warp 8, lane 0    Q of both query tiles once per unit (3-D boxes: 64
//                     dims x g heads x 128/g tokens), then K tiles through the
//                     block table into a 5-stage ring;
//   warp 11, lane 0   V tiles, the same way, into a 4-stage ring (separate
//                     streams, so a K load never waits behind a V stage that
//                     an earlier P.V still occupies, and separate warps, so
//                     neither loader's loop is serialised behind the other's);
//   warps 9, 10 (MMA) one thread per query tile issues S_t = Q_t K^T into
//                     double-buffered TMEM S tiles and O_t += P_t V into its
//                     TMEM O tile, with P read from tensor memory; the two
//                     tiles' pipelines only meet at the shared K/V rings;
//   warps 0-3 / 4-7   softmax of query tile 0 / 1: thread r of a warpgroup
//                     owns row r of its tile (TMEM lane r): reads its S row
//                     with tcgen05.ld, masks (causal, window, unit range),
//                     keeps an online softmax (a running max that is only
//                     moved - with a rescale of its O row in TMEM - when a
//                     tile raises it by more than 2^8), writes P as packed
//                     bf16 back over the S tile it came from, and at the end
//                     normalises O and stores it.
//
// Sharing K/V between two query tiles halves the K/V traffic from L2 per
// flop and leaves shared memory for deep rings; the two softmax warpgroups
// keep the tensor core fed while each works through its exponentials.
// Keeping P in tensor memory makes it double-buffered with S for free: the
// softmax of tile i+1 never waits for the P.V product of tile i, and the S
// product of tile i+2, which overwrites that buffer, is issued right behind
// that P.V (the tensor core runs one thread's MMAs in issue order).
// Every wait is bounded; a wait that gives up sets kErrTimeout and the CTA
// drains and returns.
#include <cuda.h>

#include <cfloat>

#include "fg_internal.h"
#include "rope_exact.cuh"
#include "sm100_ptx.cuh"

namespace fg {
namespace {

constexpr long long kWaitLimit = 1LL << 31;

// Cycle accounting of the kernel's roles, compiled in only with
// -DFG_PHASE_TRACE (the separate trace build, libfg_trace.so). Each role keeps
// one clock64 stamp and, at every mark, adds the cycles since the previous
// mark to one of its slots; one recording thread per role adds its slots to
// g_phase at exit, which fg_phase_trace_read returns. Slot layout: softmax
// of query tile t at 12 t (wait S, load S, max, rescale O, exponentials and
// P store, V zeroing, store wait and P arrive, epilogue wait, epilogue
// stores, unit pop, 64-key steps, wait for the exponential turn), MMA thread t at 24 + 8 t (unit
// pop, wait K, issue S, wait V, wait P, wait O free, issue P.V, steps), the
// K and V loaders at 40 and 48 (unit pop, wait Q free, wait stage free,
// issue, tiles), CTA cycles and CTAs at 56 and 57; %globaltimer (ns) of the
// first CTA start, the last CTA start and the last CTA end at 58, 59, 60
// (minimum / maximum over the launches since the last read).
#ifdef FG_PHASE_TRACE
constexpr int kPhaseSlots = 64;
__device__ unsigned long long g_phase[kPhaseSlots];
#define PH_DECL        \
  uint32_t ph_[12] = {}; \
  uint32_t ph_t_ = (uint32_t)clock()
#define PH_MARK(i)                          \
  do {                                      \
    const uint32_t t_ = (uint32_t)clock();  \
    ph_[i] += t_ - ph_t_;                   \
    ph_t_ = t_;                             \
  } while (0)
#define PH_COUNT(i, n) (ph_[i] += (n))
#define PH_FLUSH(rec, base, n)                                                     \
  do {                                                                             \
    if (rec)                                                                       \
      for (int i_ = 0; i_ < (n); ++i_) atomicAdd(&g_phase[(base) + i_], (unsigned long long)ph_[i_]); \
  } while (0)
#else
#define PH_DECL
#define PH_MARK(i) \
  do {             \
  } while (0)
#define PH_COUNT(i, n) \
  do {                 \
  } while (0)
#define PH_FLUSH(rec, base, n) \
  do {                         \
  } while (0)
#endif

template <int D>
struct TcCfg {
  static constexpr int BM = 128;  // query rows per tile
  static constexpr int NQ = 2;    // query tiles per unit
  static constexpr int BN = 64;   // keys per K/V tile
  static constexpr int KST = 5, VST = 4;
  static constexpr int DH = D / 64;  // 64-dim (128-byte) boxes per row
  static constexpr int kQBytes = BM * D * 2;
  static constexpr int kKVBytes = BN * D * 2;
  static constexpr int kOffQ = 0;
  static constexpr int kOffK = kOffQ + NQ * kQBytes;
  static constexpr int kOffV = kOffK + KST * kKVBytes;
  static constexpr int kOffBar = kOffV + VST * kKVBytes;
  // q_full, q_empty, k_full[KST], k_empty[KST], v_full[VST], v_empty[VST],
  // then per query tile: s_full[2], p_full[2], pv_done[2], o_free; the
  // exponential turns of the 4 softmax warp pairs (turn[2 r + t]); unit
  // queue; q_ready (Q rotated in place, the rotary-at-load form)
  static constexpr int kNumBars = 2 + 2 * KST + 2 * VST + NQ * 7 + 8 + 2 * UnitQueue::kDepth + 1;
  static constexpr int kSmem = kOffBar + kNumBars * 8 + 16 + UnitQueue::kDepth * 4;
  static constexpr int kThreads = 384;  // 8 softmax warps, the K loader, two MMA warps, the V loader
  static constexpr uint32_t kTmemCols = 512;
  // query tile t: S (then P) buffers at kColS0 + 2 t BN and + BN, O at kColO0 + t D
  static constexpr uint32_t kColS0 = 0;
  static constexpr uint32_t kColO0 = NQ * 2 * BN;
  static_assert(kColO0 + NQ * D <= kTmemCols, "TMEM budget");
  static_assert(kSmem + 1024 <= 228 * 1024, "shared memory budget");
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
  // the rotary-at-load form (ROPE = true): Q is read unrotated and rotated
  // in shared memory with this table ([position][d/2] (cos, sin) times
  // 2^896, pair 8 j + e at entry e * d/16 + j)
  const double2* rope;
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
// 2^x for a pair of floats on the FMA pipe, without the special-function
// unit: Cody-Waite range reduction x = j + f, j = rint(x), |f| <= 1/2, and
// 2^x = 2^j p(f), p the degree-5 polynomial of least maximum relative error
// to 2^f on [-1/2, 1/2] (float32 coefficients from exp2_poly_fit.py; relative
// error 2^-22.6 before the float32 evaluation). rint(x) is an add of
// 1.5 * 2^23, after which the low mantissa bits of the sum hold j; 2^j is
// placed by adding (sum bits) << 23 to p's bits (the constant's own low bits
// are zero, so only j << 23 remains). x is clamped at -127, so j >= -127
// with f >= 0 there and the result stays a non-negative float (a subnormal
// at the bottom); -inf, the masked keys, gives a value below 2^-148 that
// rounds to bf16 zero.
constexpr float kExp2C0 = 0x1.000002p+0f, kExp2C1 = 0x1.62e428p-1f, kExp2C2 = 0x1.ebf918p-3f,
                kExp2C3 = 0x1.c6b6e4p-5f, kExp2C4 = 0x1.3d0c52p-7f, kExp2C5 = 0x1.5c08e6p-10f;
__device__ __forceinline__ float2 ex2_fma2(float2 x) {
  x.x = fmaxf(x.x, -127.f);
  x.y = fmaxf(x.y, -127.f);
  const float2 t = __fadd2_rn(x, make_float2(12582912.f, 12582912.f));
  const float2 j = __fadd2_rn(t, make_float2(-12582912.f, -12582912.f));
  const float2 f = __ffma2_rn(j, make_float2(-1.f, -1.f), x);
  float2 p = __ffma2_rn(make_float2(kExp2C5, kExp2C5), f, make_float2(kExp2C4, kExp2C4));
  p = __ffma2_rn(p, f, make_float2(kExp2C3, kExp2C3));
  p = __ffma2_rn(p, f, make_float2(kExp2C2, kExp2C2));
  p = __ffma2_rn(p, f, make_float2(kExp2C1, kExp2C1));
  p = __ffma2_rn(p, f, make_float2(kExp2C0, kExp2C0));
  return make_float2(__int_as_float(__float_as_int(p.x) + (__float_as_int(t.x) << 23)),
                     __int_as_float(__float_as_int(p.y) + (__float_as_int(t.y) << 23)));
}
// Every kExp2FmaEvery-th pair of a row's exponentials goes to ex2_fma2, the
// rest to ex2 (0: none, the default). Measured on B200 on the long-prompt
// batch, taking a quarter or half of the exponentials off the
// special-function unit this way made the kernel slower (the softmax's
// instruction count, not the special-function unit, set its pace), so it is
// off; the path stays compiled in with -DFG_EXP2_FMA_EVERY=n.
#ifndef FG_EXP2_FMA_EVERY
#define FG_EXP2_FMA_EVERY 0
#endif
constexpr int kExp2FmaEvery = FG_EXP2_FMA_EVERY;

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

template <int D, bool ROPE>
__global__ void __launch_bounds__(384, 1) attn_tc_kernel(const __grid_constant__ CUtensorMap tm_q,
                                                        const __grid_constant__ CUtensorMap tm_kv,
                                                        TcArgs a) {
  using C = TcCfg<D>;
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  unsigned char* smem = smem_raw;
  // SMs outside the kernel's share are left to the decode kernel
  if (ptx::sm_id() >= a.sm_end) return;
#ifdef FG_PHASE_TRACE
  const long long cta_t0 = clock64();
  if (threadIdx.x == 0) {
    const unsigned long long g0 = ptx::global_timer_ns();
    atomicMin(&g_phase[58], g0);
    atomicMax(&g_phase[59], g0);
  }
#endif
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
  uint64_t* tb = v_empty + C::VST;  // query tile t: 7 barriers from tb + 7 t
  auto s_full = [tb](int t, int b) { return tb + 7 * t + b; };
  auto p_full = [tb](int t, int b) { return tb + 7 * t + 2 + b; };
  auto pv_done = [tb](int t, int b) { return tb + 7 * t + 4 + b; };
  auto o_free = [tb](int t) { return tb + 7 * t + 6; };
  // warp r of query tile 0 and warp r of tile 1 (warps r and r + 4) share an
  // SM sub-partition and its special-function unit: they take turns with
  // their exponentials, tile 0 first in each K/V tile; turn[2 r + t] is
  // completed when it is tile t's turn
  uint64_t* turn = tb + 7 * C::NQ;
  uint64_t* uq_full = turn + 8;
  uint64_t* uq_empty = uq_full + UnitQueue::kDepth;
  uint64_t* q_ready = uq_empty + UnitQueue::kDepth;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + C::kNumBars);
  // units come from a global counter through this queue (the V loader, the
  // two MMA threads and the eight softmax warps consume)
  const UnitQueue uq{reinterpret_cast<int32_t*>(tmem_slot + 4), uq_full, uq_empty, 11};

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = a.g;
  int32_t* err = a.batch.err;

  if (threadIdx.x == 0) {
    ptx::mbar_init(q_full, 1);
    // Q and every K/V stage are released by both MMA threads
    ptx::mbar_init(q_empty, C::NQ);
    for (int i = 0; i < C::KST; ++i) {
      ptx::mbar_init(&k_full[i], 1);
      ptx::mbar_init(&k_empty[i], C::NQ);
    }
    for (int i = 0; i < C::VST; ++i) {
      ptx::mbar_init(&v_full[i], 1);
      ptx::mbar_init(&v_empty[i], C::NQ);
    }
    for (int t = 0; t < C::NQ; ++t) {
      for (int i = 0; i < 2; ++i) {
        ptx::mbar_init(s_full(t, i), 1);
        ptx::mbar_init(p_full(t, i), 4);
        ptx::mbar_init(pv_done(t, i), 1);
      }
      ptx::mbar_init(o_free(t), 4);
    }
    for (int i = 0; i < 8; ++i) ptx::mbar_init(&turn[i], 1);
    ptx::mbar_init(q_ready, 8);
    uq.init();
    ptx::fence_mbar_init();
  }
  if (warp == 9) {
    ptx::tmem_alloc(tmem_slot, C::kTmemCols);
    ptx::tmem_relinquish();
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  bool ok = true;

  if (warp == 8 || warp == 11) {
    // ---------------------------------------------------------------- loads
    if (lane == 0) {
      const bool is_k = warp == 8;
      const int B = a.cache.block_size;
      const int BR = B < 64 ? B : 64;
      const int Hkv = a.cache.n_kv_heads;
      const int kv = is_k ? 0 : 1;
      const int NST = is_k ? C::KST : C::VST;
      uint64_t* full = is_k ? k_full : v_full;
      uint64_t* empty = is_k ? k_empty : v_empty;
      unsigned char* ring = is_k ? sK : sV;
      int gt = 0, un = 0;
      PH_DECL;
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
        PH_MARK(0);
        if (is_k) {
          // both query tiles' boxes (tile 1's reaches past the unit's rows
          // when R <= 128; those rows are never used)
          if (un >= 1 && !wait_or_flag(q_empty, (un - 1) & 1, err, ok)) break;
          PH_MARK(1);
          ptx::mbar_arrive_expect_tx(q_full, C::NQ * C::kQBytes);
#pragma unroll
          for (int t = 0; t < C::NQ; ++t)
#pragma unroll
            for (int dh = 0; dh < C::DH; ++dh)
              ptx::tma_load_3d(sQ + t * C::kQBytes + dh * C::BM * 128, &tm_q, dh * 64, x.h * g,
                               x.row0 + t * (C::BM / g), q_full);
        }
        const int32_t* bt = a.batch.bt + a.batch.bt_off[x.s];
        const int nb = a.batch.bt_off[x.s + 1] - a.batch.bt_off[x.s];
        // block ids of a tile's 64 / BR boxes (-1: past the table, no load);
        // the next tile's are read before this tile waits for its stage, so
        // the dependent global read is off the issue path
        constexpr int kMaxBoxes = 4;  // 64-key tile over 16-slot blocks
        auto tile_blocks = [&](int i, int32_t (&ids)[kMaxBoxes]) {
#pragma unroll
          for (int j = 0; j < kMaxBoxes; ++j) {
            const int pos = x.k00 + i * C::BN + j * BR;
            const int lb = pos / B;
            ids[j] = (j * BR < C::BN && lb < nb) ? bt[lb] : -1;
          }
        };
        int32_t cur[kMaxBoxes], nxt[kMaxBoxes];
        if (x.n_tiles > 0) tile_blocks(0, cur);
        for (int i = 0; i < x.n_tiles && ok; ++i, ++gt) {
          if (i + 1 < x.n_tiles) tile_blocks(i + 1, nxt);
          const int k0 = x.k00 + i * C::BN;
          uint32_t bytes = 0;
#pragma unroll
          for (int j = 0; j < kMaxBoxes; ++j)
            if (cur[j] >= 0 && cur[j] < a.cache.n_blocks) bytes += BR * 128 * C::DH;
          const int st = gt % NST;
          if (gt >= NST && !wait_or_flag(&empty[st], ((gt / NST) - 1) & 1, err, ok)) break;
          PH_MARK(2);
          PH_COUNT(4, 1);
          ptx::mbar_arrive_expect_tx(&full[st], bytes);
#pragma unroll
          for (int j = 0; j < kMaxBoxes; ++j) {
            const int pos = k0 + j * BR;
            const int32_t blk = cur[j];
            if (j * BR >= C::BN || (blk == -1 && pos / B >= nb)) continue;
            if (blk < 0 || blk >= a.cache.n_blocks) {
              if (is_k) atomicOr(err, kErrBadBlock);
              continue;
            }
            const int row = (int)((((int64_t)blk * 2 + kv) * Hkv + x.h) * B + (pos - (pos / B) * B));
#pragma unroll
            // the unit order puts CTAs that read the same kv head's keys side
            // by side, so these lines are read again soon: keep them in L2
            // ahead of the lines streamed once (Q, the decode kernel's K/V)
            for (int dh = 0; dh < C::DH; ++dh)
              ptx::tma_load_2d_hint(ring + st * C::kKVBytes + dh * C::BN * 128 + (pos - k0) * 128, &tm_kv,
                                    dh * 64, row, &full[st], ptx::l2_evict_last_policy());
          }
#pragma unroll
          for (int j = 0; j < kMaxBoxes; ++j) cur[j] = nxt[j];
          PH_MARK(3);
        }
      }
      PH_FLUSH(true, is_k ? 40 : 48, 5);
      // every unit is claimed: a grid launched behind this one (the decode
      // kernel) may take SMs as this kernel's CTAs leave
      if (is_k) ptx::allow_dependent_launch();
      // let in-flight loads land before the CTA can exit
      for (int t = max(0, gt - NST); t < gt && ok; ++t) wait_or_flag(&full[t % NST], (t / NST) & 1, err, ok);
      if (is_k && un >= 1) wait_or_flag(q_full, (un - 1) & 1, err, ok);
    }
  } else if (warp == 9 || warp == 10) {
    // ---------------------------------------------------------------- MMA
    // One thread per query tile, so the two tiles' pipelines only meet at
    // the shared K/V rings: each thread walks every unit and K/V tile,
    // issues its tile's S and P.V products, and releases Q and each K/V
    // stage once (with a plain arrival when its tile has no rows).
    if (lane == 0) {
      const int t = warp - 9;
      constexpr uint32_t idesc_qk = ptx::idesc_bf16_f32(C::BM, C::BN, 0, 0);
      constexpr uint32_t idesc_pv = ptx::idesc_bf16_f32(C::BM, D, 0, 1);
      const uint32_t q_addr = ptx::smem_u32(sQ) + t * C::kQBytes, k_addr = ptx::smem_u32(sK);
      const uint32_t v_addr = ptx::smem_u32(sV);
      const uint32_t col_s = C::kColS0 + t * 2 * C::BN, col_o = C::kColO0 + t * D;
      int gt = 0, un = 0, ns = 0, np = 0, nu = 0;
      PH_DECL;
      // O_t += P_t V for the tile's next P (TMEM S buffer np & 1, bf16
      // packed, 16 keys = 8 columns per MMA step); `first` starts a unit's
      // accumulation and must wait until this tile's previous epilogue has
      // read O_t.
      auto issue_pv = [&](int vs, bool first) {
        const int l = np++, pb = l & 1;
        PH_MARK(3);
        if (!wait_or_flag(p_full(t, pb), (l >> 1) & 1, err, ok)) return;
        PH_MARK(4);
        if (first && nu >= 2 && !wait_or_flag(o_free(t), (nu - 2) & 1, err, ok)) return;
        PH_MARK(5);
        ptx::tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < C::BN / 16; ++kk) {
          const uint64_t bd = ptx::smem_desc_sw128(v_addr + vs * C::kKVBytes + kk * 16 * 128, C::BN * 128, 1024);
          mma_bf16_ts(tmem + col_o, tmem + col_s + pb * C::BN + kk * 8, bd, idesc_pv, (!first || kk > 0) ? 1u : 0u);
        }
        ptx::mma_commit(pv_done(t, pb));
        PH_MARK(6);
      };
      for (;; ++un) {
        int u = -1;
        if (!uq.pop(un, false, kWaitLimit, &u)) {
          atomicOr(err, kErrTimeout);
          ok = false;
        }
        if (u < 0 || !ok) break;
        const Unit x = load_unit(a, u, C::BN);
        PH_MARK(0);
        const bool live = x.R > t * C::BM;
        if (!live) {
          // nothing to compute: release Q and the unit's K/V stages as they
          // fill (the loaders' phases must see this thread's arrivals)
          if (!wait_or_flag(q_full, un & 1, err, ok)) break;
          ptx::mbar_arrive(q_empty);
          for (int i = 0; i < x.n_tiles && ok; ++i, ++gt) {
            if (!wait_or_flag(&k_full[gt % C::KST], (gt / C::KST) & 1, err, ok)) break;
            ptx::mbar_arrive(&k_empty[gt % C::KST]);
            if (!wait_or_flag(&v_full[gt % C::VST], (gt / C::VST) & 1, err, ok)) break;
            ptx::mbar_arrive(&v_empty[gt % C::VST]);
          }
          continue;
        }
        ++nu;
        if (!wait_or_flag(ROPE ? q_ready : q_full, un & 1, err, ok)) break;
        for (int i = 0; i < x.n_tiles && ok; ++i, ++gt) {
          const int ks = gt % C::KST;
          if (!wait_or_flag(&k_full[ks], (gt / C::KST) & 1, err, ok)) break;
          PH_MARK(1);
          PH_COUNT(7, 1);
          ptx::tc_fence_after();
          // S buffer sb holds P of this tile's tile ns - 2, which the P.V
          // issued earlier reads: the tensor core runs this thread's MMAs in
          // issue order, so this S product queues behind it
          const int sb = ns++ & 1;
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const uint32_t off = (kk >> 2) * C::BM * 128 + (kk & 3) * 32;
            const uint64_t ad = ptx::smem_desc_sw128(q_addr + off, 16, 1024);
            const uint64_t bd = ptx::smem_desc_sw128(
                k_addr + ks * C::kKVBytes + (kk >> 2) * C::BN * 128 + (kk & 3) * 32, 16, 1024);
            ptx::mma_bf16(tmem + col_s + sb * C::BN, ad, bd, idesc_qk, kk > 0 ? 1u : 0u);
          }
          ptx::mma_commit(s_full(t, sb));
          ptx::mma_commit(&k_empty[ks]);
          if (i == x.n_tiles - 1) ptx::mma_commit(q_empty);
          PH_MARK(2);
          if (i >= 1) {
            const int vs = (gt - 1) % C::VST;
            if (!wait_or_flag(&v_full[vs], ((gt - 1) / C::VST) & 1, err, ok)) break;
            issue_pv(vs, i == 1);
            ptx::mma_commit(&v_empty[vs]);
          }
        }
        if (ok) {
          const int vs = (gt - 1) % C::VST;
          if (wait_or_flag(&v_full[vs], ((gt - 1) / C::VST) & 1, err, ok)) {
            issue_pv(vs, x.n_tiles == 1);
            ptx::mma_commit(&v_empty[vs]);
          }
        }
      }
      PH_FLUSH(true, 24 + 8 * t, 8);
    }
  } else {
    // ---------------------------------------------------- softmax / epilogue
    const int qt = warp >> 2;              // query tile of this warpgroup
    const int r = (warp & 3) * 32 + lane;  // row within the tile == TMEM lane
    const uint32_t lane_base = (uint32_t)((warp & 3) * 32) << 16;
    const uint32_t col_s = C::kColS0 + qt * 2 * C::BN, col_o = C::kColO0 + qt * D;
    int gt = 0, lt = 0, un = 0;  // global K/V tiles; tiles of this query tile; units
    int hs = 0;                  // K/V tiles in which this warp took its exponential turn
    PH_DECL;
    for (;; ++un) {
      int u = -1;
      if (!uq.pop(un, true, kWaitLimit, &u)) {
        if (lane == 0) atomicOr(err, kErrTimeout);
        ok = false;
      }
      if (u < 0 || !ok) break;
      const Unit x = load_unit(a, u, C::BN);
      if (ROPE) {
        // the rotary-at-load form: each thread rotates its own row of the
        // unit's Q tile in shared memory (pairs (i, i + d/2) share a row and
        // a swizzled 16-byte position: the two 64-dim halves at d = 128,
        // 16-byte chunks j and j + 4 at d = 64), with the same exact
        // arithmetic as the rotary kernel; every softmax warp arrives on
        // q_ready once it is done (rows past the unit are left alone)
        if (!wait_or_flag(q_full, un & 1, err, ok)) break;
        const int rq = qt * C::BM + r;
        if (rq < x.R) {
          constexpr int HALF = D / 2, GROUPS = HALF / 8, NCH = HALF / 8;
          const double2* rrow = a.rope + (int64_t)(x.ctx + x.tok_begin + rq / g) * HALF;
          unsigned char* qrow = sQ + qt * C::kQBytes + r * 128;
          const int sw = r & 7;
          // one 16-byte chunk pair at a time (a table prefetch one chunk
          // ahead measured slower: its registers push the kernel into spills)
#pragma unroll 1
          for (int j = 0; j < NCH; ++j) {
            uint4* pa = reinterpret_cast<uint4*>(qrow + ((j ^ sw) << 4));
            uint4* pb = D == 128 ? reinterpret_cast<uint4*>(qrow + C::BM * 128 + ((j ^ sw) << 4))
                                 : reinterpret_cast<uint4*>(qrow + (((j + 4) ^ sw) << 4));
            uint4 y1, y2;
            rope::rotate8(*pa, *pb, [&](int e) { return __ldg(rrow + e * GROUPS + j); }, y1, y2);
            *pa = y1;
            *pb = y2;
          }
        }
        ptx::fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) ptx::mbar_arrive(q_ready);
      }
      if (x.R <= qt * C::BM) {  // this query tile has no rows in the unit
        gt += x.n_tiles;
        continue;
      }
      const int rr = qt * C::BM + r;  // row within the unit
      const bool row_ok = rr < x.R;
      const int p_r = x.ctx + x.tok_begin + rr / g;
      int lower = 0, upper = 0;
      if (row_ok) {
        lower = max(x.kb, a.window > 0 ? p_r - a.window + 1 : 0);
        upper = min(x.ke, p_r + 1);
      }
      const bool warp_live = qt * C::BM + (warp & 3) * 32 < x.R;
      // this warp and its partner in the other query tile take turns when
      // both have rows in the unit (the tile-1 warp's rows are the later ones)
      const bool turns = C::BM + (warp & 3) * 32 < x.R;
      uint64_t* my_turn = &turn[2 * (warp & 3) + qt];
      uint64_t* their_turn = &turn[2 * (warp & 3) + (qt ^ 1)];
      float m_used = -INFINITY, l = 0.f;
      PH_MARK(9);
      for (int i = 0; i < x.n_tiles && ok; ++i, ++lt, ++gt) {
        const int sb = lt & 1;
        const int k0 = x.k00 + i * C::BN;
        if (!wait_or_flag(s_full(qt, sb), (lt >> 1) & 1, err, ok)) break;
        PH_MARK(0);
        PH_COUNT(10, 1);
        if (warp_live) {
          ptx::tc_fence_after();
          uint32_t raw[C::BN];
#pragma unroll
          for (int c = 0; c < C::BN / 32; ++c)
            ptx::tmem_ld32(tmem + lane_base + col_s + sb * C::BN + c * 32,
                           *reinterpret_cast<uint32_t(*)[32]>(&raw[c * 32]));
          ptx::tmem_ld_wait();
          PH_MARK(1);
          float sv[C::BN];
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
          // the tile max as a tree of 3-input maxima (8 independent chains)
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
          PH_MARK(2);
          // O may be rescaled only once the P.V of the previous tile is done
          if (i >= 1 && __any_sync(0xffffffffu, alpha != 1.f)) {
            if (!wait_or_flag(pv_done(qt, (lt - 1) & 1), ((lt - 1) >> 1) & 1, err, ok)) break;
            ptx::tc_fence_after();
            const float2 al2 = make_float2(alpha, alpha);
#pragma unroll
            for (int c = 0; c < D / 32; ++c) {
              uint32_t o[32];
              const uint32_t ta = tmem + lane_base + col_o + c * 32;
              ptx::tmem_ld32(ta, o);
              ptx::tmem_ld_wait();
#pragma unroll
              for (int e = 0; e < 32; e += 2) {
                const float2 v2 = __fmul2_rn(make_float2(__uint_as_float(o[e]), __uint_as_float(o[e + 1])), al2);
                o[e] = __float_as_uint(v2.x);
                o[e + 1] = __float_as_uint(v2.y);
              }
              ptx::tmem_st32(ta, o);
            }
            ptx::tmem_st_wait();
          }
          PH_MARK(3);
          // P = 2^(s*scale - m_used), packed two bf16 per 32-bit word, written
          // over the first BN/2 columns of this S buffer (lane r = row r);
          // the scale-and-shift and the running sums use the packed f32x2
          // FMA/add. Masked keys are -inf and give 0; a row with no key yet
          // has m_used = -inf, all its scores -inf, and neg_m = 0 keeps them 0.
          float2 ls[4] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f),
                          make_float2(0.f, 0.f)};
          const float neg_m = m_used == -INFINITY ? 0.f : -m_used;
          const float2 sc2 = make_float2(a.scale_log2, a.scale_log2), nm2 = make_float2(neg_m, neg_m);
          // wait for this warp's turn: tile 0 after tile 1's previous K/V
          // tile, tile 1 after tile 0's current one
          PH_MARK(4);
          if (turns && (qt == 1 || hs >= 1) &&
              !wait_or_flag(my_turn, (qt == 1 ? hs : hs - 1) & 1, err, ok))
            break;
          PH_MARK(11);
          uint32_t pw[C::BN / 2];
#pragma unroll
          for (int c = 0; c < C::BN / 2; ++c) {
            const float2 xx = __ffma2_rn(make_float2(sv[2 * c], sv[2 * c + 1]), sc2, nm2);
            const float2 pp = (kExp2FmaEvery > 0 && c % (kExp2FmaEvery > 0 ? kExp2FmaEvery : 1) ==
                                                         kExp2FmaEvery - 1)
                                  ? ex2_fma2(xx)
                                  : make_float2(ex2(xx.x), ex2(xx.y));
            ls[c & 3] = __fadd2_rn(ls[c & 3], pp);
            __nv_bfloat162 pr = __floats2bfloat162_rn(pp.x, pp.y);
            pw[c] = *reinterpret_cast<uint32_t*>(&pr);
          }
          ptx::tmem_st32(tmem + lane_base + col_s + sb * C::BN, pw);
          if (turns) {
            __syncwarp();
            if (lane == 0) ptx::mbar_arrive(their_turn);
            ++hs;
          }
          const float2 l01 = __fadd2_rn(ls[0], ls[1]), l23 = __fadd2_rn(ls[2], ls[3]);
          l += (l01.x + l01.y) + (l23.x + l23.y);
          PH_MARK(4);
          // keys at or past the sequence end may hold anything (unwritten
          // slots, stale stage data): zero those V rows so 0 * garbage cannot
          // reach O. Both warpgroups may do it for a stage (the same zeros),
          // each before its own P.V can be issued.
          if (k0 + C::BN > x.L) {
            const int vs = gt % C::VST;
            if (!wait_or_flag(&v_full[vs], (gt / C::VST) & 1, err, ok)) break;
            const int z0 = max(0, x.L - k0);
            const int per_dh = (C::BN - z0) * 8;  // 16-byte chunks per 64-dim half
            const int nz = per_dh * C::DH;
            const int live_rows = min(C::BM, x.R - qt * C::BM);
            const int n_live = (live_rows + 31) & ~31;  // threads of the warpgroup's live warps
            for (int z = r; z < nz; z += n_live) {
              const int dh = z / per_dh, rem = z - dh * per_dh;
              const int row = z0 + rem / 8, chn = rem % 8;
              *reinterpret_cast<uint4*>(sV + vs * C::kKVBytes + dh * C::BN * 128 + row * 128 + chn * 16) =
                  make_uint4(0, 0, 0, 0);
            }
            ptx::fence_proxy_async_smem();
          }
          PH_MARK(5);
          ptx::tmem_st_wait();
        }
        // padding warps write no P: arriving right after their s_full wait
        // is safe, because tile lt + 2 cannot start before this phase ends
        ptx::tc_fence_before();
        __syncwarp();
        if (lane == 0) ptx::mbar_arrive(p_full(qt, sb));
        PH_MARK(6);
      }
      if (!ok) break;
      // epilogue: wait for the unit's last PV, read the O row out of TMEM
      // half at a time (one wait per half), normalise and store it, and free
      // O (the next unit's first P.V may start; the stores are in flight)
      const int last = lt - 1;
      if (!wait_or_flag(pv_done(qt, last & 1), (last >> 1) & 1, err, ok)) break;
      PH_MARK(7);
      ptx::tc_fence_after();
      if (warp_live) {
        const int row = x.row0 + rr / g;
        const int qh = x.h * g + (rr % g);
        const float inv = l > 0.f ? 1.f / l : 0.f;
        const bool wide = ((reinterpret_cast<uintptr_t>(a.out) | reinterpret_cast<uintptr_t>(a.part_o)) & 31u) == 0;
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
          uint32_t o[D / 2];
#pragma unroll
          for (int c = 0; c < D / 64; ++c)
            ptx::tmem_ld32(tmem + lane_base + col_o + hh * (D / 2) + c * 32,
                           *reinterpret_cast<uint32_t(*)[32]>(&o[c * 32]));
          ptx::tmem_ld_wait();
          if (!row_ok) continue;
          // a thread writes its own row, so each store instruction touches
          // 32 rows; 32-byte stores (when the bases allow) halve their number
          if (x.part < 0) {
            __nv_bfloat16* dst = a.out + ((int64_t)row * a.Hq + qh) * D + hh * (D / 2);
#pragma unroll
            for (int q8 = 0; q8 < D / 32; ++q8) {
              uint32_t w[8];
#pragma unroll
              for (int e = 0; e < 8; ++e) {
                __nv_bfloat162 pr = __floats2bfloat162_rn(__uint_as_float(o[q8 * 16 + 2 * e]) * inv,
                                                          __uint_as_float(o[q8 * 16 + 2 * e + 1]) * inv);
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
          } else {
            float* dst = a.part_o + (int64_t)(x.part + rr) * D + hh * (D / 2);
#pragma unroll
            for (int q8 = 0; q8 < D / 16; ++q8) {
              if (wide) {
                ptx::st_global_v8(dst + q8 * 8, &o[q8 * 8]);
              } else {
                float4* d4 = reinterpret_cast<float4*>(dst + q8 * 8);
                d4[0] = make_float4(__uint_as_float(o[8 * q8]), __uint_as_float(o[8 * q8 + 1]),
                                    __uint_as_float(o[8 * q8 + 2]), __uint_as_float(o[8 * q8 + 3]));
                d4[1] = make_float4(__uint_as_float(o[8 * q8 + 4]), __uint_as_float(o[8 * q8 + 5]),
                                    __uint_as_float(o[8 * q8 + 6]), __uint_as_float(o[8 * q8 + 7]));
              }
            }
          }
        }
        if (row_ok && x.part >= 0) {
          a.part_ml[(int64_t)(x.part + rr) * 2] = m_used;
          a.part_ml[(int64_t)(x.part + rr) * 2 + 1] = l;
        }
      }
      ptx::tc_fence_before();
      __syncwarp();
      if (lane == 0) ptx::mbar_arrive(o_free(qt));
      PH_MARK(8);
    }
    PH_FLUSH(lane == 0 && (warp & 3) == 0, 12 * qt, 12);
  }
  ptx::tc_fence_before();
  __syncthreads();
  if (warp == 9) {
    ptx::tc_fence_after();
    ptx::tmem_dealloc(tmem, C::kTmemCols);
  }
#ifdef FG_PHASE_TRACE
  if (threadIdx.x == 0) {
    atomicAdd(&g_phase[56], (unsigned long long)(clock64() - cta_t0));
    atomicAdd(&g_phase[57], 1ull);
    atomicMax(&g_phase[60], ptx::global_timer_ns());
  }
#endif
}

template <int D, bool ROPE>
cudaError_t launch_tc_d(const CUtensorMap& tm_q, const CUtensorMap& tm_kv, const TcArgs& args, int grid,
                        cudaStream_t stream) {
  using C = TcCfg<D>;
  // per device: the attributes apply to the current device only
  static PerDeviceOnce configured;
  cudaError_t e0 = configured.run([] {
    cudaError_t e = cudaFuncSetAttribute(attn_tc_kernel<D, ROPE>, cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmem);
    // the largest shared-memory carveout, so CTAs of different kernels can
    // share an SM
    if (e == cudaSuccess)
      e = cudaFuncSetAttribute(attn_tc_kernel<D, ROPE>, cudaFuncAttributePreferredSharedMemoryCarveout,
                               cudaSharedmemCarveoutMaxShared);
    return e;
  });
  if (e0 != cudaSuccess) return e0;
  attn_tc_kernel<D, ROPE><<<grid, C::kThreads, C::kSmem, stream>>>(tm_q, tm_kv, args);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_attention_tc(const void* tm_q, const void* tm_kv, const CacheView& cache,
                                const BatchView& batch, const WorkItem* items, int n_items,
                                __nv_bfloat16* out, float* part_o, float* part_ml, int n_q_heads,
                                int g, float scale_log2, int window, int grid, int sm_end,
                                int* counter, cudaStream_t stream, const double2* rope) {
  if (n_items == 0) return cudaSuccess;
  TcArgs args{cache, batch, items, out, part_o, part_ml, n_q_heads, g, scale_log2, window, n_items,
              counter, sm_end, rope};
  grid = grid < 1 ? 1 : (grid > n_items ? n_items : grid);
  const CUtensorMap& q = *static_cast<const CUtensorMap*>(tm_q);
  const CUtensorMap& kv = *static_cast<const CUtensorMap*>(tm_kv);
  if (rope) {
    if (cache.head_dim == 128) return launch_tc_d<128, true>(q, kv, args, grid, stream);
    return launch_tc_d<64, true>(q, kv, args, grid, stream);
  }
  if (cache.head_dim == 128) return launch_tc_d<128, false>(q, kv, args, grid, stream);
  return launch_tc_d<64, false>(q, kv, args, grid, stream);
}

}  // namespace fg

#ifdef FG_PHASE_TRACE
// Trace build only: copies the query-tile kernel's phase-cycle table (the
// slot layout above g_phase) to `out` (n <= 64 entries, host memory) after
// synchronising the device, and zeroes it when `reset` is set. 0 on success.
extern "C" int fg_phase_trace_read(unsigned long long* out, int n, int reset) {
  if (!out || n < 0 || n > fg::kPhaseSlots) return 1;
  if (cudaDeviceSynchronize() != cudaSuccess) return 2;
  if (cudaMemcpyFromSymbol(out, fg::g_phase, (size_t)n * 8) != cudaSuccess) return 2;
  if (reset) {
    unsigned long long init[fg::kPhaseSlots] = {};
    init[58] = ~0ull;  // running minimum
    if (cudaMemcpyToSymbol(fg::g_phase, init, sizeof(init)) != cudaSuccess) return 2;
  }
  return 0;
}
#endif
