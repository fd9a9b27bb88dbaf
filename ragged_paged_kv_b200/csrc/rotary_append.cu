// Step 1 + 2 of the forward pass: rotary on Q and K, then append K_rot and V
// into the blocked KV cache ("DeepSpeed-FastGen — paper by Holmes et al.
// (2024)", Key points: blocked KV cache as in PagedAttention).
//
// Units of (token, chunk of heads) stream through a three-stage shared-memory
// ring per CTA by bulk copy; each consumer thread rotates 8 (i, i + d/2) pairs
// at a time from there and writes 16-byte stores. The rotation runs in double
// so that it rounds exactly as specified: a bf16 times a float product is
// exact in double (8 + 24 significant bits), the sum rounds once to double,
// and the double is rounded to bf16 (ties to even) by one conversion
// instruction, so no intermediate float rounding can change the result.
#include <algorithm>
#include <cfloat>

#include "fg_internal.h"
#include "rope_exact.cuh"
#include "sm100_ptx.cuh"

namespace fg {
namespace {

constexpr long long kWaitLimit = 1LL << 31;
constexpr int kChunkHeads = 32;  // heads (of q | k | v, concatenated) per unit
constexpr int kStages = 3;
constexpr int kCtasPerSm = 4;
constexpr int kConsumers = 128;

// What the producer tells the consumers about a unit.
struct UnitMeta {
  int32_t t, h0, h1, blk, slot, pos, pad[2];
};

template <int D>
struct RotCfg {
  static constexpr int ROW = D * 2;  // bytes per head row
  static constexpr int HALF = D / 2;
  static constexpr int kRows = 0;
  static constexpr int kRope = kRows + kChunkHeads * ROW;  // HALF (cos, sin) pairs of double
  static constexpr int kMeta = kRope + HALF * 16;
  static constexpr int kStage = kMeta + (int)sizeof(UnitMeta);
  static constexpr int kBar = kStages * kStage;
  static constexpr int kMetaRing = kBar + 2 * kStages * 8;  // 32 UnitMeta: the producer warp's batch
  static constexpr int kSmem = kMetaRing + 32 * (int)sizeof(UnitMeta);
};

// A unit is (token, chunk of 32 heads of the concatenated q | k | v rows).
// Warp 4 is the producer. For each batch of 32 of the CTA's units
// (blockIdx.x, + gridDim.x, ...) its lane j reads unit j's position and
// cache block (two independent loads of per-row arrays the batch put
// resolved on the host; the 32 lanes' loads run at once) into a shared batch
// table; lane 0 then, stage by
// stage, writes a unit's metadata into the stage and pulls its rows (each of
// q, k and v a contiguous run of whole heads) and the position's rotary row
// with 1-D bulk copies on the stage's mbarrier. Warps 0-3 rotate from shared
// memory and store 16-byte vectors, then free the stage.
// ROT = false: the append alone (models without rotary embedding): the head
// list is k | v (Hq = 0) and K is copied like V.
template <int D, bool ROT>
__global__ void __launch_bounds__(kConsumers + 32, kCtasPerSm) rotary_append_kernel(
    CacheView cache, BatchView batch, const __nv_bfloat16* q, const __nv_bfloat16* k,
    const __nv_bfloat16* v, __nv_bfloat16* q_rot, const double2* __restrict__ rope, int Hq, int chunks,
    int skip_tc_q) {
  using C = RotCfg<D>;
  constexpr int HALF = C::HALF;
  constexpr int GROUPS = HALF / 8;  // 8-pair groups per head
  constexpr int ROW = C::ROW;
  static_assert(kConsumers % GROUPS == 0, "consumer count must be a multiple of the groups per head");
  extern __shared__ __align__(128) unsigned char smem[];
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + C::kBar);
  uint64_t* empty = full + kStages;
  const int Hkv = cache.n_kv_heads;
  const int n_units = batch.n_tokens * chunks;
  if (threadIdx.x == 0) {
    for (int i = 0; i < kStages; ++i) {
      ptx::mbar_init(&full[i], 1);
      ptx::mbar_init(&empty[i], kConsumers / 32);
    }
    ptx::fence_mbar_init();
  }
  __syncthreads();

  if (threadIdx.x >= kConsumers) {
    // ------------------------------------------------------------ producer
    const int lane = threadIdx.x - kConsumers;
    UnitMeta* batch_meta = reinterpret_cast<UnitMeta*>(smem + C::kMetaRing);
    int it = 0;
    bool ok = true;
    for (int base = blockIdx.x; base < n_units && ok; base += 32 * gridDim.x) {
      {
        const int u = base + lane * gridDim.x;
        UnitMeta m{};
        m.t = -1;
        if (u < n_units) {
          const int t = u / chunks;
          const int h0 = (u - t * chunks) * kChunkHeads;
          const int pos = batch.tok_pos[t];
          m.t = t;
          m.h0 = h0;
          m.h1 = min(h0 + kChunkHeads, Hq + 2 * Hkv);
          // Q rows the query-tile kernel rotates itself (skip_tc_q > 0: the
          // attention call that follows reads unrotated Q for the sequences
          // it serves, the plan's rule with skip_tc_q = the largest group the
          // tensor-core decode kernel takes): the unit keeps its K and V
          if (skip_tc_q > 0 && h0 < Hq) {
            const int s = batch.tok_seq[t];
            const int qn = batch.cu_q[s + 1] - batch.cu_q[s];
            const int grp = Hq / Hkv;
            if (!(qn == 1 && ((D == 128 && grp <= skip_tc_q) || grp == 1))) m.h0 = min(Hq, m.h1);
          }
          m.blk = batch.tok_blk[t];
          m.slot = pos - (pos / cache.block_size) * cache.block_size;
          m.pos = pos;
        }
        batch_meta[lane] = m;
      }
      __syncwarp();
      if (lane == 0) {
        for (int j = 0; j < 32; ++j, ++it) {
          const UnitMeta m = batch_meta[j];
          if (m.t < 0) break;
          const int st = it % kStages;
          if (it >= kStages && !ptx::mbar_wait_bounded(&empty[st], ((it / kStages) - 1) & 1, kWaitLimit)) {
            atomicOr(batch.err, kErrTimeout);
            ok = false;  // the consumers give up on the full barrier of this stage
            break;
          }
          unsigned char* stage = smem + st * C::kStage;
          *reinterpret_cast<UnitMeta*>(stage + C::kMeta) = m;
          const int t = m.t, h0 = m.h0, h1 = m.h1, pos = m.pos;
          const bool rot = ROT && h0 < h1 && h0 < Hq + Hkv;
          ptx::mbar_arrive_expect_tx(&full[st], (uint32_t)((h1 - h0) * ROW + (rot ? HALF * 16 : 0)));
          if (rot) ptx::bulk_g2s(stage + C::kRope, rope + (int64_t)pos * HALF, HALF * 16, &full[st]);
          // [h0, h1) cut by the q, k and v ranges of the concatenated head list
          const int qa = h0, qb = min(h1, Hq);
          if (qa < qb)
            ptx::bulk_g2s(stage, q + ((int64_t)t * Hq + qa) * D, (uint32_t)((qb - qa) * ROW), &full[st]);
          const int ka = max(h0, Hq), kb = min(h1, Hq + Hkv);
          if (ka < kb)
            ptx::bulk_g2s(stage + (ka - h0) * ROW, k + ((int64_t)t * Hkv + (ka - Hq)) * D,
                          (uint32_t)((kb - ka) * ROW), &full[st]);
          const int va = max(h0, Hq + Hkv), vb = h1;
          if (va < vb)
            ptx::bulk_g2s(stage + (va - h0) * ROW, v + ((int64_t)t * Hkv + (va - Hq - Hkv)) * D,
                          (uint32_t)((vb - va) * ROW), &full[st]);
        }
      }
      ok = __shfl_sync(0xffffffffu, ok, 0);
      __syncwarp();  // the batch table is rewritten only after lane 0 has read it
    }
    return;
  }

  // -------------------------------------------------------------- consumers
  const int g = threadIdx.x % GROUPS;  // this thread's 8-pair group of every head it rotates
  const int i0 = g * 8;
  int it = 0;
  for (int u = blockIdx.x; u < n_units; u += gridDim.x, ++it) {
    const int st = it % kStages;
    // the whole warp learns together whether the stage arrived
    const bool landed = ptx::mbar_wait_bounded(&full[st], (it / kStages) & 1, kWaitLimit);
    if (!__all_sync(0xffffffffu, landed)) {
      if ((threadIdx.x & 31) == 0) atomicOr(batch.err, kErrTimeout);
      return;
    }
    const unsigned char* stage = smem + st * C::kStage;
    const UnitMeta m = *reinterpret_cast<const UnitMeta*>(stage + C::kMeta);
    const bool blk_ok = m.blk >= 0 && m.blk < cache.n_blocks;
    if (!blk_ok && threadIdx.x == 0) atomicOr(batch.err, kErrBadBlock);
    const int n_rot = ROT ? max(0, min(m.h1, Hq + Hkv) - m.h0) : 0;  // rotated heads in this unit
    if (n_rot > 0) {
      // the rotary row is stored pair 8 g + e at entry e * GROUPS + g, so
      // these loads are conflict-free
      const double2* rs = reinterpret_cast<const double2*>(stage + C::kRope);
      double cs[8], sn[8];
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        const double2 r = rs[e * GROUPS + g];
        cs[e] = r.x;
        sn[e] = r.y;
      }
      for (int hl = threadIdx.x / GROUPS; hl < n_rot; hl += kConsumers / GROUPS) {
        const int h = m.h0 + hl;
        const uint4 a = *reinterpret_cast<const uint4*>(stage + hl * ROW + i0 * 2);
        const uint4 b = *reinterpret_cast<const uint4*>(stage + hl * ROW + (HALF + i0) * 2);
        uint4 y1, y2;
        rope::rotate8(a, b, [&](int e) { return make_double2(cs[e], sn[e]); }, y1, y2);
        __nv_bfloat16* dst;
        if (h < Hq) {
          dst = q_rot + ((int64_t)m.t * Hq + h) * D;
        } else {
          if (!blk_ok) continue;
          dst = cache.base + cache_offset(cache, m.blk, 0, h - Hq, m.slot);
        }
        *reinterpret_cast<uint4*>(dst + i0) = y1;
        *reinterpret_cast<uint4*>(dst + HALF + i0) = y2;
      }
    }
    if (blk_ok) {
      // V heads (and, without rotary, K heads) of the unit: a plain copy
      // into the cache slots
      constexpr int VCH = D / 8;  // 16-byte pieces per head
      const int v0 = ROT ? max(m.h0, Hq + Hkv) : m.h0;
      const int nv = max(0, m.h1 - v0) * VCH;
      for (int ci = threadIdx.x; ci < nv; ci += kConsumers) {
        const int hl = ci / VCH, c = ci - hl * VCH;
        const int hk = v0 + hl - Hq;  // index in the k | v head list
        const int kv = hk >= Hkv ? 1 : 0;
        *reinterpret_cast<uint4*>(cache.base + cache_offset(cache, m.blk, kv, hk - kv * Hkv, m.slot) + c * 8) =
            *reinterpret_cast<const uint4*>(stage + (v0 - m.h0 + hl) * ROW + c * 16);
      }
    }
    // this warp is done with the stage
    __syncwarp();
    if ((threadIdx.x & 31) == 0) ptx::mbar_arrive(&empty[st]);
  }
}

}  // namespace

cudaError_t launch_rotary_append(const CacheView& cache, const BatchView& batch,
                                 const __nv_bfloat16* q, const __nv_bfloat16* k,
                                 const __nv_bfloat16* v, __nv_bfloat16* q_rot, const double2* rope,
                                 int n_q_heads, bool rotate, cudaStream_t stream, int skip_tc_q) {
  if (batch.n_tokens == 0) return cudaSuccess;
  if (!rotate) n_q_heads = 0;
  const int chunks = (n_q_heads + 2 * cache.n_kv_heads + kChunkHeads - 1) / kChunkHeads;
  const int64_t units = (int64_t)batch.n_tokens * chunks;
  if (units > (int64_t)1 << 30) return cudaErrorInvalidConfiguration;
  int dev = 0, sms = 148;
  if (cudaGetDevice(&dev) != cudaSuccess || cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
    sms = 148;
  const int grid = (int)std::min<int64_t>(units, (int64_t)sms * kCtasPerSm);
  if (cache.head_dim == 128) {
    if (rotate)
      rotary_append_kernel<128, true><<<grid, kConsumers + 32, RotCfg<128>::kSmem, stream>>>(
          cache, batch, q, k, v, q_rot, rope, n_q_heads, chunks, skip_tc_q);
    else
      rotary_append_kernel<128, false><<<grid, kConsumers + 32, RotCfg<128>::kSmem, stream>>>(
          cache, batch, q, k, v, q_rot, rope, n_q_heads, chunks, skip_tc_q);
  } else {
    if (rotate)
      rotary_append_kernel<64, true><<<grid, kConsumers + 32, RotCfg<64>::kSmem, stream>>>(
          cache, batch, q, k, v, q_rot, rope, n_q_heads, chunks, skip_tc_q);
    else
      rotary_append_kernel<64, false><<<grid, kConsumers + 32, RotCfg<64>::kSmem, stream>>>(
          cache, batch, q, k, v, q_rot, rope, n_q_heads, chunks, skip_tc_q);
  }
  return cudaGetLastError();
}

}  // namespace fg
