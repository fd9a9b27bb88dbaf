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
#include "sm100_ptx.cuh"

namespace fg {
namespace {

// float64 -> bf16, round to nearest even, one rounding. Truncate to float and
// force the last float bit on when the truncation dropped anything ("round
// to odd", Boldo & Melquiond 2008): with 16 spare bits between float and bf16
// the following float -> bf16 round-to-nearest-even then equals the direct
// rounding of the double, subnormals included. Exact for every double; the
// kernel uses it only for vectors the fast path below does not cover.
__device__ __noinline__ unsigned short f64_to_bf16_rne_slow(double x) {
  float f = __double2float_rz(x);
  if ((double)f != x) f = __uint_as_float(__float_as_uint(f) | 1u);
  return __bfloat16_as_ushort(__float2bfloat16_rn(f));
}

// float64 -> bf16, round to nearest even, one rounding, as one PTX
// conversion (cvt.rn.bf16.f64). On B200 it gives the same bits as the
// round-to-odd path above for every finite double tried (2^32 of them:
// random bit patterns, neighbours of bf16 midpoints, the subnormal range,
// overflow), subnormal results included.
__device__ __forceinline__ uint32_t f64_to_bf16_cvt(double y) {
  unsigned short r;
  asm("cvt.rn.bf16.f64 %0, %1;" : "=h"(r) : "d"(y));
  return r;
}

// A bf16 pattern widened to a double whose value is 2^-896 times the bf16's
// value, by moving its 8 exponent bits to the low end of the double's 11-bit
// exponent field (an arithmetic shift keeps the sign on top, the mask clears
// the three bits in between). Exact for zero, subnormal and normal patterns;
// infinities and NaNs are screened out per vector first. The rotary table is
// stored times 2^896, so each product x * cos is exact and unscaled.
__device__ __forceinline__ double bf16_lo_scaled(uint32_t w) {
  return __hiloint2double((int)(((uint32_t)((int32_t)(w << 16) >> 3)) & 0x8FFFFFFFu), 0);
}
__device__ __forceinline__ double bf16_hi_scaled(uint32_t w) {
  return __hiloint2double((int)(((uint32_t)((int32_t)w >> 3)) & 0x8FFFE000u), 0);
}
// Bit 15 or 31 is set iff the low or high bf16 of w has an all-ones exponent.
__device__ __forceinline__ uint32_t special_bits(uint32_t w) {
  return ((w & 0x7F807F80u) + 0x00800080u) & 0x80008000u;
}
__device__ __forceinline__ double bf16_lo(uint32_t w) { return (double)__uint_as_float(w << 16); }
__device__ __forceinline__ double bf16_hi(uint32_t w) { return (double)__uint_as_float(w & 0xFFFF0000u); }

// Rotation of one word pair (two pairs (x1, x2)) the plain way, for the
// vectors the fast path does not cover; the table entries are times 2^896.
__device__ __noinline__ uint2 rotate_pair_slow(uint32_t a, uint32_t b, double2 r_lo, double2 r_hi) {
  const double x1l = bf16_lo(a), x1h = bf16_hi(a), x2l = bf16_lo(b), x2h = bf16_hi(b);
  const double cl = r_lo.x * 0x1p-896, sl = r_lo.y * 0x1p-896;
  const double ch = r_hi.x * 0x1p-896, sh = r_hi.y * 0x1p-896;
  const unsigned short r1l = f64_to_bf16_rne_slow(__dsub_rn(__dmul_rn(x1l, cl), __dmul_rn(x2l, sl)));
  const unsigned short r1h = f64_to_bf16_rne_slow(__dsub_rn(__dmul_rn(x1h, ch), __dmul_rn(x2h, sh)));
  const unsigned short r2l = f64_to_bf16_rne_slow(__dadd_rn(__dmul_rn(x2l, cl), __dmul_rn(x1l, sl)));
  const unsigned short r2h = f64_to_bf16_rne_slow(__dadd_rn(__dmul_rn(x2h, ch), __dmul_rn(x1h, sh)));
  return make_uint2((uint32_t)r1l | ((uint32_t)r1h << 16), (uint32_t)r2l | ((uint32_t)r2h << 16));
}

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
// (blockIdx.x, + gridDim.x, ...) its lane j resolves unit j's sequence,
// position and cache block (a chain of dependent metadata loads; the 32
// chains run at once) into a shared batch table; lane 0 then, stage by
// stage, writes a unit's metadata into the stage and pulls its rows (each of
// q, k and v a contiguous run of whole heads) and the position's rotary row
// with 1-D bulk copies on the stage's mbarrier. Warps 0-3 rotate from shared
// memory and store 16-byte vectors, then free the stage.
// ROT = false: the append alone (models without rotary embedding): the head
// list is k | v (Hq = 0) and K is copied like V.
template <int D, bool ROT>
__global__ void __launch_bounds__(kConsumers + 32, kCtasPerSm) rotary_append_kernel(
    CacheView cache, BatchView batch, const __nv_bfloat16* q, const __nv_bfloat16* k,
    const __nv_bfloat16* v, __nv_bfloat16* q_rot, const double2* __restrict__ rope, int Hq, int chunks) {
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
          const int s = batch.tok_seq[t];
          const int pos = batch.ctx[s] + (t - batch.cu_q[s]);
          const int lb = pos / cache.block_size;
          m.t = t;
          m.h0 = h0;
          m.h1 = min(h0 + kChunkHeads, Hq + 2 * Hkv);
          m.blk = batch.bt[batch.bt_off[s] + lb];
          m.slot = pos - lb * cache.block_size;
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
          const bool rot = ROT && h0 < Hq + Hkv;
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
        const uint32_t aw[4] = {a.x, a.y, a.z, a.w};
        const uint32_t bw[4] = {b.x, b.y, b.z, b.w};
        uint32_t y1[4], y2[4];
        uint32_t special = 0;
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          special |= special_bits(aw[e]) | special_bits(bw[e]);
          const double x1l = bf16_lo_scaled(aw[e]), x1h = bf16_hi_scaled(aw[e]);
          const double x2l = bf16_lo_scaled(bw[e]), x2h = bf16_hi_scaled(bw[e]);
          const double cl = cs[2 * e], sl = sn[2 * e], ch = cs[2 * e + 1], sh = sn[2 * e + 1];
          // both products are exact, so one fused multiply-add rounds the
          // difference exactly once
          const double r1l = __fma_rn(x1l, cl, -__dmul_rn(x2l, sl));
          const double r1h = __fma_rn(x1h, ch, -__dmul_rn(x2h, sh));
          const double r2l = __fma_rn(x2l, cl, __dmul_rn(x1l, sl));
          const double r2h = __fma_rn(x2h, ch, __dmul_rn(x1h, sh));
          y1[e] = f64_to_bf16_cvt(r1l) | (f64_to_bf16_cvt(r1h) << 16);
          y2[e] = f64_to_bf16_cvt(r2l) | (f64_to_bf16_cvt(r2h) << 16);
        }
        if (special != 0u) {
          // an infinite or NaN input: redo the vector with plain widening and
          // the exact narrowing
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const uint2 r = rotate_pair_slow(aw[e], bw[e], rs[(2 * e) * GROUPS + g], rs[(2 * e + 1) * GROUPS + g]);
            y1[e] = r.x;
            y2[e] = r.y;
          }
        }
        __nv_bfloat16* dst;
        if (h < Hq) {
          dst = q_rot + ((int64_t)m.t * Hq + h) * D;
        } else {
          if (!blk_ok) continue;
          dst = cache.base + cache_offset(cache, m.blk, 0, h - Hq, m.slot);
        }
        *reinterpret_cast<uint4*>(dst + i0) = make_uint4(y1[0], y1[1], y1[2], y1[3]);
        *reinterpret_cast<uint4*>(dst + HALF + i0) = make_uint4(y2[0], y2[1], y2[2], y2[3]);
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
                                 int n_q_heads, bool rotate, cudaStream_t stream) {
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
          cache, batch, q, k, v, q_rot, rope, n_q_heads, chunks);
    else
      rotary_append_kernel<128, false><<<grid, kConsumers + 32, RotCfg<128>::kSmem, stream>>>(
          cache, batch, q, k, v, q_rot, rope, n_q_heads, chunks);
  } else {
    if (rotate)
      rotary_append_kernel<64, true><<<grid, kConsumers + 32, RotCfg<64>::kSmem, stream>>>(
          cache, batch, q, k, v, q_rot, rope, n_q_heads, chunks);
    else
      rotary_append_kernel<64, false><<<grid, kConsumers + 32, RotCfg<64>::kSmem, stream>>>(
          cache, batch, q, k, v, q_rot, rope, n_q_heads, chunks);
  }
  return cudaGetLastError();
}

}  // namespace fg
