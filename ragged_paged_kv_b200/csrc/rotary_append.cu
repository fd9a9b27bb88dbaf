// Step 1 + 2 of the forward pass: rotary on Q and K, then append K_rot and V
// into the blocked KV cache ("DeepSpeed-FastGen — paper by Holmes et al.
// (2024)", Key points: blocked KV cache as in PagedAttention).
//
// One CTA per batch row (token). Each thread rotates 8 (i, i + d/2) pairs at a
// time with 16-byte loads of both halves and writes 16-byte stores, so every
// global access is a full, aligned 16-byte vector; a thread issues the loads
// of four heads before it computes and stores any of them. The rotation runs in double
// so that it rounds exactly once: a bf16 times a float product is exact in
// double (8 + 24 significant bits), the sum rounds once, and the double is
// rounded straight to bf16 (ties to even) - no float intermediate that could
// round twice.
#include "fg_internal.h"

namespace fg {
namespace {

// float64 -> bf16, round to nearest even, one rounding. Truncate to float and
// force the last float bit on when the truncation dropped anything ("round
// to odd", Boldo & Melquiond 2008): with 16 spare bits between float and bf16
// the following float -> bf16 round-to-nearest-even then equals the direct
// rounding of the double, subnormals included.
__device__ __forceinline__ unsigned short f64_to_bf16_rne(double x) {
  float f = __double2float_rz(x);
  if ((double)f != x) f = __uint_as_float(__float_as_uint(f) | 1u);
  return __bfloat16_as_ushort(__float2bfloat16_rn(f));
}

__device__ __forceinline__ double bf16_lo(uint32_t w) { return (double)__uint_as_float(w << 16); }
__device__ __forceinline__ double bf16_hi(uint32_t w) { return (double)__uint_as_float(w & 0xFFFF0000u); }

__device__ __forceinline__ const __nv_bfloat16* k_in(const __nv_bfloat16* k, int t, int Hkv, int h, int D) {
  return k + ((int64_t)t * Hkv + h) * D;
}

template <int D>
__global__ void __launch_bounds__(128) rotary_append_kernel(CacheView cache, BatchView batch,
                                                            const __nv_bfloat16* q,
                                                            const __nv_bfloat16* __restrict__ k,
                                                            const __nv_bfloat16* __restrict__ v,
                                                            __nv_bfloat16* q_rot,
                                                            const float2* __restrict__ rope,
                                                            int Hq) {
  constexpr int HALF = D / 2;
  constexpr int GROUPS = HALF / 8;  // 8-pair groups per head
  const int t = blockIdx.x;
  const int Hkv = cache.n_kv_heads;
  const int s = batch.tok_seq[t];
  const int p = batch.ctx[s] + (t - batch.cu_q[s]);
  const int lb = p / cache.block_size;
  const int slot = p - lb * cache.block_size;
  int32_t blk = batch.bt[batch.bt_off[s] + lb];
  const bool blk_ok = blk >= 0 && blk < cache.n_blocks;
  if (!blk_ok && threadIdx.x == 0) atomicOr(batch.err, kErrBadBlock);
  // Every thread handles the same 8-pair group i0 of several heads (the block
  // size is a multiple of the groups per head), so its 8 (cos, sin) pairs are
  // loaded once; all loads of a batch of heads are issued before any store.
  static_assert(128 % GROUPS == 0, "block size must be a multiple of the groups per head");
  const int i0 = (threadIdx.x % GROUPS) * 8;
  float cs[8], sn[8];
  {
    const float4* r4 = reinterpret_cast<const float4*>(rope + (int64_t)p * HALF + i0);
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const float4 r = r4[e];
      cs[2 * e] = r.x; sn[2 * e] = r.y; cs[2 * e + 1] = r.z; sn[2 * e + 1] = r.w;
    }
  }
  constexpr int BATCH = 4;
  const int total = (Hq + Hkv) * GROUPS;
  for (int base = threadIdx.x; base < total; base += BATCH * 128) {
    uint4 a[BATCH], b[BATCH];
#pragma unroll
    for (int j = 0; j < BATCH; ++j) {
      const int gi = base + j * 128;
      if (gi >= total) break;
      const int h = gi / GROUPS;
      const __nv_bfloat16* src = h < Hq ? q + ((int64_t)t * Hq + h) * D
                                        : k_in(k, t, Hkv, h - Hq, D);
      a[j] = *reinterpret_cast<const uint4*>(src + i0);
      b[j] = *reinterpret_cast<const uint4*>(src + HALF + i0);
    }
#pragma unroll
    for (int j = 0; j < BATCH; ++j) {
      const int gi = base + j * 128;
      if (gi >= total) break;
      const int h = gi / GROUPS;
      const uint32_t aw[4] = {a[j].x, a[j].y, a[j].z, a[j].w};
      const uint32_t bw[4] = {b[j].x, b[j].y, b[j].z, b[j].w};
      uint32_t y1[4], y2[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const double x1l = bf16_lo(aw[e]), x1h = bf16_hi(aw[e]);
        const double x2l = bf16_lo(bw[e]), x2h = bf16_hi(bw[e]);
        const double cl = cs[2 * e], sl = sn[2 * e], ch = cs[2 * e + 1], sh = sn[2 * e + 1];
        const unsigned short r1l = f64_to_bf16_rne(__dsub_rn(__dmul_rn(x1l, cl), __dmul_rn(x2l, sl)));
        const unsigned short r1h = f64_to_bf16_rne(__dsub_rn(__dmul_rn(x1h, ch), __dmul_rn(x2h, sh)));
        const unsigned short r2l = f64_to_bf16_rne(__dadd_rn(__dmul_rn(x2l, cl), __dmul_rn(x1l, sl)));
        const unsigned short r2h = f64_to_bf16_rne(__dadd_rn(__dmul_rn(x2h, ch), __dmul_rn(x1h, sh)));
        y1[e] = (uint32_t)r1l | ((uint32_t)r1h << 16);
        y2[e] = (uint32_t)r2l | ((uint32_t)r2h << 16);
      }
      __nv_bfloat16* dst;
      if (h < Hq) {
        dst = q_rot + ((int64_t)t * Hq + h) * D;
      } else {
        if (!blk_ok) continue;
        dst = cache.base + cache_offset(cache, blk, 0, h - Hq, slot);
      }
      *reinterpret_cast<uint4*>(dst + i0) = make_uint4(y1[0], y1[1], y1[2], y1[3]);
      *reinterpret_cast<uint4*>(dst + HALF + i0) = make_uint4(y2[0], y2[1], y2[2], y2[3]);
    }
  }
  if (!blk_ok) return;
  constexpr int VCH = D / 8;
  const int nv = Hkv * VCH;
  for (int base = threadIdx.x; base < nv; base += BATCH * 128) {
    uint4 x[BATCH];
#pragma unroll
    for (int j = 0; j < BATCH; ++j) {
      const int ci = base + j * 128;
      if (ci >= nv) break;
      const int h = ci / VCH;
      x[j] = *reinterpret_cast<const uint4*>(v + ((int64_t)t * Hkv + h) * D + (ci - h * VCH) * 8);
    }
#pragma unroll
    for (int j = 0; j < BATCH; ++j) {
      const int ci = base + j * 128;
      if (ci >= nv) break;
      const int h = ci / VCH;
      *reinterpret_cast<uint4*>(cache.base + cache_offset(cache, blk, 1, h, slot) + (ci - h * VCH) * 8) = x[j];
    }
  }
}

}  // namespace

cudaError_t launch_rotary_append(const CacheView& cache, const BatchView& batch,
                                 const __nv_bfloat16* q, const __nv_bfloat16* k,
                                 const __nv_bfloat16* v, __nv_bfloat16* q_rot, const float2* rope,
                                 int n_q_heads, cudaStream_t stream) {
  if (batch.n_tokens == 0) return cudaSuccess;
  dim3 grid(batch.n_tokens), block(128);
  if (cache.head_dim == 128)
    rotary_append_kernel<128><<<grid, block, 0, stream>>>(cache, batch, q, k, v, q_rot, rope, n_q_heads);
  else
    rotary_append_kernel<64><<<grid, block, 0, stream>>>(cache, batch, q, k, v, q_rot, rope, n_q_heads);
  return cudaGetLastError();
}

}  // namespace fg
