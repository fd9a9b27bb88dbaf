// The exact rotary arithmetic shared by the kernels that rotate Q or K:
// rotate-half, y1 = x1 c - x2 s and y2 = x2 c + x1 s for each (i, i + d/2)
// pair, with c and s the fp32 table values, every product exact in double,
// the sum rounded once to double and the double rounded once to bf16 (ties
// to even) — the rotation of "DeepSpeed-FastGen — paper by Holmes et al.
// (2024)" (Key points: LLaMA-family models), with the rounding written out
// so that the cache and the rotated queries come out bit for bit the same
// wherever they are computed.
#pragma once

#include <cuda_bf16.h>
#include <cstdint>

namespace fg {
namespace rope {

// float64 -> bf16, round to nearest even, one rounding. Truncate to float and
// force the last float bit on when the truncation dropped anything ("round
// to odd", Boldo & Melquiond 2008): with 16 spare bits between float and bf16
// the following float -> bf16 round-to-nearest-even then equals the direct
// rounding of the double, subnormals included. Exact for every double; used
// only for vectors the fast path below does not cover.
static __device__ __noinline__ unsigned short f64_to_bf16_rne_slow(double x) {
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
static __device__ __noinline__ uint2 rotate_pair_slow(uint32_t a, uint32_t b, double2 r_lo, double2 r_hi) {
  const double x1l = bf16_lo(a), x1h = bf16_hi(a), x2l = bf16_lo(b), x2h = bf16_hi(b);
  const double cl = r_lo.x * 0x1p-896, sl = r_lo.y * 0x1p-896;
  const double ch = r_hi.x * 0x1p-896, sh = r_hi.y * 0x1p-896;
  const unsigned short r1l = f64_to_bf16_rne_slow(__dsub_rn(__dmul_rn(x1l, cl), __dmul_rn(x2l, sl)));
  const unsigned short r1h = f64_to_bf16_rne_slow(__dsub_rn(__dmul_rn(x1h, ch), __dmul_rn(x2h, sh)));
  const unsigned short r2l = f64_to_bf16_rne_slow(__dadd_rn(__dmul_rn(x2l, cl), __dmul_rn(x1l, sl)));
  const unsigned short r2h = f64_to_bf16_rne_slow(__dadd_rn(__dmul_rn(x2h, ch), __dmul_rn(x1h, sh)));
  return make_uint2((uint32_t)r1l | ((uint32_t)r1h << 16), (uint32_t)r2l | ((uint32_t)r2h << 16));
}

// Rotates 8 pairs: a holds x1 of pairs 0..7 (8 bf16), b their x2; rope(e)
// returns pair e's (cos, sin) times 2^896 as a double2. y1 gets x1 c - x2 s,
// y2 gets x2 c + x1 s, each rounded exactly as above.
template <class Rope>
__device__ __forceinline__ void rotate8(const uint4& a, const uint4& b, Rope rope, uint4& y1, uint4& y2) {
  const uint32_t aw[4] = {a.x, a.y, a.z, a.w};
  const uint32_t bw[4] = {b.x, b.y, b.z, b.w};
  uint32_t r1[4], r2[4];
  uint32_t special = 0;
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    special |= special_bits(aw[e]) | special_bits(bw[e]);
    const double x1l = bf16_lo_scaled(aw[e]), x1h = bf16_hi_scaled(aw[e]);
    const double x2l = bf16_lo_scaled(bw[e]), x2h = bf16_hi_scaled(bw[e]);
    const double2 pl = rope(2 * e), ph = rope(2 * e + 1);
    // both products are exact, so one fused multiply-add rounds the
    // difference exactly once
    const double s1l = __fma_rn(x1l, pl.x, -__dmul_rn(x2l, pl.y));
    const double s1h = __fma_rn(x1h, ph.x, -__dmul_rn(x2h, ph.y));
    const double s2l = __fma_rn(x2l, pl.x, __dmul_rn(x1l, pl.y));
    const double s2h = __fma_rn(x2h, ph.x, __dmul_rn(x1h, ph.y));
    r1[e] = f64_to_bf16_cvt(s1l) | (f64_to_bf16_cvt(s1h) << 16);
    r2[e] = f64_to_bf16_cvt(s2l) | (f64_to_bf16_cvt(s2h) << 16);
  }
  if (special != 0u) {
    // an infinite or NaN input: redo the vector with plain widening and the
    // exact narrowing
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const uint2 r = rotate_pair_slow(aw[e], bw[e], rope(2 * e), rope(2 * e + 1));
      r1[e] = r.x;
      r2[e] = r.y;
    }
  }
  y1 = make_uint4(r1[0], r1[1], r1[2], r1[3]);
  y2 = make_uint4(r2[0], r2[1], r2[2], r2[3]);
}

}  // namespace rope
}  // namespace fg
