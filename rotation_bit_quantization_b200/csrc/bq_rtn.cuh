// Exact per-group asymmetric RTN in float32, shared by the specialised kernels.
//
// Quantizer (ButterflyQuant explainer, section "training & results": 2-bit
// weights; RTN block quantizer: WUSH technical summary, section 2), per group
// of contiguous outputs with qmax = 2^bits - 1:
//   lo, hi = min, max;  scale16 = fp16_rn((hi - lo) / qmax);  s = scale16
//   (s = 1 when hi == lo or scale16 == 0);  z = clamp(rint(-lo / s), 0, qmax)
//   q = clamp(rint(y / s) + z, 0, qmax)  with IEEE float32 division, rint
//   half-to-even.
//
// Fast path: with inv = 1 / s correctly rounded, y * inv + (1.5 * 2^23 + z) is
// rounded once to an integer whose low bits are the code; when y * inv is far
// enough from every half-integer (relative to vmax, a bound on |y * inv| over
// the group) that integer is rint(RN(y / s)) + z (see rtn_codes8).  A set of 8
// values with any element near a tie (or a NaN), or a group whose extremes
// would need clamping, is redone with IEEE division.
#pragma once

#include "bq_internal.cuh"

namespace bq {

// 3-input maximum that returns NaN if any input is NaN
__device__ __forceinline__ float max_nan3(float a, float b, float c) {
  float d;
  asm("max.NaN.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}

struct RtnParams {
  float inv;   // 1 / s, correctly rounded
  float thr;   // tie threshold on |v - rint(v)|; -1 sends every set to the slow path
  float mz;    // 1.5 * 2^23 + z
  float s;     // scale as float
  uint16_t scale16, zero16;
};

// rint(RN(-lo / s)) and rint(RN(hi / s)) of a group's extremes, by the same
// exact-RTN argument as rtn_codes8 (fast path: one packed FMA pair and the tie
// test; IEEE division only when either quotient is near a half-integer).
__device__ __forceinline__ float2 rint_extremes(float lo, float hi, float s, float inv, float thr) {
  const float2 v = make_float2(-lo, hi);
  const float2 m2 = make_float2(12582912.f, 12582912.f);   // 1.5 * 2^23
  const float2 t = __ffma2_rn(v, make_float2(inv, inv), m2);
  const float2 r = __fadd2_rn(t, make_float2(-12582912.f, -12582912.f));
  const float2 e = __ffma2_rn(v, make_float2(-inv, -inv), r);
  if (fmaxf(fabsf(e.x), fabsf(e.y)) < thr) return r;        // also false for a NaN
  return make_float2(rintf(__fdiv_rn(-lo, s)), rintf(__fdiv_rn(hi, s)));
}

__device__ __forceinline__ RtnParams rtn_params(float lo, float hi, float qmax) {
  RtnParams p;
  __half h16 = __float2half_rn(__fdiv_rn(__fsub_rn(hi, lo), qmax));
  float s = __half2float(h16);
  if (hi == lo || s == 0.f) {
    s = 1.f;
    h16 = __float2half_rn(1.f);
  }
  const float inv = __frcp_rn(s);  // correctly rounded 1 / s
  const float vmax = fmaxf(fabsf(lo), fabsf(hi)) * inv * 1.000001f;
  const float thr = vmax < 4194304.f ? 0.5f - vmax * 9.5367431640625e-7f : -1.f;  // 2^22, 2^-20
  const float2 ext = rint_extremes(lo, hi, s, inv, thr);
  const float zraw = ext.x;
  const float z = __fadd_rn(fminf(fmaxf(zraw, 0.f), qmax), 0.f);  // +0 for a zero point of 0
  // codes are monotone in y: the group needs no clamping iff its extremes land in
  // [0, qmax]; the bottom is z - rint(-lo / s) (division and rint are odd functions)
  const bool inrange = zraw <= qmax && __fadd_rn(ext.y, z) <= qmax;
  p.inv = inv;
  p.thr = inrange ? thr : -1.f;
  p.mz = __fadd_rn(12582912.f, z);
  p.s = s;
  p.scale16 = __half_as_ushort(h16);
  p.zero16 = __half_as_ushort(__float2half_rn(z));
  return p;
}

// Codes of 8 values by IEEE division (slow path, out of line).
template <int BITS>
__device__ __noinline__ uint32_t rtn_codes_by_division(float y0, float y1, float y2, float y3, float y4, float y5,
                                                        float y6, float y7, float s, float z) {
  const float qmax = static_cast<float>((1 << BITS) - 1);
  const float y[8] = {y0, y1, y2, y3, y4, y5, y6, y7};
  uint32_t word = 0;
#pragma unroll
  for (int e = 0; e < 8; ++e) {
    const float t = fminf(fmaxf(__fadd_rn(rintf(__fdiv_rn(y[e], s)), z), 0.f), qmax);
    word |= static_cast<uint32_t>(t) << (BITS * e);
  }
  return word;
}

// Packed codes of 8 consecutive values (lowest element in the lowest bits):
// INT4 -> 32 bits, INT2 -> 16 bits.
//
// With P = y * inv exact and |P| < 2^22: t = RN(P + mz) = mz + rint(P) (the sum
// lies in (2^23, 2^24), where the float32 spacing is 1), r = t - mz = rint(P)
// exactly, and e = RN(r - P) is within 2^-25 of r - P.  The threshold
// thr = RN(0.5 - vmax 2^-20) then leaves P at least vmax 2^-20 - 2^-24 away
// from every half-integer whenever |e| < thr, which exceeds
// |RN(y / s) - P| <= 2^-23 vmax once vmax > 1/14; below that |P| and |y / s|
// are both under 1/2 and every code is z.  So rint(RN(y / s)) = r on the
// fast path, and t's low bits carry r + z.
template <int BITS>
__device__ __forceinline__ uint32_t rtn_codes8(const float2 (&y)[4], float inv, float thr, float mz, float s) {
  const float2 iv = make_float2(inv, inv), niv = make_float2(-inv, -inv);
  const float2 m2 = make_float2(mz, mz), nm2 = make_float2(-mz, -mz);
  uint32_t b[8];
  float emax = 0.f;
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    const float2 t = __ffma2_rn(y[q], iv, m2);        // mz + rint(y * inv)
    const float2 r = __fadd2_rn(t, nm2);               // rint(y * inv), exact
    const float2 e = __ffma2_rn(y[q], niv, r);         // r - y * inv, one rounding
    emax = max_nan3(emax, fabsf(e.x), fabsf(e.y));  // a NaN goes to the slow path
    b[2 * q] = __float_as_uint(t.x);
    b[2 * q + 1] = __float_as_uint(t.y);
  }
  uint32_t word;
  if constexpr (BITS == 4) {
    const uint32_t p0 = b[0] + (b[1] << 4), p1 = b[2] + (b[3] << 4);
    const uint32_t p2 = b[4] + (b[5] << 4), p3 = b[6] + (b[7] << 4);
    word = __byte_perm(__byte_perm(p0, p1, 0x0040), __byte_perm(p2, p3, 0x0040), 0x5410);
  } else {
    const uint32_t p0 = b[0] + (b[1] << 2) + (b[2] << 4) + (b[3] << 6);
    const uint32_t p1 = b[4] + (b[5] << 2) + (b[6] << 4) + (b[7] << 6);
    word = __byte_perm(p0, p1, 0x0040) & 0xffffu;
  }
  if (!(emax < thr))
    word = rtn_codes_by_division<BITS>(y[0].x, y[0].y, y[1].x, y[1].y, y[2].x, y[2].y, y[3].x, y[3].y, s,
                                       __fadd_rn(mz, -12582912.f));
  return word;
}

}  // namespace bq
