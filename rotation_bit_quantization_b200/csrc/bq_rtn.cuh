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
// Fast path: v = y * inv with inv = 1 / s correctly rounded, so
// |v - RN(y / s)| <= 1.5 * 2^-23 |y / s|.  When v is farther than vmax * 2^-20
// from every half-integer (vmax bounds |v| over the group), rint(RN(y / s)) =
// rint(v).  rint(v) + z is taken as the bit pattern of v + (1.5 * 2^23 + z)
// (round-half-even addition; no tie can occur on the fast path), so the code
// sits in the low bits.  A set of 8 values with any element near a tie, or a
// group whose extremes would need clamping, is redone with IEEE division.
#pragma once

#include "bq_internal.cuh"

namespace bq {

struct RtnParams {
  float inv;   // 1 / s, correctly rounded
  float thr;   // tie threshold on |v - rint(v)|; -1 sends every set to the slow path
  float mz;    // 1.5 * 2^23 + z
  float s;     // scale as float
  uint16_t scale16, zero16;
};

__device__ __forceinline__ RtnParams rtn_params(float lo, float hi, float qmax) {
  RtnParams p;
  __half h16 = __float2half_rn(__fdiv_rn(__fsub_rn(hi, lo), qmax));
  float s = __half2float(h16);
  if (hi == lo || s == 0.f) {
    s = 1.f;
    h16 = __float2half_rn(1.f);
  }
  const float zraw = rintf(__fdiv_rn(-lo, s));
  const float z = __fadd_rn(fminf(fmaxf(zraw, 0.f), qmax), 0.f);  // +0 for a zero point of 0
  const float inv = __fdiv_rn(1.f, s);
  const float vmax = fmaxf(fabsf(lo), fabsf(hi)) * inv * 1.000001f;
  const float thr = vmax < 4194304.f ? 0.5f - vmax * 9.5367431640625e-7f : -1.f;  // 2^22, 2^-20
  // codes are monotone in y: the group needs no clamping iff its extremes land in
  // [0, qmax]; the bottom is z - rint(-lo / s) (division and rint are odd functions)
  const bool inrange = zraw <= qmax && __fadd_rn(rintf(__fdiv_rn(hi, s)), z) <= qmax;
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
template <int BITS>
__device__ __forceinline__ uint32_t rtn_codes8(const float2 (&y)[4], float inv, float thr, float mz, float s) {
  const float2 iv = make_float2(inv, inv), m2 = make_float2(mz, mz);
  const float2 nm2 = make_float2(-mz, -mz), neg1 = make_float2(-1.f, -1.f);
  bool exact = true;
  uint32_t b[8];
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    const float2 v = __fmul2_rn(y[q], iv);
    const float2 t = __fadd2_rn(v, m2);
    const float2 e = __ffma2_rn(__fadd2_rn(t, nm2), neg1, v);  // v - rint(v), exact
    exact = exact & (fabsf(e.x) < thr) & (fabsf(e.y) < thr);
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
  if (!exact)
    word = rtn_codes_by_division<BITS>(y[0].x, y[0].y, y[1].x, y[1].y, y[2].x, y[2].y, y[3].x, y[3].y, s,
                                       __fadd_rn(mz, -12582912.f));
  return word;
}

}  // namespace bq
