// Device helpers shared by the generic and backward kernels: padded shared-memory
// indexing and the in-register Givens stages of the plain cos/sin form.
//
// Stage s rotates the pair (i, i + 2^s) (ButterflyQuant abstract; explainer
// article, section "butterfly"): forward y_i = c x_i - s x_j, y_j = s x_i + c x_j;
// the transpose (inverse) uses -s.  A work item holds the 8 elements whose
// index differs only in bits [b0, b0 + 3); stage s is the in-register bit
// SB = s - b0.
#pragma once

#include "bq_internal.cuh"

namespace bq {

constexpr int kBitsPerPass = 3;

__host__ __device__ __forceinline__ int pad(int i) { return i + (i >> 5); }

template <int SB, bool INV>
__device__ __forceinline__ void rot_stage(float (&v)[8], int E, int base, int b0, int s,
                                          const float2* __restrict__ cs_s) {
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    if ((j >> SB) & 1) continue;
    if (j >= E) continue;
    const int jj = j | (1 << SB);
    const int i = base | (j << b0);
    const int p = ((i >> (s + 1)) << s) | (i & ((1 << s) - 1));
    const float2 c = __ldg(&cs_s[p]);
    const float a = v[j], b = v[jj];
    if (!INV) {
      v[j] = c.x * a - c.y * b;
      v[jj] = c.y * a + c.x * b;
    } else {
      v[j] = c.x * a + c.y * b;
      v[jj] = c.x * b - c.y * a;
    }
  }
}

template <bool INV>
__device__ __forceinline__ void rot_any(float (&v)[8], int E, int base, int b0, int s, const KLayer& Ly) {
  const float2* cs_s = Ly.cs + size_t(s) * (Ly.m >> 1);
  switch (s - b0) {
    case 0: rot_stage<0, INV>(v, E, base, b0, s, cs_s); break;
    case 1: rot_stage<1, INV>(v, E, base, b0, s, cs_s); break;
    default: rot_stage<2, INV>(v, E, base, b0, s, cs_s); break;
  }
}


}  // namespace bq
