// Specialised Kronecker composite Q = B_1024 (x) O_R (n = 1024 R, R odd <= 7):
// forward with float32 / bfloat16 output, or fused with per-group RTN and
// INT2 / INT4 packing.  Non-power-of-two widths use this composite (ButterflyQuant
// explainer article, section "butterfly"), e.g. the LLaMA-2-13B hidden size
// 5120 = 1024 x 5.
//
// Element i = i1 R + i2 (i1 < 1024, i2 < R); B acts on i1, O_R on each
// contiguous group of R.  The two factors commute, so O_R is applied first.
//
// Design (B200, sm_100a):
//  * One row per CTA of 128 threads (several CTAs per SM: the tensor-memory
//    allocation is 128 columns).  Thread tau = 32 w + l holds 8 values of i1
//    and all R values of i2: 8 R elements.  The 10 stages of B run as three
//    register passes and one shuffle stage:
//        P0: i1 = 8 tau + e                                  stages 0..2
//        P1: i1 = (l & 7) | e << 3 | (l >> 3) << 6 | w << 8  stages 3..5
//        P2: i1 = (l & 15) | w << 4 | e << 6 | (l >> 4) << 9 stages 6..8,
//            then stage 9 across lanes l and l ^ 16
//    P0 holds 8 R contiguous input elements (vector loads) and O_R runs there
//    in registers.  P0 -> P1 stays inside the warp; P1 -> P2 needs the CTA's
//    barrier.  Exchange buffers hold one plane of 1024 per i2 at address
//    p + 4 floor(p / 32) + 16 floor(p / 512), conflict-free on both sides.
//  * The scaled rotation form of the prepared table (a_i += alpha a_j,
//    a_j += beta a_i with the old values; outputs times sigma) when the layer's
//    header flag allows it, else plain cos/sin.  Each thread's 88 coefficients
//    (8 per register stage, 16 for stage 9 with sigma folded in) sit in tensor
//    memory, read one stage at a time with tcgen05.ld.
//  * The result goes through shared memory in element order (upper half of the
//    row shifted by 16 floats: conflict-free for odd R) so that each thread
//    reads R chunks of 8 consecutive elements: vector stores for the float
//    outputs; for RTN, per-chunk min / max are reduced per group through
//    shared memory by one thread per group, which also writes scale and zero.
#include <cfloat>

#include "bq_rtn.cuh"

namespace bq {
namespace {

constexpr int M1 = 1024;
constexpr int kT = 128;
constexpr int kPlane = 1168;  // exchange-buffer floats per i2 plane
constexpr int kRed = 688;     // chunk-extreme slots: cg * S <= 672 for n = 5120

enum KMode { kKF32 = 0, kKBF16 = 1, kKQuant = 2 };

struct KronArgs {
  const void* x;
  void* y;
  long long rows;
  const float* fast;    // [10][1024] scaled-form coefficients
  const float* sigma;   // [1024]
  const float2* cs;     // [10][512] cos, sin
  const float* fast_inv;   // [10][1024] scaled-form coefficients of the inverse
  const float* sigma_inv;  // [1024]
  const float* hdr;     // header: hdr[0] (hdr[3]) == 1 when the scaled form (inverse) is usable
  const float* O;       // [R][R]
  uint8_t* codes;
  uint16_t* scale;
  uint16_t* zero;
  int group;            // RTN group (64, 128 or 256)
};

// ------------------------------------------------------------------ tensor memory

__device__ __forceinline__ void tld8(uint32_t addr, uint32_t (&r)[8]) {
  asm volatile("tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7])
               : "r"(addr));
}

// Waits for this thread's outstanding tensor-memory loads; the registers are
// passed through so that no use of them is scheduled before the wait.
__device__ __forceinline__ void twait(uint32_t (&r)[8]) {
  asm volatile("tcgen05.wait::ld.sync.aligned;"
               : "+r"(r[0]), "+r"(r[1]), "+r"(r[2]), "+r"(r[3]), "+r"(r[4]), "+r"(r[5]), "+r"(r[6]), "+r"(r[7])
               :
               : "memory");
}

__device__ __forceinline__ void tst8(uint32_t addr, const uint32_t (&r)[8]) {
  asm volatile("tcgen05.st.sync.aligned.32x32b.x8.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8};" ::"r"(addr), "r"(r[0]),
               "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7])
               : "memory");
}

__device__ __forceinline__ void cta_sync() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
  __syncthreads();
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

__device__ __forceinline__ float u2f(uint32_t v) { return __uint_as_float(v); }

// ------------------------------------------------------------------ layouts

__device__ __forceinline__ int pos_pass(int P, int tau, int e) {
  const int l = tau & 31, w = tau >> 5;
  if (P == 0) return 8 * tau + e;
  if (P == 1) return (l & 7) | (e << 3) | ((l >> 3) << 6) | (w << 8);
  return (l & 15) | (w << 4) | (e << 6) | ((l >> 4) << 9);
}

__host__ __device__ constexpr int e_low(int pr, int SB) { return ((pr >> SB) << (SB + 1)) | (pr & ((1 << SB) - 1)); }

// exchange-buffer address p + 4 floor(p / 32) + 16 floor(p / 512) = base + offset(e)
__device__ __forceinline__ int xbase(int P, int tau) {
  const int l = tau & 31, w = tau >> 5;
  if (P == 0) return 8 * tau + 4 * (tau >> 2) + 16 * (tau >> 6);
  if (P == 1) return (l & 7) + 72 * (l >> 3) + 288 * w + 16 * (w >> 1);
  return (l & 15) + 16 * w + 4 * (w >> 1) + 592 * (l >> 4);
}
template <int P>
__device__ __forceinline__ constexpr int xoff(int e) {
  return P == 0 ? e : (P == 1 ? 8 * e + 4 * (e >> 2) : 72 * e);
}

// ------------------------------------------------------------------ one register stage
//
// a[i2][k] holds elements (2k, 2k+1) of sub-row i2.  Coefficient block: c[pr] for the
// low end of pair pr, c[4 + pr] for its high end (alpha / beta, or cos / sin).

template <int SB, bool SCALED, int R>
__device__ __forceinline__ void stage(float2 (&a)[R][4], const uint32_t (&c)[8]) {
  if constexpr (SB == 0) {
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const float cl = u2f(c[k]), ch = u2f(c[4 + k]);
#pragma unroll
      for (int r = 0; r < R; ++r) {
        const float lo = a[r][k].x, hi = a[r][k].y;
        if constexpr (SCALED) {
          a[r][k].x = fmaf(cl, hi, lo);
          a[r][k].y = fmaf(ch, lo, hi);
        } else {
          a[r][k].x = fmaf(-ch, hi, cl * lo);
          a[r][k].y = fmaf(cl, hi, ch * lo);
        }
      }
    }
  } else {
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int il = SB == 1 ? 2 * h : h, ih = SB == 1 ? 2 * h + 1 : h + 2;
      const float2 cl = make_float2(u2f(c[2 * h]), u2f(c[2 * h + 1]));
      const float2 ch = make_float2(u2f(c[4 + 2 * h]), u2f(c[5 + 2 * h]));
#pragma unroll
      for (int r = 0; r < R; ++r) {
        const float2 lo = a[r][il], hi = a[r][ih];
        if constexpr (SCALED) {
          a[r][il] = __ffma2_rn(cl, hi, lo);
          a[r][ih] = __ffma2_rn(ch, lo, hi);
        } else {
          a[r][il] = __ffma2_rn(make_float2(-ch.x, -ch.y), hi, __fmul2_rn(cl, lo));
          a[r][ih] = __ffma2_rn(cl, hi, __fmul2_rn(ch, lo));
        }
      }
    }
  }
}

// ------------------------------------------------------------------ inputs
//
// Pass 0 holds elements [8 R tau, 8 R tau + 8 R) of the row: element 8 R tau + j is
// (e, i2) = (j / R, j % R).  They arrive as R (bf16) or 2 R (float32) 16-byte
// vectors, prefetched one row ahead.

template <typename TI, int R>
struct KPre {
  static constexpr int kVec = R * static_cast<int>(sizeof(TI)) / 2;
  uint4 v[kVec];
};

template <typename TI, int R>
__device__ __forceinline__ void kprefetch(KPre<TI, R>& p, const TI* row, int tau) {
  const uint4* s = reinterpret_cast<const uint4*>(row) + KPre<TI, R>::kVec * tau;
#pragma unroll
  for (int q = 0; q < KPre<TI, R>::kVec; ++q) p.v[q] = s[q];
}

template <typename TI, int R>
__device__ __forceinline__ void kunpack(const KPre<TI, R>& p, float2 (&a)[R][4]) {
  const uint32_t* w = reinterpret_cast<const uint32_t*>(p.v);
#pragma unroll
  for (int j = 0; j < 8 * R; ++j) {
    const int e = j / R, i2 = j % R;
    float v;
    if constexpr (sizeof(TI) == 4) {
      v = __uint_as_float(w[j]);
    } else {
      v = (j & 1) ? __uint_as_float(w[j >> 1] & 0xffff0000u) : __uint_as_float(w[j >> 1] << 16);
    }
    if (e & 1) a[i2][e >> 1].y = v;
    else a[i2][e >> 1].x = v;
  }
}

// ------------------------------------------------------------------ kernel
//
// Tensor-memory columns of a thread: 8 s (s < 9) the block of register stage s,
// 72 + e and 80 + e the stage-9 coefficients (k1, k2) of element e:
//   scaled: y = (x + k2 x') k1 with k1 = sigma, k2 = alpha (low end) or beta (high)
//   plain:  y = k1 x + k2 x'  with k1 = cos, k2 = -sin (low end) or sin (high)
// where x' is the partner element in lane l ^ 16.

template <typename TI, int MODE, int BITS, int R>
__global__ void __launch_bounds__(kT, 4) k_kron1024(const KronArgs A) {
  constexpr int N = M1 * R;
  constexpr float kQmax = static_cast<float>((1 << BITS) - 1);
  extern __shared__ __align__(16) float smem[];
  __shared__ uint32_t s_tmem;
  // one exchange buffer serves pass 0 -> 1 and pass 1 -> 2: warp w only touches
  // positions with i1 bits 8, 9 = w until the pass 1 -> 2 barrier
  float* bufA = smem;                  // [R][kPlane]
  float* bufB = bufA;
  float* nat = bufA + R * kPlane;      // [N + 16]: the row in element order
  float2* red = reinterpret_cast<float2*>(nat + N + 16);  // [kRed] chunk (min, max), transposed
  float4* par = reinterpret_cast<float4*>(red + kRed);    // [N / 64] group parameters
  const int tau = threadIdx.x, l = tau & 31, w = tau >> 5;
  const bool scaled = A.hdr[0] == 1.f;

  if (w == 0) {
    const uint32_t dst = static_cast<uint32_t>(__cvta_generic_to_shared(&s_tmem));
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], 128;" ::"r"(dst) : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  cta_sync();
  const uint32_t tb = s_tmem + (static_cast<uint32_t>(32 * w) << 16);
  {
    // this thread's coefficients into its lane
#pragma unroll 1
    for (int s = 0; s < 9; ++s) {
      const int P = s / 3, SB = s % 3;
      uint32_t c[8];
#pragma unroll
      for (int pr = 0; pr < 4; ++pr) {
        const int elo = e_low(pr, SB);
        const int ilo = pos_pass(P, tau, elo), ihi = pos_pass(P, tau, elo | (1 << SB));
        if (scaled) {
          c[pr] = __float_as_uint(A.fast[s * M1 + ilo]);
          c[4 + pr] = __float_as_uint(A.fast[s * M1 + ihi]);
        } else {
          const float2 t = A.cs[s * (M1 / 2) + (((ilo >> (s + 1)) << s) | (ilo & ((1 << s) - 1)))];
          c[pr] = __float_as_uint(t.x);
          c[4 + pr] = __float_as_uint(t.y);
        }
      }
      tst8(tb + 8 * s, c);
    }
    uint32_t k1[8], k2[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      const int i1 = pos_pass(2, tau, e);
      const bool low = ((i1 >> 9) & 1) == 0;
      if (scaled) {
        k1[e] = __float_as_uint(A.sigma[i1]);
        k2[e] = __float_as_uint(A.fast[9 * M1 + i1]);
      } else {
        const float2 t = A.cs[9 * (M1 / 2) + (i1 & 511)];
        k1[e] = __float_as_uint(t.x);
        k2[e] = __float_as_uint(low ? -t.y : t.y);
      }
    }
    tst8(tb + 72, k1);
    tst8(tb + 80, k2);
    asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
  }
  cta_sync();

  float o[R][R];
#pragma unroll
  for (int r = 0; r < R; ++r)
#pragma unroll
    for (int q = 0; q < R; ++q) o[r][q] = A.O[r * R + q];

  const int b0 = xbase(0, tau), b1 = xbase(1, tau), b2 = xbase(2, tau);
  const int nb = pos_pass(2, tau, 0) * R + 16 * (l >> 4);  // element-order address of (e, i2) = (0, 0)
  const int hsw = (tau >> 2) & 1;                          // chunk-half order of the element-order reads
  const TI* X = static_cast<const TI*>(A.x);

  KPre<TI, R> pre;
  if (blockIdx.x < A.rows) kprefetch<TI, R>(pre, X + static_cast<long long>(blockIdx.x) * N, tau);
  uint32_t ca[8], cn[8];
  tld8(tb, ca);
  twait(ca);

#pragma unroll 1
  for (long long row = blockIdx.x; row < A.rows; row += gridDim.x) {
    float2 a[R][4];
    kunpack<TI, R>(pre, a);
    if (row + gridDim.x < A.rows) kprefetch<TI, R>(pre, X + (row + gridDim.x) * N, tau);

    // O_R on every contiguous group of R (per i1), two i1 values per packed op
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      float2 in[R];
#pragma unroll
      for (int q = 0; q < R; ++q) in[q] = a[q][k];
#pragma unroll
      for (int r = 0; r < R; ++r) {
        float2 acc = __fmul2_rn(make_float2(o[r][0], o[r][0]), in[0]);
#pragma unroll
        for (int q = 1; q < R; ++q) acc = __ffma2_rn(make_float2(o[r][q], o[r][q]), in[q], acc);
        a[r][k] = acc;
      }
    }

    // stages 0..8 in registers, the block of stage s + 1 streaming in meanwhile
#define KSTEP(S, SB, CUR, NXT) \
  tld8(tb + 8 * ((S) + 1), NXT); \
  if (scaled) stage<SB, true, R>(a, CUR); else stage<SB, false, R>(a, CUR); \
  twait(NXT)
    KSTEP(0, 0, ca, cn); KSTEP(1, 1, cn, ca); KSTEP(2, 2, ca, cn);
#pragma unroll
    for (int r = 0; r < R; ++r) {
      float* p = bufA + r * kPlane + b0;
      *reinterpret_cast<float4*>(p) = make_float4(a[r][0].x, a[r][0].y, a[r][1].x, a[r][1].y);
      *reinterpret_cast<float4*>(p + 4) = make_float4(a[r][2].x, a[r][2].y, a[r][3].x, a[r][3].y);
    }
    __syncwarp();
#pragma unroll
    for (int r = 0; r < R; ++r)
#pragma unroll
      for (int k = 0; k < 4; ++k)
        a[r][k] = make_float2(bufA[r * kPlane + b1 + xoff<1>(2 * k)], bufA[r * kPlane + b1 + xoff<1>(2 * k + 1)]);
    KSTEP(3, 0, cn, ca); KSTEP(4, 1, ca, cn); KSTEP(5, 2, cn, ca);
    __syncwarp();  // every lane's pass-1 reads precede the writes into the same region
#pragma unroll
    for (int r = 0; r < R; ++r)
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        bufB[r * kPlane + b1 + xoff<1>(2 * k)] = a[r][k].x;
        bufB[r * kPlane + b1 + xoff<1>(2 * k + 1)] = a[r][k].y;
      }
    __syncthreads();
#pragma unroll
    for (int r = 0; r < R; ++r)
#pragma unroll
      for (int k = 0; k < 4; ++k)
        a[r][k] = make_float2(bufB[r * kPlane + b2 + xoff<2>(2 * k)], bufB[r * kPlane + b2 + xoff<2>(2 * k + 1)]);
    KSTEP(6, 0, ca, cn); KSTEP(7, 1, cn, ca);
    tld8(tb + 72, cn);
    if (scaled) stage<2, true, R>(a, ca); else stage<2, false, R>(a, ca);
    tld8(tb + 80, ca);
    twait(cn);  // one wait covers both loads; each array is passed through one
    twait(ca);
#undef KSTEP

    // stage 9 across lanes l and l ^ 16 (sigma folded in), then the row in element order
#pragma unroll
    for (int k = 0; k < 4; ++k)
#pragma unroll
      for (int r = 0; r < R; ++r) {
        const float x0 = a[r][k].x, x1 = a[r][k].y;
        const float p0 = __shfl_xor_sync(0xffffffffu, x0, 16), p1 = __shfl_xor_sync(0xffffffffu, x1, 16);
        const float k10 = u2f(cn[2 * k]), k11 = u2f(cn[2 * k + 1]);
        const float k20 = u2f(ca[2 * k]), k21 = u2f(ca[2 * k + 1]);
        float y0, y1;
        if (scaled) {
          y0 = fmaf(k20, p0, x0) * k10;
          y1 = fmaf(k21, p1, x1) * k11;
        } else {
          y0 = fmaf(k20, p0, k10 * x0);
          y1 = fmaf(k21, p1, k11 * x1);
        }
        nat[nb + 64 * R * (2 * k) + r] = y0;
        nat[nb + 64 * R * (2 * k + 1) + r] = y1;
      }
    tld8(tb, ca);  // block 0 for the next row
    __syncthreads();

    // chunks c = tau + 128 q (q < R) of 8 consecutive elements
    float2 yv[R][4];
#pragma unroll
    for (int q = 0; q < R; ++q) {
      const int c = tau + kT * q;
      const float* src = nat + 8 * c + (8 * c >= 512 * R ? 16 : 0);
      const float4 u = *reinterpret_cast<const float4*>(src + 4 * hsw);
      const float4 v = *reinterpret_cast<const float4*>(src + 4 * (hsw ^ 1));
      const float4 lo = hsw ? v : u, hi = hsw ? u : v;
      yv[q][0] = make_float2(lo.x, lo.y);
      yv[q][1] = make_float2(lo.z, lo.w);
      yv[q][2] = make_float2(hi.x, hi.y);
      yv[q][3] = make_float2(hi.z, hi.w);
    }
    if constexpr (MODE == kKF32) {
#pragma unroll
      for (int q = 0; q < R; ++q) {
        float4* d = reinterpret_cast<float4*>(static_cast<float*>(A.y) + row * N + 8 * (tau + kT * q));
        d[0] = make_float4(yv[q][0].x, yv[q][0].y, yv[q][1].x, yv[q][1].y);
        d[1] = make_float4(yv[q][2].x, yv[q][2].y, yv[q][3].x, yv[q][3].y);
      }
    } else if constexpr (MODE == kKBF16) {
#pragma unroll
      for (int q = 0; q < R; ++q) {
        uint4 u;
        __nv_bfloat162 b[4];
#pragma unroll
        for (int k = 0; k < 4; ++k) b[k] = __floats2bfloat162_rn(yv[q][k].x, yv[q][k].y);
        u.x = *reinterpret_cast<uint32_t*>(&b[0]);
        u.y = *reinterpret_cast<uint32_t*>(&b[1]);
        u.z = *reinterpret_cast<uint32_t*>(&b[2]);
        u.w = *reinterpret_cast<uint32_t*>(&b[3]);
        *reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(A.y) + row * N + 8 * (tau + kT * q)) = u;
      }
    } else {
      // per-chunk extremes -> per-group parameters (one thread per group) -> codes
      // chunk c of group g = c / cg, j = c % cg sits at red[j * S + g]: S odd for
      // cg >= 16 and S = 2 (mod 16) for cg = 8 keep both the writes (16 lanes per
      // phase) and the reducers' reads conflict-free
      const int cg = A.group >> 3, G = N / A.group, lcg = 31 - __clz(cg);
      const int S = cg == 8 ? G + 2 : G + 1;
#pragma unroll
      for (int q = 0; q < R; ++q) {
        float mn = fminf(yv[q][0].x, yv[q][0].y), mx = fmaxf(yv[q][0].x, yv[q][0].y);
#pragma unroll
        for (int k = 1; k < 4; ++k) {
          mn = fminf(mn, fminf(yv[q][k].x, yv[q][k].y));
          mx = fmaxf(mx, fmaxf(yv[q][k].x, yv[q][k].y));
        }
        const int c = tau + kT * q;
        red[(c & (cg - 1)) * S + (c >> lcg)] = make_float2(mn, mx);
      }
      __syncthreads();
      if (tau < G) {
        float lo = FLT_MAX, hi = -FLT_MAX;
        for (int j = 0; j < cg; ++j) {
          const float2 t = red[j * S + tau];
          lo = fminf(lo, t.x);
          hi = fmaxf(hi, t.y);
        }
        const RtnParams p = rtn_params(lo, hi, kQmax);
        par[tau] = make_float4(p.inv, p.thr, p.mz, p.s);
        A.scale[row * G + tau] = p.scale16;
        A.zero[row * G + tau] = p.zero16;
      }
      __syncthreads();
#pragma unroll
      for (int q = 0; q < R; ++q) {
        const int c = tau + kT * q;
        const float4 p = par[c >> lcg];
        const uint32_t word = rtn_codes8<BITS>(yv[q], p.x, p.y, p.z, p.w);
        if constexpr (BITS == 4) {
          *reinterpret_cast<uint32_t*>(A.codes + row * (N / 2) + 4 * c) = word;
        } else {
          *reinterpret_cast<uint16_t*>(A.codes + row * (N / 4) + 2 * c) = static_cast<uint16_t>(word);
        }
      }
    }
    twait(ca);
  }

  cta_sync();
  if (w == 0) asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, 128;" ::"r"(s_tmem) : "memory");
}

template <int R>
constexpr int kron_smem_bytes() {
  return static_cast<int>(sizeof(float)) * (R * kPlane + M1 * R + 16 + 2 * kRed + 4 * (M1 * R / 64));
}

template <typename TI, int MODE, int BITS, int R>
bq_status kron_launch(const KronArgs& A, cudaStream_t st) {
  auto kern = k_kron1024<TI, MODE, BITS, R>;
  constexpr int smem = kron_smem_bytes<R>();
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return BQ_ERR_CUDA;
  static std::atomic<int> ready[kMaxDevices];
  if (!once_per_device(ready, dev, [&] {
        return cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) == cudaSuccess;
      }))
    return BQ_ERR_CUDA;
  const int sms = device_sm_count(dev);
  if (sms <= 0) return BQ_ERR_CUDA;
  long long grid = static_cast<long long>(sms) * 4;  // four row CTAs per SM
  if (grid > A.rows) grid = A.rows;
  if (grid < 1) grid = 1;
  kern<<<static_cast<unsigned>(grid), kT, smem, st>>>(A);
  return cudaPeekAtLastError() == cudaSuccess ? BQ_OK : BQ_ERR_CUDA;
}

template <typename TI, int R>
bq_status kron_dispatch(const KronArgs& A, bq_dtype yt, const QuantArgs* q, cudaStream_t st) {
  if (q) return q->bits == 4 ? kron_launch<TI, kKQuant, 4, R>(A, st) : kron_launch<TI, kKQuant, 2, R>(A, st);
  return yt == BQ_F32 ? kron_launch<TI, kKF32, 4, R>(A, st) : kron_launch<TI, kKBF16, 4, R>(A, st);
}


// ------------------------------------------------------------------ inverse
//
// x = (B_1024^T (x) O_R^T) y: the forward's layouts visited backwards.  B^T is the
// butterfly of the transposed rotations with the stages in reverse order, so it has
// a scaled form of its own (the table's fast_inv / sigma_inv, prepared by the same
// sweep over stages 9 .. 0): every stage is then two FMAs per pair, with sigma_inv
// applied after stage 0.  When the table's inverse flag is clear the kernel runs
// the plain cos/sin rotations.  The row is read in element-order chunks into shared
// memory and picked up in pass-2 layout; stage 9 runs across lanes, stages 8..0 in
// registers with the exchanges reversed; O_R^T is applied in pass 0, which stores
// contiguously.
// Tensor-memory columns: 8 s for register stage s, 80 + e the stage-9 coefficient
// k2 of element e (pass-2 layout) and 72 + e either the stage-9 k1 (plain:
// y = k1 x + k2 x', k1 = cos, k2 = +-sin) or, scaled (y = x + k2 x'), sigma_inv of
// pass-0 element e.

template <int SB, int R>
__device__ __forceinline__ void stage_inv(float2 (&a)[R][4], const uint32_t (&c)[8]) {
  if constexpr (SB == 0) {
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const float cl = u2f(c[k]), ch = u2f(c[4 + k]);
#pragma unroll
      for (int r = 0; r < R; ++r) {
        const float lo = a[r][k].x, hi = a[r][k].y;
        a[r][k].x = fmaf(ch, hi, cl * lo);
        a[r][k].y = fmaf(-ch, lo, cl * hi);
      }
    }
  } else {
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int il = SB == 1 ? 2 * h : h, ih = SB == 1 ? 2 * h + 1 : h + 2;
      const float2 cl = make_float2(u2f(c[2 * h]), u2f(c[2 * h + 1]));
      const float2 ch = make_float2(u2f(c[4 + 2 * h]), u2f(c[5 + 2 * h]));
#pragma unroll
      for (int r = 0; r < R; ++r) {
        const float2 lo = a[r][il], hi = a[r][ih];
        a[r][il] = __ffma2_rn(ch, hi, __fmul2_rn(cl, lo));
        a[r][ih] = __ffma2_rn(make_float2(-ch.x, -ch.y), lo, __fmul2_rn(cl, hi));
      }
    }
  }
}

// chunks c = tau + 128 q (q < R) of 8 consecutive elements, one row ahead
template <typename TI, int R>
__device__ __forceinline__ void kprefetch_chunks(KPre<TI, R>& p, const TI* row, int tau) {
  constexpr int kPer = KPre<TI, R>::kVec / R;  // 16-byte vectors per chunk
#pragma unroll
  for (int q = 0; q < R; ++q) {
    const uint4* s = reinterpret_cast<const uint4*>(row + 8 * (tau + kT * q));
#pragma unroll
    for (int i = 0; i < kPer; ++i) p.v[kPer * q + i] = s[i];
  }
}

template <typename TI, int R>
__device__ __forceinline__ void kunpack_chunks(const KPre<TI, R>& p, float2 (&yv)[R][4]) {
  const uint32_t* w = reinterpret_cast<const uint32_t*>(p.v);
#pragma unroll
  for (int q = 0; q < R; ++q)
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      if constexpr (sizeof(TI) == 4) {
        yv[q][k] = make_float2(__uint_as_float(w[8 * q + 2 * k]), __uint_as_float(w[8 * q + 2 * k + 1]));
      } else {
        const uint32_t u = w[4 * q + k];
        yv[q][k] = make_float2(__uint_as_float(u << 16), __uint_as_float(u & 0xffff0000u));
      }
    }
}

template <typename TI, typename TO, int R>
__global__ void __launch_bounds__(kT, 4) k_kron1024_inv(const KronArgs A) {
  constexpr int N = M1 * R;
  extern __shared__ __align__(16) float smem[];
  __shared__ uint32_t s_tmem;
  float* xbuf = smem;              // [R][kPlane]
  float* nat = xbuf + R * kPlane;  // [N + 16]
  const int tau = threadIdx.x, l = tau & 31, w = tau >> 5;
  const bool scaled = A.hdr[3] == 1.f;

  if (w == 0) {
    const uint32_t dst = static_cast<uint32_t>(__cvta_generic_to_shared(&s_tmem));
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], 128;" ::"r"(dst) : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  cta_sync();
  const uint32_t tb = s_tmem + (static_cast<uint32_t>(32 * w) << 16);
  {
#pragma unroll 1
    for (int s = 0; s < 9; ++s) {
      const int P = s / 3, SB = s % 3;
      uint32_t c[8];
#pragma unroll
      for (int pr = 0; pr < 4; ++pr) {
        const int elo = e_low(pr, SB);
        const int ilo = pos_pass(P, tau, elo);
        if (scaled) {
          c[pr] = __float_as_uint(A.fast_inv[s * M1 + ilo]);
          c[4 + pr] = __float_as_uint(A.fast_inv[s * M1 + pos_pass(P, tau, elo | (1 << SB))]);
        } else {
          const float2 t = A.cs[s * (M1 / 2) + (((ilo >> (s + 1)) << s) | (ilo & ((1 << s) - 1)))];
          c[pr] = __float_as_uint(t.x);
          c[4 + pr] = __float_as_uint(t.y);
        }
      }
      tst8(tb + 8 * s, c);
    }
    uint32_t k1[8], k2[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      const int i1 = pos_pass(2, tau, e);
      if (scaled) {
        k1[e] = __float_as_uint(A.sigma_inv[pos_pass(0, tau, e)]);
        k2[e] = __float_as_uint(A.fast_inv[9 * M1 + i1]);
      } else {
        const float2 t = A.cs[9 * (M1 / 2) + (i1 & 511)];
        k1[e] = __float_as_uint(t.x);
        k2[e] = __float_as_uint(((i1 >> 9) & 1) ? -t.y : t.y);
      }
    }
    tst8(tb + 72, k1);
    tst8(tb + 80, k2);
    asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
  }
  cta_sync();

  float o[R][R];
#pragma unroll
  for (int r = 0; r < R; ++r)
#pragma unroll
    for (int q = 0; q < R; ++q) o[r][q] = A.O[r * R + q];

  const int b0 = xbase(0, tau), b1 = xbase(1, tau), b2 = xbase(2, tau);
  const int nb = pos_pass(2, tau, 0) * R + 16 * (l >> 4);
  const int hsw = (tau >> 2) & 1;
  const TI* Y = static_cast<const TI*>(A.x);

  KPre<TI, R> pre;
  if (blockIdx.x < A.rows) kprefetch_chunks<TI, R>(pre, Y + static_cast<long long>(blockIdx.x) * N, tau);
  uint32_t ca[8], cn[8];
  tld8(tb + 72, cn);
  tld8(tb + 80, ca);
  twait(cn);
  twait(ca);

#define KISTEP(S, SB, CUR, NXT) \
  tld8(tb + 8 * ((S) - 1), NXT); \
  if (scaled) stage<SB, true, R>(a, CUR); else stage_inv<SB, R>(a, CUR); \
  twait(NXT)

#pragma unroll 1
  for (long long row = blockIdx.x; row < A.rows; row += gridDim.x) {
    {
      float2 yv[R][4];
      kunpack_chunks<TI, R>(pre, yv);
      if (row + gridDim.x < A.rows) kprefetch_chunks<TI, R>(pre, Y + (row + gridDim.x) * N, tau);
#pragma unroll
      for (int q = 0; q < R; ++q) {
        const int c = tau + kT * q;
        float* dst = nat + 8 * c + (8 * c >= 512 * R ? 16 : 0);
        const float4 lo = make_float4(yv[q][0].x, yv[q][0].y, yv[q][1].x, yv[q][1].y);
        const float4 hi = make_float4(yv[q][2].x, yv[q][2].y, yv[q][3].x, yv[q][3].y);
        *reinterpret_cast<float4*>(dst + 4 * hsw) = hsw ? hi : lo;
        *reinterpret_cast<float4*>(dst + 4 * (hsw ^ 1)) = hsw ? lo : hi;
      }
    }
    __syncthreads();
    float2 a[R][4];
#pragma unroll
    for (int k = 0; k < 4; ++k)
#pragma unroll
      for (int r = 0; r < R; ++r) {
        const float x0 = nat[nb + 64 * R * (2 * k) + r], x1 = nat[nb + 64 * R * (2 * k + 1) + r];
        const float p0 = __shfl_xor_sync(0xffffffffu, x0, 16), p1 = __shfl_xor_sync(0xffffffffu, x1, 16);
        if (scaled)
          a[r][k] = make_float2(fmaf(u2f(ca[2 * k]), p0, x0), fmaf(u2f(ca[2 * k + 1]), p1, x1));
        else
          a[r][k] = make_float2(fmaf(u2f(ca[2 * k]), p0, u2f(cn[2 * k]) * x0),
                                fmaf(u2f(ca[2 * k + 1]), p1, u2f(cn[2 * k + 1]) * x1));
      }
    tld8(tb + 64, ca);
    twait(ca);
    KISTEP(8, 2, ca, cn); KISTEP(7, 1, cn, ca); KISTEP(6, 0, ca, cn);
#pragma unroll
    for (int r = 0; r < R; ++r)
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        xbuf[r * kPlane + b2 + xoff<2>(2 * k)] = a[r][k].x;
        xbuf[r * kPlane + b2 + xoff<2>(2 * k + 1)] = a[r][k].y;
      }
    __syncthreads();
#pragma unroll
    for (int r = 0; r < R; ++r)
#pragma unroll
      for (int k = 0; k < 4; ++k)
        a[r][k] = make_float2(xbuf[r * kPlane + b1 + xoff<1>(2 * k)], xbuf[r * kPlane + b1 + xoff<1>(2 * k + 1)]);
    KISTEP(5, 2, cn, ca); KISTEP(4, 1, ca, cn); KISTEP(3, 0, cn, ca);
    __syncwarp();  // every lane's pass-1 reads precede the writes into the same region
#pragma unroll
    for (int r = 0; r < R; ++r)
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        xbuf[r * kPlane + b1 + xoff<1>(2 * k)] = a[r][k].x;
        xbuf[r * kPlane + b1 + xoff<1>(2 * k + 1)] = a[r][k].y;
      }
    __syncwarp();
#pragma unroll
    for (int r = 0; r < R; ++r) {
      const float4 u = *reinterpret_cast<const float4*>(xbuf + r * kPlane + b0);
      const float4 v = *reinterpret_cast<const float4*>(xbuf + r * kPlane + b0 + 4);
      a[r][0] = make_float2(u.x, u.y);
      a[r][1] = make_float2(u.z, u.w);
      a[r][2] = make_float2(v.x, v.y);
      a[r][3] = make_float2(v.z, v.w);
    }
    KISTEP(2, 2, ca, cn); KISTEP(1, 1, cn, ca);
    tld8(tb + 72, cn);  // sigma_inv (scaled) or stage 9's k1 of the next row (plain)
    if (scaled) {
      stage<0, true, R>(a, ca);
      twait(cn);
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const float2 sg = make_float2(u2f(cn[2 * k]), u2f(cn[2 * k + 1]));
#pragma unroll
        for (int r = 0; r < R; ++r) a[r][k] = __fmul2_rn(a[r][k], sg);
      }
    } else {
      stage_inv<0, R>(a, ca);
    }
    tld8(tb + 80, ca);  // stage 9's k2 of the next row

    // O_R^T on every group of R, then the pass-0 elements (contiguous) to memory
    float2 out[R][4];
#pragma unroll
    for (int k = 0; k < 4; ++k)
#pragma unroll
      for (int r = 0; r < R; ++r) {
        float2 acc = __fmul2_rn(make_float2(o[0][r], o[0][r]), a[0][k]);
#pragma unroll
        for (int q = 1; q < R; ++q) acc = __ffma2_rn(make_float2(o[q][r], o[q][r]), a[q][k], acc);
        out[r][k] = acc;
      }
    // element 8 R tau + j is (e, i2) = (j / R, j % R)
    if constexpr (sizeof(TO) == 4) {
      float* dst = static_cast<float*>(A.y) + row * N + 8 * R * tau;
#pragma unroll
      for (int v = 0; v < 2 * R; ++v) {
        float f[4];
#pragma unroll
        for (int t = 0; t < 4; ++t) {
          const int j = 4 * v + t, e = j / R, r = j % R;
          f[t] = (e & 1) ? out[r][e >> 1].y : out[r][e >> 1].x;
        }
        reinterpret_cast<float4*>(dst)[v] = make_float4(f[0], f[1], f[2], f[3]);
      }
    } else {
      __nv_bfloat16* dst = static_cast<__nv_bfloat16*>(A.y) + row * N + 8 * R * tau;
#pragma unroll
      for (int v = 0; v < R; ++v) {
        uint32_t u[4];
#pragma unroll
        for (int t = 0; t < 4; ++t) {
          const int j0 = 8 * v + 2 * t, j1 = j0 + 1;
          const float f0 = ((j0 / R) & 1) ? out[j0 % R][(j0 / R) >> 1].y : out[j0 % R][(j0 / R) >> 1].x;
          const float f1 = ((j1 / R) & 1) ? out[j1 % R][(j1 / R) >> 1].y : out[j1 % R][(j1 / R) >> 1].x;
          __nv_bfloat162 b = __floats2bfloat162_rn(f0, f1);
          u[t] = *reinterpret_cast<uint32_t*>(&b);
        }
        reinterpret_cast<uint4*>(dst)[v] = make_uint4(u[0], u[1], u[2], u[3]);
      }
    }
    twait(cn);
    twait(ca);
  }
#undef KISTEP

  cta_sync();
  if (w == 0) asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, 128;" ::"r"(s_tmem) : "memory");
}

template <typename TI, typename TO, int R>
bq_status kron_inv_launch(const KronArgs& A, cudaStream_t st) {
  auto kern = k_kron1024_inv<TI, TO, R>;
  constexpr int smem = kron_smem_bytes<R>();
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return BQ_ERR_CUDA;
  static std::atomic<int> ready[kMaxDevices];
  if (!once_per_device(ready, dev, [&] {
        return cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) == cudaSuccess;
      }))
    return BQ_ERR_CUDA;
  const int sms = device_sm_count(dev);
  if (sms <= 0) return BQ_ERR_CUDA;
  long long grid = static_cast<long long>(sms) * 4;
  if (grid > A.rows) grid = A.rows;
  if (grid < 1) grid = 1;
  kern<<<static_cast<unsigned>(grid), kT, smem, st>>>(A);
  return cudaPeekAtLastError() == cudaSuccess ? BQ_OK : BQ_ERR_CUDA;
}

}  // namespace

bool kron1024_supports(const KLayer& L, const QuantArgs* q) {
  if (L.m != M1 || L.r != 5 || L.O == nullptr) return false;
  if (q && q->group != 64 && q->group != 128 && q->group != 256) return false;
  return true;
}

bq_status launch_kron1024(const KLayer& L, const void* x, bq_dtype xt, void* y, bq_dtype yt, int64_t rows,
                          const QuantArgs* q, cudaStream_t st) {
  KronArgs A;
  A.x = x;
  A.y = y;
  A.rows = rows;
  A.fast = L.fast;
  A.sigma = L.sigma;
  A.fast_inv = L.fast_inv;
  A.sigma_inv = L.sigma_inv;
  A.cs = L.cs;
  A.hdr = L.hdr;
  A.O = L.O;
  A.codes = q ? q->codes : nullptr;
  A.scale = q ? q->scale : nullptr;
  A.zero = q ? q->zero : nullptr;
  A.group = q ? q->group : 128;
  return xt == BQ_F32 ? kron_dispatch<float, 5>(A, yt, q, st) : kron_dispatch<__nv_bfloat16, 5>(A, yt, q, st);
}

bq_status launch_kron1024_inv(const KLayer& L, const void* y, bq_dtype yt, void* x, bq_dtype xt, int64_t rows,
                              cudaStream_t st) {
  KronArgs A;
  A.x = y;  // the kernel reads A.x and writes A.y
  A.y = x;
  A.rows = rows;
  A.fast = L.fast;
  A.sigma = L.sigma;
  A.fast_inv = L.fast_inv;
  A.sigma_inv = L.sigma_inv;
  A.cs = L.cs;
  A.hdr = L.hdr;
  A.O = L.O;
  A.codes = nullptr;
  A.scale = nullptr;
  A.zero = nullptr;
  A.group = 128;
  if (yt == BQ_F32)
    return xt == BQ_F32 ? kron_inv_launch<float, float, 5>(A, st) : kron_inv_launch<float, __nv_bfloat16, 5>(A, st);
  return xt == BQ_F32 ? kron_inv_launch<__nv_bfloat16, float, 5>(A, st)
                      : kron_inv_launch<__nv_bfloat16, __nv_bfloat16, 5>(A, st);
}

}  // namespace bq
