// Specialised n = 4096 butterfly kernel (m = 4096, r = 1): forward transform
// with float32 / bfloat16 output, or fused with per-group asymmetric RTN and
// INT2 / INT4 packing.  This is the hot path of the activation side Q x and the
// weight side W Q^T (ButterflyQuant abstract: y = W x = (W Q^T)(Q x)).
//
// Design (B200, sm_100a):
//  * Coefficients live in tensor memory.  The 12 stages need 192 KB of
//    per-pair coefficients per layer, more than shared memory can spare next
//    to the row buffers, and streaming them from L1/shared memory for every
//    row would cost ~384 shared-memory wavefronts per row.  Each SM therefore
//    copies the layer's 208 KB tensor-memory image (built once per layer by
//    bq_precompute_cs) into its 128 TMEM lanes x 416 columns at start-up, and
//    every thread reads its own lane with tcgen05.ld, a path separate from
//    shared memory.
//  * 128 threads (one warpgroup, thread t <-> TMEM lane t) own a row at a
//    time; each thread holds 32 of its elements.  The 12 stages run in
//    three passes with the in-register index bits
//        pass A: position bits {0..4}    stages 0..4
//        pass B: position bits {5..9}    stages 5..9
//        pass C: position bits {0,1,2,10,11}  stages 10, 11
//    and two swizzled shared-memory transposes between them (conflict-free:
//    one side uses 16-byte vectors, the other 4-byte scalars).  The A -> B
//    exchange stays inside each warp (bits 10, 11 are the warp index of both
//    layouts); only B -> C needs the row group's barrier.  Pass C's
//    layout keeps 8 consecutive positions per thread, so the RTN epilogue
//    (group statistics, packing, coalesced stores) runs in place without a
//    third transpose.
//  * Rotations use the scaled two-FMA form prepared by bq_precompute_cs
//    (a_i += alpha a_j, a_j += beta a_i; outputs times sigma), issued as packed
//    fma.rn.f32x2 where two pairs sit in adjacent registers; when the layer's
//    scaled form is out of range (table header flag 0) the same kernel runs the
//    plain cos/sin rotation instead.
//  * One CTA per SM (all 512 TMEM columns), three row groups per CTA sharing
//    the tensor-memory image (warps w, w+4, w+8 use the same lanes) for
//    latency hiding; the next row's input is prefetched into registers while
//    the current row is processed.
#include <cfloat>

#include "bq_rtn.cuh"

namespace bq {
namespace {

constexpr int M = 4096;
constexpr int kGroupThreads = 128;
constexpr int kSlots = 3;
constexpr int kThreads = kSlots * kGroupThreads;
constexpr int kColB = 160, kColC = 320, kColS = 384;
constexpr int kFillChunks = kImageCols / 16;  // 26 chunks of 16 columns, dealt round-robin to the slots

enum Mode { kOutF32 = 0, kOutBF16 = 1, kQuant = 2 };

// ------------------------------------------------------------------ tensor memory

__device__ __forceinline__ void tmem_ld32(uint32_t addr, uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
        "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
        "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(addr));
}

// Waits for this thread's outstanding tensor-memory loads; the registers are
// passed through so that no use of them can be scheduled before the wait.
__device__ __forceinline__ void tmem_wait(uint32_t (&r)[32]) {
  asm volatile("tcgen05.wait::ld.sync.aligned;"
               : "+r"(r[0]), "+r"(r[1]), "+r"(r[2]), "+r"(r[3]), "+r"(r[4]), "+r"(r[5]), "+r"(r[6]), "+r"(r[7]),
                 "+r"(r[8]), "+r"(r[9]), "+r"(r[10]), "+r"(r[11]), "+r"(r[12]), "+r"(r[13]), "+r"(r[14]),
                 "+r"(r[15]), "+r"(r[16]), "+r"(r[17]), "+r"(r[18]), "+r"(r[19]), "+r"(r[20]), "+r"(r[21]),
                 "+r"(r[22]), "+r"(r[23]), "+r"(r[24]), "+r"(r[25]), "+r"(r[26]), "+r"(r[27]), "+r"(r[28]),
                 "+r"(r[29]), "+r"(r[30]), "+r"(r[31])
               :
               : "memory");
}

__device__ __forceinline__ void tmem_st16(uint32_t addr, const uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], "
      "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" ::"r"(addr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]),
      "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15])
      : "memory");
}

__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

__device__ __forceinline__ void group_sync(int slot) {
  asm volatile("bar.sync %0, %1;" ::"r"(1 + slot), "r"(kGroupThreads) : "memory");
}

__device__ __forceinline__ float u2f(uint32_t v) { return __uint_as_float(v); }

// ------------------------------------------------------------------ one stage in registers
//
// a[r][q] holds register slots (2q, 2q+1) of row r.  For in-register bit SB the
// thread's 16 pairs are (j_k, j_k | 2^SB), j_k = ((k >> SB) << (SB+1)) | (k & (2^SB-1)),
// and coefficient column 4q + e belongs to the low element of pair 2q + e,
// column 4q + 2 + e to its high element.

template <int SB>
__host__ __device__ constexpr int low_slot(int k) {
  return ((k >> SB) << (SB + 1)) | (k & ((1 << SB) - 1));
}

template <int SB, bool SCALED, int R>
__device__ __forceinline__ void stage(float2 (&a)[2][16], const uint32_t (&c)[32]) {
  if constexpr (SB == 0) {
    // pairs (2k, 2k+1) sit inside one float2: scalar FMAs
#pragma unroll
    for (int q = 0; q < 8; ++q) {
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const int k = 2 * q + e;
        const float cl = u2f(c[4 * q + e]), ch = u2f(c[4 * q + 2 + e]);
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
    }
  } else {
#pragma unroll
    for (int q = 0; q < 8; ++q) {
      constexpr int kHalf = 1 << (SB - 1);  // float2 distance between a low slot and its partner
      const int lq = low_slot<SB>(2 * q) >> 1;
      const int hq = lq + kHalf;
      const float2 cl = make_float2(u2f(c[4 * q]), u2f(c[4 * q + 1]));
      const float2 ch = make_float2(u2f(c[4 * q + 2]), u2f(c[4 * q + 3]));
#pragma unroll
      for (int r = 0; r < R; ++r) {
        const float2 lo = a[r][lq], hi = a[r][hq];
        if constexpr (SCALED) {
          a[r][lq] = __ffma2_rn(cl, hi, lo);
          a[r][hq] = __ffma2_rn(ch, lo, hi);
        } else {
          const float2 nch = make_float2(-ch.x, -ch.y);
          a[r][lq] = __ffma2_rn(nch, hi, __fmul2_rn(cl, lo));
          a[r][hq] = __ffma2_rn(cl, hi, __fmul2_rn(ch, lo));
        }
      }
    }
  }
}

// Computes one stage from the coefficient block in `cur` while the block at
// `next_addr` streams into `nxt`; returns after `nxt` has arrived.
template <int SB, bool SCALED, int R>
__device__ __forceinline__ void stage_step(float2 (&a)[2][16], uint32_t (&cur)[32], uint32_t (&nxt)[32],
                                           uint32_t next_addr) {
  tmem_ld32(next_addr, nxt);
  stage<SB, SCALED, R>(a, cur);
  tmem_wait(nxt);
}

// ------------------------------------------------------------------ inputs

template <typename TI>
struct Prefetch;
template <>
struct Prefetch<__nv_bfloat16> {
  static constexpr int kVec = 4;  // 16-byte vectors per row per thread (32 bf16)
  uint4 v[2][kVec];
};
template <>
struct Prefetch<float> {
  static constexpr int kVec = 8;
  uint4 v[2][kVec];
};

template <typename TI>
__device__ __forceinline__ void prefetch(Prefetch<TI>& p, const TI* x, long long row, int cnt, int tau) {
#pragma unroll
  for (int r = 0; r < 2; ++r) {
    if (r < cnt) {
      const uint4* src = reinterpret_cast<const uint4*>(x + (row + r) * M + tau * 32);
#pragma unroll
      for (int i = 0; i < Prefetch<TI>::kVec; ++i) p.v[r][i] = src[i];
    }
  }
}

template <int R>
__device__ __forceinline__ void unpack_input(const Prefetch<__nv_bfloat16>& p, float2 (&a)[2][16]) {
#pragma unroll
  for (int r = 0; r < R; ++r)
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const uint32_t w[4] = {p.v[r][i].x, p.v[r][i].y, p.v[r][i].z, p.v[r][i].w};
#pragma unroll
      for (int k = 0; k < 4; ++k)
        a[r][4 * i + k] = make_float2(__uint_as_float(w[k] << 16), __uint_as_float(w[k] & 0xffff0000u));
    }
}

template <int R>
__device__ __forceinline__ void unpack_input(const Prefetch<float>& p, float2 (&a)[2][16]) {
#pragma unroll
  for (int r = 0; r < R; ++r)
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      a[r][2 * i] = make_float2(__uint_as_float(p.v[r][i].x), __uint_as_float(p.v[r][i].y));
      a[r][2 * i + 1] = make_float2(__uint_as_float(p.v[r][i].z), __uint_as_float(p.v[r][i].w));
    }
}

// ------------------------------------------------------------------ kernel

struct FastArgs {
  const void* x;
  void* y;
  long long rows;
  const float* image;
  const float* hdr;
  uint8_t* codes;
  uint16_t* scale;
  uint16_t* zero;
};

template <int N>
__host__ __device__ constexpr int clog2(int v) {
  return v <= 1 ? 0 : 1 + clog2<N>(v / 2);
}

template <int S>
__device__ __forceinline__ int bitrev(int k) {
  int r = 0;
#pragma unroll
  for (int i = 0; i < clog2<0>(S); ++i) r |= ((k >> i) & 1) << (clog2<0>(S) - 1 - i);
  return r;
}

__device__ __forceinline__ float min3(float a, float b, float c) {
  float d;
  asm("min.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}
__device__ __forceinline__ float max3(float a, float b, float c) {
  float d;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}

// Per-group asymmetric RTN of the R rows held in pass-C layout, packing and stores.
//
// Group extremes: 3-input min / max over each 8-value set, then a recursive-halving
// shuffle reduction after which lane l holds set bitrev(l & (S-1)) of its group.
// Every lane computes that group's parameters (scale16, s, z, 1 / s and the tie
// threshold, as in rtn_params); each set then takes them by shuffle from the lane
// that holds them and is coded by rtn_codes8 (exact RTN: see bq_rtn.cuh).  One
// reducing warp per row group with the parameters in shared memory issues fewer
// instructions but adds two row-group barriers, and measured slower at 2048 rows.
template <int BITS, int GLANES, int R>
__device__ __forceinline__ void quant_epilogue(const float2 (&a)[2][16], const FastArgs& A, long long row0, int tau,
                                               int lane) {
  constexpr int S = 4 * R;               // (row, hi2) sets per thread
  constexpr int LOGS = clog2<0>(S);
  constexpr int LOGG = clog2<0>(GLANES);  // lanes sharing one group
  constexpr int GROUP = 8 * GLANES;
  constexpr int GPR = M / GROUP;          // groups per row
  constexpr int QMAX = (1 << BITS) - 1;
  const float qmax = static_cast<float>(QMAX);
  float mn[S], mx[S];
#pragma unroll
  for (int k = 0; k < S; ++k) {
    const int r = k >> 2, h = k & 3;
    const float2 p0 = a[r][4 * h], p1 = a[r][4 * h + 1], p2 = a[r][4 * h + 2], p3 = a[r][4 * h + 3];
    mn[k] = fminf(min3(p0.x, p0.y, p1.x), min3(p1.y, p2.x, min3(p2.y, p3.x, p3.y)));
    mx[k] = fmaxf(max3(p0.x, p0.y, p1.x), max3(p1.y, p2.x, max3(p2.y, p3.x, p3.y)));
  }
  // recursive halving over lane bits 0..LOGS-1: afterwards lane l holds set bitrev(l & (S-1))
#pragma unroll
  for (int i = 0; i < LOGS; ++i) {
    const int half = (S >> i) >> 1;
    const bool up = (lane >> i) & 1;
#pragma unroll
    for (int k = 0; k < half; ++k) {
      const float smn = up ? mn[k] : mn[k + half], kmn = up ? mn[k + half] : mn[k];
      const float smx = up ? mx[k] : mx[k + half], kmx = up ? mx[k + half] : mx[k];
      mn[k] = fminf(kmn, __shfl_xor_sync(0xffffffffu, smn, 1 << i));
      mx[k] = fmaxf(kmx, __shfl_xor_sync(0xffffffffu, smx, 1 << i));
    }
  }
#pragma unroll
  for (int i = LOGS; i < LOGG; ++i) {
    mn[0] = fminf(mn[0], __shfl_xor_sync(0xffffffffu, mn[0], 1 << i));
    mx[0] = fmaxf(mx[0], __shfl_xor_sync(0xffffffffu, mx[0], 1 << i));
  }
  const float lo = mn[0], hi = mx[0];
  __half h16 = __float2half_rn(__fdiv_rn(__fsub_rn(hi, lo), qmax));
  float s = __half2float(h16);
  if (hi == lo || s == 0.f) {
    s = 1.f;
    h16 = __float2half_rn(1.f);
  }
  const float zraw = rintf(__fdiv_rn(-lo, s));
  const float z = __fadd_rn(fminf(fmaxf(zraw, 0.f), qmax), 0.f);  // +0 for a zero point of 0
  const float inv = __fdiv_rn(1.f, s);
  // tie margin for the whole group: every |v| <= max(|lo|, |hi|) * inv * (1 + 2^-20)
  const float vmax = fmaxf(fabsf(lo), fabsf(hi)) * inv * 1.000001f;
  const float thr = vmax < 4194304.f ? 0.5f - vmax * 9.5367431640625e-7f : -1.f;  // 2^22, 2^-20
  // codes are monotone in y: when the group's extremes quantize inside [0, qmax],
  // no element needs clamping.  Division and rint are both odd functions, so the
  // code of lo is z - rint(-lo/s) exactly: in range at the bottom iff
  // rint(-lo/s) <= qmax.  The top is checked with one IEEE division.
  const bool inrange = zraw <= qmax && __fadd_rn(rintf(__fdiv_rn(hi, s)), z) <= qmax;
  const float thr_in = inrange ? thr : -1.f;  // -1 sends the whole set to the slow path
  {
    const int k = bitrev<S>(lane & (S - 1));
    if (((lane >> LOGS) & ((1 << (LOGG - LOGS)) - 1)) == 0) {
      const long long row = row0 + (k >> 2);
      const int g = (k & 3) * (1024 / GROUP) + (tau >> LOGG);
      A.scale[row * GPR + g] = __half_as_ushort(h16);
      A.zero[row * GPR + g] = __half_as_ushort(__float2half_rn(z));
    }
  }
  // codes of each set with its group's parameters (from the lane that reduced it)
  const float mz = __fadd_rn(12582912.f, z);
#pragma unroll
  for (int k = 0; k < S; ++k) {
    const int src = (lane & ~(S - 1)) | bitrev<S>(k);
    const float invk = __shfl_sync(0xffffffffu, inv, src);
    const float thrk = __shfl_sync(0xffffffffu, thr_in, src);
    const float mzk = __shfl_sync(0xffffffffu, mz, src);
    const float sk = __shfl_sync(0xffffffffu, s, src);
    const int r = k >> 2, h = k & 3;
    const float2 y[4] = {a[r][4 * h], a[r][4 * h + 1], a[r][4 * h + 2], a[r][4 * h + 3]};
    const uint32_t word = rtn_codes8<BITS>(y, invk, thrk, mzk, sk);
    const long long row = row0 + r;
    if constexpr (BITS == 4) {
      *reinterpret_cast<uint32_t*>(A.codes + row * (M / 2) + h * 512 + tau * 4) = word;
    } else {
      *reinterpret_cast<uint16_t*>(A.codes + row * (M / 4) + h * 256 + tau * 2) = static_cast<uint16_t>(word);
    }
  }
}

template <int MODE, int R>
__device__ __forceinline__ void store_epilogue(const float2 (&a)[2][16], const FastArgs& A, long long row0, int tau) {
#pragma unroll
  for (int r = 0; r < R; ++r)
#pragma unroll
    for (int h = 0; h < 4; ++h) {
      const long long off = (row0 + r) * M + h * 1024 + tau * 8;
      if constexpr (MODE == kOutF32) {
        float4* dst = reinterpret_cast<float4*>(static_cast<float*>(A.y) + off);
        dst[0] = make_float4(a[r][4 * h].x, a[r][4 * h].y, a[r][4 * h + 1].x, a[r][4 * h + 1].y);
        dst[1] = make_float4(a[r][4 * h + 2].x, a[r][4 * h + 2].y, a[r][4 * h + 3].x, a[r][4 * h + 3].y);
      } else {
        uint4 w;
        __nv_bfloat162 b0 = __floats2bfloat162_rn(a[r][4 * h].x, a[r][4 * h].y);
        __nv_bfloat162 b1 = __floats2bfloat162_rn(a[r][4 * h + 1].x, a[r][4 * h + 1].y);
        __nv_bfloat162 b2 = __floats2bfloat162_rn(a[r][4 * h + 2].x, a[r][4 * h + 2].y);
        __nv_bfloat162 b3 = __floats2bfloat162_rn(a[r][4 * h + 3].x, a[r][4 * h + 3].y);
        w.x = *reinterpret_cast<uint32_t*>(&b0);
        w.y = *reinterpret_cast<uint32_t*>(&b1);
        w.z = *reinterpret_cast<uint32_t*>(&b2);
        w.w = *reinterpret_cast<uint32_t*>(&b3);
        *reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(A.y) + off) = w;
      }
    }
}

// One group of R rows through all twelve stages and the epilogue.  On entry
// c0 holds coefficient block 0 (waited for) and `pre` holds the rows' input;
// on return c0 again holds block 0 and `pre` holds the next rows' input.
template <typename TI, int MODE, int BITS, int GLANES, bool SCALED, int R>
__device__ __forceinline__ void process(const FastArgs& A, long long row0, long long nrow, int ncnt, int slot,
                                        int tau, int lane, uint32_t tb, float* bufAB, float* bufBC,
                                        Prefetch<TI>& pre, uint32_t (&c0)[32], uint32_t (&c1)[32]) {
  float2 a[2][16];
  unpack_input<R>(pre, a);
  prefetch(pre, static_cast<const TI*>(A.x), nrow, ncnt, tau);

  // pass A: stages 0..4 on position bits 0..4
  stage_step<0, SCALED, R>(a, c0, c1, tb + 32);
  stage_step<1, SCALED, R>(a, c1, c0, tb + 64);
  stage_step<2, SCALED, R>(a, c0, c1, tb + 96);
  stage_step<3, SCALED, R>(a, c1, c0, tb + 128);
  stage_step<4, SCALED, R>(a, c0, c1, tb + kColB);
#pragma unroll
  for (int r = 0; r < R; ++r)
#pragma unroll
    for (int c = 0; c < 8; ++c)
      *reinterpret_cast<float4*>(bufAB + r * M + tau * 32 + 4 * (c ^ (tau & 7))) =
          make_float4(a[r][2 * c].x, a[r][2 * c].y, a[r][2 * c + 1].x, a[r][2 * c + 1].y);
  // pass-A thread t writes row t (positions 32t..32t+31); pass-B thread t reads rows
  // 32(t >> 5) .. 32(t >> 5) + 31: position bits 10, 11 are the warp index in both
  // layouts, so this exchange stays inside the warp
  __syncwarp();
  {
    const int base = ((tau >> 5) << 10) + (tau & 3), cq = (tau & 31) >> 2;
#pragma unroll
    for (int r = 0; r < R; ++r)
#pragma unroll
      for (int rb = 0; rb < 32; rb += 2) {
        const float v0 = bufAB[r * M + base + 32 * rb + 4 * (cq ^ (rb & 7))];
        const float v1 = bufAB[r * M + base + 32 * (rb + 1) + 4 * (cq ^ ((rb + 1) & 7))];
        a[r][rb >> 1] = make_float2(v0, v1);
      }
  }
  // pass B: stages 5..9 on position bits 5..9
  stage_step<0, SCALED, R>(a, c1, c0, tb + kColB + 32);
  stage_step<1, SCALED, R>(a, c0, c1, tb + kColB + 64);
  stage_step<2, SCALED, R>(a, c1, c0, tb + kColB + 96);
  stage_step<3, SCALED, R>(a, c0, c1, tb + kColB + 128);
  stage_step<4, SCALED, R>(a, c1, c0, tb + kColC);
  {
    const int base = (tau >> 5) * 1024 + ((tau & 31) >> 3) * 8 + (tau & 3), sw = (tau >> 2) & 1;
#pragma unroll
    for (int r = 0; r < R; ++r)
#pragma unroll
      for (int rb = 0; rb < 32; rb += 2) {
        bufBC[r * M + base + 32 * rb + 4 * (sw ^ 0)] = a[r][rb >> 1].x;
        bufBC[r * M + base + 32 * (rb + 1) + 4 * (sw ^ 1)] = a[r][rb >> 1].y;
      }
  }
  group_sync(slot);
  {
    const int sw = (tau >> 2) & 1;
#pragma unroll
    for (int r = 0; r < R; ++r)
#pragma unroll
      for (int h = 0; h < 4; ++h)
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
          const float4 v = *reinterpret_cast<const float4*>(bufBC + r * M + h * 1024 + tau * 8 + 4 * (hh ^ sw));
          a[r][4 * h + 2 * hh] = make_float2(v.x, v.y);
          a[r][4 * h + 2 * hh + 1] = make_float2(v.z, v.w);
        }
  }
  // pass C: stages 10, 11 on slot bits 3, 4 (position bits 10, 11)
  stage_step<3, SCALED, R>(a, c0, c1, tb + kColC + 32);
  stage_step<4, SCALED, R>(a, c1, c0, tb + kColS);
  // output scale (1 for the plain rotation), then start loading the next group's block 0
#pragma unroll
  for (int r = 0; r < R; ++r)
#pragma unroll
    for (int q = 0; q < 16; ++q) a[r][q] = __fmul2_rn(a[r][q], make_float2(u2f(c0[2 * q]), u2f(c0[2 * q + 1])));
  tmem_ld32(tb, c0);
  if constexpr (MODE == kQuant) {
    quant_epilogue<BITS, GLANES, R>(a, A, row0, tau, lane);
  } else {
    store_epilogue<MODE, R>(a, A, row0, tau);
  }
  tmem_wait(c0);
}

template <typename TI, int MODE, int BITS, int GLANES, bool SCALED>
__device__ __forceinline__ void run_rows(const FastArgs& A, long long rb, long long re, int slot, int tau, int lane,
                                         uint32_t tb, float* bufAB, float* bufBC, Prefetch<TI>& pre,
                                         uint32_t (&c0)[32], uint32_t (&c1)[32]) {
  // the B -> C buffer alternates between rows: with only a warp-level sync before
  // the next row's B -> C writes, row i's readers and row i+2's writers are kept
  // apart by row i+1's row-group barrier
#pragma unroll 1
  for (long long row = rb; row < re; ++row)
    process<TI, MODE, BITS, GLANES, SCALED, 1>(A, row, row + 1, row + 1 < re ? 1 : 0, slot, tau, lane, tb, bufAB,
                                               bufBC + ((row - rb) & 1) * M, pre, c0, c1);
}

// Copies this thread's share of a tensor-memory image (NCHUNK chunks of 16
// columns, dealt round-robin to the slots) into its lane: all loads in flight
// first (each warp load is one contiguous 512-byte run of the [column/4][lane]
// image), then the stores.  Every CTA reads the same image at the same moment,
// so each starts at a different chunk (block index mod NCHUNK): the requests in
// flight then spread over the L2 slices instead of queueing on the same few.
// (Sharing one L2 read per CTA pair through distributed shared memory was
// slower: gathering 208 KB per SM that way costs more than the L2 reads saved.)
template <int NCHUNK>
__device__ __forceinline__ void fill_tmem(const float* image, uint32_t tb, int slot, int tau) {
  const float4* src = reinterpret_cast<const float4*>(image) + tau;  // block q of lane tau at [q * 128]
  constexpr int kMine = (NCHUNK + kSlots - 1) / kSlots;
  float4 f[kMine * 4];
  const int rot = blockIdx.x % NCHUNK;
#pragma unroll
  for (int i = 0; i < kMine; ++i) {
    const int c0 = slot + i * kSlots;
    if (c0 < NCHUNK) {
      const int c = c0 + rot < NCHUNK ? c0 + rot : c0 + rot - NCHUNK;
#pragma unroll
      for (int j = 0; j < 4; ++j) f[4 * i + j] = src[(4 * c + j) * kImageLanes];
    }
  }
#pragma unroll
  for (int i = 0; i < kMine; ++i) {
    const int c0 = slot + i * kSlots;
    if (c0 < NCHUNK) {
      const int c = c0 + rot < NCHUNK ? c0 + rot : c0 + rot - NCHUNK;
      uint32_t v[16];
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        v[4 * j] = __float_as_uint(f[4 * i + j].x);
        v[4 * j + 1] = __float_as_uint(f[4 * i + j].y);
        v[4 * j + 2] = __float_as_uint(f[4 * i + j].z);
        v[4 * j + 3] = __float_as_uint(f[4 * i + j].w);
      }
      tmem_st16(tb + 16 * c, v);
    }
  }
  asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}

template <typename TI, int MODE, int BITS, int GLANES>
__global__ void __launch_bounds__(kThreads, 1) k_fast4096(const FastArgs A) {
  extern __shared__ __align__(16) float smem[];
  __shared__ uint32_t s_tmem;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int slot = warp >> 2, wq = warp & 3, tau = wq * 32 + lane;
  float* bufAB = smem + slot * (3 * M);
  float* bufBC = bufAB + M;  // two buffers, used alternately
  const long long G = static_cast<long long>(gridDim.x) * kSlots;
  const long long g = static_cast<long long>(blockIdx.x) * kSlots + slot;
  const long long rb = g * A.rows / G, re = (g + 1) * A.rows / G;

  Prefetch<TI> pre;
  prefetch(pre, static_cast<const TI*>(A.x), rb, re > rb ? 1 : 0, tau);

  if (warp == 0) {
    const uint32_t dst = static_cast<uint32_t>(__cvta_generic_to_shared(&s_tmem));
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], 512;" ::"r"(dst) : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tb = s_tmem + (static_cast<uint32_t>(wq * 32) << 16);
  fill_tmem<kFillChunks>(A.image, tb, slot, tau);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();

  const bool scaled = A.hdr[0] == 1.f;
  uint32_t c0[32], c1[32];
  tmem_ld32(tb, c0);
  tmem_wait(c0);
  if (scaled)
    run_rows<TI, MODE, BITS, GLANES, true>(A, rb, re, slot, tau, lane, tb, bufAB, bufBC, pre, c0, c1);
  else
    run_rows<TI, MODE, BITS, GLANES, false>(A, rb, re, slot, tau, lane, tb, bufAB, bufBC, pre, c0, c1);

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 0) {
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, 512;" ::"r"(s_tmem) : "memory");
  }
}

template <typename TI, int MODE, int BITS, int GLANES>
bq_status launch(const FastArgs& A, cudaStream_t st) {
  auto kern = k_fast4096<TI, MODE, BITS, GLANES>;
  const int smem = kSlots * 3 * M * static_cast<int>(sizeof(float));
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return BQ_ERR_CUDA;
  // per device: the shared-memory opt-in and the SM count, set up on first use
  static int sms_of[64] = {};
  if (sms_of[dev] == 0) {
    int sms = 0;
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess ||
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || sms <= 0)
      return BQ_ERR_CUDA;
    sms_of[dev] = sms;
  }
  const int sms = sms_of[dev];
  long long grid = (A.rows + kSlots - 1) / kSlots;
  if (grid > sms) grid = sms;
  if (grid < 1) grid = 1;
  kern<<<static_cast<unsigned>(grid), kThreads, smem, st>>>(A);
  return cudaPeekAtLastError() == cudaSuccess ? BQ_OK : BQ_ERR_CUDA;
}

template <typename TI>
bq_status dispatch_quant(const FastArgs& A, int bits, int group, cudaStream_t st) {
  if (bits == 4) {
    if (group == 64) return launch<TI, kQuant, 4, 8>(A, st);
    if (group == 128) return launch<TI, kQuant, 4, 16>(A, st);
    return launch<TI, kQuant, 4, 32>(A, st);
  }
  if (group == 64) return launch<TI, kQuant, 2, 8>(A, st);
  if (group == 128) return launch<TI, kQuant, 2, 16>(A, st);
  return launch<TI, kQuant, 2, 32>(A, st);
}


// ------------------------------------------------------------------ inverse
//
// x = Q^T y: stages 11 .. 0, each the transpose [[c, s], [-s, c]] of its rotation,
// in the forward's thread layouts visited backwards (pass C, then B, then A) with
// the two transposes reversed.  Coefficients: the plain (cos, sin) image, whose
// stage-s block sits at column 32 s; the scaled form's [[1, alpha], [beta, 1]]
// steps do not invert into steps of the same shape.

template <int SB>
__device__ __forceinline__ void stage_inv(float2 (&a)[2][16], const uint32_t (&c)[32]) {
  if constexpr (SB == 0) {
#pragma unroll
    for (int q = 0; q < 8; ++q)
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const int k = 2 * q + e;
        const float cl = u2f(c[4 * q + e]), ch = u2f(c[4 * q + 2 + e]);
        const float lo = a[0][k].x, hi = a[0][k].y;
        a[0][k].x = fmaf(ch, hi, cl * lo);
        a[0][k].y = fmaf(-ch, lo, cl * hi);
      }
  } else {
#pragma unroll
    for (int q = 0; q < 8; ++q) {
      constexpr int kHalf = 1 << (SB - 1);
      const int lq = low_slot<SB>(2 * q) >> 1;
      const int hq = lq + kHalf;
      const float2 cl = make_float2(u2f(c[4 * q]), u2f(c[4 * q + 1]));
      const float2 ch = make_float2(u2f(c[4 * q + 2]), u2f(c[4 * q + 3]));
      const float2 lo = a[0][lq], hi = a[0][hq];
      a[0][lq] = __ffma2_rn(ch, hi, __fmul2_rn(cl, lo));
      a[0][hq] = __ffma2_rn(make_float2(-ch.x, -ch.y), lo, __fmul2_rn(cl, hi));
    }
  }
}

// stage S of the inverse from `cur`, while the block of stage S - 1 streams into `nxt`
template <int S, int SB>
__device__ __forceinline__ void inv_step(float2 (&a)[2][16], uint32_t (&cur)[32], uint32_t (&nxt)[32], uint32_t tb) {
  if constexpr (S > 0) tmem_ld32(tb + 32 * (S - 1), nxt);
  stage_inv<SB>(a, cur);
  if constexpr (S > 0) tmem_wait(nxt);
}

// Pass-C layout input: thread tau holds positions 8 tau + 1024 h + (0..7), h < 4.
template <typename TI>
__device__ __forceinline__ void prefetch_c(Prefetch<TI>& p, const TI* x, long long row, int cnt, int tau) {
  if (cnt > 0) {
    constexpr int kPer = Prefetch<TI>::kVec / 4;  // 16-byte vectors per group of 8 elements
#pragma unroll
    for (int h = 0; h < 4; ++h) {
      const uint4* src = reinterpret_cast<const uint4*>(x + row * M + h * 1024 + tau * 8);
#pragma unroll
      for (int i = 0; i < kPer; ++i) p.v[0][kPer * h + i] = src[i];
    }
  }
}

template <typename TI, typename TO>
__device__ __forceinline__ void inv_row(const FastArgs& A, long long row, int ncnt, int slot, int tau, uint32_t tb,
                                        float* bufAB, float* bufBC, Prefetch<TI>& pre, uint32_t (&c0)[32],
                                        uint32_t (&c1)[32]) {
  float2 a[2][16];
  unpack_input<1>(pre, a);
  prefetch_c(pre, static_cast<const TI*>(A.x), row + 1, ncnt, tau);
  // pass C: stages 11, 10 (slot bits 4, 3); c0 holds block 11 on entry
  inv_step<11, 4>(a, c0, c1, tb);
  inv_step<10, 3>(a, c1, c0, tb);
  {
    const int sw = (tau >> 2) & 1;
#pragma unroll
    for (int h = 0; h < 4; ++h)
#pragma unroll
      for (int hh = 0; hh < 2; ++hh)
        *reinterpret_cast<float4*>(bufBC + h * 1024 + tau * 8 + 4 * (hh ^ sw)) =
            make_float4(a[0][4 * h + 2 * hh].x, a[0][4 * h + 2 * hh].y, a[0][4 * h + 2 * hh + 1].x,
                        a[0][4 * h + 2 * hh + 1].y);
  }
  group_sync(slot);
  {
    const int base = (tau >> 5) * 1024 + ((tau & 31) >> 3) * 8 + (tau & 3), sw = (tau >> 2) & 1;
#pragma unroll
    for (int rb = 0; rb < 32; rb += 2)
      a[0][rb >> 1] = make_float2(bufBC[base + 32 * rb + 4 * sw], bufBC[base + 32 * (rb + 1) + 4 * (sw ^ 1)]);
  }
  // pass B: stages 9 .. 5
  inv_step<9, 4>(a, c0, c1, tb);
  inv_step<8, 3>(a, c1, c0, tb);
  inv_step<7, 2>(a, c0, c1, tb);
  inv_step<6, 1>(a, c1, c0, tb);
  inv_step<5, 0>(a, c0, c1, tb);
  {
    const int base = ((tau >> 5) << 10) + (tau & 3), cq = (tau & 31) >> 2;
#pragma unroll
    for (int rb = 0; rb < 32; rb += 2) {
      bufAB[base + 32 * rb + 4 * (cq ^ (rb & 7))] = a[0][rb >> 1].x;
      bufAB[base + 32 * (rb + 1) + 4 * (cq ^ ((rb + 1) & 7))] = a[0][rb >> 1].y;
    }
  }
  __syncwarp();  // the B -> A exchange stays inside the warp (position bits 10, 11)
#pragma unroll
  for (int c = 0; c < 8; ++c) {
    const float4 v = *reinterpret_cast<const float4*>(bufAB + tau * 32 + 4 * (c ^ (tau & 7)));
    a[0][2 * c] = make_float2(v.x, v.y);
    a[0][2 * c + 1] = make_float2(v.z, v.w);
  }
  // pass A: stages 4 .. 0, then block 11 again for the next row
  inv_step<4, 4>(a, c1, c0, tb);
  inv_step<3, 3>(a, c0, c1, tb);
  inv_step<2, 2>(a, c1, c0, tb);
  inv_step<1, 1>(a, c0, c1, tb);
  tmem_ld32(tb + 32 * 11, c0);
  stage_inv<0>(a, c1);
  // pass-A layout output: 32 consecutive positions at 32 tau
  const long long off = row * M + tau * 32;
  if constexpr (sizeof(TO) == 4) {
    float4* dst = reinterpret_cast<float4*>(static_cast<float*>(A.y) + off);
#pragma unroll
    for (int c = 0; c < 8; ++c) dst[c] = make_float4(a[0][2 * c].x, a[0][2 * c].y, a[0][2 * c + 1].x, a[0][2 * c + 1].y);
  } else {
    uint4* dst = reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(A.y) + off);
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      uint32_t w[4];
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        __nv_bfloat162 b = __floats2bfloat162_rn(a[0][4 * c + k].x, a[0][4 * c + k].y);
        w[k] = *reinterpret_cast<uint32_t*>(&b);
      }
      dst[c] = make_uint4(w[0], w[1], w[2], w[3]);
    }
  }
  tmem_wait(c0);
}

template <typename TI, typename TO>
__global__ void __launch_bounds__(kThreads, 1) k_inv4096(const FastArgs A) {
  extern __shared__ __align__(16) float smem[];
  __shared__ uint32_t s_tmem;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int slot = warp >> 2, wq = warp & 3, tau = wq * 32 + lane;
  float* bufAB = smem + slot * (3 * M);
  float* bufBC = bufAB + M;  // two buffers, used alternately
  const long long G = static_cast<long long>(gridDim.x) * kSlots;
  const long long g = static_cast<long long>(blockIdx.x) * kSlots + slot;
  const long long rb = g * A.rows / G, re = (g + 1) * A.rows / G;

  Prefetch<TI> pre;
  prefetch_c(pre, static_cast<const TI*>(A.x), rb, re > rb ? 1 : 0, tau);
  if (warp == 0) {
    const uint32_t dst = static_cast<uint32_t>(__cvta_generic_to_shared(&s_tmem));
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], 512;" ::"r"(dst) : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tb = s_tmem + (static_cast<uint32_t>(wq * 32) << 16);
  fill_tmem<kImageInvCols / 16>(A.image, tb, slot, tau);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();

  uint32_t c0[32], c1[32];
  tmem_ld32(tb + 32 * 11, c0);
  tmem_wait(c0);
  // the C -> B buffer alternates between rows (row i's readers and row i+2's
  // writers are kept apart by row i+1's barrier)
#pragma unroll 1
  for (long long row = rb; row < re; ++row)
    inv_row<TI, TO>(A, row, row + 1 < re ? 1 : 0, slot, tau, tb, bufAB, bufBC + ((row - rb) & 1) * M, pre, c0, c1);

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 0) {
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, 512;" ::"r"(s_tmem) : "memory");
  }
}

template <typename TI, typename TO>
bq_status launch_inv(const FastArgs& A, cudaStream_t st) {
  auto kern = k_inv4096<TI, TO>;
  const int smem = kSlots * 3 * M * static_cast<int>(sizeof(float));
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return BQ_ERR_CUDA;
  static int sms_of[64] = {};
  if (sms_of[dev] == 0) {
    int sms = 0;
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess ||
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || sms <= 0)
      return BQ_ERR_CUDA;
    sms_of[dev] = sms;
  }
  long long grid = (A.rows + kSlots - 1) / kSlots;
  if (grid > sms_of[dev]) grid = sms_of[dev];
  if (grid < 1) grid = 1;
  kern<<<static_cast<unsigned>(grid), kThreads, smem, st>>>(A);
  return cudaPeekAtLastError() == cudaSuccess ? BQ_OK : BQ_ERR_CUDA;
}

}  // namespace

bool fast4096_supports(const KLayer& L, const QuantArgs* q) {
  if (L.m != M || L.r != 1 || L.image == nullptr) return false;
  if (q && q->group != 64 && q->group != 128 && q->group != 256) return false;
  return true;
}

bq_status launch_fast4096(const KLayer& L, const void* x, bq_dtype xt, void* y, bq_dtype yt, int64_t rows,
                          const QuantArgs* q, cudaStream_t st) {
  FastArgs A;
  A.x = x;
  A.y = y;
  A.rows = rows;
  A.image = L.image;
  A.hdr = L.hdr;
  A.codes = q ? q->codes : nullptr;
  A.scale = q ? q->scale : nullptr;
  A.zero = q ? q->zero : nullptr;
  if (q) {
    return xt == BQ_F32 ? dispatch_quant<float>(A, q->bits, q->group, st)
                        : dispatch_quant<__nv_bfloat16>(A, q->bits, q->group, st);
  }
  if (xt == BQ_F32)
    return yt == BQ_F32 ? launch<float, kOutF32, 4, 16>(A, st) : launch<float, kOutBF16, 4, 16>(A, st);
  return yt == BQ_F32 ? launch<__nv_bfloat16, kOutF32, 4, 16>(A, st) : launch<__nv_bfloat16, kOutBF16, 4, 16>(A, st);
}

bq_status launch_inv4096(const KLayer& L, const void* y, bq_dtype yt, void* x, bq_dtype xt, int64_t rows,
                         cudaStream_t st) {
  FastArgs A;
  A.x = y;  // the kernel reads A.x and writes A.y
  A.y = x;
  A.rows = rows;
  A.image = L.image_inv;
  A.hdr = L.hdr;
  A.codes = nullptr;
  A.scale = nullptr;
  A.zero = nullptr;
  if (yt == BQ_F32) return xt == BQ_F32 ? launch_inv<float, float>(A, st) : launch_inv<float, __nv_bfloat16>(A, st);
  return xt == BQ_F32 ? launch_inv<__nv_bfloat16, float>(A, st) : launch_inv<__nv_bfloat16, __nv_bfloat16>(A, st);
}

}  // namespace bq
