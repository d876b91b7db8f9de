// W2A16 consumer GEMM on the fifth-generation tensor cores.
//
// The transform leaves a layer's output unchanged because y = W x = (W Q^T)(Q x)
// (ButterflyQuant abstract), and the pages deploy it with 2-bit weights and
// 16-bit activations (explainer article, section "training & results": W2A16).
// The quantized layer is therefore a GEMM of the rotated bfloat16 activations
// x~ = Q x with the dequantized codes of W Q^T:
//   out[t][o] = sum_k x~[t][k] * bf16((q[o][k] - z[o][g]) * s[o][g]),  g = k / group,
// with codes, scales and zero points in the layout bq_weight_rotate_pack writes
// (4-bit codes, W4A16, use the same kernel).
//
// The MMA computes D[o][t] (output features along M, tokens along N) with the
// dequantized weights as its A operand in TENSOR memory, so they never pass
// through shared memory: shared memory carries only the activation tiles (written
// once by the tensor memory accelerator, read once by the MMAs) and the packed
// codes, which halves its traffic per flop against staging both operands there
// (shared-memory bandwidth, not the tensor cores, bounds the two-operand form).
//
// One CTA per SM, persistent over tiles of 128 output features x 256 tokens, K in
// stages of 64:
//  * a 5-deep ring of stages, each an activation tile (up to 256 tokens x 64,
//    128-byte swizzled, the layout the MMA reads) with the packed codes of the
//    tile's 128 features in shared memory, and the A operand they become in
//    tensor memory (lane = feature, 32 columns of bf16 pairs); one "empty"
//    barrier per stage, committed by the MMAs, frees both halves;
//  * warp 12 (one thread) waits for a stage to be empty and loads it with the
//    tensor memory accelerator, completing on "full_x";
//  * warps 4-11 (two threads per feature, 32 of its 64 codes each) wait for
//    full_x, expand the codes to bfloat16 (q - z) * s in registers, store them
//    with tcgen05.st into the stage's A slot and arrive on "full_w".  full_x of
//    a round completes only after the copy was issued, which was after the
//    stage's previous MMAs had committed, so the A slot is free by then;
//  * warp 13 (one thread) waits for full_w alone (every dequantizing thread
//    acquired full_x before arriving, so the activation tile is ordered before
//    the MMAs too) and issues tcgen05.mma (bf16 x bf16 -> fp32, M = 128,
//    N = up to 256, K = 16), so each dequantized weight feeds up to 256 tokens;
//    one commit per stage frees it, one per work unit hands the accumulator
//    (256 columns) to the epilogue;
//  * warps 0-3 read the accumulator (lane = feature), transpose 32 x 32 blocks
//    through shared memory so that each thread holds one token's 32 consecutive
//    features, and store them; split-K partial rows ([token][128 features]) are
//    stored straight from the accumulator's layout, one token row per warp store.
//    For bfloat16 output the accumulator is first drained (rounded to bf16 pairs,
//    six chunks parked in spare tensor-memory columns, two in registers) and
//    handed back, so the next unit's MMAs do not wait for the transposes.
// Dequantization is exact up to the final bfloat16 rounding.  2-bit codes: a
// group has four possible weights, bf16((q - z) s) for q = 0..3 (the product is
// exact in float32, one cvt.rn rounds it); their low and high bytes form two
// 4-byte tables, and each pair of codes becomes one bf16x2 word by a byte
// permutation whose selector (q0, q0 + 4, q1, q1 + 4) one integer multiply-add
// builds from the codes.  4-bit codes: a code is placed in the mantissa of 2^23
// (one LOP3), (v - (2^23 + z 2^(b j))) is the exact integer (q - z) 2^(b j), the
// product with s 2^-(b j) is the exact (q - z) s, and one cvt.rn.bf16x2 rounds
// it; the packed f32x2 forms do two elements per instruction.
//
// Every wait on a barrier is bounded (one second): a wait that runs out sets the
// CTA's abort flag and a bit in the caller's status word, the other roles leave
// their loops when they see the flag, the copies and MMAs already issued are
// waited for (again bounded), and the tensor memory is freed before the kernel
// returns.
#include <cuda.h>
#include <cudaTypedefs.h>

#include <mutex>

#include "bq_internal.cuh"

namespace bq {
namespace {

constexpr int kBM = 128;                                 // output features per tile (the MMA's M)
constexpr int kBN = 256;                                 // largest token tile (the MMA's N; smaller for few tokens)
constexpr int kBK = 64;                                  // K per stage: one 128-byte row of bf16
constexpr int kStages = 5;                               // ring depth: activations + codes (shared memory)
                                                         // and the weights they pair with (tensor memory)
constexpr int kXBytes = kBN * kBK * 2;                   // 32 KiB activation tile
constexpr int kCodeBytes = kBM * kBK / 2;                // packed codes of a stage (4-bit size), 4 KiB
constexpr int kStageBytes = kXBytes + kCodeBytes;        // 36 KiB, a multiple of 1024
constexpr int kEpiOff = kStages * kStageBytes;           // epilogue transposes: 4 warps x 32 x 33 floats
constexpr int kBarOff = kEpiOff + 4 * 32 * 33 * 4;
constexpr int kSmemBytes = kBarOff + 320 + 1024;         // barriers, then slack for 1024-byte alignment
constexpr int kEpiWarps = 4, kDeqWarps = 8, kTmaWarp = 12, kMmaWarp = 13;
constexpr int kThreads = 32 * 14;
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColW = 256;                          // weight ring: stage s at columns 256 + 32 s
constexpr uint32_t kColSpare = kColW + 32 * kStages;    // 96 spare columns: six drained bf16 chunks
static_assert(kColSpare + 6 * 16 <= kTmemCols, "spare tensor-memory columns");
constexpr unsigned long long kWaitLimitNs = 1000000000ull;

// barrier block (byte offsets from kBarOff)
constexpr int kFullX = 0, kFullW = 64, kEmpty = 128, kAccFull = 192, kAccEmpty = 200, kDrain = 208,
              kTmemSlot = 216, kAbort = 220;

// status bits: which wait ran out
constexpr int kStTma = 1, kStDeq = 2, kStMmaOperands = 4, kStMmaAcc = 8, kStEpi = 16, kStDrain = 32;

// instruction descriptor: fp32 accumulate, bf16 A and B, both K-major, M = 128, N = ntok
__host__ __device__ constexpr uint32_t make_idesc(int ntok) {
  return (1u << 4) | (1u << 7) | (1u << 10) | (uint32_t(ntok >> 3) << 17) | (uint32_t(kBM >> 4) << 24);
}

// ------------------------------------------------------------------ PTX wrappers

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ unsigned long long gtimer() {
  unsigned long long t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}

__device__ __forceinline__ void mbar_expect_tx(uint32_t bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes) : "memory");
}

__device__ __forceinline__ bool mbar_try(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n selp.u32 %0, 1, 0, p;\n}"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}

// Wait for the phase of `parity` to complete.  Returns false when the CTA's abort
// flag is raised or the wait runs out (then it raises the flag and records `code`).
__device__ __forceinline__ bool wait_bar(uint32_t bar, uint32_t parity, volatile int* abort_flag, int32_t* status,
                                      int code) {
  if (mbar_try(bar, parity)) return true;
  const unsigned long long t0 = gtimer();
  for (uint32_t i = 1;; ++i) {
    if (mbar_try(bar, parity)) return true;
    if ((i & 15u) == 0) {
      if (*abort_flag) return false;
      if (gtimer() - t0 > kWaitLimitNs) {
        *abort_flag = 1;
        if (status) atomicOr(status, code);
        return false;
      }
    }
  }
}

// A wait that ignores the abort flag (for work already issued), still bounded.
__device__ __forceinline__ bool wait_bar_drain(uint32_t bar, uint32_t parity, int32_t* status) {
  const unsigned long long t0 = gtimer();
  while (!mbar_try(bar, parity)) {
    if (gtimer() - t0 > kWaitLimitNs) {
      if (status) atomicOr(status, kStDrain);
      return false;
    }
  }
  return true;
}

__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

__device__ __forceinline__ void tma_2d(uint32_t dst, const CUtensorMap* map, int x, int y, uint32_t bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];"
      ::"r"(dst), "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(bar)
      : "memory");
}

// shared-memory matrix descriptor: K-major, 128-byte swizzle, 8-row groups 1024 bytes apart
__device__ __forceinline__ uint64_t sw128_desc(uint32_t addr) {
  return static_cast<uint64_t>((addr >> 4) & 0x3FFFu) | (1ull << 16) | (64ull << 32) | (1ull << 46) | (2ull << 61);
}

// D (tensor memory) (+)= A (tensor memory, 128 lanes x 16 bf16) x B (shared memory, descriptor)
__device__ __forceinline__ void umma_bf16_ta(uint32_t d, uint32_t a, uint64_t b, uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n"
      " tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n}"
      ::"r"(d), "r"(a), "l"(b), "r"(idesc), "r"(accumulate)
      : "memory");
}

__device__ __forceinline__ void umma_commit(uint32_t bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar) : "memory");
}

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

__device__ __forceinline__ void tmem_wait_ld(uint32_t (&r)[32]) {
  asm volatile("tcgen05.wait::ld.sync.aligned;"
               : "+r"(r[0]), "+r"(r[1]), "+r"(r[2]), "+r"(r[3]), "+r"(r[4]), "+r"(r[5]), "+r"(r[6]), "+r"(r[7]),
                 "+r"(r[8]), "+r"(r[9]), "+r"(r[10]), "+r"(r[11]), "+r"(r[12]), "+r"(r[13]), "+r"(r[14]),
                 "+r"(r[15]), "+r"(r[16]), "+r"(r[17]), "+r"(r[18]), "+r"(r[19]), "+r"(r[20]), "+r"(r[21]),
                 "+r"(r[22]), "+r"(r[23]), "+r"(r[24]), "+r"(r[25]), "+r"(r[26]), "+r"(r[27]), "+r"(r[28]),
                 "+r"(r[29]), "+r"(r[30]), "+r"(r[31])::"memory");
}

__device__ __forceinline__ void tmem_st16(uint32_t addr, const uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], "
      "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};"
      ::"r"(addr), "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),
        "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15])
      : "memory");
}

__device__ __forceinline__ void tmem_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

__device__ __forceinline__ void tmem_ld16(uint32_t addr, uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
      : "r"(addr));
}

__device__ __forceinline__ void tmem_wait_ld16(uint32_t (&r)[16]) {
  asm volatile("tcgen05.wait::ld.sync.aligned;"
               : "+r"(r[0]), "+r"(r[1]), "+r"(r[2]), "+r"(r[3]), "+r"(r[4]), "+r"(r[5]), "+r"(r[6]), "+r"(r[7]),
                 "+r"(r[8]), "+r"(r[9]), "+r"(r[10]), "+r"(r[11]), "+r"(r[12]), "+r"(r[13]), "+r"(r[14]),
                 "+r"(r[15])::"memory");
}

__device__ __forceinline__ uint4 ld_shared_v4(uint32_t addr) {
  uint4 v;
  asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(addr)
               : "memory");
  return v;
}

__device__ __forceinline__ uint32_t bf16x2(float lo, float hi) {
  const __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<const uint32_t*>(&v);
}

// ------------------------------------------------------------------ dequantization

// Per-group constants of one output feature: for the code at position j of a
// 16-bit half (bit offset BITS j), nc[j] = -(2^23 + z 2^(BITS j)) and
// sf[j] = s 2^-(BITS j), held as pairs (j, j + 1) for the f32x2 forms.
template <int BITS>
struct Dequant {
  static constexpr int J = 16 / BITS;  // codes per 16-bit half
  float2 nc[J / 2], sf[J / 2];

  __device__ __forceinline__ void set(float s, float z) {
#pragma unroll
    for (int p = 0; p < J / 2; ++p) {
      const float w0 = static_cast<float>(1u << (BITS * 2 * p)), w1 = static_cast<float>(1u << (BITS * (2 * p + 1)));
      nc[p] = make_float2(-(8388608.f + z * w0), -(8388608.f + z * w1));
      sf[p] = make_float2(s * (1.f / w0), s * (1.f / w1));
    }
  }

  // J codes at the bottom 16 bits of x -> J / 2 words of two bfloat16 each
  __device__ __forceinline__ void half(uint32_t x, uint32_t* out) const {
#pragma unroll
    for (int p = 0; p < J / 2; ++p) {
      constexpr uint32_t kMask = (1u << BITS) - 1u;
      const uint32_t m0 = kMask << (BITS * 2 * p), m1 = kMask << (BITS * (2 * p + 1));
      const float2 v = make_float2(__uint_as_float((x & m0) | 0x4B000000u), __uint_as_float((x & m1) | 0x4B000000u));
      const float2 f = __fmul2_rn(__fadd2_rn(v, nc[p]), sf[p]);
      out[p] = bf16x2(f.x, f.y);
    }
  }
};

// The four weights a 2-bit group can hold as byte tables: byte q of `lo` / `hi` is
// the low / high byte of bf16((q - z) s).
struct Lut2 {
  uint32_t lo, hi;

  __device__ __forceinline__ void set(float s, float z) {
    const uint32_t p01 = bf16x2((0.f - z) * s, (1.f - z) * s);
    const uint32_t p23 = bf16x2((2.f - z) * s, (3.f - z) * s);
    lo = __byte_perm(p01, p23, 0x6420);
    hi = __byte_perm(p01, p23, 0x7531);
  }

  // 16 codes of one word (code i at bits 2i) -> 8 words of bf16 pairs (codes 2j, 2j + 1)
  __device__ __forceinline__ void word(uint32_t c, uint32_t* out) const {
    const uint32_t m0 = c & 0x03030303u, m1 = (c >> 2) & 0x03030303u;  // byte b: codes 4b, 4b + 1
    const uint32_t m2 = (c >> 4) & 0x03030303u, m3 = (c >> 6) & 0x03030303u;  // codes 4b + 2, 4b + 3
    // bytes (qa, qb, qc, qd) -> selector nibbles (qa, qa + 4, qb, qb + 4, qc, qc + 4, qd, qd + 4)
    const uint32_t g0 = __byte_perm(m0, m1, 0x5140) * 0x11u + 0x40404040u;  // codes 0, 1, 4, 5
    const uint32_t g1 = __byte_perm(m2, m3, 0x5140) * 0x11u + 0x40404040u;  // codes 2, 3, 6, 7
    const uint32_t g2 = __byte_perm(m0, m1, 0x7362) * 0x11u + 0x40404040u;  // codes 8, 9, 12, 13
    const uint32_t g3 = __byte_perm(m2, m3, 0x7362) * 0x11u + 0x40404040u;  // codes 10, 11, 14, 15
    out[0] = __byte_perm(lo, hi, g0);
    out[1] = __byte_perm(lo, hi, g1);
    out[2] = __byte_perm(lo, hi, g0 >> 16);
    out[3] = __byte_perm(lo, hi, g1 >> 16);
    out[4] = __byte_perm(lo, hi, g2);
    out[5] = __byte_perm(lo, hi, g3);
    out[6] = __byte_perm(lo, hi, g2 >> 16);
    out[7] = __byte_perm(lo, hi, g3 >> 16);
  }
};

// Per-group expansion state: the byte tables for 2-bit codes, the f32x2 constants
// for 4-bit codes.
template <int BITS>
struct Expand;

template <>
struct Expand<2> {
  Lut2 t;
  __device__ __forceinline__ void set(float s, float z) { t.set(s, z); }
  // 32 codes (8 bytes at `codes` in shared memory) -> 16 words
  __device__ __forceinline__ void run(uint32_t codes, uint32_t (&v)[16]) const {
    uint32_t a, b;
    asm volatile("ld.shared.v2.b32 {%0, %1}, [%2];" : "=r"(a), "=r"(b) : "r"(codes) : "memory");
    t.word(a, v);
    t.word(b, v + 8);
  }
};

template <>
struct Expand<4> {
  Dequant<4> dq;
  __device__ __forceinline__ void set(float s, float z) { dq.set(s, z); }
  // 32 codes (16 bytes at `codes` in shared memory) -> 16 words
  __device__ __forceinline__ void run(uint32_t codes, uint32_t (&v)[16]) const {
    const uint4 a = ld_shared_v4(codes);
    const uint32_t w[4] = {a.x, a.y, a.z, a.w};
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      dq.half(w[c], v + 4 * c);
      dq.half(w[c] >> 16, v + 4 * c + 2);
    }
  }
};

// ------------------------------------------------------------------ epilogue store

// 32 consecutive features o0 .. o0 + 31 of token t
template <bool BF16>
__device__ __forceinline__ void store_row32(void* out, long long t, int out_features, int o0, bool vec,
                                            const float (&r)[32]) {
  if (BF16) {
    __nv_bfloat16* row = static_cast<__nv_bfloat16*>(out) + t * out_features;
    if (vec && o0 + 32 <= out_features) {
      uint4* dst = reinterpret_cast<uint4*>(row + o0);
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int e = 8 * i;
        dst[i] = make_uint4(bf16x2(r[e], r[e + 1]), bf16x2(r[e + 2], r[e + 3]), bf16x2(r[e + 4], r[e + 5]),
                            bf16x2(r[e + 6], r[e + 7]));
      }
    } else {
#pragma unroll
      for (int e = 0; e < 32; ++e)
        if (o0 + e < out_features) row[o0 + e] = __float2bfloat16_rn(r[e]);
    }
  } else {
    float* row = static_cast<float*>(out) + t * out_features;
    if (vec && o0 + 32 <= out_features) {
      float4* dst = reinterpret_cast<float4*>(row + o0);
#pragma unroll
      for (int i = 0; i < 8; ++i) dst[i] = make_float4(r[4 * i], r[4 * i + 1], r[4 * i + 2], r[4 * i + 3]);
    } else {
#pragma unroll
      for (int e = 0; e < 32; ++e)
        if (o0 + e < out_features) row[o0 + e] = r[e];
    }
  }
}

// ------------------------------------------------------------------ kernel

struct GemmArgs {
  const uint16_t* scale;  // [out_features][n / group] fp16 bits
  const uint16_t* zero;
  void* out;              // [tokens][out_features]
  float* part;            // split-K partial sums [f_tile][t_tile][ksplit][ntok][128] (ksplit > 1)
  int tokens, out_features, n, group;
  int ntok, npad;         // tokens per tile (the MMA's N, a multiple of 16) and its 32-rounded width
  uint32_t idesc;
  int kblocks, ksplit;    // K stages of 64, and the slices K is cut into
  int t_tiles, units;     // token tiles; work units = t_tiles x ksplit x feature tiles
  int vec;                // epilogue may use 16-byte stores
  int32_t* status;
};

// Work unit u: token tile fastest, then K slice, then feature tile.
struct Unit {
  int t_tile, ks, f_tile, t0, o0, kb0, kb1;
};

__device__ __forceinline__ Unit unit_of(const GemmArgs& a, int u) {
  Unit r;
  r.t_tile = u % a.t_tiles;
  const int rest = u / a.t_tiles;
  r.ks = rest % a.ksplit;
  r.f_tile = rest / a.ksplit;
  r.t0 = r.t_tile * a.ntok;
  r.o0 = r.f_tile * kBM;
  r.kb0 = r.ks * a.kblocks / a.ksplit;
  r.kb1 = (r.ks + 1) * a.kblocks / a.ksplit;
  return r;
}

template <int BITS, bool BF16>
__global__ void __launch_bounds__(kThreads, 1)
    k_w2a16(const __grid_constant__ CUtensorMap map_x, const __grid_constant__ CUtensorMap map_codes,
            const GemmArgs args) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* gbase = smem_raw + (base - raw);
  const uint32_t bars = base + kBarOff;
  volatile int* abort_flag = reinterpret_cast<volatile int*>(gbase + kBarOff + kAbort);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(gbase + kBarOff + kTmemSlot);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  constexpr uint32_t kCodeRow = kBK * BITS / 8;             // packed bytes of one feature per stage
  const uint32_t tx = static_cast<uint32_t>(args.ntok) * (kBK * 2) + kBM * kCodeRow;  // bytes of a stage's copies

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(bars + kFullX + 8 * s, 1);
      mbar_init(bars + kFullW + 8 * s, 32 * kDeqWarps);
      mbar_init(bars + kEmpty + 8 * s, 1);
    }
    mbar_init(bars + kAccFull, 1);
    mbar_init(bars + kAccEmpty, 32 * kEpiWarps);
    mbar_init(bars + kDrain, 1);
    *abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == kMmaWarp) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(tmem_slot)),
                 "r"(kTmemCols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  if (warp == kTmaWarp && lane == 0) {
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&map_x)) : "memory");
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&map_codes)) : "memory");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == kTmaWarp) {
    // ---------------------------------------------------------------- loads
    if (lane == 0) {
      uint32_t s = 0, par = 0, issued = 0, last_parity = 0;
      bool ok = true;
      for (int u = blockIdx.x; ok && u < args.units; u += gridDim.x) {
        const Unit U = unit_of(args, u);
        for (int kb = U.kb0; kb < U.kb1; ++kb) {
          if (!wait_bar(bars + kEmpty + 8 * s, par ^ 1u, abort_flag, args.status, kStTma)) {
            ok = false;
            break;
          }
          const uint32_t st = base + s * kStageBytes;
          mbar_expect_tx(bars + kFullX + 8 * s, tx);
          tma_2d(st, &map_x, kb * kBK, U.t0, bars + kFullX + 8 * s);
          tma_2d(st + kXBytes, &map_codes, kb * kCodeRow, U.o0, bars + kFullX + 8 * s);
          issued |= 1u << s;
          last_parity = (last_parity & ~(1u << s)) | (par << s);
          if (++s == kStages) {
            s = 0;
            par ^= 1u;
          }
        }
      }
      // copies still in flight land before the CTA exits
      for (int s = 0; s < kStages; ++s)
        if ((issued >> s) & 1u) wait_bar_drain(bars + kFullX + 8 * s, (last_parity >> s) & 1u, args.status);
    }
    __syncwarp();
  } else if (warp == kMmaWarp) {
    // ---------------------------------------------------------------- MMA issue
    if (lane == 0) {
      uint32_t s = 0, par = 0;
      const uint32_t idesc = args.idesc;
      bool ok = true;
      int i = 0;
      for (int u = blockIdx.x; ok && u < args.units; u += gridDim.x, ++i) {
        const Unit U = unit_of(args, u);
        // one accumulator: unit i starts once the epilogue has read unit i - 1
        if (!wait_bar(bars + kAccEmpty, (i & 1) ^ 1, abort_flag, args.status, kStMmaAcc)) break;
        tc_fence_after();
        uint32_t acc = 0;
        for (int kb = U.kb0; kb < U.kb1; ++kb) {
          if (!wait_bar(bars + kFullW + 8 * s, par, abort_flag, args.status, kStMmaOperands)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint64_t xd = sw128_desc(base + s * kStageBytes);
          const uint32_t a = tmem + kColW + 32u * s;
#pragma unroll
          for (int j = 0; j < kBK / 16; ++j) {
            umma_bf16_ta(tmem, a + 8 * j, xd + 2 * j, idesc, acc);  // +32 bytes of K per step
            acc = 1;
          }
          umma_commit(bars + kEmpty + 8 * s);
          if (++s == kStages) {
            s = 0;
            par ^= 1u;
          }
        }
        if (ok) umma_commit(bars + kAccFull);
      }
      // every MMA issued has completed before the tensor memory is freed
      umma_commit(bars + kDrain);
      wait_bar_drain(bars + kDrain, 0, args.status);
    }
    __syncwarp();
  } else if (warp >= kEpiWarps) {
    // ---------------------------------------------------------------- dequantization
    const int dw = warp - kEpiWarps;             // 0 .. 7
    const int f = 32 * (dw & 3) + lane;          // feature of the tile = tensor-memory lane, 0 .. 127
    const int kh = dw >> 2;                      // which 32 of the stage's 64 codes
    const uint32_t lane_base = static_cast<uint32_t>(32 * (warp & 3)) << 16;
    const uint32_t col = 16u * kh;
    const int gpr = args.n / args.group, kb_per_group = args.group / kBK;
    Expand<BITS> ex;
    // (s, z) of the next group this thread expands: units in CTA order, each from
    // the group of its first stage to the group of its last; the unit's geometry
    // is computed once per unit
    int pu = blockIdx.x, pg = 0, pg_last = -1;
    long long po = 0;
    auto enter = [&]() {
      if (pu < args.units) {
        const Unit P = unit_of(args, pu);
        pg = P.kb0 / kb_per_group;
        pg_last = (P.kb1 - 1) / kb_per_group;
        po = static_cast<long long>(P.o0) + f;
      }
    };
    float s_next = 0.f, z_next = 0.f;
    auto load_sz = [&]() {
      s_next = 0.f;
      z_next = 0.f;
      if (pu < args.units && po < args.out_features) {
        s_next = __half2float(__ushort_as_half(__ldg(args.scale + po * gpr + pg)));
        z_next = __half2float(__ushort_as_half(__ldg(args.zero + po * gpr + pg)));
      }
    };
    auto advance = [&]() {
      if (pg < pg_last) {
        ++pg;
      } else {
        pu += gridDim.x;
        enter();
      }
    };
    enter();
    load_sz();
    uint32_t s = 0, par = 0;
    bool ok = true;
    for (int u = blockIdx.x; ok && u < args.units; u += gridDim.x) {
      const Unit U = unit_of(args, u);
      for (int kb = U.kb0; kb < U.kb1; ++kb) {
        if (kb == U.kb0 || (kb & (kb_per_group - 1)) == 0) {  // kb_per_group is 1, 2 or 4
          ex.set(s_next, z_next);
          advance();
          load_sz();
        }
        // full_x: the stage's copies landed, so its previous MMAs (which read the A
        // slot too) have committed
        if (!wait_bar(bars + kFullX + 8 * s, par, abort_flag, args.status, kStDeq)) {
          ok = false;
          break;
        }
        tc_fence_after();
        uint32_t v[16];
        ex.run(base + s * kStageBytes + kXBytes + f * kCodeRow + kh * (kCodeRow / 2), v);
        tmem_st16(tmem + lane_base + kColW + 32u * s + col, v);
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(bars + kFullW + 8 * s);
        if (++s == kStages) {
          s = 0;
          par ^= 1u;
        }
      }
    }
  } else {
    // ---------------------------------------------------------------- epilogue
    float* buf = reinterpret_cast<float*>(gbase + kEpiOff) + warp * (32 * 33);
    const int nchunks = args.npad / 32;
    int i = 0;
    for (int u = blockIdx.x; u < args.units; u += gridDim.x, ++i) {
      if (!wait_bar(bars + kAccFull, i & 1, abort_flag, args.status, kStEpi)) break;
      tc_fence_after();
      const Unit U = unit_of(args, u);
      // split K: this slice's partial sums, rows of 128 features per token of the tile
      float* slice = args.ksplit > 1 ? args.part + ((static_cast<size_t>(U.f_tile) * args.t_tiles + U.t_tile) *
                                                        args.ksplit + U.ks) * args.ntok * kBM
                                     : nullptr;
      // Chunk q: r[j] = D[feature 32 warp + lane][token 32 q + j].  The load of
      // chunk q + 1 into the same registers starts as soon as r has been consumed,
      // and the accumulator is handed back right after its last load.
      const uint32_t lane_base = static_cast<uint32_t>(32 * warp) << 16;
      const int tmax = min(args.ntok, args.tokens - U.t0);  // valid tokens of the tile
      uint32_t r[32];
      tmem_ld32(tmem + lane_base, r);
      if (slice) {
        // split-K partial rows [token][128 features]: each warp store writes one
        // token's 32 features of this warp (128 contiguous bytes), no transpose
        float* d = slice + 32 * warp + lane;
#pragma unroll 1
        for (int q = 0; q < nchunks; ++q) {
          tmem_wait_ld(r);
          if (q + 1 == nchunks) {
            tc_fence_before();
            mbar_arrive(bars + kAccEmpty);
          }
          float c[32];
#pragma unroll
          for (int j = 0; j < 32; ++j) c[j] = __uint_as_float(r[j]);
          if (q + 1 < nchunks) tmem_ld32(tmem + lane_base + 32u * (q + 1), r);
#pragma unroll
          for (int j = 0; j < 32; ++j)
            if (32 * q + j < tmax) d[static_cast<size_t>(32 * q + j) * kBM] = c[j];
        }
      } else if (BF16) {
        // bfloat16 rows: the accumulator is drained before anything is stored.  Each
        // chunk is rounded to bf16 pairs at once (word k = tokens 2k, 2k + 1 of the
        // chunk); chunks 0-5 go to the spare tensor-memory columns, chunks 6-7 stay
        // in registers, and the accumulator is handed back to the MMAs; the
        // transposes and stores then overlap the next unit's MMAs.
        uint32_t keep[2][16];
#pragma unroll
        for (int q = 0; q < 8; ++q) {
          if (q < nchunks) {
            tmem_wait_ld(r);
            uint32_t p[16];
#pragma unroll
            for (int k = 0; k < 16; ++k) p[k] = bf16x2(__uint_as_float(r[2 * k]), __uint_as_float(r[2 * k + 1]));
            if (q + 1 < nchunks) tmem_ld32(tmem + lane_base + 32u * (q + 1), r);
            if (q < 6) {
              tmem_st16(tmem + lane_base + kColSpare + 16u * q, p);
            } else {
#pragma unroll
              for (int k = 0; k < 16; ++k) keep[q - 6][k] = p[k];
            }
          }
        }
        tc_fence_before();
        mbar_arrive(bars + kAccEmpty);
        tmem_wait_st();
        // per warp [32 tokens][40 halves]: rows of 80 bytes, 16-byte aligned
        uint16_t* b16 = reinterpret_cast<uint16_t*>(buf);
        const int o = U.o0 + 32 * warp;  // first feature of this warp
#pragma unroll
        for (int q = 0; q < 8; ++q) {
          if (q < nchunks) {
            uint32_t w[16];
            if (q < 6) {
              tmem_ld16(tmem + lane_base + kColSpare + 16u * q, w);
              tmem_wait_ld16(w);
            } else {
#pragma unroll
              for (int k = 0; k < 16; ++k) w[k] = keep[q - 6][k];
            }
#pragma unroll
            for (int k = 0; k < 16; ++k) {
              b16[(2 * k) * 40 + lane] = static_cast<uint16_t>(w[k] & 0xffffu);
              b16[(2 * k + 1) * 40 + lane] = static_cast<uint16_t>(w[k] >> 16);
            }
            __syncwarp();
            const int tt = 32 * q + lane;  // token within the tile
            if (tt < tmax) {
              const uint16_t* src = b16 + lane * 40;
              uint16_t* row = static_cast<uint16_t*>(args.out) +
                              (static_cast<long long>(U.t0) + tt) * args.out_features;
              if (args.vec != 0 && o + 32 <= args.out_features) {
                uint4* dst = reinterpret_cast<uint4*>(row + o);
#pragma unroll
                for (int i = 0; i < 4; ++i) dst[i] = reinterpret_cast<const uint4*>(src)[i];
              } else {
#pragma unroll
                for (int e = 0; e < 32; ++e)
                  if (o + e < args.out_features) row[o + e] = src[e];
              }
            }
            __syncwarp();
          }
        }
      } else {
        // float32 rows: transposed through shared memory so that this thread holds
        // token 32 q + lane's 32 consecutive features (16-byte stores)
#pragma unroll 1
        for (int q = 0; q < nchunks; ++q) {
          tmem_wait_ld(r);
          if (q + 1 == nchunks) {
            tc_fence_before();
            mbar_arrive(bars + kAccEmpty);
          }
#pragma unroll
          for (int j = 0; j < 32; ++j) buf[j * 33 + lane] = __uint_as_float(r[j]);
          if (q + 1 < nchunks) tmem_ld32(tmem + lane_base + 32u * (q + 1), r);
          __syncwarp();
          float c[32];
#pragma unroll
          for (int j = 0; j < 32; ++j) c[j] = buf[lane * 33 + j];
          __syncwarp();
          const int tt = 32 * q + lane;  // token within the tile
          if (tt < tmax)
            store_row32<BF16>(args.out, static_cast<long long>(U.t0) + tt, args.out_features, U.o0 + 32 * warp,
                              args.vec != 0, c);
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == kMmaWarp) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kTmemCols) : "memory");
  }
}

// Split K: out[t][o] = sum over the slices, in slice order, of the partial sums.
// One thread per output element, features fastest (coalesced reads and writes).
template <bool BF16>
__global__ void __launch_bounds__(256) k_splitk_reduce(const float* __restrict__ part, void* __restrict__ out,
                                                       int tokens, int out_features, int ntok, int t_tiles,
                                                       int ksplit) {
  const long long total = static_cast<long long>(tokens) * out_features;
  for (long long e = blockIdx.x * 256LL + threadIdx.x; e < total; e += static_cast<long long>(gridDim.x) * 256) {
    const int t = static_cast<int>(e / out_features), o = static_cast<int>(e % out_features);
    const int t_tile = t / ntok, f_tile = o / kBM;
    const float* p = part + ((static_cast<size_t>(f_tile) * t_tiles + t_tile) * ksplit * ntok + (t % ntok)) * kBM +
                     (o % kBM);
    float v = 0.f;
    for (int k = 0; k < ksplit; ++k) v += __ldg(p + static_cast<size_t>(k) * ntok * kBM);
    if (BF16)
      static_cast<__nv_bfloat16*>(out)[e] = __float2bfloat16_rn(v);
    else
      static_cast<float*>(out)[e] = v;
  }
}

// ------------------------------------------------------------------ decode path (1-8 tokens)
//
// With a handful of tokens each dequantized weight feeds only T products, and the
// tensor-core GEMM is bound by its MMA issue rate (four instructions per K stage of
// 128 features whatever N is).  Here the weights are expanded in registers straight
// into the A fragments of warp-level bf16 MMAs (mma.sync m16n8k16, float32
// accumulation) with the tokens as N (an 8-token fragment), so the products
// and sums leave the CUDA cores: what remains per weight is the expansion (about 1.5
// instructions per weight for 2-bit codes: the byte tables' selectors and permutes).
//
// A block is four warps on 16 output features; warp w takes a quarter of K in windows
// of 256, the next window's codes loading while one is expanded.  Lane (g, c) = (lane / 4, lane % 4) owns features f0 + g and f0 + g + 8 and,
// in window j, the 64 channels k = 256 j + 64 c .. + 63, so that its codes of a
// window are one contiguous 16- or 32-byte run per feature and its group parameters
// one pair per feature (groups are multiples of 64).  The MMA's 16-wide K slice s of
// the window maps its positions 2c, 2c + 1, 2c + 8, 2c + 9 to the channels
// k + 4 s + 0, 1, 2, 3 of lane c's run; A (weights) and B (activations) use the same
// map, so the contraction is the plain dot product.  The four warps' partial sums are
// added in warp order: the result is reproducible bitwise, and its error stays within
// one float32 rounding per 16 products plus the final adds (the GEMM's bound).
constexpr int kDecMaxTokens = 8;
constexpr int kDecWarps = 4;


__device__ __forceinline__ void mma_16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                          uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
      "{%0, %1, %2, %3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// 16 consecutive codes of one feature (bits 2i or 4i of `c`: one word of 2-bit codes, or
// the low / high half of two words of 4-bit codes) -> 8 words of bf16 pairs
template <int BITS>
__device__ __forceinline__ void expand16(const Expand<BITS>& ex, const uint32_t* c, uint32_t (&w)[8]) {
  if constexpr (BITS == 2) {
    ex.t.word(c[0], w);
  } else {
    ex.dq.half(c[0], w);
    ex.dq.half(c[0] >> 16, w + 2);
    ex.dq.half(c[1], w + 4);
    ex.dq.half(c[1] >> 16, w + 6);
  }
}

template <int BITS, int NB, bool BF16>
__global__ void __launch_bounds__(32 * kDecWarps)
    k_w2a16_dec(const __nv_bfloat16* __restrict__ x, int tokens, const uint8_t* __restrict__ codes,
                const uint16_t* __restrict__ scale, const uint16_t* __restrict__ zero, void* __restrict__ out, int n,
                int out_features, int group) {
  __shared__ float red[kDecWarps][16][8 * NB];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = lane >> 2, c = lane & 3;
  const int f0 = blockIdx.x * 16;
  const int fa = f0 + g, fb = f0 + g + 8;
  const bool la = fa < out_features, lb = fb < out_features;
  const int nwin = n / 256;
  const int j0 = (warp * nwin) / kDecWarps, j1 = ((warp + 1) * nwin) / kDecWarps;
  constexpr int kRun = 64 * BITS / 8;  // code bytes of a lane's run
  const size_t row_bytes = static_cast<size_t>(n) * BITS / 8;
  const uint8_t* ca = codes + static_cast<size_t>(la ? fa : 0) * row_bytes;
  const uint8_t* cb = codes + static_cast<size_t>(lb ? fb : 0) * row_bytes;
  const int gpr = n / group;
  // activations of token g (and g + 8): rows past the last token read token 0 and are
  // never stored
  const __nv_bfloat16* xr[NB];
#pragma unroll
  for (int h = 0; h < NB; ++h) xr[h] = x + static_cast<size_t>(g + 8 * h < tokens ? g + 8 * h : 0) * n;

  float d[NB][4];
#pragma unroll
  for (int h = 0; h < NB; ++h) d[h][0] = d[h][1] = d[h][2] = d[h][3] = 0.f;

  auto load_run = [&](const uint8_t* base, int j, uint32_t (&r)[kRun / 4]) {
    const uint4* src = reinterpret_cast<const uint4*>(base + static_cast<size_t>(256 * j + 64 * c) * BITS / 8);
#pragma unroll
    for (int q = 0; q < kRun / 16; ++q) {
      const uint4 v = __ldcs(src + q);
      r[4 * q] = v.x;
      r[4 * q + 1] = v.y;
      r[4 * q + 2] = v.z;
      r[4 * q + 3] = v.w;
    }
  };
  uint32_t ra[kRun / 4], rb[kRun / 4];
  if (j0 < j1) {
    load_run(ca, j0, ra);
    load_run(cb, j0, rb);
  }
#pragma unroll 1
  for (int j = j0; j < j1; ++j) {
    const int k = 256 * j + 64 * c;
    const int gi = k / group;
    Expand<BITS> ea, eb;
    ea.set(la ? __half2float(__ushort_as_half(__ldg(scale + static_cast<size_t>(fa) * gpr + gi))) : 0.f,
           la ? __half2float(__ushort_as_half(__ldg(zero + static_cast<size_t>(fa) * gpr + gi))) : 0.f);
    eb.set(lb ? __half2float(__ushort_as_half(__ldg(scale + static_cast<size_t>(fb) * gpr + gi))) : 0.f,
           lb ? __half2float(__ushort_as_half(__ldg(zero + static_cast<size_t>(fb) * gpr + gi))) : 0.f);
    uint32_t qa[kRun / 4], qb[kRun / 4];
#pragma unroll
    for (int i = 0; i < kRun / 4; ++i) {
      qa[i] = ra[i];
      qb[i] = rb[i];
    }
    if (j + 1 < j1) {  // the next window's codes in flight meanwhile
      load_run(ca, j + 1, ra);
      load_run(cb, j + 1, rb);
    }
#pragma unroll
    for (int sub = 0; sub < 4; ++sub) {  // 16 channels: four K slices of the MMA
      uint32_t wa[8], wb[8];
      expand16<BITS>(ea, qa + sub * (BITS / 2), wa);
      expand16<BITS>(eb, qb + sub * (BITS / 2), wb);
      uint4 xv[NB][2];
#pragma unroll
      for (int h = 0; h < NB; ++h) {
        const uint4* xs = reinterpret_cast<const uint4*>(xr[h] + k + 16 * sub);
        xv[h][0] = __ldg(xs);
        xv[h][1] = __ldg(xs + 1);
      }
#pragma unroll
      for (int s = 0; s < 4; ++s) {
#pragma unroll
        for (int h = 0; h < NB; ++h) {
          const uint4& v = xv[h][s >> 1];
          const uint32_t b0 = (s & 1) ? v.z : v.x, b1 = (s & 1) ? v.w : v.y;
          mma_16816(d[h], wa[2 * s], wb[2 * s], wa[2 * s + 1], wb[2 * s + 1], b0, b1);
        }
      }
    }
  }
  // d[h]: (feature g, tokens 8 h + 2 c, + 1), (feature g + 8, the same tokens)
#pragma unroll
  for (int h = 0; h < NB; ++h) {
    red[warp][g][8 * h + 2 * c] = d[h][0];
    red[warp][g][8 * h + 2 * c + 1] = d[h][1];
    red[warp][g + 8][8 * h + 2 * c] = d[h][2];
    red[warp][g + 8][8 * h + 2 * c + 1] = d[h][3];
  }
  __syncthreads();
  for (int e = threadIdx.x; e < 16 * 8 * NB; e += 32 * kDecWarps) {
    const int t = e / 16, f = e % 16;  // features fastest: coalesced stores
    if (t < tokens && f0 + f < out_features) {
      float v = red[0][f][t];
#pragma unroll
      for (int w = 1; w < kDecWarps; ++w) v += red[w][f][t];
      const size_t o = static_cast<size_t>(t) * out_features + f0 + f;
      if (BF16)
        static_cast<__nv_bfloat16*>(out)[o] = __float2bfloat16_rn(v);
      else
        static_cast<float*>(out)[o] = v;
    }
  }
}

template <int BITS, bool BF16>
bq_status run_dec(const void* x, int tokens, int n, const uint8_t* codes, const uint16_t* scale, const uint16_t* zero,
                  void* out, int out_features, int group, cudaStream_t st) {
  const unsigned grid = static_cast<unsigned>((out_features + 15) / 16);
  const auto* xb = static_cast<const __nv_bfloat16*>(x);
  k_w2a16_dec<BITS, 1, BF16><<<grid, 32 * kDecWarps, 0, st>>>(xb, tokens, codes, scale, zero, out, n, out_features,
                                                               group);
  return cudaPeekAtLastError() == cudaSuccess ? BQ_OK : BQ_ERR_CUDA;
}

bool dec_applies(long long tokens, int n) { return tokens >= 1 && tokens <= kDecMaxTokens && n % 256 == 0; }

// ------------------------------------------------------------------ host side

PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q{};
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

bool encode_2d(CUtensorMap* map, CUtensorMapDataType type, const void* ptr, uint64_t inner, uint64_t outer,
               uint64_t row_bytes, uint32_t box_inner, uint32_t box_outer, CUtensorMapSwizzle swizzle) {
  const PFN_cuTensorMapEncodeTiled_v12000 fn = tensor_map_encoder();
  if (!fn) return false;
  const cuuint64_t dims[2] = {inner, outer};
  const cuuint64_t strides[1] = {row_bytes};
  const cuuint32_t box[2] = {box_inner, box_outer};
  const cuuint32_t elem[2] = {1, 1};
  return fn(map, type, 2, const_cast<void*>(ptr), dims, strides, box, elem, CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}


template <int BITS, bool BF16>
bq_status run_gemm(const CUtensorMap& mx, const CUtensorMap& mc, const GemmArgs& a, int grid, cudaStream_t st) {
  auto kern = k_w2a16<BITS, BF16>;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes) != cudaSuccess)
    return BQ_ERR_CUDA;
  kern<<<grid, kThreads, kSmemBytes, st>>>(mx, mc, a);
  return cudaPeekAtLastError() == cudaSuccess ? BQ_OK : BQ_ERR_CUDA;
}

int sm_count() {
  int dev = 0, sms = 148;
  if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  return sms > 0 ? sms : 148;
}

// The launch shape: token tile (the MMA's N), tiles, and the K split that gives at
// least two work units per SM when there are few tiles (at least 4 K stages each).
struct Plan {
  int ntok, npad, t_tiles, f_tiles, kblocks, ksplit;
  size_t part_bytes;
};

Plan plan_of(long long tokens, int n, long long out_features, int sms) {
  Plan p;
  p.ntok = tokens >= kBN ? kBN : static_cast<int>((tokens + 15) / 16 * 16);
  if (p.ntok < 16) p.ntok = 16;
  p.npad = (p.ntok + 31) / 32 * 32;
  p.t_tiles = static_cast<int>((tokens + p.ntok - 1) / p.ntok);
  p.f_tiles = static_cast<int>((out_features + kBM - 1) / kBM);
  p.kblocks = n / kBK;
  const long long tiles = static_cast<long long>(p.t_tiles) * p.f_tiles;
  long long k = 1;
  if (tiles < sms) {
    k = (2LL * sms + tiles - 1) / tiles;
    const long long kmax = p.kblocks / 4 > 0 ? p.kblocks / 4 : 1;
    if (k > kmax) k = kmax;
  }
  p.ksplit = static_cast<int>(k);
  p.part_bytes = p.ksplit > 1 ? static_cast<size_t>(tiles) * p.ksplit * kBM * p.ntok * sizeof(float) : 0;
  return p;
}

bool valid_gemm_shape(long long tokens, int n, long long out_features, int bits, int group) {
  if (tokens < 0 || out_features < 0 || n <= 0 || n % kBK != 0 || (bits != 2 && bits != 4)) return false;
  if ((group != 64 && group != 128 && group != 256) || n % group != 0) return false;
  return true;
}

}  // namespace
}  // namespace bq

using namespace bq;

extern "C" size_t bq_w2a16_gemm_workspace_size(int64_t tokens, int32_t n, int64_t out_features) {
  if (tokens <= 0 || out_features <= 0 || n <= 0 || n % kBK != 0) return 0;
  if (dec_applies(tokens, n)) return 0;
  const Plan p = plan_of(tokens, n, out_features, sm_count());
  return p.part_bytes;
}

extern "C" bq_status bq_w2a16_gemm(const void* x, int64_t tokens, int32_t n, const uint8_t* codes,
                                   const uint16_t* scale_f16, const uint16_t* zero_f16, int64_t out_features,
                                   int32_t bits, int32_t group, void* out, bq_dtype out_t, void* workspace,
                                   size_t workspace_bytes, int32_t* status, void* stream) {
  if (!valid_gemm_shape(tokens, n, out_features, bits, group)) return BQ_ERR_INVALID_ARG;
  if (out_t != BQ_F32 && out_t != BQ_BF16) return BQ_ERR_INVALID_ARG;
  if (tokens > 0x7fffffffLL || out_features > 0x7fffffffLL) return BQ_ERR_UNSUPPORTED;
  if (tokens == 0 || out_features == 0) return BQ_OK;
  if (!x || !codes || !scale_f16 || !zero_f16 || !out) return BQ_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(codes)) return BQ_ERR_INVALID_ARG;
  if (workspace && (reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return BQ_ERR_INVALID_ARG;
  if (dec_applies(tokens, n)) {  // decode-sized: warp-level MMAs, weights expanded in registers
    auto st = static_cast<cudaStream_t>(stream);
    const int t = static_cast<int>(tokens), of = static_cast<int>(out_features);
    if (bits == 2)
      return out_t == BQ_BF16 ? run_dec<2, true>(x, t, n, codes, scale_f16, zero_f16, out, of, group, st)
                              : run_dec<2, false>(x, t, n, codes, scale_f16, zero_f16, out, of, group, st);
    return out_t == BQ_BF16 ? run_dec<4, true>(x, t, n, codes, scale_f16, zero_f16, out, of, group, st)
                            : run_dec<4, false>(x, t, n, codes, scale_f16, zero_f16, out, of, group, st);
  }
  const int sms = sm_count();
  Plan p = plan_of(tokens, n, out_features, sms);
  // without a workspace big enough for the split-K partial sums, K is not split
  if (p.ksplit > 1 && (!workspace || workspace_bytes < p.part_bytes)) {
    p.ksplit = 1;
    p.part_bytes = 0;
  }
  const long long units = static_cast<long long>(p.t_tiles) * p.f_tiles * p.ksplit;
  if (units > 0x7fffffffLL) return BQ_ERR_UNSUPPORTED;
  CUtensorMap mx, mc;
  if (!encode_2d(&mx, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, x, static_cast<uint64_t>(n), static_cast<uint64_t>(tokens),
                 static_cast<uint64_t>(n) * 2, kBK, static_cast<uint32_t>(p.ntok), CU_TENSOR_MAP_SWIZZLE_128B))
    return BQ_ERR_UNSUPPORTED;
  const uint64_t row_bytes = static_cast<uint64_t>(n) * bits / 8;
  if (!encode_2d(&mc, CU_TENSOR_MAP_DATA_TYPE_UINT8, codes, row_bytes, static_cast<uint64_t>(out_features), row_bytes,
                 kBK * bits / 8, kBM, CU_TENSOR_MAP_SWIZZLE_NONE))
    return BQ_ERR_UNSUPPORTED;
  GemmArgs a;
  a.scale = scale_f16;
  a.zero = zero_f16;
  a.out = out;
  a.part = p.ksplit > 1 ? static_cast<float*>(workspace) : nullptr;
  a.tokens = static_cast<int>(tokens);
  a.out_features = static_cast<int>(out_features);
  a.n = n;
  a.group = group;
  a.ntok = p.ntok;
  a.npad = p.npad;
  a.idesc = make_idesc(p.ntok);
  a.kblocks = p.kblocks;
  a.ksplit = p.ksplit;
  a.t_tiles = p.t_tiles;
  a.units = static_cast<int>(units);
  a.vec = aligned16(out) && out_features % (out_t == BQ_BF16 ? 8 : 4) == 0;
  a.status = status;
  auto st = static_cast<cudaStream_t>(stream);
  const int grid = units < sms ? static_cast<int>(units) : sms;
  bq_status s;
  if (bits == 2)
    s = out_t == BQ_BF16 ? run_gemm<2, true>(mx, mc, a, grid, st) : run_gemm<2, false>(mx, mc, a, grid, st);
  else
    s = out_t == BQ_BF16 ? run_gemm<4, true>(mx, mc, a, grid, st) : run_gemm<4, false>(mx, mc, a, grid, st);
  if (s != BQ_OK || p.ksplit == 1) return s;
  const long long total = tokens * out_features;
  long long rgrid = (total + 255) / 256;
  if (rgrid > 8LL * sms) rgrid = 8LL * sms;
  if (out_t == BQ_BF16)
    k_splitk_reduce<true><<<static_cast<unsigned>(rgrid), 256, 0, st>>>(a.part, out, a.tokens, a.out_features, a.ntok,
                                                                        a.t_tiles, a.ksplit);
  else
    k_splitk_reduce<false><<<static_cast<unsigned>(rgrid), 256, 0, st>>>(a.part, out, a.tokens, a.out_features,
                                                                         a.ntok, a.t_tiles, a.ksplit);
  return cudaPeekAtLastError() == cudaSuccess ? BQ_OK : BQ_ERR_CUDA;
}

namespace {
size_t act_bytes(int32_t n, int64_t tokens) {
  return (static_cast<size_t>(tokens) * static_cast<size_t>(n) * 2 + 255) & ~static_cast<size_t>(255);
}
}  // namespace

extern "C" size_t bq_w2a16_linear_workspace_size(int32_t n, int64_t tokens, int64_t out_features) {
  if (n <= 0 || tokens < 0 || out_features < 0) return 0;
  return act_bytes(n, tokens) + bq_w2a16_gemm_workspace_size(tokens, n, out_features);
}

extern "C" bq_status bq_w2a16_linear(const bq_layer* layer, const void* x, bq_dtype xt, int64_t tokens,
                                     const uint8_t* codes, const uint16_t* scale_f16, const uint16_t* zero_f16,
                                     int64_t out_features, int32_t bits, int32_t group, void* out, bq_dtype out_t,
                                     void* workspace, size_t workspace_bytes, int32_t* status, void* stream) {
  if (!layer || tokens < 0) return BQ_ERR_INVALID_ARG;
  if (!valid_gemm_shape(tokens, layer->n, out_features, bits, group) || (out_t != BQ_F32 && out_t != BQ_BF16))
    return BQ_ERR_INVALID_ARG;
  if (tokens == 0) return BQ_OK;
  if (!workspace || (reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return BQ_ERR_INVALID_ARG;
  const size_t xb = act_bytes(layer->n, tokens);
  if (workspace_bytes < xb) return BQ_ERR_WORKSPACE;
  const bq_status s = bq_butterfly_fwd(layer, x, xt, workspace, BQ_BF16, tokens, stream);
  if (s != BQ_OK) return s;
  return bq_w2a16_gemm(workspace, tokens, layer->n, codes, scale_f16, zero_f16, out_features, bits, group, out, out_t,
                       static_cast<uint8_t*>(workspace) + xb, workspace_bytes - xb, status, stream);
}
