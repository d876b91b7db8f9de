// Block-wise transform fused with AbsMax block quantization (the WUSH workload;
// WUSH technical summary, section 2 "method" and "implementation"): every block of
// G channels of an activation row gets its own G x G linear transform,
//     y[b G + o] = sum_k T[b][o][k] x[b G + k],
// and the result is quantized per block with a round-to-nearest quantizer whose
// scale comes from the block's absolute maximum: MXFP4 (E2M1 elements, E8M0
// power-of-two scale, G = 32), NVFP4 (E2M1 elements, E4M3 scale, G = 16) or
// symmetric INT4 (fp16 scale, G = 32); or written out unquantized.
//
// Design (B200, sm_100a): the transform is a dense contraction, so it runs on the
// tensor cores.  A work unit is 128 rows x 256 channels, loaded as four
// 64-channel sub-tiles (the last unit of a row may have fewer):
//  * one thread issues the tensor-memory-accelerator copies of each sub-tile's
//    activations (128 x 64 bf16, 128-byte swizzle) and of its blocks'
//    transforms (G x 64 bf16: the prepared table puts the 64 / G blocks of a
//    64-channel tile side by side) into a ring of shared-memory stages;
//  * one thread issues, per block and per 16 channels of K,
//    tcgen05.mma.cta_group::1.kind::f16 (M = 128 rows, N = G outputs, bf16
//    operands from shared memory, fp32 accumulate) into a tensor-memory
//    accumulator (256 columns per unit, two accumulators alternating);
//  * eight (MXFP4) or sixteen (NVFP4, INT4, unquantized output) epilogue warps
//    read the accumulator (thread = row and a half or a quarter of the unit's
//    columns: tcgen05.ld of 32 outputs at a time), compute each block's absolute
//    maximum and scale in registers (a quantization group is one thread's run of
//    G values: no cross-lane reduction) and write its code bytes of the unit with
//    32-byte stores and its scales with one store: the wide unit is what
//    keeps the scale stores few (per-row scale runs of 1 or 2 bytes cost as much
//    store bandwidth as the codes); they convert two values per instruction with
//    cvt.rn.satfinite.e2m1x2.f32 (exact for MXFP4: the division by a power of
//    two is exact; NVFP4 takes the codes of the IEEE float32 quotient by the E4M3
//    scale through a checked reciprocal product) or the exact RTN path of the INT4
//    codes.
// Every barrier wait gives up after one second: the CTA raises its abort flag,
// records the role in the caller's status word and leaves its loop after the
// work already issued has completed; the caller checks the status word.
#include <cuda.h>
#include <cudaTypedefs.h>

#include <mutex>

#include "bq_rtn.cuh"

namespace bq {
namespace {

constexpr int kBM = 128;   // rows per unit (the MMA's M)
constexpr int kBC = 64;    // channels per sub-tile (one 128-byte swizzle row of bf16)
constexpr int kSub = 4;            // sub-tiles per unit
constexpr int kUC = kBC * kSub;    // channels per unit
constexpr int kStages = 6;         // sub-tile stages
constexpr int kAStageBytes = kBM * kBC * 2;  // 16 KB
constexpr int kBStageBytes = 32 * kBC * 2;   // up to G = 32 rows: 4 KB
constexpr int kStageBytes = kAStageBytes + kBStageBytes;
constexpr int kBarOff = kStages * kStageBytes;
constexpr int kSmemBytes = 1024 + kBarOff + 256;  // 1024-byte alignment slack, barriers
static_assert(kSmemBytes <= 227 * 1024, "shared memory per CTA");
static_assert(16 * kStages + 16 + 16 + 8 + 4 + 4 <= 256, "barrier block");
constexpr int kTmemCols = 2 * kUC;                 // two accumulators
static_assert(kTmemCols <= 512 && (kTmemCols & (kTmemCols - 1)) == 0, "tensor memory allocation");
constexpr unsigned long long kWaitLimitNs = 1000000000ull;

// barrier block (byte offsets from kBarOff): a full and an empty barrier per stage,
// a full and an empty barrier per accumulator, the drain barrier, the TMEM slot and
// the abort flag
constexpr int kFull = 0, kEmpty = 8 * kStages, kAccFull = 16 * kStages, kAccEmpty = kAccFull + 16,
              kDrain = kAccEmpty + 16, kTmemSlot = kDrain + 8, kAbort = kTmemSlot + 4;
constexpr int kStTma = 1, kStMma = 2, kStEpi = 4, kStDrain = 8;

enum Format { kNone = 0, kMxfp4 = 1, kNvfp4 = 2, kInt4 = 3 };

// Epilogue shape per format: warps per TMEM lane quarter (each takes kUC / parts
// columns of a unit).  MXFP4's codes are cheap (a power-of-two scale, one conversion
// per two values): two warps per quarter keep up and leave the smaller CTA; the
// NVFP4 and INT4 epilogues do more arithmetic per value, and the unquantized output
// more stores, and take four.
template <int FMT>
struct Epi {
  static constexpr int kParts = FMT == kMxfp4 ? 2 : 4;
  static constexpr int kWarps = 4 * kParts;
  static constexpr int kCols = kUC / kParts;        // columns of a unit per epilogue thread
  static constexpr int kChunks = kCols / 32;        // tcgen05.ld of 32 columns each
  static constexpr int kThreads = 32 * (kWarps + 2);  // epilogue warps, TMA warp, MMA warp
  static_assert(kChunks >= 1 && kCols % 32 == 0, "epilogue columns");
};

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

// Waits for the phase of `parity`; false when the abort flag is up or the wait ran
// out (then it raises the flag and records `code` in the status word).
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

// A wait for work already issued (ignores the abort flag), still bounded.
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

// 2D tiled copy global -> shared, completing on an mbarrier (no multicast)
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

// instruction descriptor: fp32 accumulate, bf16 A and B, both K-major, M = 128, N = n
__host__ __device__ constexpr uint32_t make_idesc(int n) {
  return (1u << 4) | (1u << 7) | (1u << 10) | (uint32_t(n >> 3) << 17) | (uint32_t(kBM >> 4) << 24);
}

// D (tensor memory) (+)= A (shared memory) x B (shared memory)
__device__ __forceinline__ void umma_ss(uint32_t d, uint64_t a, uint64_t b, uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n"
      " tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n}"
      ::"r"(d), "l"(a), "l"(b), "r"(idesc), "r"(accumulate)
      : "memory");
}

__device__ __forceinline__ void umma_commit(uint32_t bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar) : "memory");
}

__device__ __forceinline__ void tmem_ld32(uint32_t addr, float (&r)[32]) {
  uint32_t (&u)[32] = reinterpret_cast<uint32_t (&)[32]>(r);
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
      : "=r"(u[0]), "=r"(u[1]), "=r"(u[2]), "=r"(u[3]), "=r"(u[4]), "=r"(u[5]), "=r"(u[6]), "=r"(u[7]),
        "=r"(u[8]), "=r"(u[9]), "=r"(u[10]), "=r"(u[11]), "=r"(u[12]), "=r"(u[13]), "=r"(u[14]), "=r"(u[15]),
        "=r"(u[16]), "=r"(u[17]), "=r"(u[18]), "=r"(u[19]), "=r"(u[20]), "=r"(u[21]), "=r"(u[22]), "=r"(u[23]),
        "=r"(u[24]), "=r"(u[25]), "=r"(u[26]), "=r"(u[27]), "=r"(u[28]), "=r"(u[29]), "=r"(u[30]), "=r"(u[31])
      : "r"(addr));
}

__device__ __forceinline__ void tmem_wait_ld1(float (&a)[32]) {
  uint32_t (&u)[32] = reinterpret_cast<uint32_t (&)[32]>(a);
  asm volatile("tcgen05.wait::ld.sync.aligned;"
               : "+r"(u[0]), "+r"(u[1]), "+r"(u[2]), "+r"(u[3]), "+r"(u[4]), "+r"(u[5]), "+r"(u[6]), "+r"(u[7]),
                 "+r"(u[8]), "+r"(u[9]), "+r"(u[10]), "+r"(u[11]), "+r"(u[12]), "+r"(u[13]), "+r"(u[14]),
                 "+r"(u[15]), "+r"(u[16]), "+r"(u[17]), "+r"(u[18]), "+r"(u[19]), "+r"(u[20]), "+r"(u[21]),
                 "+r"(u[22]), "+r"(u[23]), "+r"(u[24]), "+r"(u[25]), "+r"(u[26]), "+r"(u[27]), "+r"(u[28]),
                 "+r"(u[29]), "+r"(u[30]), "+r"(u[31])
               :
               : "memory");
}

// 32-byte store (one full L2 sector); p 32-byte aligned
__device__ __forceinline__ void st_global_32B(void* p, const uint4& a, const uint4& b) {
  asm volatile("st.global.v8.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};" ::"l"(p), "r"(a.x), "r"(a.y), "r"(a.z),
               "r"(a.w), "r"(b.x), "r"(b.y), "r"(b.z), "r"(b.w)
               : "memory");
}

// keeps the registers of a chunk loaded before the preceding wait::ld from being
// read earlier (the wait itself is issued once, by tmem_wait_ld1)
__device__ __forceinline__ void tmem_bind(float (&a)[32]) {
  uint32_t (&u)[32] = reinterpret_cast<uint32_t (&)[32]>(a);
  asm volatile(""
               : "+r"(u[0]), "+r"(u[1]), "+r"(u[2]), "+r"(u[3]), "+r"(u[4]), "+r"(u[5]), "+r"(u[6]), "+r"(u[7]),
                 "+r"(u[8]), "+r"(u[9]), "+r"(u[10]), "+r"(u[11]), "+r"(u[12]), "+r"(u[13]), "+r"(u[14]),
                 "+r"(u[15]), "+r"(u[16]), "+r"(u[17]), "+r"(u[18]), "+r"(u[19]), "+r"(u[20]), "+r"(u[21]),
                 "+r"(u[22]), "+r"(u[23]), "+r"(u[24]), "+r"(u[25]), "+r"(u[26]), "+r"(u[27]), "+r"(u[28]),
                 "+r"(u[29]), "+r"(u[30]), "+r"(u[31])
               :
               : "memory");
}

// two float32 -> one byte of two E2M1 codes (hi in bits 4..7), round to nearest even,
// saturating at +-6
__device__ __forceinline__ uint32_t e2m1x2(float hi, float lo) {
  uint16_t d;
  asm("{\n .reg .b8 t;\n cvt.rn.satfinite.e2m1x2.f32 t, %1, %2;\n cvt.u16.u8 %0, t;\n}" : "=h"(d) : "f"(hi), "f"(lo));
  return d;
}

// float32 -> FP8 E4M3 byte (round to nearest even, saturating at +-448)
__device__ __forceinline__ uint32_t e4m3_byte(float v) {
  uint16_t d;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(d) : "f"(0.f), "f"(v));
  return d & 0xffu;
}

// FP8 E4M3 byte -> float32 (exact)
__device__ __forceinline__ float e4m3_value(uint32_t byte) {
  uint32_t h2;
  const uint16_t in = static_cast<uint16_t>(byte);
  asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h2) : "h"(in));
  return __half2float(__ushort_as_half(static_cast<uint16_t>(h2 & 0xffffu)));
}

// eight float32 -> four bytes of E2M1 code pairs (element 2k in the low nibble of
// byte k), round to nearest even, saturating at +-6
__device__ __forceinline__ uint32_t e2m1x8(float2 a, float2 b, float2 c, float2 d) {
  uint32_t w;
  asm("{\n .reg .b8 b0, b1, b2, b3;\n"
      " cvt.rn.satfinite.e2m1x2.f32 b0, %2, %1;\n"
      " cvt.rn.satfinite.e2m1x2.f32 b1, %4, %3;\n"
      " cvt.rn.satfinite.e2m1x2.f32 b2, %6, %5;\n"
      " cvt.rn.satfinite.e2m1x2.f32 b3, %8, %7;\n"
      " mov.b32 %0, {b0, b1, b2, b3};\n}"
      : "=r"(w)
      : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y), "f"(c.x), "f"(c.y), "f"(d.x), "f"(d.y));
  return w;
}

__device__ __forceinline__ float max3f(float a, float b, float c) {
  float d;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}

// largest |v[k]| of N values (N even, N >= 8): three-input maxima in two chains
template <int N>
__device__ __forceinline__ float absmax(const float* v) {
  float m0 = max3f(fabsf(v[0]), fabsf(v[1]), fabsf(v[2]));
  float m1 = max3f(fabsf(v[3]), fabsf(v[4]), fabsf(v[5]));
  int k = 6;
#pragma unroll
  for (; k + 4 <= N; k += 4) {
    m0 = max3f(m0, fabsf(v[k]), fabsf(v[k + 1]));
    m1 = max3f(m1, fabsf(v[k + 2]), fabsf(v[k + 3]));
  }
#pragma unroll
  for (; k < N; k += 2) m0 = max3f(m0, fabsf(v[k]), fabsf(v[k + 1]));
  return fmaxf(m0, m1);
}

// ------------------------------------------------------------------ epilogue: one row's 64 outputs

struct BlkArgs {
  int rows, C, G;
  int col_tiles, col_units, units;  // 64-channel sub-tiles, units per row tile, all units
  float gscale;           // NVFP4 per-tensor scale
  void* y;                // kNone: [rows][C] float32 or bf16
  int y_bf16;
  uint8_t* codes;         // [rows][C / 2]
  void* scales;           // [rows][C / G]: bytes (MXFP4, NVFP4) or fp16 bits (INT4)
  int32_t* status;
  uint32_t idesc;
};

// MXFP4: 32 values -> 16 code bytes and the E8M0 scale byte.
__device__ __forceinline__ void quant_mxfp4(const float* v, uint4& codes, uint32_t& scale) {
  const float amax = absmax<32>(v);
  const int biased = static_cast<int>((__float_as_uint(amax) >> 23) & 0xffu);
  const int X = biased - 129 > -127 ? biased - 129 : -127;   // floor(log2 amax) - 2, at least -127
  scale = static_cast<uint32_t>(X + 127);
  const float inv = __uint_as_float(static_cast<uint32_t>(127 - X) << 23);  // 2^-X, exact
  const float2 iv = make_float2(inv, inv);
  uint32_t w[4];
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    const float* p = v + 8 * q;
    w[q] = e2m1x8(__fmul2_rn(make_float2(p[0], p[1]), iv), __fmul2_rn(make_float2(p[2], p[3]), iv),
                  __fmul2_rn(make_float2(p[4], p[5]), iv), __fmul2_rn(make_float2(p[6], p[7]), iv));
  }
  codes = make_uint4(w[0], w[1], w[2], w[3]);
}

// NVFP4: 16 values -> 8 code bytes and the E4M3 scale byte.  The codes are those of
// RN32(y / den).  Fast path: q = RN32(y * RN32(1 / den)) is within 1.5 ulp of the
// correctly rounded quotient (two roundings of relative size 2^-24 each), so when
// q (1 - 2^-20) and q (1 + 2^-20) receive the same E2M1 code, that code -- the code is
// monotone in the value -- is also the code of RN32(y / den); elements where the two
// differ (a quotient within about 2^-20 relative of a rounding boundary of the E2M1
// grid), and groups whose den or quotients leave the range where those error bounds
// hold, take IEEE division.
__device__ __forceinline__ void quant_nvfp4(const float* v, float gscale, uint2& codes, uint32_t& scale) {
  const float amax = absmax<16>(v);
  scale = e4m3_byte(__fdiv_rn(amax, 6.f));
  const float den = __fmul_rn(e4m3_value(scale), gscale);
  if (den == 0.f) {
    codes = make_uint2(0u, 0u);
    return;
  }
  const float r = __frcp_rn(den);
  bool ok = den >= 0x1p-100f && den <= 0x1p100f && amax * r < 0x1p100f;
  const float2 up = make_float2(1.00000095367431640625f, 1.00000095367431640625f);   // 1 + 2^-20
  const float2 dn = make_float2(0.99999904632568359375f, 0.99999904632568359375f);   // 1 - 2^-20
  const float2 r2 = make_float2(r, r);
  uint32_t w[2];
#pragma unroll
  for (int q = 0; q < 2; ++q) {
    float2 qu[4], qd[4];
#pragma unroll
    for (int b = 0; b < 4; ++b) {
      const float2 qv = __fmul2_rn(make_float2(v[8 * q + 2 * b], v[8 * q + 2 * b + 1]), r2);
      qu[b] = __fmul2_rn(qv, up);
      qd[b] = __fmul2_rn(qv, dn);
    }
    w[q] = e2m1x8(qu[0], qu[1], qu[2], qu[3]);
    ok = ok && w[q] == e2m1x8(qd[0], qd[1], qd[2], qd[3]);
  }
  if (!ok) {
#pragma unroll
    for (int q = 0; q < 2; ++q) {
      uint32_t word = 0;
#pragma unroll
      for (int b = 0; b < 4; ++b) {
        const int k = 8 * q + 2 * b;
        word |= e2m1x2(__fdiv_rn(v[k + 1], den), __fdiv_rn(v[k], den)) << (8 * b);
      }
      w[q] = word;
    }
  }
  codes = make_uint2(w[0], w[1]);
}

// Symmetric INT4 codes of 32 values (two's complement nibbles, lowest element in the
// lowest bits): rint(y / s) as in the exact RTN path of the asymmetric quantizer, with
// the offset 8 (codes 1..15 for -7..7; XOR 8 gives the nibble).  y * inv + (1.5 2^23 + 8)
// rounds to the integer rint(y inv) + 8 in the low mantissa bits; the residual
// e = rint - y inv, taken with one rounding, shows how far y inv is from a tie.  The
// group takes IEEE division and clamping when a residual comes within the error bound
// of the product of a tie, or the group's extreme lands outside [-7, 7].
__device__ __forceinline__ void quant_int4(const float* v, uint4& codes, uint32_t& scale16) {
  const float amax = absmax<32>(v);
  __half h16 = __float2half_rn(__fdiv_rn(amax, 7.f));
  float s = __half2float(h16);
  if (amax == 0.f || s == 0.f) {
    s = 1.f;
    h16 = __float2half_rn(1.f);
  }
  scale16 = __half_as_ushort(h16);
  const float inv = __frcp_rn(s);
  const float vmax = amax * inv * 1.000001f;
  float thr = vmax < 4194304.f ? 0.5f - vmax * 9.5367431640625e-7f : -1.f;  // 2^22, 2^-20
  // |y| <= amax: no code leaves [-7, 7] when rint(amax / s) <= 7
  if (!(rintf(__fdiv_rn(amax, s)) <= 7.f)) thr = -1.f;
  const float2 iv = make_float2(inv, inv), niv = make_float2(-inv, -inv);
  const float2 m2 = make_float2(12582920.f, 12582920.f);   // 1.5 * 2^23 + 8
  const float2 nm2 = make_float2(-12582920.f, -12582920.f);
  float emax = 0.f;
  uint32_t w[4];
#pragma unroll
  for (int g = 0; g < 4; ++g) {
    uint32_t b[8];
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const float2 yv = make_float2(v[8 * g + 2 * q], v[8 * g + 2 * q + 1]);
      const float2 t = __ffma2_rn(yv, iv, m2);
      const float2 rr = __fadd2_rn(t, nm2);
      const float2 e = __ffma2_rn(yv, niv, rr);
      emax = max_nan3(emax, fabsf(e.x), fabsf(e.y));
      b[2 * q] = __float_as_uint(t.x);
      b[2 * q + 1] = __float_as_uint(t.y);
    }
    // low byte of t = rint + 8 in 1..15: two codes per byte, then the four bytes
    const uint32_t p0 = b[0] + (b[1] << 4), p1 = b[2] + (b[3] << 4);
    const uint32_t p2 = b[4] + (b[5] << 4), p3 = b[6] + (b[7] << 4);
    w[g] = __byte_perm(__byte_perm(p0, p1, 0x0040), __byte_perm(p2, p3, 0x0040), 0x5410) ^ 0x88888888u;
  }
  if (!(emax < thr)) {
#pragma unroll
    for (int g = 0; g < 4; ++g) {
      uint32_t word = 0;
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        const float t = fminf(fmaxf(rintf(__fdiv_rn(v[8 * g + e], s)), -7.f), 7.f);
        word |= (static_cast<uint32_t>(static_cast<int>(t)) & 0xfu) << (4 * e);
      }
      w[g] = word;
    }
  }
  codes = make_uint4(w[0], w[1], w[2], w[3]);
}

// 32 outputs -> 16 code bytes and their scales: one byte (MXFP4), two bytes (NVFP4:
// two groups of 16) or the fp16 bits (INT4)
template <int FMT>
__device__ __forceinline__ void chunk_quant(const float* v, float gscale, uint4& codes, uint32_t& scales) {
  if constexpr (FMT == kMxfp4) {
    quant_mxfp4(v, codes, scales);
  } else if constexpr (FMT == kNvfp4) {
    uint2 c0, c1;
    uint32_t s0, s1;
    quant_nvfp4(v, gscale, c0, s0);
    quant_nvfp4(v + 16, gscale, c1, s1);
    codes = make_uint4(c0.x, c0.y, c1.x, c1.y);
    scales = s0 | (s1 << 8);
  } else {
    quant_int4(v, codes, scales);
  }
}

// One row's outputs c0 .. c0 + 32 nch - 1 (v[c] holds c0 + 32 c ..), nch <= kChunks.
template <int FMT, int G, int kChunks>
__device__ __forceinline__ void epilogue_part(const BlkArgs& a, long long row, int c0, float (&v)[kChunks][32],
                                              int nch) {
  if constexpr (FMT == kNone) {
#pragma unroll
    for (int c = 0; c < kChunks; ++c) {
      if (c >= nch) break;
      if (a.y_bf16) {
        uint4* dst = reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(a.y) + row * a.C + c0 + 32 * c);
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          uint32_t w[4];
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            __nv_bfloat162 h = __floats2bfloat162_rn(v[c][8 * q + 2 * k], v[c][8 * q + 2 * k + 1]);
            w[k] = *reinterpret_cast<uint32_t*>(&h);
          }
          dst[q] = make_uint4(w[0], w[1], w[2], w[3]);
        }
      } else {
        float4* dst = reinterpret_cast<float4*>(static_cast<float*>(a.y) + row * a.C + c0 + 32 * c);
#pragma unroll
        for (int q = 0; q < 8; ++q)
          dst[q] = make_float4(v[c][4 * q], v[c][4 * q + 1], v[c][4 * q + 2], v[c][4 * q + 3]);
      }
    }
  } else {
    constexpr int kSb = FMT == kMxfp4 ? 1 : 2;   // scale bytes per 32 outputs
    constexpr int kBytes = kSb * kChunks;
    uint4* crow = reinterpret_cast<uint4*>(a.codes + row * (a.C / 2) + c0 / 2);
    uint8_t* sp = static_cast<uint8_t*>(a.scales) + (row * (a.C / G) + c0 / G) * (FMT == kInt4 ? 2 : 1);
    uint64_t sc = 0;
    uint4 q[kChunks];
#pragma unroll
    for (int c = 0; c < kChunks; ++c) {
      if (c >= nch) break;
      uint32_t s;
      chunk_quant<FMT>(v[c], a.gscale, q[c], s);
      sc |= static_cast<uint64_t>(s) << (8 * kSb * c);
    }
    // codes: 32-byte stores (whole sectors) where the run allows
    const bool wide = (reinterpret_cast<uintptr_t>(crow) & 31u) == 0;
#pragma unroll
    for (int c = 0; c < kChunks; c += 2) {
      if (c >= nch) break;
      if (c + 1 < nch && wide) {
        st_global_32B(crow + c, q[c], q[c + 1]);
      } else {
        crow[c] = q[c];
        if (c + 1 < nch) crow[c + 1] = q[c + 1];
      }
    }
    if (nch == kChunks && (reinterpret_cast<uintptr_t>(sp) & (kBytes - 1)) == 0) {
      if constexpr (kBytes == 8) *reinterpret_cast<uint64_t*>(sp) = sc;
      else if constexpr (kBytes == 4) *reinterpret_cast<uint32_t*>(sp) = static_cast<uint32_t>(sc);
      else if constexpr (kBytes == 2) *reinterpret_cast<uint16_t*>(sp) = static_cast<uint16_t>(sc);
      else *sp = static_cast<uint8_t>(sc);
    } else {
#pragma unroll
      for (int c = 0; c < kChunks; ++c) {
        if (c >= nch) break;
        if constexpr (kSb == 1) sp[c] = static_cast<uint8_t>(sc >> (8 * c));
        else reinterpret_cast<uint16_t*>(sp)[c] = static_cast<uint16_t>(sc >> (16 * c));
      }
    }
  }
}

template <int FMT, int G>
__global__ void __launch_bounds__(Epi<FMT>::kThreads, 1)
    k_blockq(const __grid_constant__ CUtensorMap map_x, const __grid_constant__ CUtensorMap map_t, const BlkArgs args) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* gbase = smem_raw + (base - raw);
  const uint32_t bars = base + kBarOff;
  volatile int* abort_flag = reinterpret_cast<volatile int*>(gbase + kBarOff + kAbort);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(gbase + kBarOff + kTmemSlot);
  using E = Epi<FMT>;
  constexpr int kTmaWarp = E::kWarps, kMmaWarp = E::kWarps + 1;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int row_tiles = (args.rows + kBM - 1) / kBM;
  constexpr uint32_t kTx = kAStageBytes + G * kBC * 2;  // bytes a stage's two copies deliver

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(bars + kFull + 8 * s, 1);
      mbar_init(bars + kEmpty + 8 * s, 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(bars + kAccFull + 8 * a, 1);
      mbar_init(bars + kAccEmpty + 8 * a, 32 * E::kWarps);
    }
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
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&map_t)) : "memory");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == kTmaWarp) {
    // ---------------------------------------------------------------- loads
    if (lane == 0) {
      uint32_t s = 0, par = 0, issued = 0, last_parity = 0;
      bool stop = false;
      for (int u = blockIdx.x; u < args.units && !stop; u += gridDim.x) {
        const int rt = u % row_tiles, cu = u / row_tiles;
        const int nsub = min(kSub, args.col_tiles - kSub * cu);
        for (int j = 0; j < nsub; ++j) {
          if (!wait_bar(bars + kEmpty + 8 * s, par ^ 1u, abort_flag, args.status, kStTma)) {
            stop = true;
            break;
          }
          const int ct = kSub * cu + j;
          const uint32_t st = base + s * kStageBytes;
          mbar_expect_tx(bars + kFull + 8 * s, kTx);
          tma_2d(st, &map_x, ct * kBC, rt * kBM, bars + kFull + 8 * s);
          tma_2d(st + kAStageBytes, &map_t, 0, ct * G, bars + kFull + 8 * s);
          issued |= 1u << s;
          last_parity = (last_parity & ~(1u << s)) | (par << s);
          if (++s == kStages) {
            s = 0;
            par ^= 1u;
          }
        }
      }
      // copies still in flight land before the CTA exits
      for (int s2 = 0; s2 < kStages; ++s2)
        if ((issued >> s2) & 1u) wait_bar_drain(bars + kFull + 8 * s2, (last_parity >> s2) & 1u, args.status);
    }
    __syncwarp();
  } else if (warp == kMmaWarp) {
    // ---------------------------------------------------------------- MMA issue
    if (lane == 0) {
      uint32_t s = 0, par = 0;
      int i = 0;
      bool stop = false;
      for (int u = blockIdx.x; u < args.units && !stop; u += gridDim.x, ++i) {
        const int acc = i & 1;
        if (!wait_bar(bars + kAccEmpty + 8 * acc, ((i >> 1) & 1) ^ 1, abort_flag, args.status, kStMma)) break;
        const int nsub = min(kSub, args.col_tiles - kSub * (u / row_tiles));
        for (int j = 0; j < nsub; ++j) {
          if (!wait_bar(bars + kFull + 8 * s, par, abort_flag, args.status, kStMma)) {
            stop = true;
            break;
          }
          tc_fence_after();
          const uint32_t st = base + s * kStageBytes;
          const uint64_t ad = sw128_desc(st), bd = sw128_desc(st + kAStageBytes);
          const uint32_t d0 = tmem + static_cast<uint32_t>(kUC * acc + kBC * j);
#pragma unroll
          for (int b = 0; b < kBC / G; ++b) {
#pragma unroll
            for (int kk = 0; kk < G / 16; ++kk) {
              const uint64_t koff = static_cast<uint64_t>((b * G + 16 * kk) * 2 / 16);  // +32 bytes per 16 of K
              umma_ss(d0 + static_cast<uint32_t>(b * G), ad + koff, bd + koff, args.idesc, kk > 0 ? 1u : 0u);
            }
          }
          umma_commit(bars + kEmpty + 8 * s);
          if (++s == kStages) {
            s = 0;
            par ^= 1u;
          }
        }
        if (stop) break;
        umma_commit(bars + kAccFull + 8 * acc);
      }
      // every MMA issued has completed before the tensor memory is freed
      umma_commit(bars + kDrain);
      wait_bar_drain(bars + kDrain, 0, args.status);
    }
    __syncwarp();
  } else {
    // ---------------------------------------------------------------- epilogue
    // warp w: rows 32 (w & 3) .. + 31 (its TMEM lane quarter), the unit's columns
    // E::kCols (w >> 2) .. + E::kCols - 1
    const uint32_t lane_base = static_cast<uint32_t>(32 * (warp & 3)) << 16;
    const int part = warp >> 2;
    int i = 0;
    for (int u = blockIdx.x; u < args.units; u += gridDim.x, ++i) {
      const int acc = i & 1;
      if (!wait_bar(bars + kAccFull + 8 * acc, (i >> 1) & 1, abort_flag, args.status, kStEpi)) break;
      tc_fence_after();
      const int rt = u % row_tiles, cu = u / row_tiles;
      const int valid = kBC * min(kSub, args.col_tiles - kSub * cu) - E::kCols * part;  // warp-uniform
      const int nch = valid <= 0 ? 0 : min(E::kChunks, valid / 32);
      float v[E::kChunks][32];
      const uint32_t t0 = tmem + lane_base + static_cast<uint32_t>(kUC * acc + E::kCols * part);
#pragma unroll
      for (int c = 0; c < E::kChunks; ++c)
        if (c < nch) tmem_ld32(t0 + 32 * c, v[c]);
      tmem_wait_ld1(v[0]);
#pragma unroll
      for (int c = 1; c < E::kChunks; ++c) tmem_bind(v[c]);
      tc_fence_before();
      mbar_arrive(bars + kAccEmpty + 8 * acc);
      const long long row = static_cast<long long>(rt) * kBM + 32 * (warp & 3) + lane;
      if (row < args.rows && nch > 0) epilogue_part<FMT, G, E::kChunks>(args, row, kUC * cu + E::kCols * part, v, nch);
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == kMmaWarp) {
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kTmemCols) : "memory");
  }
}

// Prepared table: the blocks of each 64-channel tile side by side,
//   P[tile][o][c] = T[(64 tile + c) / G][o][(64 tile + c) % G]   (bf16, [C / 64][G][64]),
// so that one 2D tile copy brings the G x 64 B operand of a unit.
__global__ void k_blockq_prepare(const uint16_t* __restrict__ T, uint16_t* __restrict__ P, int C, int G) {
  const long long total = static_cast<long long>(C / kBC) * G * kBC;
  for (long long i = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; i < total;
       i += static_cast<long long>(gridDim.x) * blockDim.x) {
    const int c = static_cast<int>(i % kBC);
    const int o = static_cast<int>((i / kBC) % G);
    const long long tile = i / (static_cast<long long>(kBC) * G);
    const long long ch = tile * kBC + c;
    const long long b = ch / G;
    const int k = static_cast<int>(ch % G);
    P[i] = T[(b * G + o) * G + k];
  }
}

// ------------------------------------------------------------------ host side

PFN_cuTensorMapEncodeTiled_v12000 encoder() {
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

bool encode_bf16_2d(CUtensorMap* map, const void* ptr, uint64_t inner, uint64_t outer, uint32_t box_outer) {
  const PFN_cuTensorMapEncodeTiled_v12000 fn = encoder();
  if (!fn) return false;
  const cuuint64_t dims[2] = {inner, outer};
  const cuuint64_t strides[1] = {inner * 2};
  const cuuint32_t box[2] = {static_cast<cuuint32_t>(kBC), box_outer};
  const cuuint32_t elem[2] = {1, 1};
  return fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(ptr), dims, strides, box, elem,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int FMT, int G>
bq_status run(const CUtensorMap& mx, const CUtensorMap& mt, const BlkArgs& a, int grid, cudaStream_t st) {
  auto kern = k_blockq<FMT, G>;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return BQ_ERR_CUDA;
  static std::atomic<int> ready[kMaxDevices];
  if (!once_per_device(ready, dev, [&] {
        return cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes) == cudaSuccess;
      }))
    return BQ_ERR_CUDA;
  kern<<<grid, Epi<FMT>::kThreads, kSmemBytes, st>>>(mx, mt, a);
  return cudaPeekAtLastError() == cudaSuccess ? BQ_OK : BQ_ERR_CUDA;
}

int group_of(bq_block_format f, int G) {
  switch (f) {
    case BQ_BLOCK_MXFP4: return 32;
    case BQ_BLOCK_NVFP4: return 16;
    case BQ_BLOCK_INT4: return 32;
    case BQ_BLOCK_NONE: return G == 16 || G == 32 ? G : 0;
  }
  return 0;
}

}  // namespace
}  // namespace bq

using namespace bq;

extern "C" size_t bq_block_table_bytes(int32_t C, int32_t G) {
  if ((G != 16 && G != 32) || C <= 0 || C % kBC != 0) return 0;
  return static_cast<size_t>(C) * G * 2;
}

extern "C" bq_status bq_block_prepare(const uint16_t* T, int32_t C, int32_t G, uint16_t* table, void* stream) {
  if (bq_block_table_bytes(C, G) == 0 || !T || !table || !aligned16(table) ||
      (reinterpret_cast<uintptr_t>(T) & 1u))
    return BQ_ERR_INVALID_ARG;
  const long long total = static_cast<long long>(C) * G;
  long long grid = (total + 255) / 256;
  if (grid > 4096) grid = 4096;
  k_blockq_prepare<<<static_cast<unsigned>(grid), 256, 0, static_cast<cudaStream_t>(stream)>>>(T, table, C, G);
  return cudaPeekAtLastError() == cudaSuccess ? BQ_OK : BQ_ERR_CUDA;
}

extern "C" bq_status bq_block_transform_quantize(const uint16_t* table, int32_t C, int32_t G, const void* x,
                                                 int64_t rows, bq_block_format format, float gscale, void* y,
                                                 bq_dtype yt, uint8_t* codes, void* scales, int32_t* status,
                                                 void* stream) {
  if (bq_block_table_bytes(C, G) == 0 || group_of(format, G) != G) return BQ_ERR_INVALID_ARG;
  if (rows < 0 || rows > 0x7fffffffLL) return rows < 0 ? BQ_ERR_INVALID_ARG : BQ_ERR_UNSUPPORTED;
  if (rows == 0) return BQ_OK;
  if (!table || !x || !aligned16(table) || !aligned16(x)) return BQ_ERR_INVALID_ARG;
  if (format == BQ_BLOCK_NONE) {
    if (!y || !aligned16(y) || (yt != BQ_F32 && yt != BQ_BF16)) return BQ_ERR_INVALID_ARG;
  } else {
    if (!codes || !scales || !aligned16(codes) || (reinterpret_cast<uintptr_t>(scales) & 1u)) return BQ_ERR_INVALID_ARG;
    if (format == BQ_BLOCK_NVFP4 && !(gscale > 0.f && gscale < 3.0e38f)) return BQ_ERR_INVALID_ARG;
  }
  CUtensorMap mx, mt;
  if (!encode_bf16_2d(&mx, x, static_cast<uint64_t>(C), static_cast<uint64_t>(rows), kBM) ||
      !encode_bf16_2d(&mt, table, kBC, static_cast<uint64_t>(C / kBC) * G, static_cast<uint32_t>(G)))
    return BQ_ERR_UNSUPPORTED;
  BlkArgs a;
  a.rows = static_cast<int>(rows);
  a.C = C;
  a.G = G;
  a.col_tiles = C / kBC;
  a.col_units = (a.col_tiles + kSub - 1) / kSub;
  const long long units = ((rows + kBM - 1) / kBM) * static_cast<long long>(a.col_units);
  if (units > 0x7fffffffLL) return BQ_ERR_UNSUPPORTED;
  a.units = static_cast<int>(units);
  a.gscale = gscale;
  a.y = y;
  a.y_bf16 = yt == BQ_BF16;
  a.codes = codes;
  a.scales = scales;
  a.status = status;
  a.idesc = make_idesc(G);
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return BQ_ERR_CUDA;
  const int sms = device_sm_count(dev);
  if (sms <= 0) return BQ_ERR_CUDA;
  const int grid = a.units < sms ? a.units : sms;
  auto st = static_cast<cudaStream_t>(stream);
  switch (format) {
    case BQ_BLOCK_MXFP4: return run<kMxfp4, 32>(mx, mt, a, grid, st);
    case BQ_BLOCK_NVFP4: return run<kNvfp4, 16>(mx, mt, a, grid, st);
    case BQ_BLOCK_INT4: return run<kInt4, 32>(mx, mt, a, grid, st);
    case BQ_BLOCK_NONE: return G == 16 ? run<kNone, 16>(mx, mt, a, grid, st) : run<kNone, 32>(mx, mt, a, grid, st);
  }
  return BQ_ERR_INVALID_ARG;
}
