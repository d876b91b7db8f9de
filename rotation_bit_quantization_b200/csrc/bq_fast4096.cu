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
//    layouts); only B -> C crosses the row group's warps.  Pass C's
//    layout keeps 8 consecutive positions per thread, so the RTN epilogue
//    (group statistics, packing, coalesced stores) runs in place without a
//    third transpose.
//  * The B -> C exchange is a split barrier (an mbarrier per buffer): a
//    thread arrives after writing its part of row j and waits for row j's
//    phase only in the next iteration, after row j + 1's pass A, which parks
//    in the warp's A -> B buffer meanwhile; so the warps of a row group need
//    not meet at the exchange.  Waits are bounded (bq_wait_faults).
//  * Rotations use the scaled two-FMA form prepared by bq_precompute_cs
//    (a_i += alpha a_j, a_j += beta a_i; outputs times sigma), issued as packed
//    fma.rn.f32x2 where two pairs sit in adjacent registers; when the layer's
//    scaled form is out of range (table header flag 0) the same kernel runs the
//    plain cos/sin rotation instead.
//  * One CTA per SM (all 512 TMEM columns) with kSlots row groups sharing the
//    tensor-memory image (warps w, w + 4, ... use the same lanes); each thread
//    reads the next stage's coefficients while it computes the current one
//    (kDoubleBuf) and the next row's input is prefetched into registers.
//  * Programmatic dependent launch: both kernels are launched with programmatic
//    stream serialization and let their dependents launch as soon as they start,
//    so a launch's CTAs take SMs as the previous launch's CTAs leave them and do
//    their set-up (mbarriers, TMEM allocation) meanwhile.  griddepcontrol.wait
//    comes before the first global-memory access of any thread (input prefetch,
//    coefficient image, table header, outputs), so every read sees the previous
//    kernel's writes and no write lands before that kernel has finished reading.
#include <cfloat>

#include "bq_rtn.cuh"

namespace bq {
namespace {

constexpr int M = 4096;
constexpr int kGroupThreads = 128;
constexpr int kColB = 160, kColC = 320, kColS = 384;
constexpr int kFillChunks = kImageCols / 16;  // 26 chunks of 16 columns

// forward kernel: kSlots row groups, each with an A -> B buffer, two alternating
// B -> C buffers and the epilogue's parameter slots (the inverse's buffers below)
// Three row groups with double-buffered coefficient loads (168 registers) and four
// with single-buffered loads (128 registers) measured the same at 16384 rows; three
// were 6% faster at 2048 rows and for the inverse.
constexpr int kSlots = 3;
constexpr bool kDoubleBuf = true;
constexpr int kThreads = kSlots * kGroupThreads;
constexpr int kBufFloats = M;
constexpr int kParamFloats = 4 * 32 * 4;  // 4 warps x 32 slots x float4
constexpr int kSlotFloats = 3 * kBufFloats + kParamFloats;
constexpr int kFwdSmemBytes = kSlots * kSlotFloats * static_cast<int>(sizeof(float));
static_assert(kFwdSmemBytes <= 227 * 1024, "shared memory per CTA");
// the inverse: per row group one B -> A buffer and kInvBufs rotating C -> B buffers
constexpr int kInvBufs = 3;
constexpr int kInvSlotFloats = (1 + kInvBufs) * kBufFloats;
constexpr int kInvSmemBytes = kSlots * kInvSlotFloats * static_cast<int>(sizeof(float));
static_assert(kInvSmemBytes <= 227 * 1024, "shared memory per CTA");
// image chunks a thread loads per round of the start-up fill: all of its chunks at
// once where registers allow (three row groups: 9 chunks, 144 registers), four at a
// time with more row groups
constexpr int kFillRound = kSlots >= 4 ? 4 : (kFillChunks + kSlots - 1) / kSlots;

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


__device__ __forceinline__ float u2f(uint32_t v) { return __uint_as_float(v); }

// ------------------------------------------------------------------ row-group barriers
//
// The forward's B -> C exchange uses a split barrier: every thread of the row
// group arrives on the buffer's mbarrier after writing its part of a row, and
// waits for that phase only when it comes to read the row, with the next row's
// first pass in between.  A wait gives up after one second and records it in the
// library's wait-fault word (read and cleared by bq_wait_faults), so that no
// failure can hold the SM.

constexpr unsigned long long kWaitLimitNs = 1000000000ull;

__device__ __forceinline__ unsigned long long gtimer() {
  unsigned long long t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

__device__ __forceinline__ uint32_t smem_addr(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
  asm volatile("{\n .reg .b64 st;\n mbarrier.arrive.shared::cta.b64 st, [%0];\n}" ::"r"(bar) : "memory");
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

}  // namespace

__device__ int g_wait_faults = 0;

// Lets the next kernel of the stream launch (if it was launched with programmatic
// stream serialization); it still waits for this grid in its own griddep_wait.
__device__ __forceinline__ void griddep_launch_dependents() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}
// Returns once the grids this one depends on have completed and their memory
// operations are visible; a no-op when the launch had no programmatic dependency.
__device__ __forceinline__ void griddep_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

namespace {

__device__ __forceinline__ void mbar_wait(uint32_t bar, uint32_t parity) {
  if (mbar_try(bar, parity)) return;
  const unsigned long long t0 = gtimer();
  while (!mbar_try(bar, parity)) {
    if (gtimer() - t0 > kWaitLimitNs) {
      atomicOr(&g_wait_faults, 1);
      return;
    }
  }
}

// ------------------------------------------------------------------ one stage in registers
//
// a[q] holds register slots (2q, 2q+1).  For in-register bit SB the thread's 16
// pairs are (j_k, j_k | 2^SB), j_k = ((k >> SB) << (SB+1)) | (k & (2^SB-1)), and
// coefficient column 4q + e belongs to the low element of pair 2q + e, column
// 4q + 2 + e to its high element.

template <int SB>
__host__ __device__ constexpr int low_slot(int k) {
  return ((k >> SB) << (SB + 1)) | (k & ((1 << SB) - 1));
}

template <int SB, bool SCALED>
__device__ __forceinline__ void stage(float2 (&a)[16], const uint32_t (&c)[32]) {
  if constexpr (SB == 0) {
    // pairs (2k, 2k+1) sit inside one float2: scalar FMAs
#pragma unroll
    for (int q = 0; q < 8; ++q) {
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const int k = 2 * q + e;
        const float cl = u2f(c[4 * q + e]), ch = u2f(c[4 * q + 2 + e]);
        const float lo = a[k].x, hi = a[k].y;
        if constexpr (SCALED) {
          a[k].x = fmaf(cl, hi, lo);
          a[k].y = fmaf(ch, lo, hi);
        } else {
          a[k].x = fmaf(-ch, hi, cl * lo);
          a[k].y = fmaf(cl, hi, ch * lo);
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
      const float2 lo = a[lq], hi = a[hq];
      if constexpr (SCALED) {
        a[lq] = __ffma2_rn(cl, hi, lo);
        a[hq] = __ffma2_rn(ch, lo, hi);
      } else {
        const float2 nch = make_float2(-ch.x, -ch.y);
        a[lq] = __ffma2_rn(nch, hi, __fmul2_rn(cl, lo));
        a[hq] = __ffma2_rn(cl, hi, __fmul2_rn(ch, lo));
      }
    }
  }
}

// One stage.  Double-buffered: computes from `cur` while the block at `next_addr`
// streams into `nxt` and returns after it has arrived.  Single-buffered: loads
// this stage's block at `addr` into `cur` and waits for it first (other warps of
// the SM cover the wait).
template <int SB, bool SCALED>
__device__ __forceinline__ void stage_step(float2 (&a)[16], uint32_t (&cur)[32], uint32_t (&nxt)[32],
                                           uint32_t addr, uint32_t next_addr) {
  if constexpr (kDoubleBuf) {
    tmem_ld32(next_addr, nxt);
    stage<SB, SCALED>(a, cur);
    tmem_wait(nxt);
  } else {
    tmem_ld32(addr, cur);
    tmem_wait(cur);
    stage<SB, SCALED>(a, cur);
  }
}

// ------------------------------------------------------------------ inputs

template <typename TI>
struct Prefetch;
template <>
struct Prefetch<__nv_bfloat16> {
  static constexpr int kVec = 4;  // 16-byte vectors per row per thread (32 bf16)
  uint4 v[kVec];
};
template <>
struct Prefetch<float> {
  static constexpr int kVec = 8;
  uint4 v[kVec];
};

// Pass-A layout input of one row (if cnt > 0): thread tau holds positions 32 tau .. 32 tau + 31.
template <typename TI>
__device__ __forceinline__ void prefetch(Prefetch<TI>& p, const TI* x, long long row, int cnt, int tau) {
  if (cnt > 0) {
    const uint4* src = reinterpret_cast<const uint4*>(x + row * M + tau * 32);
#pragma unroll
    for (int i = 0; i < Prefetch<TI>::kVec; ++i) p.v[i] = src[i];
  }
}

__device__ __forceinline__ void unpack_input(const Prefetch<__nv_bfloat16>& p, float2 (&a)[16]) {
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const uint32_t w[4] = {p.v[i].x, p.v[i].y, p.v[i].z, p.v[i].w};
#pragma unroll
    for (int k = 0; k < 4; ++k)
      a[4 * i + k] = make_float2(__uint_as_float(w[k] << 16), __uint_as_float(w[k] & 0xffff0000u));
  }
}

__device__ __forceinline__ void unpack_input(const Prefetch<float>& p, float2 (&a)[16]) {
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    a[2 * i] = make_float2(__uint_as_float(p.v[i].x), __uint_as_float(p.v[i].y));
    a[2 * i + 1] = make_float2(__uint_as_float(p.v[i].z), __uint_as_float(p.v[i].w));
  }
}

// ------------------------------------------------------------------ transposes
//
// A -> B: pass-A thread t writes its 32 positions as 16-byte vectors at float
// 32 t + 4 (c ^ (t & 7)); pass-B threads read single floats.  B -> C: pass-B
// threads write single floats, pass-C threads read 16-byte vectors, the two
// halves of each 8-position run swapped by bit 2 of the thread index.  Every
// access of a warp covers distinct banks in each of its phases.

__device__ __forceinline__ void xpose_ab_write(const float2 (&a)[16], float* buf, int tau) {
#pragma unroll
  for (int c = 0; c < 8; ++c)
    *reinterpret_cast<float4*>(buf + tau * 32 + 4 * (c ^ (tau & 7))) =
        make_float4(a[2 * c].x, a[2 * c].y, a[2 * c + 1].x, a[2 * c + 1].y);
  // pass-A thread t writes positions 32 t .. 32 t + 31; pass-B thread t reads the
  // positions of pass-A threads 32 (t >> 5) .. 32 (t >> 5) + 31: position bits 10, 11
  // are the warp index in both layouts, so this exchange stays inside the warp
  __syncwarp();
}

__device__ __forceinline__ void xpose_ab_read(float2 (&a)[16], const float* buf, int tau) {
  const int base = ((tau >> 5) << 10) + (tau & 3), cq = (tau & 31) >> 2;
#pragma unroll
  for (int rb = 0; rb < 32; rb += 2) {
    const float v0 = buf[base + 32 * rb + 4 * (cq ^ (rb & 7))];
    const float v1 = buf[base + 32 * (rb + 1) + 4 * (cq ^ ((rb + 1) & 7))];
    a[rb >> 1] = make_float2(v0, v1);
  }
}

__device__ __forceinline__ void xpose_ab(float2 (&a)[16], float* buf, int tau) {
  xpose_ab_write(a, buf, tau);
  xpose_ab_read(a, buf, tau);
}

__device__ __forceinline__ void xpose_bc_write(const float2 (&a)[16], float* buf, int tau) {
  const int base = (tau >> 5) * 1024 + ((tau & 31) >> 3) * 8 + (tau & 3), sw = (tau >> 2) & 1;
#pragma unroll
  for (int rb = 0; rb < 32; rb += 2) {
    buf[base + 32 * rb + 4 * (sw ^ 0)] = a[rb >> 1].x;
    buf[base + 32 * (rb + 1) + 4 * (sw ^ 1)] = a[rb >> 1].y;
  }
}

__device__ __forceinline__ void xpose_bc_read(float2 (&a)[16], const float* buf, int tau) {
  const int sw = (tau >> 2) & 1;
#pragma unroll
  for (int h = 0; h < 4; ++h)
#pragma unroll
    for (int hh = 0; hh < 2; ++hh) {
      const float4 v = *reinterpret_cast<const float4*>(buf + h * 1024 + tau * 8 + 4 * (hh ^ sw));
      a[4 * h + 2 * hh] = make_float2(v.x, v.y);
      a[4 * h + 2 * hh + 1] = make_float2(v.z, v.w);
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

// Per-group asymmetric RTN of the row held in pass-C layout, packing and stores.
//
// Each thread holds 4 sets of 8 consecutive values (position bits 10, 11 = h); a
// group of GROUP = 8 GLANES positions spans GLANES lanes.  Group extremes: 3-input
// min / max over each set, then a recursive-halving shuffle reduction after which
// lane l holds set bitrev(l & 3) of its group, and plain xor levels for the
// remaining group lanes.  Every lane computes the parameters of the set it holds
// (as in rtn_params); one lane per (group, set) stores scale and zero and puts
// (1/s, tie threshold, 1.5 2^23 + z, s) into the warp's parameter slots in shared
// memory, from which every lane reads the parameters of each of its sets after a
// warp barrier (one broadcast load per set instead of four shuffles).  The codes
// then come from rtn_codes8 (exact RTN: see bq_rtn.cuh).
template <int BITS, int GLANES>
__device__ __forceinline__ void quant_epilogue(const float2 (&a)[16], const FastArgs& A, long long row, int tau,
                                               int lane, float4* params) {
  constexpr int S = 4;                    // sets per thread
  constexpr int LOGS = 2;
  constexpr int LOGG = clog2<0>(GLANES);  // lanes sharing one group
  static_assert(LOGS <= LOGG, "a group must span at least S lanes");
  constexpr int GROUP = 8 * GLANES;
  constexpr int GPR = M / GROUP;          // groups per row
  constexpr int QMAX = (1 << BITS) - 1;
  const float qmax = static_cast<float>(QMAX);
  float mn[S], mx[S];
#pragma unroll
  for (int h = 0; h < S; ++h) {
    const float2 p0 = a[4 * h], p1 = a[4 * h + 1], p2 = a[4 * h + 2], p3 = a[4 * h + 3];
    mn[h] = fminf(min3(p0.x, p0.y, p1.x), min3(p1.y, p2.x, min3(p2.y, p3.x, p3.y)));
    mx[h] = fmaxf(max3(p0.x, p0.y, p1.x), max3(p1.y, p2.x, max3(p2.y, p3.x, p3.y)));
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
  const RtnParams P = rtn_params(mn[0], mx[0], qmax);
  const int slot0 = (lane >> LOGG) * S;
  if (((lane >> LOGS) & ((1 << (LOGG - LOGS)) - 1)) == 0) {
    const int h = bitrev<S>(lane & (S - 1));
    const int g = h * (1024 / GROUP) + (tau >> LOGG);
    A.scale[row * GPR + g] = P.scale16;
    A.zero[row * GPR + g] = P.zero16;
    params[slot0 + h] = make_float4(P.inv, P.thr, P.mz, P.s);
  }
  __syncwarp();
#pragma unroll
  for (int h = 0; h < S; ++h) {
    const float4 q = params[slot0 + h];
    const float2 y[4] = {a[4 * h], a[4 * h + 1], a[4 * h + 2], a[4 * h + 3]};
    const uint32_t word = rtn_codes8<BITS>(y, q.x, q.y, q.z, q.w);
    if constexpr (BITS == 4) {
      *reinterpret_cast<uint32_t*>(A.codes + row * (M / 2) + h * 512 + tau * 4) = word;
    } else {
      *reinterpret_cast<uint16_t*>(A.codes + row * (M / 4) + h * 256 + tau * 2) = static_cast<uint16_t>(word);
    }
  }
}

template <int MODE>
__device__ __forceinline__ void store_epilogue(const float2 (&a)[16], const FastArgs& A, long long row, int tau) {
#pragma unroll
  for (int h = 0; h < 4; ++h) {
    const long long off = row * M + h * 1024 + tau * 8;
    if constexpr (MODE == kOutF32) {
      float4* dst = reinterpret_cast<float4*>(static_cast<float*>(A.y) + off);
      dst[0] = make_float4(a[4 * h].x, a[4 * h].y, a[4 * h + 1].x, a[4 * h + 1].y);
      dst[1] = make_float4(a[4 * h + 2].x, a[4 * h + 2].y, a[4 * h + 3].x, a[4 * h + 3].y);
    } else {
      uint4 w;
      __nv_bfloat162 b0 = __floats2bfloat162_rn(a[4 * h].x, a[4 * h].y);
      __nv_bfloat162 b1 = __floats2bfloat162_rn(a[4 * h + 1].x, a[4 * h + 1].y);
      __nv_bfloat162 b2 = __floats2bfloat162_rn(a[4 * h + 2].x, a[4 * h + 2].y);
      __nv_bfloat162 b3 = __floats2bfloat162_rn(a[4 * h + 3].x, a[4 * h + 3].y);
      w.x = *reinterpret_cast<uint32_t*>(&b0);
      w.y = *reinterpret_cast<uint32_t*>(&b1);
      w.z = *reinterpret_cast<uint32_t*>(&b2);
      w.w = *reinterpret_cast<uint32_t*>(&b3);
      *reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(A.y) + off) = w;
    }
  }
}

static_assert(kDoubleBuf, "the forward's pass sequence assumes double-buffered coefficient loads");

// The forward's three passes on the row in registers.  Each starts with the
// coefficient block of its first stage in `x` and returns with the block at `next`
// in `y` (pass C: in `x` again, loaded while the epilogue runs).
template <bool SCALED>
__device__ __forceinline__ void pass_a(float2 (&a)[16], uint32_t (&x)[32], uint32_t (&y)[32], uint32_t tb,
                                       uint32_t next) {
  stage_step<0, SCALED>(a, x, y, tb, tb + 32);
  stage_step<1, SCALED>(a, y, x, tb + 32, tb + 64);
  stage_step<2, SCALED>(a, x, y, tb + 64, tb + 96);
  stage_step<3, SCALED>(a, y, x, tb + 96, tb + 128);
  stage_step<4, SCALED>(a, x, y, tb + 128, next);
}

template <bool SCALED>
__device__ __forceinline__ void pass_b(float2 (&a)[16], uint32_t (&x)[32], uint32_t (&y)[32], uint32_t tb,
                                       uint32_t next) {
  stage_step<0, SCALED>(a, x, y, tb + kColB, tb + kColB + 32);
  stage_step<1, SCALED>(a, y, x, tb + kColB + 32, tb + kColB + 64);
  stage_step<2, SCALED>(a, x, y, tb + kColB + 64, tb + kColB + 96);
  stage_step<3, SCALED>(a, y, x, tb + kColB + 96, tb + kColB + 128);
  stage_step<4, SCALED>(a, x, y, tb + kColB + 128, next);
}

// Pass C (stages 10, 11 on slot bits 3, 4: position bits 10, 11), the output scale
// (1 for the plain rotation) and the epilogue of row `row`.
template <typename TI, int MODE, int BITS, int GLANES, bool SCALED>
__device__ __forceinline__ void pass_c(float2 (&a)[16], uint32_t (&x)[32], uint32_t (&y)[32], const FastArgs& A,
                                       long long row, int tau, int lane, uint32_t tb, float4* params,
                                       uint32_t next) {
  stage_step<3, SCALED>(a, x, y, tb + kColC, tb + kColC + 32);
  stage_step<4, SCALED>(a, y, x, tb + kColC + 32, tb + kColS);
#pragma unroll
  for (int q = 0; q < 16; ++q) a[q] = __fmul2_rn(a[q], make_float2(u2f(x[2 * q]), u2f(x[2 * q + 1])));
  tmem_ld32(next, x);
  if constexpr (MODE == kQuant) {
    quant_epilogue<BITS, GLANES>(a, A, row, tau, lane, params);
  } else {
    store_epilogue<MODE>(a, A, row, tau);
  }
  tmem_wait(x);
}

// Rows rb .. re - 1 of one row group, software-pipelined around the B -> C
// exchange: row j's pass A runs, and the row parks in the A -> B buffer, before
// the group waits for row j - 1's B -> C buffer; then row j - 1's pass C and
// epilogue, row j's pass B and its B -> C writes.  The B -> C buffers and their
// mbarriers alternate by row.  Buffer reuse: a thread writes row j's B -> C
// buffer after its wait for row j - 1, which every thread of the group arrives
// at only after reading row j - 2 from that buffer.  On entry `pre` holds row
// rb's input and c0 coefficient block 0.
template <typename TI, int MODE, int BITS, int GLANES, bool SCALED>
__device__ __forceinline__ void run_rows(const FastArgs& A, long long rb, long long re, int tau, int lane,
                                         uint32_t tb, float* bufAB, float* bufBC, float4* params, uint32_t bars,
                                         Prefetch<TI>& pre, uint32_t (&c0)[32], uint32_t (&c1)[32]) {
  const TI* X = static_cast<const TI*>(A.x);
  float2 a[16];
#pragma unroll 1
  for (long long row = rb; row < re; ++row) {
    const int j = static_cast<int>(row - rb);
    unpack_input(pre, a);
    prefetch(pre, X, row + 1, row + 1 < re ? 1 : 0, tau);
    if (j == 0) {
      pass_a<SCALED>(a, c0, c1, tb, tb + kColB);
      xpose_ab(a, bufAB, tau);
    } else {
      pass_a<SCALED>(a, c0, c1, tb, tb + kColC);
      xpose_ab_write(a, bufAB, tau);  // row j parks here
      const int jp = j - 1;
      mbar_wait(bars + 8 * (jp & 1), (jp >> 1) & 1);
      xpose_bc_read(a, bufBC + (jp & 1) * kBufFloats, tau);
      pass_c<TI, MODE, BITS, GLANES, SCALED>(a, c1, c0, A, row - 1, tau, lane, tb, params, tb + kColB);
      xpose_ab_read(a, bufAB, tau);
    }
    pass_b<SCALED>(a, c1, c0, tb, tb);
    xpose_bc_write(a, bufBC + (j & 1) * kBufFloats, tau);
    mbar_arrive(bars + 8 * (j & 1));
  }
  if (re > rb) {
    const int jl = static_cast<int>(re - 1 - rb);
    tmem_ld32(tb + kColC, c1);
    mbar_wait(bars + 8 * (jl & 1), (jl >> 1) & 1);
    xpose_bc_read(a, bufBC + (jl & 1) * kBufFloats, tau);
    tmem_wait(c1);
    pass_c<TI, MODE, BITS, GLANES, SCALED>(a, c1, c0, A, re - 1, tau, lane, tb, params, tb);
  }
}

// Copies this thread's share of a tensor-memory image (NCHUNK chunks of 16
// columns, dealt round-robin to the NSLOT row groups) into its lane, ROUND chunks
// at a time: all loads of a round in flight first (each warp load is one
// contiguous 512-byte run of the [column/4][lane] image), then the stores.  Every
// CTA reads the same image at the same moment, so each starts at a different
// chunk (block index mod NCHUNK): the requests in flight then spread over the L2
// slices instead of queueing on the same few.
template <int NCHUNK, int NSLOT, int ROUND>
__device__ __forceinline__ void fill_tmem(const float* image, uint32_t tb, int slot, int tau) {
  const float4* src = reinterpret_cast<const float4*>(image) + tau;  // block q of lane tau at [q * 128]
  constexpr int kMine = (NCHUNK + NSLOT - 1) / NSLOT;
  const int rot = blockIdx.x % NCHUNK;
#pragma unroll
  for (int base = 0; base < kMine; base += ROUND) {
    float4 f[ROUND * 4];
#pragma unroll
    for (int i = 0; i < ROUND; ++i) {
      const int c0 = slot + (base + i) * NSLOT;
      if (base + i < kMine && c0 < NCHUNK) {
        const int c = c0 + rot < NCHUNK ? c0 + rot : c0 + rot - NCHUNK;
#pragma unroll
        for (int j = 0; j < 4; ++j) f[4 * i + j] = src[(4 * c + j) * kImageLanes];
      }
    }
#pragma unroll
    for (int i = 0; i < ROUND; ++i) {
      const int c0 = slot + (base + i) * NSLOT;
      if (base + i < kMine && c0 < NCHUNK) {
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
  }
  asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}

template <typename TI, int MODE, int BITS, int GLANES>
__global__ void __launch_bounds__(kThreads, 1) k_fast4096(const FastArgs A) {
  extern __shared__ __align__(16) float smem[];
  __shared__ uint32_t s_tmem;
  __shared__ __align__(8) unsigned long long s_bars[kSlots][2];  // B -> C buffer of rows j, j + 1
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int slot = warp >> 2, wq = warp & 3, tau = wq * 32 + lane;
  float* sbase = smem + slot * kSlotFloats;
  float* bufAB = sbase;
  float* bufBC = sbase + kBufFloats;  // two buffers, used alternately
  float4* params = reinterpret_cast<float4*>(sbase + 3 * kBufFloats) + wq * 32;
  const long long G = static_cast<long long>(gridDim.x) * kSlots;
  const long long g = static_cast<long long>(blockIdx.x) * kSlots + slot;
  const long long rb = g * A.rows / G, re = (g + 1) * A.rows / G;

  Prefetch<TI> pre;
  griddep_launch_dependents();

  if (threadIdx.x == 0) {
#pragma unroll
    for (int i = 0; i < kSlots; ++i) {
      mbar_init(smem_addr(&s_bars[i][0]), kGroupThreads);
      mbar_init(smem_addr(&s_bars[i][1]), kGroupThreads);
    }
  }
  if (warp == 0) {
    const uint32_t dst = static_cast<uint32_t>(__cvta_generic_to_shared(&s_tmem));
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], 512;" ::"r"(dst) : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tb = s_tmem + (static_cast<uint32_t>(wq * 32) << 16);
  griddep_wait();  // everything above touches only shared and tensor memory
  prefetch(pre, static_cast<const TI*>(A.x), rb, re > rb ? 1 : 0, tau);
  fill_tmem<kFillChunks, kSlots, kFillRound>(A.image, tb, slot, tau);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();

  const bool scaled = A.hdr[0] == 1.f;
  const uint32_t bars = smem_addr(&s_bars[slot][0]);
  uint32_t c0[32], c1[32];
  if constexpr (kDoubleBuf) {
    tmem_ld32(tb, c0);
    tmem_wait(c0);
  }
  if (scaled)
    run_rows<TI, MODE, BITS, GLANES, true>(A, rb, re, tau, lane, tb, bufAB, bufBC, params, bars, pre, c0, c1);
  else
    run_rows<TI, MODE, BITS, GLANES, false>(A, rb, re, tau, lane, tb, bufAB, bufBC, params, bars, pre, c0, c1);

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 0) {
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, 512;" ::"r"(s_tmem) : "memory");
  }
}

// Launches one of this file's kernels with programmatic stream serialization: it may
// start while the previous kernel of the stream is still running, and waits for it
// (griddep_wait) before its first global-memory access.
template <typename K>
bq_status launch_dependent(K kern, long long grid, int smem_bytes, const FastArgs& A, cudaStream_t st) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(grid), 1, 1);
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.dynamicSmemBytes = static_cast<size_t>(smem_bytes);
  cfg.stream = st;
  cudaLaunchAttribute at[1];
  at[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  at[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = at;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, A) == cudaSuccess ? BQ_OK : BQ_ERR_CUDA;
}

template <typename TI, int MODE, int BITS, int GLANES>
bq_status launch(const FastArgs& A, cudaStream_t st) {
  auto kern = k_fast4096<TI, MODE, BITS, GLANES>;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return BQ_ERR_CUDA;
  static std::atomic<int> ready[kMaxDevices];
  if (!once_per_device(ready, dev, [&] {
        return cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kFwdSmemBytes) ==
               cudaSuccess;
      }))
    return BQ_ERR_CUDA;
  const int sms = device_sm_count(dev);
  if (sms <= 0) return BQ_ERR_CUDA;
  long long grid = (A.rows + kSlots - 1) / kSlots;
  if (grid > sms) grid = sms;
  if (grid < 1) grid = 1;
  return launch_dependent(kern, grid, kFwdSmemBytes, A, st);
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
// x = Q^T y: stages 11 .. 0, each the transposed rotation, in the forward's thread
// layouts visited backwards (pass C, then B, then A) with the two transposes
// reversed.  The rotation by -theta has the same scaled two-FMA form as the
// forward, with its own coefficients and output scale prepared by
// bq_precompute_cs (table header[3]); the image holds them in the forward's
// columns (stage s at column 32 s, the output scale of the pass-A positions at
// column 384), or (cos, sin) when that form is out of range, in which case the
// plain transposed rotation [[c, s], [-s, c]] runs.  Same row groups and
// coefficient loads as the forward; the C -> B exchange is split the same way, with
// three buffers rotating by row (see run_inv_rows).

template <int SB>
__device__ __forceinline__ void stage_inv_plain(float2 (&a)[16], const uint32_t (&c)[32]) {
  if constexpr (SB == 0) {
#pragma unroll
    for (int q = 0; q < 8; ++q)
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const int k = 2 * q + e;
        const float cl = u2f(c[4 * q + e]), ch = u2f(c[4 * q + 2 + e]);
        const float lo = a[k].x, hi = a[k].y;
        a[k].x = fmaf(ch, hi, cl * lo);
        a[k].y = fmaf(-ch, lo, cl * hi);
      }
  } else {
#pragma unroll
    for (int q = 0; q < 8; ++q) {
      constexpr int kHalf = 1 << (SB - 1);
      const int lq = low_slot<SB>(2 * q) >> 1;
      const int hq = lq + kHalf;
      const float2 cl = make_float2(u2f(c[4 * q]), u2f(c[4 * q + 1]));
      const float2 ch = make_float2(u2f(c[4 * q + 2]), u2f(c[4 * q + 3]));
      const float2 lo = a[lq], hi = a[hq];
      a[lq] = __ffma2_rn(ch, hi, __fmul2_rn(cl, lo));
      a[hq] = __ffma2_rn(make_float2(-ch.x, -ch.y), lo, __fmul2_rn(cl, hi));
    }
  }
}

// Stage S (in-register bit SB) of the inverse; the next stage in visiting order
// is S - 1 (after stage 0: stage 11 of the next row).
template <int S, int SB, bool SCALED>
__device__ __forceinline__ void inv_step(float2 (&a)[16], uint32_t (&cur)[32], uint32_t (&nxt)[32], uint32_t tb) {
  if constexpr (kDoubleBuf) {
    tmem_ld32(tb + 32 * (S > 0 ? S - 1 : 11), nxt);
  } else {
    tmem_ld32(tb + 32 * S, cur);
    tmem_wait(cur);
  }
  if constexpr (SCALED) {
    stage<SB, true>(a, cur);
  } else {
    stage_inv_plain<SB>(a, cur);
  }
  if constexpr (kDoubleBuf) tmem_wait(nxt);
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
      for (int i = 0; i < kPer; ++i) p.v[kPer * h + i] = src[i];
    }
  }
}

// Pass C of the inverse (stages 11, 10 on slot bits 4, 3); c0 holds block 11 on
// entry and block 9 on return.
template <bool SCALED>
__device__ __forceinline__ void inv_pass_c(float2 (&a)[16], uint32_t (&c0)[32], uint32_t (&c1)[32], uint32_t tb) {
  inv_step<11, 4, SCALED>(a, c0, c1, tb);
  inv_step<10, 3, SCALED>(a, c1, c0, tb);
}

// C -> B exchange (across the row group's warps): pass-C threads write 16-byte
// vectors, pass-B threads read single floats.
__device__ __forceinline__ void inv_c2b_write(const float2 (&a)[16], float* buf, int tau) {
  const int sw = (tau >> 2) & 1;
#pragma unroll
  for (int h = 0; h < 4; ++h)
#pragma unroll
    for (int hh = 0; hh < 2; ++hh)
      *reinterpret_cast<float4*>(buf + h * 1024 + tau * 8 + 4 * (hh ^ sw)) =
          make_float4(a[4 * h + 2 * hh].x, a[4 * h + 2 * hh].y, a[4 * h + 2 * hh + 1].x, a[4 * h + 2 * hh + 1].y);
}

__device__ __forceinline__ void inv_c2b_read(float2 (&a)[16], const float* buf, int tau) {
  const int base = (tau >> 5) * 1024 + ((tau & 31) >> 3) * 8 + (tau & 3), sw = (tau >> 2) & 1;
#pragma unroll
  for (int rb = 0; rb < 32; rb += 2)
    a[rb >> 1] = make_float2(buf[base + 32 * rb + 4 * sw], buf[base + 32 * (rb + 1) + 4 * (sw ^ 1)]);
}

// Passes B and A of the inverse (stages 9 .. 0, the B -> A exchange inside the
// warp), the output scale and the store of row `row`; c0 holds block 9 on entry and
// block 11 on return.
template <typename TO, bool SCALED>
__device__ __forceinline__ void inv_pass_ba(float2 (&a)[16], uint32_t (&c0)[32], uint32_t (&c1)[32], uint32_t tb,
                                            float* bufAB, const FastArgs& A, long long row, int tau) {
  inv_step<9, 4, SCALED>(a, c0, c1, tb);
  inv_step<8, 3, SCALED>(a, c1, c0, tb);
  inv_step<7, 2, SCALED>(a, c0, c1, tb);
  inv_step<6, 1, SCALED>(a, c1, c0, tb);
  inv_step<5, 0, SCALED>(a, c0, c1, tb);
  {
    const int base = ((tau >> 5) << 10) + (tau & 3), cq = (tau & 31) >> 2;
#pragma unroll
    for (int rb = 0; rb < 32; rb += 2) {
      bufAB[base + 32 * rb + 4 * (cq ^ (rb & 7))] = a[rb >> 1].x;
      bufAB[base + 32 * (rb + 1) + 4 * (cq ^ ((rb + 1) & 7))] = a[rb >> 1].y;
    }
  }
  __syncwarp();  // the B -> A exchange stays inside the warp (position bits 10, 11)
#pragma unroll
  for (int c = 0; c < 8; ++c) {
    const float4 v = *reinterpret_cast<const float4*>(bufAB + tau * 32 + 4 * (c ^ (tau & 7)));
    a[2 * c] = make_float2(v.x, v.y);
    a[2 * c + 1] = make_float2(v.z, v.w);
  }
  // pass A: stages 4 .. 0 (the last one loads block 11 of the next row)
  inv_step<4, 4, SCALED>(a, c1, c0, tb);
  inv_step<3, 3, SCALED>(a, c0, c1, tb);
  inv_step<2, 2, SCALED>(a, c1, c0, tb);
  inv_step<1, 1, SCALED>(a, c0, c1, tb);
  inv_step<0, 0, SCALED>(a, c1, c0, tb);
  if constexpr (SCALED) {
    // output scale of the pass-A positions
    tmem_ld32(tb + kColS, c1);
    tmem_wait(c1);
#pragma unroll
    for (int q = 0; q < 16; ++q) a[q] = __fmul2_rn(a[q], make_float2(u2f(c1[2 * q]), u2f(c1[2 * q + 1])));
  }
  // pass-A layout output: 32 consecutive positions at 32 tau
  const long long off = row * M + tau * 32;
  if constexpr (sizeof(TO) == 4) {
    float4* dst = reinterpret_cast<float4*>(static_cast<float*>(A.y) + off);
#pragma unroll
    for (int c = 0; c < 8; ++c) dst[c] = make_float4(a[2 * c].x, a[2 * c].y, a[2 * c + 1].x, a[2 * c + 1].y);
  } else {
    uint4* dst = reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(A.y) + off);
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      uint32_t w[4];
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        __nv_bfloat162 b = __floats2bfloat162_rn(a[4 * c + k].x, a[4 * c + k].y);
        w[k] = *reinterpret_cast<uint32_t*>(&b);
      }
      dst[c] = make_uint4(w[0], w[1], w[2], w[3]);
    }
  }
}

// Rows rb .. re - 1 of one row group, software-pipelined around the C -> B
// exchange: row j's pass C runs and the row goes into its C -> B buffer before the
// group waits for row j - 1's; then row j - 1's passes B and A and its store.
// Three C -> B buffers (and mbarriers) rotate by row, and a thread arrives for row
// j only after it has read row j - 1: a thread writes row j into the buffer of row
// j - 3 after its wait for row j - 2, which every thread arrives at only after
// reading row j - 3.  On entry `pre` holds row rb's input and c0 block 11.
template <typename TI, typename TO, bool SCALED>
__device__ __forceinline__ void run_inv_rows(const FastArgs& A, long long rb, long long re, int tau, uint32_t tb,
                                             float* bufAB, float* bufCB, uint32_t bars, Prefetch<TI>& pre,
                                             uint32_t (&c0)[32], uint32_t (&c1)[32]) {
  const TI* X = static_cast<const TI*>(A.x);
  float2 a[16];
#pragma unroll 1
  for (long long row = rb; row < re; ++row) {
    const int j = static_cast<int>(row - rb), b = j % kInvBufs;
    unpack_input(pre, a);
    prefetch_c(pre, X, row + 1, row + 1 < re ? 1 : 0, tau);
    inv_pass_c<SCALED>(a, c0, c1, tb);
    inv_c2b_write(a, bufCB + b * kBufFloats, tau);
    if (j == 0) {
      mbar_arrive(bars + 8 * b);
      tmem_ld32(tb + 32 * 11, c0);  // pass C of the next row comes first
      tmem_wait(c0);
    } else {
      const int jp = j - 1, bp = jp % kInvBufs;
      mbar_wait(bars + 8 * bp, (jp / kInvBufs) & 1);
      inv_c2b_read(a, bufCB + bp * kBufFloats, tau);
      mbar_arrive(bars + 8 * b);
      inv_pass_ba<TO, SCALED>(a, c0, c1, tb, bufAB, A, row - 1, tau);
    }
  }
  if (re > rb) {
    const int jl = static_cast<int>(re - 1 - rb), bl = jl % kInvBufs;
    tmem_ld32(tb + 32 * 9, c0);
    mbar_wait(bars + 8 * bl, (jl / kInvBufs) & 1);
    inv_c2b_read(a, bufCB + bl * kBufFloats, tau);
    tmem_wait(c0);
    inv_pass_ba<TO, SCALED>(a, c0, c1, tb, bufAB, A, re - 1, tau);
  }
}

template <typename TI, typename TO>
__global__ void __launch_bounds__(kThreads, 1) k_inv4096(const FastArgs A) {
  extern __shared__ __align__(16) float smem[];
  __shared__ uint32_t s_tmem;
  __shared__ __align__(8) unsigned long long s_bars[kSlots][kInvBufs];  // one per C -> B buffer
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int slot = warp >> 2, wq = warp & 3, tau = wq * 32 + lane;
  float* bufAB = smem + slot * kInvSlotFloats;
  float* bufCB = bufAB + kBufFloats;  // kInvBufs buffers, rotating by row
  const long long G = static_cast<long long>(gridDim.x) * kSlots;
  const long long g = static_cast<long long>(blockIdx.x) * kSlots + slot;
  const long long rb = g * A.rows / G, re = (g + 1) * A.rows / G;

  Prefetch<TI> pre;
  griddep_launch_dependents();
  if (threadIdx.x == 0) {
#pragma unroll
    for (int i = 0; i < kSlots; ++i)
#pragma unroll
      for (int b = 0; b < kInvBufs; ++b) mbar_init(smem_addr(&s_bars[i][b]), kGroupThreads);
  }
  if (warp == 0) {
    const uint32_t dst = static_cast<uint32_t>(__cvta_generic_to_shared(&s_tmem));
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], 512;" ::"r"(dst) : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tb = s_tmem + (static_cast<uint32_t>(wq * 32) << 16);
  griddep_wait();  // everything above touches only shared and tensor memory
  prefetch_c(pre, static_cast<const TI*>(A.x), rb, re > rb ? 1 : 0, tau);
  fill_tmem<kImageInvCols / 16, kSlots, kFillRound>(A.image, tb, slot, tau);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();

  const bool scaled = A.hdr[3] == 1.f;
  const uint32_t bars = smem_addr(&s_bars[slot][0]);
  uint32_t c0[32], c1[32];
  tmem_ld32(tb + 32 * 11, c0);
  tmem_wait(c0);
  if (scaled)
    run_inv_rows<TI, TO, true>(A, rb, re, tau, tb, bufAB, bufCB, bars, pre, c0, c1);
  else
    run_inv_rows<TI, TO, false>(A, rb, re, tau, tb, bufAB, bufCB, bars, pre, c0, c1);

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
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return BQ_ERR_CUDA;
  static std::atomic<int> ready[kMaxDevices];
  if (!once_per_device(ready, dev, [&] {
        return cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kInvSmemBytes) ==
               cudaSuccess;
      }))
    return BQ_ERR_CUDA;
  const int sms = device_sm_count(dev);
  if (sms <= 0) return BQ_ERR_CUDA;
  long long grid = (A.rows + kSlots - 1) / kSlots;
  if (grid > sms) grid = sms;
  if (grid < 1) grid = 1;
  return launch_dependent(kern, grid, kInvSmemBytes, A, st);
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

bq_status read_wait_faults(int32_t* value, bool clear, cudaStream_t st) {
  int v = 0;
  if (cudaMemcpyFromSymbolAsync(&v, g_wait_faults, sizeof(int), 0, cudaMemcpyDeviceToHost, st) != cudaSuccess)
    return BQ_ERR_CUDA;
  static const int kZero = 0;
  if (clear && cudaMemcpyToSymbolAsync(g_wait_faults, &kZero, sizeof(int), 0, cudaMemcpyHostToDevice, st) != cudaSuccess)
    return BQ_ERR_CUDA;
  if (cudaStreamSynchronize(st) != cudaSuccess) return BQ_ERR_CUDA;
  *value = v;
  return BQ_OK;
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
