// Specialised calibration backward for m = 4096 (r = 1): Y = Q X, dX = Q^T dY
// and dtheta summed over tokens, every layer in one launch.
//
// The angles are learned by gradient descent (ButterflyQuant abstract).  For a
// rotation y_i = c x_i - s x_j, y_j = s x_i + c x_j with g = dloss/dy, the chain
// rule gives dloss/dtheta = g_j y_i - g_i y_j and dloss/dx = B^T g, so the
// reverse sweep walks the stages s = 11 .. 0 with v (the stage outputs) and g,
// accumulating g_j v_i - g_i v_j per pair.
//
// Design (B200, sm_100a):
//  * One CTA per SM, 512 threads on one token at a time; each thread holds 8
//    elements of the row.  The 12 stages run as four passes of three stages,
//    the pass-P layout keeping position bits 3P .. 3P+2 in registers:
//        P0: 8 tau + e                                 (contiguous: vector I/O)
//        P1: (l & 7) | e << 3 | (l >> 3) << 6 | w << 8  (warp-local with P0)
//        P2: l | (w & 1) << 5 | e << 6 | (w >> 1) << 9   (warp pairs with P1)
//        P3: l | w << 5 | e << 9                        (coalesced dY / Y)
//    with tau = 32 w + l.  The exchanges go through shared memory padded by 4
//    floats every 32, which keeps every exchange conflict-free on both sides
//    and makes each thread's addresses a base plus compile-time offsets.
//  * The layer's cos/sin (96 per thread: 12 stages x 4 pairs x 2) sit in tensor
//    memory, gathered from the prepared table whenever the CTA moves to a new
//    layer; each stage reads its 8 values with one tcgen05.ld.
//  * The 48 dtheta sums of a thread (12 stages x 4 pairs) stay in registers for
//    a whole token chunk.  v at the end of passes 0..2 is kept from the forward
//    in the exchange buffers and re-read by the reverse sweep, which recovers
//    the other stage outputs of a pass by the inverse rotation.
//  * Determinism: tokens are cut into fixed chunks (independent of the grid);
//    each chunk's sums go to its own workspace slot and the last chunk of a
//    layer to finish (atomic ticket, no waiting) adds the slots in chunk order.
#include "bq_internal.cuh"

namespace bq {
namespace {

constexpr int M = 4096;
constexpr int kStages = 12;
constexpr int kThreads = 512;
constexpr int kBuf = 4608;     // floats per exchange buffer: 4096 + 4 per 32
constexpr int kColsPer = 96;   // tensor-memory columns per thread
constexpr int kAcc = 48;       // dtheta sums per thread
constexpr int kCounterBytes = 512;

struct B4Args {
  int layers, chunks;  // chunks per layer
  long long rows;      // tokens per layer
  const void* x;
  void* y;
  const float* dy;
  float* dx;
  float* dtheta;
  float* part;
  unsigned* counters;
  const float2* cs[kMaxBwdLayers];
};

// ------------------------------------------------------------------ tensor memory

__device__ __forceinline__ void tld8(uint32_t addr, uint32_t (&r)[8]) {
  asm volatile("tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7])
               : "r"(addr));
}

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

__device__ __forceinline__ void fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

__device__ __forceinline__ void cta_sync() {
  fence_before();
  __syncthreads();
  fence_after();
}

__device__ __forceinline__ void pair_sync(int w) {
  asm volatile("bar.sync %0, %1;" ::"r"(1 + (w >> 1)), "r"(64) : "memory");
}

__device__ __forceinline__ float u2f(uint32_t v) { return __uint_as_float(v); }

// ------------------------------------------------------------------ layouts

// position of element e of thread tau in pass P
__device__ __forceinline__ int pos_pass(int P, int tau, int e) {
  const int l = tau & 31, w = tau >> 5;
  if (P == 0) return 8 * tau + e;
  if (P == 1) return (l & 7) | (e << 3) | ((l >> 3) << 6) | (w << 8);
  if (P == 2) return l | ((w & 1) << 5) | (e << 6) | ((w >> 1) << 9);
  return l | (w << 5) | (e << 9);
}

// pr-th element (ascending) whose in-register bit SB is clear: the low end of pair pr
__host__ __device__ constexpr int e_low(int pr, int SB) { return ((pr >> SB) << (SB + 1)) | (pr & ((1 << SB) - 1)); }

// angle index of pair pr of thread tau at stage s
__device__ __forceinline__ int pair_index(int tau, int s, int pr) {
  const int i = pos_pass(s / 3, tau, e_low(pr, s % 3));
  return ((i >> (s + 1)) << s) | (i & ((1 << s) - 1));
}

// ------------------------------------------------------------------ one stage
//
// a[k] holds elements (2k, 2k+1) of the thread.  Coefficient block: c[pr] = cos,
// c[4 + pr] = sin of pair pr.  For SB >= 1 pairs (0, 1) and (2, 3) use packed
// f32x2 arithmetic: their low ends are adjacent elements, as are the high ends.

template <int SB>
__device__ __forceinline__ void lo_hi(int h, int& lo, int& hi) {
  // float2 indices of the low and high ends of pairs (2h, 2h+1)
  if constexpr (SB == 1) {
    lo = 2 * h;
    hi = 2 * h + 1;
  } else {
    lo = h;
    hi = h + 2;
  }
}

// v <- B_s v (INV = false) or v <- B_s^T v (INV = true)
template <int SB, bool INV>
__device__ __forceinline__ void rotate(float2 (&a)[4], const uint32_t (&c)[8]) {
  if constexpr (SB == 0) {
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const float co = u2f(c[k]), si = INV ? -u2f(c[4 + k]) : u2f(c[4 + k]);
      const float lo = a[k].x, hi = a[k].y;
      a[k].x = fmaf(co, lo, -si * hi);
      a[k].y = fmaf(si, lo, co * hi);
    }
  } else {
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      int il, ih;
      lo_hi<SB>(h, il, ih);
      const float2 C = make_float2(u2f(c[2 * h]), u2f(c[2 * h + 1]));
      const float2 S = INV ? make_float2(-u2f(c[4 + 2 * h]), -u2f(c[5 + 2 * h]))
                           : make_float2(u2f(c[4 + 2 * h]), u2f(c[5 + 2 * h]));
      const float2 nS = make_float2(-S.x, -S.y);
      const float2 lo = a[il], hi = a[ih];
      a[il] = __ffma2_rn(C, lo, __fmul2_rn(nS, hi));
      a[ih] = __ffma2_rn(S, lo, __fmul2_rn(C, hi));
    }
  }
}

// dtheta sums of one stage: acc[pr] += g_hi v_lo - g_lo v_hi
template <int SB>
__device__ __forceinline__ void accumulate(float2 (&acc)[2], const float2 (&v)[4], const float2 (&g)[4]) {
  if constexpr (SB == 0) {
    acc[0].x = fmaf(-g[0].x, v[0].y, fmaf(g[0].y, v[0].x, acc[0].x));
    acc[0].y = fmaf(-g[1].x, v[1].y, fmaf(g[1].y, v[1].x, acc[0].y));
    acc[1].x = fmaf(-g[2].x, v[2].y, fmaf(g[2].y, v[2].x, acc[1].x));
    acc[1].y = fmaf(-g[3].x, v[3].y, fmaf(g[3].y, v[3].x, acc[1].y));
  } else {
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      int il, ih;
      lo_hi<SB>(h, il, ih);
      const float2 ng = make_float2(-g[il].x, -g[il].y);
      acc[h] = __ffma2_rn(ng, v[ih], __ffma2_rn(g[ih], v[il], acc[h]));
    }
  }
}

// ------------------------------------------------------------------ shared-memory exchange
//
// Buffer address of position p: p + 4 * (p >> 5).  Per thread this is a base
// plus a compile-time offset in every pass:
//   P0: 8 tau + 4 (tau >> 2) + e (+4 for the second float4)
//   P1: (l & 7) + 72 (l >> 3) + 288 w + 8 e + 4 (e >> 2)
//   P2: l + 36 (w & 1) + 576 (w >> 1) + 72 e
//   P3: l + 36 w + 576 e

struct Bases {
  int b0, b1, b2, b3;  // exchange-buffer bases of passes 0..3
  int p3;              // row position of element 0 in pass 3 (l + 32 w)
};

__device__ __forceinline__ Bases make_bases(int tau) {
  const int l = tau & 31, w = tau >> 5;
  Bases b;
  b.b0 = 8 * tau + 4 * (tau >> 2);
  b.b1 = (l & 7) + 72 * (l >> 3) + 288 * w;
  b.b2 = l + 36 * (w & 1) + 576 * (w >> 1);
  b.b3 = l + 36 * w;
  b.p3 = l + 32 * w;
  return b;
}

template <int P>
__device__ __forceinline__ int off(int e) {
  if constexpr (P == 1) return 8 * e + 4 * (e >> 2);
  if constexpr (P == 2) return 72 * e;
  return 576 * e;
}

template <int P>
__device__ __forceinline__ void put(float* buf, int base, const float2 (&a)[4]) {
  if constexpr (P == 0) {
    *reinterpret_cast<float4*>(buf + base) = make_float4(a[0].x, a[0].y, a[1].x, a[1].y);
    *reinterpret_cast<float4*>(buf + base + 4) = make_float4(a[2].x, a[2].y, a[3].x, a[3].y);
  } else {
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      buf[base + off<P>(2 * k)] = a[k].x;
      buf[base + off<P>(2 * k + 1)] = a[k].y;
    }
  }
}

template <int P>
__device__ __forceinline__ void get(const float* buf, int base, float2 (&a)[4]) {
  if constexpr (P == 0) {
    const float4 u = *reinterpret_cast<const float4*>(buf + base);
    const float4 v = *reinterpret_cast<const float4*>(buf + base + 4);
    a[0] = make_float2(u.x, u.y);
    a[1] = make_float2(u.z, u.w);
    a[2] = make_float2(v.x, v.y);
    a[3] = make_float2(v.z, v.w);
  } else {
#pragma unroll
    for (int k = 0; k < 4; ++k) a[k] = make_float2(buf[base + off<P>(2 * k)], buf[base + off<P>(2 * k + 1)]);
  }
}

// ------------------------------------------------------------------ token I/O

// The next token's X and dY are copied into shared memory with cp.async while the
// current token runs.  Thread tau copies the 16-byte pieces at byte offsets
// 16 (tau + 512 q) of each row: for X these are its own pass-0 elements (bf16:
// one piece, fp32: two), for dY it is a share that other threads read in pass 3,
// after a barrier.
__device__ __forceinline__ void cp16(void* dst, const void* src) {
  const uint32_t d = static_cast<uint32_t>(__cvta_generic_to_shared(dst));
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(d), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
__device__ __forceinline__ void cp_wait_all() { asm volatile("cp.async.wait_group 0;" ::: "memory"); }

template <typename TI>
__device__ __forceinline__ void issue_token(const TI* x, const float* dy, float* xs, float* dys, int tau) {
  const char* xb = reinterpret_cast<const char*>(x);
  char* xd = reinterpret_cast<char*>(xs);
  if constexpr (sizeof(TI) == 4) {
    cp16(xd + 32 * tau, xb + 32 * tau);
    cp16(xd + 32 * tau + 16, xb + 32 * tau + 16);
  } else {
    cp16(xd + 16 * tau, xb + 16 * tau);
  }
  const char* yb = reinterpret_cast<const char*>(dy);
  char* yd = reinterpret_cast<char*>(dys);
  cp16(yd + 16 * tau, yb + 16 * tau);
  cp16(yd + 16 * (tau + 512), yb + 16 * (tau + 512));
}

__device__ __forceinline__ void read_x(const float* xs, int tau, float2 (&a)[4], float) {
  const float4 u = reinterpret_cast<const float4*>(xs)[2 * tau];
  const float4 v = reinterpret_cast<const float4*>(xs)[2 * tau + 1];
  a[0] = make_float2(u.x, u.y);
  a[1] = make_float2(u.z, u.w);
  a[2] = make_float2(v.x, v.y);
  a[3] = make_float2(v.z, v.w);
}
__device__ __forceinline__ void read_x(const float* xs, int tau, float2 (&a)[4], __nv_bfloat16) {
  const uint4 p = reinterpret_cast<const uint4*>(xs)[tau];
  const uint32_t w[4] = {p.x, p.y, p.z, p.w};
#pragma unroll
  for (int k = 0; k < 4; ++k) a[k] = make_float2(__uint_as_float(w[k] << 16), __uint_as_float(w[k] & 0xffff0000u));
}

__device__ __forceinline__ void store_y(float* y, int b3, const float2 (&a)[4]) {
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    y[b3 + 512 * (2 * k)] = a[k].x;
    y[b3 + 512 * (2 * k + 1)] = a[k].y;
  }
}
__device__ __forceinline__ void store_y(__nv_bfloat16* y, int b3, const float2 (&a)[4]) {
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    y[b3 + 512 * (2 * k)] = __float2bfloat16_rn(a[k].x);
    y[b3 + 512 * (2 * k + 1)] = __float2bfloat16_rn(a[k].y);
  }
}


__device__ __forceinline__ void store_dx(float* dx, int tau, const float2 (&a)[4]) {
  float4* d = reinterpret_cast<float4*>(dx + 8 * tau);
  d[0] = make_float4(a[0].x, a[0].y, a[1].x, a[1].y);
  d[1] = make_float4(a[2].x, a[2].y, a[3].x, a[3].y);
}

// ------------------------------------------------------------------ kernel
//
// Coefficient blocks ping-pong between ca and cn: stage s always uses ca when s
// is even and cn when s is odd, in both sweeps, while the next block streams
// into the other array.  Between tokens ca holds block 0.

template <typename TI, typename TO>
__global__ void __launch_bounds__(kThreads, 1) k_bwd4096(const __grid_constant__ B4Args A) {
  extern __shared__ __align__(16) float smem[];
  __shared__ uint32_t s_tmem;
  __shared__ int s_last;
  float* E1 = smem;        // v after stage 2  (forward pass 0 -> 1)
  float* E2 = E1 + kBuf;   // v after stage 5  (pass 1 -> 2)
  float* E3 = E2 + kBuf;   // v after stage 8  (pass 2 -> 3)
  float* Ga = E3 + kBuf;   // g: reverse pass 3 -> 2 and 1 -> 0
  float* Gb = Ga + kBuf;   // g: reverse pass 2 -> 1
  float* Xs = Gb + kBuf;   // [2][M] floats: X of the current / next token (bf16 uses half)
  float* Ds = Xs + 2 * M;  // [2][M]: dY of the current / next token
  const int tau = threadIdx.x, w = tau >> 5;
  const Bases B = make_bases(tau);

  if (w == 0) {
    const uint32_t dst = static_cast<uint32_t>(__cvta_generic_to_shared(&s_tmem));
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], 512;" ::"r"(dst) : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  cta_sync();
  const uint32_t tb =
      s_tmem + (static_cast<uint32_t>(32 * (w & 3)) << 16) + static_cast<uint32_t>(kColsPer * (w >> 2));

  const long long total = static_cast<long long>(A.layers) * A.chunks;
  const long long cb = blockIdx.x * total / gridDim.x, ce = (blockIdx.x + 1) * total / gridDim.x;
  int cur_layer = -1;

#pragma unroll 1
  for (long long ch = cb; ch < ce; ++ch) {
    const int layer = static_cast<int>(ch / A.chunks), j = static_cast<int>(ch % A.chunks);
    if (layer != cur_layer) {
      // gather this thread's 96 cos/sin values of the new layer into its lane
      cta_sync();  // every thread is done with the previous layer's values
      const float2* cs = A.cs[layer];
#pragma unroll 1
      for (int s = 0; s < kStages; ++s) {
        uint32_t v[8];
#pragma unroll
        for (int pr = 0; pr < 4; ++pr) {
          const float2 t = cs[s * (M / 2) + pair_index(tau, s, pr)];
          v[pr] = __float_as_uint(t.x);
          v[4 + pr] = __float_as_uint(t.y);
        }
        tst8(tb + 8 * s, v);
      }
      asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
      cta_sync();
      cur_layer = layer;
    }
    const long long t0 = j * A.rows / A.chunks, t1 = (j + 1) * A.rows / A.chunks;
    const size_t lbase = static_cast<size_t>(layer) * static_cast<size_t>(A.rows) * M;
    const TI* X = static_cast<const TI*>(A.x) + lbase;
    TO* Y = static_cast<TO*>(A.y) + lbase;
    const float* DY = A.dy + lbase;
    float* DX = A.dx + lbase;

    float2 acc[kStages][2];
#pragma unroll
    for (int s = 0; s < kStages; ++s) acc[s][0] = acc[s][1] = make_float2(0.f, 0.f);

    issue_token(X + t0 * M, DY + t0 * M, Xs + (t0 & 1) * M, Ds + (t0 & 1) * M, tau);
    cp_commit();
    uint32_t ca[8], cn[8];
    tld8(tb, ca);
    twait(ca);

#pragma unroll 1
    for (long long t = t0; t < t1; ++t) {
      const int par = static_cast<int>(t & 1);
      cp_wait_all();  // this thread's copies of token t have landed
      float2 v[4];
      read_x(Xs + par * M, tau, v, TI());
      if (t + 1 < t1) issue_token(X + (t + 1) * M, DY + (t + 1) * M, Xs + (par ^ 1) * M, Ds + (par ^ 1) * M, tau);
      cp_commit();

      // ---------------- forward: v <- Q v, leaving v at the ends of passes 0..2 in E1..E3
      tld8(tb + 8, cn);  rotate<0, false>(v, ca); twait(cn);
      tld8(tb + 16, ca); rotate<1, false>(v, cn); twait(ca);
      tld8(tb + 24, cn); rotate<2, false>(v, ca); twait(cn);
      put<0>(E1, B.b0, v);
      __syncwarp();
      get<1>(E1, B.b1, v);
      tld8(tb + 32, ca); rotate<0, false>(v, cn); twait(ca);
      tld8(tb + 40, cn); rotate<1, false>(v, ca); twait(cn);
      tld8(tb + 48, ca); rotate<2, false>(v, cn); twait(ca);
      put<1>(E2, B.b1, v);
      pair_sync(w);
      get<2>(E2, B.b2, v);
      tld8(tb + 56, cn); rotate<0, false>(v, ca); twait(cn);
      tld8(tb + 64, ca); rotate<1, false>(v, cn); twait(ca);
      tld8(tb + 72, cn); rotate<2, false>(v, ca); twait(cn);
      put<2>(E3, B.b2, v);
      __syncthreads();
      get<3>(E3, B.b3, v);
      tld8(tb + 80, ca); rotate<0, false>(v, cn); twait(ca);
      tld8(tb + 88, cn); rotate<1, false>(v, ca); twait(cn);
      rotate<2, false>(v, cn);  // stage 11: v = Y, block 11 stays in cn
      store_y(Y + t * M + B.p3, 0, v);

      // ---------------- reverse sweep: s = 11 .. 0
      float2 g[4];
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        // dY of token t: every thread's copies landed before the pass 2 -> 3 barrier
        const float* d = Ds + par * M + B.p3;
        g[k] = make_float2(d[512 * (2 * k)], d[512 * (2 * k + 1)]);
      }
      // pass 3
      tld8(tb + 80, ca);
      accumulate<2>(acc[11], v, g); rotate<2, true>(g, cn); rotate<2, true>(v, cn);
      twait(ca);
      tld8(tb + 72, cn);
      accumulate<1>(acc[10], v, g); rotate<1, true>(g, ca); rotate<1, true>(v, ca);
      twait(cn);
      tld8(tb + 64, ca);
      accumulate<0>(acc[9], v, g); rotate<0, true>(g, cn);
      put<3>(Ga, B.b3, g);
      get<2>(E3, B.b2, v);  // v after stage 8: this thread's own forward values
      twait(ca);
      __syncthreads();
      get<2>(Ga, B.b2, g);
      // pass 2
      tld8(tb + 56, cn);
      accumulate<2>(acc[8], v, g); rotate<2, true>(g, ca); rotate<2, true>(v, ca);
      twait(cn);
      tld8(tb + 48, ca);
      accumulate<1>(acc[7], v, g); rotate<1, true>(g, cn); rotate<1, true>(v, cn);
      twait(ca);
      tld8(tb + 40, cn);
      accumulate<0>(acc[6], v, g); rotate<0, true>(g, ca);
      put<2>(Gb, B.b2, g);
      get<1>(E2, B.b1, v);  // v after stage 5
      twait(cn);
      pair_sync(w);
      get<1>(Gb, B.b1, g);
      // pass 1
      tld8(tb + 32, ca);
      accumulate<2>(acc[5], v, g); rotate<2, true>(g, cn); rotate<2, true>(v, cn);
      twait(ca);
      tld8(tb + 24, cn);
      accumulate<1>(acc[4], v, g); rotate<1, true>(g, ca); rotate<1, true>(v, ca);
      twait(cn);
      tld8(tb + 16, ca);
      accumulate<0>(acc[3], v, g); rotate<0, true>(g, cn);
      put<1>(Ga, B.b1, g);
      get<0>(E1, B.b0, v);  // v after stage 2
      twait(ca);
      __syncwarp();
      get<0>(Ga, B.b0, g);
      // pass 0
      tld8(tb + 8, cn);
      accumulate<2>(acc[2], v, g); rotate<2, true>(g, ca); rotate<2, true>(v, ca);
      twait(cn);
      tld8(tb, ca);
      accumulate<1>(acc[1], v, g); rotate<1, true>(g, cn); rotate<1, true>(v, cn);
      twait(ca);
      accumulate<0>(acc[0], v, g); rotate<0, true>(g, ca);
      store_dx(DX + t * M, tau, g);
    }

    // this chunk's sums -> its workspace slot [chunk][k][tau], k = 4 s + pr
    float* pp = A.part + (static_cast<size_t>(layer) * A.chunks + j) * (kAcc * kThreads) + tau;
#pragma unroll
    for (int s = 0; s < kStages; ++s) {
      pp[(4 * s + 0) * kThreads] = acc[s][0].x;
      pp[(4 * s + 1) * kThreads] = acc[s][0].y;
      pp[(4 * s + 2) * kThreads] = acc[s][1].x;
      pp[(4 * s + 3) * kThreads] = acc[s][1].y;
    }
    __threadfence();
    __syncthreads();
    if (tau == 0) {
      const unsigned prev = atomicAdd(&A.counters[layer], 1u);
      s_last = prev == static_cast<unsigned>(A.chunks - 1);
    }
    __syncthreads();
    if (s_last) {
      // last chunk of this layer: add every chunk's slot in chunk order
      __threadfence();
      const float* base = A.part + static_cast<size_t>(layer) * A.chunks * (kAcc * kThreads) + tau;
      float* out = A.dtheta + static_cast<size_t>(layer) * (kStages * (M / 2));
      // one chunk per step, all 48 of its loads independent (the reduction is
      // latency-bound otherwise: it runs on one CTA per layer)
      float sum[kAcc];
#pragma unroll
      for (int k = 0; k < kAcc; ++k) sum[k] = 0.f;
#pragma unroll 1
      for (int c = 0; c < A.chunks; ++c) {
        const float* q = base + static_cast<size_t>(c) * (kAcc * kThreads);
#pragma unroll
        for (int k = 0; k < kAcc; ++k) sum[k] += __ldcg(q + k * kThreads);
      }
#pragma unroll
      for (int k = 0; k < kAcc; ++k) out[(k >> 2) * (M / 2) + pair_index(tau, k >> 2, k & 3)] = sum[k];
      if (tau == 0) A.counters[layer] = 0u;
    }
  }

  cta_sync();
  if (w == 0) asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, 512;" ::"r"(s_tmem) : "memory");
}

template <typename TI, typename TO>
bq_status run(const B4Args& A, cudaStream_t st) {
  auto kern = k_bwd4096<TI, TO>;
  constexpr int smem = (5 * kBuf + 4 * M) * static_cast<int>(sizeof(float));
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return BQ_ERR_CUDA;
  static std::atomic<int> ready[kMaxDevices];
  if (!once_per_device(ready, dev, [&] {
        return cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) == cudaSuccess;
      }))
    return BQ_ERR_CUDA;
  const int sms = device_sm_count(dev);
  if (sms <= 0) return BQ_ERR_CUDA;
  long long grid = static_cast<long long>(A.layers) * A.chunks;
  if (grid > sms) grid = sms;
  kern<<<static_cast<unsigned>(grid), kThreads, smem, st>>>(A);
  return cudaPeekAtLastError() == cudaSuccess ? BQ_OK : BQ_ERR_CUDA;
}

}  // namespace

int bwd4096_chunks(int num_layers, int64_t rows) {
  // about eight chunks per SM of a B200 (148 SMs), at most one per token
  long long c = (148LL * 8 + num_layers - 1) / num_layers;
  if (c > rows) c = rows;
  if (c < 1) c = 1;
  return static_cast<int>(c);
}

bq_status launch_bwd4096(const KLayer* layers, int num_layers, const void* x, bq_dtype xt, void* y, bq_dtype yt,
                         const float* dy, float* dx, float* dtheta, int64_t rows, void* ws, int chunks,
                         cudaStream_t st) {
  B4Args A;
  A.layers = num_layers;
  A.chunks = chunks;
  A.rows = rows;
  A.x = x; A.y = y; A.dy = dy; A.dx = dx; A.dtheta = dtheta;
  A.counters = static_cast<unsigned*>(ws);
  A.part = reinterpret_cast<float*>(static_cast<char*>(ws) + kCounterBytes);
  for (int l = 0; l < kMaxBwdLayers; ++l) A.cs[l] = l < num_layers ? layers[l].cs : nullptr;
  if (cudaMemsetAsync(ws, 0, kCounterBytes, st) != cudaSuccess) return BQ_ERR_CUDA;
  if (xt == BQ_F32 && yt == BQ_F32) return run<float, float>(A, st);
  if (xt == BQ_F32 && yt == BQ_BF16) return run<float, __nv_bfloat16>(A, st);
  if (xt == BQ_BF16 && yt == BQ_F32) return run<__nv_bfloat16, float>(A, st);
  return run<__nv_bfloat16, __nv_bfloat16>(A, st);
}

}  // namespace bq
