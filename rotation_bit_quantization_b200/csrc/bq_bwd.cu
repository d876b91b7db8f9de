// K4: backward of the butterfly transform for angle calibration, all layers in
// one launch, with a deterministic token reduction of dtheta.
//
// The angles are learned by gradient descent (ButterflyQuant abstract).  With
// the loss linear in Y = Q X and upstream gradient dY, the chain rule through
// one rotation y_i = c x_i - s x_j, y_j = s x_i + c x_j gives
//     d loss / d theta = g_j y_i - g_i y_j      (g = d loss / d y)
//     d loss / d x     = B^T g.
// The reverse sweep therefore starts from v = Y, g = dY and, for stage
// s = L-1 .. 0, accumulates g_j v_i - g_i v_j into dtheta[s][p] and maps both
// v and g back through B_s^T.  v is recovered by the inverse rotation instead
// of being stored (Q is orthogonal), so no per-stage activations are kept.
//
// Work split: block b handles layer b / chunks and a fixed contiguous token
// range of it, two tokens at a time, keeping a float32 dtheta partial for the
// whole layer in shared memory.  Each block writes its partial to the
// workspace; the last block of a layer to finish (atomic ticket, no waiting)
// sums the partials in chunk order, so dtheta is bitwise reproducible.
#include <cfloat>

#include "bq_passes.cuh"

namespace bq {
namespace {

constexpr int kBwdThreads = 512;
constexpr int kTokens = 2;          // tokens per batch held in shared memory
constexpr int kCounterBytes = 512;  // ticket counters at the start of the workspace

struct BwdArgs {
  int m, L, chunks, layers;
  long long rows;
  const void* x;
  void* y;
  const float* dy;
  float* dx;
  float* dtheta;
  float* part;
  unsigned* counters;
  const float2* cs[kMaxBwdLayers];
};

template <int SB>
__device__ __forceinline__ void bwd_stage(float (&v)[8], float (&g)[8], float (&acc)[4], int E, int base,
                                          int b0, int s, const float2* __restrict__ cs_s) {
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    if ((j >> SB) & 1) continue;
    if (j >= E) continue;
    const int jj = j | (1 << SB);
    const int pl = ((j >> (SB + 1)) << SB) | (j & ((1 << SB) - 1));
    const int i = base | (j << b0);
    const int p = ((i >> (s + 1)) << s) | (i & ((1 << s) - 1));
    const float2 c = __ldg(&cs_s[p]);
    acc[pl] = fmaf(g[jj], v[j], acc[pl]);
    acc[pl] = fmaf(-g[j], v[jj], acc[pl]);
    const float a = v[j], b = v[jj];
    v[j] = c.x * a + c.y * b;
    v[jj] = c.x * b - c.y * a;
    const float ga = g[j], gb = g[jj];
    g[j] = c.x * ga + c.y * gb;
    g[jj] = c.x * gb - c.y * ga;
  }
}

__device__ __forceinline__ void bwd_any(float (&v)[8], float (&g)[8], float (&acc)[4], int E, int base, int b0,
                                        int s, const float2* cs_s) {
  switch (s - b0) {
    case 0: bwd_stage<0>(v, g, acc, E, base, b0, s, cs_s); break;
    case 1: bwd_stage<1>(v, g, acc, E, base, b0, s, cs_s); break;
    default: bwd_stage<2>(v, g, acc, E, base, b0, s, cs_s); break;
  }
}

template <int SB>
__device__ __forceinline__ void add_acc(float* dth, const float (&acc)[4], int E, int base, int b0, int s, int half) {
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    if ((j >> SB) & 1) continue;
    if (j >= E) continue;
    const int pl = ((j >> (SB + 1)) << SB) | (j & ((1 << SB) - 1));
    const int i = base | (j << b0);
    const int p = ((i >> (s + 1)) << s) | (i & ((1 << s) - 1));
    dth[s * half + p] += acc[pl];
  }
}

template <typename TI, typename TO>
__global__ void __launch_bounds__(kBwdThreads, 1) k_bwd(const __grid_constant__ BwdArgs A) {
  extern __shared__ float smem[];
  const int m = A.m, L = A.L, half = m >> 1, nang = L * half;
  const int tid = threadIdx.x, T = blockDim.x;
  const int layer = blockIdx.x / A.chunks, chunk = blockIdx.x % A.chunks;
  const long long R = A.rows;
  const long long t0 = chunk * R / A.chunks, t1 = (chunk + 1) * R / A.chunks;
  const int stride = pad(m) + 1;
  float* dth = smem;
  float* vb = smem + round4(size_t(nang));
  float* gb = vb + kTokens * stride;
  KLayer Ly;
  Ly.m = m; Ly.L = L; Ly.r = 1; Ly.n = m;
  Ly.cs = A.cs[layer];
  const TI* X = static_cast<const TI*>(A.x) + static_cast<long long>(layer) * R * m;
  TO* Y = static_cast<TO*>(A.y) + static_cast<long long>(layer) * R * m;
  const float* DY = A.dy + static_cast<long long>(layer) * R * m;
  float* DX = A.dx + static_cast<long long>(layer) * R * m;

  const int ec = L < kBitsPerPass ? L : kBitsPerPass;
  const int E = 1 << ec;
  const int per = m >> ec;
  const int passes = (L + kBitsPerPass - 1) / kBitsPerPass;

  for (int k = tid; k < nang; k += T) dth[k] = 0.f;
  __syncthreads();

  for (long long tb = t0; tb < t1; tb += kTokens) {
    const int nt = static_cast<int>(t1 - tb < kTokens ? t1 - tb : kTokens);
    for (int idx = tid; idx < nt * m; idx += T) {
      const int t = idx / m, i = idx % m;
      vb[t * stride + pad(i)] = load_elem(X + (tb + t) * m + i);
    }
    __syncthreads();
    // forward: v <- Q v
    for (int k = 0; k < passes; ++k) {
      const int s0 = k * kBitsPerPass, s1 = s0 + kBitsPerPass < L ? s0 + kBitsPerPass : L;
      const int b0 = s0 < L - ec ? s0 : L - ec;
      const int lowmask = (1 << b0) - 1;
      for (int w = tid; w < nt * per; w += T) {
        const int t = w / per, q = w % per;
        const int base = (q & lowmask) | ((q >> b0) << (b0 + ec));
        float* buf = vb + t * stride;
        float v[8];
#pragma unroll
        for (int j = 0; j < 8; ++j)
          if (j < E) v[j] = buf[pad(base | (j << b0))];
        for (int s = s0; s < s1; ++s) rot_any<false>(v, E, base, b0, s, Ly);
#pragma unroll
        for (int j = 0; j < 8; ++j)
          if (j < E) buf[pad(base | (j << b0))] = v[j];
      }
      __syncthreads();
    }
    for (int idx = tid; idx < nt * m; idx += T) {
      const int t = idx / m, i = idx % m;
      store_elem(Y + (tb + t) * m + i, vb[t * stride + pad(i)]);
      gb[t * stride + pad(i)] = DY[(tb + t) * m + i];
    }
    __syncthreads();
    // reverse sweep with dtheta accumulation
    for (int k = passes - 1; k >= 0; --k) {
      const int s0 = k * kBitsPerPass, s1 = s0 + kBitsPerPass < L ? s0 + kBitsPerPass : L;
      const int b0 = s0 < L - ec ? s0 : L - ec;
      const int lowmask = (1 << b0) - 1;
      for (int q = tid; q < per; q += T) {
        const int base = (q & lowmask) | ((q >> b0) << (b0 + ec));
        float acc[3][4];
#pragma unroll
        for (int a = 0; a < 3; ++a)
#pragma unroll
          for (int b = 0; b < 4; ++b) acc[a][b] = 0.f;
        for (int t = 0; t < nt; ++t) {
          float* bv = vb + t * stride;
          float* bg = gb + t * stride;
          float v[8], g[8];
#pragma unroll
          for (int j = 0; j < 8; ++j)
            if (j < E) {
              v[j] = bv[pad(base | (j << b0))];
              g[j] = bg[pad(base | (j << b0))];
            }
#pragma unroll
          for (int sl = kBitsPerPass - 1; sl >= 0; --sl) {
            const int s = s0 + sl;
            if (s < s1) bwd_any(v, g, acc[sl], E, base, b0, s, Ly.cs + size_t(s) * half);
          }
#pragma unroll
          for (int j = 0; j < 8; ++j)
            if (j < E) {
              bv[pad(base | (j << b0))] = v[j];
              bg[pad(base | (j << b0))] = g[j];
            }
        }
#pragma unroll
        for (int sl = 0; sl < kBitsPerPass; ++sl) {
          const int s = s0 + sl;
          if (s >= s1) continue;
          switch (s - b0) {
            case 0: add_acc<0>(dth, acc[sl], E, base, b0, s, half); break;
            case 1: add_acc<1>(dth, acc[sl], E, base, b0, s, half); break;
            default: add_acc<2>(dth, acc[sl], E, base, b0, s, half); break;
          }
        }
      }
      __syncthreads();
    }
    for (int idx = tid; idx < nt * m; idx += T) {
      const int t = idx / m, i = idx % m;
      DX[(tb + t) * m + i] = gb[t * stride + pad(i)];
    }
    __syncthreads();
  }

  // deterministic cross-block reduction: partial -> workspace, last block sums in chunk order
  float* mine = A.part + (static_cast<size_t>(layer) * A.chunks + chunk) * nang;
  for (int k = tid; k < nang; k += T) mine[k] = dth[k];
  __threadfence();
  __syncthreads();
  __shared__ int is_last;
  if (tid == 0) {
    const unsigned prev = atomicAdd(&A.counters[layer], 1u);
    is_last = (prev == static_cast<unsigned>(A.chunks - 1));
  }
  __syncthreads();
  if (is_last) {
    __threadfence();
    const float* base = A.part + static_cast<size_t>(layer) * A.chunks * nang;
    float* out = A.dtheta + static_cast<size_t>(layer) * nang;
    for (int k = tid; k < nang; k += T) {
      float sum = 0.f;
      for (int c = 0; c < A.chunks; ++c) sum += __ldcg(base + static_cast<size_t>(c) * nang + k);
      out[k] = sum;
    }
    if (tid == 0) A.counters[layer] = 0u;
  }
}

template <typename TI, typename TO>
bq_status run_bwd(const BwdArgs& A, cudaStream_t st) {
  auto kern = k_bwd<TI, TO>;
  const size_t smem = sizeof(float) * (round4(size_t(A.L) * (A.m >> 1)) + size_t(2 * kTokens) * (pad(A.m) + 1));
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem)) != cudaSuccess)
    return BQ_ERR_CUDA;
  const unsigned grid = static_cast<unsigned>(A.layers * A.chunks);
  kern<<<grid, kBwdThreads, smem, st>>>(A);
  return cudaPeekAtLastError() == cudaSuccess ? BQ_OK : BQ_ERR_CUDA;
}

}  // namespace

int bwd_chunks(int m, int num_layers, int64_t rows) {
  if (m == 4096) return bwd4096_chunks(num_layers, rows);
  const int target_blocks = 148 * 4;
  long long c = (target_blocks + num_layers - 1) / num_layers;
  if (c > rows) c = rows;
  if (c < 1) c = 1;
  return static_cast<int>(c);
}

size_t bwd_workspace_bytes(int m, int num_layers, int chunks) {
  const int L = ilog2(m);
  return kCounterBytes + sizeof(float) * size_t(num_layers) * chunks * size_t(L) * (m >> 1);
}

bq_status launch_bwd(const KLayer* layers, int num_layers, const void* x, bq_dtype xt, void* y, bq_dtype yt,
                     const float* dy, float* dx, float* dtheta, int64_t rows, void* ws, int chunks,
                     cudaStream_t st) {
  if (layers[0].m == 4096)
    return launch_bwd4096(layers, num_layers, x, xt, y, yt, dy, dx, dtheta, rows, ws, chunks, st);
  BwdArgs A;
  A.m = layers[0].m;
  A.L = layers[0].L;
  A.chunks = chunks;
  A.layers = num_layers;
  A.rows = rows;
  A.x = x; A.y = y; A.dy = dy; A.dx = dx; A.dtheta = dtheta;
  A.counters = static_cast<unsigned*>(ws);
  A.part = reinterpret_cast<float*>(static_cast<char*>(ws) + kCounterBytes);
  for (int l = 0; l < kMaxBwdLayers; ++l) A.cs[l] = l < num_layers ? layers[l].cs : nullptr;
  if (cudaMemsetAsync(ws, 0, kCounterBytes, st) != cudaSuccess) return BQ_ERR_CUDA;
  if (xt == BQ_F32 && yt == BQ_F32) return run_bwd<float, float>(A, st);
  if (xt == BQ_F32 && yt == BQ_BF16) return run_bwd<float, __nv_bfloat16>(A, st);
  if (xt == BQ_BF16 && yt == BQ_F32) return run_bwd<__nv_bfloat16, float>(A, st);
  return run_bwd<__nv_bfloat16, __nv_bfloat16>(A, st);
}

}  // namespace bq
