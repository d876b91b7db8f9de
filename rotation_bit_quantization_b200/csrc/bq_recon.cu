// Reconstruction loss of one linear layer under weight quantization, with a
// straight-through estimator, for calibrating the angles.
//
// The calibration loss keeps the quantized layer's output close to the original
// one (explainer article, section "training & results"), using the invariance
// y = W x = (W Q^T)(Q x) (ButterflyQuant abstract).  For weights W [out][n] and T
// calibration tokens x [T][n]:
//   V = W Q^T (row o is Q w_o),  W_hat = dequantize(RTN(V)),  x~_t = Q x_t,
//   r[t][o] = (W_hat x~_t)_o - (W x_t)_o,      loss = (1/T) sum ||r_t||^2,
// and with dW_hat / dV taken as the identity (straight-through estimator)
//   G_x = (2/T) r W_hat  [T][n],   G_v = (2/T) r^T x~  [out][n],
//   dtheta = backward(x, G_x) + backward(W, G_v).
//
// Composition of the library's own calls: bq_weight_rotate_pack gives RTN(V)
// (bitwise the quantizer applied to the float32 forward output), a dequantize
// kernel gives W_hat, bq_butterfly_fwd gives x~, four small tiled FP32 GEMMs give
// W_hat x~^T, W x^T, G_x and G_v, a residual kernel forms r and its squares
// (summed in a fixed order), and two bq_butterfly_bwd calls plus an add give
// dtheta.  Everything is deterministic.
#include "bq_internal.cuh"

namespace bq {
namespace {

// ------------------------------------------------------------------ FP32 GEMM
//
// C[i][j] = alpha * sum_k A(i, k) B(k, j) + beta * C[i][j], with A(i, k) =
// A[i * sam + k * sak] and B(k, j) = B[k * sbk + j * sbn] (so any transposition is a
// choice of strides).  64 x 64 tiles, 16-deep k slices, 4 x 4 outputs per thread;
// each output's sum runs over k in order, so results are reproducible.
constexpr int kTM = 64, kTN = 64, kTK = 16;

__global__ void __launch_bounds__(256) k_sgemm(int M, int N, int K, float alpha, const float* __restrict__ A,
                                               long long sam, long long sak, const float* __restrict__ B,
                                               long long sbk, long long sbn, float beta, float* __restrict__ C,
                                               long long ldc) {
  __shared__ float As[kTK][kTM + 4];
  __shared__ float Bs[kTK][kTN + 4];
  const int tid = threadIdx.x, tx = tid % 16, ty = tid / 16;
  const int m0 = blockIdx.y * kTM, n0 = blockIdx.x * kTN;
  float acc[4][4] = {};
  for (int k0 = 0; k0 < K; k0 += kTK) {
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int idx = tid + 256 * i;
      // A tile: k fastest when A is k-contiguous, else i fastest
      int mm, kk;
      if (sak == 1) { mm = idx / kTK; kk = idx % kTK; } else { kk = idx / kTM; mm = idx % kTM; }
      const int gm = m0 + mm, gk = k0 + kk;
      As[kk][mm] = (gm < M && gk < K) ? A[gm * sam + gk * sak] : 0.f;
      int nn, kb;
      if (sbn == 1) { kb = idx / kTN; nn = idx % kTN; } else { nn = idx / kTK; kb = idx % kTK; }
      const int gn = n0 + nn, gkb = k0 + kb;
      Bs[kb][nn] = (gn < N && gkb < K) ? B[gkb * sbk + gn * sbn] : 0.f;
    }
    __syncthreads();
#pragma unroll
    for (int kk = 0; kk < kTK; ++kk) {
      float a[4], b[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) a[i] = As[kk][ty * 4 + i];
#pragma unroll
      for (int j = 0; j < 4; ++j) b[j] = Bs[kk][tx * 4 + j];
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(a[i], b[j], acc[i][j]);
    }
    __syncthreads();
  }
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int gm = m0 + ty * 4 + i, gn = n0 + tx * 4 + j;
      if (gm < M && gn < N) {
        float* c = C + gm * ldc + gn;
        *c = beta == 0.f ? alpha * acc[i][j] : fmaf(beta, *c, alpha * acc[i][j]);
      }
    }
}

bq_status sgemm(int M, int N, int K, float alpha, const float* A, long long sam, long long sak, const float* B,
                long long sbk, long long sbn, float beta, float* C, long long ldc, cudaStream_t st) {
  dim3 grid((N + kTN - 1) / kTN, (M + kTM - 1) / kTM);
  k_sgemm<<<grid, 256, 0, st>>>(M, N, K, alpha, A, sam, sak, B, sbk, sbn, beta, C, ldc);
  return cudaPeekAtLastError() == cudaSuccess ? BQ_OK : BQ_ERR_CUDA;
}

// ------------------------------------------------------------------ elementwise pieces

// W_hat = (q - z) s per group, from packed little-endian codes and fp16 scale / zero
__global__ void k_dequant(const uint8_t* __restrict__ codes, const uint16_t* __restrict__ scale,
                          const uint16_t* __restrict__ zero, long long rows, int n, int bits, int group,
                          float* __restrict__ out) {
  const long long total = rows * n;
  for (long long i = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; i < total;
       i += static_cast<long long>(gridDim.x) * blockDim.x) {
    const long long row = i / n;
    const int col = static_cast<int>(i % n);
    const int per = 8 / bits;
    const uint8_t byte = codes[row * (n / per) + col / per];
    const int q = (byte >> (bits * (col % per))) & ((1 << bits) - 1);
    const long long gi = row * (n / group) + col / group;
    const float s = __half2float(__ushort_as_half(scale[gi]));
    const float z = __half2float(__ushort_as_half(zero[gi]));
    out[i] = (static_cast<float>(q) - z) * s;
  }
}

// r = P - R in place, and per-block sums of r^2 (fixed order) into part[block]
__global__ void __launch_bounds__(256) k_residual(float* __restrict__ p, const float* __restrict__ r, long long count,
                                                  double* __restrict__ part) {
  __shared__ double sh[256];
  double acc = 0.0;
  for (long long i = blockIdx.x * 256LL + threadIdx.x; i < count; i += static_cast<long long>(gridDim.x) * 256) {
    const float d = p[i] - r[i];
    p[i] = d;
    acc += static_cast<double>(d) * d;
  }
  sh[threadIdx.x] = acc;
  __syncthreads();
  for (int h = 128; h > 0; h >>= 1) {
    if (threadIdx.x < h) sh[threadIdx.x] += sh[threadIdx.x + h];
    __syncthreads();
  }
  if (threadIdx.x == 0) part[blockIdx.x] = sh[0];
}

__global__ void k_finish(const double* __restrict__ part, int nparts, double scale, float* __restrict__ loss,
                         float* __restrict__ a, const float* __restrict__ b, long long count) {
  if (blockIdx.x == 0 && threadIdx.x == 0) {
    double s = 0.0;
    for (int i = 0; i < nparts; ++i) s += part[i];
    *loss = static_cast<float>(s * scale);
  }
  for (long long i = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; i < count;
       i += static_cast<long long>(gridDim.x) * blockDim.x)
    a[i] += b[i];
}

constexpr int kResidualBlocks = 512;

struct ReconLayout {
  size_t codes, scale, zero, what, xt, p, r, gx, gv, ybuf, dxbuf, dthx, dthv, part, bwdws, total;
};

size_t align256(size_t v) { return (v + 255) & ~size_t(255); }

ReconLayout recon_layout(int n, long long out, long long T, int bits, int group) {
  const int L = ilog2(n);
  const long long rmax = out > T ? out : T;
  const size_t bwd = bwd_workspace_bytes(n, 1, bwd_chunks(n, 1, rmax));
  ReconLayout l;
  size_t o = 0;
  auto take = [&](size_t bytes) { const size_t at = o; o = align256(o + bytes); return at; };
  l.codes = take(size_t(out) * n * bits / 8);
  l.scale = take(sizeof(uint16_t) * size_t(out) * (n / group));
  l.zero = take(sizeof(uint16_t) * size_t(out) * (n / group));
  l.what = take(sizeof(float) * size_t(out) * n);
  l.xt = take(sizeof(float) * size_t(T) * n);
  l.p = take(sizeof(float) * size_t(T) * out);
  l.r = take(sizeof(float) * size_t(T) * out);
  l.gx = take(sizeof(float) * size_t(T) * n);
  l.gv = take(sizeof(float) * size_t(out) * n);
  l.ybuf = take(sizeof(float) * size_t(rmax) * n);
  l.dxbuf = take(sizeof(float) * size_t(rmax) * n);
  l.dthx = take(sizeof(float) * size_t(L) * (n / 2));
  l.dthv = take(sizeof(float) * size_t(L) * (n / 2));
  l.part = take(sizeof(double) * kResidualBlocks);
  l.bwdws = take(bwd);
  l.total = o;
  return l;
}

bool ok_group(int n, int bits, int group) {
  return (bits == 2 || bits == 4) && group >= 32 && group % 32 == 0 && group <= kMaxGroup && n % group == 0;
}

}  // namespace
}  // namespace bq

using namespace bq;

extern "C" size_t bq_reconstruction_workspace_size(int32_t n, int64_t out_features, int64_t tokens, int32_t bits,
                                                   int32_t group) {
  if (n < 2 || n > kMaxM || (n & (n - 1)) || out_features < 1 || tokens < 1 || !ok_group(n, bits, group)) return 0;
  return recon_layout(n, out_features, tokens, bits, group).total;
}

extern "C" bq_status bq_reconstruction_loss(const bq_layer* layer, const float* w, int64_t out_features,
                                            const float* x, int64_t tokens, int32_t bits, int32_t group,
                                            float* dtheta, float* loss, void* workspace, size_t workspace_bytes,
                                            void* stream) {
  if (!layer || !w || !x || !dtheta || !loss || !workspace) return BQ_ERR_INVALID_ARG;
  const int n = layer->n;
  if (layer->r != 1 || layer->m != n || layer->O) return layer->r != 1 ? BQ_ERR_UNSUPPORTED : BQ_ERR_INVALID_ARG;
  const size_t need = bq_reconstruction_workspace_size(n, out_features, tokens, bits, group);
  if (need == 0) return BQ_ERR_INVALID_ARG;
  if (workspace_bytes < need || (reinterpret_cast<uintptr_t>(workspace) & 255u)) return BQ_ERR_WORKSPACE;
  const ReconLayout lay = recon_layout(n, out_features, tokens, bits, group);
  char* ws = static_cast<char*>(workspace);
  auto F = [&](size_t off) { return reinterpret_cast<float*>(ws + off); };
  auto st = static_cast<cudaStream_t>(stream);
  const long long out = out_features, T = tokens;
  bq_status s;
  // W_hat = dequantize(RTN(W Q^T));  x~ = Q x
  uint8_t* codes = reinterpret_cast<uint8_t*>(ws + lay.codes);
  uint16_t* scale = reinterpret_cast<uint16_t*>(ws + lay.scale);
  uint16_t* zero = reinterpret_cast<uint16_t*>(ws + lay.zero);
  if ((s = bq_weight_rotate_pack(layer, w, BQ_F32, out, bits, group, codes, scale, zero, stream)) != BQ_OK) return s;
  {
    long long grid = (out * n + 255) / 256;
    if (grid > 4096) grid = 4096;
    k_dequant<<<static_cast<unsigned>(grid), 256, 0, st>>>(codes, scale, zero, out, n, bits, group, F(lay.what));
    if (cudaPeekAtLastError() != cudaSuccess) return BQ_ERR_CUDA;
  }
  if ((s = bq_butterfly_fwd(layer, x, BQ_F32, F(lay.xt), BQ_F32, T, stream)) != BQ_OK) return s;
  // P = x~ W_hat^T, R = x W^T  ([T][out]);  r = P - R and sum r^2
  if ((s = sgemm(T, out, n, 1.f, F(lay.xt), n, 1, F(lay.what), 1, n, 0.f, F(lay.p), out, st)) != BQ_OK) return s;
  if ((s = sgemm(T, out, n, 1.f, x, n, 1, w, 1, n, 0.f, F(lay.r), out, st)) != BQ_OK) return s;
  double* part = reinterpret_cast<double*>(ws + lay.part);
  k_residual<<<kResidualBlocks, 256, 0, st>>>(F(lay.p), F(lay.r), T * out, part);
  if (cudaPeekAtLastError() != cudaSuccess) return BQ_ERR_CUDA;
  // G_x = (2/T) r W_hat  [T][n];  G_v = (2/T) r^T x~  [out][n]
  const float g = static_cast<float>(2.0 / static_cast<double>(T));
  if ((s = sgemm(T, n, out, g, F(lay.p), out, 1, F(lay.what), n, 1, 0.f, F(lay.gx), n, st)) != BQ_OK) return s;
  if ((s = sgemm(out, n, T, g, F(lay.p), 1, out, F(lay.xt), n, 1, 0.f, F(lay.gv), n, st)) != BQ_OK) return s;
  // dtheta = backward(x, G_x) + backward(W, G_v)
  const size_t bwdbytes = workspace_bytes - lay.bwdws;
  if ((s = bq_butterfly_bwd(layer, 1, x, BQ_F32, F(lay.ybuf), BQ_F32, F(lay.gx), F(lay.dxbuf), F(lay.dthx), T,
                            ws + lay.bwdws, bwdbytes, stream)) != BQ_OK)
    return s;
  if ((s = bq_butterfly_bwd(layer, 1, w, BQ_F32, F(lay.ybuf), BQ_F32, F(lay.gv), F(lay.dxbuf), dtheta, out,
                            ws + lay.bwdws, bwdbytes, stream)) != BQ_OK)
    return s;
  const long long nth = static_cast<long long>(ilog2(n)) * (n / 2);
  k_finish<<<static_cast<unsigned>((nth + 255) / 256), 256, 0, st>>>(part, kResidualBlocks, 1.0 / static_cast<double>(T),
                                                                    loss, dtheta, F(lay.dthx), nth);
  return cudaPeekAtLastError() == cudaSuccess ? BQ_OK : BQ_ERR_CUDA;
}
