// K0: per-layer angle preparation.
//
// The butterfly's rotations are parameterised by continuous angles
// (ButterflyQuant abstract; explainer article, section "butterfly").  This
// kernel turns one layer's angles into the table every transform kernel reads:
//
//  * cs[s][p] = (cos, sin) of theta[s][p], float64 sincos rounded to float32;
//  * the scaled ("square-root-free") rotation form.  A rotation
//        y_i = c x_i - s x_j,   y_j = s x_i + c x_j
//    equals c * (x_i - t x_j, x_j + t x_i) with t = s / c.  Carrying every
//    element as x_i = d_i a_i with a data-independent scale d_i turns each
//    rotation into two FMAs on the a's:
//        a_i <- a_i + alpha a_j,  alpha = -t d_j / d_i
//        a_j <- a_j + beta  a_i,  beta  =  t d_i / d_j     (old a_i, a_j)
//    with d_i, d_j <- c d_i, c d_j.  The scales depend only on the angles, so
//    they are tracked here in float64 stage by stage and the final d becomes
//    the per-position output scale sigma.  Rounding error per rotation stays
//    within a few ulps of |c x_i| + |s x_j|, the same order as the plain form.
//    When any scale leaves [2^-60, 1] or any coefficient exceeds 2^60 (angles
//    near +-pi/2 chained over many stages), header[0] is cleared and the
//    kernels use the plain cos/sin form for this layer.
#include "bq_internal.cuh"

namespace bq {

namespace {

__global__ void k_prepare(const float* __restrict__ theta, float* __restrict__ table, TableLayout tl) {
  extern __shared__ double d[];  // running scale of every position
  __shared__ int bad;
  const int m = tl.m, L = tl.L, half = m / 2;
  const int tid = threadIdx.x, T = blockDim.x;
  float2* cs = reinterpret_cast<float2*>(table + tl.off_cs);
  float* fast = table + tl.off_fast;
  float* sigma = table + tl.off_sigma;

  for (int k = tid; k < L * half; k += T) {
    double sn, c;
    sincos(static_cast<double>(theta[k]), &sn, &c);
    cs[k] = make_float2(static_cast<float>(c), static_cast<float>(sn));
  }
  for (int i = tid; i < m; i += T) d[i] = 1.0;
  if (tid == 0) bad = 0;
  __syncthreads();

  const double kCoefMax = 0x1p60, kScaleMin = 0x1p-60;
  for (int s = 0; s < L; ++s) {
    for (int p = tid; p < half; p += T) {
      const int lowmask = (1 << s) - 1;
      const int i = ((p >> s) << (s + 1)) | (p & lowmask);
      const int j = i + (1 << s);
      double sn, c;
      sincos(static_cast<double>(theta[s * half + p]), &sn, &c);
      const double di = d[i], dj = d[j];
      const double t = sn / c;
      const double alpha = -t * dj / di;
      const double beta = t * di / dj;
      if (!(fabs(alpha) <= kCoefMax && fabs(beta) <= kCoefMax)) bad = 1;  // also NaN
      fast[size_t(s) * m + i] = static_cast<float>(alpha);
      fast[size_t(s) * m + j] = static_cast<float>(beta);
      const double ndi = di * c, ndj = dj * c;
      if (!(fabs(ndi) >= kScaleMin && fabs(ndj) >= kScaleMin)) bad = 1;
      d[i] = ndi;
      d[j] = ndj;
    }
    __syncthreads();
  }
  for (int i = tid; i < m; i += T) sigma[i] = static_cast<float>(d[i]);
  __syncthreads();
  if (tid < 16) {
    float v = 0.f;
    if (tid == 0) v = bad ? 0.f : 1.f;
    if (tid == 1) v = static_cast<float>(m);
    if (tid == 2) v = static_cast<float>(L);
    table[tid] = v;
  }
}

}  // namespace

bq_status launch_prepare(const float* theta, int m, float* table, cudaStream_t st) {
  TableLayout tl = table_layout(m);
  const size_t smem = sizeof(double) * size_t(m);
  if (smem > 48 * 1024) {
    if (cudaFuncSetAttribute(k_prepare, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem)) != cudaSuccess)
      return BQ_ERR_CUDA;
  }
  k_prepare<<<1, 1024, smem, st>>>(theta, table, tl);
  return cudaPeekAtLastError() == cudaSuccess ? BQ_OK : BQ_ERR_CUDA;
}

}  // namespace bq
