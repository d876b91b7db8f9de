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
//  * the same scaled form of the inverse Q^T (stages L-1 .. 0, each rotation by
//    the negated angle), with its own coefficients, output scale and flag
//    (header[3]).
#include "bq_internal.cuh"

namespace bq {

namespace {

// One sweep of the scaled form over all stages: forward (stages 0 .. L-1, angle
// theta) or inverse (stages L-1 .. 0, angle -theta: the transposed rotation).  The
// running scale of every position starts at 1 and is multiplied by the pair's
// cosine at every stage; the coefficients of the pair (i, j) at that stage are
// alpha = -t d_j / d_i (position i) and beta = t d_i / d_j (position j), with
// t = tan of the stage's angle (negated for the inverse), both applied to the old
// values.  Returns (in *bad) 1 when a coefficient exceeds 2^60 or a scale falls
// below 2^-60 (or is NaN).
template <typename CS>
__device__ void scaled_sweep(CS cs_of, const TableLayout& tl, bool inverse, float* __restrict__ fast,
                             float* __restrict__ sigma, double* d, int* bad) {
  const int m = tl.m, L = tl.L, half = m / 2;
  const int tid = threadIdx.x, T = blockDim.x;
  for (int i = tid; i < m; i += T) d[i] = 1.0;
  __syncthreads();
  const double kCoefMax = 0x1p60, kScaleMin = 0x1p-60;
  for (int k = 0; k < L; ++k) {
    const int s = inverse ? L - 1 - k : k;
    for (int p = tid; p < half; p += T) {
      const int lowmask = (1 << s) - 1;
      const int i = ((p >> s) << (s + 1)) | (p & lowmask);
      const int j = i + (1 << s);
      double sn, c;
      cs_of(s, p, sn, c);
      const double di = d[i], dj = d[j];
      const double t = inverse ? -sn / c : sn / c;
      const double alpha = -t * dj / di;
      const double beta = t * di / dj;
      if (!(fabs(alpha) <= kCoefMax && fabs(beta) <= kCoefMax)) *bad = 1;  // also NaN
      fast[size_t(s) * m + i] = static_cast<float>(alpha);
      fast[size_t(s) * m + j] = static_cast<float>(beta);
      const double ndi = di * c, ndj = dj * c;
      if (!(fabs(ndi) >= kScaleMin && fabs(ndj) >= kScaleMin)) *bad = 1;
      d[i] = ndi;
      d[j] = ndj;
    }
    __syncthreads();
  }
  for (int i = tid; i < m; i += T) sigma[i] = static_cast<float>(d[i]);
  __syncthreads();
}

__device__ __forceinline__ void write_header(float* table, const TableLayout& tl, int bad, int bad_inv) {
  const int tid = threadIdx.x;
  if (tid < 16) {
    float v = 0.f;
    if (tid == 0) v = bad ? 0.f : 1.f;
    if (tid == 1) v = static_cast<float>(tl.m);
    if (tid == 2) v = static_cast<float>(tl.L);
    if (tid == 3) v = bad_inv ? 0.f : 1.f;
    table[tid] = v;
  }
}

__global__ void k_prepare(const float* __restrict__ theta, float* __restrict__ table, TableLayout tl) {
  extern __shared__ double d[];  // running scale of every position
  __shared__ int bad, bad_inv;
  const int half = tl.m / 2;
  const int tid = threadIdx.x, T = blockDim.x;
  float2* cs = reinterpret_cast<float2*>(table + tl.off_cs);

  for (int k = tid; k < tl.L * half; k += T) {
    double sn, c;
    sincos(static_cast<double>(theta[k]), &sn, &c);
    cs[k] = make_float2(static_cast<float>(c), static_cast<float>(sn));
  }
  if (tid == 0) bad = bad_inv = 0;
  __syncthreads();
  auto cs_of = [&](int s, int p, double& sn, double& c) { sincos(static_cast<double>(theta[s * half + p]), &sn, &c); };
  scaled_sweep(cs_of, tl, false, table + tl.off_fast, table + tl.off_sigma, d, &bad);
  scaled_sweep(cs_of, tl, true, table + tl.off_fast_inv, table + tl.off_sigma_inv, d, &bad_inv);
  write_header(table, tl, bad, bad_inv);
}

// Hadamard presets.  H_n is the butterfly at particular angles (explainer
// article, section "butterfly"): at theta = pi/4 every rotation is
// [[1, -1], [1, 1]] / sqrt(2).  theta = pi/4 + k pi/2 (k = 0..3) gives the four
// rotations with entries +-1/sqrt(2), so a product of such stages has every entry
// +-1/sqrt(n): k = 0 everywhere is the fixed Hadamard transform, random k per
// rotation a randomized one.  The angles' cos and sin are +-1/sqrt(2) exactly in
// float64 here (not float32 angles through sincos), so t = s / c is +-1, every
// coefficient of the scaled form is exactly +-1 (all positions carry the same
// |scale| at each stage) and the output scale is +-(1/sqrt(2))^L: the forward
// and inverse kernels then compute the butterfly with exact coefficient products.
__global__ void k_prepare_hadamard(const uint8_t* __restrict__ quadrant, float* __restrict__ table,
                                   float* __restrict__ theta_out, TableLayout tl) {
  extern __shared__ double d[];
  __shared__ int bad, bad_inv;
  const int half = tl.m / 2;
  const int tid = threadIdx.x, T = blockDim.x;
  float2* cs = reinterpret_cast<float2*>(table + tl.off_cs);
  const double r = 0.70710678118654752440;  // 1 / sqrt(2)
  const double kPi = 3.14159265358979323846;
  auto cs_of = [&](int s, int p, double& sn, double& c) {
    const int k = quadrant ? (quadrant[s * half + p] & 3) : 0;
    c = (k == 0 || k == 3) ? r : -r;   // cos(pi/4 + k pi/2)
    sn = (k <= 1) ? r : -r;            // sin(pi/4 + k pi/2)
  };
  for (int q = tid; q < tl.L * half; q += T) {
    double sn, c;
    cs_of(q / half, q % half, sn, c);
    cs[q] = make_float2(static_cast<float>(c), static_cast<float>(sn));
    const int k = quadrant ? (quadrant[q] & 3) : 0;
    if (theta_out) theta_out[q] = static_cast<float>(kPi / 4 + (k < 2 ? k : k - 4) * (kPi / 2));
  }
  if (tid == 0) bad = bad_inv = 0;
  __syncthreads();
  // every coefficient of both sweeps is exactly +-1 (t = +-1 and all positions carry
  // the same |scale| at each stage), so the range checks always pass
  scaled_sweep(cs_of, tl, false, table + tl.off_fast, table + tl.off_sigma, d, &bad);
  scaled_sweep(cs_of, tl, true, table + tl.off_fast_inv, table + tl.off_sigma_inv, d, &bad_inv);
  write_header(table, tl, bad, bad_inv);
}

// Position held in register slot e by thread t of a 128-thread row group, for
// the three passes of the specialised n = 4096 kernel (see bq_fast4096.cu).
__device__ __forceinline__ int pos_pass(int pass, int t, int e) {
  if (pass == 0) return t * 32 + e;
  if (pass == 1) return (t & 31) | (e << 5) | ((t >> 5) << 10);
  return (e & 7) | (t << 3) | ((e >> 3) << 10);
}

// Tensor-memory image of the n = 4096 kernel: lane t, column c, stored as float4
// blocks [c / 4][t] so that a warp filling four consecutive columns of its 32
// lanes reads one contiguous 512-byte run.
//   columns [0,160):   pass 0 stages 0..4   (32 columns per stage)
//   columns [160,320): pass 1 stages 5..9
//   columns [320,384): pass 2 stages 10, 11
//   columns [384,416): output scale of the 32 positions thread t ends with
//                      (pass-2 layout for the forward, pass-0 for the inverse)
// Inside a stage block, column 4q + e (e = 0, 1) is the coefficient of the low
// element of the thread's (2q + e)-th pair and column 4q + 2 + e that of its
// high element: (alpha, beta) of the scaled form, or (cos, sin) when the
// scaled form is out of range (header flag 0; the output scale is then 1).
// The inverse image has the same stage columns, filled from the inverse's own
// scaled form (header[3]) or with (cos, sin).
__global__ void k_image4096(float* __restrict__ table, TableLayout tl) {
  int idx = blockIdx.x * blockDim.x + threadIdx.x;
  const bool inv = idx >= kImageLanes * kImageCols;
  if (inv) idx -= kImageLanes * kImageCols;
  if (idx >= kImageLanes * (inv ? kImageInvCols : kImageCols)) return;
  const int ncol = inv ? kImageInvCols : kImageCols;
  const int t = idx / ncol, col = idx % ncol;
  const bool scaled = inv ? table[3] == 1.f : table[0] == 1.f;
  const float2* cs = reinterpret_cast<const float2*>(table + tl.off_cs);
  const float* fast = table + (inv ? tl.off_fast_inv : tl.off_fast);
  const float* sigma = table + (inv ? tl.off_sigma_inv : tl.off_sigma);
  float v;
  if (col >= 384) {
    v = scaled ? sigma[pos_pass(inv ? 0 : 2, t, col - 384)] : 1.f;
  } else {
    int pass, stage, sb;
    if (col < 160) { pass = 0; stage = col / 32; sb = stage; }
    else if (col < 320) { pass = 1; stage = 5 + (col - 160) / 32; sb = stage - 5; }
    else { pass = 2; stage = 10 + (col - 320) / 32; sb = stage - 7; }
    const int w = col & 31, q = w >> 2, high = (w >> 1) & 1, e = w & 1;
    const int k = 2 * q + e;
    const int j = ((k >> sb) << (sb + 1)) | (k & ((1 << sb) - 1));
    const int low = pos_pass(pass, t, j);
    if (scaled) {
      v = fast[size_t(stage) * tl.m + (high ? pos_pass(pass, t, j | (1 << sb)) : low)];
    } else {
      const int p = ((low >> (stage + 1)) << stage) | (low & ((1 << stage) - 1));
      const float2 c = cs[size_t(stage) * (tl.m >> 1) + p];
      v = high ? c.y : c.x;
    }
  }
  table[(inv ? tl.off_image_inv : tl.off_image) + (size_t(col >> 2) * kImageLanes + t) * 4 + (col & 3)] = v;
}

}  // namespace

bq_status launch_prepare_any(const float* theta, const uint8_t* quadrant, float* theta_out, bool hadamard, int m,
                             float* table, cudaStream_t st);

bq_status launch_prepare(const float* theta, int m, float* table, cudaStream_t st) {
  return launch_prepare_any(theta, nullptr, nullptr, false, m, table, st);
}

bq_status launch_prepare_hadamard(const uint8_t* quadrant, float* theta_out, int m, float* table, cudaStream_t st) {
  return launch_prepare_any(nullptr, quadrant, theta_out, true, m, table, st);
}

bq_status launch_prepare_any(const float* theta, const uint8_t* quadrant, float* theta_out, bool hadamard, int m,
                             float* table, cudaStream_t st) {
  TableLayout tl = table_layout(m);
  const size_t smem = sizeof(double) * size_t(m);
  if (smem > 48 * 1024) {
    const cudaError_t e =
        hadamard ? cudaFuncSetAttribute(k_prepare_hadamard, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem))
                 : cudaFuncSetAttribute(k_prepare, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem));
    if (e != cudaSuccess) return BQ_ERR_CUDA;
  }
  if (hadamard)
    k_prepare_hadamard<<<1, 1024, smem, st>>>(quadrant, table, theta_out, tl);
  else
    k_prepare<<<1, 1024, smem, st>>>(theta, table, tl);
  if (m == 4096) {
    const int total = kImageLanes * (kImageCols + kImageInvCols);
    k_image4096<<<(total + 255) / 256, 256, 0, st>>>(table, tl);
  }
  return cudaPeekAtLastError() == cudaSuccess ? BQ_OK : BQ_ERR_CUDA;
}

}  // namespace bq
