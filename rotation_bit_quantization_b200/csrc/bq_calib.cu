// Calibration support: the uniformity regulariser of the rotated activations and
// a plain gradient step on the angles.
//
// The angles are learned with a loss that includes a uniformity regularisation on
// the post-transformation activations (ButterflyQuant abstract): the KL
// divergence between the rotated activations' distribution and the uniform
// distribution over the quantization intervals (explainer article, section
// "training & results").  Per group of `group` outputs of a row:
//   s, z      the group's RTN scale and zero point (rtn_params: the quantizer's
//             own float32 rules, so the bins are the levels the codes use);
//   u_i       = y_i / s + z clamped to [0, qmax], spread over its two nearest
//             levels with the triangular kernel max(0, 1 - |u - c|);
//   p_c       = (1/g) sum_i w_c(u_i),  p~_c = (p_c + eps) / (1 + B eps),  B = qmax + 1;
//   KL        = sum_c p~_c log(B p~_c);  loss = mean of KL over all groups.
// Gradient (s, z held constant; zero outside 0 < u < qmax): for u in (k, k+1)
//   dloss/dy = (log p~_{k+1} - log p~_k) / (s g G (1 + B eps)),  G = number of groups.
//
// One warp per group.  Each lane accumulates its values' weights into its own
// column of a per-warp [B][32] histogram in shared memory (no atomics: the sum
// order is fixed, so results are reproducible), the columns are added in a fixed
// order, and each level's logarithm is taken once and fetched by shuffle.
#include <cfloat>

#include "bq_rtn.cuh"

namespace bq {
namespace {

constexpr int kCalWarps = 8;

template <int BITS, int GROUP>
__global__ void __launch_bounds__(32 * kCalWarps) k_uniformity(const float* __restrict__ y, long long groups,
                                                               float eps, float gscale, float* __restrict__ kl_group,
                                                               float* __restrict__ dy) {
  constexpr int B = 1 << BITS, QMAX = B - 1, E = GROUP / 32;
  __shared__ float hist[kCalWarps][B][32];
  const int lane = threadIdx.x & 31, wl = threadIdx.x >> 5;
  const float qmax = static_cast<float>(QMAX);
  const long long stride = static_cast<long long>(gridDim.x) * kCalWarps;
#pragma unroll 1
  for (long long g = static_cast<long long>(blockIdx.x) * kCalWarps + wl; g < groups; g += stride) {
    const float* src = y + g * GROUP + lane * E;
    float v[E];
#pragma unroll
    for (int q = 0; q < E; q += (E >= 4 ? 4 : E)) {
      if constexpr (E >= 4) {
        const float4 t = *reinterpret_cast<const float4*>(src + q);
        v[q] = t.x; v[q + 1] = t.y; v[q + 2] = t.z; v[q + 3] = t.w;
      } else {
        const float2 t = *reinterpret_cast<const float2*>(src + q);
        v[q] = t.x; v[q + 1] = t.y;
      }
    }
    float lo = v[0], hi = v[0];
#pragma unroll
    for (int q = 1; q < E; ++q) {
      lo = fminf(lo, v[q]);
      hi = fmaxf(hi, v[q]);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      lo = fminf(lo, __shfl_xor_sync(0xffffffffu, lo, o));
      hi = fmaxf(hi, __shfl_xor_sync(0xffffffffu, hi, o));
    }
    const RtnParams p = rtn_params(lo, hi, qmax);
    const float z = __fadd_rn(p.mz, -12582912.f);
#pragma unroll
    for (int c = 0; c < B; ++c) hist[wl][c][lane] = 0.f;
    float u[E];
    int k[E];
#pragma unroll
    for (int q = 0; q < E; ++q) {
      u[q] = fmaf(v[q], p.inv, z);
      const float uc = fminf(fmaxf(u[q], 0.f), qmax);
      k[q] = min(static_cast<int>(uc), QMAX - 1);  // uc >= 0: truncation is floor
      const float f = uc - static_cast<float>(k[q]);
      hist[wl][k[q]][lane] += 1.f - f;
      hist[wl][k[q] + 1][lane] += f;
    }
    __syncwarp();
    // level c = lane % B: add the columns in a fixed order per level, level c starting
    // at column c so that the lanes of one step hit distinct banks
    const int c = lane % B;
    float cnt = 0.f;
#pragma unroll 8
    for (int l = 0; l < 32; ++l) cnt += hist[wl][c][(l + c) & 31];
    const float pt = (cnt * (1.f / static_cast<float>(GROUP)) + eps) / (1.f + static_cast<float>(B) * eps);
    const float lg = logf(static_cast<float>(B) * pt);
    float term = lane < B ? pt * lg : 0.f;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) term += __shfl_xor_sync(0xffffffffu, term, o);
    if (lane == 0) kl_group[g] = term;
    if (dy) {
      const float sc = gscale / p.s;
      float d[E];
#pragma unroll
      for (int q = 0; q < E; ++q) {
        const float l0 = __shfl_sync(0xffffffffu, lg, k[q]), l1 = __shfl_sync(0xffffffffu, lg, k[q] + 1);
        d[q] = (u[q] > 0.f && u[q] < qmax) ? (l1 - l0) * sc : 0.f;
      }
      float* dst = dy + g * GROUP + lane * E;
#pragma unroll
      for (int q = 0; q < E; q += (E >= 4 ? 4 : E)) {
        if constexpr (E >= 4) *reinterpret_cast<float4*>(dst + q) = make_float4(d[q], d[q + 1], d[q + 2], d[q + 3]);
        else *reinterpret_cast<float2*>(dst + q) = make_float2(d[q], d[q + 1]);
      }
    }
    __syncwarp();  // the histogram columns are reused by the next group
  }
}

// loss = (sum of kl_group) / count, summed in a fixed order by one CTA
__global__ void __launch_bounds__(1024) k_mean(const float* __restrict__ v, long long count, float* __restrict__ out) {
  __shared__ double part[1024];
  double acc = 0.0;
  for (long long i = threadIdx.x; i < count; i += 1024) acc += static_cast<double>(v[i]);
  part[threadIdx.x] = acc;
  __syncthreads();
  for (int h = 512; h > 0; h >>= 1) {
    if (threadIdx.x < h) part[threadIdx.x] += part[threadIdx.x + h];
    __syncthreads();
  }
  if (threadIdx.x == 0) *out = static_cast<float>(part[0] / static_cast<double>(count));
}

__global__ void k_sgd(float* __restrict__ theta, const float* __restrict__ dtheta, long long count, float lr) {
  for (long long i = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; i < count;
       i += static_cast<long long>(gridDim.x) * blockDim.x)
    theta[i] = fmaf(-lr, dtheta[i], theta[i]);
}

template <int BITS, int GROUP>
bq_status run_uniformity(const float* y, long long groups, float eps, float gscale, float* kl, float* dy,
                         cudaStream_t st) {
  int dev = 0, sms = 148;
  if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  long long grid = (groups + kCalWarps - 1) / kCalWarps;
  const long long cap = static_cast<long long>(sms) * 8;
  if (grid > cap) grid = cap;
  if (grid < 1) grid = 1;
  k_uniformity<BITS, GROUP><<<static_cast<unsigned>(grid), 32 * kCalWarps, 0, st>>>(y, groups, eps, gscale, kl, dy);
  return cudaPeekAtLastError() == cudaSuccess ? BQ_OK : BQ_ERR_CUDA;
}

template <int BITS>
bq_status uniformity_bits(const float* y, long long groups, int group, float eps, float gscale, float* kl, float* dy,
                          cudaStream_t st) {
  switch (group) {
    case 64: return run_uniformity<BITS, 64>(y, groups, eps, gscale, kl, dy, st);
    case 128: return run_uniformity<BITS, 128>(y, groups, eps, gscale, kl, dy, st);
    default: return run_uniformity<BITS, 256>(y, groups, eps, gscale, kl, dy, st);
  }
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace
}  // namespace bq

using namespace bq;

extern "C" bq_status bq_uniformity_loss(const float* y, int64_t rows, int32_t n, int32_t bits, int32_t group,
                                        float eps, float* kl_group, float* dy, float* loss, void* stream) {
  if (rows < 0 || n <= 0 || (bits != 2 && bits != 4)) return BQ_ERR_INVALID_ARG;
  if (group != 64 && group != 128 && group != 256) return BQ_ERR_INVALID_ARG;
  if (n % group != 0 || !(eps > 0.f && eps < 1.f)) return BQ_ERR_INVALID_ARG;
  if (rows == 0) return BQ_OK;
  if (!y || !kl_group || !aligned16(y) || (dy && !aligned16(dy))) return BQ_ERR_INVALID_ARG;
  const long long groups = static_cast<long long>(rows) * (n / group);
  const int B = 1 << bits;
  const double gscale = 1.0 / (static_cast<double>(group) * static_cast<double>(groups) * (1.0 + B * double(eps)));
  auto st = static_cast<cudaStream_t>(stream);
  bq_status s = bits == 4 ? uniformity_bits<4>(y, groups, group, eps, static_cast<float>(gscale), kl_group, dy, st)
                          : uniformity_bits<2>(y, groups, group, eps, static_cast<float>(gscale), kl_group, dy, st);
  if (s != BQ_OK || !loss) return s;
  k_mean<<<1, 1024, 0, st>>>(kl_group, groups, loss);
  return cudaPeekAtLastError() == cudaSuccess ? BQ_OK : BQ_ERR_CUDA;
}

extern "C" bq_status bq_angle_sgd(float* theta, const float* dtheta, int64_t count, float lr, void* stream) {
  if (count < 0 || !(lr == lr)) return BQ_ERR_INVALID_ARG;
  if (count == 0) return BQ_OK;
  if (!theta || !dtheta) return BQ_ERR_INVALID_ARG;
  long long grid = (count + 255) / 256;
  if (grid > 4096) grid = 4096;
  k_sgd<<<static_cast<unsigned>(grid), 256, 0, static_cast<cudaStream_t>(stream)>>>(theta, dtheta, count, lr);
  return cudaPeekAtLastError() == cudaSuccess ? BQ_OK : BQ_ERR_CUDA;
}
