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
// Each lane accumulates its values' weights into its own column of a per-warp
// [B][32] histogram in shared memory (each address has one writer, so the order
// of the additions is fixed and results are reproducible), a group's columns are
// added in a fixed order, and each level's logarithm is taken once; the
// differences of successive logarithms (the gradient's numerators) go back into
// each lane's own column, one read per value for the gradient.  (Two copies per lane, even
// and odd values, measured slower: the chains of read-modify-writes are not the
// limit.)  The loss (the mean over groups) is summed by a cluster of eight CTAs,
// each over a fixed eighth, and added up in rank order by the first: one CTA alone
// took about 100 us for the 2M per-group values of a 65536 x 4096 batch.
#include <cfloat>

#include "bq_rtn.cuh"

namespace bq {
namespace {

constexpr int kCalWarps = 8;

// Each warp handles NG = 32 / GL groups at once with GL = GROUP / 32 lanes per
// group and 32 values per lane (float4 chunks GL j + q of the group for lane q),
// so the per-group work (scale and zero point, the histogram's column sums, the
// logarithms) is spread over the warp instead of repeated by all of its lanes.
template <int BITS, int GROUP>
__global__ void __launch_bounds__(32 * kCalWarps) k_uniformity(const float* __restrict__ y, long long groups,
                                                               float eps, float gscale, float* __restrict__ kl_group,
                                                               float* __restrict__ dy) {
  constexpr int B = 1 << BITS, QMAX = B - 1, GL = GROUP / 32, NG = 32 / GL;
  constexpr int BPL = B >= GL ? B / GL : 1;  // levels each lane of a group sums
  __shared__ float hist[kCalWarps][B][32];
  const int lane = threadIdx.x & 31, wl = threadIdx.x >> 5;
  const int gi = lane / GL, q = lane % GL;
  const float qmax = static_cast<float>(QMAX);
  const long long stride = static_cast<long long>(gridDim.x) * kCalWarps * NG;
#pragma unroll 1
  for (long long g0 = (static_cast<long long>(blockIdx.x) * kCalWarps + wl) * NG; g0 < groups; g0 += stride) {
    const long long g = g0 + gi;
    const bool live = g < groups;  // the last warp may hold fewer than NG groups
    const float* src = y + (live ? g : g0) * GROUP;
    float v[32];
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const float4 t = *reinterpret_cast<const float4*>(src + 4 * (GL * j + q));
      v[4 * j] = t.x; v[4 * j + 1] = t.y; v[4 * j + 2] = t.z; v[4 * j + 3] = t.w;
    }
    float lo = v[0], hi = v[0];
#pragma unroll
    for (int e = 1; e < 32; ++e) {
      lo = fminf(lo, v[e]);
      hi = fmaxf(hi, v[e]);
    }
#pragma unroll
    for (int o = GL / 2; o > 0; o >>= 1) {
      lo = fminf(lo, __shfl_xor_sync(0xffffffffu, lo, o));
      hi = fmaxf(hi, __shfl_xor_sync(0xffffffffu, hi, o));
    }
    const RtnParams p = rtn_params(lo, hi, qmax);
    const float z = __fadd_rn(p.mz, -12582912.f);
#pragma unroll
    for (int c = 0; c < B; ++c) hist[wl][c][lane] = 0.f;
    __syncwarp();
    // soft histogram: each lane adds into its own column (the only writer of those
    // addresses, so a plain read-modify-write in program order)
#pragma unroll
    for (int e = 0; e < 32; ++e) {
      const float uc = fminf(fmaxf(fmaf(v[e], p.inv, z), 0.f), qmax);
      const int k = min(static_cast<int>(uc), QMAX - 1);  // uc >= 0: truncation is floor
      const float f = uc - static_cast<float>(k);
      hist[wl][k][lane] += 1.f - f;
      hist[wl][k + 1][lane] += f;
    }
    __syncwarp();
    // levels q BPL .. q BPL + BPL - 1 of this lane's group: its GL columns, in a fixed
    // order per level that starts at column q (the group's lanes hit distinct banks)
    float term = 0.f, lgv[BPL];
#pragma unroll
    for (int b = 0; b < BPL; ++b) {
      const int c = q * BPL + b;
      lgv[b] = 0.f;
      if (c < B) {
        float cnt = 0.f;
#pragma unroll
        for (int l = 0; l < GL; ++l) cnt += hist[wl][c][gi * GL + ((l + q) & (GL - 1))];
        const float pt = (cnt * (1.f / static_cast<float>(GROUP)) + eps) / (1.f + static_cast<float>(B) * eps);
        lgv[b] = logf(static_cast<float>(B) * pt);
        term = fmaf(pt, lgv[b], term);
      }
    }
#pragma unroll
    for (int o = GL / 2; o > 0; o >>= 1) term += __shfl_xor_sync(0xffffffffu, term, o);
    if (live && q == 0) kl_group[g] = term;
    // every lane gets its group's B logarithms, and puts their successive differences
    // (the gradient's numerator for u in (k, k + 1)) into its own column
    float lgc[B];
#pragma unroll
    for (int c = 0; c < B; ++c) lgc[c] = __shfl_sync(0xffffffffu, lgv[c % BPL], gi * GL + c / BPL);
    __syncwarp();
#pragma unroll
    for (int c = 0; c < QMAX; ++c) hist[wl][c][lane] = lgc[c + 1] - lgc[c];
    __syncwarp();
    if (dy) {
      const float sc = gscale / p.s;
      float* dst = dy + (live ? g : g0) * GROUP;
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        float d[4];
#pragma unroll
        for (int t = 0; t < 4; ++t) {
          const float u = fmaf(v[4 * j + t], p.inv, z);
          const float uc = fminf(fmaxf(u, 0.f), qmax);
          const int k = min(static_cast<int>(uc), QMAX - 1);
          d[t] = (u > 0.f && u < qmax) ? hist[wl][k][lane] * sc : 0.f;
        }
        if (live) *reinterpret_cast<float4*>(dst + 4 * (GL * j + q)) = make_float4(d[0], d[1], d[2], d[3]);
      }
    }
    __syncwarp();  // the columns are reused by the next groups
  }
}

// loss = (sum of kl_group) / count: a cluster of kMeanCtas CTAs, CTA r summing the
// r-th of kMeanCtas equal slices (each thread a fixed strided subset in four fixed
// partial sums, then a fixed tree), and CTA 0 adding the CTAs' totals in rank order
// from their shared memory.  Fixed order throughout, and no memory outside the
// cluster, so concurrent calls on other streams do not interfere.
constexpr int kMeanCtas = 8;

__global__ void __cluster_dims__(kMeanCtas, 1, 1) __launch_bounds__(1024)
    k_mean(const float* __restrict__ v, long long count, float* __restrict__ out) {
  __shared__ double part[1024];
  uint32_t rank;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(rank));
  const long long slice = (count + kMeanCtas - 1) / kMeanCtas;
  const long long b0 = static_cast<long long>(rank) * slice;
  const long long b1 = b0 + slice < count ? b0 + slice : count;
  double acc[4] = {0.0, 0.0, 0.0, 0.0};
  long long i = b0 + threadIdx.x;
  for (; i + 3 * 1024 < b1; i += 4 * 1024) {
#pragma unroll
    for (int k = 0; k < 4; ++k) acc[k] += static_cast<double>(v[i + k * 1024]);
  }
  for (; i < b1; i += 1024) acc[0] += static_cast<double>(v[i]);  // the tail
  part[threadIdx.x] = (acc[0] + acc[1]) + (acc[2] + acc[3]);
  __syncthreads();
  for (int h = 512; h > 0; h >>= 1) {
    if (threadIdx.x < h) part[threadIdx.x] += part[threadIdx.x + h];
    __syncthreads();
  }
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
  if (rank == 0 && threadIdx.x == 0) {
    const uint32_t local = static_cast<uint32_t>(__cvta_generic_to_shared(&part[0]));
    double total = 0.0;
    for (uint32_t r = 0; r < kMeanCtas; ++r) {
      uint32_t addr;
      double t;
      asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(addr) : "r"(local), "r"(r));
      asm volatile("ld.shared::cluster.f64 %0, [%1];" : "=d"(t) : "r"(addr) : "memory");
      total += t;
    }
    *out = static_cast<float>(total / static_cast<double>(count));
  }
  // the peers' totals stay in place until the first CTA has read them
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
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
  constexpr int kGroupsPerBlock = kCalWarps * (32 / (GROUP / 32));
  long long grid = (groups + kGroupsPerBlock - 1) / kGroupsPerBlock;
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
  k_mean<<<kMeanCtas, 1024, 0, st>>>(kl_group, groups, loss);
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
