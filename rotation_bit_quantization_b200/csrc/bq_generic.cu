// Generic row-resident butterfly kernels: forward / inverse / fused RTN for any
// supported width (m a power of two <= 4096, optional dense Kronecker factor
// O_r, r <= 8).  They use the plain cos/sin rotation and serve every layer
// the specialised kernels do not take (and layers whose scaled form is out
// of range).
//
// Method (ButterflyQuant abstract; explainer article, section "butterfly"):
// Q = B_{L-1} ... B_0, stage s rotating pairs (i, i + 2^s) by the Givens
// matrix [[c, -s], [s, c]]; composite Q = B_m (x) O_r for n = m*r with O_r on
// contiguous groups of r and B_m on the stride-r index.  The inverse applies
// the stages in reverse order with negated angles, then O_r^T.
//
// Layout: one CTA works on one row at a time, the row held in shared memory
// as float32 (index i padded by i/32 to spread banks).  Stages are grouped
// three at a time: each work item loads the 8 elements whose index differs
// only in the three bits of the group, applies the three stages in registers
// and writes them back.
#include <cfloat>

#include "bq_passes.cuh"

namespace bq {
namespace {

constexpr int kThreads = 256;
// One group of up to three stages [s0, s1) over every sub-row of the row in `buf`.
template <bool INV>
__device__ void butterfly_pass(float* buf, const KLayer& Ly, int s0, int s1, int tid, int T) {
  const int m = Ly.m, r = Ly.r, L = Ly.L;
  const int ec = L < kBitsPerPass ? L : kBitsPerPass;
  const int b0 = s0 < L - ec ? s0 : L - ec;
  const int E = 1 << ec;
  const int items = r * (m >> ec);
  const int lowmask = (1 << b0) - 1;
  for (int w = tid; w < items; w += T) {
    const int i2 = w % r;
    const int q = w / r;
    const int base = (q & lowmask) | ((q >> b0) << (b0 + ec));
    float v[8];
#pragma unroll
    for (int j = 0; j < 8; ++j)
      if (j < E) v[j] = buf[pad((base | (j << b0)) * r + i2)];
    if (!INV) {
      for (int s = s0; s < s1; ++s) rot_any<false>(v, E, base, b0, s, Ly);
    } else {
      for (int s = s1 - 1; s >= s0; --s) rot_any<true>(v, E, base, b0, s, Ly);
    }
#pragma unroll
    for (int j = 0; j < 8; ++j)
      if (j < E) buf[pad((base | (j << b0)) * r + i2)] = v[j];
  }
}

// O_r (or O_r^T) applied to every contiguous group of r elements.
template <bool TRANSPOSE>
__device__ void apply_dense(float* buf, const KLayer& Ly, int tid, int T) {
  const int r = Ly.r;
  for (int g = tid; g < Ly.m; g += T) {
    float v[kMaxR], o[kMaxR];
#pragma unroll
    for (int k = 0; k < kMaxR; ++k)
      if (k < r) v[k] = buf[pad(g * r + k)];
#pragma unroll
    for (int a = 0; a < kMaxR; ++a) {
      if (a >= r) continue;
      float acc = 0.f;
#pragma unroll
      for (int b = 0; b < kMaxR; ++b) {
        if (b >= r) continue;
        const float w = TRANSPOSE ? __ldg(&Ly.O[b * r + a]) : __ldg(&Ly.O[a * r + b]);
        acc = fmaf(w, v[b], acc);
      }
      o[a] = acc;
    }
#pragma unroll
    for (int k = 0; k < kMaxR; ++k)
      if (k < r) buf[pad(g * r + k)] = o[k];
  }
}

template <bool INV>
__device__ void transform_row(float* buf, const KLayer& Ly, int tid, int T) {
  const int L = Ly.L;
  const int passes = (L + kBitsPerPass - 1) / kBitsPerPass;
  if (!INV) {
    if (Ly.r > 1) {
      apply_dense<false>(buf, Ly, tid, T);
      __syncthreads();
    }
    for (int k = 0; k < passes; ++k) {
      const int s0 = k * kBitsPerPass;
      const int s1 = s0 + kBitsPerPass < L ? s0 + kBitsPerPass : L;
      butterfly_pass<false>(buf, Ly, s0, s1, tid, T);
      __syncthreads();
    }
  } else {
    for (int k = passes - 1; k >= 0; --k) {
      const int s0 = k * kBitsPerPass;
      const int s1 = s0 + kBitsPerPass < L ? s0 + kBitsPerPass : L;
      butterfly_pass<true>(buf, Ly, s0, s1, tid, T);
      __syncthreads();
    }
    if (Ly.r > 1) {
      apply_dense<true>(buf, Ly, tid, T);
      __syncthreads();
    }
  }
}

// Per-group asymmetric RTN + packing of one row held in `buf` (one warp per group).
__device__ void quant_row(const float* buf, int n, const QuantArgs& qa, long long row, int tid, int T) {
  const int lane = tid & 31, warp = tid >> 5, nw = T >> 5;
  const int g = qa.group, C = g >> 5, bits = qa.bits;
  const float qmax = static_cast<float>((1 << bits) - 1);
  const int G = n / g;
  const int lane_bits = C * bits;
  uint8_t* crow = qa.codes + row * static_cast<long long>(n / 8 * bits);
  for (int gi = warp; gi < G; gi += nw) {
    const int e0 = gi * g + lane * C;
    float v[8];
    float lo = FLT_MAX, hi = -FLT_MAX;
#pragma unroll
    for (int c = 0; c < 8; ++c) {
      if (c < C) {
        v[c] = buf[pad(e0 + c)];
        lo = fminf(lo, v[c]);
        hi = fmaxf(hi, v[c]);
      }
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
      lo = fminf(lo, __shfl_xor_sync(0xffffffffu, lo, off));
      hi = fmaxf(hi, __shfl_xor_sync(0xffffffffu, hi, off));
    }
    const float range = __fsub_rn(hi, lo);
    __half h = __float2half_rn(__fdiv_rn(range, qmax));
    float s = __half2float(h);
    if (hi == lo || s == 0.f) {
      s = 1.f;
      h = __float2half_rn(1.f);
    }
    const float z = __fadd_rn(fminf(fmaxf(rintf(__fdiv_rn(-lo, s)), 0.f), qmax), 0.f);  // +0 for a zero point of 0
    uint32_t word = 0;
#pragma unroll
    for (int c = 0; c < 8; ++c) {
      if (c < C) {
        float t = __fadd_rn(rintf(__fdiv_rn(v[c], s)), z);
        t = fminf(fmaxf(t, 0.f), qmax);
        word |= static_cast<uint32_t>(t) << (c * bits);
      }
    }
    if (lane_bits >= 8) {
      uint8_t* dst = crow + (static_cast<size_t>(e0) * bits) / 8;
      if (lane_bits == 8) *dst = static_cast<uint8_t>(word);
      else if (lane_bits == 16) *reinterpret_cast<uint16_t*>(dst) = static_cast<uint16_t>(word);
      else *reinterpret_cast<uint32_t*>(dst) = word;
    } else {
      const int per = 8 / lane_bits;  // lanes sharing one byte (2 or 4)
      uint32_t byte = 0;
      for (int k = 0; k < per; ++k) {
        const uint32_t w2 = __shfl_sync(0xffffffffu, word, (lane & ~(per - 1)) + k);
        byte |= w2 << (k * lane_bits);
      }
      if ((lane & (per - 1)) == 0) crow[(static_cast<size_t>(e0) * bits) / 8] = static_cast<uint8_t>(byte);
    }
    if (lane == 0) {
      qa.scale[row * G + gi] = __half_as_ushort(h);
      qa.zero[row * G + gi] = __half_as_ushort(__float2half_rn(z));
    }
  }
}

template <typename TI, typename TO, bool INV, bool QUANT>
__global__ void __launch_bounds__(kThreads) k_generic(KLayer Ly, const TI* x, TO* y, long long rows, QuantArgs qa) {
  extern __shared__ float buf[];
  const int n = Ly.n;
  const int tid = threadIdx.x, T = blockDim.x;
  for (long long row = blockIdx.x; row < rows; row += gridDim.x) {
    const TI* xr = x + row * n;
    for (int i = tid; i < n; i += T) buf[pad(i)] = load_elem(xr + i);
    __syncthreads();
    transform_row<INV>(buf, Ly, tid, T);
    if (!QUANT) {
      TO* yr = y + row * n;
      for (int i = tid; i < n; i += T) store_elem(yr + i, buf[pad(i)]);
    } else {
      quant_row(buf, n, qa, row, tid, T);
    }
    __syncthreads();
  }
}

template <typename TI, typename TO, bool INV, bool QUANT>
bq_status run(const KLayer& Ly, const void* x, void* y, int64_t rows, const QuantArgs& qa, cudaStream_t st) {
  auto kern = k_generic<TI, TO, INV, QUANT>;
  const size_t smem = sizeof(float) * size_t(pad(Ly.n) + 1);
  if (smem > 48 * 1024) {
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem)) != cudaSuccess)
      return BQ_ERR_CUDA;
  }
  int dev = 0, sms = 148, per_sm = 1;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, kThreads, smem);
  if (per_sm < 1) per_sm = 1;
  long long grid = static_cast<long long>(sms) * per_sm;
  if (grid > rows) grid = rows;
  if (grid < 1) return BQ_OK;
  kern<<<static_cast<unsigned>(grid), kThreads, smem, st>>>(Ly, static_cast<const TI*>(x), static_cast<TO*>(y),
                                                           rows, qa);
  return cudaPeekAtLastError() == cudaSuccess ? BQ_OK : BQ_ERR_CUDA;
}

template <bool INV>
bq_status dispatch_io(const KLayer& Ly, const void* x, bq_dtype xt, void* y, bq_dtype yt, int64_t rows,
                      cudaStream_t st) {
  QuantArgs none{0, 0, nullptr, nullptr, nullptr};
  if (xt == BQ_F32 && yt == BQ_F32) return run<float, float, INV, false>(Ly, x, y, rows, none, st);
  if (xt == BQ_F32 && yt == BQ_BF16) return run<float, __nv_bfloat16, INV, false>(Ly, x, y, rows, none, st);
  if (xt == BQ_BF16 && yt == BQ_F32) return run<__nv_bfloat16, float, INV, false>(Ly, x, y, rows, none, st);
  return run<__nv_bfloat16, __nv_bfloat16, INV, false>(Ly, x, y, rows, none, st);
}

}  // namespace

bq_status launch_generic(const KLayer& Ly, const void* x, bq_dtype xt, void* y, bq_dtype yt, int64_t rows,
                         bool inverse, const QuantArgs* q, cudaStream_t st) {
  if (q) {
    if (xt == BQ_F32) return run<float, float, false, true>(Ly, x, nullptr, rows, *q, st);
    return run<__nv_bfloat16, float, false, true>(Ly, x, nullptr, rows, *q, st);
  }
  return inverse ? dispatch_io<true>(Ly, x, xt, y, yt, rows, st) : dispatch_io<false>(Ly, x, xt, y, yt, rows, st);
}

}  // namespace bq
