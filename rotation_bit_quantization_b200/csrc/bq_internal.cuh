// Internal declarations shared by the libbq CUDA sources (not part of the C ABI).
#pragma once

#include <atomic>
#include <cstdint>
#include <mutex>
#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "bq.h"

namespace bq {

constexpr int kMaxM = 4096;        // largest butterfly width (power of two)
constexpr int kMaxR = 8;           // largest dense Kronecker factor
constexpr int kMaxN = 16384;       // largest row width m*r
constexpr int kMaxBwdLayers = 128; // layers per backward launch (kernel-parameter array)
constexpr int kMaxGroup = 256;     // largest quantization group

// Prepared-table layout (floats), per layer of width m with L = log2(m) stages:
//   [0, 16)            header: [0] = 1.0 when the scaled (fast) rotation form is
//                      usable for this layer, else 0.0; [1] = m; [2] = L;
//                      [3] = 1.0 when the scaled form of the inverse is usable
//   cs     [L][m/2]    float2 (cos, sin) of every angle
//   fast   [L][m]      per-position coefficient of the scaled form: at stage s
//                      position i is updated as a_i += fast[s][i] * a_{i ^ 2^s}
//                      (the low element of a pair first, then the high one)
//   sigma  [m]         per-position output scale of the scaled form
//   fast_inv [L][m]    the same for the inverse (stages L-1 .. 0, transposed
//                      rotations), low element first
//   sigma_inv [m]      per-position output scale of the scaled inverse
//   image  [104][128][4] (m == 4096 only) tensor-memory image of the specialised
//                      n = 4096 kernel: lane t, column c (float4 block c/4 of
//                      lane t) holds the coefficient thread t needs at that
//                      column (see bq_fast4096.cu)
//   image_inv [104][128][4] (m == 4096 only) the same lanes and stage columns
//                      for the inverse kernel: its scaled-form coefficients and
//                      output scale, or (cos, sin) and 1 when header[3] is 0
struct TableLayout {
  int m, L;
  size_t off_cs, off_fast, off_sigma, off_fast_inv, off_sigma_inv, off_image, off_image_inv, total;
};

constexpr int kImageLanes = 128;
constexpr int kImageCols = 416;
constexpr int kImageInvCols = 416;

__host__ __device__ inline int ilog2(int v) {
  int l = 0;
  while ((1 << l) < v) ++l;
  return l;
}

__host__ __device__ inline size_t round4(size_t v) { return (v + 3) & ~size_t(3); }

__host__ __device__ inline TableLayout table_layout(int m) {
  TableLayout t;
  t.m = m;
  t.L = ilog2(m);
  t.off_cs = 16;
  t.off_fast = t.off_cs + round4(size_t(t.L) * m);
  t.off_sigma = t.off_fast + round4(size_t(t.L) * m);
  t.off_fast_inv = t.off_sigma + round4(size_t(m));
  t.off_sigma_inv = t.off_fast_inv + round4(size_t(t.L) * m);
  t.off_image = t.off_sigma_inv + round4(size_t(m));
  t.off_image_inv = t.off_image + (m == 4096 ? size_t(kImageLanes) * kImageCols : 0);
  t.total = t.off_image_inv + (m == 4096 ? size_t(kImageLanes) * kImageInvCols : 0);
  return t;
}

// Everything a kernel needs about one layer, passed by value.
struct KLayer {
  int n, m, r, L;
  const float2* cs;     // [L][m/2]
  const float* fast;    // [L][m]
  const float* sigma;   // [m]
  const float* fast_inv;   // [L][m]
  const float* sigma_inv;  // [m]
  const float* hdr;     // header (flags at hdr[0], hdr[3])
  const float* image;   // tensor-memory image (m == 4096) or nullptr
  const float* image_inv;  // plain-form image for the inverse (m == 4096) or nullptr
  const float* O;       // [r][r] or nullptr
};

inline KLayer make_klayer(const bq_layer& l) {
  TableLayout t = table_layout(l.m);
  KLayer k;
  k.n = l.n; k.m = l.m; k.r = l.r; k.L = t.L;
  k.cs = reinterpret_cast<const float2*>(l.table + t.off_cs);
  k.fast = l.table + t.off_fast;
  k.sigma = l.table + t.off_sigma;
  k.fast_inv = l.table + t.off_fast_inv;
  k.sigma_inv = l.table + t.off_sigma_inv;
  k.hdr = l.table;
  k.image = l.m == 4096 ? l.table + t.off_image : nullptr;
  k.image_inv = l.m == 4096 ? l.table + t.off_image_inv : nullptr;
  k.O = l.O;
  return k;
}

struct QuantArgs {
  int bits, group;
  uint8_t* codes;
  uint16_t* scale;
  uint16_t* zero;
};

// Launchers (defined in the .cu files).  Each returns BQ_OK or BQ_ERR_CUDA.
bq_status launch_prepare(const float* theta, int m, float* table, cudaStream_t st);
bq_status launch_prepare_hadamard(const uint8_t* quadrant, float* theta_out, int m, float* table, cudaStream_t st);
bq_status launch_fast4096(const KLayer& L, const void* x, bq_dtype xt, void* y, bq_dtype yt, int64_t rows,
                          const QuantArgs* q, cudaStream_t st);
bool fast4096_supports(const KLayer& L, const QuantArgs* q);
bq_status launch_inv4096(const KLayer& L, const void* y, bq_dtype yt, void* x, bq_dtype xt, int64_t rows,
                         cudaStream_t st);
bq_status launch_kron1024(const KLayer& L, const void* x, bq_dtype xt, void* y, bq_dtype yt, int64_t rows,
                          const QuantArgs* q, cudaStream_t st);
bool kron1024_supports(const KLayer& L, const QuantArgs* q);
bq_status launch_kron1024_inv(const KLayer& L, const void* y, bq_dtype yt, void* x, bq_dtype xt, int64_t rows,
                              cudaStream_t st);
bq_status launch_generic(const KLayer& L, const void* x, bq_dtype xt, void* y, bq_dtype yt,
                         int64_t rows, bool inverse, const QuantArgs* q, cudaStream_t st);
bq_status launch_bwd(const KLayer* layers, int num_layers, const void* x, bq_dtype xt,
                     void* y, bq_dtype yt, const float* dy, float* dx, float* dtheta,
                     int64_t rows, void* ws, int chunks, cudaStream_t st);
bq_status launch_bwd4096(const KLayer* layers, int num_layers, const void* x, bq_dtype xt, void* y, bq_dtype yt,
                         const float* dy, float* dx, float* dtheta, int64_t rows, void* ws, int chunks,
                         cudaStream_t st);
int bwd4096_chunks(int num_layers, int64_t rows);
int bwd_chunks(int m, int num_layers, int64_t rows);
size_t bwd_workspace_bytes(int m, int num_layers, int chunks);

// ---------------------------------------------------------------- host validation
//
// Shared by every entry point, so that the same bad argument gives the same
// status from each of them.

inline bool valid_m(int m) { return m >= 2 && m <= kMaxM && (m & (m - 1)) == 0; }
inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
inline bool valid_dtype(bq_dtype t) { return t == BQ_F32 || t == BQ_BF16; }

inline bq_status check_layer(const bq_layer* l) {
  if (!l) return BQ_ERR_INVALID_ARG;
  if (!valid_m(l->m) || l->r < 1 || l->r > kMaxR) return BQ_ERR_INVALID_ARG;
  if (static_cast<long long>(l->m) * l->r != l->n || l->n > kMaxN) return BQ_ERR_INVALID_ARG;
  if (!l->table || !aligned16(l->table)) return BQ_ERR_INVALID_ARG;
  if ((l->r > 1) != (l->O != nullptr)) return BQ_ERR_INVALID_ARG;
  if (l->O && (reinterpret_cast<uintptr_t>(l->O) & 3u)) return BQ_ERR_INVALID_ARG;
  return BQ_OK;
}

// The layer list and dtypes of a backward call (both backward entry points):
// every layer valid, one width m, no dense factor (r == 1), rows >= 1.  Fills kl.
inline bq_status check_bwd_layers(const bq_layer* layers, int32_t num_layers, bq_dtype xt, bq_dtype yt,
                                  int64_t rows_per_layer, KLayer* kl) {
  if (!layers || num_layers < 1 || num_layers > kMaxBwdLayers) return BQ_ERR_INVALID_ARG;
  if (!valid_dtype(xt) || !valid_dtype(yt)) return BQ_ERR_INVALID_ARG;
  const int m = layers[0].m;
  for (int l = 0; l < num_layers; ++l) {
    bq_status s = check_layer(&layers[l]);
    if (s != BQ_OK) return s;
    if (layers[l].m != m) return BQ_ERR_INVALID_ARG;
    if (layers[l].r != 1) return BQ_ERR_UNSUPPORTED;
    kl[l] = make_klayer(layers[l]);
  }
  if (rows_per_layer < 1) return BQ_ERR_INVALID_ARG;
  return BQ_OK;
}

// ---------------------------------------------------------------- host helpers

// Runs `fn` once per device for the given flag array (a per-kernel static), under
// one process-wide lock: concurrent first calls from several host threads set a
// kernel's attributes exactly once and every caller sees the result.  Returns
// false, leaving the flag clear, if fn fails.
inline std::mutex& setup_mutex() {
  static std::mutex mu;
  return mu;
}

constexpr int kMaxDevices = 64;

template <typename Fn>
inline bool once_per_device(std::atomic<int> (&flags)[kMaxDevices], int dev, Fn fn) {
  if (dev < 0 || dev >= kMaxDevices) return false;
  if (flags[dev].load(std::memory_order_acquire)) return true;
  std::lock_guard<std::mutex> lock(setup_mutex());
  if (flags[dev].load(std::memory_order_relaxed)) return true;
  if (!fn()) return false;
  flags[dev].store(1, std::memory_order_release);
  return true;
}

// Multiprocessor count of device `dev` (cached; 0 on failure).
inline int device_sm_count(int dev) {
  static std::atomic<int> sms[kMaxDevices];
  if (dev < 0 || dev >= kMaxDevices) return 0;
  int v = sms[dev].load(std::memory_order_acquire);
  if (v > 0) return v;
  if (cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || v <= 0) return 0;
  sms[dev].store(v, std::memory_order_release);
  return v;
}

// ---------------------------------------------------------------- device helpers

__device__ __forceinline__ float load_elem(const float* p) { return *p; }
__device__ __forceinline__ float load_elem(const __nv_bfloat16* p) { return __bfloat162float(*p); }
__device__ __forceinline__ void store_elem(float* p, float v) { *p = v; }
__device__ __forceinline__ void store_elem(__nv_bfloat16* p, float v) { *p = __float2bfloat16_rn(v); }

}  // namespace bq
