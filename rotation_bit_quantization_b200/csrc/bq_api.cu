// C ABI entry points of libbq.so: host-side validation and dispatch.  Every
// check runs before anything is launched; a failed check returns a status and
// launches nothing.  See include/bq.h for the contract of each call.
#include "bq_internal.cuh"

namespace bq {

// The wait-fault word of the m = 4096 kernels on the current device (bq_fast4096.cu,
// the translation unit that holds the word).
bq_status read_wait_faults(int32_t* value, bool clear, cudaStream_t st);

namespace {

bq_status check_rows(const void* a, const void* b, int64_t rows) {
  if (rows < 0) return BQ_ERR_INVALID_ARG;
  if (rows == 0) return BQ_OK;
  if (!a || !b || !aligned16(a) || !aligned16(b)) return BQ_ERR_INVALID_ARG;
  return BQ_OK;
}

bq_status transform(const bq_layer* layer, const void* x, bq_dtype xt, void* y, bq_dtype yt, int64_t rows,
                    void* stream, bool inverse) {
  bq_status s = check_layer(layer);
  if (s != BQ_OK) return s;
  if (!valid_dtype(xt) || !valid_dtype(yt)) return BQ_ERR_INVALID_ARG;
  if ((s = check_rows(x, y, rows)) != BQ_OK) return s;
  if (rows == 0) return BQ_OK;
  if (x == y && xt != yt) return BQ_ERR_INVALID_ARG;
  const KLayer L = make_klayer(*layer);
  if (!inverse && fast4096_supports(L, nullptr))
    return launch_fast4096(L, x, xt, y, yt, rows, nullptr, static_cast<cudaStream_t>(stream));
  if (inverse && fast4096_supports(L, nullptr))
    return launch_inv4096(L, x, xt, y, yt, rows, static_cast<cudaStream_t>(stream));
  if (inverse && kron1024_supports(L, nullptr))
    return launch_kron1024_inv(L, x, xt, y, yt, rows, static_cast<cudaStream_t>(stream));
  if (!inverse && kron1024_supports(L, nullptr))
    return launch_kron1024(L, x, xt, y, yt, rows, nullptr, static_cast<cudaStream_t>(stream));
  return launch_generic(L, x, xt, y, yt, rows, inverse, nullptr, static_cast<cudaStream_t>(stream));
}

bq_status quantize(const bq_layer* layer, const void* x, bq_dtype xt, int64_t rows, int32_t bits, int32_t group,
                   uint8_t* codes, uint16_t* scale, uint16_t* zero, void* stream) {
  bq_status s = check_layer(layer);
  if (s != BQ_OK) return s;
  if (!valid_dtype(xt)) return BQ_ERR_INVALID_ARG;
  if (bits != 2 && bits != 4) return BQ_ERR_INVALID_ARG;
  if (group < 32 || group > kMaxGroup || (group & 31) || layer->n % group) return BQ_ERR_INVALID_ARG;
  if (rows < 0) return BQ_ERR_INVALID_ARG;
  if (rows == 0) return BQ_OK;
  if (!x || !codes || !scale || !zero) return BQ_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(codes) || !aligned16(scale) || !aligned16(zero)) return BQ_ERR_INVALID_ARG;
  const KLayer L = make_klayer(*layer);
  QuantArgs q{bits, group, codes, scale, zero};
  if (fast4096_supports(L, &q))
    return launch_fast4096(L, x, xt, nullptr, BQ_F32, rows, &q, static_cast<cudaStream_t>(stream));
  if (kron1024_supports(L, &q))
    return launch_kron1024(L, x, xt, nullptr, BQ_F32, rows, &q, static_cast<cudaStream_t>(stream));
  return launch_generic(L, x, xt, nullptr, BQ_F32, rows, false, &q, static_cast<cudaStream_t>(stream));
}

}  // namespace
}  // namespace bq

using namespace bq;

extern "C" {

int32_t bq_cuda_last_error(void) { return static_cast<int32_t>(cudaGetLastError()); }

const char* bq_cuda_error_string(int32_t code) { return cudaGetErrorString(static_cast<cudaError_t>(code)); }

size_t bq_table_floats(int32_t m) {
  if (!valid_m(m)) return 0;
  return table_layout(m).total;
}

bq_status bq_precompute_cs(const float* theta, int32_t m, float* table, void* stream) {
  if (!valid_m(m) || !theta || !table || !aligned16(table) || (reinterpret_cast<uintptr_t>(theta) & 3u))
    return BQ_ERR_INVALID_ARG;
  return launch_prepare(theta, m, table, static_cast<cudaStream_t>(stream));
}

bq_status bq_precompute_hadamard(int32_t m, const uint8_t* quadrant, float* table, float* theta, void* stream) {
  if (!valid_m(m) || !table || !aligned16(table) || (reinterpret_cast<uintptr_t>(theta) & 3u)) return BQ_ERR_INVALID_ARG;
  return launch_prepare_hadamard(quadrant, theta, m, table, static_cast<cudaStream_t>(stream));
}

bq_status bq_butterfly_fwd(const bq_layer* layer, const void* x, bq_dtype xt, void* y, bq_dtype yt, int64_t rows,
                           void* stream) {
  return transform(layer, x, xt, y, yt, rows, stream, false);
}

bq_status bq_butterfly_inv(const bq_layer* layer, const void* y, bq_dtype yt, void* x, bq_dtype xt, int64_t rows,
                           void* stream) {
  return transform(layer, y, yt, x, xt, rows, stream, true);
}

size_t bq_butterfly_bwd_workspace_size(int32_t m, int32_t num_layers, int64_t rows_per_layer) {
  if (!valid_m(m) || num_layers < 1 || num_layers > kMaxBwdLayers || rows_per_layer < 1) return 0;
  return bwd_workspace_bytes(m, num_layers, bwd_chunks(m, num_layers, rows_per_layer));
}

bq_status bq_butterfly_bwd(const bq_layer* layers, int32_t num_layers, const void* x, bq_dtype xt, void* y,
                           bq_dtype yt, const float* dy, float* dx, float* dtheta, int64_t rows_per_layer,
                           void* workspace, size_t workspace_bytes, void* stream) {
  KLayer kl[kMaxBwdLayers];
  const bq_status s = check_bwd_layers(layers, num_layers, xt, yt, rows_per_layer, kl);
  if (s != BQ_OK) return s;
  const int m = layers[0].m;
  const void* ptrs[] = {x, y, dy, dx, dtheta, workspace};
  for (const void* p : ptrs)
    if (!p || !aligned16(p)) return BQ_ERR_INVALID_ARG;
  const int chunks = bwd_chunks(m, num_layers, rows_per_layer);
  if (workspace_bytes < bwd_workspace_bytes(m, num_layers, chunks)) return BQ_ERR_WORKSPACE;
  return launch_bwd(kl, num_layers, x, xt, y, yt, dy, dx, dtheta, rows_per_layer, workspace, chunks,
                    static_cast<cudaStream_t>(stream));
}

bq_status bq_transform_quantize(const bq_layer* layer, const void* x, bq_dtype xt, int64_t rows, int32_t bits,
                                int32_t group, uint8_t* codes, uint16_t* scale_f16, uint16_t* zero_f16,
                                void* stream) {
  return quantize(layer, x, xt, rows, bits, group, codes, scale_f16, zero_f16, stream);
}

bq_status bq_weight_rotate_pack(const bq_layer* layer, const void* w, bq_dtype wt, int64_t out_features,
                                int32_t bits, int32_t group, uint8_t* codes, uint16_t* scale_f16,
                                uint16_t* zero_f16, void* stream) {
  return quantize(layer, w, wt, out_features, bits, group, codes, scale_f16, zero_f16, stream);
}

bq_status bq_wait_faults(int32_t* value, int32_t clear, void* stream) {
  if (value == nullptr) return BQ_ERR_INVALID_ARG;
  return bq::read_wait_faults(value, clear != 0, static_cast<cudaStream_t>(stream));
}

const char* bq_status_string(bq_status status) {
  switch (status) {
    case BQ_OK: return "ok";
    case BQ_ERR_INVALID_ARG: return "invalid argument";
    case BQ_ERR_UNSUPPORTED: return "unsupported configuration";
    case BQ_ERR_WORKSPACE: return "workspace too small";
    case BQ_ERR_CUDA: return "CUDA launch error";
  }
  return "unknown status";
}

}  // extern "C"
