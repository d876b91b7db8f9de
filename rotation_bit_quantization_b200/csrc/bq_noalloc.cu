// bq_butterfly_bwd_noalloc: the calibration backward with its scratch memory in
// a fixed device array instead of a caller-provided workspace.
//
// Some callers cannot allocate device memory at the moment they need the
// backward: code that runs while another framework owns the device allocator
// (a plugin handed only its inputs and outputs), a real-time loop that must not
// block in the allocator, or a process whose device memory is fully reserved
// by a pool.  They still pass every input and output; the only scratch the
// backward uses (per-block dtheta partials and the per-layer tickets of the
// deterministic reduction) lives in the file-scope array below, which every GPU
// that loads this library keeps until the process exits.
//
// The paper has no counterpart to this entry point.
#include <mutex>

#include "bq_internal.cuh"

namespace bq {
namespace {

constexpr size_t kScratchBytes = size_t(8) << 20;  // 8 MiB (BQ_NOALLOC_SCRATCH_BYTES)

static __device__ __align__(256) unsigned char g_scratch[kScratchBytes];

std::mutex g_mu;
void* g_scratch_ptr[kMaxDevices] = {};

// Device address of g_scratch on the current device, looked up once per device.
// In host code `g_scratch` names a host-side stand-in, not device memory, so the
// address must come from cudaGetSymbolAddress with the device current.
bq_status scratch_for_current_device(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return BQ_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_mu);
  if (!g_scratch_ptr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_scratch) != cudaSuccess || !p) return BQ_ERR_CUDA;
    g_scratch_ptr[dev] = p;
  }
  *out = g_scratch_ptr[dev];
  return BQ_OK;
}

}  // namespace
}  // namespace bq

using namespace bq;

extern "C" bq_status bq_butterfly_bwd_noalloc(const bq_layer* layers, int32_t num_layers, const void* x, bq_dtype xt,
                                              void* y, bq_dtype yt, const float* dy, float* dx, float* dtheta,
                                              int64_t rows_per_layer, void* stream) {
  // the same layer and dtype checks, in the same order, as bq_butterfly_bwd
  KLayer kl[kMaxBwdLayers];
  const bq_status s = check_bwd_layers(layers, num_layers, xt, yt, rows_per_layer, kl);
  if (s != BQ_OK) return s;
  const int m = layers[0].m;
  const void* ptrs[] = {x, y, dy, dx, dtheta};
  for (const void* p : ptrs)
    if (!p || !aligned16(p)) return BQ_ERR_INVALID_ARG;
  // as many token chunks per layer as the default backward uses, reduced until the
  // partials fit the fixed scratch; at least one chunk per layer must fit
  int chunks = bwd_chunks(m, num_layers, rows_per_layer);
  while (chunks > 1 && bwd_workspace_bytes(m, num_layers, chunks) > kScratchBytes) --chunks;
  if (bwd_workspace_bytes(m, num_layers, chunks) > kScratchBytes) return BQ_ERR_WORKSPACE;
  void* scratch = nullptr;
  const bq_status st = scratch_for_current_device(&scratch);
  if (st != BQ_OK) return st;
  return launch_bwd(kl, num_layers, x, xt, y, yt, dy, dx, dtheta, rows_per_layer, scratch, chunks,
                    static_cast<cudaStream_t>(stream));
}
