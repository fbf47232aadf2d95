// Prefill for callers that cannot allocate device memory.
//
// Some callers of this library may not call cudaMalloc: a plugin loaded into a
// host runtime that owns all device memory through its own pool (a foreign
// allocation is forbidden there, or breaks its accounting), or code on a
// latency-critical path that cannot afford an allocation's implicit
// synchronisation.  mamba2_conv_ssd_prefill_noalloc serves them: it runs the
// ordinary prefill with its scratch taken from a fixed array in this file
// instead of a caller-provided workspace.
//
// The array is MAMBA2_STATIC_SCRATCH_BYTES large and lives in every GPU that
// loads this library until the process exits.  Host code cannot use the
// array's name as a device address, so its address is looked up once per
// device (with that device current) and cached.  Every call shares the array:
// calls that overlap on the GPU (different streams, or different host threads
// on the same device) race on it.  The prefill writes each part of its
// scratch before reading it, so stale contents from an earlier call do no
// harm and nothing needs clearing.
#include <mutex>

#include "common.cuh"

namespace m2 {
namespace {

static __device__ __align__(256) unsigned char g_static_scratch[MAMBA2_STATIC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
std::mutex g_scratch_mu;
void *g_scratch_addr[kMaxDevices] = {};

// Device address of g_static_scratch on the current device (set up on first use).
cudaError_t static_scratch_address(void **out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  if (g_scratch_addr[dev] == nullptr) {
    void *p = nullptr;
    e = cudaGetSymbolAddress(&p, g_static_scratch);
    if (e != cudaSuccess) return e;
    g_scratch_addr[dev] = p;
  }
  *out = g_scratch_addr[dev];
  return cudaSuccess;
}

}  // namespace
}  // namespace m2

extern "C" MAMBA2_API int mamba2_conv_ssd_prefill_noalloc(
    const mamba2_dims *dims, const mamba2_params *params, const void *xBC,
    int64_t xBC_row_stride, const void *z, int64_t z_row_stride, const void *dt_raw,
    int64_t dt_row_stride, void *y, void *conv_state, float *ssm_state, int32_t states_in,
    void *stream) {
  // Sizes are validated by the ordinary entry point below; only the scratch
  // limit is checked here.
  if (mamba2_prefill_workspace_size(dims) > (size_t)MAMBA2_STATIC_SCRATCH_BYTES)
    return MAMBA2_ERR_WORKSPACE;
  void *scratch = nullptr;
  if (m2::static_scratch_address(&scratch) != cudaSuccess) return MAMBA2_ERR_CUDA;
  return mamba2_conv_ssd_prefill(dims, params, xBC, xBC_row_stride, z, z_row_stride, dt_raw,
                                 dt_row_stride, y, conv_state, ssm_state, states_in, scratch,
                                 (size_t)MAMBA2_STATIC_SCRATCH_BYTES, stream);
}
