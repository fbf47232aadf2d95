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
// array's name as a device address, so its address is looked up with the
// device current and cached per CUDA context: a context that is destroyed and
// re-created (cudaDeviceReset, or the primary context released and retained
// again) reloads this module, the array may move, and the new context's id
// forces a fresh lookup.  Every call shares the array: calls that overlap on
// the GPU (different streams, or different host threads on the same device)
// race on it.  The prefill writes each part of its scratch before reading it,
// so stale contents from an earlier call do no harm and nothing needs clearing.
#include <mutex>

#include "common.cuh"

namespace m2 {
namespace {

static __device__ __align__(256) unsigned char g_static_scratch[MAMBA2_STATIC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
struct ScratchEntry {
  unsigned long long ctx_id;  // 0: not looked up
  void *addr;
};
std::mutex g_scratch_mu;
ScratchEntry g_scratch[kMaxDevices] = {};

// Device address of g_static_scratch in the current device's context.
cudaError_t static_scratch_address(void **out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  const unsigned long long id = current_context_id();
  ScratchEntry &c = g_scratch[dev];
  if (id == 0 || c.ctx_id != id || c.addr == nullptr) {
    void *p = nullptr;
    e = cudaGetSymbolAddress(&p, g_static_scratch);  // makes the primary context current
    if (e != cudaSuccess) return e;
    c.addr = p;
    c.ctx_id = current_context_id();
  }
  *out = c.addr;
  return cudaSuccess;
}

}  // namespace
}  // namespace m2

extern "C" MAMBA2_API int mamba2_conv_ssd_prefill_noalloc(
    const mamba2_dims *dims, const mamba2_params *params, const void *xBC,
    int64_t xBC_row_stride, const void *z, int64_t z_row_stride, const void *dt_raw,
    int64_t dt_row_stride, void *y, void *conv_state, float *ssm_state, int32_t states_in,
    void *stream) {
  struct Disarm {  // stage events are disarmed on every return, as for the other entries
    ~Disarm() { m2::g_stage_events.n = 0; }
  } disarm;
  const int st = m2::validate_prefill_dims(dims);
  if (st != MAMBA2_OK) return st;
  if (mamba2_prefill_workspace_size(dims) > (size_t)MAMBA2_STATIC_SCRATCH_BYTES)
    return MAMBA2_ERR_WORKSPACE;
  void *scratch = nullptr;
  if (m2::static_scratch_address(&scratch) != cudaSuccess) return MAMBA2_ERR_CUDA;
  return mamba2_conv_ssd_prefill(dims, params, xBC, xBC_row_stride, z, z_row_stride, dt_raw,
                                 dt_row_stride, y, conv_state, ssm_state, states_in, scratch,
                                 (size_t)MAMBA2_STATIC_SCRATCH_BYTES, stream);
}
