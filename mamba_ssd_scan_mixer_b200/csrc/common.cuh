// Device helpers and the internal problem description shared by the kernels
// of libmamba2ssd.so.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "mamba2ssd.h"

namespace m2 {

// Resolved problem sizes (validated by the C ABI before any launch).
struct Problem {
  int64_t batch, L;
  int H, P, N, G, K, Q;
  int io;       // mamba2_dtype
  int nbg;      // norm_before_gate
  float eps;
  int64_t d_inner, conv_dim;
  int64_t nchunks;  // ceil(L / Q)
  __host__ __device__ int heads_per_group() const { return H / G; }
};

// Everything one prefill call needs, with device pointers already checked.
struct PrefillArgs {
  Problem pr;
  mamba2_params prm;
  const void *xBC;
  int64_t ld_xbc;
  const void *z;
  int64_t ld_z;
  const void *dt_raw;
  int64_t ld_dt;
  void *y;
  void *conv_state;
  float *ssm_state;
  int states_in;
  char *ws;
  cudaStream_t stream;
};

struct StepArgs {
  Problem pr;
  mamba2_params prm;
  const void *xBC;
  int64_t ld_xbc;
  const void *z;
  int64_t ld_z;
  const void *dt_raw;
  int64_t ld_dt;
  void *y;
  void *conv_state;
  float *ssm_state;
  cudaStream_t stream;
};

// ---------------------------------------------------------------- conversions
__device__ __forceinline__ float to_f(float v) { return v; }
__device__ __forceinline__ float to_f(__nv_bfloat16 v) { return __bfloat162float(v); }

template <typename T> __device__ __forceinline__ T from_f(float v);
template <> __device__ __forceinline__ float from_f<float>(float v) { return v; }
template <> __device__ __forceinline__ __nv_bfloat16 from_f<__nv_bfloat16>(float v) {
  return __float2bfloat16_rn(v);
}

// ---------------------------------------------------------------- activations
// Accurate forms (CUDA's expf / log1pf); the fp32 path relies on them.
__device__ __forceinline__ float silu_f(float v) { return v / (1.0f + expf(-v)); }
__device__ __forceinline__ float softplus_f(float s) {
  return fmaxf(s, 0.0f) + log1pf(expf(-fabsf(s)));
}

// ---------------------------------------------------------------- reductions
__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// Sum over the block (blockDim.x a multiple of 32, <= 1024); every thread gets
// the total.  `red` is shared scratch of >= 33 floats.
__device__ __forceinline__ float block_sum(float v, float *red) {
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5, nw = blockDim.x >> 5;
  v = warp_sum(v);
  __syncthreads();  // red may still be read by a previous call
  if (lane == 0) red[wid] = v;
  __syncthreads();
  float t = (lane < nw) ? red[lane] : 0.0f;
  t = warp_sum(t);
  return t;
}

inline int64_t ceil_div(int64_t a, int64_t b) { return (a + b - 1) / b; }

// Optional per-stage timing events (profiling aid, see
// mamba2_record_stage_events): when armed, stage_mark(s, i) records event i
// on stream s.  Armed per host thread, for one call.
constexpr int kMaxStageEvents = 16;
struct StageEvents {
  cudaEvent_t ev[kMaxStageEvents];
  int n;  // 0 = disarmed
};
extern thread_local StageEvents g_stage_events;
inline void stage_mark(cudaStream_t s, int i) {
  if (i < g_stage_events.n && g_stage_events.ev[i] != nullptr)
    cudaEventRecord(g_stage_events.ev[i], s);
}

// Names of the kernel stages each path enqueues, in order.
extern const char *const kPrefillSimtStages[];
extern const int kPrefillSimtStageCount;
extern const char *const kStepSimtStages[];
extern const int kStepSimtStageCount;
inline size_t align_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

// Launchers (one per translation unit).
cudaError_t prefill_simt(const PrefillArgs &a);
size_t prefill_simt_workspace(const Problem &pr);
cudaError_t step_simt(const StepArgs &a);

}  // namespace m2
