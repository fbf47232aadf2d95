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

// ---------------------------------------------------------------- async copies
namespace m2 {

// Each translation unit that waits on mbarriers keeps its own error word (a
// file-scope __device__ variable, so no relocatable device code is needed),
// passes its address to mbar_wait_bounded, and exposes a host function that
// reads and clears it for mamba2_device_errors.  Bit values: kErrWaitTimeout.
constexpr unsigned int kErrWaitTimeout = 1u;
constexpr unsigned long long kWaitLimitNs = 2000000000ull;  // 2 s

__device__ __forceinline__ uint32_t smem_u32(const void *p) {
  return (uint32_t)__cvta_generic_to_shared(p);
}
__device__ __forceinline__ unsigned long long globaltimer_ns() {
  unsigned long long t;
  asm volatile("mov.u64 %0, %globaltimer;" : "=l"(t));
  return t;
}
__device__ __forceinline__ void mbar_init(uint64_t *bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count)
               : "memory");
}
__device__ __forceinline__ void fence_mbar_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}
__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}
__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t *bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)),
               "r"(bytes)
               : "memory");
}
// Bulk (non-tensor) global -> shared copy completing on `bar`; 16-byte aligned
// addresses, size a multiple of 16.
__device__ __forceinline__ void bulk_g2s(void *dst, const void *src, uint32_t bytes,
                                         uint64_t *bar) {
  asm volatile(
      "cp.async.bulk.shared::cta.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
          smem_u32(dst)),
      "l"(src), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint64_t *bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n"
      " selp.u32 %0, 1, 0, p;\n}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}
// Waits for phase `parity` of `bar` to complete, for at most kWaitLimitNs;
// returns false (and raises the device error flag) if it never did.
__device__ __forceinline__ bool mbar_wait_bounded(uint64_t *bar, uint32_t parity,
                                                  unsigned int *err) {
  if (mbar_try_wait(bar, parity)) return true;
  const unsigned long long t0 = globaltimer_ns();
  while (!mbar_try_wait(bar, parity)) {
    if (globaltimer_ns() - t0 > kWaitLimitNs) {
      atomicOr(err, kErrWaitTimeout);
      return false;
    }
  }
  return true;
}

// Host: read and clear the error words of the kernels that wait (one per
// translation unit).  Synchronous.
cudaError_t take_step_errors(unsigned int *out);

}  // namespace m2
