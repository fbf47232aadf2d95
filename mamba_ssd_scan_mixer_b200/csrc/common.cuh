// Device helpers and the internal problem description shared by the kernels
// of libmamba2ssd.so.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <nvtx3/nvToolsExt.h>
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
  // packed sequences of different lengths (batch = sequences, pr.L = total
  // tokens): device [batch + 1] first token of each sequence; null otherwise
  const int32_t *cu_seqlens = nullptr;
};

// One backward call of the prefill (device pointers checked by the C ABI).
struct BackwardArgs {
  Problem pr;
  mamba2_params prm;
  const void *xBC;
  int64_t ld_xbc;
  const void *z;
  int64_t ld_z;
  const void *dt_raw;
  int64_t ld_dt;
  const void *conv_state_in;      // or null (zero left context)
  const float *ssm_state_in;      // or null (zero initial state)
  const void *dy;                 // [b][L][d_inner]
  const float *d_ssm_state_out;   // or null
  void *d_xBC, *d_z, *d_dt_raw;   // [b][L][conv_dim], [b][L][d_inner], [b][L][H]
  float *d_conv_w, *d_conv_b, *d_dt_bias, *d_A, *d_D, *d_norm_w;
  void *d_conv_state_in;          // or null
  float *d_ssm_state_in;          // or null
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

// NVTX range for the lifetime of the object (header-only NVTX 3: without a
// profiler attached the calls return at once).  Each entry point and each
// kernel stage it enqueues is named, so a timeline shows the call structure.
struct NvtxRange {
  explicit NvtxRange(const char *name) { nvtxRangePushA(name); }
  ~NvtxRange() { nvtxRangePop(); }
  NvtxRange(const NvtxRange &) = delete;
  NvtxRange &operator=(const NvtxRange &) = delete;
};

// Names of the kernel stages each path enqueues, in order.
extern const char *const kPrefillSimtStages[];
extern const int kPrefillSimtStageCount;
extern const char *const kStepSimtStages[];
extern const int kStepSimtStageCount;
extern const char *const kBackwardStages[];
extern const int kBackwardStageCount;
inline size_t align_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

// MAMBA2_OK if `dims` describe a valid prefill problem, else the status the
// prefill entry point would return for them.
int validate_prefill_dims(const mamba2_dims *dims);

// Launchers (one per translation unit).
cudaError_t prefill_simt(const PrefillArgs &a);
size_t prefill_simt_workspace(const Problem &pr);
cudaError_t step_simt(const StepArgs &a);
cudaError_t prefill_backward(const BackwardArgs &a);
size_t backward_workspace(const Problem &pr);

}  // namespace m2

// ---------------------------------------------------------------- async copies
namespace m2 {

// Programmatic dependent launch: a kernel launched with programmatic stream
// serialization may start while the previous kernel of the stream drains;
// grid_dependency_wait blocks until that kernel has completed and its memory
// operations are visible.  launch_dependents lets the next kernel's CTAs be
// scheduled once every CTA of this one has called it (or exited).
__device__ __forceinline__ void grid_dependency_wait() {
  asm volatile("griddepcontrol.wait;" ::: "memory");
}
__device__ __forceinline__ void launch_dependents() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

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
__device__ __forceinline__ void mbar_arrive(uint64_t *bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
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

// Waits for phase `parity` of `bar` for at most `limit_ns`; returns false (and
// raises the device error flag) if it never completed.
__device__ __forceinline__ bool mbar_wait_bounded_ns(uint64_t *bar, uint32_t parity,
                                                     unsigned int *err,
                                                     unsigned long long limit_ns) {
  if (mbar_try_wait(bar, parity)) return true;
  const unsigned long long t0 = globaltimer_ns();
  while (!mbar_try_wait(bar, parity)) {
    if (globaltimer_ns() - t0 > limit_ns) {
      atomicOr(err, kErrWaitTimeout);
      return false;
    }
  }
  return true;
}

// Test aid behind mamba2_debug_stall_waits: when the translation unit's stall
// word is set, thread 0 of every CTA waits on a barrier that nothing completes
// until the (short) limit runs out, which raises kErrWaitTimeout exactly as a
// timed-out wait in the kernel's main loop does; the caller then returns before
// it has issued any asynchronous copy, MMA or cluster access, so nothing is in
// flight.  Every CTA of a launch reads the same word, so a cluster's CTAs all
// return together.
constexpr unsigned long long kTestStallNs = 20000000ull;  // 20 ms
__device__ __forceinline__ bool test_stall(const unsigned int *stall, unsigned int *err) {
  if (*reinterpret_cast<const volatile unsigned int *>(stall) == 0u) return false;
  __shared__ uint64_t dead;
  if (threadIdx.x == 0) {
    mbar_init(&dead, 1);
    mbar_wait_bounded_ns(&dead, 0, err, kTestStallNs);
  }
  return true;
}

// ---------------------------------------------------------------- checked build
// Built with -DMAMBA2_BOUNDS_CHECK (libmamba2ssd_checked.so, a debugging aid in
// place of a memory checker), every plain global load and store of the
// tensor-core prefill kernels and of the decode kernel is checked against the
// byte range of the buffer it addresses and against the alignment of its
// access size; an access that fails is skipped and raises kErrBounds in the
// kernel's error word (mamba2_device_errors bit 1).  Tensor-memory copies
// (TMA) are bounded by their tensor maps and need no check.  In the ordinary
// build the checks compile to nothing.
constexpr unsigned int kErrBounds = 2u;
// bit 2 of mamba2_device_errors: a packed-sequence prefill got sequence offsets
// that do not start at 0, decrease, or do not end at the total token count
constexpr unsigned int kErrSeqlens = 4u;
struct Span {  // [lo, hi) byte addresses of one device buffer (lo == hi: none)
  unsigned long long lo, hi;
};
inline Span span_of(const void *p, size_t bytes) {
  const unsigned long long a = reinterpret_cast<unsigned long long>(p);
  return Span{a, p == nullptr ? a : a + bytes};
}
#ifdef MAMBA2_BOUNDS_CHECK
__device__ __forceinline__ bool span_ok(const void *p, unsigned int bytes, unsigned int align,
                                        const Span &s, unsigned int *err) {
  const unsigned long long a = reinterpret_cast<unsigned long long>(p);
  if (a >= s.lo && a + bytes <= s.hi && (a & (unsigned long long)(align - 1)) == 0) return true;
  atomicOr(err, kErrBounds);
  return false;
}
// an access of `bytes` (1, 2, 4, 8 or 16) at p, aligned to its size
#define M2_OK(p, bytes, span, err) ::m2::span_ok((p), (bytes), (bytes), (span), (err))
// a bulk copy of `bytes` at p (16-byte aligned)
#define M2_OK_BULK(p, bytes, span, err) ::m2::span_ok((p), (bytes), 16u, (span), (err))
#else
#define M2_OK(p, bytes, span, err) true
#define M2_OK_BULK(p, bytes, span, err) true
#endif

// Host: read and clear the error words of the kernels that wait (one per
// translation unit).  Synchronous.
cudaError_t take_step_errors(unsigned int *out);
// Host: set the stall word of every translation unit whose kernels wait.
cudaError_t set_step_stall(unsigned int v);
cudaError_t set_prefill_tc_stall(unsigned int v);

// Host: true exactly once per CUDA context for each `slot` (0 .. 15): launch
// attributes (cudaFuncSetAttribute) belong to a context and are set again
// when the context is re-created.
bool first_use_in_context(int slot);
// Host: unique id of the calling thread's current CUDA context (0 if none).
unsigned long long current_context_id();

}  // namespace m2

// ---------------------------------------------------------------- tcgen05 / TMEM
namespace m2 {

// Shared-memory matrix descriptor, 128-byte swizzle, K-major canonical layout:
// rows of 64 16-bit elements (128 B), 8-row groups 1024 B apart (SBO); the
// tile base must be 1024-byte aligned.  LBO is unused for this layout.
__device__ __forceinline__ uint64_t umma_desc_sw128(uint32_t saddr) {
  uint64_t d = (uint64_t)((saddr >> 4) & 0x3FFFu);
  d |= (uint64_t)(16u >> 4) << 16;    // LBO (ignored)
  d |= (uint64_t)(1024u >> 4) << 32;  // SBO: 8 rows x 128 B
  d |= (uint64_t)1 << 46;             // descriptor version
  d |= (uint64_t)2 << 61;             // SWIZZLE_128B
  return d;
}
// Instruction descriptor of tcgen05.mma kind::f16: fp16 A and B (both K-major),
// fp32 accumulator, M x N.
__host__ __device__ constexpr uint32_t umma_idesc_f16(int M, int N) {
  return (1u << 4) | (0u << 7) | (0u << 10) | ((uint32_t)(N >> 3) << 17) |
         ((uint32_t)(M >> 4) << 24);
}
// Byte offset of element (r, k) in a K-major SW128 tile of 64-element rows.
__device__ __forceinline__ uint32_t sw128_off(int r, int k) {
  return (uint32_t)(r * 128 + ((((k >> 3) ^ r) & 7) << 4) + ((k & 7) << 1));
}
// Byte offset of the 16-byte chunk holding elements k..k+7 (k % 8 == 0).
__device__ __forceinline__ uint32_t sw128_chunk(int r, int k) {
  return (uint32_t)(r * 128 + ((((k >> 3) ^ r) & 7) << 4));
}

__device__ __forceinline__ void tmem_alloc(uint32_t *holder, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                   smem_u32(holder)),
               "r"(ncols)
               : "memory");
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}
// D[tmem] (+)= A[smem] * B[smem]^T, issued by one thread.
__device__ __forceinline__ void umma_f16(uint32_t tmem_d, uint64_t adesc, uint64_t bdesc,
                                         uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n"
      " tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n}" ::"r"(tmem_d),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}
// Arrive on `bar` when every MMA issued so far by this thread has completed.
__device__ __forceinline__ void umma_commit(uint64_t *bar) {
  asm volatile(
      "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
          smem_u32(bar))
      : "memory");
}
// 32 consecutive fp32 columns of this thread's TMEM lane (warp w reads lanes
// 32*(w%4) .. +31; taddr carries that lane offset in bits 16..31).
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, float (&v)[32]) {
  uint32_t r[32];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,"
      "%15,%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]),
        "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]),
        "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
  for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
}
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, float (&v)[16]) {
  uint32_t r[16];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,"
      "%15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15])
      : "r"(taddr));
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
  for (int i = 0; i < 16; ++i) v[i] = __uint_as_float(r[i]);
}
// Two 16-column loads (a, b) with one wait: both are in flight together.  The
// wait sits in the same asm statement, so no copy of an output register can
// be made before the data has arrived.
__device__ __forceinline__ void tmem_ld16x2(uint32_t ta, float (&va)[16], uint32_t tb,
                                            float (&vb)[16]) {
  uint32_t r[32];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,"
      "%15}, [%32];\n\t"
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,"
      "%28,%29,%30,%31}, [%33];\n\t"
      "tcgen05.wait::ld.sync.aligned;"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]),
        "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]),
        "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(ta), "r"(tb)
      : "memory");
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    va[i] = __uint_as_float(r[i]);
    vb[i] = __uint_as_float(r[16 + i]);
  }
}
// A 32-column load (a) and a 16-column load (b) with one wait.
__device__ __forceinline__ void tmem_ld32x16(uint32_t ta, float (&va)[32], uint32_t tb,
                                             float (&vb)[16]) {
  uint32_t r[48];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,"
      "%15,%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%48];\n\t"
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%32,%33,%34,%35,%36,%37,%38,%39,%40,%41,%42,%43,"
      "%44,%45,%46,%47}, [%49];\n\t"
      "tcgen05.wait::ld.sync.aligned;"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]),
        "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]),
        "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31]),
        "=r"(r[32]), "=r"(r[33]), "=r"(r[34]), "=r"(r[35]), "=r"(r[36]), "=r"(r[37]),
        "=r"(r[38]), "=r"(r[39]), "=r"(r[40]), "=r"(r[41]), "=r"(r[42]), "=r"(r[43]),
        "=r"(r[44]), "=r"(r[45]), "=r"(r[46]), "=r"(r[47])
      : "r"(ta), "r"(tb)
      : "memory");
#pragma unroll
  for (int i = 0; i < 32; ++i) va[i] = __uint_as_float(r[i]);
#pragma unroll
  for (int i = 0; i < 16; ++i) vb[i] = __uint_as_float(r[32 + i]);
}
// tcgen05.st of 16 columns without waiting for it to land; tmem_wait_st() before
// anything reads those columns back (this thread) or hands them to others.
__device__ __forceinline__ void tmem_st16_async(uint32_t taddr, const float (&v)[16]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,"
      "%14,%15,%16};" ::"r"(taddr),
      "r"(__float_as_uint(v[0])), "r"(__float_as_uint(v[1])), "r"(__float_as_uint(v[2])),
      "r"(__float_as_uint(v[3])), "r"(__float_as_uint(v[4])), "r"(__float_as_uint(v[5])),
      "r"(__float_as_uint(v[6])), "r"(__float_as_uint(v[7])), "r"(__float_as_uint(v[8])),
      "r"(__float_as_uint(v[9])), "r"(__float_as_uint(v[10])), "r"(__float_as_uint(v[11])),
      "r"(__float_as_uint(v[12])), "r"(__float_as_uint(v[13])), "r"(__float_as_uint(v[14])),
      "r"(__float_as_uint(v[15]))
      : "memory");
}
__device__ __forceinline__ void tmem_wait_st() {
  asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_st16(uint32_t taddr, const float (&v)[16]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,"
      "%14,%15,%16};" ::"r"(taddr),
      "r"(__float_as_uint(v[0])), "r"(__float_as_uint(v[1])), "r"(__float_as_uint(v[2])),
      "r"(__float_as_uint(v[3])), "r"(__float_as_uint(v[4])), "r"(__float_as_uint(v[5])),
      "r"(__float_as_uint(v[6])), "r"(__float_as_uint(v[7])), "r"(__float_as_uint(v[8])),
      "r"(__float_as_uint(v[9])), "r"(__float_as_uint(v[10])), "r"(__float_as_uint(v[11])),
      "r"(__float_as_uint(v[12])), "r"(__float_as_uint(v[13])), "r"(__float_as_uint(v[14])),
      "r"(__float_as_uint(v[15]))
      : "memory");
  asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_st32(uint32_t taddr, const float (&v)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,"
      "%14,%15,%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};" ::"r"(taddr),
      "r"(__float_as_uint(v[0])), "r"(__float_as_uint(v[1])), "r"(__float_as_uint(v[2])),
      "r"(__float_as_uint(v[3])), "r"(__float_as_uint(v[4])), "r"(__float_as_uint(v[5])),
      "r"(__float_as_uint(v[6])), "r"(__float_as_uint(v[7])), "r"(__float_as_uint(v[8])),
      "r"(__float_as_uint(v[9])), "r"(__float_as_uint(v[10])), "r"(__float_as_uint(v[11])),
      "r"(__float_as_uint(v[12])), "r"(__float_as_uint(v[13])), "r"(__float_as_uint(v[14])),
      "r"(__float_as_uint(v[15])), "r"(__float_as_uint(v[16])), "r"(__float_as_uint(v[17])),
      "r"(__float_as_uint(v[18])), "r"(__float_as_uint(v[19])), "r"(__float_as_uint(v[20])),
      "r"(__float_as_uint(v[21])), "r"(__float_as_uint(v[22])), "r"(__float_as_uint(v[23])),
      "r"(__float_as_uint(v[24])), "r"(__float_as_uint(v[25])), "r"(__float_as_uint(v[26])),
      "r"(__float_as_uint(v[27])), "r"(__float_as_uint(v[28])), "r"(__float_as_uint(v[29])),
      "r"(__float_as_uint(v[30])), "r"(__float_as_uint(v[31]))
      : "memory");
  asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}

// Two floats -> packed fp16x2 (round to nearest, saturating to the finite range).
__device__ __forceinline__ uint32_t pack_half2(float lo, float hi) {
  uint32_t r;
  asm("cvt.rn.satfinite.f16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
  return r;
}
__device__ __forceinline__ float2 unpack_half2(uint32_t v) {
  __half2 h = *reinterpret_cast<__half2 *>(&v);
  return __half22float2(h);
}

cudaError_t prefill_tc(const PrefillArgs &a);
size_t prefill_tc_workspace(const Problem &pr, bool varlen = false);
bool prefill_tc_supported(const Problem &pr, bool varlen = false);
cudaError_t take_prefill_tc_errors(unsigned int *out);
extern const char *const kPrefillTcStages[];
extern const int kPrefillTcStageCount;

}  // namespace m2
