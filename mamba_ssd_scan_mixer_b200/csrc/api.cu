// C ABI of libmamba2ssd.so: argument validation and launch.  See
// include/mamba2ssd.h for the contract of every entry point.
#include <cuda.h>

#include <cmath>
#include <cstring>
#include <mutex>

#include "common.cuh"

namespace m2 {
namespace {

bool aligned(const void *p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

bool pow2_in(int v, int lo, int hi) { return v >= lo && v <= hi && (v & (v - 1)) == 0; }

// Validates the sizes shared by prefill and decode and fills `pr`.
int make_problem(const mamba2_dims *d, bool prefill, Problem *pr) {
  if (d == nullptr) return MAMBA2_ERR_INVALID_ARG;
  if (d->batch < 0 || d->nheads < 1 || d->ngroups < 1 || d->headdim < 1 || d->dstate < 1 ||
      d->d_conv < 1)
    return MAMBA2_ERR_INVALID_ARG;
  if (prefill && d->seqlen < 0) return MAMBA2_ERR_INVALID_ARG;
  if (d->nheads % d->ngroups != 0) return MAMBA2_ERR_INVALID_ARG;
  if (d->io_dtype != MAMBA2_F32 && d->io_dtype != MAMBA2_BF16) return MAMBA2_ERR_INVALID_ARG;
  if (d->norm_before_gate != 0 && d->norm_before_gate != 1) return MAMBA2_ERR_INVALID_ARG;
  if (!(d->norm_eps > 0.0f) || !std::isfinite(d->norm_eps)) return MAMBA2_ERR_INVALID_ARG;
  if (d->d_conv != 4) return MAMBA2_ERR_UNSUPPORTED;
  if (!pow2_in(d->headdim, 16, 64) || !pow2_in(d->dstate, 16, 128))
    return MAMBA2_ERR_UNSUPPORTED;
  if (prefill && d->chunk_size != 64 && d->chunk_size != 128 && d->chunk_size != 256)
    return MAMBA2_ERR_UNSUPPORTED;
  if (d->batch > 65535 || d->nheads > 65535) return MAMBA2_ERR_UNSUPPORTED;  // grid y/z limits
  pr->batch = d->batch;
  pr->L = prefill ? d->seqlen : 1;
  pr->H = d->nheads;
  pr->P = d->headdim;
  pr->N = d->dstate;
  pr->G = d->ngroups;
  pr->K = d->d_conv;
  pr->Q = prefill ? d->chunk_size : 1;
  pr->io = d->io_dtype;
  pr->nbg = d->norm_before_gate;
  pr->eps = d->norm_eps;
  pr->d_inner = (int64_t)pr->H * pr->P;
  pr->conv_dim = pr->d_inner + 2LL * pr->G * pr->N;
  pr->nchunks = prefill ? ceil_div(pr->L, pr->Q) : 1;
  if (prefill && pr->L > (int64_t)1 << 31) return MAMBA2_ERR_UNSUPPORTED;  // grid x limit
  return MAMBA2_OK;
}

// The prefill kernels a problem runs on: the tensor-core path for bf16 I/O at
// headdim 64 / d_state 64, the fp32 CUDA-core path otherwise.
bool use_tc(const Problem &pr) { return prefill_tc_supported(pr); }

size_t prefill_workspace(const Problem &pr) {
  return use_tc(pr) ? prefill_tc_workspace(pr) : prefill_simt_workspace(pr);
}

bool params_ok(const mamba2_params *p) {
  return p != nullptr && p->conv_w && p->conv_b && p->dt_bias && p->A && p->D && p->norm_w &&
         aligned(p->conv_w, 16);
}

// Disarms the stage events when a call returns, whatever the path taken.
struct DisarmOnExit {
  ~DisarmOnExit() { g_stage_events.n = 0; }
};

}  // namespace

thread_local StageEvents g_stage_events = {{}, 0};

// Driver entry points fetched through the runtime, so that the library has no
// load-time dependency on libcuda (it loads, and its host logic is testable,
// on a machine without a driver).
template <typename F>
F driver_fn(const char *name) {
  void *p = nullptr;
  cudaDriverEntryPointQueryResult q;
  if (cudaGetDriverEntryPoint(name, &p, cudaEnableDefault, &q) != cudaSuccess ||
      q != cudaDriverEntryPointSuccess) {
    cudaGetLastError();
    return nullptr;
  }
  return reinterpret_cast<F>(p);
}

unsigned long long current_context_id() {
  using GetCurrent = CUresult (*)(CUcontext *);
  using GetId = CUresult (*)(CUcontext, unsigned long long *);
  static const GetCurrent get_current = driver_fn<GetCurrent>("cuCtxGetCurrent");
  static const GetId get_id = driver_fn<GetId>("cuCtxGetId");
  if (get_current == nullptr || get_id == nullptr) return 0;
  CUcontext ctx = nullptr;
  unsigned long long id = 0;
  if (get_current(&ctx) != CUDA_SUCCESS || ctx == nullptr || get_id(ctx, &id) != CUDA_SUCCESS)
    return 0;
  return id;
}

bool first_use_in_context(int slot) {
  static std::mutex mu;
  static unsigned long long seen[64][16] = {};
  int dev = 0;
  if (slot < 0 || slot >= 16 || cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64)
    return true;
  const unsigned long long id = current_context_id();
  if (id == 0) return true;
  std::lock_guard<std::mutex> lock(mu);
  if (seen[dev][slot] == id) return false;
  seen[dev][slot] = id;
  return true;
}

int validate_prefill_dims(const mamba2_dims *dims) {
  Problem pr;
  return make_problem(dims, true, &pr);
}

}  // namespace m2

using namespace m2;

extern "C" {

MAMBA2_API const char *mamba2_status_string(int status) {
  switch (status) {
    case MAMBA2_OK: return "ok";
    case MAMBA2_ERR_INVALID_ARG: return "invalid argument";
    case MAMBA2_ERR_UNSUPPORTED: return "unsupported configuration";
    case MAMBA2_ERR_WORKSPACE: return "workspace missing or too small";
    case MAMBA2_ERR_CUDA: return "CUDA error";
    default: return "unknown status";
  }
}

MAMBA2_API int mamba2_version(void) { return 100; }

MAMBA2_API int mamba2_record_stage_events(void *const *events, int n_events) {
  if (n_events < 0 || n_events > kMaxStageEvents || (n_events > 0 && events == nullptr))
    return MAMBA2_ERR_INVALID_ARG;
  for (int i = 0; i < n_events; ++i) g_stage_events.ev[i] = static_cast<cudaEvent_t>(events[i]);
  g_stage_events.n = n_events;
  return MAMBA2_OK;
}

MAMBA2_API int mamba2_device_errors(unsigned int *flags) {
  if (flags == nullptr) return MAMBA2_ERR_INVALID_ARG;
  *flags = 0;
  if (cudaDeviceSynchronize() != cudaSuccess) return MAMBA2_ERR_CUDA;
  unsigned int f = 0;
  if (take_step_errors(&f) != cudaSuccess) return MAMBA2_ERR_CUDA;
  *flags |= f;
  if (take_prefill_tc_errors(&f) != cudaSuccess) return MAMBA2_ERR_CUDA;
  *flags |= f;
  return MAMBA2_OK;
}

MAMBA2_API int mamba2_debug_stall_waits(int enable) {
  if (enable != 0 && enable != 1) return MAMBA2_ERR_INVALID_ARG;
  if (cudaDeviceSynchronize() != cudaSuccess) return MAMBA2_ERR_CUDA;
  if (set_step_stall((unsigned)enable) != cudaSuccess ||
      set_prefill_tc_stall((unsigned)enable) != cudaSuccess)
    return MAMBA2_ERR_CUDA;
  return MAMBA2_OK;
}

MAMBA2_API int mamba2_stage_names(int kind, const mamba2_dims *dims, const char **names,
                                  int max_names) {
  Problem pr;
  if (kind != 0 && kind != 1 && kind != 2) return MAMBA2_ERR_INVALID_ARG;
  if (make_problem(dims, kind != 1, &pr) != MAMBA2_OK) return MAMBA2_ERR_INVALID_ARG;
  const bool tc = kind == 0 && use_tc(pr);
  const char *const *list = kind == 2   ? kBackwardStages
                            : kind == 1 ? kStepSimtStages
                            : tc        ? kPrefillTcStages
                                        : kPrefillSimtStages;
  const int n = kind == 2   ? kBackwardStageCount
                : kind == 1 ? kStepSimtStageCount
                : tc        ? kPrefillTcStageCount
                            : kPrefillSimtStageCount;
  for (int i = 0; names != nullptr && i < n && i < max_names; ++i) names[i] = list[i];
  return n;
}

MAMBA2_API size_t mamba2_prefill_workspace_size(const mamba2_dims *dims) {
  Problem pr;
  if (make_problem(dims, true, &pr) != MAMBA2_OK) return 0;
  return prefill_workspace(pr);
}

namespace m2 {
namespace {
// The shared body of the fixed-length and the packed-sequence prefill: dims,
// pointers and strides checked, the no-token case, then the launch.
int prefill_entry(const mamba2_dims *dims, const mamba2_params *params, const void *xBC,
                  int64_t xBC_row_stride, const void *z, int64_t z_row_stride,
                  const void *dt_raw, int64_t dt_row_stride, const int32_t *cu_seqlens,
                  void *y, void *conv_state, float *ssm_state, int32_t states_in,
                  void *workspace, size_t workspace_bytes, void *stream) {
  Problem pr;
  int st = make_problem(dims, true, &pr);
  if (st != MAMBA2_OK) return st;
  const bool varlen = cu_seqlens != nullptr;
  if (!params_ok(params)) return MAMBA2_ERR_INVALID_ARG;
  if (states_in != 0 && states_in != 1) return MAMBA2_ERR_INVALID_ARG;
  if (states_in && (conv_state == nullptr || ssm_state == nullptr)) return MAMBA2_ERR_INVALID_ARG;
  if (ssm_state != nullptr && !aligned(ssm_state, 16)) return MAMBA2_ERR_INVALID_ARG;
  const size_t esz = pr.io == MAMBA2_BF16 ? 2 : 4;
  if (conv_state != nullptr && !aligned(conv_state, esz)) return MAMBA2_ERR_INVALID_ARG;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (pr.batch == 0) return MAMBA2_OK;
  if (pr.L > 0) {
    if (xBC == nullptr || z == nullptr || dt_raw == nullptr || y == nullptr)
      return MAMBA2_ERR_INVALID_ARG;
    if (xBC_row_stride < pr.conv_dim || z_row_stride < pr.d_inner || dt_row_stride < pr.H)
      return MAMBA2_ERR_INVALID_ARG;
    if (xBC_row_stride % 8 != 0 || z_row_stride % 8 != 0) return MAMBA2_ERR_INVALID_ARG;
    if (!aligned(xBC, 16) || !aligned(z, 16) || !aligned(y, 16) || !aligned(dt_raw, esz))
      return MAMBA2_ERR_INVALID_ARG;
    if (varlen && !prefill_tc_supported(pr, true)) return MAMBA2_ERR_UNSUPPORTED;
    const size_t need = varlen ? prefill_tc_workspace(pr, true) : prefill_workspace(pr);
    if (workspace == nullptr || workspace_bytes < need || !aligned(workspace, 256))
      return MAMBA2_ERR_WORKSPACE;
  } else {
    // no new tokens: the states pass through, or start (and stay) at zero
    if (!states_in) {
      if (conv_state != nullptr &&
          cudaMemsetAsync(conv_state, 0, (size_t)pr.batch * pr.conv_dim * pr.K * esz, s) !=
              cudaSuccess)
        return MAMBA2_ERR_CUDA;
      if (ssm_state != nullptr &&
          cudaMemsetAsync(ssm_state, 0, (size_t)pr.batch * pr.H * pr.P * pr.N * 4, s) !=
              cudaSuccess)
        return MAMBA2_ERR_CUDA;
    }
    return MAMBA2_OK;
  }
  PrefillArgs a;
  a.pr = pr;
  a.prm = *params;
  a.xBC = xBC;
  a.ld_xbc = xBC_row_stride;
  a.z = z;
  a.ld_z = z_row_stride;
  a.dt_raw = dt_raw;
  a.ld_dt = dt_row_stride;
  a.y = y;
  a.conv_state = conv_state;
  a.ssm_state = ssm_state;
  a.states_in = states_in;
  a.ws = static_cast<char *>(workspace);
  a.stream = s;
  a.cu_seqlens = cu_seqlens;
  return (varlen || use_tc(pr) ? prefill_tc(a) : prefill_simt(a)) == cudaSuccess
             ? MAMBA2_OK
             : MAMBA2_ERR_CUDA;
}
}  // namespace
}  // namespace m2

MAMBA2_API int mamba2_conv_ssd_prefill(const mamba2_dims *dims, const mamba2_params *params,
                                       const void *xBC, int64_t xBC_row_stride, const void *z,
                                       int64_t z_row_stride, const void *dt_raw,
                                       int64_t dt_row_stride, void *y, void *conv_state,
                                       float *ssm_state, int32_t states_in, void *workspace,
                                       size_t workspace_bytes, void *stream) {
  NvtxRange range("mamba2_conv_ssd_prefill");
  DisarmOnExit disarm;
  return m2::prefill_entry(dims, params, xBC, xBC_row_stride, z, z_row_stride, dt_raw,
                           dt_row_stride, nullptr, y, conv_state, ssm_state, states_in,
                           workspace, workspace_bytes, stream);
}

MAMBA2_API size_t mamba2_prefill_varlen_workspace_size(const mamba2_dims *dims) {
  Problem pr;
  if (make_problem(dims, true, &pr) != MAMBA2_OK || pr.L < 1 || !prefill_tc_supported(pr, true))
    return 0;
  return prefill_tc_workspace(pr, true);
}

MAMBA2_API int mamba2_conv_ssd_prefill_varlen(
    const mamba2_dims *dims, const mamba2_params *params, const void *xBC,
    int64_t xBC_row_stride, const void *z, int64_t z_row_stride, const void *dt_raw,
    int64_t dt_row_stride, const int32_t *cu_seqlens, void *y, void *conv_state,
    float *ssm_state, int32_t states_in, void *workspace, size_t workspace_bytes, void *stream) {
  NvtxRange range("mamba2_conv_ssd_prefill_varlen");
  DisarmOnExit disarm;
  if (cu_seqlens == nullptr || !m2::aligned(cu_seqlens, 4)) return MAMBA2_ERR_INVALID_ARG;
  return m2::prefill_entry(dims, params, xBC, xBC_row_stride, z, z_row_stride, dt_raw,
                           dt_row_stride, cu_seqlens, y, conv_state, ssm_state, states_in,
                           workspace, workspace_bytes, stream);
}

MAMBA2_API int mamba2_ssd_step(const mamba2_dims *dims, const mamba2_params *params,
                               const void *xBC, int64_t xBC_row_stride, const void *z,
                               int64_t z_row_stride, const void *dt_raw, int64_t dt_row_stride,
                               void *y, void *conv_state, float *ssm_state, void *stream) {
  NvtxRange range("mamba2_ssd_step");
  DisarmOnExit disarm;
  Problem pr;
  int st = make_problem(dims, false, &pr);
  if (st != MAMBA2_OK) return st;
  if (!params_ok(params)) return MAMBA2_ERR_INVALID_ARG;
  if (pr.batch == 0) return MAMBA2_OK;
  if (xBC == nullptr || z == nullptr || dt_raw == nullptr || y == nullptr ||
      conv_state == nullptr || ssm_state == nullptr)
    return MAMBA2_ERR_INVALID_ARG;
  const size_t esz = pr.io == MAMBA2_BF16 ? 2 : 4;
  if (xBC_row_stride < pr.conv_dim || z_row_stride < pr.d_inner || dt_row_stride < pr.H)
    return MAMBA2_ERR_INVALID_ARG;
  if (xBC_row_stride % 8 != 0 || z_row_stride % 8 != 0) return MAMBA2_ERR_INVALID_ARG;
  if (!aligned(xBC, 16) || !aligned(z, 16) || !aligned(y, 16) || !aligned(ssm_state, 16) ||
      !aligned(conv_state, 16) || !aligned(dt_raw, esz))
    return MAMBA2_ERR_INVALID_ARG;
  StepArgs a;
  a.pr = pr;
  a.prm = *params;
  a.xBC = xBC;
  a.ld_xbc = xBC_row_stride;
  a.z = z;
  a.ld_z = z_row_stride;
  a.dt_raw = dt_raw;
  a.ld_dt = dt_row_stride;
  a.y = y;
  a.conv_state = conv_state;
  a.ssm_state = ssm_state;
  a.stream = static_cast<cudaStream_t>(stream);
  return step_simt(a) == cudaSuccess ? MAMBA2_OK : MAMBA2_ERR_CUDA;
}

MAMBA2_API size_t mamba2_prefill_backward_workspace_size(const mamba2_dims *dims) {
  Problem pr;
  if (make_problem(dims, true, &pr) != MAMBA2_OK) return 0;
  return backward_workspace(pr);
}

MAMBA2_API int mamba2_conv_ssd_prefill_backward(
    const mamba2_dims *dims, const mamba2_params *params, const void *xBC,
    int64_t xBC_row_stride, const void *z, int64_t z_row_stride, const void *dt_raw,
    int64_t dt_row_stride, const void *conv_state_in, const float *ssm_state_in, const void *dy,
    const float *d_ssm_state_out, void *d_xBC, void *d_z, void *d_dt_raw, float *d_conv_w,
    float *d_conv_b, float *d_dt_bias, float *d_A, float *d_D, float *d_norm_w,
    void *d_conv_state_in, float *d_ssm_state_in, void *workspace, size_t workspace_bytes,
    void *stream) {
  NvtxRange range("mamba2_conv_ssd_prefill_backward");
  DisarmOnExit disarm;
  Problem pr;
  int st = make_problem(dims, true, &pr);
  if (st != MAMBA2_OK) return st;
  if (!params_ok(params)) return MAMBA2_ERR_INVALID_ARG;
  if (d_conv_w == nullptr || d_conv_b == nullptr || d_dt_bias == nullptr || d_A == nullptr ||
      d_D == nullptr || d_norm_w == nullptr)
    return MAMBA2_ERR_INVALID_ARG;
  const int64_t bl = pr.batch * pr.L;
  if (bl > 0 && (xBC == nullptr || z == nullptr || dt_raw == nullptr || dy == nullptr ||
                 d_xBC == nullptr || d_z == nullptr || d_dt_raw == nullptr))
    return MAMBA2_ERR_INVALID_ARG;
  const size_t esz = pr.io == MAMBA2_BF16 ? 2 : 4;
  if (xBC_row_stride < pr.conv_dim || z_row_stride < pr.d_inner || dt_row_stride < pr.H)
    return MAMBA2_ERR_INVALID_ARG;
  const void *io_ptrs[] = {xBC, z, dt_raw, dy, d_xBC, d_z, d_dt_raw, conv_state_in,
                           d_conv_state_in};  // element-aligned
  const void *f32_ptrs[] = {ssm_state_in, d_ssm_state_out, d_ssm_state_in, d_conv_w,
                            d_conv_b,     d_dt_bias,       d_A,            d_D, d_norm_w};
  for (const void *q : io_ptrs)
    if (!aligned(q, esz)) return MAMBA2_ERR_INVALID_ARG;
  for (const void *q : f32_ptrs)
    if (!aligned(q, 4)) return MAMBA2_ERR_INVALID_ARG;
  if (workspace == nullptr || !aligned(workspace, 256)) return MAMBA2_ERR_WORKSPACE;
  if (workspace_bytes < backward_workspace(pr)) return MAMBA2_ERR_WORKSPACE;
  BackwardArgs a;
  a.pr = pr;
  a.prm = *params;
  a.xBC = xBC;
  a.ld_xbc = xBC_row_stride;
  a.z = z;
  a.ld_z = z_row_stride;
  a.dt_raw = dt_raw;
  a.ld_dt = dt_row_stride;
  a.conv_state_in = conv_state_in;
  a.ssm_state_in = ssm_state_in;
  a.dy = dy;
  a.d_ssm_state_out = d_ssm_state_out;
  a.d_xBC = d_xBC;
  a.d_z = d_z;
  a.d_dt_raw = d_dt_raw;
  a.d_conv_w = d_conv_w;
  a.d_conv_b = d_conv_b;
  a.d_dt_bias = d_dt_bias;
  a.d_A = d_A;
  a.d_D = d_D;
  a.d_norm_w = d_norm_w;
  a.d_conv_state_in = d_conv_state_in;
  a.d_ssm_state_in = d_ssm_state_in;
  a.ws = static_cast<char *>(workspace);
  a.stream = static_cast<cudaStream_t>(stream);
  return prefill_backward(a) == cudaSuccess ? MAMBA2_OK : MAMBA2_ERR_CUDA;
}

}  // extern "C"
