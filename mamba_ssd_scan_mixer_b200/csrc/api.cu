// C ABI of libmamba2ssd.so: argument validation and launch.  See
// include/mamba2ssd.h for the contract of every entry point.
#include <cuda.h>

#include <algorithm>
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

namespace m2 {
namespace {
// Device memory of the host-buffer prefill: two staged input pieces, two output
// pieces, the carried states and the prefill workspace of one piece.
struct HostPlan {
  int64_t Lp, ldx, ldz, ldd;  // tokens per piece; staged row strides (elements)
  size_t x, z, d, in, y, cs, hs, ws, total;
};
size_t up256(size_t v) { return (v + 255) / 256 * 256; }
bool host_plan(const mamba2_dims *dims, const Problem &pr, HostPlan *o) {
  // pieces of whole chunks for every chunk size (multiples of 256 tokens), about
  // an eighth of the sequence each, so that the copies of the first and last
  // pieces, which nothing overlaps, are short (sixteenths were measured slower:
  // the per-piece launches and waits add up)
  const int64_t part = (pr.L + 7) / 8;
  o->Lp = std::min<int64_t>(std::max<int64_t>((part + 255) / 256 * 256, 256),
                            std::max<int64_t>(pr.L, 1));
  const size_t esz = pr.io == MAMBA2_BF16 ? 2 : 4;
  o->ldx = (pr.conv_dim + 7) / 8 * 8;
  o->ldz = (pr.d_inner + 7) / 8 * 8;
  o->ldd = (pr.H + 7) / 8 * 8;
  const size_t rows = (size_t)pr.batch * (size_t)o->Lp;
  o->x = up256(rows * o->ldx * esz);
  o->z = up256(rows * o->ldz * esz);
  o->d = up256(rows * o->ldd * esz);
  o->in = o->x + o->z + o->d;
  o->y = up256(rows * pr.d_inner * esz);
  o->cs = up256((size_t)pr.batch * pr.conv_dim * pr.K * esz);
  o->hs = up256((size_t)pr.batch * pr.H * pr.P * pr.N * 4);
  mamba2_dims dp = *dims;
  dp.seqlen = (int32_t)o->Lp;
  Problem pp;
  if (make_problem(&dp, true, &pp) != MAMBA2_OK) return false;
  o->ws = up256(prefill_workspace(pp));
  o->total = 2 * o->in + 2 * o->y + o->cs + o->hs + o->ws;
  return true;
}
// The two streams and eight events of the host-buffer prefill, kept per host
// thread and device for the thread's lifetime; a context that was destroyed and
// created again gets new ones (the old handles died with it).  Without a
// context id they are made for the call and released after it (owned).
struct HostPipe {
  unsigned long long ctx = 0;
  cudaStream_t up = nullptr, dn = nullptr;
  cudaEvent_t ev[8] = {};
};
bool make_pipe(HostPipe *p) {
  *p = HostPipe{};
  bool ok = cudaStreamCreateWithFlags(&p->up, cudaStreamNonBlocking) == cudaSuccess &&
            cudaStreamCreateWithFlags(&p->dn, cudaStreamNonBlocking) == cudaSuccess;
  for (int i = 0; ok && i < 8; ++i)
    ok = cudaEventCreateWithFlags(&p->ev[i], cudaEventDisableTiming) == cudaSuccess;
  return ok;
}
void release_pipe(HostPipe *p) {  // once their work is complete
  for (int i = 0; i < 8; ++i)
    if (p->ev[i] != nullptr) cudaEventDestroy(p->ev[i]);
  if (p->up != nullptr) cudaStreamDestroy(p->up);
  if (p->dn != nullptr) cudaStreamDestroy(p->dn);
  *p = HostPipe{};
}
bool host_pipe(HostPipe *call_owned, HostPipe **out, bool *owned) {
  thread_local HostPipe pipes[64];
  int dev = 0;
  const unsigned long long id = current_context_id();
  *owned = id == 0 || cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64;
  if (*owned) {
    *out = call_owned;
    return make_pipe(call_owned);
  }
  HostPipe &p = pipes[dev];
  if (p.ctx != id) {
    if (!make_pipe(&p)) {
      release_pipe(&p);
      return false;
    }
    p.ctx = id;
  }
  *out = &p;
  return true;
}
}  // namespace
}  // namespace m2

MAMBA2_API size_t mamba2_prefill_host_workspace_size(const mamba2_dims *dims) {
  Problem pr;
  m2::HostPlan plan;
  if (make_problem(dims, true, &pr) != MAMBA2_OK || !m2::host_plan(dims, pr, &plan)) return 0;
  return plan.total;
}

MAMBA2_API int mamba2_conv_ssd_prefill_host(
    const mamba2_dims *dims, const mamba2_params *params, const void *xBC,
    int64_t xBC_row_stride, const void *z, int64_t z_row_stride, const void *dt_raw,
    int64_t dt_row_stride, void *y, void *conv_state, float *ssm_state, int32_t states_in,
    void *workspace, size_t workspace_bytes, void *stream) {
  NvtxRange range("mamba2_conv_ssd_prefill_host");
  g_stage_events.n = 0;  // stage events are not recorded by this entry
  DisarmOnExit disarm;
  Problem pr;
  int st = make_problem(dims, true, &pr);
  if (st != MAMBA2_OK) return st;
  if (!params_ok(params)) return MAMBA2_ERR_INVALID_ARG;
  if (states_in != 0 && states_in != 1) return MAMBA2_ERR_INVALID_ARG;
  if (states_in && (conv_state == nullptr || ssm_state == nullptr)) return MAMBA2_ERR_INVALID_ARG;
  if (pr.batch == 0) return MAMBA2_OK;
  if (pr.L > 0 && (xBC == nullptr || z == nullptr || dt_raw == nullptr || y == nullptr))
    return MAMBA2_ERR_INVALID_ARG;
  if (pr.L > 0 &&
      (xBC_row_stride < pr.conv_dim || z_row_stride < pr.d_inner || dt_row_stride < pr.H))
    return MAMBA2_ERR_INVALID_ARG;
  m2::HostPlan pl;
  if (!m2::host_plan(dims, pr, &pl)) return MAMBA2_ERR_INVALID_ARG;
  if (workspace == nullptr || workspace_bytes < pl.total || !aligned(workspace, 256))
    return MAMBA2_ERR_WORKSPACE;
  const size_t esz = pr.io == MAMBA2_BF16 ? 2 : 4;
  char *w = static_cast<char *>(workspace);
  char *in[2] = {w, w + pl.in};
  char *yb[2] = {w + 2 * pl.in, w + 2 * pl.in + pl.y};
  char *cs_d = w + 2 * pl.in + 2 * pl.y;
  float *hs_d = reinterpret_cast<float *>(cs_d + pl.cs);
  char *ws_d = cs_d + pl.cs + pl.hs;
  const size_t cs_bytes = (size_t)pr.batch * pr.conv_dim * pr.K * esz;
  const size_t hs_bytes = (size_t)pr.batch * pr.H * pr.P * pr.N * 4;
  cudaStream_t cs_ = static_cast<cudaStream_t>(stream);
  // The usual layout, the three views side by side in one packed row (an in_proj
  // output): copy each row's span once and point the staged views into it, which
  // avoids copies of narrow rows (dt_raw's are a few hundred bytes).  Needs one
  // row stride, the device entry's alignments at the views' offsets in the row,
  // and a staged row that fits the slot.
  const char *hx = static_cast<const char *>(xBC), *hz = static_cast<const char *>(z),
             *hd = static_cast<const char *>(dt_raw);
  const char *base = std::min(hx, std::min(hz, hd));
  const char *span_end = std::max(hx + pr.conv_dim * esz,
                                  std::max(hz + pr.d_inner * esz, hd + pr.H * esz));
  const int64_t S = xBC_row_stride;
  const bool packed = pr.L > 0 && z_row_stride == S && dt_row_stride == S && S % 8 == 0 &&
                      span_end - base <= S * (int64_t)esz &&
                      (size_t)S <= (size_t)(pl.ldx + pl.ldz + pl.ldd) &&
                      (hx - base) % 16 == 0 && (hz - base) % 16 == 0 && (hd - base) % esz == 0;

  // Copies in on one stream, the prefill of each piece on the caller's stream,
  // copies out on a third: piece i + 1 arrives and piece i - 1 leaves while piece
  // i runs.  Two staging slots per direction; every reuse waits for its reader.
  m2::HostPipe own, *pipe = nullptr;
  bool owned = false;
  const bool ok = m2::host_pipe(&own, &pipe, &owned);
  if (!ok) {
    if (owned) m2::release_pipe(&own);
    return MAMBA2_ERR_CUDA;
  }
  cudaStream_t upl = pipe->up, dnl = pipe->dn;
  cudaEvent_t *ev = pipe->ev;  // start, in_ready[2], comp_done[2], out_free[2], done
  cudaEvent_t start = ev[0], done = ev[7];
  cudaEvent_t *in_ready = ev + 1, *comp_done = ev + 3, *out_free = ev + 5;
  int rc = MAMBA2_OK;
  auto chk = [&](cudaError_t e) {
    if (e != cudaSuccess && rc == MAMBA2_OK) rc = MAMBA2_ERR_CUDA;
    return rc == MAMBA2_OK;
  };
  if (ok) {
    // nothing of this call starts before the caller's earlier work on its stream
    chk(cudaEventRecord(start, cs_));
    chk(cudaStreamWaitEvent(upl, start, 0));
    chk(cudaStreamWaitEvent(dnl, start, 0));
    const int64_t np = pr.L > 0 ? (pr.L + pl.Lp - 1) / pl.Lp : 0;
    if (states_in && np > 0) {
      chk(cudaMemcpyAsync(cs_d, conv_state, cs_bytes, cudaMemcpyHostToDevice, upl));
      chk(cudaMemcpyAsync(hs_d, ssm_state, hs_bytes, cudaMemcpyHostToDevice, upl));
    }
    if (np == 0 && !states_in) {  // no tokens and no carried states: they start at zero
      chk(cudaMemsetAsync(cs_d, 0, cs_bytes, dnl));
      chk(cudaMemsetAsync(hs_d, 0, hs_bytes, dnl));
    }
    for (int64_t i = 0; i < np && rc == MAMBA2_OK; ++i) {
      const int s = (int)(i & 1);
      const int64_t t0 = i * pl.Lp, Li = std::min<int64_t>(pl.Lp, pr.L - t0);
      char *xs = in[s], *zs = in[s] + pl.x, *ds = in[s] + pl.x + pl.z;
      int64_t lx = pl.ldx, lz = pl.ldz, ld = pl.ldd;
      if (packed) {
        xs = in[s] + (hx - base);
        zs = in[s] + (hz - base);
        ds = in[s] + (hd - base);
        lx = lz = ld = S;
      }
      if (i >= 2) chk(cudaStreamWaitEvent(upl, comp_done[s], 0));  // slot s read by piece i - 2
      if (packed) {  // rows bi L + t0 .. + Li of every batch row: their spans
        const size_t row = (size_t)S * esz, span = (size_t)(span_end - base);
        for (int64_t bi = 0; bi < pr.batch && rc == MAMBA2_OK; ++bi) {
          const size_t r0 = (size_t)(bi * pr.L + t0), d0 = (size_t)(bi * pl.Lp);
          if (span == row)
            chk(cudaMemcpyAsync(in[s] + d0 * row, base + r0 * row, (size_t)Li * row,
                                cudaMemcpyHostToDevice, upl));
          else
            chk(cudaMemcpy2DAsync(in[s] + d0 * row, row, base + r0 * row, row, span, Li,
                                  cudaMemcpyHostToDevice, upl));
        }
      }
      for (int64_t bi = 0; !packed && bi < pr.batch && rc == MAMBA2_OK; ++bi) {
        const size_t r0 = (size_t)(bi * pr.L + t0), d0 = (size_t)(bi * pl.Lp);
        chk(cudaMemcpy2DAsync(xs + d0 * pl.ldx * esz, pl.ldx * esz,
                              static_cast<const char *>(xBC) + r0 * xBC_row_stride * esz,
                              xBC_row_stride * esz, pr.conv_dim * esz, Li,
                              cudaMemcpyHostToDevice, upl));
        chk(cudaMemcpy2DAsync(zs + d0 * pl.ldz * esz, pl.ldz * esz,
                              static_cast<const char *>(z) + r0 * z_row_stride * esz,
                              z_row_stride * esz, pr.d_inner * esz, Li, cudaMemcpyHostToDevice,
                              upl));
        chk(cudaMemcpy2DAsync(ds + d0 * pl.ldd * esz, pl.ldd * esz,
                              static_cast<const char *>(dt_raw) + r0 * dt_row_stride * esz,
                              dt_row_stride * esz, pr.H * esz, Li, cudaMemcpyHostToDevice, upl));
      }
      chk(cudaEventRecord(in_ready[s], upl));
      chk(cudaStreamWaitEvent(cs_, in_ready[s], 0));
      if (i >= 2) chk(cudaStreamWaitEvent(cs_, out_free[s], 0));  // y slot s copied out
      if (rc != MAMBA2_OK) break;
      // the piece's batch rows are Lp apart in the staging slot: one batch row at
      // a time when the last piece is shorter, else all rows in one call
      mamba2_dims di = *dims;
      di.seqlen = (int32_t)Li;
      const int32_t sin = (i > 0 || states_in) ? 1 : 0;
      if (Li == pl.Lp || pr.batch == 1) {
        rc = m2::prefill_entry(&di, params, xs, lx, zs, lz, ds, ld, nullptr, yb[s], cs_d, hs_d,
                               sin, ws_d, pl.ws, cs_);
      } else {
        di.batch = 1;
        for (int64_t bi = 0; bi < pr.batch && rc == MAMBA2_OK; ++bi) {
          const size_t d0 = (size_t)(bi * pl.Lp);
          rc = m2::prefill_entry(&di, params, xs + d0 * lx * esz, lx, zs + d0 * lz * esz, lz,
                                 ds + d0 * ld * esz, ld, nullptr, yb[s] + d0 * pr.d_inner * esz,
                                 cs_d + (size_t)bi * pr.conv_dim * pr.K * esz,
                                 hs_d + (size_t)bi * pr.H * pr.P * pr.N, sin, ws_d, pl.ws, cs_);
        }
      }
      if (rc != MAMBA2_OK) break;
      chk(cudaEventRecord(comp_done[s], cs_));
      chk(cudaStreamWaitEvent(dnl, comp_done[s], 0));
      // y rows of the piece: batch row bi of the slot at bi Lp rows
      chk(cudaMemcpy2DAsync(static_cast<char *>(y) + (size_t)t0 * pr.d_inner * esz,
                            (size_t)pr.L * pr.d_inner * esz, yb[s],
                            (size_t)pl.Lp * pr.d_inner * esz, (size_t)Li * pr.d_inner * esz,
                            pr.batch, cudaMemcpyDeviceToHost, dnl));
      chk(cudaEventRecord(out_free[s], dnl));
    }
    if (rc == MAMBA2_OK && (np > 0 || !states_in)) {  // (no tokens: carried states unchanged)
      if (conv_state != nullptr)
        chk(cudaMemcpyAsync(conv_state, cs_d, cs_bytes, cudaMemcpyDeviceToHost, dnl));
      if (ssm_state != nullptr)
        chk(cudaMemcpyAsync(ssm_state, hs_d, hs_bytes, cudaMemcpyDeviceToHost, dnl));
    }
    // the caller's stream resumes after everything this call enqueued
    cudaEventRecord(in_ready[0], upl);
    cudaEventRecord(done, dnl);
    cudaStreamWaitEvent(cs_, in_ready[0], 0);
    cudaStreamWaitEvent(cs_, done, 0);
  } else {
    rc = MAMBA2_ERR_CUDA;
  }
  if (owned) m2::release_pipe(&own);
  return rc;
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
