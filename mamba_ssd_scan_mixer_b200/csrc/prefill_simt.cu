// Prefill of the Mamba-2 mixer core with CUDA-core fp32 arithmetic.
//
// This is the path for fp32 I/O (whose 1e-3 relative bound bf16 tensor-core
// operands cannot meet) and the reference-grade GPU path for any shape.  It
// evaluates the chunked (state-space duality) form of the selective scan of
// the Mamba-2 layer named on the state-spaces/mamba repository page
// (opendeer.net, "About the project"), in the order of the "Zamba2 hybrid
// architecture in Transformers" page (qwbw.cn), section 三 steps 2-4:
//
//   conv_silu      u = silu(conv1d(xBC) + b)        [b, L, conv_dim] fp32
//   conv_state_out last d_conv raw inputs -> conv state
//   dt_cumsum      dt = softplus(dt_raw + dt_bias); cum = chunk-local
//                  inclusive prefix sum of dt * A    [b, H, L] fp32 each
//   chunk_state    S_c = sum_s exp(cum_end - cum_s) dt_s x_s B_s^T
//   state_pass     H_0 = h_in; H_{c+1} = exp(cum_end) H_c + S_c  (S_c replaced
//                  in place by H_c, the state entering chunk c)
//   chunk_out      y_pre = diag block (C B^T o decay) (dt x) + exp(cum) C H_c^T + D x
//   gated_norm     y = rmsnorm(y_pre * silu(z)) * w over ngroups groups
//
// Workspace: u, dt, cum, chunk states, y_pre (all fp32), 256-byte aligned.
#include "common.cuh"

namespace m2 {
namespace {

constexpr int kConvTokens = 64;   // tokens per conv thread
constexpr int kTileT = 64;        // tokens per chunk_out block
constexpr int kTileS = 32;        // source tokens per chunk_out / chunk_state step
constexpr int kMaxOutPerThread = 32;  // P * N / 256 for P <= 64, N <= 128

struct Workspace {
  float *u, *dt, *cum, *states, *ypre;
};

Workspace carve(const Problem &pr, char *base) {
  Workspace w;
  size_t off = 0;
  auto take = [&](size_t bytes) {
    char *p = base + off;
    off += align_up(bytes, 256);
    return reinterpret_cast<float *>(p);
  };
  const size_t bL = (size_t)pr.batch * (size_t)pr.L;
  w.u = take(bL * pr.conv_dim * 4);
  w.dt = take(bL * pr.H * 4);
  w.cum = take(bL * pr.H * 4);
  w.states = take((size_t)pr.batch * pr.nchunks * pr.H * pr.P * pr.N * 4);
  w.ypre = take(bL * pr.d_inner * 4);
  return w;
}

// ---------------------------------------------------------------- conv + SiLU
template <typename T>
__global__ void conv_silu_kernel(Problem pr, const T *__restrict__ xBC, int64_t ld,
                                 const T *__restrict__ cs, int states_in,
                                 const float *__restrict__ w, const float *__restrict__ bias,
                                 float *__restrict__ u) {
  grid_dependency_wait();  // (launched as a dependent of the previous kernel)
  launch_dependents();
  const int64_t c = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (c >= pr.conv_dim) return;
  const int64_t bi = blockIdx.z, t0 = (int64_t)blockIdx.y * kConvTokens;
  const T *xb = xBC + bi * pr.L * ld;
  auto val = [&](int64_t tau) -> float {
    if (tau >= 0) return to_f(xb[tau * ld + c]);
    if (!states_in) return 0.0f;
    return to_f(cs[(bi * pr.conv_dim + c) * 4 + 4 + tau]);
  };
  const float w0 = w[c * 4 + 0], w1 = w[c * 4 + 1], w2 = w[c * 4 + 2], w3 = w[c * 4 + 3];
  const float b = bias[c];
  float v0 = val(t0 - 3), v1 = val(t0 - 2), v2 = val(t0 - 1);
  const int64_t t1 = min(t0 + kConvTokens, pr.L);
  for (int64_t t = t0; t < t1; ++t) {
    const float v3 = to_f(xb[t * ld + c]);
    const float pre = b + w0 * v0 + w1 * v1 + w2 * v2 + w3 * v3;
    u[(bi * pr.L + t) * pr.conv_dim + c] = silu_f(pre);
    v0 = v1;
    v1 = v2;
    v2 = v3;
  }
}

// Final conv state = last 4 raw inputs of [old state | new tokens].  Each
// thread reads all four inputs before writing, so the update is in place.
template <typename T>
__global__ void conv_state_out_kernel(Problem pr, const T *__restrict__ xBC, int64_t ld, T *cs,
                                      int states_in) {
  grid_dependency_wait();  // (launched as a dependent of the previous kernel)
  launch_dependents();
  const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= pr.batch * pr.conv_dim) return;
  const int64_t bi = i / pr.conv_dim, c = i % pr.conv_dim;
  const T *xb = xBC + bi * pr.L * ld;
  T v[4];
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    const int64_t tau = pr.L - 4 + k;
    if (tau >= 0) v[k] = xb[tau * ld + c];
    else v[k] = states_in ? cs[i * 4 + 4 + tau] : from_f<T>(0.0f);
  }
#pragma unroll
  for (int k = 0; k < 4; ++k) cs[i * 4 + k] = v[k];
}

// ---------------------------------------------------------------- dt, cumsum
// One block per (chunk, head, batch row), blockDim.x == Q.
template <typename T>
__global__ void dt_cumsum_kernel(Problem pr, const T *__restrict__ dt_raw, int64_t ld,
                                 const float *__restrict__ dt_bias, const float *__restrict__ A,
                                 float *__restrict__ dt_out, float *__restrict__ cum_out) {
  grid_dependency_wait();  // (launched as a dependent of the previous kernel)
  launch_dependents();
  __shared__ float warp_tot[32];
  const int h = blockIdx.y;
  const int64_t bi = blockIdx.z, t = (int64_t)blockIdx.x * pr.Q + threadIdx.x;
  const bool valid = t < pr.L;
  float dt = 0.0f;
  if (valid) dt = softplus_f(to_f(dt_raw[(bi * pr.L + t) * ld + h]) + dt_bias[h]);
  float v = dt * A[h];
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const float n = __shfl_up_sync(0xffffffffu, v, o);
    if (lane >= o) v += n;
  }
  if (lane == 31) warp_tot[wid] = v;
  __syncthreads();
  float prefix = 0.0f;
  for (int k = 0; k < wid; ++k) prefix += warp_tot[k];
  v += prefix;
  if (valid) {
    const int64_t o = (bi * pr.H + h) * pr.L + t;
    dt_out[o] = dt;
    cum_out[o] = v;
  }
}

// ---------------------------------------------------------------- chunk states
// One block (256 threads) per (chunk, head, batch row); output o = p * N + n.
__global__ void chunk_state_kernel(Problem pr, const float *__restrict__ u,
                                   const float *__restrict__ dtw, const float *__restrict__ cum,
                                   float *__restrict__ states) {
  grid_dependency_wait();  // (launched as a dependent of the previous kernel)
  launch_dependents();
  extern __shared__ float smem[];
  const int P = pr.P, N = pr.N;
  float *xs = smem;                 // [kTileS][P]
  float *bs = xs + kTileS * P;      // [kTileS][N]
  float *ws = bs + kTileS * N;      // [kTileS]
  const int chunk = blockIdx.x, h = blockIdx.y;
  const int64_t bi = blockIdx.z;
  const int g = h / pr.heads_per_group();
  const int64_t c0 = (int64_t)chunk * pr.Q, c1 = min(c0 + pr.Q, pr.L);
  const float *dth = dtw + (bi * pr.H + h) * pr.L;
  const float *cumh = cum + (bi * pr.H + h) * pr.L;
  const float cum_end = cumh[c1 - 1];
  const int nout = P * N;
  float acc[kMaxOutPerThread];
#pragma unroll
  for (int k = 0; k < kMaxOutPerThread; ++k) acc[k] = 0.0f;
  for (int64_t s0 = c0; s0 < c1; s0 += kTileS) {
    for (int i = threadIdx.x; i < kTileS * P; i += blockDim.x) {
      const int64_t s = s0 + i / P;
      xs[i] = (s < c1) ? u[(bi * pr.L + s) * pr.conv_dim + (int64_t)h * P + i % P] : 0.0f;
    }
    for (int i = threadIdx.x; i < kTileS * N; i += blockDim.x) {
      const int64_t s = s0 + i / N;
      bs[i] = (s < c1) ? u[(bi * pr.L + s) * pr.conv_dim + pr.d_inner + (int64_t)g * N + i % N]
                       : 0.0f;
    }
    if (threadIdx.x < kTileS) {
      const int64_t s = s0 + threadIdx.x;
      ws[threadIdx.x] = (s < c1) ? expf(cum_end - cumh[s]) * dth[s] : 0.0f;
    }
    __syncthreads();
#pragma unroll
    for (int k = 0; k < kMaxOutPerThread; ++k) {
      const int o = threadIdx.x + k * blockDim.x;
      if (o < nout) {
        const int p = o / N, n = o % N;
        float a = acc[k];
        for (int j = 0; j < kTileS; ++j) a += ws[j] * xs[j * P + p] * bs[j * N + n];
        acc[k] = a;
      }
    }
    __syncthreads();
  }
  float *out = states + ((bi * pr.nchunks + chunk) * pr.H + h) * (int64_t)nout;
#pragma unroll
  for (int k = 0; k < kMaxOutPerThread; ++k) {
    const int o = threadIdx.x + k * blockDim.x;
    if (o < nout) out[o] = acc[k];
  }
}

// ---------------------------------------------------------------- state passing
// states[c] holds S_c on entry and H_c (state entering chunk c) on exit.
__global__ void state_pass_kernel(Problem pr, float *__restrict__ states,
                                  const float *__restrict__ cum, float *ssm_state,
                                  int states_in) {
  grid_dependency_wait();  // (launched as a dependent of the previous kernel)
  launch_dependents();
  const int nout = pr.P * pr.N;
  const int o = blockIdx.x * blockDim.x + threadIdx.x;
  if (o >= nout) return;
  const int h = blockIdx.y;
  const int64_t bi = blockIdx.z;
  const int64_t hs_idx = (bi * pr.H + h) * (int64_t)nout + o;
  float hc = states_in ? ssm_state[hs_idx] : 0.0f;
  const float *cumh = cum + (bi * pr.H + h) * pr.L;
  for (int64_t c = 0; c < pr.nchunks; ++c) {
    const int64_t idx = ((bi * pr.nchunks + c) * pr.H + h) * (int64_t)nout + o;
    const float S = states[idx];
    states[idx] = hc;
    const int64_t last = min((c + 1) * pr.Q, pr.L) - 1;
    hc = expf(cumh[last]) * hc + S;
  }
  if (ssm_state != nullptr) ssm_state[hs_idx] = hc;
}

// ---------------------------------------------------------------- chunk output
// One block (256 threads) per (64-token tile, head, batch row).  Thread owns
// tokens ti = tid/16 + 16k (k < 4) and lanes p = tid%16 + 16j (j < P/16).
__global__ void chunk_out_kernel(Problem pr, const float *__restrict__ u,
                                 const float *__restrict__ dtw, const float *__restrict__ cum,
                                 const float *__restrict__ states, const float *__restrict__ Dp,
                                 float *__restrict__ ypre) {
  grid_dependency_wait();  // (launched as a dependent of the previous kernel)
  launch_dependents();
  extern __shared__ float smem[];
  const int P = pr.P, N = pr.N, NP = N + 1;
  float *Cs = smem;                   // [kTileT][N+1]
  float *Hs = Cs + kTileT * NP;       // [P][N+1]
  float *Bs = Hs + P * NP;            // [kTileS][N+1]
  float *xs = Bs + kTileS * NP;       // [kTileS][P]
  float *W = xs + kTileS * P;         // [kTileT][kTileS+1]
  float *cumT = W + kTileT * (kTileS + 1);  // [kTileT]
  float *cumS = cumT + kTileT;        // [kTileS]
  float *dtS = cumS + kTileS;         // [kTileS]

  const int h = blockIdx.y;
  const int64_t bi = blockIdx.z;
  const int g = h / pr.heads_per_group();
  const int64_t t0 = (int64_t)blockIdx.x * kTileT;
  const int64_t chunk = t0 / pr.Q, c0 = chunk * pr.Q;
  const int64_t tend = min(t0 + kTileT, pr.L);
  const float *dth = dtw + (bi * pr.H + h) * pr.L;
  const float *cumh = cum + (bi * pr.H + h) * pr.L;
  const int64_t offC = pr.d_inner + (int64_t)pr.G * N + (int64_t)g * N;
  const int64_t offB = pr.d_inner + (int64_t)g * N;

  for (int i = threadIdx.x; i < kTileT * N; i += blockDim.x) {
    const int ti = i / N, n = i % N;
    const int64_t t = t0 + ti;
    Cs[ti * NP + n] = (t < tend) ? u[(bi * pr.L + t) * pr.conv_dim + offC + n] : 0.0f;
  }
  const float *Hc = states + ((bi * pr.nchunks + chunk) * pr.H + h) * (int64_t)(P * N);
  for (int i = threadIdx.x; i < P * N; i += blockDim.x) Hs[(i / N) * NP + i % N] = Hc[i];
  for (int i = threadIdx.x; i < kTileT; i += blockDim.x)
    cumT[i] = (t0 + i < tend) ? cumh[t0 + i] : 0.0f;

  const int tq = threadIdx.x / 16, pq = threadIdx.x % 16, nj = P / 16;
  float acc[4][4];
#pragma unroll
  for (int k = 0; k < 4; ++k)
#pragma unroll
    for (int j = 0; j < 4; ++j) acc[k][j] = 0.0f;

  for (int64_t s0 = c0; s0 < tend; s0 += kTileS) {
    __syncthreads();
    for (int i = threadIdx.x; i < kTileS * N; i += blockDim.x) {
      const int sj = i / N, n = i % N;
      const int64_t s = s0 + sj;
      Bs[sj * NP + n] = (s < tend) ? u[(bi * pr.L + s) * pr.conv_dim + offB + n] : 0.0f;
    }
    for (int i = threadIdx.x; i < kTileS * P; i += blockDim.x) {
      const int64_t s = s0 + i / P;
      xs[i] = (s < tend) ? u[(bi * pr.L + s) * pr.conv_dim + (int64_t)h * P + i % P] : 0.0f;
    }
    if (threadIdx.x < kTileS) {
      const int64_t s = s0 + threadIdx.x;
      cumS[threadIdx.x] = (s < tend) ? cumh[s] : 0.0f;
      dtS[threadIdx.x] = (s < tend) ? dth[s] : 0.0f;
    }
    __syncthreads();
    for (int i = threadIdx.x; i < kTileT * kTileS; i += blockDim.x) {
      const int ti = i / kTileS, sj = i % kTileS;
      const int64_t t = t0 + ti, s = s0 + sj;
      float wv = 0.0f;
      if (s <= t && t < tend) {
        float cb = 0.0f;
        for (int n = 0; n < N; ++n) cb += Cs[ti * NP + n] * Bs[sj * NP + n];
        wv = cb * expf(cumT[ti] - cumS[sj]) * dtS[sj];
      }
      W[ti * (kTileS + 1) + sj] = wv;
    }
    __syncthreads();
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const int ti = tq + 16 * k;
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        if (j < nj) {
          const int p = pq + 16 * j;
          float a = acc[k][j];
          for (int sj = 0; sj < kTileS; ++sj) a += W[ti * (kTileS + 1) + sj] * xs[sj * P + p];
          acc[k][j] = a;
        }
      }
    }
  }
  // carried state, D skip, store
  const float Dh = Dp[h];
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    const int ti = tq + 16 * k;
    const int64_t t = t0 + ti;
    if (t >= tend) continue;
    const float carry = expf(cumT[ti]);
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      if (j < nj) {
        const int p = pq + 16 * j;
        float ch = 0.0f;
        for (int n = 0; n < N; ++n) ch += Cs[ti * NP + n] * Hs[p * NP + n];
        const float xv = u[(bi * pr.L + t) * pr.conv_dim + (int64_t)h * P + p];
        ypre[(bi * pr.L + t) * pr.d_inner + (int64_t)h * P + p] = acc[k][j] + carry * ch + Dh * xv;
      }
    }
  }
}

// ---------------------------------------------------------------- gated norm
// One block (256 threads) per (token, batch row).
template <typename T>
__global__ void gated_norm_kernel(Problem pr, const float *__restrict__ ypre,
                                  const T *__restrict__ z, int64_t ld_z,
                                  const float *__restrict__ w, T *__restrict__ y) {
  grid_dependency_wait();  // (launched as a dependent of the previous kernel)
  launch_dependents();
  __shared__ float red[33];
  const int64_t t = blockIdx.x, bi = blockIdx.y;
  const int64_t row = bi * pr.L + t;
  const float *yr = ypre + row * pr.d_inner;
  const T *zr = z + row * ld_z;
  T *outr = y + row * pr.d_inner;
  const int64_t gs = pr.d_inner / pr.G;
  for (int k = 0; k < pr.G; ++k) {
    float ss = 0.0f;
    for (int64_t i = threadIdx.x; i < gs; i += blockDim.x) {
      const int64_t c = k * gs + i;
      const float v = pr.nbg ? yr[c] : yr[c] * silu_f(to_f(zr[c]));
      ss += v * v;
    }
    ss = block_sum(ss, red);
    const float inv = rsqrtf(ss / (float)gs + pr.eps);
    for (int64_t i = threadIdx.x; i < gs; i += blockDim.x) {
      const int64_t c = k * gs + i;
      const float sz = silu_f(to_f(zr[c]));
      float o = pr.nbg ? yr[c] * inv * w[c] * sz : yr[c] * sz * inv * w[c];
      outr[c] = from_f<T>(o);
    }
  }
}

size_t chunk_out_smem(const Problem &pr) {
  const int NP = pr.N + 1;
  return sizeof(float) * (size_t)(kTileT * NP + pr.P * NP + kTileS * NP + kTileS * pr.P +
                                  kTileT * (kTileS + 1) + kTileT + 2 * kTileS);
}

size_t chunk_state_smem(const Problem &pr) {
  return sizeof(float) * (size_t)(kTileS * pr.P + kTileS * pr.N + kTileS);
}

// Launch of a kernel that may start while the previous one on the stream drains
// (programmatic dependent launch): each kernel waits for its predecessor before
// its first memory access, so only the launch latency overlaps.
template <typename... KArgs, typename... Args>
cudaError_t launch_dependent(void (*k)(KArgs...), dim3 grid, dim3 block, size_t smem,
                             cudaStream_t st, Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, k, static_cast<KArgs>(args)...);
}

template <typename T>
cudaError_t run(const PrefillArgs &a) {
  const Problem &pr = a.pr;
  cudaStream_t st = a.stream;
  const T *xBC = static_cast<const T *>(a.xBC);
  T *cs = static_cast<T *>(a.conv_state);
  Workspace w = carve(pr, a.ws);

  dim3 g1((unsigned)ceil_div(pr.conv_dim, 128), (unsigned)ceil_div(pr.L, kConvTokens),
          (unsigned)pr.batch);
  stage_mark(st, 0);
  conv_silu_kernel<T><<<g1, 128, 0, st>>>(pr, xBC, a.ld_xbc, cs, a.states_in, a.prm.conv_w,
                                          a.prm.conv_b, w.u);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  stage_mark(st, 1);
  if (cs != nullptr) {
    const int64_t n = pr.batch * pr.conv_dim;
    e = launch_dependent(conv_state_out_kernel<T>, dim3((unsigned)ceil_div(n, 256)), dim3(256), 0,
                         st, pr, xBC, a.ld_xbc, cs, a.states_in);
    if (e != cudaSuccess) return e;
  }
  dim3 g2((unsigned)pr.nchunks, pr.H, (unsigned)pr.batch);
  stage_mark(st, 2);
  e = launch_dependent(dt_cumsum_kernel<T>, g2, dim3(pr.Q), 0, st, pr,
                       static_cast<const T *>(a.dt_raw), a.ld_dt, a.prm.dt_bias, a.prm.A, w.dt,
                       w.cum);
  if (e != cudaSuccess) return e;
  stage_mark(st, 3);
  e = launch_dependent(chunk_state_kernel, g2, dim3(256), chunk_state_smem(pr), st, pr, w.u, w.dt,
                       w.cum, w.states);
  if (e != cudaSuccess) return e;
  dim3 g3((unsigned)ceil_div(pr.P * pr.N, 256), pr.H, (unsigned)pr.batch);
  stage_mark(st, 4);
  e = launch_dependent(state_pass_kernel, g3, dim3(256), 0, st, pr, w.states, w.cum, a.ssm_state,
                       a.states_in);
  if (e != cudaSuccess) return e;
  dim3 g4((unsigned)ceil_div(pr.L, kTileT), pr.H, (unsigned)pr.batch);
  stage_mark(st, 5);
  e = launch_dependent(chunk_out_kernel, g4, dim3(256), chunk_out_smem(pr), st, pr, w.u, w.dt,
                       w.cum, w.states, a.prm.D, w.ypre);
  if (e != cudaSuccess) return e;
  dim3 g5((unsigned)pr.L, (unsigned)pr.batch);
  stage_mark(st, 6);
  e = launch_dependent(gated_norm_kernel<T>, g5, dim3(256), 0, st, pr, w.ypre,
                       static_cast<const T *>(a.z), a.ld_z, a.prm.norm_w, static_cast<T *>(a.y));
  if (e != cudaSuccess) return e;
  stage_mark(st, 7);
  return cudaGetLastError();
}

}  // namespace

const char *const kPrefillSimtStages[] = {"conv_silu",   "conv_state_out", "dt_cumsum",
                                          "chunk_state", "state_pass",     "chunk_out",
                                          "gated_norm"};
const int kPrefillSimtStageCount = 7;

size_t prefill_simt_workspace(const Problem &pr) {
  const size_t bL = (size_t)pr.batch * (size_t)pr.L;
  return align_up(bL * pr.conv_dim * 4, 256) + 2 * align_up(bL * pr.H * 4, 256) +
         align_up((size_t)pr.batch * pr.nchunks * pr.H * pr.P * pr.N * 4, 256) +
         align_up(bL * pr.d_inner * 4, 256);
}

cudaError_t prefill_simt(const PrefillArgs &a) {
  // chunk_out needs up to ~100 KB of dynamic shared memory (N = 128, P = 64);
  // the attribute is per device, so it is set on every call (a host-side call)
  cudaError_t e = cudaFuncSetAttribute(chunk_out_kernel,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)chunk_out_smem(a.pr));
  if (e != cudaSuccess) return e;
  return a.pr.io == MAMBA2_BF16 ? run<__nv_bfloat16>(a) : run<float>(a);
}

}  // namespace m2
