// Single-token decode step of the Mamba-2 mixer core ("Zamba2 hybrid
// architecture in Transformers", qwbw.cn, section 三 step 3: with the states
// cached and one new token, the scan becomes one recurrent state update).
//
// One block per batch row does the whole row: conv-state shift and conv +
// SiLU for all conv_dim channels into shared memory, dt per head, the state
// update and C contraction head by head (the fp32 state is streamed as
// float4, updated in place), then the gated group RMSNorm over the row.
#include "common.cuh"

namespace m2 {
namespace {

template <typename T>
__global__ void __launch_bounds__(256)
    ssd_step_kernel(Problem pr, mamba2_params prm, const T *__restrict__ xBC, int64_t ld_x,
                    const T *__restrict__ z, int64_t ld_z, const T *__restrict__ dt_raw,
                    int64_t ld_dt, T *__restrict__ y, T *__restrict__ conv_state,
                    float *__restrict__ ssm) {
  extern __shared__ float smem[];
  const int H = pr.H, P = pr.P, N = pr.N;
  float *u_s = smem;                   // [conv_dim]
  float *y_s = u_s + pr.conv_dim;      // [d_inner]
  float *dt_s = y_s + pr.d_inner;      // [H]
  float *dA_s = dt_s + H;              // [H]
  __shared__ float red[33];
  const int64_t bi = blockIdx.x;

  // conv-state shift + conv + SiLU
  for (int64_t c = threadIdx.x; c < pr.conv_dim; c += blockDim.x) {
    T *cs = conv_state + (bi * pr.conv_dim + c) * 4;
    const T n0 = cs[1], n1 = cs[2], n2 = cs[3], n3 = xBC[bi * ld_x + c];
    cs[0] = n0;
    cs[1] = n1;
    cs[2] = n2;
    cs[3] = n3;
    const float *w = prm.conv_w + c * 4;
    const float pre = prm.conv_b[c] + w[0] * to_f(n0) + w[1] * to_f(n1) + w[2] * to_f(n2) +
                      w[3] * to_f(n3);
    u_s[c] = silu_f(pre);
  }
  for (int h = threadIdx.x; h < H; h += blockDim.x) {
    const float dt = softplus_f(to_f(dt_raw[bi * ld_dt + h]) + prm.dt_bias[h]);
    dt_s[h] = dt;
    dA_s[h] = expf(dt * prm.A[h]);
  }
  __syncthreads();

  // state update + C contraction, head by head.  nq = N/4 consecutive threads
  // share a row p of the state (nq divides 32), reduced with xor shuffles.
  const int nq = N / 4;
  const int hpg = pr.heads_per_group();
  for (int h = 0; h < H; ++h) {
    const int g = h / hpg;
    const float *xh = u_s + (int64_t)h * P;
    const float *Bv = u_s + pr.d_inner + (int64_t)g * N;
    const float *Cv = u_s + pr.d_inner + (int64_t)pr.G * N + (int64_t)g * N;
    const float dt = dt_s[h], dA = dA_s[h], Dh = prm.D[h];
    float4 *st = reinterpret_cast<float4 *>(ssm + (bi * H + h) * (int64_t)(P * N));
    for (int idx = threadIdx.x; idx < P * nq; idx += blockDim.x) {
      const int p = idx / nq, q = idx % nq;
      const float xdt = xh[p] * dt;
      float4 s = st[idx];
      s.x = dA * s.x + xdt * Bv[4 * q + 0];
      s.y = dA * s.y + xdt * Bv[4 * q + 1];
      s.z = dA * s.z + xdt * Bv[4 * q + 2];
      s.w = dA * s.w + xdt * Bv[4 * q + 3];
      st[idx] = s;
      float part = s.x * Cv[4 * q + 0] + s.y * Cv[4 * q + 1] + s.z * Cv[4 * q + 2] +
                   s.w * Cv[4 * q + 3];
      for (int o = nq / 2; o > 0; o >>= 1) part += __shfl_xor_sync(0xffffffffu, part, o);
      if (q == 0) y_s[(int64_t)h * P + p] = part + Dh * xh[p];
    }
  }
  __syncthreads();

  // gated group RMSNorm over the row
  const T *zr = z + bi * ld_z;
  T *outr = y + bi * pr.d_inner;
  const int64_t gs = pr.d_inner / pr.G;
  for (int k = 0; k < pr.G; ++k) {
    float ss = 0.0f;
    for (int64_t i = threadIdx.x; i < gs; i += blockDim.x) {
      const int64_t c = k * gs + i;
      const float v = pr.nbg ? y_s[c] : y_s[c] * silu_f(to_f(zr[c]));
      ss += v * v;
    }
    ss = block_sum(ss, red);
    const float inv = rsqrtf(ss / (float)gs + pr.eps);
    for (int64_t i = threadIdx.x; i < gs; i += blockDim.x) {
      const int64_t c = k * gs + i;
      const float sz = silu_f(to_f(zr[c]));
      const float o = pr.nbg ? y_s[c] * inv * prm.norm_w[c] * sz : y_s[c] * sz * inv * prm.norm_w[c];
      outr[c] = from_f<T>(o);
    }
  }
}

template <typename T>
cudaError_t run(const StepArgs &a) {
  const Problem &pr = a.pr;
  const size_t smem = sizeof(float) * (size_t)(pr.conv_dim + pr.d_inner + 2 * pr.H);
  cudaError_t e = cudaFuncSetAttribute(ssd_step_kernel<T>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  stage_mark(a.stream, 0);
  ssd_step_kernel<T><<<(unsigned)pr.batch, 256, smem, a.stream>>>(
      pr, a.prm, static_cast<const T *>(a.xBC), a.ld_xbc, static_cast<const T *>(a.z), a.ld_z,
      static_cast<const T *>(a.dt_raw), a.ld_dt, static_cast<T *>(a.y),
      static_cast<T *>(a.conv_state), a.ssm_state);
  stage_mark(a.stream, 1);
  return cudaGetLastError();
}

}  // namespace

const char *const kStepSimtStages[] = {"ssd_step"};
const int kStepSimtStageCount = 1;

cudaError_t step_simt(const StepArgs &a) {
  return a.pr.io == MAMBA2_BF16 ? run<__nv_bfloat16>(a) : run<float>(a);
}

}  // namespace m2
