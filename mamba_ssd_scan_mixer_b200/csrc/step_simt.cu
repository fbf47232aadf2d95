// Single-token decode step of the Mamba-2 mixer core ("Zamba2 hybrid
// architecture in Transformers", qwbw.cn, section 三 step 3: with the states
// cached and one new token, the scan becomes one recurrent state update).
//
// The step is bound by streaming the fp32 SSM state (read + write, 32 KB per
// head at P = N = 64).  Each batch row is handled by a thread-block cluster of
// `cs` CTAs that split the row's heads; a CTA:
//   0. starts bulk asynchronous copies (cp.async.bulk, completing on mbarriers)
//      of its first heads' state into a ring of shared-memory buffers;
//   1. meanwhile shifts the conv state of its own x channels and computes conv
//      + SiLU for them and for all B/C channels (cheap, recomputed by every CTA);
//   2. per head: waits for its buffer (bounded wait), updates the state in
//      registers and stores it to global memory, contracts it with C
//      (xor-shuffle reduction over the N/4 lanes that share a row p), and
//      refills the buffer with a later head;
//   3. gates with silu(z), sums squares per norm group, exchanges the partial
//      sums through distributed shared memory (rank 0 holds the table) and
//      scales its own channels.
// The B/C conv state is shared by the cluster, so it is written (channel j by
// rank j % cs) only after the cluster barrier that follows every CTA's reads.
#include <cooperative_groups.h>

#include <algorithm>

#include "common.cuh"

namespace cg = cooperative_groups;

namespace m2 {
namespace {

constexpr int kStepThreads = 256;
constexpr int kMaxQuads = 8;   // float4s of one head's state per thread: P*N/4/256, P<=64, N<=128
constexpr int kMaxStages = 4;  // shared-memory ring of per-head state buffers

static __device__ unsigned int g_step_errors = 0;

template <typename T>
__device__ __forceinline__ float conv4(const float *w, float b, T a0, T a1, T a2, T a3) {
  return b + w[0] * to_f(a0) + w[1] * to_f(a1) + w[2] * to_f(a2) + w[3] * to_f(a3);
}

template <typename T>
__global__ void __launch_bounds__(kStepThreads)
    ssd_step_kernel(Problem pr, mamba2_params prm, const T *__restrict__ xBC, int64_t ld_x,
                    const T *__restrict__ z, int64_t ld_z, const T *__restrict__ dt_raw,
                    int64_t ld_dt, T *__restrict__ y, T *__restrict__ conv_state,
                    float *__restrict__ ssm, int hpc, int stages) {
  cg::cluster_group cluster = cg::this_cluster();
  const int cs = (int)cluster.num_blocks();
  const int rank = (int)cluster.block_rank();
  const int64_t bi = blockIdx.y;
  const int H = pr.H, P = pr.P, N = pr.N, G = pr.G;
  const int hpg = pr.heads_per_group();
  const int h0 = rank * hpc;
  const int GN = G * N;
  const int head_floats = P * N;
  const uint32_t head_bytes = (uint32_t)head_floats * 4u;
  extern __shared__ __align__(128) unsigned char smem_raw[];
  float *sbuf = reinterpret_cast<float *>(smem_raw);                 // [stages][P*N]
  uint64_t *full = reinterpret_cast<uint64_t *>(sbuf + stages * head_floats);  // [kMaxStages]
  float *ubc = reinterpret_cast<float *>(full + kMaxStages);         // [2*G*N] B | C
  float *ux = ubc + 2 * GN;          // [hpc*P]
  float *ys = ux + hpc * P;          // [hpc*P]
  float *dts = ys + hpc * P;         // [hpc]
  float *dAs = dts + hpc;            // [hpc]
  float *part = dAs + hpc;           // [cs*G] partial sums of squares (rank 0's is used)
  float *inv = part + cs * G;        // [G]
  __shared__ float red[33];

  // 0. start streaming this CTA's heads of the state (contiguous in memory)
  float *st_row = ssm + (bi * H + h0) * (int64_t)head_floats;
  if (threadIdx.x == 0) {
    for (int k = 0; k < stages; ++k) mbar_init(&full[k], 1);
    fence_mbar_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    for (int k = 0; k < stages && k < hpc; ++k) {
      mbar_arrive_expect_tx(&full[k], head_bytes);
      bulk_g2s(sbuf + k * head_floats, st_row + (int64_t)k * head_floats, head_bytes, &full[k]);
    }
  }

  // 1. conv: own x channels (state written now), all B/C channels (read only)
  const T *xr = xBC + bi * ld_x;
  T *csr = conv_state + bi * pr.conv_dim * 4;
  for (int i = threadIdx.x; i < hpc * P; i += blockDim.x) {
    const int64_t c = (int64_t)h0 * P + i;
    T *w4 = csr + c * 4;
    const T a0 = w4[1], a1 = w4[2], a2 = w4[3], a3 = xr[c];
    w4[0] = a0;
    w4[1] = a1;
    w4[2] = a2;
    w4[3] = a3;
    ux[i] = silu_f(conv4(prm.conv_w + c * 4, prm.conv_b[c], a0, a1, a2, a3));
  }
  for (int j = threadIdx.x; j < 2 * GN; j += blockDim.x) {
    const int64_t c = pr.d_inner + j;
    const T *w4 = csr + c * 4;
    ubc[j] = silu_f(conv4(prm.conv_w + c * 4, prm.conv_b[c], w4[1], w4[2], w4[3], xr[c]));
  }
  for (int i = threadIdx.x; i < hpc; i += blockDim.x) {
    const int h = h0 + i;
    const float dt = softplus_f(to_f(dt_raw[bi * ld_dt + h]) + prm.dt_bias[h]);
    dts[i] = dt;
    dAs[i] = expf(dt * prm.A[h]);
  }
  __syncthreads();

  // 2. per head: wait for its buffer, update in registers, store to global,
  //    contract with C (xor-shuffle over the N/4 lanes sharing a row p), refill
  const int nq = N / 4, total = P * nq;
  bool ok = true;
  int j = 0;
  for (; j < hpc; ++j) {
    const int k = j % stages;
    const bool got = mbar_wait_bounded(&full[k], (uint32_t)((j / stages) & 1), &g_step_errors);
    ok = __syncthreads_and(got) != 0;
    if (!ok) break;
    const int g = (h0 + j) / hpg;
    const float *xh = ux + j * P;
    const float4 *B4 = reinterpret_cast<const float4 *>(ubc + g * N);
    const float4 *C4 = reinterpret_cast<const float4 *>(ubc + GN + g * N);
    const float dt = dts[j], dA = dAs[j], Dh = prm.D[h0 + j];
    const float4 *src = reinterpret_cast<const float4 *>(sbuf + k * head_floats);
    float4 *dst = reinterpret_cast<float4 *>(st_row + (int64_t)j * head_floats);
#pragma unroll
    for (int kq = 0; kq < kMaxQuads; ++kq) {
      const int idx = threadIdx.x + kq * kStepThreads;
      if (idx < total) {  // warp-uniform: total is a multiple of 64
        const int p = idx / nq, q = idx % nq;
        const float xdt = xh[p] * dt;
        const float4 b = B4[q], cc = C4[q];
        float4 v = src[idx];
        v.x = dA * v.x + xdt * b.x;
        v.y = dA * v.y + xdt * b.y;
        v.z = dA * v.z + xdt * b.z;
        v.w = dA * v.w + xdt * b.w;
        dst[idx] = v;
        float pt = v.x * cc.x + v.y * cc.y + v.z * cc.z + v.w * cc.w;
        for (int o = nq / 2; o > 0; o >>= 1) pt += __shfl_xor_sync(0xffffffffu, pt, o);
        if (q == 0) ys[j * P + p] = pt + Dh * xh[p];
      }
    }
    __syncthreads();  // every thread is done with buffer k
    if (threadIdx.x == 0 && j + stages < hpc) {
      fence_proxy_async_smem();
      mbar_arrive_expect_tx(&full[k], head_bytes);
      bulk_g2s(sbuf + k * head_floats, st_row + (int64_t)(j + stages) * head_floats, head_bytes,
               &full[k]);
    }
  }
  if (!ok && threadIdx.x == 0) {
    // a wait ran out: let the copies still in flight land before the CTA exits
    for (int jj = j; jj < hpc && jj < j + stages; ++jj)
      mbar_wait_bounded(&full[jj % stages], (uint32_t)((jj / stages) & 1), &g_step_errors);
  }
  __syncthreads();

  // 3. gate, partial sums of squares per norm group (= head group), exchange
  const T *zr = z + bi * ld_z + (int64_t)h0 * P;
  const int g_lo = h0 / hpg, g_hi = (h0 + hpc - 1) / hpg;
  float *part0 = cluster.map_shared_rank(part, 0);
  for (int g = threadIdx.x; g < G; g += blockDim.x)
    if (g < g_lo || g > g_hi) part0[rank * G + g] = 0.0f;
  for (int g = g_lo; g <= g_hi; ++g) {
    const int c0 = max(g * hpg, h0) * P - h0 * P, c1 = min((g + 1) * hpg, h0 + hpc) * P - h0 * P;
    float ss = 0.0f;
    for (int c = c0 + threadIdx.x; c < c1; c += blockDim.x) {
      const float v = pr.nbg ? ys[c] : ys[c] * silu_f(to_f(zr[c]));
      ss += v * v;
    }
    ss = block_sum(ss, red);
    if (threadIdx.x == 0) part0[rank * G + g] = ss;
  }
  cluster.sync();
  const float gs = (float)(hpg * P);
  for (int g = g_lo + (int)threadIdx.x; g <= g_hi; g += blockDim.x) {
    float tot = 0.0f;
    for (int r = 0; r < cs; ++r) tot += part0[r * G + g];
    inv[g] = rsqrtf(tot / gs + pr.eps);
  }
  __syncthreads();
  T *yr = y + bi * pr.d_inner + (int64_t)h0 * P;
  const float *nw = prm.norm_w + (int64_t)h0 * P;
  for (int c = threadIdx.x; c < hpc * P; c += blockDim.x) {
    const float sc = inv[(h0 + c / P) / hpg];
    const float sz = silu_f(to_f(zr[c]));
    const float o = pr.nbg ? ys[c] * sc * nw[c] * sz : ys[c] * sz * sc * nw[c];
    yr[c] = from_f<T>(o);
  }
  // 4. shared B/C conv state, now that every CTA of the cluster has read it
  for (int jb = rank + cs * (int)threadIdx.x; jb < 2 * GN; jb += cs * blockDim.x) {
    const int64_t c = pr.d_inner + jb;
    T *w4 = csr + c * 4;
    const T a0 = w4[1], a1 = w4[2], a2 = w4[3], a3 = xr[c];
    w4[0] = a0;
    w4[1] = a1;
    w4[2] = a2;
    w4[3] = a3;
  }
  cluster.sync();  // rank 0's partial-sum table stays alive until all have read it
}

int cluster_size_for(int H) {
  for (int cs : {8, 4, 2})
    if (H % cs == 0) return cs;
  return 1;
}

template <typename T>
cudaError_t run(const StepArgs &a) {
  const Problem &pr = a.pr;
  const int cs = cluster_size_for(pr.H), hpc = pr.H / cs;
  const size_t head_bytes = sizeof(float) * (size_t)pr.P * pr.N;
  const int stages = (int)std::max<size_t>(2, std::min<size_t>(kMaxStages, 65536 / head_bytes));
  const size_t smem = stages * head_bytes + sizeof(uint64_t) * kMaxStages +
                      sizeof(float) * (size_t)(2 * pr.G * pr.N + 2 * hpc * pr.P + 2 * hpc +
                                               cs * pr.G + pr.G);
  cudaError_t e = cudaFuncSetAttribute(ssd_step_kernel<T>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)cs, (unsigned)pr.batch, 1);
  cfg.blockDim = dim3(kStepThreads, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = a.stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = (unsigned)cs;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  stage_mark(a.stream, 0);
  e = cudaLaunchKernelEx(&cfg, ssd_step_kernel<T>, pr, a.prm, static_cast<const T *>(a.xBC),
                         a.ld_xbc, static_cast<const T *>(a.z), a.ld_z,
                         static_cast<const T *>(a.dt_raw), a.ld_dt, static_cast<T *>(a.y),
                         static_cast<T *>(a.conv_state), a.ssm_state, hpc, stages);
  stage_mark(a.stream, 1);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace

const char *const kStepSimtStages[] = {"ssd_step"};
const int kStepSimtStageCount = 1;

cudaError_t take_step_errors(unsigned int *out) {
  unsigned int v = 0, zero = 0;
  cudaError_t e = cudaMemcpyFromSymbol(&v, g_step_errors, sizeof(v));
  if (e == cudaSuccess) e = cudaMemcpyToSymbol(g_step_errors, &zero, sizeof(zero));
  *out = v;
  return e;
}

cudaError_t step_simt(const StepArgs &a) {
  return a.pr.io == MAMBA2_BF16 ? run<__nv_bfloat16>(a) : run<float>(a);
}

}  // namespace m2
