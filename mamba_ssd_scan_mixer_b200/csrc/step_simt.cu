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
constexpr int kMaxStages = 4;  // shared-memory ring of per-head state buffers

static __device__ unsigned int g_step_errors = 0;

// silu with the fast exponential and reciprocal (relative error ~1e-6)
__device__ __forceinline__ float silu_fast(float v) { return __fdividef(v, 1.0f + __expf(-v)); }

template <typename T>
__device__ __forceinline__ float conv4(const float *w, float b, T a0, T a1, T a2, T a3) {
  return b + w[0] * to_f(a0) + w[1] * to_f(a1) + w[2] * to_f(a2) + w[3] * to_f(a3);
}

template <typename T, int N>
__global__ void __launch_bounds__(kStepThreads)
    ssd_step_kernel(Problem pr, mamba2_params prm, const T *__restrict__ xBC, int64_t ld_x,
                    const T *__restrict__ z, int64_t ld_z, const T *__restrict__ dt_raw,
                    int64_t ld_dt, T *__restrict__ y, T *__restrict__ conv_state,
                    float *__restrict__ ssm, int hpc, int stages, int nclusters) {
  cg::cluster_group cluster = cg::this_cluster();
  const int cs = (int)cluster.num_blocks();
  const int rank = (int)cluster.block_rank();
  const int cid = blockIdx.y;  // this cluster's index; it handles rows cid, cid + nclusters, ...
  constexpr int NQ = N / 4;               // float4s per state row (compile time)
  constexpr int kRowsPerPass = kStepThreads / NQ;
  const int H = pr.H, P = pr.P, G = pr.G;
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

  // Work items k = (row iteration, head): row cid + (k / hpc) * nclusters, head h0 + k % hpc.
  // The ring runs across rows, so the next row's state is already arriving while
  // this row finishes its norm exchange and the next row its conv.
  const int64_t rows_mine = pr.batch > cid ? (pr.batch - cid + nclusters - 1) / nclusters : 0;
  const int64_t n_items = rows_mine * hpc;
  auto item_src = [&](int64_t k) -> float * {
    const int64_t r = cid + (k / hpc) * nclusters;
    return ssm + (r * H + h0 + (int)(k % hpc)) * (int64_t)head_floats;
  };
  if (threadIdx.x == 0) {
    for (int s = 0; s < stages; ++s) mbar_init(&full[s], 1);
    fence_mbar_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    for (int s = 0; s < stages && s < n_items; ++s) {
      mbar_arrive_expect_tx(&full[s], head_bytes);
      bulk_g2s(sbuf + s * head_floats, item_src(s), head_bytes, &full[s]);
    }
  }

  // this thread's column of float4s (q) and first row (p0); rows p0 + kRowsPerPass * i
  const int q = threadIdx.x % NQ, p0 = threadIdx.x / NQ;
  const int passes = P / kRowsPerPass > 0 ? P / kRowsPerPass : 1;
  const bool active = p0 < P;  // P * NQ may be smaller than the block
  bool ok = true;
  int64_t k = 0;  // next item to consume
  for (int64_t rr = 0; rr < rows_mine; ++rr) {
    const int64_t bi = cid + rr * nclusters;
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
      ux[i] = silu_fast(conv4(prm.conv_w + c * 4, prm.conv_b[c], a0, a1, a2, a3));
    }
    for (int j = threadIdx.x; j < 2 * GN; j += blockDim.x) {
      const int64_t c = pr.d_inner + j;
      const T *w4 = csr + c * 4;
      ubc[j] = silu_fast(conv4(prm.conv_w + c * 4, prm.conv_b[c], w4[1], w4[2], w4[3], xr[c]));
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
    float *st_row = ssm + (bi * H + h0) * (int64_t)head_floats;
    for (int j = 0; j < hpc; ++j, ++k) {
      const int s = (int)(k % stages);
      const bool got =
          ok && mbar_wait_bounded(&full[s], (uint32_t)((k / stages) & 1), &g_step_errors);
      ok = __syncthreads_and(got) != 0;
      if (ok && active) {
        const int g = (h0 + j) / hpg;
        const float *xh = ux + j * P;
        const float4 b = reinterpret_cast<const float4 *>(ubc + g * N)[q];
        const float4 cc = reinterpret_cast<const float4 *>(ubc + GN + g * N)[q];
        const float dt = dts[j], dA = dAs[j], Dh = prm.D[h0 + j];
        const float4 *src = reinterpret_cast<const float4 *>(sbuf + s * head_floats);
        float4 *dst = reinterpret_cast<float4 *>(st_row + (int64_t)j * head_floats);
        for (int i = 0; i < passes; ++i) {
          const int p = p0 + i * kRowsPerPass, idx = p * NQ + q;
          const float xv = xh[p], xdt = xv * dt;
          float4 v = src[idx];
          v.x = fmaf(dA, v.x, xdt * b.x);
          v.y = fmaf(dA, v.y, xdt * b.y);
          v.z = fmaf(dA, v.z, xdt * b.z);
          v.w = fmaf(dA, v.w, xdt * b.w);
          dst[idx] = v;
          float pt = fmaf(v.x, cc.x, fmaf(v.y, cc.y, fmaf(v.z, cc.z, v.w * cc.w)));
#pragma unroll
          for (int o = NQ / 2; o > 0; o >>= 1) pt += __shfl_xor_sync(0xffffffffu, pt, o);
          if (q == 0) ys[j * P + p] = fmaf(Dh, xv, pt);
        }
      }
      __syncthreads();  // every thread is done with buffer s
      if (threadIdx.x == 0 && ok && k + stages < n_items) {
        fence_proxy_async_smem();
        mbar_arrive_expect_tx(&full[s], head_bytes);
        bulk_g2s(sbuf + s * head_floats, item_src(k + stages), head_bytes, &full[s]);
      }
    }

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
        const float v = pr.nbg ? ys[c] : ys[c] * silu_fast(to_f(zr[c]));
        if (!pr.nbg) ys[c] = v;  // keep the gated value for the scaling below
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
      const float o = pr.nbg ? ys[c] * sc * nw[c] * silu_fast(to_f(zr[c])) : ys[c] * sc * nw[c];
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
    cluster.sync();  // rank 0's table and this row's smem stay valid until all are done
  }
  if (!ok && threadIdx.x == 0) {
    // a wait ran out: let the copies still in flight land before the CTA exits
    for (int64_t kk = k; kk < n_items && kk < k + stages; ++kk)
      mbar_wait_bounded(&full[kk % stages], (uint32_t)((kk / stages) & 1), &g_step_errors);
  }
}

int cluster_size_for(int H) {
  for (int cs : {8, 4, 2})
    if (H % cs == 0) return cs;
  return 1;
}

template <typename T, int N>
cudaError_t run(const StepArgs &a) {
  const Problem &pr = a.pr;
  const int cs = cluster_size_for(pr.H), hpc = pr.H / cs;
  const size_t head_bytes = sizeof(float) * (size_t)pr.P * pr.N;
  const int stages = (int)std::max<size_t>(2, std::min<size_t>(kMaxStages, 65536 / head_bytes));
  const size_t smem = stages * head_bytes + sizeof(uint64_t) * kMaxStages +
                      sizeof(float) * (size_t)(2 * pr.G * pr.N + 2 * hpc * pr.P + 2 * hpc +
                                               cs * pr.G + pr.G);
  cudaError_t e = cudaFuncSetAttribute(ssd_step_kernel<T, N>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  if (cs > 8) {
    e = cudaFuncSetAttribute(ssd_step_kernel<T, N>, cudaFuncAttributeNonPortableClusterSizeAllowed,
                             1);
    if (e != cudaSuccess) return e;
  }
  cudaLaunchConfig_t cfg = {};
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
  // as many clusters as fit on the device at once, each looping over rows
  cfg.gridDim = dim3((unsigned)cs, 1, 1);
  int max_clusters = 0;
  if (cudaOccupancyMaxActiveClusters(&max_clusters, ssd_step_kernel<T, N>, &cfg) != cudaSuccess ||
      max_clusters <= 0) {
    cudaGetLastError();  // clear a failed query; fall back to one cluster per row
    max_clusters = (int)std::min<int64_t>(pr.batch, 65535);
  }
  // the fewest clusters that keep the largest per-cluster row count: no cluster idles
  // at the end while others still have a row left
  const int64_t fit = std::max<int64_t>(1, std::min<int64_t>(pr.batch, max_clusters));
  const int64_t rows_per = (pr.batch + fit - 1) / fit;
  const int nclusters = (int)std::max<int64_t>(1, (pr.batch + rows_per - 1) / rows_per);
  cfg.gridDim = dim3((unsigned)cs, (unsigned)nclusters, 1);
  stage_mark(a.stream, 0);
  e = cudaLaunchKernelEx(&cfg, ssd_step_kernel<T, N>, pr, a.prm, static_cast<const T *>(a.xBC),
                         a.ld_xbc, static_cast<const T *>(a.z), a.ld_z,
                         static_cast<const T *>(a.dt_raw), a.ld_dt, static_cast<T *>(a.y),
                         static_cast<T *>(a.conv_state), a.ssm_state, hpc, stages, nclusters);
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

template <typename T>
cudaError_t run_n(const StepArgs &a) {
  switch (a.pr.N) {
    case 16: return run<T, 16>(a);
    case 32: return run<T, 32>(a);
    case 64: return run<T, 64>(a);
    default: return run<T, 128>(a);
  }
}

cudaError_t step_simt(const StepArgs &a) {
  return a.pr.io == MAMBA2_BF16 ? run_n<__nv_bfloat16>(a) : run_n<float>(a);
}

}  // namespace m2
