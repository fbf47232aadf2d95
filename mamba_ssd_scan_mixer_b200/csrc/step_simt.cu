// Single-token decode step of the Mamba-2 mixer core ("Zamba2 hybrid
// architecture in Transformers", qwbw.cn, section 三 step 3: with the states
// cached and one new token, the scan becomes one recurrent state update).
//
// The step is bound by streaming the fp32 SSM state (read + write, 32 KB per
// head at P = N = 64).  Each batch row is handled by a thread-block cluster of
// `cs` CTAs that split the row's heads; persistent clusters loop over rows.
// A CTA has 8 compute warps and one producer warp:
//   producer: bulk asynchronous copies (cp.async.bulk, completing on mbarriers)
//     of its heads' state, row after row, into a ring of shared-memory
//     buffers; a buffer is refilled as soon as the compute warps release it;
//   compute, per row r:
//   1. conv + SiLU of the CTA's own x channels and of all B/C channels, from
//      the row's conv state, new xBC column and z, which were copied into
//      shared memory (cp.async) while row r - 1 streamed; the shifted conv
//      state of the own channels goes back to global memory; dt;
//   2. start the copies of row r + 1's inputs; per head: wait for its buffer
//      (bounded wait), update the state in registers, store it to global
//      memory, contract it with C (xor-shuffle reduction over the N/4 lanes
//      that share a row p), release the buffer;
//   3. gate with silu(z) and sum squares per norm group;
//   4. finish row r - 1: wait until every rank of the cluster has signalled
//      it, scale and store its output, write this rank's share of its shifted
//      B/C conv state (all ranks have read it by then);
//   5. send row r's partial sums into every rank's table (distributed shared
//      memory, asynchronous stores that complete bytes on that rank's mbarrier).
// So the norm exchange of a row completes while the next row streams.  The
// tables, mbarriers and per-row buffers alternate between rows; step 4 comes
// before step 5 so that no rank can overwrite a table this CTA still reads.
#include <algorithm>

#include <mutex>

#include "common.cuh"

namespace m2 {
namespace {

constexpr int kStepThreads = 256;                 // compute threads
constexpr int kStepBlock = kStepThreads + 32;     // + the producer warp
constexpr int kMaxStages = 4;  // shared-memory ring of per-head state buffers (at most)
constexpr uint32_t kStepSmemPerCta = 112 * 1024;  // two CTAs per SM

static __device__ unsigned int g_step_errors = 0;
static __device__ unsigned int g_step_stall = 0;  // mamba2_debug_stall_waits

// silu with the fast exponential and reciprocal (relative error ~1e-6)
__device__ __forceinline__ float silu_fast(float v) { return __fdividef(v, 1.0f + __expf(-v)); }

template <typename T>
__device__ __forceinline__ float conv4(const float *w, float b, T a0, T a1, T a2, T a3) {
  return b + w[0] * to_f(a0) + w[1] * to_f(a1) + w[2] * to_f(a2) + w[3] * to_f(a3);
}

// Bulk (non-tensor) shared -> global copy in this thread's bulk async-group, and
// the waits for this thread's groups: until at most n are still reading their
// shared-memory source, or until at most n are still in flight at all.
__device__ __forceinline__ void bulk_s2g(void *dst, const void *src, uint32_t bytes) {
  asm volatile("cp.async.bulk.global.shared::cta.bulk_group [%0], [%1], %2;" ::"l"(dst),
               "r"(smem_u32(src)), "r"(bytes)
               : "memory");
  asm volatile("cp.async.bulk.commit_group;" ::: "memory");
}
__device__ __forceinline__ void bulk_wait_read_all() {
  asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
}
__device__ __forceinline__ void bulk_wait_all() {
  asm volatile("cp.async.bulk.wait_group 0;" ::: "memory");
}

// barrier of the compute warps only (the producer warp never joins it)
__device__ __forceinline__ void step_bar() { asm volatile("bar.sync 1, 256;" ::: "memory"); }

__device__ __forceinline__ float step_block_sum(float v, float *red) {
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
  v = warp_sum(v);
  step_bar();  // red may still be read by a previous call
  if (lane == 0) red[wid] = v;
  step_bar();
  float t = (lane < kStepThreads / 32) ? red[lane] : 0.0f;
  return warp_sum(t);
}

// shared::cluster address of `p` (this CTA's shared memory) in rank `r`
__device__ __forceinline__ uint32_t cluster_addr(const void *p, int r) {
  uint32_t a;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(a) : "r"(smem_u32(p)), "r"(r));
  return a;
}
// asynchronous 4-byte store into another rank's shared memory that completes
// 4 transaction bytes on that rank's mbarrier
__device__ __forceinline__ void st_async_cluster(uint32_t addr, float v, uint32_t bar) {
  asm volatile("st.async.shared::cluster.mbarrier::complete_tx::bytes.b32 [%0], %1, [%2];" ::"r"(addr),
               "r"(__float_as_uint(v)), "r"(bar)
               : "memory");
}
__device__ __forceinline__ bool mbar_try_wait_cluster(uint64_t *bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n .reg .pred p;\n mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2;\n"
      " selp.u32 %0, 1, 0, p;\n}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}
__device__ __forceinline__ bool mbar_wait_cluster_bounded(uint64_t *bar, uint32_t parity) {
  if (mbar_try_wait_cluster(bar, parity)) return true;
  const unsigned long long t0 = globaltimer_ns();
  while (!mbar_try_wait_cluster(bar, parity)) {
    if (globaltimer_ns() - t0 > kWaitLimitNs) {
      atomicOr(&g_step_errors, kErrWaitTimeout);
      return false;
    }
  }
  return true;
}
__device__ __forceinline__ void cluster_arrive_wait() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n barrier.cluster.wait.acquire.aligned;" :::
                   "memory");
}

__device__ __forceinline__ void cp_async16(void *dst_smem, const void *src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_u32(dst_smem)), "l"(src)
               : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_all;" ::: "memory"); }

// four consecutive conv-state elements (8 or 16 bytes, aligned)
__device__ __forceinline__ void store4(__nv_bfloat16 *p, __nv_bfloat16 a0, __nv_bfloat16 a1,
                                       __nv_bfloat16 a2, __nv_bfloat16 a3) {
  uint2 v;
  v.x = (uint32_t)__bfloat16_as_ushort(a0) | ((uint32_t)__bfloat16_as_ushort(a1) << 16);
  v.y = (uint32_t)__bfloat16_as_ushort(a2) | ((uint32_t)__bfloat16_as_ushort(a3) << 16);
  *reinterpret_cast<uint2 *>(p) = v;
}
__device__ __forceinline__ void store4(float *p, float a0, float a1, float a2, float a3) {
  *reinterpret_cast<float4 *>(p) = make_float4(a0, a1, a2, a3);
}

// Shared-memory layout of a CTA (byte offsets; every 16-byte-accessed array is
// 16-byte aligned).  C = own x channels (hpc * P), BC = B and C channels.
struct StepLayout {
  uint32_t bar, pre, pre_elems, cw, cb, nw, ubc, ux, ys, zk, bcn, dts, dAs, dtr, dtb, Ah, Dh, part,
      mysum, inv, total;
};
template <typename T>
__host__ __device__ inline StepLayout step_layout(int stages, int hpc, int P, int G, int N, int cs) {
  const uint32_t C = (uint32_t)(hpc * P), BC = (uint32_t)(2 * G * N), t = (uint32_t)sizeof(T);
  StepLayout L;
  uint32_t o = (uint32_t)(stages * P * N * 4);  // ring of per-head state buffers
  L.bar = o;  o += 8 * (2 * kMaxStages + 2);     // full, empty, sums_ready[2]
  // per-row inputs, two buffers: conv state of own channels [C][4] | of B/C [BC][4] |
  // new x [C] | new B/C [BC] | z [C]
  L.pre_elems = 4 * C + 4 * BC + C + BC + C;
  L.pre = o;  o += 2 * t * L.pre_elems;
  L.cw = o;   o += 16 * (C + BC);  // conv taps (float4) of own then B/C channels
  L.cb = o;   o += 4 * (C + BC);
  L.nw = o;   o += 4 * C;
  L.ubc = o;  o += 4 * BC;         // post-conv B | C
  L.ux = o;   o += 4 * C;          // post-conv x
  L.ys = o;   o += 4 * 2 * C;      // per row parity: y, then the gated y
  L.zk = o;   o += t * 2 * C;      // per row parity: z kept for the norm-before-gate order
  L.bcn = o;  o += t * 2 * 4 * BC; // per row parity: shifted B/C conv state
  L.dts = o;  o += 4 * hpc;
  L.dAs = o;  o += 4 * hpc;
  L.dtr = o;  o += 4 * 2 * hpc;    // per row parity: raw dt
  L.dtb = o;  o += 4 * hpc;
  L.Ah = o;   o += 4 * hpc;
  L.Dh = o;   o += 4 * hpc;
  L.part = o; o += 4 * 2 * cs * G; // per row parity: partial sums of every rank
  L.mysum = o; o += 4 * G;
  L.inv = o;  o += 4 * G;
  L.total = o;
  return L;
}

// Byte ranges of the decode step's buffers (checked build, see M2_OK).
struct StepSpans {
  Span xbc, z, dt, y, conv, ssm, conv_w, conv_b, norm_w, dt_bias, A, D;
};

template <typename T, int N>
__global__ void __launch_bounds__(kStepBlock, 2)
    ssd_step_kernel(Problem pr, mamba2_params prm, const T *__restrict__ xBC, int64_t ld_x,
                    const T *__restrict__ z, int64_t ld_z, const T *__restrict__ dt_raw,
                    int64_t ld_dt, T *__restrict__ y, T *__restrict__ conv_state,
                    float *__restrict__ ssm, int hpc, int stages, int nclusters,
                    const StepSpans sp) {
  if (test_stall(&g_step_stall, &g_step_errors)) return;  // every CTA alike (test aid)
  int cs, rank;
  asm volatile("mov.u32 %0, %%cluster_nctarank;" : "=r"(cs));
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(rank));
  const int cid = blockIdx.y;  // this cluster's index; it handles rows cid, cid + nclusters, ...
  constexpr int NQ = N / 4;               // float4s per state row (compile time)
  constexpr int kRowsPerPass = kStepThreads / NQ;
  const int H = pr.H, P = pr.P, G = pr.G;
  const int hpg = pr.heads_per_group();
  const int h0 = rank * hpc;
  const int GN = G * N, C = hpc * P, BC = 2 * GN;
  const int head_floats = P * N;
  const uint32_t head_bytes = (uint32_t)head_floats * 4u;
  extern __shared__ __align__(128) unsigned char smem_raw[];
  const StepLayout Lo = step_layout<T>(stages, hpc, P, G, N, cs);
  float *sbuf = reinterpret_cast<float *>(smem_raw);  // [stages][P*N]
  uint64_t *full = reinterpret_cast<uint64_t *>(smem_raw + Lo.bar);
  uint64_t *empty = full + kMaxStages;
  uint64_t *sums_ready = empty + kMaxStages;  // [2] (row parity)
  T *pre0 = reinterpret_cast<T *>(smem_raw + Lo.pre);
  const float4 *cw = reinterpret_cast<const float4 *>(smem_raw + Lo.cw);
  const float *cb = reinterpret_cast<const float *>(smem_raw + Lo.cb);
  const float *nw = reinterpret_cast<const float *>(smem_raw + Lo.nw);
  float *ubc = reinterpret_cast<float *>(smem_raw + Lo.ubc);
  float *ux = reinterpret_cast<float *>(smem_raw + Lo.ux);
  float *ys = reinterpret_cast<float *>(smem_raw + Lo.ys);
  T *zk = reinterpret_cast<T *>(smem_raw + Lo.zk);
  T *bcn = reinterpret_cast<T *>(smem_raw + Lo.bcn);
  float *dts = reinterpret_cast<float *>(smem_raw + Lo.dts);
  float *dAs = reinterpret_cast<float *>(smem_raw + Lo.dAs);
  float *dtr = reinterpret_cast<float *>(smem_raw + Lo.dtr);
  const float *dtb = reinterpret_cast<const float *>(smem_raw + Lo.dtb);
  const float *Ah = reinterpret_cast<const float *>(smem_raw + Lo.Ah);
  const float *Dh = reinterpret_cast<const float *>(smem_raw + Lo.Dh);
  float *part = reinterpret_cast<float *>(smem_raw + Lo.part);
  float *mysum = reinterpret_cast<float *>(smem_raw + Lo.mysum);
  float *inv = reinterpret_cast<float *>(smem_raw + Lo.inv);
  __shared__ float red[33];

  // Work items k = (row iteration, head): row cid + (k / hpc) * nclusters, head h0 + k % hpc.
  const int64_t rows_mine = pr.batch > cid ? (pr.batch - cid + nclusters - 1) / nclusters : 0;
  const int64_t n_items = rows_mine * hpc;
  if (threadIdx.x == 0) {
    for (int s = 0; s < stages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], kStepThreads);
    }
    // one local arrival (carrying the expected bytes: cs * G partial sums) and
    // the ranks' asynchronous stores complete a phase; rows 0 and 1 armed here
    for (int s = 0; s < 2; ++s) {
      mbar_init(&sums_ready[s], 1);
      mbar_arrive_expect_tx(&sums_ready[s], (uint32_t)(cs * G * 4));
    }
    fence_mbar_init();
  }
  // row-independent parameters of the CTA's channels and heads
  for (int i = threadIdx.x; i < C + BC; i += blockDim.x) {
    const int64_t ch = i < C ? (int64_t)h0 * P + i : pr.d_inner + (i - C);
    const float4 *wp = reinterpret_cast<const float4 *>(prm.conv_w) + ch;
    reinterpret_cast<float4 *>(smem_raw + Lo.cw)[i] =
        M2_OK(wp, 16, sp.conv_w, &g_step_errors) ? __ldg(wp) : make_float4(0.f, 0.f, 0.f, 0.f);
    reinterpret_cast<float *>(smem_raw + Lo.cb)[i] =
        M2_OK(prm.conv_b + ch, 4, sp.conv_b, &g_step_errors) ? __ldg(prm.conv_b + ch) : 0.0f;
    if (i < C)
      reinterpret_cast<float *>(smem_raw + Lo.nw)[i] =
          M2_OK(prm.norm_w + ch, 4, sp.norm_w, &g_step_errors) ? __ldg(prm.norm_w + ch) : 0.0f;
  }
  for (int i = threadIdx.x; i < hpc; i += blockDim.x) {
    reinterpret_cast<float *>(smem_raw + Lo.dtb)[i] =
        M2_OK(prm.dt_bias + h0 + i, 4, sp.dt_bias, &g_step_errors) ? prm.dt_bias[h0 + i] : 0.0f;
    reinterpret_cast<float *>(smem_raw + Lo.Ah)[i] =
        M2_OK(prm.A + h0 + i, 4, sp.A, &g_step_errors) ? prm.A[h0 + i] : 0.0f;
    reinterpret_cast<float *>(smem_raw + Lo.Dh)[i] =
        M2_OK(prm.D + h0 + i, 4, sp.D, &g_step_errors) ? prm.D[h0 + i] : 0.0f;
  }
  __syncthreads();
  // every CTA of the cluster runs (and has initialised its barriers) before any
  // remote store or arrive
  cluster_arrive_wait();

  if (threadIdx.x >= kStepThreads) {
    // ---------------- producer warp: streams each head's state in, and (once the
    // compute warps have updated it in place) back out, both as bulk copies
    if (threadIdx.x == kStepThreads) {
      auto head_state = [&](int64_t item) -> float * {  // global state of item (row, head)
        const int64_t r = cid + (item / hpc) * nclusters;
        return ssm + (r * H + h0 + (int)(item % hpc)) * (int64_t)head_floats;
      };
      // item j's updated state (buffer j % stages) back to global memory, once the
      // compute warps are done with it; the buffer is free when the copy has read it
      auto write_back = [&](int64_t j) -> bool {
        const int s = (int)(j % stages);
        if (!mbar_wait_bounded(&empty[s], (uint32_t)((j / stages) & 1), &g_step_errors))
          return false;
        float *dst = head_state(j);
        if (M2_OK_BULK(dst, head_bytes, sp.ssm, &g_step_errors)) {
          bulk_s2g(dst, sbuf + s * head_floats, head_bytes);
          bulk_wait_read_all();
        }
        return true;
      };
      int64_t np = 0;  // items issued
      bool wb_ok = true;
      for (; np < n_items; ++np) {
        const int s = (int)(np % stages);
        if (np >= stages && !(wb_ok = write_back(np - stages))) break;
        const float *src = head_state(np);
        if (M2_OK_BULK(src, head_bytes, sp.ssm, &g_step_errors)) {
          mbar_arrive_expect_tx(&full[s], head_bytes);
          bulk_g2s(sbuf + s * head_floats, src, head_bytes, &full[s]);
        } else {
          mbar_arrive(&full[s]);  // nothing copied: the stage completes without bytes
        }
      }
      // the last heads' write-backs; then no copy may be in flight when the CTA
      // exits (each stage's last load, every store)
      for (int64_t kk = std::max<int64_t>(0, np - stages); wb_ok && kk < np; ++kk)
        wb_ok = write_back(kk);
      for (int64_t kk = std::max<int64_t>(0, np - stages); kk < np; ++kk)
        mbar_wait_bounded(&full[kk % stages], (uint32_t)((kk / stages) & 1), &g_step_errors);
      bulk_wait_all();
    }
    __syncwarp();
    cluster_arrive_wait();
    return;
  }

  // ---------------- compute warps
  const int tid = threadIdx.x;
  // this thread's column of float4s (q) and first row (p0); rows p0 + kRowsPerPass * i
  const int q = tid % NQ, p0 = tid / NQ;
  const int passes = P / kRowsPerPass > 0 ? P / kRowsPerPass : 1;
  const bool active = p0 < P;  // P * NQ may be smaller than the block
  const int g_lo = h0 / hpg, g_hi = (h0 + hpc - 1) / hpg;
  const float gs = (float)(hpg * P);
  bool ok = true;
  int64_t k = 0;  // next item to consume

  // copies of row rr's inputs into buffer rr % 2 (16-byte pieces, one commit group)
  auto prefetch = [&](int64_t rr) {
    const int64_t bi = cid + rr * nclusters;
    char *pb = reinterpret_cast<char *>(pre0 + (rr & 1) * Lo.pre_elems);
    const char *csr = reinterpret_cast<const char *>(conv_state + bi * pr.conv_dim * 4);
    const int tsz = (int)sizeof(T);
    const int n0 = 4 * C * tsz / 16, n1 = n0 + 4 * BC * tsz / 16, n2 = n1 + C * tsz / 16,
              n3 = n2 + BC * tsz / 16, n4 = n3 + C * tsz / 16;
    for (int i = tid; i < n4; i += kStepThreads) {
      const char *src;
      if (i < n0) src = csr + (int64_t)h0 * P * 4 * tsz + 16 * i;
      else if (i < n1) src = csr + pr.d_inner * 4 * tsz + 16 * (i - n0);
      else if (i < n2) src = reinterpret_cast<const char *>(xBC + bi * ld_x + (int64_t)h0 * P) + 16 * (i - n1);
      else if (i < n3) src = reinterpret_cast<const char *>(xBC + bi * ld_x + pr.d_inner) + 16 * (i - n2);
      else src = reinterpret_cast<const char *>(z + bi * ld_z + (int64_t)h0 * P) + 16 * (i - n3);
      if (M2_OK(src, 16, i < n1 ? sp.conv : (i < n3 ? sp.xbc : sp.z), &g_step_errors))
        cp_async16(pb + 16 * i, src);
    }
    cp_async_commit();
  };

  // step 4 for row rr: wait for every rank's partial sums, scale, store y; this
  // rank's share of the shifted B/C conv state
  auto finish = [&](int64_t rr) {
    const int par = (int)(rr & 1);
    const int64_t bi = cid + rr * nclusters;
    ok = __all_sync(0xffffffffu,
                    ok && mbar_wait_cluster_bounded(&sums_ready[par], (uint32_t)((rr >> 1) & 1)));
    for (int g = g_lo + tid; g <= g_hi; g += kStepThreads) {
      float tot = 0.0f;
      for (int r = 0; r < cs; ++r) tot += part[(par * cs + r) * G + g];
      inv[g] = rsqrtf(tot / gs + pr.eps);
    }
    step_bar();
    // re-arm this parity for row rr + 2: no rank sends that row before this CTA
    // has sent row rr + 1, which happens after this point
    if (tid == 0 && rr + 2 < rows_mine) mbar_arrive_expect_tx(&sums_ready[par], (uint32_t)(cs * G * 4));
    T *yr = y + bi * pr.d_inner + (int64_t)h0 * P;
    const float *ysr = ys + par * C;
    for (int c = tid; c < C; c += kStepThreads) {
      float o = ysr[c] * inv[(h0 + c / P) / hpg] * nw[c];
      if (pr.nbg) o *= silu_fast(to_f(zk[par * C + c]));
      if (M2_OK(yr + c, (unsigned)sizeof(T), sp.y, &g_step_errors)) yr[c] = from_f<T>(o);
    }
    T *csr = conv_state + bi * pr.conv_dim * 4;
    const T *bn = bcn + par * 4 * BC;
    for (int jb = rank + cs * tid; jb < BC; jb += cs * kStepThreads)
      if (M2_OK(csr + (pr.d_inner + jb) * 4, 4 * (unsigned)sizeof(T), sp.conv, &g_step_errors))
        store4(csr + (pr.d_inner + jb) * 4, bn[jb * 4], bn[jb * 4 + 1], bn[jb * 4 + 2],
               bn[jb * 4 + 3]);
  };

  if (rows_mine > 0) {
    prefetch(0);
    if (tid < hpc)
      dtr[tid] = M2_OK(dt_raw + (int64_t)cid * ld_dt + h0 + tid, (unsigned)sizeof(T), sp.dt,
                       &g_step_errors)
                     ? to_f(dt_raw[(int64_t)cid * ld_dt + h0 + tid])
                     : 0.0f;
  }
  for (int64_t rr = 0; rr < rows_mine; ++rr) {
    const int64_t bi = cid + rr * nclusters;
    const int par = (int)(rr & 1);
    cp_async_wait_all();
    step_bar();  // row rr's inputs (and raw dt) in shared memory
    const T *pb = pre0 + par * Lo.pre_elems;
    const T *pcx = pb, *pcbc = pb + 4 * C, *px = pcbc + 4 * BC, *pxbc = px + C, *pz = pxbc + BC;
    // 1. conv + SiLU; own channels' shifted state back to global memory
    T *csr = conv_state + bi * pr.conv_dim * 4;
    for (int i = tid; i < C + BC; i += kStepThreads) {
      const float4 w4 = cw[i];
      const float w[4] = {w4.x, w4.y, w4.z, w4.w};
      if (i < C) {
        const T a0 = pcx[i * 4 + 1], a1 = pcx[i * 4 + 2], a2 = pcx[i * 4 + 3], a3 = px[i];
        if (M2_OK(csr + ((int64_t)h0 * P + i) * 4, 4 * (unsigned)sizeof(T), sp.conv, &g_step_errors))
          store4(csr + ((int64_t)h0 * P + i) * 4, a0, a1, a2, a3);
        ux[i] = silu_fast(conv4(w, cb[i], a0, a1, a2, a3));
        if (pr.nbg) zk[par * C + i] = pz[i];
      } else {
        const int j = i - C;
        const T a0 = pcbc[j * 4 + 1], a1 = pcbc[j * 4 + 2], a2 = pcbc[j * 4 + 3], a3 = pxbc[j];
        ubc[j] = silu_fast(conv4(w, cb[i], a0, a1, a2, a3));
        T *bn = bcn + par * 4 * BC + j * 4;
        bn[0] = a0;
        bn[1] = a1;
        bn[2] = a2;
        bn[3] = a3;
      }
    }
    if (tid < hpc) {
      const float dt = softplus_f(dtr[par * hpc + tid] + dtb[tid]);
      dts[tid] = dt;
      dAs[tid] = expf(dt * Ah[tid]);
    }
    step_bar();

    // 2. the next row's inputs start to arrive; per head: wait for its buffer,
    //    update in registers, store to global, contract with C, release
    float dtn = 0.0f;
    if (rr + 1 < rows_mine) {
      prefetch(rr + 1);
      if (tid < hpc)
        dtn = M2_OK(dt_raw + (bi + nclusters) * ld_dt + h0 + tid, (unsigned)sizeof(T), sp.dt,
                    &g_step_errors)
                  ? to_f(dt_raw[(bi + nclusters) * ld_dt + h0 + tid])
                  : 0.0f;
    }
    float *ysr = ys + par * C;
    for (int j = 0; j < hpc; ++j, ++k) {
      const int s = (int)(k % stages);
      ok = __all_sync(0xffffffffu,
                      ok && mbar_wait_bounded(&full[s], (uint32_t)((k / stages) & 1), &g_step_errors));
      if (ok && active) {
        const int g = (h0 + j) / hpg;
        const float *xh = ux + j * P;
        const float4 b = reinterpret_cast<const float4 *>(ubc + g * N)[q];
        const float4 cc = reinterpret_cast<const float4 *>(ubc + GN + g * N)[q];
        const float dt = dts[j], dA = dAs[j], Dj = Dh[j];
        // updated in place: the producer copies the buffer back to global memory
        float4 *src = reinterpret_cast<float4 *>(sbuf + s * head_floats);
        // up to 4 rows per thread, independent: their reductions interleave
        constexpr int kPass = 4;
        float pt[kPass], xs[kPass];
#pragma unroll
        for (int i = 0; i < kPass; ++i) {
          pt[i] = 0.0f;
          xs[i] = 0.0f;
          if (i < passes) {
            const int p = p0 + i * kRowsPerPass, idx = p * NQ + q;
            const float xv = xh[p], xdt = xv * dt;
            float4 v = src[idx];
            v.x = fmaf(dA, v.x, xdt * b.x);
            v.y = fmaf(dA, v.y, xdt * b.y);
            v.z = fmaf(dA, v.z, xdt * b.z);
            v.w = fmaf(dA, v.w, xdt * b.w);
            src[idx] = v;
            pt[i] = fmaf(v.x, cc.x, fmaf(v.y, cc.y, fmaf(v.z, cc.z, v.w * cc.w)));
            xs[i] = xv;
          }
        }
#pragma unroll
        for (int o = NQ / 2; o > 0; o >>= 1)
#pragma unroll
          for (int i = 0; i < kPass; ++i) pt[i] += __shfl_xor_sync(0xffffffffu, pt[i], o);
#pragma unroll
        for (int i = 0; i < kPass; ++i)
          if (i < passes && q == 0) ysr[j * P + p0 + i * kRowsPerPass] = fmaf(Dj, xs[i], pt[i]);
        // rows beyond the first kPass passes (P / kRowsPerPass > kPass)
        for (int i = kPass; i < passes; ++i) {
          const int p = p0 + i * kRowsPerPass, idx = p * NQ + q;
          const float xv = xh[p], xdt = xv * dt;
          float4 v = src[idx];
          v.x = fmaf(dA, v.x, xdt * b.x);
          v.y = fmaf(dA, v.y, xdt * b.y);
          v.z = fmaf(dA, v.z, xdt * b.z);
          v.w = fmaf(dA, v.w, xdt * b.w);
          src[idx] = v;
          float t = fmaf(v.x, cc.x, fmaf(v.y, cc.y, fmaf(v.z, cc.z, v.w * cc.w)));
#pragma unroll
          for (int o = NQ / 2; o > 0; o >>= 1) t += __shfl_xor_sync(0xffffffffu, t, o);
          if (q == 0) ysr[j * P + p] = fmaf(Dj, xv, t);
        }
      }
      // this thread is done with buffer s: its updates visible to the bulk copy out
      fence_proxy_async_smem();
      mbar_arrive(&empty[s]);
    }
    if (tid < hpc) dtr[(par ^ 1) * hpc + tid] = dtn;
    step_bar();  // y of the row complete

    // 3. gate, partial sums of squares per norm group (= head group)
    for (int g = tid; g < G; g += kStepThreads)
      if (g < g_lo || g > g_hi) mysum[g] = 0.0f;
    for (int g = g_lo; g <= g_hi; ++g) {
      const int c0 = max(g * hpg, h0) * P - h0 * P, c1 = min((g + 1) * hpg, h0 + hpc) * P - h0 * P;
      float ss = 0.0f;
      for (int c = c0 + tid; c < c1; c += kStepThreads) {
        float v = ysr[c];
        if (!pr.nbg) {
          v *= silu_fast(to_f(pz[c]));
          ysr[c] = v;  // the gated value, scaled in step 4
        }
        ss += v * v;
      }
      ss = step_block_sum(ss, red);
      if (tid == 0) mysum[g] = ss;
    }
    step_bar();
    // 4. the previous row, whose partial sums have had a row's time to arrive
    if (rr > 0) finish(rr - 1);
    // 5. this row's partials into part[par][rank][*] of every rank; thread r
    //    sends rank r's, completing bytes on its barrier
    if (tid < cs) {
      const uint32_t bar = cluster_addr(&sums_ready[par], tid);
      for (int g = 0; g < G; ++g)
        st_async_cluster(cluster_addr(part + (par * cs + rank) * G + g, tid), mysum[g], bar);
    }
  }
  if (rows_mine > 0) finish(rows_mine - 1);
  // no rank may exit while another can still store into its shared memory
  cluster_arrive_wait();
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
  // the deepest ring (2 .. 4 heads) that still lets two CTAs share an SM
  int stages = kMaxStages;
  while (stages > 2 &&
         step_layout<T>(stages, hpc, pr.P, pr.G, pr.N, cs).total > kStepSmemPerCta)
    --stages;
  if ((size_t)stages * head_bytes > 65536) stages = 2;
  const size_t smem = step_layout<T>(stages, hpc, pr.P, pr.G, pr.N, cs).total;
  if (smem > 227 * 1024) return cudaErrorInvalidValue;
  // The shared-memory attribute (per context) and the occupancy answer (per
  // device, shared-memory size and cluster size) are kept from the previous
  // call with the same key, so a decode loop pays for neither on every step.
  struct LaunchCache {
    unsigned long long ctx;
    size_t smem;
    int cs, max_clusters;
  };
  static std::mutex mu;
  static LaunchCache cache[64] = {};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  const unsigned long long ctx = current_context_id();
  LaunchCache hit = {};
  const bool cacheable = dev >= 0 && dev < 64 && ctx != 0;
  if (cacheable) {
    std::lock_guard<std::mutex> lock(mu);
    hit = cache[dev];
  }
  const bool fresh = !(cacheable && hit.ctx == ctx && hit.smem == smem && hit.cs == cs);
  if (fresh) {
    e = cudaFuncSetAttribute(ssd_step_kernel<T, N>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)smem);
    if (e != cudaSuccess) return e;
    if (cs > 8) {
      e = cudaFuncSetAttribute(ssd_step_kernel<T, N>,
                               cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
      if (e != cudaSuccess) return e;
    }
  }
  cudaLaunchConfig_t cfg = {};
  cfg.blockDim = dim3(kStepBlock, 1, 1);
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
  int max_clusters = fresh ? 0 : hit.max_clusters;
  if (fresh) {
    if (cudaOccupancyMaxActiveClusters(&max_clusters, ssd_step_kernel<T, N>, &cfg) !=
            cudaSuccess ||
        max_clusters <= 0) {
      cudaGetLastError();  // clear a failed query; fall back to one cluster per row
      max_clusters = 0;
    } else if (cacheable) {
      std::lock_guard<std::mutex> lock(mu);
      cache[dev] = LaunchCache{ctx, smem, cs, max_clusters};
    }
  }
  if (max_clusters <= 0) max_clusters = (int)std::min<int64_t>(pr.batch, 65535);
  // the fewest clusters that keep the largest per-cluster row count: no cluster idles
  // at the end while others still have a row left
  const int64_t fit = std::max<int64_t>(1, std::min<int64_t>(pr.batch, max_clusters));
  const int64_t rows_per = (pr.batch + fit - 1) / fit;
  const int nclusters = (int)std::max<int64_t>(1, (pr.batch + rows_per - 1) / rows_per);
  cfg.gridDim = dim3((unsigned)cs, (unsigned)nclusters, 1);
  stage_mark(a.stream, 0);
  StepSpans sp;
  {
    const size_t ts = sizeof(T), b = (size_t)pr.batch;
    sp.xbc = span_of(a.xBC, ((b - 1) * a.ld_xbc + pr.conv_dim) * ts);
    sp.z = span_of(a.z, ((b - 1) * a.ld_z + pr.d_inner) * ts);
    sp.dt = span_of(a.dt_raw, ((b - 1) * a.ld_dt + pr.H) * ts);
    sp.y = span_of(a.y, b * pr.d_inner * ts);
    sp.conv = span_of(a.conv_state, b * pr.conv_dim * 4 * ts);
    sp.ssm = span_of(a.ssm_state, b * pr.H * pr.P * pr.N * 4);
    sp.conv_w = span_of(a.prm.conv_w, (size_t)pr.conv_dim * 16);
    sp.conv_b = span_of(a.prm.conv_b, (size_t)pr.conv_dim * 4);
    sp.norm_w = span_of(a.prm.norm_w, (size_t)pr.d_inner * 4);
    sp.dt_bias = span_of(a.prm.dt_bias, (size_t)pr.H * 4);
    sp.A = span_of(a.prm.A, (size_t)pr.H * 4);
    sp.D = span_of(a.prm.D, (size_t)pr.H * 4);
  }
  e = cudaLaunchKernelEx(&cfg, ssd_step_kernel<T, N>, pr, a.prm, static_cast<const T *>(a.xBC),
                         a.ld_xbc, static_cast<const T *>(a.z), a.ld_z,
                         static_cast<const T *>(a.dt_raw), a.ld_dt, static_cast<T *>(a.y),
                         static_cast<T *>(a.conv_state), a.ssm_state, hpc, stages, nclusters, sp);
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

cudaError_t set_step_stall(unsigned int v) {
  return cudaMemcpyToSymbol(g_step_stall, &v, sizeof(v));
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
