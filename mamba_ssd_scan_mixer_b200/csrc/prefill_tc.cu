// Prefill of the Mamba-2 mixer core on the 5th-generation tensor cores
// (tcgen05.mma, accumulators in tensor memory), for bf16 I/O with headdim 64
// and d_state 64.
//
// It evaluates the chunked state-space-duality form of the scan (the Mamba-2
// layer named on the state-spaces/mamba repository page, opendeer.net, "About
// the project"; chunked prefill per "Zamba2 hybrid architecture in
// Transformers", qwbw.cn, section 三 step 3) with 128-token chunks, so that
// a chunk's tokens are the MMA's M = 128 rows:
//
//   tc_chunk_state  conv+SiLU of x (two heads) and B, dt/cumsum, then
//                   S_c = (x o w)^T B with w_s = exp(cum_end - cum_s) dt_s:
//                   M = 128 (2 heads x 64 lanes), N = 64, K = 128 tokens.
//   tc_state_pass   H_{c+1} = exp(cum_end) H_c + S_c over chunks in fp32; the
//                   state entering each chunk is kept as the fp16 MMA operand,
//                   the final state in fp32.
//   tc_chunk_out    persistent clusters; per (row, chunk, group) unit the
//                   cluster's CTAs split the heads of the group:
//                   CB = C B^T (M = N = 128, K = 64) once; per head the
//                   operand CB o exp(cum_t - cum_s) dt_s (causal, D on the
//                   diagonal) times x (K = 128) and C times H_c^T (K = 64, a
//                   second accumulator scaled by exp(cum_t)) give y_pre in TMEM;
//                   the silu(z) gate and sums of squares follow, the per-token
//                   sums are exchanged through distributed shared memory, and
//                   the normalised output is written in bf16.
//
// Operands are fp16 (11-bit significand; bf16's 8 bits cannot meet the output
// tolerance on these workloads), accumulation is fp32.  The chunk-state
// product uses a two-term fp16 split of both operands (hi*hi + hi*lo + lo*hi),
// because the returned final state must hold 2e-2 of its RMS.
#include <cuda.h>
#include <cudaTypedefs.h>

#include <algorithm>

#include "common.cuh"


namespace m2 {
namespace {

constexpr int kQ = 128;          // tokens per chunk = MMA M
constexpr int kThreads = 512;    // 16 compute warps
constexpr int kWsThreads = kThreads + 64;   // + TMA producer warp + MMA issuer warp
constexpr int kK1Threads = kThreads + 96;   // + 2 producer warps (even / odd items) + MMA warp
constexpr int kHP = 64;          // headdim
constexpr int kNS = 64;          // d_state
constexpr int kMaxHeadsPerCta = 5;  // TMEM: 128 (CB) + 5 x 64 (y) + 64 (C H_c^T) = 512 columns
constexpr uint32_t kTmemT = 128 + 64 * kMaxHeadsPerCta;  // column of the C H_c^T accumulator
constexpr float kLog2e = 1.4426950408889634f;

static __device__ unsigned int g_tc_errors = 0;
static __device__ unsigned int g_tc_stall = 0;  // mamba2_debug_stall_waits

struct TcArgs {
  Problem pr;
  mamba2_params prm;
  const __nv_bfloat16 *xBC;
  int64_t ld_x;
  const __nv_bfloat16 *z;
  int64_t ld_z;
  const __nv_bfloat16 *dt_raw;
  int64_t ld_dt;
  __nv_bfloat16 *y;
  const __nv_bfloat16 *conv_in;  // conv state read for the left context (or null)
  float *ssm_state;              // in (if states_in) / out (may be null)
  int states_in;
  int nch;                       // chunks of kQ tokens
  float *S;                      // [b][nch][H][n/4 16][p 64][4] chunk states
  float *cum_end;                // [b][nch][H] chunk sum of dt*A
  float *cum;                    // [b][nch][H][128] running sum of dt*A inside the chunk
  float *dtv;                    // [b][nch][H][128] dt (0 past the end of the sequence)
  __half *Hc;                    // [b][nch][H][n 64][p 64] state entering each chunk
  __half *u;                     // [b][L][conv_dim] post-conv x | B | C, fp16
  int hpc;                       // max heads per CTA in tc_chunk_out
};

// silu(v) = v * sigmoid(v) with sigmoid(v) = (1 + tanh(v / 2)) / 2, using the
// hardware tanh approximation (one special-function op per element).
__device__ __forceinline__ float tanh_approx(float x) {
  float y;
  asm("tanh.approx.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
__device__ __forceinline__ float silu_fast(float v) {
  const float h = 0.5f * v;
  return fmaf(h, tanh_approx(h), h);
}

__device__ __forceinline__ float ex2_approx(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// Inclusive prefix sum over the 32 lanes of a warp.
__device__ __forceinline__ float warp_scan(float v, int lane) {
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const float n = __shfl_up_sync(0xffffffffu, v, o);
    if (lane >= o) v += n;
  }
  return v;
}

// Post-conv activations of 8 channels x 4 tokens -> u (fp16), tokens < L only.
__device__ __forceinline__ void store_u(const TcArgs &a, int64_t bi, int64_t t0, int64_t ch,
                                        const float (&v)[4][8]) {
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    const int64_t t = t0 + k;
    if (t < a.pr.L) {
      uint4 o;
      o.x = pack_half2(v[k][0], v[k][1]);
      o.y = pack_half2(v[k][2], v[k][3]);
      o.z = pack_half2(v[k][4], v[k][5]);
      o.w = pack_half2(v[k][6], v[k][7]);
      *reinterpret_cast<uint4 *>(a.u + (bi * a.pr.L + t) * a.pr.conv_dim + ch) = o;
    }
  }
}

__device__ __forceinline__ void st_shared_v2(uint32_t addr, uint32_t a, uint32_t b) {
  asm volatile("st.shared.v2.b32 [%0], {%1, %2};" ::"r"(addr), "r"(a), "r"(b) : "memory");
}
__device__ __forceinline__ void st_shared_v4(uint32_t addr, uint32_t a, uint32_t b, uint32_t c,
                                             uint32_t d) {
  asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(a), "r"(b), "r"(c),
               "r"(d)
               : "memory");
}
__device__ __forceinline__ uint4 ld_shared_v4(uint32_t addr) {
  uint4 v;
  asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "r"(addr));
  return v;
}


__device__ __forceinline__ void tma_load_3d(uint32_t dst, const CUtensorMap *map, int c0, int c1,
                                            int c2, uint64_t *bar) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3, %4}], [%5];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(c2), "r"(smem_u32(bar))
      : "memory");
}
__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap *map, int c0, int c1,
                                            uint64_t *bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3}], [%4];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(smem_u32(bar))
      : "memory");
}
__device__ __forceinline__ void tma_store_3d(const CUtensorMap *map, uint32_t src, int c0, int c1,
                                             int c2) {
  asm volatile("cp.async.bulk.tensor.3d.global.shared::cta.tile.bulk_group [%0, {%2, %3, %4}], [%1];"
               ::"l"(reinterpret_cast<uint64_t>(map)), "r"(src), "r"(c0), "r"(c1), "r"(c2)
               : "memory");
}
// Bulk-store groups: commit the stores issued so far; wait until at most one /
// none of the committed groups still reads shared memory.
__device__ __forceinline__ void bulk_commit() {
  asm volatile("cp.async.bulk.commit_group;" ::: "memory");
}
// (the group count of wait_group is an immediate: the cases used are spelled out)
__device__ __forceinline__ void bulk_wait_read_le(int n) {
  if (n >= 4) asm volatile("cp.async.bulk.wait_group.read 4;" ::: "memory");
  else if (n == 3) asm volatile("cp.async.bulk.wait_group.read 3;" ::: "memory");
  else if (n == 2) asm volatile("cp.async.bulk.wait_group.read 2;" ::: "memory");
  else if (n == 1) asm volatile("cp.async.bulk.wait_group.read 1;" ::: "memory");
  else asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
}
__device__ __forceinline__ void bulk_wait_read_all() {
  asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
}
__device__ __forceinline__ void cluster_arrive_relaxed() {
  asm volatile("barrier.cluster.arrive.relaxed.aligned;" ::: "memory");
}
__device__ __forceinline__ void cluster_arrive_release() {
  asm volatile("barrier.cluster.arrive.release.aligned;" ::: "memory");
}
__device__ __forceinline__ void cluster_wait() {
  asm volatile("barrier.cluster.wait.acquire.aligned;" ::: "memory");
}
// barrier over the 512 compute threads only (the producer warp never joins)
__device__ __forceinline__ void compute_sync() {
  asm volatile("bar.sync 1, 512;" ::: "memory");
}
__device__ __forceinline__ bool compute_all(bool v) {
  int r;
  asm volatile("{\n .reg .pred p, q;\n setp.ne.s32 p, %1, 0;\n bar.red.and.pred q, 1, 512, p;\n"
               " selp.s32 %0, 1, 0, q;\n}"
               : "=r"(r)
               : "r"((int)v)
               : "memory");
  return r != 0;
}
__device__ __forceinline__ bool wait_compute(uint64_t *bar, uint32_t parity, bool ok) {
  const bool got = ok ? mbar_wait_bounded(bar, parity, &g_tc_errors) : false;
  return compute_all(got);
}
// Smem descriptor for an MN-major SW128 operand: 8-row (K) atoms of 64
// elements (N) x 128 B, K atoms 1024 B apart (SBO), N atoms `lbo` apart.
__device__ __forceinline__ uint64_t umma_desc_sw128_mn(uint32_t saddr, uint32_t lbo) {
  uint64_t d = (uint64_t)((saddr >> 4) & 0x3FFFu);
  d |= (uint64_t)((lbo >> 4) & 0x3FFFu) << 16;
  d |= (uint64_t)(1024u >> 4) << 32;
  d |= (uint64_t)1 << 46;
  d |= (uint64_t)2 << 61;
  return d;
}

// ============================================================== chunk states
// Persistent: grid = one CTA per SM; CTA k takes a contiguous range of work
// items ordered (row, chunk, group, item), where the items of a (row, chunk,
// group) are its head pairs followed by one C item:
//   pair item: conv + SiLU of x (2 heads) and of B (only when the CTA's previous
//     item had another (row, chunk, group): B's operands stay in shared memory),
//     post-conv values to u, then S = (x o w)^T B on the tensor cores;
//   C item: conv + SiLU of the group's C channels -> u.
// 16 compute warps + 2 producer warps + 1 MMA-issuer warp.  The producer of an
// item (one per ring stage, so they alternate) TMA-loads its raw bf16 tiles
// [136 tokens c0-3 .. c0+132][64 ch] (128-byte swizzle) into its stage,
// computes its dt weights (stored also as per-token dt and cumsum rows for the
// output kernel) and stages its conv taps while the compute warps work on the
// previous item; the MMA warp
// issues a pair item's products once its operands are in shared memory, and
// they run under the next item's convolution.
// Smem (1024-aligned): ring [2][x_A | x_B | B (a C item uses slot 0)], then the
// operands A_hi, A_lo [2 k-blocks][128 rows][128 B] and B_hi, B_lo [2][64][128 B].
constexpr uint32_t kRawRows = 136, kRawBytes = kRawRows * 128;  // 17 KB, 1024-multiple
constexpr uint32_t kK1Stage = 3 * kRawBytes;
constexpr uint32_t kK1A = 2 * 128 * 128, kK1B = 2 * 64 * 128;
constexpr uint32_t kK1Ahi = 2 * kK1Stage, kK1Alo = kK1Ahi + kK1A, kK1Bhi = kK1Alo + kK1A,
                   kK1Blo = kK1Bhi + kK1B, kK1Tiles = kK1Blo + kK1B;

struct K1Maps {
  CUtensorMap xbc;  // [b][L][conv_dim] bf16 (row stride ld_x), box 64 ch x 136 tokens
};

// conv1d + SiLU of the 8 channels in 16-byte column `cg` of a raw tile, for
// output tokens at tile rows s0+3 .. s0+6 (inputs: rows s0 .. s0+6); taps and
// bias of the tile's 64 channels in shared memory, channel 8 g + i at [i][g]
// (wt[8][8] float4, bs[8][8]) so that neighbouring groups read neighbouring words,
// stored halved: the sum is then h = pre / 2 exactly, and silu(pre) = h + h tanh(h).
__device__ __forceinline__ void conv8x4_smem(uint32_t tile, int s0, int cg, const float4 *wt,
                                             const float *bs, float (&out)[4][8]) {
  float w[8][4], bias[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const float4 wv = wt[i * 8 + cg];
    w[i][0] = wv.x;
    w[i][1] = wv.y;
    w[i][2] = wv.z;
    w[i][3] = wv.w;
    bias[i] = bs[i * 8 + cg];
  }
  float rows[7][8];
#pragma unroll
  for (int r = 0; r < 7; ++r) {
    const int R = s0 + r;
    const uint4 raw = ld_shared_v4(tile + R * 128 + (((cg ^ R) & 7) << 4));
    const __nv_bfloat162 *h2 = reinterpret_cast<const __nv_bfloat162 *>(&raw);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float2 f = __bfloat1622float2(h2[i]);
      rows[r][2 * i] = f.x;
      rows[r][2 * i + 1] = f.y;
    }
  }
#pragma unroll
  for (int k = 0; k < 4; ++k)
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const float h = bias[i] + w[i][0] * rows[k][i] + w[i][1] * rows[k + 1][i] +
                      w[i][2] * rows[k + 2][i] + w[i][3] * rows[k + 3][i];
      out[k][i] = fmaf(h, tanh_approx(h), h);
    }
}

struct K1Item {
  int64_t bi;
  int c, g, pair;
  bool isC;
  bool freshB;  // B must be convolved (the CTA's previous item had another key)
};

// Item `it`, the k-th of its CTA.  Items are ordered (row, chunk, group, r) with
// r = 0 .. pairs - 1 the head pairs and r = pairs the C item; every index fits
// in 32 bits (the launch checks the item count).
__device__ __forceinline__ K1Item k1_item(const Problem &pr, int nch, int pairs, int it, int k) {
  const unsigned key = (unsigned)it / (unsigned)(pairs + 1);
  const int r = it - (int)key * (pairs + 1);
  const unsigned bc = key / (unsigned)pr.G;
  K1Item w;
  w.g = (int)(key - bc * (unsigned)pr.G);
  w.bi = (int64_t)(bc / (unsigned)nch);
  w.c = (int)(bc - (unsigned)w.bi * (unsigned)nch);
  w.isC = r == pairs;
  w.pair = w.isC ? 0 : r;
  w.freshB = !w.isC && (k == 0 || r == 0);
  return w;
}

__global__ void __launch_bounds__(kK1Threads, 1)
    tc_chunk_state_kernel(TcArgs a, const __grid_constant__ K1Maps maps, int n_items) {
  if (test_stall(&g_tc_stall, &g_tc_errors)) return;  // every CTA alike (test aid)
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  __shared__ float ws[2][2][kQ];          // [stage][head of pair][token] chunk weights
  __shared__ float4 wts[2][3][64];        // [stage][slot][channel] conv taps
  __shared__ float bss[2][3][64];         // [stage][slot][channel] conv bias
  __shared__ uint64_t full[2], empty[2], ops_ready, mbar;
  __shared__ uint32_t tmem_holder;
  const Problem &pr = a.pr;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const uint32_t base = (smem_u32(smem_raw) + 1023u) & ~1023u;
  const uint32_t sAhi = base + kK1Ahi, sAlo = base + kK1Alo, sBhi = base + kK1Bhi,
                 sBlo = base + kK1Blo;
  const int hpg = pr.heads_per_group();
  const int pairs = (hpg + 1) / 2;
  const int it0 = (int)((int64_t)n_items * blockIdx.x / gridDim.x),
            it1 = (int)((int64_t)n_items * (blockIdx.x + 1) / gridDim.x);

  if (warp == 0) tmem_alloc(&tmem_holder, 64);
  if (tid == 0) {
    for (int k = 0; k < 2; ++k) {
      mbar_init(&full[k], 2);  // the tiles' transaction bytes + the producer's weights
      mbar_init(&empty[k], 1);
    }
    mbar_init(&ops_ready, 1);  // operands of a pair item written (compute thread 0)
    mbar_init(&mbar, 1);       // its MMAs completed (tcgen05.commit)
    fence_mbar_init();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_holder;

  if (warp == kThreads / 32 || warp == kThreads / 32 + 2) {
    // ---------------- producers: warp 16 takes the CTA's even items (ring stage
    // 0), warp 18 the odd ones (stage 1).
    const int mine = warp == kThreads / 32 ? 0 : 1;
    int k = 0;
    for (int it = it0; it < it1; ++it, ++k) {
      const int st = k & 1;
      if (st != mine) continue;
      const K1Item w = k1_item(pr, a.nch, pairs, it, k);
      const bool freshB = w.freshB;
      const int64_t c0 = (int64_t)w.c * kQ;
      const int hA = w.g * hpg + 2 * w.pair;
      const bool hasB = 2 * w.pair + 1 < hpg;
      // everything that needs no shared memory first, while the stage may still be
      // in use: the item's global loads (one round trip: dt of both heads for this
      // lane's 4 tokens, their dt_bias and A, the conv taps of its slots), the dt
      // weights, and the per-token dt and cumsum rows for the output kernel
      float dtr[2][4], dtb[2] = {0.0f, 0.0f}, Ah[2] = {0.0f, 0.0f};
      float4 tw[3][2];
      float tb[3][2];
      bool son[3];
#pragma unroll
      for (int sl = 0; sl < 3; ++sl) {
        son[sl] = w.isC ? sl == 0 : (sl == 1 ? hasB : (sl == 2 ? freshB : true));
        const int64_t ch0 = w.isC ? pr.d_inner + (int64_t)(pr.G + w.g) * kNS
                                  : (sl < 2 ? (int64_t)(hA + sl) * kHP : pr.d_inner + (int64_t)w.g * kNS);
#pragma unroll
        for (int j = 0; j < 2; ++j) {
          if (son[sl]) {
            tw[sl][j] = __ldg(reinterpret_cast<const float4 *>(a.prm.conv_w) + ch0 + lane + 32 * j);
            tb[sl][j] = __ldg(a.prm.conv_b + ch0 + lane + 32 * j);
          }
        }
      }
#pragma unroll
      for (int half = 0; half < 2; ++half) {
        const bool hv = !w.isC && (half == 0 || hasB);
        if (hv) {
          dtb[half] = __ldg(a.prm.dt_bias + hA + half);
          Ah[half] = __ldg(a.prm.A + hA + half);
        }
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const int64_t tt = c0 + 4 * lane + q;
          dtr[half][q] = (hv && tt < pr.L)
                             ? __bfloat162float(a.dt_raw[(w.bi * pr.L + tt) * a.ld_dt + hA + half])
                             : -INFINITY;
        }
      }
      float wsv[2][4];
      if (!w.isC) {
#pragma unroll
        for (int half = 0; half < 2; ++half) {
          const bool hv = half == 0 || hasB;
          float dt4[4], a4[4];
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            dt4[q] = dtr[half][q] != -INFINITY ? softplus_f(dtr[half][q] + dtb[half]) : 0.0f;
            a4[q] = dt4[q] * Ah[half];
          }
          const float tot = a4[0] + a4[1] + a4[2] + a4[3];
          float run = warp_scan(tot, lane) - tot;
          const float cum_end = __shfl_sync(0xffffffffu, run + tot, 31);
          float cq[4];
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            run += a4[q];
            cq[q] = run;
            wsv[half][q] = expf(cum_end - run) * dt4[q];
          }
          if (hv) {
            const int64_t row = (w.bi * a.nch + w.c) * pr.H + hA + half;
            reinterpret_cast<float4 *>(a.cum + row * kQ)[lane] = make_float4(cq[0], cq[1], cq[2], cq[3]);
            reinterpret_cast<float4 *>(a.dtv + row * kQ)[lane] = make_float4(dt4[0], dt4[1], dt4[2], dt4[3]);
            if (lane == 0) a.cum_end[row] = cum_end;
          }
        }
      }
      // the stage is free once the compute warps are done with item k - 2
      if (k >= 2) {
        bool got = lane == 0 ? mbar_wait_bounded(&empty[st], (uint32_t)(((k >> 1) - 1) & 1),
                                                 &g_tc_errors)
                             : true;
        if (!__all_sync(0xffffffffu, got)) break;
      }
      if (lane == 0) {
        const uint32_t stage = base + st * kK1Stage;
        if (w.isC) {
          mbar_arrive_expect_tx(&full[st], kRawBytes);
          tma_load_3d(stage, &maps.xbc, (int)(pr.d_inner + (int64_t)(pr.G + w.g) * kNS),
                      (int)c0 - 3, (int)w.bi, &full[st]);
        } else {
          mbar_arrive_expect_tx(&full[st],
                                (1u + (hasB ? 1u : 0u) + (freshB ? 1u : 0u)) * kRawBytes);
          tma_load_3d(stage, &maps.xbc, hA * kHP, (int)c0 - 3, (int)w.bi, &full[st]);
          if (hasB)
            tma_load_3d(stage + kRawBytes, &maps.xbc, (hA + 1) * kHP, (int)c0 - 3, (int)w.bi,
                        &full[st]);
          if (freshB)
            tma_load_3d(stage + 2 * kRawBytes, &maps.xbc, (int)(pr.d_inner + (int64_t)w.g * kNS),
                        (int)c0 - 3, (int)w.bi, &full[st]);
        }
      }
      if (!w.isC) {
#pragma unroll
        for (int half = 0; half < 2; ++half)
#pragma unroll
          for (int q = 0; q < 4; ++q) ws[st][half][4 * lane + q] = wsv[half][q];
      }
      // conv taps and bias of the item's slots, channel 8 g + i at [i][g]
#pragma unroll
      for (int sl = 0; sl < 3; ++sl) {
        if (!son[sl]) continue;
#pragma unroll
        for (int j = 0; j < 2; ++j) {
          const int i = lane + 32 * j, d = (i & 7) * 8 + (i >> 3);
          const float4 w4 = tw[sl][j];  // halved (exact), see conv8x4_smem
          wts[st][sl][d] = make_float4(0.5f * w4.x, 0.5f * w4.y, 0.5f * w4.z, 0.5f * w4.w);
          bss[st][sl][d] = 0.5f * tb[sl][j];
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&full[st]);  // weights of this stage written
    }
  } else if (warp == kThreads / 32 + 1) {
    // ---------------- MMA issuer: S = x_hi B_hi + x_hi B_lo + x_lo B_hi per pair item
    if (lane == 0) {
      const uint32_t idesc = umma_idesc_f16(128, 64);
      const uint32_t As[3] = {sAhi, sAhi, sAlo}, Bs[3] = {sBhi, sBlo, sBhi};
      int n = 0;
      for (int it = it0; it < it1; ++it) {
        if (k1_item(pr, a.nch, pairs, it, 1).isC) continue;
        if (!mbar_wait_bounded(&ops_ready, (uint32_t)(n & 1), &g_tc_errors)) break;
        ++n;
        tc_fence_after();
        for (int prod = 0; prod < 3; ++prod)
          for (int ks = 0; ks < 8; ++ks) {
            const int blk = ks >> 2, kin = ks & 3;
            umma_f16(tmem, umma_desc_sw128(As[prod] + blk * 16384 + kin * 32),
                     umma_desc_sw128(Bs[prod] + blk * 8192 + kin * 32), idesc,
                     (prod > 0 || ks > 0) ? 1u : 0u);
          }
        umma_commit(&mbar);
      }
    }
  } else {
    // ---------------- compute warps
    bool ok = true;
    int k = 0, npair_done = 0;
    // the pair item whose MMA is in flight: its chunk states are stored from TMEM
    // (rows m = 32 (warp % 4) + lane, 16 columns per warp / 4; S is kept
    // [n/4][p][4] per head so that a warp's float4 stores are contiguous)
    struct Pending {
      int64_t bi;
      int c, hA;
      bool hasB;
    } pw{};
    bool pending = false;
    auto store_states = [&](const Pending &q) {
      tc_fence_after();
      const int m = 32 * (warp & 3) + lane, half = m >> 6, p = m & 63, cb = warp >> 2;
      float sv[16];
      tmem_ld16(tmem + ((uint32_t)(32 * (warp & 3)) << 16) + 16 * cb, sv);
      if (half == 0 || q.hasB) {
        float4 *dst = reinterpret_cast<float4 *>(
            a.S + ((q.bi * a.nch + q.c) * pr.H + q.hA + half) * (int64_t)(kHP * kNS));
#pragma unroll
        for (int i = 0; i < 4; ++i)
          dst[(4 * cb + i) * kHP + p] =
              make_float4(sv[4 * i], sv[4 * i + 1], sv[4 * i + 2], sv[4 * i + 3]);
      }
      tc_fence_before();  // TMEM read before the next MMA is issued
    };
    for (int it = it0; ok && it < it1; ++it, ++k) {
      const int st = k & 1;
      const uint32_t stage = base + st * kK1Stage;
      ok = wait_compute(&full[st], (uint32_t)((k >> 1) & 1), ok);
      if (!ok) break;
      const K1Item w = k1_item(pr, a.nch, pairs, it, k);
      const bool freshB = w.freshB;
      const int64_t c0 = (int64_t)w.c * kQ;
      const int hA = w.g * hpg + 2 * w.pair;
      const bool hasB = 2 * w.pair + 1 < hpg;
      // channel of slot s (C items use slot 0 for C)
      auto slot_ch = [&](int sl) -> int64_t {
        if (w.isC) return pr.d_inner + (int64_t)(pr.G + w.g) * kNS;
        return sl < 2 ? (int64_t)(hA + sl) * kHP : pr.d_inner + (int64_t)w.g * kNS;
      };
      auto slot_on = [&](int sl) -> bool {
        return w.isC ? sl == 0 : (sl == 1 ? hasB : (sl == 2 ? freshB : true));
      };
      // missing second head: zero rows 64..127 of the x operands
      auto zero_tile = [&](int cg, int s0) {
        const int blk = s0 >> 6, kq = s0 & 63;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const uint32_t off = blk * 16384 + sw128_off(64 + cg * 8 + i, kq);
          st_shared_v2(sAhi + off, 0u, 0u);
          st_shared_v2(sAlo + off, 0u, 0u);
        }
      };
      // operands of one tile: x o w (slots 0, 1) or B (slot 2), split into fp16 hi + lo
      auto put_operands = [&](int sl, int cg, int s0, const float (&v)[4][8]) {
        const int blk = s0 >> 6, kq = s0 & 63;
        float wk[4] = {1.0f, 1.0f, 1.0f, 1.0f};  // x is weighted per token, B is not
        if (sl < 2) {
          const float4 w4 = *reinterpret_cast<const float4 *>(&ws[st][sl][s0]);
          wk[0] = w4.x;
          wk[1] = w4.y;
          wk[2] = w4.z;
          wk[3] = w4.w;
        }
        const bool rot = (cg & 1) != 0;
        const uint32_t hi_base = sl < 2 ? sAhi + blk * 16384 : sBhi + blk * 8192;
        const uint32_t lo_base = sl < 2 ? sAlo + blk * 16384 : sBlo + blk * 8192;
        const int row0 = (sl < 2 ? sl * 64 : 0) + cg * 8;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          float hq[4], lq[4];
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) {
            const float x = (rot ? v[kk][i ^ 4] : v[kk][i]) * wk[kk];
            // hi: x cut to 11 significant bits (an fp16 value), lo: the exact rest
            hq[kk] = __uint_as_float(__float_as_uint(x) & 0xFFFFE000u);
            lq[kk] = x - hq[kk];
          }
          const uint32_t off = sw128_off(row0 + (rot ? (i ^ 4) : i), kq);
          st_shared_v2(hi_base + off, pack_half2(hq[0], hq[1]), pack_half2(hq[2], hq[3]));
          st_shared_v2(lo_base + off, pack_half2(lq[0], lq[1]), pack_half2(lq[2], lq[3]));
        }
      };
      const int nslots = w.isC ? 1 : 3;
      // first chunk: the 3 rows before token 0 come from the carried conv state
      if (c0 == 0 && a.states_in) {
        for (int idx = tid; idx < nslots * 3 * 64; idx += kThreads) {
          const int sl = idx / 192, r = (idx / 64) % 3, chn = idx % 64;
          if (!slot_on(sl)) continue;
          const __nv_bfloat16 v = a.conv_in[(w.bi * pr.conv_dim + slot_ch(sl) + chn) * 4 + 1 + r];
          const uint32_t addr = stage + sl * kRawBytes + r * 128 +
                                ((((chn >> 3) ^ r) & 7) << 4) + ((chn & 7) << 1);
          asm volatile("st.shared.b16 [%0], %1;" ::"r"(addr), "h"(__bfloat16_as_ushort(v))
                       : "memory");
        }
        compute_sync();
      }
      // conv + SiLU.  Warp tile: one slot x 4 groups of 8 channels x 8 quads of
      // tokens (lane = group lane % 4, quad lane / 4).  This tile reads the
      // swizzled raw rows, stores u (64 contiguous bytes per token) and, with the
      // channel order of odd groups rotated by 4, stores the swizzled operands
      // without shared-memory bank conflicts.
      //
      // A pair item whose B operand is already in shared memory has exactly one
      // tile per warp: its values stay in registers until the previous item's MMA
      // has completed, so that MMA runs under this item's convolution.  Other pair
      // items first wait for that MMA, then write their operands tile by tile.
      const bool overlap = !w.isC && !freshB;
      if (!w.isC && !overlap && pending) {
        ok = wait_compute(&mbar, (uint32_t)(npair_done & 1), ok);
        if (ok) {
          store_states(pw);
          pending = false;
          ++npair_done;
        }
      }
      const int ntiles = 8 * (w.isC ? 1 : (freshB ? 3 : 2));
      float v[4][8];
      int keep_sl = 0, keep_cg = 0, keep_s0 = 0;
      for (int wt = warp; wt < ntiles; wt += kThreads / 32) {
        const int sl = wt >> 3;
        const int cg = 4 * ((wt >> 2) & 1) + (lane & 3);
        const int s0 = 4 * (8 * (wt & 3) + (lane >> 2));
        keep_sl = sl;
        keep_cg = cg;
        keep_s0 = s0;
        if (sl == 1 && !hasB) {  // missing second head: zero rows 64..127
          if (!overlap) zero_tile(cg, s0);
          continue;
        }
        conv8x4_smem(stage + sl * kRawBytes, s0, cg, wts[st][sl], bss[st][sl], v);
        if (w.isC || sl < 2 || w.pair == 0) store_u(a, w.bi, c0 + s0, slot_ch(sl) + cg * 8, v);
        if (!w.isC && !overlap) put_operands(sl, cg, s0, v);
      }
      if (overlap) {
        if (pending) {
          ok = wait_compute(&mbar, (uint32_t)(npair_done & 1), ok);
          if (ok) {
            store_states(pw);
            pending = false;
            ++npair_done;
          }
        }
        if (ok) {
          if (keep_sl == 1 && !hasB) zero_tile(keep_cg, keep_s0);
          else put_operands(keep_sl, keep_cg, keep_s0, v);
        }
      }
      fence_proxy_async_smem();
      tc_fence_before();
      compute_sync();
      if (tid == 0) mbar_arrive(&empty[st]);  // raw tiles and taps of this stage consumed
      if (w.isC || !ok) continue;
      if (tid == 0) mbar_arrive(&ops_ready);  // the MMA warp issues S = (x o w)^T B
      pending = true;
      pw.bi = w.bi;
      pw.c = w.c;
      pw.hA = hA;
      pw.hasB = hasB;
    }
    if (ok && pending) {
      ok = wait_compute(&mbar, (uint32_t)(npair_done & 1), ok);
      if (ok) {
        store_states(pw);
        pending = false;
      }
    }
    if (!ok && tid == 0) {
      // a wait ran out: let the MMA and the copies already issued land before the
      // CTA frees its tensor memory and exits
      if (pending) mbar_wait_bounded(&mbar, (uint32_t)(npair_done & 1), &g_tc_errors);
      for (int s2 = 0; s2 < 2; ++s2) mbar_wait_bounded(&full[s2], 0, &g_tc_errors);
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) tmem_dealloc(tmem, 64);
}

// ============================================================== state passing
// grid (P*N/1024 + conv-state blocks, H, b): one thread per 4 state elements of
// one p and consecutive n (four independent recurrences, 16-byte loads of the
// chunk states), sequential over chunks.
// Blocks with blockIdx.x >= P*N/1024 (only for h = 0) write the final conv
// state instead: the last 4 raw inputs of [old state | new tokens], in place
// (the chunk-state kernel, which reads the old state, has finished by now).
constexpr int kPassBlocks = (kHP * kNS) / 1024;

__global__ void __launch_bounds__(256) tc_state_pass_kernel(TcArgs a, __nv_bfloat16 *cs) {
  const Problem &pr = a.pr;
  const int h = blockIdx.y;
  const int64_t bi = blockIdx.z;
  if ((int)blockIdx.x >= kPassBlocks) {
    if (h != 0 || cs == nullptr) return;
    const int64_t ch = (int64_t)(blockIdx.x - kPassBlocks) * 256 + threadIdx.x;
    if (ch >= pr.conv_dim) return;
    const int64_t i = bi * pr.conv_dim + ch;
    __nv_bfloat16 v[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const int64_t tau = pr.L - 4 + k;
      if (tau >= 0) v[k] = a.xBC[(bi * pr.L + tau) * a.ld_x + ch];
      else v[k] = a.states_in ? cs[i * 4 + 4 + tau] : __float2bfloat16(0.0f);
    }
#pragma unroll
    for (int k = 0; k < 4; ++k) cs[i * 4 + k] = v[k];
    return;
  }
  // float4 slot j of a head's 64 x 64 state: n = 4 (j / 64) .. +3, p = j % 64 (the
  // chunk-state layout [n/4][p][4]); H_c is stored [n][p] (the MN-major MMA operand)
  const int j = blockIdx.x * 256 + threadIdx.x, n4 = j >> 6, p = j & 63;
  const int64_t hs = (bi * pr.H + h) * (int64_t)(kHP * kNS) + p * kNS + 4 * n4;
  float4 hc = a.states_in ? *reinterpret_cast<const float4 *>(a.ssm_state + hs)
                          : make_float4(0.f, 0.f, 0.f, 0.f);
  const int64_t stride = (int64_t)pr.H * kHP * kNS;
  const float *S = a.S + (bi * a.nch * pr.H + h) * (int64_t)(kHP * kNS) + 4 * j;
  __half *Hc = a.Hc + (bi * a.nch * pr.H + h) * (int64_t)(kHP * kNS) + (4 * n4) * kHP + p;
  const float *ce = a.cum_end + bi * a.nch * pr.H + h;
  auto put = [&](int64_t c) {
    __half *o = Hc + c * stride;
    o[0] = __float2half_rn(hc.x);
    o[kHP] = __float2half_rn(hc.y);
    o[2 * kHP] = __float2half_rn(hc.z);
    o[3 * kHP] = __float2half_rn(hc.w);
  };
  // loads run 8 chunks ahead of the (sequential) recurrence
  constexpr int kAhead = 8;
  int c = 0;
  for (; c + kAhead <= a.nch; c += kAhead) {
    float4 sv[kAhead];
    float d[kAhead];
#pragma unroll
    for (int k = 0; k < kAhead; ++k) {
      sv[k] = *reinterpret_cast<const float4 *>(S + (c + k) * stride);
      d[k] = ce[(int64_t)(c + k) * pr.H];
    }
#pragma unroll
    for (int k = 0; k < kAhead; ++k) {
      put(c + k);
      const float f = expf(d[k]);
      hc = make_float4(fmaf(f, hc.x, sv[k].x), fmaf(f, hc.y, sv[k].y), fmaf(f, hc.z, sv[k].z),
                       fmaf(f, hc.w, sv[k].w));
    }
  }
  for (; c < a.nch; ++c) {
    put(c);
    const float4 sv = *reinterpret_cast<const float4 *>(S + c * stride);
    const float f = expf(ce[(int64_t)c * pr.H]);
    hc = make_float4(fmaf(f, hc.x, sv.x), fmaf(f, hc.y, sv.y), fmaf(f, hc.z, sv.z),
                     fmaf(f, hc.w, sv.w));
  }
  if (a.ssm_state != nullptr) *reinterpret_cast<float4 *>(a.ssm_state + hs) = hc;
}

// ============================================================== chunk output
// Persistent clusters: grid (cs, ncl, 1), cluster (cs, 1, 1).  Cluster k takes
// the units (row, chunk, group) k, k + ncl, ...; its cs CTAs split the group's
// heads.  16 compute warps + 1 TMA producer warp + 1 MMA-issuer warp.  Tiles
// arrive by TMA in 128-byte-swizzled layouts (1024-aligned).  Per head the
// intra-chunk part [CB o L o dt (+D)] x is one K = 128 MMA into the head's TMEM
// columns, and the carried-state part C H_c^T a K = 64 MMA with the C tile
// itself as operand into a shared TMEM accumulator, scaled by exp(cum_t) in
// the epilogue.  The operand A is double-buffered so that the A-build of head
// j + 1 overlaps the MMA of head j; buffer 1 reuses the B tile once CB is
// formed.  The next unit's C and B tiles, its CB product and its first
// x / H_c / z tiles arrive while the current unit exchanges its norm sums and
// writes its output.
constexpr uint32_t kCt = 0;                      // C   [128 t][64 n] fp16     16 KB (u)
constexpr uint32_t kBt = kCt + 16384;            // B   [128 s][64 n] fp16     16 KB (u)
constexpr int kXhStages = 2, kZStages = 2;
constexpr uint32_t kXhBytes = 16384 + 8192;      // per stage: x [128 s][64 p] + H_c [64 n][64 p]
constexpr uint32_t kXh = kBt + 16384;            // x / H_c ring  2 x 24 KB (x at +0, H_c at +16 KB)
constexpr uint32_t kZt = kXh + kXhStages * kXhBytes;  // z ring [128 t][64 p] bf16  2 x 16 KB
constexpr uint32_t kA0 = kZt + kZStages * 16384;      // A buffer 0: [2][128 t][64 k] fp16  32 KB
constexpr uint32_t kA1 = kA0 + 2 * 16384;             // A buffer 1, block 1 (block 0 at kBt)
constexpr uint32_t kYst = kA1 + 16384;                // two output staging tiles  32 KB
constexpr uint32_t kTcOutTiles = kYst + 2 * 16384;    // 192 KB
// output staging: [128 t][64 p] bf16 tiles, idle while a unit writes its output:
// A buffer 0, block 1 of buffer 1 and the two staging tiles
constexpr int kYTiles = 5;
__device__ __forceinline__ uint32_t y_tile(int slot) {
  return slot < 2 ? kA0 + slot * 16384 : (slot == 2 ? kA1 : kYst + (slot - 3) * 16384);
}

// Byte offset of k-block `blk` (CB columns s 0..63, 64..127) of A buffer `buf`.
__device__ __forceinline__ uint32_t a_block(int buf, int blk) {
  return buf == 0 ? kA0 + blk * 16384 : (blk == 0 ? kBt : kA1);
}

struct OutShared {
  float cum2[kMaxHeadsPerCta][kQ];  // cumsum * log2(e)
  float dt[kMaxHeadsPerCta][kQ];
  float beta[kMaxHeadsPerCta][kQ];  // exp(cum_r - cum_s) dt_s, r = end of s's 32-token group
  float betad[kMaxHeadsPerCta][kQ]; // exp(cum_s0 - cum_s) dt_s, s0 = start of s's group
  int span_ok[kMaxHeadsPerCta][4];  // group's log2-decay span <= 60: factorise its diagonal
  float nw[kMaxHeadsPerCta][kHP];   // norm weight of the CTA's channels
  float ss[4][kQ];
  float part[2][16][kQ];            // [unit parity][rank]: partial sums of squares per token
  float mine[kQ];                   // this CTA's partial sums
  float inv[kQ];
  float Dh[kMaxHeadsPerCta];
  uint64_t full_cb, full_xh[kXhStages], empty_xh[kXhStages], full_z[kZStages],
      empty_z[kZStages], a_ready[2], mbar_cb, mbar_mma[2], tiles_free, sums_ready[2], t_free;
  uint32_t tmem_holder;
  int ok_flag;
};

struct OutMaps {
  CUtensorMap u;   // [b][L][conv_dim] fp16, box 64 ch x 128 tokens
  CUtensorMap z;   // [b][L][d_inner] bf16 (row stride ld_z), box 64 x 128
  CUtensorMap hc;  // [rows][64] fp16, box 64 x 64
  CUtensorMap y;   // [b][L][d_inner] bf16, box 64 x 128 (stores)
};

// 16-byte asynchronous store into another rank's shared memory that completes
// 16 transaction bytes on that rank's mbarrier
__device__ __forceinline__ void st_async_v4(uint32_t addr, float4 v, uint32_t bar) {
  asm volatile(
      "st.async.shared::cluster.mbarrier::complete_tx::bytes.v4.b32 [%0], {%1, %2, %3, %4}, [%5];" ::"r"(addr),
      "r"(__float_as_uint(v.x)), "r"(__float_as_uint(v.y)), "r"(__float_as_uint(v.z)),
      "r"(__float_as_uint(v.w)), "r"(bar)
      : "memory");
}
__device__ __forceinline__ uint32_t cluster_addr(const void *p, int r) {
  uint32_t out;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(out) : "r"(smem_u32(p)), "r"(r));
  return out;
}
__device__ __forceinline__ bool mbar_wait_cluster_bounded(uint64_t *bar, uint32_t parity) {
  auto probe = [&]() {
    uint32_t ok;
    asm volatile(
        "{\n .reg .pred p;\n mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2;\n"
        " selp.u32 %0, 1, 0, p;\n}"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity)
        : "memory");
    return ok != 0;
  };
  if (probe()) return true;
  const unsigned long long t0 = globaltimer_ns();
  while (!probe()) {
    if (globaltimer_ns() - t0 > kWaitLimitNs) {
      atomicOr(&g_tc_errors, kErrWaitTimeout);
      return false;
    }
  }
  return true;
}

// Unit n of cluster `cid`: (row bi, chunk c, group g).
__device__ __forceinline__ void out_unit(const Problem &pr, int nch, int ncl, int cid, int n,
                                         int64_t &bi, int &c, int &g) {
  const int64_t u = cid + (int64_t)n * ncl;
  g = (int)(u % pr.G);
  const int64_t bc = u / pr.G;
  c = (int)(bc % nch);
  bi = bc / nch;
}

__global__ void __launch_bounds__(kWsThreads, 1)
    tc_chunk_out_kernel(TcArgs a, const __grid_constant__ OutMaps maps, int ncl) {
  if (test_stall(&g_tc_stall, &g_tc_errors)) return;  // every CTA of every cluster alike
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  int cs, rank;
  asm volatile("mov.u32 %0, %%cluster_nctarank;" : "=r"(cs));
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(rank));
  const Problem &pr = a.pr;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const uint32_t base = (smem_u32(smem_raw) + 1023u) & ~1023u;
  OutShared &sh = *reinterpret_cast<OutShared *>(smem_raw + (base - smem_u32(smem_raw)) +
                                                 kTcOutTiles);
  const int cid = blockIdx.y;
  const int hpg = pr.heads_per_group();
  const int lh0 = rank * a.hpc;
  const int nh = max(0, min(a.hpc, hpg - lh0));  // heads of this CTA in every unit
  const int64_t n_all = pr.batch * (int64_t)a.nch * pr.G;
  const int n_units = n_all > cid ? (int)((n_all - cid + ncl - 1) / ncl) : 0;
  const uint32_t sum_bytes = (uint32_t)cs * kQ * 4;  // partial sums this CTA receives per unit

  if (warp == 0) tmem_alloc(&sh.tmem_holder, 512);
  if (tid == 0) {
    mbar_init(&sh.full_cb, 1);
    for (int k = 0; k < kXhStages; ++k) {
      mbar_init(&sh.full_xh[k], 1);
      mbar_init(&sh.empty_xh[k], 1);  // arrived by tcgen05.commit of the head's MMA
    }
    for (int k = 0; k < kZStages; ++k) {
      mbar_init(&sh.full_z[k], 1);
      mbar_init(&sh.empty_z[k], kThreads);  // every compute thread after its epilogue
    }
    for (int k = 0; k < 2; ++k) {
      mbar_init(&sh.a_ready[k], kThreads);  // every compute thread after its A-build
      mbar_init(&sh.mbar_mma[k], 1);        // MMA of a head that used A buffer k
      // the local arrival carries the bytes the ranks' partial sums complete;
      // units 0 and 1 are armed here, unit n + 2 once unit n's sums are read
      mbar_init(&sh.sums_ready[k], 1);
      mbar_arrive_expect_tx(&sh.sums_ready[k], sum_bytes);
    }
    mbar_init(&sh.mbar_cb, 1);
    mbar_init(&sh.tiles_free, 1);  // a unit's C / B tiles and CB columns no longer read
    mbar_init(&sh.t_free, kThreads);  // every compute thread has read the C H_c^T columns
    fence_mbar_init();
    sh.ok_flag = 1;
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  cluster_arrive_relaxed();  // waited for before the first remote store
  bool started = false;
  const uint32_t tmem = sh.tmem_holder;

  if (warp == kThreads / 32) {
    // ---------------- producer: per unit, x / H_c / z of each head (rings released
    // by the head's MMA and epilogue); after the first head's, the unit's C and B
    // tiles, once the previous unit has finished reading them
    if (lane == 0 && nh > 0) {
      int J = 0;    // heads issued so far (ring position)
      int ncb = 0;  // C / B loads issued
      bool ok = true;
      for (int n = 0; ok && n < n_units; ++n) {
        int64_t bi;
        int c, g;
        out_unit(pr, a.nch, ncl, cid, n, bi, c, g);
        const int h0 = g * hpg + lh0;
        const int c0 = c * kQ;
        for (int j = 0; ok && j < nh; ++j, ++J) {
          const int h = h0 + j, sx = J % kXhStages, sz = J % kZStages;
          ok = J < kXhStages ||
               mbar_wait_bounded(&sh.empty_xh[sx], (uint32_t)((J / kXhStages - 1) & 1), &g_tc_errors);
          if (!ok) break;
          mbar_arrive_expect_tx(&sh.full_xh[sx], kXhBytes);
          tma_load_3d(base + kXh + sx * kXhBytes, &maps.u, h * kHP, c0, (int)bi, &sh.full_xh[sx]);
          tma_load_2d(base + kXh + sx * kXhBytes + 16384, &maps.hc, 0,
                      (int)(((bi * a.nch + c) * pr.H + h) * kHP), &sh.full_xh[sx]);
          ok = J < kZStages ||
               mbar_wait_bounded(&sh.empty_z[sz], (uint32_t)((J / kZStages - 1) & 1), &g_tc_errors);
          if (!ok) break;
          mbar_arrive_expect_tx(&sh.full_z[sz], 16384);
          tma_load_3d(base + kZt + sz * 16384, &maps.z, h * kHP, c0, (int)bi, &sh.full_z[sz]);
          if (j == 0) {
            ok = n == 0 || mbar_wait_bounded(&sh.tiles_free, (uint32_t)((n - 1) & 1), &g_tc_errors);
            if (!ok) break;
            mbar_arrive_expect_tx(&sh.full_cb, 2 * 16384);
            tma_load_3d(base + kCt, &maps.u, (int)(pr.d_inner + (int64_t)(pr.G + g) * kNS), c0,
                        (int)bi, &sh.full_cb);
            tma_load_3d(base + kBt, &maps.u, (int)(pr.d_inner + (int64_t)g * kNS), c0, (int)bi,
                        &sh.full_cb);
            ++ncb;
          }
        }
      }
      // no copy may be in flight when the CTA exits: the last copy into each buffer
      if (ncb > 0) mbar_wait_bounded(&sh.full_cb, (uint32_t)((ncb - 1) & 1), &g_tc_errors);
      for (int k = max(0, J - 2); k < J; ++k) {
        mbar_wait_bounded(&sh.full_xh[k % kXhStages], (uint32_t)((k / kXhStages) & 1), &g_tc_errors);
        mbar_wait_bounded(&sh.full_z[k % kZStages], (uint32_t)((k / kZStages) & 1), &g_tc_errors);
      }
    }
  } else if (warp == kThreads / 32 + 1) {
    // ---------------- MMA issuer: per unit CB once, then per head the K = 128 and K = 64 MMAs
    if (lane == 0 && nh > 0) {
      const uint32_t idesc_cb = umma_idesc_f16(128, 128);
      const uint32_t idesc_mn = umma_idesc_f16(128, 64) | (1u << 16);  // B operand MN-major
      int J = 0;
      bool ok = true;
      for (int n = 0; ok && n < n_units; ++n) {
        // CB = C B^T : M = 128 (t), N = 128 (s), K = 64 (n)
        ok = mbar_wait_bounded(&sh.full_cb, (uint32_t)(n & 1), &g_tc_errors);
        if (!ok) break;
        tc_fence_after();
        for (int kin = 0; kin < 4; ++kin)
          umma_f16(tmem, umma_desc_sw128(base + kCt + kin * 32),
                   umma_desc_sw128(base + kBt + kin * 32), idesc_cb, kin > 0 ? 1u : 0u);
        umma_commit(&sh.mbar_cb);
        for (int j = 0; j < nh; ++j, ++J) {
          ok = mbar_wait_bounded(&sh.a_ready[J & 1], (uint32_t)((J >> 1) & 1), &g_tc_errors) &&
               mbar_wait_bounded(&sh.full_xh[J % kXhStages], (uint32_t)((J / kXhStages) & 1),
                                 &g_tc_errors);
          if (!ok) break;
          tc_fence_after();
          const uint32_t xt = base + kXh + (J % kXhStages) * kXhBytes, ht = xt + 16384;
          // y_j = [CB o L o dt (+D)] x : K = 128 (x [s][p] MN-major)
          for (int ks = 0; ks < 8; ++ks)
            umma_f16(tmem + 128 + 64 * j, umma_desc_sw128(base + a_block(J & 1, ks >> 2) + (ks & 3) * 32),
                     umma_desc_sw128_mn(xt + ks * 2048, 16384), idesc_mn, ks > 0 ? 1u : 0u);
          // T = C H_c^T : K = 64, the C tile as operand (H_c [n][p] MN-major), once the
          // previous head's epilogue has read T
          if (J > 0 && !mbar_wait_bounded(&sh.t_free, (uint32_t)((J - 1) & 1), &g_tc_errors)) {
            ok = false;
            break;
          }
          tc_fence_after();
          for (int kin = 0; kin < 4; ++kin)
            umma_f16(tmem + kTmemT, umma_desc_sw128(base + kCt + kin * 32),
                     umma_desc_sw128_mn(ht + kin * 2048, 8192), idesc_mn, kin > 0 ? 1u : 0u);
          umma_commit(&sh.mbar_mma[J & 1]);
          umma_commit(&sh.empty_xh[J % kXhStages]);  // its x / H_c stage is free once it completes
        }
      }
      if (!ok) sh.ok_flag = 0;
      // no MMA may be in flight when the CTA frees its tensor memory
      if (J > 0) mbar_wait_bounded(&sh.mbar_mma[(J - 1) & 1], (uint32_t)(((J - 1) >> 1) & 1), &g_tc_errors);
    }
  } else {
    // ---------------- compute warps
    const int t = 32 * (warp & 3) + lane, hf = warp >> 2, q = warp & 3;
    const uint32_t lane_off = (uint32_t)(32 * (warp & 3)) << 16;
    float ss_acc = 0.0f;
    bool ok = true;
    int J = 0;  // heads processed so far (ring and A-buffer position)
    auto wait_warp = [&](uint64_t *bar, uint32_t parity) {
      const bool got = ok && mbar_wait_bounded(bar, parity, &g_tc_errors);
      ok = __all_sync(0xffffffffu, got) != 0;
    };

    // epilogue, part 1: gate with silu(z) (z tile in smem), sum of squares, g -> TMEM.
    // Warp w handles rows 32*(w%4) .. +31 and columns 16*(w/4) .. +15 of a head.
    auto epilogue1 = [&](int j, int zslot) {
      float v[16], w[16];
      const uint32_t col = 128 + 64 * j + 16 * hf;
      tmem_ld16(tmem + lane_off + col, v);
      tmem_ld16(tmem + lane_off + kTmemT + 16 * hf, w);
      tc_fence_before();
      mbar_arrive(&sh.t_free);  // the C H_c^T columns may take the next head's product
      const float ec = ex2_approx(sh.cum2[j][t]);  // exp(cum_t)
#pragma unroll
      for (int i = 0; i < 16; ++i) v[i] = fmaf(ec, w[i], v[i]);
      if (!pr.nbg) {
        const uint32_t zt = base + kZt + zslot * 16384;
#pragma unroll
        for (int qq = 0; qq < 2; ++qq) {
          const uint4 raw = ld_shared_v4(zt + sw128_chunk(t, 16 * hf + 8 * qq));
          const __nv_bfloat162 *h2 = reinterpret_cast<const __nv_bfloat162 *>(&raw);
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const float2 f = __bfloat1622float2(h2[i]);
            v[8 * qq + 2 * i] *= silu_fast(f.x);
            v[8 * qq + 2 * i + 1] *= silu_fast(f.y);
          }
        }
      }
#pragma unroll
      for (int i = 0; i < 16; ++i) ss_acc = fmaf(v[i], v[i], ss_acc);
      tmem_st16(tmem + lane_off + col, v);
    };

    // the per-chunk dt and cumsum rows (written by the chunk-state kernel) of a
    // unit's heads: one warp per head, 4 consecutive tokens per lane; the next
    // unit's are loaded before this unit's norm exchange and used after it
    float4 cu = make_float4(0.f, 0.f, 0.f, 0.f), dv = cu;
    auto load_rows = [&](int n) {
      if (warp < nh && n < n_units) {
        int64_t bi;
        int c, g;
        out_unit(pr, a.nch, ncl, cid, n, bi, c, g);
        const int64_t row = (bi * a.nch + c) * pr.H + g * hpg + lh0 + warp;
        cu = reinterpret_cast<const float4 *>(a.cum + row * kQ)[lane];
        dv = reinterpret_cast<const float4 *>(a.dtv + row * kQ)[lane];
      }
    };
    load_rows(0);
    int nw_h0 = -1;  // heads whose norm weights are in shared memory
    for (int n = 0; ok && n < n_units; ++n) {
      int64_t bi;
      int c, g;
      out_unit(pr, a.nch, ncl, cid, n, bi, c, g);
      const int h0 = g * hpg + lh0;
      const int64_t c0 = (int64_t)c * kQ;
      const int par = n & 1;
      // decay terms of the unit's heads
      if (warp < nh) {
        const int j = warp;
        const float cum4[4] = {cu.x, cu.y, cu.z, cu.w}, dt4[4] = {dv.x, dv.y, dv.z, dv.w};
        float c2[4];
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          c2[k] = cum4[k] * kLog2e;
          sh.cum2[j][4 * lane + k] = c2[k];
          sh.dt[j][4 * lane + k] = dt4[k];
        }
        const float c2r = __shfl_sync(0xffffffffu, c2[3], (lane | 7));
        const float c2s0 = __shfl_sync(0xffffffffu, c2[0], (lane & ~7));
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          sh.beta[j][4 * lane + k] = ex2_approx(c2r - c2[k]) * dt4[k];
          sh.betad[j][4 * lane + k] = ex2_approx(fminf(c2s0 - c2[k], 60.0f)) * dt4[k];
        }
        if ((lane & 7) == 7) sh.span_ok[j][lane >> 3] = (c2s0 - c2r) <= 60.0f;
      }
      if (h0 != nw_h0) {  // norm weights and D of the CTA's heads (same in every unit if G = 1)
        for (int i = tid; i < nh * kHP; i += kThreads)
          sh.nw[i / kHP][i % kHP] = a.prm.norm_w[(int64_t)h0 * kHP + i];
        if (tid < nh) sh.Dh[tid] = a.prm.D[h0 + tid];
        nw_h0 = h0;
      }
      if (n > 0 && tid == 0) bulk_wait_read_all();  // the previous unit's output staging
      compute_sync();  // decay terms, weights and D visible; staging tiles free
      ss_acc = 0.0f;

      for (int j = 0; j < nh; ++j, ++J) {
        // A buffer J % 2 is free: the MMA of head J - 2 was waited for by its
        // epilogue in the previous iteration (or the previous unit)
        if (j == 0) {
          wait_warp(&sh.full_cb, (uint32_t)(n & 1));  // the C tile (read for the scaled-C block)
          wait_warp(&sh.mbar_cb, (uint32_t)(n & 1));  // CB in TMEM; the B tile is free (A buffer 1)
        }
        if (!ok) break;
        tc_fence_after();
        const uint32_t abuf = base + a_block(J & 1, 0), abuf1 = base + a_block(J & 1, 1);
      // A_j = CB o exp(cum_t - cum_s) dt_s (s <= t), D on the diagonal;
      // 32-column groups k above the row quarter q are zero, below it the decay
      // factorises as alpha_t beta_s (both <= 1), on it exponentials are direct.
      {
        const int k = hf, s0 = 32 * k;  // this warp's 32-column group
        const uint32_t at = (k >> 1) == 0 ? abuf : abuf1;
        const int kc = 32 * (k & 1);       // column of the group inside its 64-wide block
        const float c2t = sh.cum2[j][t];
        if (k > q) {
#pragma unroll
          for (int qq = 0; qq < 4; ++qq) st_shared_v4(at + sw128_chunk(t, kc + 8 * qq), 0u, 0u, 0u, 0u);
        } else {
          float cb[32];
          tmem_ld32(tmem + lane_off + s0, cb);
          if (k < q) {
            const float alpha = ex2_approx(c2t - sh.cum2[j][s0 + 31]);
            const float4 *b4 = reinterpret_cast<const float4 *>(&sh.beta[j][s0]);
#pragma unroll
            for (int qq = 0; qq < 4; ++qq) {
              const float4 bA = b4[2 * qq], bB = b4[2 * qq + 1];
              const float bb[8] = {bA.x, bA.y, bA.z, bA.w, bB.x, bB.y, bB.z, bB.w};
              uint32_t w4[4];
#pragma unroll
              for (int e = 0; e < 4; ++e) {
                const int sl = 8 * qq + 2 * e;
                w4[e] = pack_half2(cb[sl] * alpha * bb[2 * e], cb[sl + 1] * alpha * bb[2 * e + 1]);
              }
              st_shared_v4(at + sw128_chunk(t, kc + 8 * qq), w4[0], w4[1], w4[2], w4[3]);
            }
          } else if (sh.span_ok[j][k]) {
            // diagonal group, decay span <= 2^60: alpha_t = exp(cum_t - cum_s0) and
            // betad_s = exp(cum_s0 - cum_s) dt_s stay within [2^-60, 2^60]
            const float Dh = sh.Dh[j];
            const float alpha = ex2_approx(c2t - sh.cum2[j][s0]);
            const float4 *b4 = reinterpret_cast<const float4 *>(&sh.betad[j][s0]);
#pragma unroll
            for (int qq = 0; qq < 4; ++qq) {
              const float4 bA = b4[2 * qq], bB = b4[2 * qq + 1];
              const float bb[8] = {bA.x, bA.y, bA.z, bA.w, bB.x, bB.y, bB.z, bB.w};
              uint32_t w4[4];
#pragma unroll
              for (int e = 0; e < 4; ++e) {
                float val[2];
#pragma unroll
                for (int u = 0; u < 2; ++u) {
                  const int sl = 8 * qq + 2 * e + u, s = s0 + sl;
                  float vv = cb[sl] * alpha * bb[2 * e + u];
                  if (s == t) vv += Dh;
                  val[u] = (s <= t) ? vv : 0.0f;
                }
                w4[e] = pack_half2(val[0], val[1]);
              }
              st_shared_v4(at + sw128_chunk(t, kc + 8 * qq), w4[0], w4[1], w4[2], w4[3]);
            }
          } else {
            const float Dh = sh.Dh[j];
            const float4 *c4 = reinterpret_cast<const float4 *>(&sh.cum2[j][s0]);
            const float4 *d4 = reinterpret_cast<const float4 *>(&sh.dt[j][s0]);
#pragma unroll
            for (int qq = 0; qq < 4; ++qq) {
              const float4 cA = c4[2 * qq], cB = c4[2 * qq + 1];
              const float4 dA = d4[2 * qq], dB = d4[2 * qq + 1];
              const float cc[8] = {cA.x, cA.y, cA.z, cA.w, cB.x, cB.y, cB.z, cB.w};
              const float dd[8] = {dA.x, dA.y, dA.z, dA.w, dB.x, dB.y, dB.z, dB.w};
              uint32_t w4[4];
#pragma unroll
              for (int e = 0; e < 4; ++e) {
                float val[2];
#pragma unroll
                for (int u = 0; u < 2; ++u) {
                  const int sl = 8 * qq + 2 * e + u, s = s0 + sl;
                  float vv = cb[sl] * ex2_approx(fminf(c2t - cc[2 * e + u], 0.0f)) * dd[2 * e + u];
                  if (s == t) vv += Dh;
                  val[u] = (s <= t) ? vv : 0.0f;
                }
                w4[e] = pack_half2(val[0], val[1]);
              }
              st_shared_v4(at + sw128_chunk(t, kc + 8 * qq), w4[0], w4[1], w4[2], w4[3]);
            }
          }
        }
      }
        fence_proxy_async_smem();
        tc_fence_before();
        mbar_arrive(&sh.a_ready[J & 1]);
        if (j > 0) {  // epilogue of the previous head overlaps this head's MMA
          const int P1 = J - 1;
          wait_warp(&sh.mbar_mma[P1 & 1], (uint32_t)((P1 >> 1) & 1));
          wait_warp(&sh.full_z[P1 % kZStages], (uint32_t)((P1 / kZStages) & 1));
          if (!ok) break;
          tc_fence_after();
          epilogue1(j - 1, P1 % kZStages);
          mbar_arrive(&sh.empty_z[P1 % kZStages]);
        }
      }
      if (ok && nh > 0) {
        const int P1 = J - 1;
        wait_warp(&sh.mbar_mma[P1 & 1], (uint32_t)((P1 >> 1) & 1));
        wait_warp(&sh.full_z[P1 % kZStages], (uint32_t)((P1 / kZStages) & 1));
        tc_fence_after();
        if (ok) {
          epilogue1(nh - 1, P1 % kZStages);
          mbar_arrive(&sh.empty_z[P1 % kZStages]);
        }
      }
      sh.ss[hf][t] = ss_acc;
      load_rows(n + 1);
      tc_fence_before();
      compute_sync();
      // the unit's C and B tiles and CB columns are no longer read; its last MMA is done
      if (tid == 0) mbar_arrive(&sh.tiles_free);

      // per-token partial sums of this CTA into part[par][rank][*] of every rank
      // (asynchronous stores completing bytes on that rank's barrier)
      if (tid < kQ) sh.mine[tid] = (sh.ss[0][tid] + sh.ss[1][tid]) + (sh.ss[2][tid] + sh.ss[3][tid]);
      if (!started) {
        cluster_wait();  // (arrived at the start) every CTA of the cluster is running
        started = true;
      }
      compute_sync();
      for (int i = tid; i < cs * (kQ / 4); i += kThreads) {
        const int r = i / (kQ / 4), f = i % (kQ / 4);
        st_async_v4(cluster_addr(&sh.part[par][rank][4 * f], r),
                    reinterpret_cast<const float4 *>(sh.mine)[f], cluster_addr(&sh.sums_ready[par], r));
      }
      ok = __all_sync(0xffffffffu,
                      ok && mbar_wait_cluster_bounded(&sh.sums_ready[par], (uint32_t)((n >> 1) & 1))) != 0;
      if (tid < kQ) {
        float tot = 0.0f;
        for (int r = 0; r < cs; ++r) tot += sh.part[par][r][tid];
        sh.inv[tid] = rsqrtf(tot / (float)(hpg * kHP) + pr.eps);
      }
      compute_sync();
      // unit n + 2 uses this parity again; no rank sends it before this CTA has
      // sent unit n + 1's sums, which happens after this point
      if (tid == 0 && n + 2 < n_units) mbar_arrive_expect_tx(&sh.sums_ready[par], sum_bytes);
      tc_fence_after();
      // normalised bf16 output: each head's [128 t][64 p] tile is written into a
      // staging tile (128-byte swizzle) and stored by TMA, which drops the rows past
      // the end of the sequence.  The five staging tiles are the A buffers' blocks
      // other than the B tile (the next unit's B may be arriving there) and two
      // tiles of their own.
      if (ok && sh.ok_flag) {
        const bool t_valid = c0 + t < pr.L;
        const float sc = sh.inv[t];
        for (int j = 0; j < nh; ++j) {
          const int h = h0 + j;
          const int slot = j % kYTiles;
          const uint32_t ybuf = base + y_tile(slot);
          if (j == kYTiles) {  // the store of head 0 has read its tile
            if (tid == 0) bulk_wait_read_le(kYTiles - 1);
            compute_sync();
          }
          float v[16];
          tmem_ld16(tmem + lane_off + 128 + 64 * j + 16 * hf, v);
          const float4 *nw4 = reinterpret_cast<const float4 *>(&sh.nw[j][16 * hf]);
          if (pr.nbg && t_valid) {
            const int64_t row = bi * pr.L + c0 + t;
            const uint4 *zp =
                reinterpret_cast<const uint4 *>(a.z + row * a.ld_z + (int64_t)h * kHP + 16 * hf);
#pragma unroll
            for (int qq = 0; qq < 2; ++qq) {
              const uint4 raw = __ldg(zp + qq);
              const __nv_bfloat162 *h2 = reinterpret_cast<const __nv_bfloat162 *>(&raw);
#pragma unroll
              for (int i = 0; i < 4; ++i) {
                const float2 f = __bfloat1622float2(h2[i]);
                v[8 * qq + 2 * i] *= silu_fast(f.x);
                v[8 * qq + 2 * i + 1] *= silu_fast(f.y);
              }
            }
          }
#pragma unroll
          for (int qq = 0; qq < 2; ++qq) {
            uint32_t o[4];
            const float4 wA = nw4[2 * qq], wB = nw4[2 * qq + 1];
            const float ww[8] = {wA.x, wA.y, wA.z, wA.w, wB.x, wB.y, wB.z, wB.w};
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const int i = 8 * qq + 2 * e;
              const __nv_bfloat162 b2 =
                  __floats2bfloat162_rn(v[i] * sc * ww[2 * e], v[i + 1] * sc * ww[2 * e + 1]);
              o[e] = *reinterpret_cast<const uint32_t *>(&b2);
            }
            st_shared_v4(ybuf + sw128_chunk(t, 16 * hf + 8 * qq), o[0], o[1], o[2], o[3]);
          }
          fence_proxy_async_smem();
          compute_sync();  // head j's tile is complete: store it while the next one is built
          if (tid == 0) {
            tma_store_3d(&maps.y, ybuf, h * kHP, (int)c0, (int)bi);
            bulk_commit();
          }
        }
      }
      // the y columns of TMEM are read before the next unit's MMAs; its A-builds
      // wait for the stores to have read the staging tiles
      tc_fence_before();
      compute_sync();
    }
    if (tid == 0) bulk_wait_read_all();  // the last unit's stores have read their tiles
    if (!ok) sh.ok_flag = 0;
  }
  // every thread: the cluster's start barrier (if not waited for yet), then one
  // more: no CTA exits while another may still store into its shared memory
  __syncwarp();
  if (!started) cluster_wait();
  cluster_arrive_release();
  cluster_wait();
  tc_fence_before();
  __syncthreads();
  if (warp == 0) tmem_dealloc(tmem, 512);
}


// Heads per CTA and cluster size of tc_chunk_out for hpg heads per group.
// Most clusters of `cs` output-kernel CTAs resident at once on the current
// device (cached per device; -1 if the query fails).
int out_max_clusters(int cs);

// Cluster size of the output kernel: every size from ceil(hpg / 6) to 16 whose
// heads per CTA fit tensor memory is scored by the rounds of units its resident
// clusters need times (heads per CTA + a per-unit cost of about 2.5 heads).
void out_choose(int hpg, int64_t units, int *cs, int *hpc, int *ncl) {
  const int lo = (hpg + kMaxHeadsPerCta - 1) / kMaxHeadsPerCta;
  int64_t best = -1;
  for (int c = std::max(lo, 1); c <= 16; ++c) {
    const int h = (hpg + c - 1) / c;
    if (h > kMaxHeadsPerCta) continue;
    const int m = out_max_clusters(c);
    if (m <= 0) continue;
    const int64_t rounds = (units + m - 1) / m;
    const int64_t score = rounds * (2 * h + 5);
    if (best < 0 || score < best) {
      best = score;
      *cs = c;
      *hpc = h;
      *ncl = (int)std::min<int64_t>(units, m);
    }
  }
  if (best < 0) {  // no occupancy answer: the smallest cluster, one per unit
    *cs = std::max(lo, 1);
    *hpc = (hpg + *cs - 1) / *cs;
    *ncl = (int)std::min<int64_t>(units, 65535);
  }
}

struct TcWorkspace {
  float *S, *cum_end, *cum, *dtv;
  __half *Hc, *u;
};

TcWorkspace tc_carve(const Problem &pr, char *base) {
  const int64_t nch = ceil_div(pr.L, kQ);
  const size_t st = (size_t)pr.batch * nch * pr.H * kHP * kNS;
  TcWorkspace w;
  size_t off = 0;
  w.S = reinterpret_cast<float *>(base + off);
  off += align_up(st * 4, 256);
  w.cum_end = reinterpret_cast<float *>(base + off);
  off += align_up((size_t)pr.batch * nch * pr.H * 4, 256);
  w.cum = reinterpret_cast<float *>(base + off);
  off += align_up((size_t)pr.batch * nch * pr.H * kQ * 4, 256);
  w.dtv = reinterpret_cast<float *>(base + off);
  off += align_up((size_t)pr.batch * nch * pr.H * kQ * 4, 256);
  w.Hc = reinterpret_cast<__half *>(base + off);
  off += align_up(st * 2, 256);
  w.u = reinterpret_cast<__half *>(base + off);
  return w;
}

// Number of SMs of the current device (cached per device).
int sm_count() {
  static int cache[64] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 132;
  if (cache[dev] == 0) {
    int n = 0;
    cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    cache[dev] = n > 0 ? n : 132;
  }
  return cache[dev];
}

// cuTensorMapEncodeTiled, fetched once through the runtime (no libcuda link-time dependency).
PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = []() {
    void *p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) !=
            cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      return (PFN_cuTensorMapEncodeTiled_v12000) nullptr;
    return reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  }();
  return fn;
}

// 3-D (channel, token, batch) or 2-D (column, row) map of a 16-bit array with
// 128-byte swizzle; out-of-range boxes read zeros.
bool make_map(CUtensorMap *m, CUtensorMapDataType dt, const void *base, int rank,
              const uint64_t *dims, const uint64_t *strides_bytes, const uint32_t *box) {
  PFN_cuTensorMapEncodeTiled_v12000 enc = tensor_map_encoder();
  if (enc == nullptr) return false;
  cuuint64_t d[3], st[2];
  cuuint32_t b[3], es[3] = {1, 1, 1};
  for (int i = 0; i < rank; ++i) {
    d[i] = dims[i];
    b[i] = box[i];
  }
  for (int i = 0; i + 1 < rank; ++i) st[i] = strides_bytes[i];
  return enc(m, dt, (cuuint32_t)rank, const_cast<void *>(base), d, st, b, es,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_128B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) ==
         CUDA_SUCCESS;
}

constexpr size_t kK1Smem = kK1Tiles + 1024;
constexpr size_t kK3Smem = kTcOutTiles + sizeof(OutShared) + 1024;
static_assert(kK1Smem <= 227 * 1024 && kK3Smem <= 227 * 1024, "shared memory per CTA");

int out_max_clusters(int cs) {
  static int cache[64][17] = {};  // 0: not asked yet
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64 || cs < 1 || cs > 16) return -1;
  int &m = cache[dev][cs];
  if (m == 0) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)cs, 1, 1);
    cfg.blockDim = dim3(kWsThreads, 1, 1);
    cfg.dynamicSmemBytes = kK3Smem;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = (unsigned)cs;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    int v = 0;
    if (cudaOccupancyMaxActiveClusters(&v, tc_chunk_out_kernel, &cfg) != cudaSuccess) {
      cudaGetLastError();  // clear the failed query
      v = -1;
    }
    m = v > 0 ? v : -1;
  }
  return m;
}

}  // namespace

const char *const kPrefillTcStages[] = {"tc_chunk_state", "tc_state_pass", "tc_chunk_out"};
const int kPrefillTcStageCount = 3;

bool prefill_tc_supported(const Problem &pr) {
  const int64_t nch = ceil_div(pr.L, kQ);
  return pr.io == MAMBA2_BF16 && pr.P == kHP && pr.N == kNS && pr.K == 4 &&
         pr.heads_per_group() <= 16 * kMaxHeadsPerCta && pr.L > 0 && nch <= 65535 &&
         pr.L < ((int64_t)1 << 31) && pr.batch * nch * pr.H * kHP < ((int64_t)1 << 31);
}

size_t prefill_tc_workspace(const Problem &pr) {
  const int64_t nch = ceil_div(pr.L, kQ);
  const size_t st = (size_t)pr.batch * nch * pr.H * kHP * kNS;
  return align_up(st * 4, 256) + align_up((size_t)pr.batch * nch * pr.H * 4, 256) +
         2 * align_up((size_t)pr.batch * nch * pr.H * kQ * 4, 256) + align_up(st * 2, 256) +
         align_up((size_t)pr.batch * pr.L * pr.conv_dim * 2, 256);
}

cudaError_t set_prefill_tc_stall(unsigned int v) {
  return cudaMemcpyToSymbol(g_tc_stall, &v, sizeof(v));
}

cudaError_t take_prefill_tc_errors(unsigned int *out) {
  unsigned int v = 0, zero = 0;
  cudaError_t e = cudaMemcpyFromSymbol(&v, g_tc_errors, sizeof(v));
  if (e == cudaSuccess) e = cudaMemcpyToSymbol(g_tc_errors, &zero, sizeof(zero));
  *out = v;
  return e;
}

cudaError_t prefill_tc(const PrefillArgs &pa) {
  const Problem &pr = pa.pr;
  cudaStream_t st = pa.stream;
  TcArgs a;
  a.pr = pr;
  a.prm = pa.prm;
  a.xBC = static_cast<const __nv_bfloat16 *>(pa.xBC);
  a.ld_x = pa.ld_xbc;
  a.z = static_cast<const __nv_bfloat16 *>(pa.z);
  a.ld_z = pa.ld_z;
  a.dt_raw = static_cast<const __nv_bfloat16 *>(pa.dt_raw);
  a.ld_dt = pa.ld_dt;
  a.y = static_cast<__nv_bfloat16 *>(pa.y);
  a.conv_in = static_cast<const __nv_bfloat16 *>(pa.conv_state);
  a.ssm_state = pa.ssm_state;
  a.states_in = pa.states_in;
  a.nch = (int)ceil_div(pr.L, kQ);
  TcWorkspace w = tc_carve(pr, pa.ws);
  a.S = w.S;
  a.cum_end = w.cum_end;
  a.cum = w.cum;
  a.dtv = w.dtv;
  a.Hc = w.Hc;
  a.u = w.u;
  const int hpg = pr.heads_per_group();
  cudaError_t e;
  if (first_use_in_context(0)) {  // attributes belong to the context: set them once in each
    e = cudaFuncSetAttribute(tc_chunk_state_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)kK1Smem);
    if (e != cudaSuccess) return e;
    e = cudaFuncSetAttribute(tc_chunk_out_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)kK3Smem);
    if (e != cudaSuccess) return e;
    e = cudaFuncSetAttribute(tc_chunk_out_kernel, cudaFuncAttributeNonPortableClusterSizeAllowed,
                             1);
    if (e != cudaSuccess) return e;
  }
  int cs = 1, hpc = 1, ncl = 1;
  out_choose(hpg, pr.batch * a.nch * (int64_t)pr.G, &cs, &hpc, &ncl);
  a.hpc = hpc;

  stage_mark(st, 0);
  const int64_t n_items = pr.batch * a.nch * (int64_t)pr.G * ((hpg + 1) / 2 + 1);
  const unsigned g1 = (unsigned)std::min<int64_t>(n_items, sm_count());
  {
    K1Maps m1;
    const uint64_t dx[3] = {(uint64_t)pr.conv_dim, (uint64_t)pr.L, (uint64_t)pr.batch};
    const uint64_t sx[2] = {(uint64_t)pa.ld_xbc * 2, (uint64_t)pr.L * pa.ld_xbc * 2};
    const uint32_t bx[3] = {64, kRawRows, 1};
    if (!make_map(&m1.xbc, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, a.xBC, 3, dx, sx, bx))
      return cudaErrorInvalidValue;
    tc_chunk_state_kernel<<<g1, kK1Threads, kK1Smem, st>>>(a, m1, (int)n_items);
  }
  stage_mark(st, 1);
  dim3 g2((unsigned)(kPassBlocks + ceil_div(pr.conv_dim, 256)), (unsigned)pr.H,
          (unsigned)pr.batch);
  tc_state_pass_kernel<<<g2, 256, 0, st>>>(a, static_cast<__nv_bfloat16 *>(pa.conv_state));
  stage_mark(st, 2);
  {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)cs, (unsigned)ncl, 1);
    cfg.blockDim = dim3(kWsThreads, 1, 1);
    cfg.dynamicSmemBytes = kK3Smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = (unsigned)cs;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    OutMaps maps;
    {
      const uint64_t du[3] = {(uint64_t)pr.conv_dim, (uint64_t)pr.L, (uint64_t)pr.batch};
      const uint64_t su[2] = {(uint64_t)pr.conv_dim * 2, (uint64_t)pr.L * pr.conv_dim * 2};
      const uint32_t bu[3] = {64, kQ, 1};
      const uint64_t dz[3] = {(uint64_t)pr.d_inner, (uint64_t)pr.L, (uint64_t)pr.batch};
      const uint64_t sz[2] = {(uint64_t)pa.ld_z * 2, (uint64_t)pr.L * pa.ld_z * 2};
      const uint64_t dh[2] = {(uint64_t)kNS, (uint64_t)pr.batch * a.nch * pr.H * kHP};
      const uint64_t shc[1] = {(uint64_t)kNS * 2};
      const uint32_t bh[2] = {64, 64};
      const uint64_t dy[3] = {(uint64_t)pr.d_inner, (uint64_t)pr.L, (uint64_t)pr.batch};
      const uint64_t sy[2] = {(uint64_t)pr.d_inner * 2, (uint64_t)pr.L * pr.d_inner * 2};
      if (!make_map(&maps.u, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, a.u, 3, du, su, bu) ||
          !make_map(&maps.z, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, a.z, 3, dz, sz, bu) ||
          !make_map(&maps.hc, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, a.Hc, 2, dh, shc, bh) ||
          !make_map(&maps.y, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, a.y, 3, dy, sy, bu))
        return cudaErrorInvalidValue;
    }
    e = cudaLaunchKernelEx(&cfg, tc_chunk_out_kernel, a, maps, ncl);
    if (e != cudaSuccess) return e;
  }
  stage_mark(st, 3);
  return cudaGetLastError();
}

}  // namespace m2
