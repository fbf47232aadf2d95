// Backward pass of the mixer-core prefill (training).  The Zamba2 layers
// support gradient checkpointing ("Zamba2 hybrid architecture in
// Transformers", qwbw.cn, section 三), so the forward is recomputed here from
// the layer's inputs and then differentiated; nothing is kept from a
// forward call.
//
// Forward (the definitions of the prefill, per batch row):
//   pre_t = b + sum_k w_k in_{t-3+k},  u_t = silu(pre_t)  -> x | B | C   (conv, 4 taps)
//   dt_t  = softplus(dt_raw_t + dt_bias),  a_t = exp(dt_t A)
//   h_t   = a_t h_{t-1} + dt_t x_t B_t^T,  ypre_t = h_t C_t + D x_t       (per head)
//   y_t   = gated group RMSNorm of ypre_t with z_t
// Backward, in the reverse order, for the loss sum(y dy) + sum(h_L dh_L):
//   bwd_prologue    u and dt again (fp32);
//   bwd_scan_fwd    h_t of every token kept in the workspace, and ypre;
//   bwd_norm        dypre, dz, and the per-token terms of dnorm_w;
//   bwd_scan_rev    reverse over tokens with dh in registers: dx, and per-warp
//                   shares of dB, dC and ddt, dA, dD, dh_0;
//   bwd_reduce_bc   dB, dC over the heads of a group and their warps; ddt;
//   bwd_dt          ddt_raw and the per-token terms of ddt_bias;
//   bwd_conv        through the SiLU and the conv: dxBC, dconv_state, dw, db;
//   col_sum         sums of the per-token terms over the tokens.
// Everything is fp32 on CUDA cores.  The scan kernels give each warp of a
// head's block rows p = warp, warp + 16, ... of the state and each lane the
// columns n = lane, lane + 32, ...: sums over n are warp shuffles, and the
// sums over p that span warps are written per warp and added afterwards, so
// no kernel synchronises a block inside its token loop (a block barrier per
// token cost more than the separate sum).
#include <algorithm>
#include <type_traits>

#include "common.cuh"

namespace m2 {
namespace {

constexpr int kScanWarps = 16;  // warps of a head's block in the scan kernels (P >= 16)

__device__ __forceinline__ float sigmoid_f(float s) { return 1.0f / (1.0f + expf(-s)); }
// d silu(s) / ds = sigmoid(s) (1 + s (1 - sigmoid(s)))
__device__ __forceinline__ float dsilu_f(float s) {
  const float g = sigmoid_f(s);
  return g * (1.0f + s * (1.0f - g));
}

// Raw conv input in_tau of row bi, channel c: token tau of xBC, or for tau < 0
// entry 4 + tau of the carried conv state (zero without one).
template <typename T>
__device__ __forceinline__ float conv_in(const T *xBC, int64_t ld_x, const T *cs, int64_t L,
                                         int64_t conv_dim, int64_t bi, int64_t c, int64_t tau) {
  if (tau >= 0) return to_f(xBC[(bi * L + tau) * ld_x + c]);
  if (cs == nullptr) return 0.0f;
  return to_f(cs[(bi * conv_dim + c) * 4 + 4 + tau]);
}

// u = silu(conv) for every (row, token, channel); dt = softplus(dt_raw + dt_bias).
template <typename T>
__global__ void bwd_prologue_kernel(Problem pr, mamba2_params prm, const T *xBC, int64_t ld_x,
                                    const T *dt_raw, int64_t ld_dt, const T *cs, float *u,
                                    float *dtv) {
  const int64_t n = pr.batch * pr.L * pr.conv_dim;
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < n;
       i += (int64_t)gridDim.x * blockDim.x) {
    const int64_t c = i % pr.conv_dim, bt = i / pr.conv_dim, t = bt % pr.L, bi = bt / pr.L;
    float pre = prm.conv_b[c];
#pragma unroll
    for (int k = 0; k < 4; ++k)
      pre += prm.conv_w[c * 4 + k] * conv_in(xBC, ld_x, cs, pr.L, pr.conv_dim, bi, c, t - 3 + k);
    u[i] = silu_f(pre);
  }
  const int64_t nd = pr.batch * pr.L * pr.H;
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < nd;
       i += (int64_t)gridDim.x * blockDim.x) {
    const int64_t h = i % pr.H, bt = i / pr.H;
    dtv[i] = softplus_f(to_f(dt_raw[bt * ld_dt + h]) + prm.dt_bias[h]);
  }
}

// The per-token inputs of one head that a warp of the scan kernels reads: dt,
// the lane's B and C columns, and x (and, backwards, dypre) of the warp's rows.
template <int ROWS, int COLS>
struct ScanTok {
  float dt, bv[COLS], cv[COLS], x[ROWS], dy[ROWS];
};
template <int ROWS, int COLS>
__device__ __forceinline__ void scan_load_tok(const Problem &pr, const float *__restrict__ u,
                                              const float *__restrict__ dtv,
                                              const float *__restrict__ dypre, int64_t bi,
                                              int h, int g, int gw, int nwh, int lane,
                                              int64_t t, ScanTok<ROWS, COLS> &k) {
  const int N = pr.N;
  const float *ut = u + (bi * pr.L + t) * pr.conv_dim;
  k.dt = dtv[(bi * pr.L + t) * pr.H + h];
#pragma unroll
  for (int j = 0; j < COLS; ++j) {
    const int n = lane + 32 * j;
    k.bv[j] = n < N ? ut[pr.d_inner + (int64_t)g * N + n] : 0.0f;
    k.cv[j] = n < N ? ut[pr.d_inner + (int64_t)(pr.G + g) * N + n] : 0.0f;
  }
#pragma unroll
  for (int r = 0; r < ROWS; ++r) {
    const int p = gw + nwh * r;
    k.x[r] = ut[(int64_t)h * pr.P + p];
    k.dy[r] = dypre != nullptr ? dypre[(bi * pr.L + t) * pr.d_inner + (int64_t)h * pr.P + p]
                               : 0.0f;
  }
}

// The warp layout of the scan kernels: a head's P / ROWS warps take rows p = gw,
// gw + P / ROWS, ... (gw the warp's index in the head), split over blocks of
// WARPS warps (grid.x = heads x blocks per head); each lane takes columns
// n = lane, lane + 32, ... (COLS = ceil(N / 32)).
//
// The recurrence forward: every row is independent, so one row per warp and
// several blocks per head keep all SMs busy; the next token's inputs are loaded
// while this one is computed.  The state after every token into hs
// [b][H][L][P][N]; ypre [b][L][d_inner].
template <int ROWS, int COLS, int WARPS>
__global__ void __launch_bounds__(32 * WARPS)
    bwd_scan_fwd_kernel(Problem pr, mamba2_params prm, const float *__restrict__ u,
                        const float *__restrict__ dtv, const float *__restrict__ h0,
                        float *__restrict__ hs, float *__restrict__ ypre) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nwh = pr.P / ROWS, bph = nwh / WARPS;
  const int h = blockIdx.x / bph, gw = (blockIdx.x % bph) * WARPS + warp;
  const int64_t bi = blockIdx.y;
  const int P = pr.P, N = pr.N, g = h / pr.heads_per_group();
  const float A = prm.A[h], D = prm.D[h];
  float st[ROWS][COLS];
  const int64_t head = bi * pr.H + h;
#pragma unroll
  for (int r = 0; r < ROWS; ++r)
#pragma unroll
    for (int j = 0; j < COLS; ++j) {
      const int p = gw + nwh * r, n = lane + 32 * j;
      st[r][j] = (n < N && h0 != nullptr) ? h0[(head * P + p) * N + n] : 0.0f;
    }
  ScanTok<ROWS, COLS> cur, nxt;
  if (pr.L > 0) scan_load_tok(pr, u, dtv, nullptr, bi, h, g, gw, nwh, lane, 0, cur);
  for (int64_t t = 0; t < pr.L; ++t) {
    if (t + 1 < pr.L) scan_load_tok(pr, u, dtv, nullptr, bi, h, g, gw, nwh, lane, t + 1, nxt);
    const float a = expf(cur.dt * A);
    float *hst = hs + (head * pr.L + t) * (int64_t)(P * N);
#pragma unroll
    for (int r = 0; r < ROWS; ++r) {
      const int p = gw + nwh * r;
      const float xdt = cur.x[r] * cur.dt;
      float acc = 0.0f;
#pragma unroll
      for (int j = 0; j < COLS; ++j) {
        const int n = lane + 32 * j;
        st[r][j] = fmaf(a, st[r][j], xdt * cur.bv[j]);
        if (n < N) hst[p * N + n] = st[r][j];
        acc = fmaf(st[r][j], cur.cv[j], acc);
      }
      acc = warp_sum(acc);
      if (lane == 0) ypre[(bi * pr.L + t) * pr.d_inner + (int64_t)h * P + p] = acc + D * cur.x[r];
    }
    cur = nxt;
  }
}

// Gated group RMSNorm backward, one block per (row, token): dypre, dz (io type)
// and the token's dnorm_w terms (dwt [b * L][d_inner]).
template <typename T>
__global__ void bwd_norm_kernel(Problem pr, mamba2_params prm, const float *ypre, const T *z,
                                int64_t ld_z, const T *dy, float *dypre, T *dz, float *dwt) {
  __shared__ float red[33];
  const int64_t bt = blockIdx.x;
  const int64_t gs = pr.d_inner / pr.G;
  const float *yp = ypre + bt * pr.d_inner;
  const T *zt = z + bt * ld_z;
  const T *dyt = dy + bt * pr.d_inner;
  for (int g = 0; g < pr.G; ++g) {
    float ss = 0.0f, sd = 0.0f;  // sum v^2 and sum w dout' v over the group
    for (int64_t i = threadIdx.x; i < gs; i += blockDim.x) {
      const int64_t c = g * gs + i;
      const float zs = to_f(zt[c]), s = silu_f(zs);
      const float v = pr.nbg ? yp[c] : yp[c] * s;
      const float dop = pr.nbg ? to_f(dyt[c]) * s : to_f(dyt[c]);
      ss = fmaf(v, v, ss);
      sd = fmaf(prm.norm_w[c] * dop, v, sd);
    }
    ss = block_sum(ss, red);
    sd = block_sum(sd, red);
    const float r = rsqrtf(ss / (float)gs + pr.eps), r3n = r * r * r / (float)gs;
    for (int64_t i = threadIdx.x; i < gs; i += blockDim.x) {
      const int64_t c = g * gs + i;
      const float zs = to_f(zt[c]), s = silu_f(zs), ds = dsilu_f(zs);
      const float v = pr.nbg ? yp[c] : yp[c] * s;
      const float dout = to_f(dyt[c]), dop = pr.nbg ? dout * s : dout;
      const float dv = r * prm.norm_w[c] * dop - r3n * v * sd;
      dwt[bt * pr.d_inner + c] = dop * v * r;
      if (pr.nbg) {
        dypre[bt * pr.d_inner + c] = dv;
        dz[bt * pr.d_inner + c] = from_f<T>(dout * v * r * prm.norm_w[c] * ds);
      } else {
        dypre[bt * pr.d_inner + c] = dv * s;
        dz[bt * pr.d_inner + c] = from_f<T>(dv * yp[c] * ds);
      }
    }
  }
}

// The recurrence backward, reverse over tokens, in the warp layout above with
// kScanWarps warps per head (ROWS = P / kScanWarps); the inputs and the stored
// states of the next token (t - 1) are loaded while token t is computed.
// du gets dx (x channels); each warp's shares of dB (times dt), dC and ddt of
// every token go to pbc [b][L][2][H][warp][N] and pdt [b][L][H][warp] (token
// major, so that the sums over a group's heads and warps read one contiguous
// span per token); dA, dD by atomics; dh0 the gradient of the initial state.
template <int ROWS, int COLS, int WARPS>
__global__ void __launch_bounds__(32 * WARPS)
    bwd_scan_rev_kernel(Problem pr, mamba2_params prm, const float *__restrict__ u,
                        const float *__restrict__ dtv, const float *__restrict__ h0,
                        const float *__restrict__ hs, const float *__restrict__ dypre,
                        const float *__restrict__ dhL, float *__restrict__ du,
                        float *__restrict__ pbc, float *__restrict__ pdt, float *dA, float *dD,
                        float *__restrict__ dh0) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nwh = pr.P / ROWS, bph = nwh / WARPS;  // nwh = kScanWarps
  const int h = blockIdx.x / bph, gw = (blockIdx.x % bph) * WARPS + warp;
  const int64_t bi = blockIdx.y;
  const int P = pr.P, N = pr.N, g = h / pr.heads_per_group();
  const float A = prm.A[h], D = prm.D[h];
  const int64_t head = bi * pr.H + h;
  const int64_t PN = (int64_t)P * N;
  // the state before token t (h_{t-1}): from hs, or the initial state (zero without one)
  auto load_prev = [&](int64_t t, float (&hp)[ROWS][COLS]) {
    const float *src = t > 0 ? hs + (head * pr.L + t - 1) * PN
                             : (h0 != nullptr ? h0 + head * PN : nullptr);
#pragma unroll
    for (int r = 0; r < ROWS; ++r)
#pragma unroll
      for (int j = 0; j < COLS; ++j) {
        const int p = gw + nwh * r, n = lane + 32 * j;
        hp[r][j] = (src != nullptr && n < N) ? src[p * N + n] : 0.0f;
      }
  };
  float dh[ROWS][COLS], hcur[ROWS][COLS], hprv[ROWS][COLS], hnx[ROWS][COLS];
#pragma unroll
  for (int r = 0; r < ROWS; ++r)
#pragma unroll
    for (int j = 0; j < COLS; ++j) {
      const int p = gw + nwh * r, n = lane + 32 * j;
      dh[r][j] = (dhL != nullptr && n < N) ? dhL[(head * P + p) * N + n] : 0.0f;
    }
  float dA_acc = 0.0f, dD_acc = 0.0f;
  ScanTok<ROWS, COLS> cur, nxt;
  if (pr.L > 0) {
    scan_load_tok(pr, u, dtv, dypre, bi, h, g, gw, nwh, lane, pr.L - 1, cur);
    load_prev(pr.L, hcur);      // h_{L-1}
    load_prev(pr.L - 1, hprv);  // h_{L-2}
  }
  for (int64_t t = pr.L - 1; t >= 0; --t) {
    if (t > 0) {  // token t - 1: its inputs and the state before it
      scan_load_tok(pr, u, dtv, dypre, bi, h, g, gw, nwh, lane, t - 1, nxt);
      load_prev(t - 1, hnx);
    }
    const float dt = cur.dt, a = expf(dt * A);
    float dbp[COLS], dcp[COLS];
#pragma unroll
    for (int j = 0; j < COLS; ++j) {
      dbp[j] = 0.0f;
      dcp[j] = 0.0f;
    }
    float ddt_dir = 0.0f, da = 0.0f;  // sum dh x B, sum dh h_{t-1}
#pragma unroll
    for (int r = 0; r < ROWS; ++r) {
      const int p = gw + nwh * r;
      const float x = cur.x[r], dyp = cur.dy[r];
      float sb = 0.0f;
#pragma unroll
      for (int j = 0; j < COLS; ++j) {
        dh[r][j] = fmaf(dyp, cur.cv[j], dh[r][j]);  // y_t = h_t C_t + D x_t
        dcp[j] = fmaf(dyp, hcur[r][j], dcp[j]);
        sb = fmaf(dh[r][j], cur.bv[j], sb);
        dbp[j] = fmaf(dh[r][j], x, dbp[j]);
        da = fmaf(dh[r][j], hprv[r][j], da);
      }
      sb = warp_sum(sb);
      ddt_dir = fmaf(x, sb, ddt_dir);
      if (lane == 0) {
        du[(bi * pr.L + t) * pr.conv_dim + (int64_t)h * P + p] = fmaf(D, dyp, dt * sb);
        dD_acc = fmaf(dyp, x, dD_acc);
      }
#pragma unroll
      for (int j = 0; j < COLS; ++j) dh[r][j] *= a;  // -> dL/dh_{t-1}
    }
    da = warp_sum(da);
    // this warp's shares of dB (times dt) and dC, and of ddt
    const int64_t bt = bi * pr.L + t;
    float *pb = pbc + ((bt * 2 * pr.H + h) * kScanWarps + gw) * N;
    const int64_t cstride = (int64_t)pr.H * kScanWarps * N;  // B -> C
#pragma unroll
    for (int j = 0; j < COLS; ++j) {
      const int n = lane + 32 * j;
      if (n < N) {
        pb[n] = dt * dbp[j];
        pb[cstride + n] = dcp[j];
      }
    }
    if (lane == 0) {
      pdt[(bt * pr.H + h) * kScanWarps + gw] = ddt_dir + da * a * A;
      dA_acc = fmaf(da * a, dt, dA_acc);
    }
    cur = nxt;
#pragma unroll
    for (int r = 0; r < ROWS; ++r)
#pragma unroll
      for (int j = 0; j < COLS; ++j) {
        hcur[r][j] = hprv[r][j];
        hprv[r][j] = hnx[r][j];
      }
  }
  if (lane == 0) {
    atomicAdd(dA + h, dA_acc);
    atomicAdd(dD + h, dD_acc);
  }
  if (dh0 != nullptr) {
#pragma unroll
    for (int r = 0; r < ROWS; ++r)
#pragma unroll
      for (int j = 0; j < COLS; ++j) {
        const int p = gw + nwh * r, n = lane + 32 * j;
        if (n < N) dh0[(head * P + p) * N + n] = dh[r][j];
      }
  }
}

// dB, dC per (row, token, group, n): the group's heads and their warps added in
// order; ddt per (row, token, head): its warps added.
__global__ void bwd_reduce_bc_kernel(Problem pr, const float *pbc, const float *pdt, float *du,
                                     float *ddt) {
  const int N = pr.N, hpg = pr.heads_per_group();
  const int64_t nbc = pr.batch * pr.L * pr.G * 2 * N;
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < nbc;
       i += (int64_t)gridDim.x * blockDim.x) {
    const int n = (int)(i % N);
    int64_t r = i / N;
    const int which = (int)(r % 2);  // 0: B, 1: C
    r /= 2;
    const int g = (int)(r % pr.G);
    const int64_t bt = r / pr.G;
    // the group's heads and their warps: hpg * kScanWarps rows of N, contiguous
    const float *src = pbc + ((bt * 2 + which) * pr.H + (int64_t)g * hpg) * kScanWarps * N + n;
    float s = 0.0f;
    for (int k = 0; k < hpg * kScanWarps; ++k) s += src[(int64_t)k * N];
    du[bt * pr.conv_dim + pr.d_inner + (int64_t)(which * pr.G + g) * N + n] = s;
  }
  const int64_t nd = pr.batch * pr.L * pr.H;
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < nd;
       i += (int64_t)gridDim.x * blockDim.x) {
    float s = 0.0f;
#pragma unroll
    for (int w = 0; w < kScanWarps; ++w) s += pdt[i * kScanWarps + w];
    ddt[i] = s;
  }
}

// ddt_raw = ddt * sigmoid(dt_raw + dt_bias) (io type), and the same value as the
// token's ddt_bias term (dbt [b * L][H]).
template <typename T>
__global__ void bwd_dt_kernel(Problem pr, mamba2_params prm, const T *dt_raw, int64_t ld_dt,
                              const float *ddt, T *ddt_raw, float *dbt) {
  const int64_t nd = pr.batch * pr.L * pr.H;
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < nd;
       i += (int64_t)gridDim.x * blockDim.x) {
    const int64_t h = i % pr.H, bt = i / pr.H;
    const float v = ddt[i] * sigmoid_f(to_f(dt_raw[bt * ld_dt + h]) + prm.dt_bias[h]);
    ddt_raw[i] = from_f<T>(v);
    dbt[i] = v;
  }
}

// Through SiLU and the conv for (row, channel, segment of kSeg tokens):
// dpre_t = du_t silu'(pre_t); d in_tau = sum_k w_k dpre_{tau + 3 - k}, for the
// tokens of the segment (dxBC) and, in the first segment, the three carried
// inputs (dconv_state, column 0 unused: zero); dw_k and db by atomics.
constexpr int kSeg = 64;
template <typename T>
__global__ void bwd_conv_kernel(Problem pr, mamba2_params prm, const T *xBC, int64_t ld_x,
                                const T *cs, const float *du, T *dxbc, T *dcs, float *dw,
                                float *db) {
  const int64_t nseg = (pr.L + kSeg - 1) / kSeg;
  const int64_t n = pr.batch * nseg * pr.conv_dim;
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < n;
       i += (int64_t)gridDim.x * blockDim.x) {
    const int64_t c = i % pr.conv_dim, r = i / pr.conv_dim, sg = r % nseg, bi = r / nseg;
    const float w0 = prm.conv_w[c * 4], w1 = prm.conv_w[c * 4 + 1], w2 = prm.conv_w[c * 4 + 2],
                w3 = prm.conv_w[c * 4 + 3], bias = prm.conv_b[c];
    const int64_t t0 = sg * kSeg, t1 = min(pr.L, t0 + kSeg);
    // dpre of tokens t0 .. t1 + 2 feed d in_tau for tau in [t0 - 3, t1): the window
    // of the last three dpre values rolls forward with tau
    auto dpre_at = [&](int64_t t) -> float {
      if (t < 0 || t >= pr.L) return 0.0f;
      float pre = bias;
      pre += w0 * conv_in(xBC, ld_x, cs, pr.L, pr.conv_dim, bi, c, t - 3);
      pre += w1 * conv_in(xBC, ld_x, cs, pr.L, pr.conv_dim, bi, c, t - 2);
      pre += w2 * conv_in(xBC, ld_x, cs, pr.L, pr.conv_dim, bi, c, t - 1);
      pre += w3 * conv_in(xBC, ld_x, cs, pr.L, pr.conv_dim, bi, c, t);
      return du[(bi * pr.L + t) * pr.conv_dim + c] * dsilu_f(pre);
    };
    float gw0 = 0.f, gw1 = 0.f, gw2 = 0.f, gw3 = 0.f, gb = 0.f;
    // weight and bias gradients over the segment's own tokens
    for (int64_t t = t0; t < t1; ++t) {
      const float d = dpre_at(t);
      gb += d;
      gw0 = fmaf(d, conv_in(xBC, ld_x, cs, pr.L, pr.conv_dim, bi, c, t - 3), gw0);
      gw1 = fmaf(d, conv_in(xBC, ld_x, cs, pr.L, pr.conv_dim, bi, c, t - 2), gw1);
      gw2 = fmaf(d, conv_in(xBC, ld_x, cs, pr.L, pr.conv_dim, bi, c, t - 1), gw2);
      gw3 = fmaf(d, conv_in(xBC, ld_x, cs, pr.L, pr.conv_dim, bi, c, t), gw3);
    }
    atomicAdd(dw + c * 4, gw0);
    atomicAdd(dw + c * 4 + 1, gw1);
    atomicAdd(dw + c * 4 + 2, gw2);
    atomicAdd(dw + c * 4 + 3, gw3);
    atomicAdd(db + c, gb);
    // input gradients: in_tau feeds pre_{tau + 3 - k} through tap k
    const int64_t tau0 = sg == 0 ? -3 : t0;
    for (int64_t tau = tau0; tau < t1; ++tau) {
      const float g = w0 * dpre_at(tau + 3) + w1 * dpre_at(tau + 2) + w2 * dpre_at(tau + 1) +
                      w3 * dpre_at(tau);
      if (tau >= 0) dxbc[(bi * pr.L + tau) * pr.conv_dim + c] = from_f<T>(g);
      else if (dcs != nullptr) dcs[(bi * pr.conv_dim + c) * 4 + 4 + tau] = from_f<T>(g);
    }
    if (sg == 0 && dcs != nullptr) dcs[(bi * pr.conv_dim + c) * 4] = from_f<T>(0.0f);
  }
}

// out[c] = sum over rows r of m[r][c] (m [rows][cols], fp32), rows split over
// blockIdx.y with atomics.
__global__ void col_sum_kernel(const float *m, int64_t rows, int64_t cols, float *out) {
  const int64_t c = blockIdx.x * (int64_t)blockDim.x + threadIdx.x;
  if (c >= cols) return;
  const int64_t per = (rows + gridDim.y - 1) / gridDim.y;
  const int64_t r0 = blockIdx.y * per, r1 = min(rows, r0 + per);
  float s = 0.0f;
  for (int64_t r = r0; r < r1; ++r) s += m[r * cols + c];
  if (r1 > r0) atomicAdd(out + c, s);
}

// Calls f(rows, cols) with the compile-time warp layout of the scan kernels for
// P (16, 32, 64: rows P / 16 per warp) and N (16 .. 128: ceil(N / 32) per lane).
template <typename F>
void launch_scan(const Problem &pr, F f) {
  auto with_rows = [&](auto cols) {
    switch (pr.P / kScanWarps) {
      case 1: f(std::integral_constant<int, 1>(), cols); break;
      case 2: f(std::integral_constant<int, 2>(), cols); break;
      default: f(std::integral_constant<int, 4>(), cols); break;
    }
  };
  switch ((pr.N + 31) / 32) {
    case 1: with_rows(std::integral_constant<int, 1>()); break;
    case 2: with_rows(std::integral_constant<int, 2>()); break;
    default: with_rows(std::integral_constant<int, 4>()); break;
  }
}

struct BwdWorkspace {
  float *u, *dtv, *hs, *ypre, *dypre, *du, *pbc, *pdt, *ddt, *tok;
};

size_t bwd_carve(const Problem &pr, char *base, BwdWorkspace *w) {
  size_t off = 0;
  auto take = [&](size_t n) -> float * {
    float *p = base == nullptr ? nullptr : reinterpret_cast<float *>(base + off);
    off += align_up(n * 4, 256);
    return p;
  };
  const size_t bl = (size_t)pr.batch * pr.L;
  BwdWorkspace t;
  t.u = take(bl * pr.conv_dim);
  t.dtv = take(bl * pr.H);
  t.hs = take(bl * pr.H * pr.P * pr.N);
  t.ypre = take(bl * pr.d_inner);
  t.dypre = take(bl * pr.d_inner);
  t.du = take(bl * pr.conv_dim);
  t.pbc = take(bl * 2 * pr.H * kScanWarps * pr.N);
  t.pdt = take(bl * pr.H * kScanWarps);
  t.ddt = take(bl * pr.H);
  t.tok = take(bl * std::max<int64_t>(pr.d_inner, pr.H));  // per-token terms of a sum
  if (w != nullptr) *w = t;
  return off;
}

template <typename T>
cudaError_t run_backward(const BackwardArgs &a) {
  const Problem &pr = a.pr;
  cudaStream_t st = a.stream;
  BwdWorkspace w;
  bwd_carve(pr, a.ws, &w);
  const T *xBC = static_cast<const T *>(a.xBC), *z = static_cast<const T *>(a.z),
          *dt_raw = static_cast<const T *>(a.dt_raw), *dy = static_cast<const T *>(a.dy),
          *cs = static_cast<const T *>(a.conv_state_in);
  const int64_t bl = pr.batch * pr.L;
  auto grid_for = [](int64_t n) { return (unsigned)std::min<int64_t>((n + 255) / 256, 1 << 20); };
  cudaError_t e;
  for (auto p : {std::make_pair((void *)a.d_conv_w, (size_t)pr.conv_dim * 4),
                 std::make_pair((void *)a.d_conv_b, (size_t)pr.conv_dim),
                 std::make_pair((void *)a.d_dt_bias, (size_t)pr.H),
                 std::make_pair((void *)a.d_A, (size_t)pr.H),
                 std::make_pair((void *)a.d_D, (size_t)pr.H),
                 std::make_pair((void *)a.d_norm_w, (size_t)pr.d_inner)}) {
    e = cudaMemsetAsync(p.first, 0, p.second * sizeof(float), st);
    if (e != cudaSuccess) return e;
  }
  if (bl == 0) {  // no token: h_L = h_0, every other gradient is zero
    if (a.d_ssm_state_in != nullptr) {
      const size_t sb = (size_t)pr.batch * pr.H * pr.P * pr.N * sizeof(float);
      e = a.d_ssm_state_out != nullptr
              ? cudaMemcpyAsync(a.d_ssm_state_in, a.d_ssm_state_out, sb, cudaMemcpyDeviceToDevice, st)
              : cudaMemsetAsync(a.d_ssm_state_in, 0, sb, st);
      if (e != cudaSuccess) return e;
    }
    if (a.d_conv_state_in != nullptr) {
      e = cudaMemsetAsync(a.d_conv_state_in, 0, (size_t)pr.batch * pr.conv_dim * 4 * sizeof(T), st);
      if (e != cudaSuccess) return e;
    }
    return cudaGetLastError();
  }
  NvtxRange r("prefill_backward");
  stage_mark(st, 0);
  bwd_prologue_kernel<T><<<grid_for(bl * pr.conv_dim), 256, 0, st>>>(pr, a.prm, xBC, a.ld_xbc,
                                                                      dt_raw, a.ld_dt, cs, w.u,
                                                                      w.dtv);
  stage_mark(st, 1);
  launch_scan(pr, [&](auto, auto cols) {  // one row per warp, 16-warp blocks
    const dim3 grid((unsigned)(pr.H * (pr.P / 16)), (unsigned)pr.batch);
    bwd_scan_fwd_kernel<1, decltype(cols)::value, 16>
        <<<grid, 32 * 16, 0, st>>>(pr, a.prm, w.u, w.dtv, a.ssm_state_in, w.hs, w.ypre);
  });
  stage_mark(st, 2);
  bwd_norm_kernel<T><<<(unsigned)bl, 256, 0, st>>>(pr, a.prm, w.ypre, z, a.ld_z, dy, w.dypre,
                                                   static_cast<T *>(a.d_z), w.tok);
  stage_mark(st, 3);
  col_sum_kernel<<<dim3((unsigned)ceil_div(pr.d_inner, 256), 64), 256, 0, st>>>(
      w.tok, bl, pr.d_inner, a.d_norm_w);
  stage_mark(st, 4);
  launch_scan(pr, [&](auto rows, auto cols) {  // kScanWarps warps per head, 4-warp blocks
    const dim3 grid((unsigned)(pr.H * (kScanWarps / 4)), (unsigned)pr.batch);
    bwd_scan_rev_kernel<decltype(rows)::value, decltype(cols)::value, 4>
        <<<grid, 32 * 4, 0, st>>>(pr, a.prm, w.u, w.dtv, a.ssm_state_in, w.hs, w.dypre,
                                  a.d_ssm_state_out, w.du, w.pbc, w.pdt, a.d_A, a.d_D,
                                  a.d_ssm_state_in);
  });
  stage_mark(st, 5);
  bwd_reduce_bc_kernel<<<grid_for(bl * pr.G * 2 * pr.N), 256, 0, st>>>(pr, w.pbc, w.pdt, w.du,
                                                                       w.ddt);
  stage_mark(st, 6);
  bwd_dt_kernel<T><<<grid_for(bl * pr.H), 256, 0, st>>>(pr, a.prm, dt_raw, a.ld_dt, w.ddt,
                                                        static_cast<T *>(a.d_dt_raw), w.tok);
  col_sum_kernel<<<dim3((unsigned)ceil_div(pr.H, 256), 64), 256, 0, st>>>(w.tok, bl, pr.H,
                                                                          a.d_dt_bias);
  stage_mark(st, 7);
  const int64_t nconv = pr.batch * ((pr.L + kSeg - 1) / kSeg) * pr.conv_dim;
  bwd_conv_kernel<T><<<grid_for(nconv), 256, 0, st>>>(pr, a.prm, xBC, a.ld_xbc, cs, w.du,
                                                      static_cast<T *>(a.d_xBC),
                                                      static_cast<T *>(a.d_conv_state_in),
                                                      a.d_conv_w, a.d_conv_b);
  stage_mark(st, 8);
  return cudaGetLastError();
}

}  // namespace

const char *const kBackwardStages[] = {"bwd_prologue", "bwd_scan_fwd", "bwd_norm",
                                       "bwd_norm_w_sum", "bwd_scan_rev", "bwd_reduce_bc",
                                       "bwd_dt", "bwd_conv"};
const int kBackwardStageCount = 8;

size_t backward_workspace(const Problem &pr) { return bwd_carve(pr, nullptr, nullptr); }

cudaError_t prefill_backward(const BackwardArgs &a) {
  return a.pr.io == MAMBA2_BF16 ? run_backward<__nv_bfloat16>(a) : run_backward<float>(a);
}

}  // namespace m2
