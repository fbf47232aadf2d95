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
//   tc_chunk_out    persistent, one CTA per SM; the heads of a (row, chunk,
//                   group) are split into blocks of up to 5 taken by different
//                   CTAs in the same round; per block
//                   CB = C B^T (M = N = 128, K = 64) once; per head the
//                   operand CB o exp(cum_t - cum_s) dt_s (causal, D on the
//                   diagonal) times x (K = 128) and C times H_c^T (K = 64, a
//                   second accumulator scaled by exp(cum_t)) give y_pre in TMEM;
//                   the silu(z) gate and sums of squares follow, the blocks'
//                   per-token sums are exchanged through global memory (L2),
//                   and the normalised output is written in bf16.
//
// Operands are fp16 (11-bit significand; bf16's 8 bits cannot meet the output
// tolerance on these workloads), accumulation is fp32.  The chunk-state
// product uses a two-term fp16 split of both operands (hi*hi + hi*lo + lo*hi),
// because the returned final state must hold 2e-2 of its RMS.
#include <cuda.h>
#include <cudaTypedefs.h>

#include <algorithm>
#include <cstddef>
#include <cstring>

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
  __half *Hc;                    // [b][nch][H][n 64][p 64] state entering each chunk, scaled
  float *hsc;                    // [b][nch][H][32] 2^s: H_c rows p = 2i, 2i + 1 hold H / 2^s
  float *smax;                   // [b][nch][H] max |S_c| of each chunk's states (bounds |H_c|)
  float *cbd;                    // [b][G][nch * 128] C_t . B_t in fp32 (the decay operand's diagonal)
  // byte ranges of every buffer, for the checked build (see M2_OK)
  struct Spans {
    Span xbc, z, dt, y, conv, ssm, S, cum_end, cum, dtv, Hc, hsc, smax, cbd, u, xpart, xcnt,
        conv_w, conv_b, dt_bias, A, D, norm_w, h0max;
  } sp;
  __half *u;                     // [b][L][conv_dim] post-conv x | B | C, fp16
  int hpc;                       // most heads of a head block in tc_chunk_out
  int nhb;                       // head blocks per group in tc_chunk_out
  float *xpart;                  // [b][nch][G][nhb][128] per-token sums of squares of each block
  unsigned *xcnt;                // [b][nch][G] blocks that have published their sums
  int64_t xkeys;                 // (chunk, group) pairs the workspace holds counters for
  int y32;                       // y is 32-byte aligned: rows are written in whole 32-byte sectors
  // packed sequences of different lengths (batch = sequences, L = total tokens):
  // chunk positions come from vl_chunks, written by tc_varlen_prep_kernel
  int varlen;
  const int4 *vl_chunks;         // [chunk capacity] {sequence, chunk in it, valid tokens, first token}
  const int *vl_chunk0;          // [batch + 2] first global chunk of each sequence, the total,
                                 // then 1 if the offsets were valid (0: the call does nothing)
  const int *cu_seqlens;         // [batch + 1] first token of each sequence (last: L)
  const float *vl_h0max;         // [batch][H] max |initial state| of each (sequence, head) when
                                 // states_in, else null (the state pass reduces it itself)
};

// Where global chunk gc lies: its sequence, its index in that sequence, its
// valid tokens (1 .. 128) and its first token in the packed token order (row
// r of a fixed-length batch starts at token r L).
struct ChunkPos {
  int seq, c, nv;
  int64_t t0;
};
__device__ __forceinline__ ChunkPos chunk_pos(const TcArgs &a, int64_t gc) {
  ChunkPos p;
  if (a.varlen) {
    const int4 e = a.vl_chunks[gc];
    p.seq = e.x;
    p.c = e.y;
    p.nv = e.z;
    p.t0 = (int64_t)(uint32_t)e.w;
  } else {
    p.seq = (int)(gc / a.nch);
    p.c = (int)(gc - (int64_t)p.seq * a.nch);
    p.t0 = (int64_t)p.seq * a.pr.L + (int64_t)p.c * 128;
    p.nv = (int)min((int64_t)128, a.pr.L - (int64_t)p.c * 128);
  }
  return p;
}
// Chunks of the call: b * chunks per row, or (packed sequences) as counted by
// the prep kernel.
__device__ __forceinline__ int64_t total_chunks(const TcArgs &a) {
  return a.varlen ? (int64_t)a.vl_chunk0[a.pr.batch] : a.pr.batch * (int64_t)a.nch;
}

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

// Post-conv activations of 8 channels x 4 tokens (rows s0 .. s0 + 3 of the chunk
// starting at token t0) -> u (fp16), the chunk's nv valid tokens only.
__device__ __forceinline__ void store_u(const TcArgs &a, int64_t t0, int s0, int nv, int64_t ch,
                                        const float (&v)[4][8]) {
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    const int64_t t = t0 + s0 + k;
    if (s0 + k < nv) {
      uint4 o;
      o.x = pack_half2(v[k][0], v[k][1]);
      o.y = pack_half2(v[k][2], v[k][3]);
      o.z = pack_half2(v[k][4], v[k][5]);
      o.w = pack_half2(v[k][6], v[k][7]);
      uint4 *dst = reinterpret_cast<uint4 *>(a.u + t * a.pr.conv_dim + ch);
      if (M2_OK(dst, 16, a.sp.u, &g_tc_errors)) *dst = o;
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


// Asynchronous global -> shared copies of 16 and 4 bytes (no registers held),
// and an arrival on an mbarrier once all of this thread's earlier copies have
// landed (.noinc: the barrier's expected count includes these arrivals).
__device__ __forceinline__ void cp_async_ca16(uint32_t dst, const void *src) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 16;" ::"r"(dst), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_ca4(uint32_t dst, const void *src) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(dst), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_mbar_arrive_noinc(uint64_t *bar) {
  asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" ::"r"(smem_u32(bar))
               : "memory");
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
// group) key are its head pairs followed by one C item:
//   pair item: conv + SiLU of x (2 heads) and, for the first pair item of a key
//     in the CTA ("fresh"), of B; post-conv values to u (fp16); then
//     S = (x o w)^T B on the tensor cores (w_s = exp(cum_end - cum_s) dt_s);
//   C item: conv + SiLU of the key's C channels -> u.
// 16 compute warps + 2 producer warps + 1 MMA-issuer warp.  The producer of an
// item (one per x-ring stage; they alternate) computes its dt weights (and the
// per-token dt and cumsum rows the output kernel reads), stages its conv taps
// and TMA-loads its raw bf16 tiles [136 tokens c0-3 .. c0+132][64 ch] (128-byte
// swizzle, rows before the sequence read as zeros): the x tiles into the
// item's ring stage, the B or C tile into the key's B/C buffer (two, by key
// parity, so the next key's B arrives while this key is being worked on).
// The compute warps keep a pair item's convolved tile in registers until the
// previous pair item's MMA (the reader of the single operand buffer) has
// completed, write the fp16 hi/lo operands, release them to the MMA warp, and
// then store the previous item's chunk states from its TMEM accumulator (two
// accumulators alternate) while the current item multiplies.  No CTA-wide
// barrier is taken per item: every hand-over is an mbarrier.
// Smem (1024-aligned): x ring [2 stages][2 slots] raw tiles, B/C raw [2], then
// the operands A_hi, A_lo [2 k-blocks][128 rows][128 B] and B_hi, B_lo
// [2][64][128 B].
constexpr uint32_t kRawRows = 136, kRawBytes = kRawRows * 128;  // 17 KB, 1024-multiple
constexpr uint32_t kK1Stage = 2 * kRawBytes;
constexpr uint32_t kK1BC = 2 * kK1Stage;                      // B/C raw buffers [2]
constexpr uint32_t kK1A = 2 * 128 * 128, kK1B = 2 * 64 * 128;
constexpr uint32_t kK1Ahi = kK1BC + 2 * kRawBytes, kK1Alo = kK1Ahi + kK1A, kK1Bhi = kK1Alo + kK1A,
                   kK1Blo = kK1Bhi + kK1B, kK1Tiles = kK1Blo + kK1B;

struct K1Maps {
  CUtensorMap xbc;   // [b][L][conv_dim] bf16 (row stride ld_x), box 64 ch x 136 tokens
  CUtensorMap xbc2;  // packed sequences: [L tokens][conv_dim], the same box
};

// conv1d + SiLU of the 8 channels in 16-byte column `cg` of a raw tile, for
// output tokens at tile rows s0+3 .. s0+6 (inputs: rows s0 .. s0+6); taps and
// bias of the tile's 64 channels in shared memory, channel 8 g + i at [i][g]
// (wt[8][8] float4, bs[8][8]) so that neighbouring groups read neighbouring words.
// With h = pre / 2 (exact), silu(pre) = h + h tanh(h).
// The 7 rows stay packed (2 bf16 per register) and are widened one channel at a
// time, so that only 28 registers of inputs and one channel's taps are live.
// hrows, if not 0, holds rows 0..2 (the 3 tokens before a sequence's first
// chunk) in the tile's layout; they are read from there instead of the tile.
__device__ __forceinline__ void conv8x4_smem(uint32_t tile, int s0, int cg, const float4 *wt,
                                             const float *bs, float (&out)[4][8],
                                             uint32_t hrows = 0) {
  uint32_t raw[7][4];
#pragma unroll
  for (int r = 0; r < 7; ++r) {
    const int R = s0 + r;
    const uint32_t src = (hrows != 0 && R < 3) ? hrows : tile;
    const uint4 q = ld_shared_v4(src + R * 128 + (((cg ^ R) & 7) << 4));
    raw[r][0] = q.x;
    raw[r][1] = q.y;
    raw[r][2] = q.z;
    raw[r][3] = q.w;
  }
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const float4 wv = wt[i * 8 + cg];
    const float bias = bs[i * 8 + cg];
    float col[7];  // channel i of the rows: bf16 -> fp32 is a 16-bit shift
#pragma unroll
    for (int r = 0; r < 7; ++r)
      col[r] = __uint_as_float((i & 1) ? (raw[r][i >> 1] & 0xFFFF0000u) : (raw[r][i >> 1] << 16));
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const float h = 0.5f * (bias + wv.x * col[k] + wv.y * col[k + 1] + wv.z * col[k + 2] +
                              wv.w * col[k + 3]);
      out[k][i] = fmaf(h, tanh_approx(h), h);
    }
  }
}

struct K1Item {
  int gc;        // global chunk (every index of the item fits in 32 bits)
  int seq, c;    // its sequence (row) and chunk in the sequence
  int nv;        // valid tokens of the chunk
  int64_t t0;    // first token of the chunk
  int g, pair;
  unsigned key;  // (global chunk, group) index
  bool isC;
  bool freshB;  // B must be convolved (the CTA's previous item had another key)
};

// Item `it`, the k-th of its CTA.  Items are ordered (global chunk, group, r)
// with r = 0 .. pairs - 1 the head pairs and r = pairs the C item; every index
// fits in 32 bits (the launch checks the item count).
__device__ __forceinline__ bool k1_is_c(int pairs, int it) {
  return it % (pairs + 1) == pairs;
}
__device__ __forceinline__ K1Item k1_item(const TcArgs &a, int pairs, int it, int k) {
  const unsigned key = (unsigned)it / (unsigned)(pairs + 1);
  const int r = it - (int)key * (pairs + 1);
  const unsigned gc = key / (unsigned)a.pr.G;
  K1Item w;
  w.key = key;
  w.g = (int)(key - gc * (unsigned)a.pr.G);
  w.gc = (int)gc;
  const ChunkPos pos = chunk_pos(a, gc);
  w.seq = pos.seq;
  w.c = pos.c;
  w.nv = pos.nv;
  w.t0 = pos.t0;
  w.isC = r == pairs;
  w.pair = w.isC ? 0 : r;
  w.freshB = !w.isC && (k == 0 || r == 0);
  return w;
}

__global__ void __launch_bounds__(kK1Threads, 1)
    tc_chunk_state_kernel(TcArgs a, const __grid_constant__ K1Maps maps, int n_items) {
  if (test_stall(&g_tc_stall, &g_tc_errors)) return;  // every CTA alike (test aid)
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  __shared__ __align__(16) float ws[2][2][kQ];    // [stage][head of pair][token] chunk weights (read as float4)
  __shared__ float4 wts[2][3][64];                // [stage][slot x_A, x_B, B/C][channel] conv taps
  __shared__ __align__(16) float bss[2][3][64];   // [stage][slot][channel] conv bias
  __shared__ uint64_t full[2], empty[2], bc_empty[2], ops_ready, mma_done[2], tmem_free[2],
      mma_final, cbd_bar, park_bar;
  // rows 0..2 (the conv's left context) of a sequence's first chunk: per stage and
  // x slot, and per B/C buffer; the tiles' own rows 0..2 are not read then
  __shared__ __align__(16) unsigned char hrow_x[2][2][3 * 128];
  __shared__ __align__(16) unsigned char hrow_bc[2][3 * 128];
  __shared__ __align__(16) float cbd_s[2][kQ];  // C-item parity: per-token partials of channel groups 4-7
  __shared__ uint32_t tmem_holder;
  const Problem &pr = a.pr;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const uint32_t base = (smem_u32(smem_raw) + 1023u) & ~1023u;
  const uint32_t sAhi = base + kK1Ahi, sAlo = base + kK1Alo, sBhi = base + kK1Bhi,
                 sBlo = base + kK1Blo;
  const int hpg = pr.heads_per_group();
  const int pairs = (hpg + 1) / 2;
  // the call's items (for packed sequences n_items is a capacity and the count
  // comes from the chunk table), split evenly over the CTAs
  const int n_real = (int)min((int64_t)n_items, total_chunks(a) * pr.G * (pairs + 1));
  const int it0 = (int)((int64_t)n_real * blockIdx.x / gridDim.x),
            it1 = (int)((int64_t)n_real * (blockIdx.x + 1) / gridDim.x);

  if (warp == 0) tmem_alloc(&tmem_holder, 128);
  if (tid == 0) {
    for (int k = 0; k < 2; ++k) {
      // the tiles' transaction bytes + the producer's weights + each producer lane's tap copies
      mbar_init(&full[k], 2 + 32);
      mbar_init(&empty[k], kThreads);  // every compute thread has read the stage's x tiles
      mbar_init(&bc_empty[k], 256);    // warps 0-7 have read the B/C tile
      mbar_init(&mma_done[k], 1);      // tcgen05.commit of a pair item's MMAs
      mbar_init(&tmem_free[k], kThreads);  // its chunk states read out of TMEM
    }
    mbar_init(&ops_ready, kThreads);  // operands of a pair item written
    mbar_init(&mma_final, 1);
    mbar_init(&cbd_bar, 128);   // warps 12-15 have written a C item's diagonal partials
    mbar_init(&park_bar, 256);  // warps 0-7 have parked a C item's convolved C values
    fence_mbar_init();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_holder;

  if (warp == kThreads / 32 || warp == kThreads / 32 + 2) {
    // ---------------- producers: warp 16 takes the CTA's even items (ring stage
    // 0), warp 18 the odd ones (stage 1).  Both walk every item to count the
    // uses of the two B/C buffers.
    const int mine = warp == kThreads / 32 ? 0 : 1;
    int k = 0;
    int bc_use0 = 0, bc_use1 = 0;  // (scalars: no local memory)
    bool ok = true;
    for (int it = it0; ok && it < it1; ++it, ++k) {
      const int st = k & 1;
      const K1Item w = k1_item(a, pairs, it, k);
      const bool useBC = w.isC || w.freshB;
      const int bcb = (int)(w.key & 1u);
      const int bc_use = !useBC ? 0 : (bcb ? bc_use1++ : bc_use0++);
      if (st != mine) continue;
      const int64_t c0 = (int64_t)w.c * kQ;
      const int hA = w.g * hpg + 2 * w.pair;
      const bool hasB = 2 * w.pair + 1 < hpg;
      // everything that needs no shared memory first, while the stage may still be
      // in use: the item's global loads (one round trip: dt of both heads for this
      // lane's 4 tokens, their dt_bias and A), the dt weights, and the per-token dt
      // and cumsum rows for the output kernel.  The conv taps are read after the
      // stage's tiles are requested (not held in registers across the wait)
      float dtr[2][4], dtb[2] = {0.0f, 0.0f}, Ah[2] = {0.0f, 0.0f};
      // slots in use (a C item convolves the key's C channels (B/C buffer) and its B
      // channels (x slot 0) to form the fp32 diagonal C_t . B_t) and their first channel
      auto slot_on = [&](int sl) -> bool {
        return w.isC ? sl != 1 : (sl == 1 ? hasB : (sl == 2 ? w.freshB : true));
      };
      auto slot_ch = [&](int sl) -> int64_t {
        return (w.isC && sl == 0) ? pr.d_inner + (int64_t)w.g * kNS
               : sl < 2           ? (int64_t)(hA + sl) * kHP
                                  : pr.d_inner + (int64_t)((w.isC ? pr.G : 0) + w.g) * kNS;
      };
#pragma unroll
      for (int half = 0; half < 2; ++half) {
        const bool hv = !w.isC && (half == 0 || hasB);
        if (hv && M2_OK(a.prm.dt_bias + hA + half, 4, a.sp.dt_bias, &g_tc_errors) &&
            M2_OK(a.prm.A + hA + half, 4, a.sp.A, &g_tc_errors)) {
          dtb[half] = __ldg(a.prm.dt_bias + hA + half);
          Ah[half] = __ldg(a.prm.A + hA + half);
        }
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const int li = 4 * lane + q;  // token of the chunk
          const __nv_bfloat16 *dp = a.dt_raw + (w.t0 + li) * a.ld_dt + hA + half;
          dtr[half][q] = (hv && li < w.nv && M2_OK(dp, 2, a.sp.dt, &g_tc_errors))
                             ? __bfloat162float(*dp)
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
          // decay from token s to the chunk end, sum_{r > s} dt_r A, summed directly
          // (exclusive suffix sums) rather than as cum_end - cum_s: with strong decays
          // |cum| is large and that difference would lose the small exponents that matter
          const float r3 = a4[3], r2 = a4[2] + r3, r1 = a4[1] + r2, r0 = a4[0] + r1;
          float e = __shfl_down_sync(0xffffffffu, r0, 1);
          if (lane == 31) e = 0.0f;
#pragma unroll
          for (int o = 1; o < 32; o <<= 1) {
            const float nx = __shfl_down_sync(0xffffffffu, e, o);
            if (lane + o < 32) e += nx;
          }
          const float sfx[4] = {e + r1, e + r2, e + r3, e};
          float cq[4];
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            run += a4[q];
            cq[q] = run;
            wsv[half][q] = expf(sfx[q]) * dt4[q];
          }
          if (hv) {
            const int64_t row = (int64_t)w.gc * pr.H + hA + half;
            float4 *cp = reinterpret_cast<float4 *>(a.cum + row * kQ) + lane;
            float4 *dp = reinterpret_cast<float4 *>(a.dtv + row * kQ) + lane;
            if (M2_OK(cp, 16, a.sp.cum, &g_tc_errors)) *cp = make_float4(cq[0], cq[1], cq[2], cq[3]);
            if (M2_OK(dp, 16, a.sp.dtv, &g_tc_errors)) *dp = make_float4(dt4[0], dt4[1], dt4[2], dt4[3]);
            if (lane == 0 && M2_OK(a.cum_end + row, 4, a.sp.cum_end, &g_tc_errors))
              a.cum_end[row] = cum_end;
            // max |S_c| of this head: raised by the compute warps' atomics after the MMA
            if (lane == 0 && M2_OK(a.smax + row, 4, a.sp.smax, &g_tc_errors)) a.smax[row] = 0.0f;
          }
        }
      }
      // the stage is free once the compute warps are done with item k - 2, the B/C
      // buffer once warps 0-7 are done with its previous use
      bool got = true;
      if (lane == 0) {
        if (k >= 2) got = mbar_wait_bounded(&empty[st], (uint32_t)(((k >> 1) - 1) & 1), &g_tc_errors);
        if (got && useBC && bc_use >= 1)
          got = mbar_wait_bounded(&bc_empty[bcb], (uint32_t)((bc_use - 1) & 1), &g_tc_errors);
      }
      ok = __shfl_sync(0xffffffffu, got ? 1 : 0, 0) != 0;
      if (!ok) break;
      // the first chunk of a sequence that continues from a carried conv state (or of
      // a packed sequence, whose rows before it belong to the previous one): its
      // left context (tokens -3 .. -1: that state, or zeros) goes to the side rows,
      // which the compute warps read instead of the tiles' rows 0..2
      const bool halo = w.c == 0 && (a.states_in || a.varlen);
      const uint32_t stage = base + st * kK1Stage;
      const uint32_t bcbuf = base + kK1BC + bcb * kRawBytes;
      const int64_t bc_ch = pr.d_inner + (int64_t)((w.isC ? pr.G : 0) + w.g) * kNS;
      if (lane == 0) {
        uint64_t *bar = &full[st];
        const uint32_t nbytes =
            (w.isC ? 1u : (1u + (hasB ? 1u : 0u))) * kRawBytes + (useBC ? kRawBytes : 0u);
        mbar_arrive_expect_tx(bar, nbytes);
        // raw rows c0 - 3 .. c0 + 132 of the item's channels starting at `ch`
        auto load_raw = [&](uint32_t dst, int ch) {
          if (a.varlen) tma_load_2d(dst, &maps.xbc2, ch, (int)(w.t0 - 3), bar);
          else tma_load_3d(dst, &maps.xbc, ch, (int)c0 - 3, w.seq, bar);
        };
        if (w.isC) load_raw(stage, (int)(pr.d_inner + (int64_t)w.g * kNS));
        if (!w.isC) {
          load_raw(stage, hA * kHP);
          if (hasB) load_raw(stage + kRawBytes, (hA + 1) * kHP);
        }
        if (useBC) load_raw(bcbuf, (int)bc_ch);
      }
      if (halo) {
        // slot x_A, x_B (if any) and the B/C tile: 3 rows x 64 channels each
        for (int idx = lane; idx < 3 * 3 * 64; idx += 32) {
          const int sl = idx / 192, r = (idx / 64) % 3, chn = idx % 64;
          if (!slot_on(sl)) continue;
          const int64_t ch = slot_ch(sl) + chn;
          const __nv_bfloat16 *hp = a.conv_in + ((int64_t)w.seq * pr.conv_dim + ch) * 4 + 1 + r;
          const __nv_bfloat16 v = a.states_in && M2_OK(hp, 2, a.sp.conv, &g_tc_errors)
                                      ? *hp
                                      : __float2bfloat16(0.0f);
          const uint32_t rows = sl < 2 ? smem_u32(&hrow_x[st][sl][0]) : smem_u32(&hrow_bc[bcb][0]);
          const uint32_t addr = rows + r * 128 + ((((chn >> 3) ^ r) & 7) << 4) + ((chn & 7) << 1);
          asm volatile("st.shared.b16 [%0], %1;" ::"r"(addr), "h"(__bfloat16_as_ushort(v))
                       : "memory");
        }
      }
      if (!w.isC) {
#pragma unroll
        for (int half = 0; half < 2; ++half)
#pragma unroll
          for (int q = 0; q < 4; ++q) ws[st][half][4 * lane + q] = wsv[half][q];
      }
      // conv taps and bias of the item's slots, channel 8 g + i at [i][g], copied
      // asynchronously; each lane's copies complete on the stage's barrier
#pragma unroll 1
      for (int sl = 0; sl < 3; ++sl) {
        if (!slot_on(sl)) continue;
        const int64_t ch0 = slot_ch(sl);
#pragma unroll
        for (int j = 0; j < 2; ++j) {
          const int i = lane + 32 * j, d = (i & 7) * 8 + (i >> 3);
          const float4 *wp = reinterpret_cast<const float4 *>(a.prm.conv_w) + ch0 + i;
          const float *bp = a.prm.conv_b + ch0 + i;
          if (M2_OK(wp, 16, a.sp.conv_w, &g_tc_errors)) cp_async_ca16(smem_u32(&wts[st][sl][d]), wp);
          else wts[st][sl][d] = make_float4(0.f, 0.f, 0.f, 0.f);
          if (M2_OK(bp, 4, a.sp.conv_b, &g_tc_errors)) cp_async_ca4(smem_u32(&bss[st][sl][d]), bp);
          else bss[st][sl][d] = 0.0f;
        }
      }
      cp_async_mbar_arrive_noinc(&full[st]);
      __syncwarp();
      if (lane == 0) mbar_arrive(&full[st]);  // weights of this stage written
    }
    // no copy may be in flight when the CTA exits: the last stage loads issued
    if (lane == 0) {
      for (int kk = max(0, k - 2); kk < k; ++kk)
        if ((kk & 1) == mine) mbar_wait_bounded(&full[kk & 1], (uint32_t)((kk >> 1) & 1), &g_tc_errors);
    }
  } else if (warp == kThreads / 32 + 1) {
    // ---------------- MMA issuer: S = x_hi B_hi + x_hi B_lo + x_lo B_hi per pair item,
    // into TMEM accumulator np % 2
    if (lane == 0) {
      const uint32_t idesc = umma_idesc_f16(128, 64);
      const uint32_t As[3] = {sAhi, sAhi, sAlo}, Bs[3] = {sBhi, sBlo, sBhi};
      int np = 0;
      for (int it = it0; it < it1; ++it) {
        if (k1_is_c(pairs, it)) continue;
        if (!mbar_wait_bounded(&ops_ready, (uint32_t)(np & 1), &g_tc_errors)) break;
        if (np >= 2 &&
            !mbar_wait_bounded(&tmem_free[np & 1], (uint32_t)(((np - 2) >> 1) & 1), &g_tc_errors))
          break;
        tc_fence_after();
        const uint32_t acc = tmem + 64 * (np & 1);
        for (int prod = 0; prod < 3; ++prod)
          for (int ks = 0; ks < 8; ++ks) {
            const int blk = ks >> 2, kin = ks & 3;
            umma_f16(acc, umma_desc_sw128(As[prod] + blk * 16384 + kin * 32),
                     umma_desc_sw128(Bs[prod] + blk * 8192 + kin * 32), idesc,
                     (prod > 0 || ks > 0) ? 1u : 0u);
          }
        umma_commit(&mma_done[np & 1]);
        ++np;
      }
      // no MMA may be in flight when the CTA frees its tensor memory
      umma_commit(&mma_final);
      mbar_wait_bounded(&mma_final, 0, &g_tc_errors);
    }
  } else {
    // ---------------- compute warps
    bool ok = true;
    int k = 0, np = 0, nc = 0;  // items, pair items and C items so far
    // chunk states of pair item q out of TMEM accumulator q % 2: rows m = 32 (warp % 4)
    // + lane (head half m / 64, lane p = m % 64), 16 columns per warp / 4; S is kept
    // [n/4][p][4] per head so that a warp's float4 stores are contiguous
    struct Pending {
      int gc, hA;
      bool hasB;
    } pw{};
    auto store_states = [&](const Pending &q, int acc) {
      const int m = 32 * (warp & 3) + lane, half = m >> 6, p = m & 63, cb = warp >> 2;
      float sv[16];
      tmem_ld16(tmem + ((uint32_t)(32 * (warp & 3)) << 16) + 64 * acc + 16 * cb, sv);
      tc_fence_before();  // TMEM read before the accumulator takes the next item
      mbar_arrive(&tmem_free[acc]);
      // max |S| over the warp's 32 rows x 16 columns (all of one head) into the head's
      // bound (non-negative floats order as their bit patterns)
      float mx = 0.0f;
#pragma unroll
      for (int i = 0; i < 16; ++i) mx = fmaxf(mx, fabsf(sv[i]));
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
      if (half == 0 || q.hasB) {
        float *mp = a.smax + (int64_t)q.gc * pr.H + q.hA + half;
        if (lane == 0 && M2_OK(mp, 4, a.sp.smax, &g_tc_errors))
          atomicMax(reinterpret_cast<int *>(mp), __float_as_int(mx));

        float4 *dst = reinterpret_cast<float4 *>(
            a.S + ((int64_t)q.gc * pr.H + q.hA + half) * (int64_t)(kHP * kNS));
#pragma unroll
        for (int i = 0; i < 4; ++i)
          if (M2_OK(dst + (4 * cb + i) * kHP + p, 16, a.sp.S, &g_tc_errors))
            dst[(4 * cb + i) * kHP + p] =
                make_float4(sv[4 * i], sv[4 * i + 1], sv[4 * i + 2], sv[4 * i + 3]);
      }
    };
    auto wait_mma = [&](int q) {  // pair item q's MMAs completed (operands free, S in TMEM)
      const bool got = ok && mbar_wait_bounded(&mma_done[q & 1], (uint32_t)((q >> 1) & 1), &g_tc_errors);
      ok = __all_sync(0xffffffffu, got) != 0;
    };
    for (int it = it0; ok && it < it1; ++it, ++k) {
      const int st = k & 1;
      const uint32_t stage = base + st * kK1Stage;
      const K1Item w = k1_item(a, pairs, it, k);
      const int bcb = (int)(w.key & 1u);
      {
        const bool got = mbar_wait_bounded(&full[st], (uint32_t)((k >> 1) & 1), &g_tc_errors);
        ok = __all_sync(0xffffffffu, got) != 0;
      }
      if (!ok) break;
      const int hA = w.g * hpg + 2 * w.pair;
      const bool hasB = 2 * w.pair + 1 < hpg;
      const uint32_t bcbuf = base + kK1BC + bcb * kRawBytes;
      const int64_t bc_ch = pr.d_inner + (int64_t)((w.isC ? pr.G : 0) + w.g) * kNS;
      // a sequence's first chunk: its left context lives in the side rows
      const bool halo = w.c == 0 && (a.states_in || a.varlen);
      auto hx = [&](int sl) -> uint32_t { return halo ? smem_u32(&hrow_x[st][sl][0]) : 0u; };
      const uint32_t hbc = halo ? smem_u32(&hrow_bc[bcb][0]) : 0u;
      // warp tile: 4 groups of 8 channels x 8 quads of tokens (lane = group lane % 4,
      // quad lane / 4); it reads the swizzled raw rows, stores u (64 contiguous bytes
      // per token) and, with the channel order of odd groups rotated by 4, stores the
      // swizzled operands without shared-memory bank conflicts
      const int cg = 4 * ((warp >> 2) & 1) + (lane & 3);
      const int s0 = 4 * (8 * (warp & 3) + (lane >> 2));
      // the tile's 4 token weights (x slots; B is not weighted).  Read before the
      // stage is released: the producer of item k + 2 overwrites ws[st] after that
      auto tile_weights = [&](int sl) -> float4 {
        return sl < 2 ? *reinterpret_cast<const float4 *>(&ws[st][sl][s0])
                      : make_float4(1.0f, 1.0f, 1.0f, 1.0f);
      };
      // operands of one tile: x o w (slots 0, 1) or B (slot 2), split into fp16 hi + lo
      auto put_operands = [&](int sl, const float (&v)[4][8], float4 w4) {
        const int blk = s0 >> 6, kq = s0 & 63;
        const float wk[4] = {w4.x, w4.y, w4.z, w4.w};
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
      // missing second head: zero rows 64..127 of the x operands
      auto zero_tile = [&]() {
        const int blk = s0 >> 6, kq = s0 & 63;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const uint32_t off = blk * 16384 + sw128_off(64 + cg * 8 + i, kq);
          st_shared_v2(sAhi + off, 0u, 0u);
          st_shared_v2(sAlo + off, 0u, 0u);
        }
      };
      float v[4][8];
      if (w.isC) {
        // C item: warps 0-7 convolve the C channels (B/C buffer) into u and park the
        // values, fp32, in the B operand buffers (free once the last pair item's MMAs
        // are done); warps 8-15, whose lanes hold the same 8 channels x 4 tokens,
        // convolve the B channels (x slot 0) and form C_t . B_t in fp32: summed over
        // the 4 lanes of a token quad, then warps 12-15 (channel groups 4-7) hand
        // their sums to warps 8-11 through shared memory
        if (np >= 1) wait_mma(np - 1);
        if (!ok) break;
        const uint32_t park = sBhi + (uint32_t)(((warp & 7) * 32 + lane) * 16);  // [8][256] float4
        if (warp < 8) {
          conv8x4_smem(bcbuf, s0, cg, wts[st][2], bss[st][2], v, hbc);
          mbar_arrive(&bc_empty[bcb]);
          store_u(a, w.t0, s0, w.nv, bc_ch + cg * 8, v);
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
#pragma unroll
            for (int h = 0; h < 2; ++h)
              st_shared_v4(park + (2 * kk + h) * 4096, __float_as_uint(v[kk][4 * h]),
                           __float_as_uint(v[kk][4 * h + 1]), __float_as_uint(v[kk][4 * h + 2]),
                           __float_as_uint(v[kk][4 * h + 3]));
          mbar_arrive(&empty[st]);
          mbar_arrive(&park_bar);
        } else {
          conv8x4_smem(stage, s0, cg, wts[st][0], bss[st][0], v, hx(0));
          mbar_arrive(&empty[st]);
          {
            const bool got = mbar_wait_bounded(&park_bar, (uint32_t)(nc & 1), &g_tc_errors);
            ok = __all_sync(0xffffffffu, got) != 0;
          }
          if (!ok) break;
          float d4[4];
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) {
            float acc = 0.0f;
#pragma unroll
            for (int h = 0; h < 2; ++h) {
              const uint4 q = ld_shared_v4(park + (2 * kk + h) * 4096);
              acc = fmaf(__uint_as_float(q.x), v[kk][4 * h], acc);
              acc = fmaf(__uint_as_float(q.y), v[kk][4 * h + 1], acc);
              acc = fmaf(__uint_as_float(q.z), v[kk][4 * h + 2], acc);
              acc = fmaf(__uint_as_float(q.w), v[kk][4 * h + 3], acc);
            }
            acc += __shfl_xor_sync(0xffffffffu, acc, 1);
            acc += __shfl_xor_sync(0xffffffffu, acc, 2);
            d4[kk] = acc;
          }
          const int cpar = nc & 1;
          if (warp >= 12) {
            if ((lane & 3) == 0)
              *reinterpret_cast<float4 *>(&cbd_s[cpar][s0]) = make_float4(d4[0], d4[1], d4[2], d4[3]);
            mbar_arrive(&cbd_bar);
          } else {
            const bool got = mbar_wait_bounded(&cbd_bar, (uint32_t)(nc & 1), &g_tc_errors);
            ok = __all_sync(0xffffffffu, got) != 0;
            if (ok && (lane & 3) == 0) {
              const float4 o = *reinterpret_cast<const float4 *>(&cbd_s[cpar][s0]);
              float4 *dp = reinterpret_cast<float4 *>(a.cbd + ((int64_t)w.gc * pr.G + w.g) * kQ + s0);
              if (M2_OK(dp, 16, a.sp.cbd, &g_tc_errors))
                *dp = make_float4(d4[0] + o.x, d4[1] + o.y, d4[2] + o.z, d4[3] + o.w);
            }
          }
        }
        ++nc;
        continue;
      }
      const int sl = warp >> 3;  // x slot of this warp: head A (warps 0-7) or B
      const int64_t xch = (int64_t)(hA + sl) * kHP;
      if (w.freshB) {
        // B changes: the previous pair item's MMAs must have read the old operands
        if (np >= 1) wait_mma(np - 1);
        if (!ok) break;
        if (warp < 8) {
          conv8x4_smem(bcbuf, s0, cg, wts[st][2], bss[st][2], v, hbc);
          if (w.pair == 0) store_u(a, w.t0, s0, w.nv, bc_ch + cg * 8, v);
          put_operands(2, v, tile_weights(2));
          mbar_arrive(&bc_empty[bcb]);
        }
        if (sl == 1 && !hasB) zero_tile();
        else {
          conv8x4_smem(stage + sl * kRawBytes, s0, cg, wts[st][sl], bss[st][sl], v, hx(sl));
          store_u(a, w.t0, s0, w.nv, xch + cg * 8, v);
          put_operands(sl, v, tile_weights(sl));
        }
        mbar_arrive(&empty[st]);
      } else {
        // the previous pair item's MMAs (the readers of the single operand buffer) are
        // normally done by now; waiting first keeps the tile out of registers across
        // the wait.  The u stores follow the operand hand-off, so the MMA does not wait
        // behind them
        const bool has_tile = !(sl == 1 && !hasB);
        if (np >= 1) wait_mma(np - 1);
        if (!ok) break;
        if (has_tile) {
          conv8x4_smem(stage + sl * kRawBytes, s0, cg, wts[st][sl], bss[st][sl], v, hx(sl));
          const float4 wk4 = tile_weights(sl);
          mbar_arrive(&empty[st]);  // nothing of the stage is read after this
          put_operands(sl, v, wk4);
        } else {
          mbar_arrive(&empty[st]);
          zero_tile();
        }
        fence_proxy_async_smem();
        mbar_arrive(&ops_ready);  // the MMA warp issues S = (x o w)^T B into accumulator np % 2
        if (has_tile) store_u(a, w.t0, s0, w.nv, xch + cg * 8, v);
      }
      if (w.freshB) {
        fence_proxy_async_smem();
        mbar_arrive(&ops_ready);
      }
      // meanwhile: the previous pair item's chunk states out of its accumulator
      if (np >= 1) store_states(pw, (np - 1) & 1);
      pw.gc = w.gc;
      pw.hA = hA;
      pw.hasB = hasB;
      ++np;
    }
    if (ok && np >= 1) {
      wait_mma(np - 1);
      if (ok) store_states(pw, (np - 1) & 1);
    }
  }
  tc_fence_before();
  __syncthreads();
  launch_dependents();
  if (warp == 0) tmem_dealloc(tmem, 128);
}

// ============================================================== packed sequences
// One block: checks the sequence offsets (0 first, non-decreasing, the total
// token count last), counts each sequence's chunks, scans the counts into
// chunk0 and writes every chunk's position {sequence, chunk in it, valid tokens,
// first token}; chunk0[nseq + 1] = 1.  Offsets that fail the check raise
// kErrSeqlens and leave zero chunks and chunk0[nseq + 1] = 0, so that the
// kernels after it do nothing.
// With carried states, blocks 1 .. nseq H each reduce one (sequence, head)'s
// initial state to max |h0| (the state pass's first bound B_0), once, instead of
// every state-pass block of the head reading the whole state again: the packed
// sequences' many short chains then start without that round trip.
constexpr int kPrepThreads = 1024;  // = the 4096 floats of a 64 x 64 state, as float4
__global__ void __launch_bounds__(kPrepThreads)
    tc_varlen_prep_kernel(const int *cu, int nseq, int64_t L, int64_t cap, int4 *chunks,
                          int *chunk0, const float *ssm, float *h0max, Span ssm_span) {
  __shared__ int bad;
  __shared__ int wsum[kPrepThreads / 32];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  if (blockIdx.x > 0) {
    const int64_t pair = blockIdx.x - 1;  // sequence * H + head
    const float4 *src = reinterpret_cast<const float4 *>(ssm + pair * (int64_t)(kHP * kNS)) + tid;
    float m = 0.0f;
    if (M2_OK(src, 16, ssm_span, &g_tc_errors)) {
      const float4 v = *src;
      m = fmaxf(fmaxf(fabsf(v.x), fabsf(v.y)), fmaxf(fabsf(v.z), fabsf(v.w)));
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    __shared__ float red[kPrepThreads / 32];
    if (lane == 0) red[warp] = m;
    __syncthreads();
    if (tid == 0) {
      float r = 0.0f;
      for (int w = 0; w < kPrepThreads / 32; ++w) r = fmaxf(r, red[w]);
      h0max[pair] = r;
    }
    return;
  }
  if (tid == 0) bad = (cu[0] != 0 || (int64_t)cu[nseq] != L) ? 1 : 0;
  __syncthreads();
  // thread tid takes sequences [s0, s1)
  const int per = (nseq + kPrepThreads - 1) / kPrepThreads;
  const int s0 = min(nseq, tid * per), s1 = min(nseq, s0 + per);
  int local = 0;
  for (int s = s0; s < s1; ++s) {
    const int len = cu[s + 1] - cu[s];
    if (len < 0) bad = 1;
    local += len > 0 ? (len + kQ - 1) / kQ : 0;
  }
  // exclusive scan of the per-thread counts
  int incl = local;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int v = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += v;
  }
  if (lane == 31) wsum[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    int v = lane < kPrepThreads / 32 ? wsum[lane] : 0;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int u = __shfl_up_sync(0xffffffffu, v, o);
      if (lane >= o) v += u;
    }
    if (lane < kPrepThreads / 32) wsum[lane] = v;  // inclusive over warps
  }
  __syncthreads();
  const bool ok = bad == 0;
  int run = incl - local + (warp > 0 ? wsum[warp - 1] : 0);  // chunks before s0
  if (!ok || (int64_t)wsum[kPrepThreads / 32 - 1] > cap) {
    if (tid == 0) atomicOr(&g_tc_errors, kErrSeqlens);
    for (int s = tid; s <= nseq + 1; s += kPrepThreads) chunk0[s] = 0;
    return;
  }
  for (int s = s0; s < s1; ++s) {
    chunk0[s] = run;
    const int len = cu[s + 1] - cu[s];
    const int n = len > 0 ? (len + kQ - 1) / kQ : 0;
    for (int c = 0; c < n; ++c)
      chunks[run + c] = make_int4(s, c, min(kQ, len - c * kQ), cu[s] + c * kQ);
    run += n;
  }
  if (tid == kPrepThreads - 1) {
    chunk0[nseq] = wsum[kPrepThreads / 32 - 1];
    chunk0[nseq + 1] = 1;
  }
}

// ============================================================== state passing
// grid (H * 8 + conv-state blocks, b) of 128-thread blocks, five per SM, so that
// a launch is one wave.  Block 8 h + q runs the recurrence
// H_{c+1} = exp(cum_end_c) H_c + S_c in fp32 for the float4 slots j = 128 q +
// thread of head h's chunk states ([n/4][p][4]: columns n = 4 (j / 64) .. +3 of
// row p = j % 64), sequential over chunks.  The chain waits on memory, so loads
// are issued 16 chunks at a time (one round trip per 16 chunks; the batch's
// scalars come through shared memory to leave the registers to the states): a
// warp reads 512 contiguous bytes per chunk and writes the fp16 state
// entering each chunk as H_c [n][p] (the output kernel's MN-major operand), four
// coalesced 64-byte rows.
// H_c is stored divided by 2^s, one power of two per (chunk, head), so that fp16
// cannot overflow whatever the state's size: s comes from a bound on max |H_c|
// that every thread of the head computes alike, B_0 = max |initial state| and
// B_{c+1} = exp(cum_end_c) B_c + max |S_c| (the chunk-state kernel supplies the
// last term), with s = max(0, floor(log2 B_c) - 13) so that |H_c| / 2^s < 2^14.
// Overestimating B only moves small values towards fp16's subnormals, whose
// absolute spacing 2^-24 2^s stays below 2^-37 B.  The output kernel multiplies
// C H_c^T by 2^s (exact); the scale table keeps one entry per row pair, here all
// equal.
// Blocks 4 H and up write the final conv state instead: the last 4 raw inputs of
// [old state | new tokens], in place (the chunk-state kernel, which reads the old
// state, has finished by now).
constexpr int kPassBlocks = 8;     // blocks per head
constexpr int kPassThreads = 128;  // x 8 = the 1024 float4 slots of a head's 64 x 64 state
constexpr int kPassAhead = 16;     // chunks whose loads are in flight together

// s = max(0, floor(log2 m) - 13), so that m / 2^s < 2^14; 2^s and 2^-s are then
// built from their exponent bits (both normal: s <= 100).
__device__ __forceinline__ int state_shift(float m) {
  const int e = (int)((__float_as_uint(m) >> 23) & 0xFFu) - 127;  // floor(log2 m) for normal m
  return min(max(e - 13, 0), 100);
}

__global__ void __launch_bounds__(kPassThreads, 5) tc_state_pass_kernel(TcArgs a, __nv_bfloat16 *cs) {
  __shared__ float red[kPassThreads / 32];
  grid_dependency_wait();  // the chunk-state kernel's results (launched early, see prefill_tc)
  launch_dependents();
  const Problem &pr = a.pr;
  {  // the output kernel's exchange counters start from zero
    const int64_t stride = (int64_t)gridDim.x * gridDim.y * blockDim.x;
    for (int64_t i = ((int64_t)blockIdx.y * gridDim.x + blockIdx.x) * blockDim.x + threadIdx.x;
         i < a.xkeys; i += stride)
      if (M2_OK(a.xcnt + i, 4, a.sp.xcnt, &g_tc_errors)) a.xcnt[i] = 0u;
  }
  const int64_t bi = blockIdx.y;  // sequence (row)
  if (a.varlen && a.vl_chunk0[pr.batch + 1] == 0) return;  // invalid offsets: nothing to do
  // its chunks [cb0, cb0 + nchs) and tokens [t0s, t0s + Ls)
  int64_t cb0, nchs, t0s, Ls;
  if (a.varlen) {
    cb0 = a.vl_chunk0[bi];
    nchs = a.vl_chunk0[bi + 1] - cb0;
    t0s = a.cu_seqlens[bi];
    Ls = a.cu_seqlens[bi + 1] - t0s;
  } else {
    cb0 = bi * a.nch;
    nchs = a.nch;
    t0s = bi * pr.L;
    Ls = pr.L;
  }
  const int nrb = pr.H * kPassBlocks;
  if ((int)blockIdx.x >= nrb) {
    if (cs == nullptr) return;
    const int64_t ch = (int64_t)(blockIdx.x - nrb) * kPassThreads + threadIdx.x;
    if (ch >= pr.conv_dim) return;
    const int64_t i = bi * pr.conv_dim + ch;
    __nv_bfloat16 v[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const int64_t tau = Ls - 4 + k;
      const __nv_bfloat16 *xp = a.xBC + (t0s + tau) * a.ld_x + ch;
      v[k] = __float2bfloat16(0.0f);
      if (tau >= 0) {
        if (M2_OK(xp, 2, a.sp.xbc, &g_tc_errors)) v[k] = *xp;
      } else if (a.states_in && M2_OK(cs + i * 4 + 4 + tau, 2, a.sp.conv, &g_tc_errors)) {
        v[k] = cs[i * 4 + 4 + tau];
      }
    }
#pragma unroll
    for (int k = 0; k < 4; ++k)
      if (M2_OK(cs + i * 4 + k, 2, a.sp.conv, &g_tc_errors)) cs[i * 4 + k] = v[k];
    return;
  }
  const int h = blockIdx.x / kPassBlocks, q = blockIdx.x % kPassBlocks;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int j = q * kPassThreads + tid, n4 = j >> 6, p = j & 63;
  const int64_t head = bi * pr.H + h;
  const int64_t hs = head * (int64_t)(kHP * kNS) + p * kNS + 4 * n4;
  float4 hc = (a.states_in && M2_OK(a.ssm_state + hs, 16, a.sp.ssm, &g_tc_errors))
                  ? *reinterpret_cast<const float4 *>(a.ssm_state + hs)
                  : make_float4(0.f, 0.f, 0.f, 0.f);
  // B_0: max |initial state| over the whole head (each block of the head alike)
  float bnd = 0.0f;
  if (a.states_in && a.vl_h0max != nullptr) {
    // (packed sequences: reduced once per (sequence, head) by the prep kernel)
    bnd = M2_OK(a.vl_h0max + head, 4, a.sp.h0max, &g_tc_errors) ? a.vl_h0max[head] : 0.0f;
  } else if (a.states_in) {
    const float4 *h0 = reinterpret_cast<const float4 *>(a.ssm_state + head * (int64_t)(kHP * kNS));
    float m = 0.0f;
    for (int i = tid; i < kHP * kNS / 4; i += kPassThreads) {
      if (!M2_OK(h0 + i, 16, a.sp.ssm, &g_tc_errors)) continue;
      const float4 v = h0[i];
      m = fmaxf(m, fmaxf(fmaxf(fabsf(v.x), fabsf(v.y)), fmaxf(fabsf(v.z), fabsf(v.w))));
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    if (lane == 0) red[warp] = m;
    __syncthreads();
#pragma unroll
    for (int w = 0; w < kPassThreads / 32; ++w) bnd = fmaxf(bnd, red[w]);
  }
  // Each chunk's step is kept short: pointers advance by one chunk, 2^-s comes
  // from its exponent bits, and the decay factor is one ex2.approx of
  // cum_end log2(e).
  const int64_t stride = (int64_t)pr.H * kHP * kNS;  // one chunk further
  const int64_t c0h = cb0 * pr.H + h;                  // (first chunk, head)
  const float *S = a.S + c0h * (int64_t)(kHP * kNS) + 4 * j;
  __half *Hc = a.Hc + c0h * (int64_t)(kHP * kNS) + (4 * n4) * kHP + p;
  const float *ce = a.cum_end + c0h;
  const float *sm = a.smax + c0h;
  float *hp = a.hsc + c0h * 32 + lane;
  const int64_t hstep = (int64_t)pr.H * 32;
  const bool scale_writer = q == 0 && warp == 0;  // the head's 32 scale entries per chunk
  // H_c / 2^s into the operand (4 coalesced 2-byte stores), 2^s into the scale table
  auto put = [&]() {
    const uint32_t sh = (uint32_t)state_shift(bnd);
    const float inv = __uint_as_float((127u - sh) << 23);  // 2^-s, exact
    if (M2_OK(Hc, 2, a.sp.Hc, &g_tc_errors) && M2_OK(Hc + 3 * kHP, 2, a.sp.Hc, &g_tc_errors)) {
      Hc[0] = __float2half_rn(hc.x * inv);
      Hc[kHP] = __float2half_rn(hc.y * inv);
      Hc[2 * kHP] = __float2half_rn(hc.z * inv);
      Hc[3 * kHP] = __float2half_rn(hc.w * inv);
    }
    if (scale_writer && M2_OK(hp, 4, a.sp.hsc, &g_tc_errors))
      *hp = __uint_as_float((127u + sh) << 23);  // 2^s
  };
  auto step = [&](float4 sv, float d, float msv) {
    const float f = ex2_approx(d * kLog2e);
    hc = make_float4(fmaf(f, hc.x, sv.x), fmaf(f, hc.y, sv.y), fmaf(f, hc.z, sv.z),
                     fmaf(f, hc.w, sv.w));
    bnd = fmaf(f, bnd, msv);
  };
  // loads run kPassAhead chunks ahead of the (sequential) recurrence; the batch's
  // decay and bound scalars, the same for the whole block, are loaded by warp 0
  // (lanes 0-15 cum_end, 16-31 smax) and shared through a double buffer
  constexpr int kAhead = kPassAhead;
  static_assert(2 * kAhead == 32, "one lane of warp 0 per scalar of a batch");
  __shared__ float s_dm[2][2 * kAhead];
  // chunks [c, c + nb) of the chain, nb <= kAhead (a constant in the main loop, so
  // that only the last, shorter batch carries the predicates)
  auto run_batch = [&](int64_t c, int nb) {
    const int par = (int)((c / kAhead) & 1);
    float sl = 0.0f;
    if (warp == 0 && (lane & (kAhead - 1)) < nb) {
      const float *src = lane < kAhead ? ce + lane * pr.H : sm + (lane - kAhead) * pr.H;
      const bool okp = lane < kAhead ? M2_OK(src, 4, a.sp.cum_end, &g_tc_errors)
                                     : M2_OK(src, 4, a.sp.smax, &g_tc_errors);
      sl = okp ? *src : 0.0f;
    }
    float4 sv[kAhead];
#pragma unroll
    for (int k = 0; k < kAhead; ++k) {
      const float *sp = S + k * stride;
      sv[k] = (k < nb && M2_OK(sp, 16, a.sp.S, &g_tc_errors))
                  ? *reinterpret_cast<const float4 *>(sp)
                  : make_float4(0.f, 0.f, 0.f, 0.f);
    }
    S += kAhead * stride;
    ce += kAhead * pr.H;
    sm += kAhead * pr.H;
    if (warp == 0) s_dm[par][lane] = sl;
    __syncthreads();  // (the buffer written here was last read two batches ago)
#pragma unroll
    for (int k = 0; k < kAhead; ++k) {
      if (k < nb) {
        put();
        step(sv[k], s_dm[par][k], s_dm[par][kAhead + k]);
        Hc += stride;
        hp += hstep;
      }
    }
  };
  int64_t c = 0;
  for (; c + kAhead <= nchs; c += kAhead) run_batch(c, kAhead);
  if (c < nchs) run_batch(c, (int)(nchs - c));
  if (a.ssm_state != nullptr && M2_OK(a.ssm_state + hs, 16, a.sp.ssm, &g_tc_errors))
    *reinterpret_cast<float4 *>(a.ssm_state + hs) = hc;
}

// ============================================================== chunk output
// Persistent grid of P CTAs, one per SM.  A unit is (row, chunk, group, head
// block): the group's heads are cut into nhb blocks of at most 5 heads, and the
// units are numbered with the head block fastest, so that the nhb units of one
// (chunk, group) are neighbours.  CTA i takes units i, i + P, ...; P is a
// multiple of nhb, so the blocks of one (chunk, group) are worked on in the same
// round by nhb different CTAs.  Per CTA:
//   warp 16      TMA producer: per unit the C and B tiles of u (C double-
//                buffered, so the next unit's arrive during this one), per head
//                the x and H_c tiles (ring of 2) and the z tile (ring of 2);
//   warp 17      MMA issuer: CB = C B^T once per unit (M = N = 128, K = 64), per
//                head y_j = A_j x_j (K = 128, into the head's 64 TMEM columns)
//                and T = C H_c^T (K = 64, one shared 64-column accumulator);
//   warps 0-7    decay operand: A_j = CB o exp(cum_t - cum_s) dt_s (s <= t, D_h
//                on the diagonal) in fp16, double-buffered, up to two heads
//                ahead of the epilogue; warp w builds rows 32 (w % 4) .. +31
//                (its TMEM lane quarter) and columns 64 (w / 4) .. +63;
//   warps 8-15   epilogue: y_j + exp(cum_t) 2^s T, gate by silu(z), per-token
//                sums of squares, the gated value back into TMEM; after the
//                unit's last head the per-token sums of the block go to global
//                memory (row hb of the (chunk, group)'s exchange slot) and a
//                counter of the (chunk, group) counts the blocks that have
//                published.  Once it reaches nhb every block adds the nhb rows,
//                in block order (the same sum, bit for bit, in every CTA and run),
//                and each head is scaled by the norm and the norm weight and
//                written to y (32-byte stores).  That output phase overlaps the
//                next unit's operand builds and MMAs: a head's TMEM columns are
//                handed back to the MMA warp one by one.
// A CTA waits only for blocks of its own (chunk, group), which other CTAs reach
// in the same round or, for a CTA that has more units, the next: with all P CTAs
// resident (P <= SMs, one CTA per SM) every wait ends.  The counters are zeroed
// by the state-pass kernel, which runs before this one.
// All waits are bounded (they raise the error flag and the CTA leaves its loop).
constexpr uint32_t kCt0 = 0;                       // C [2][128 t][64 n] fp16 (u), 2 x 16 KB
constexpr uint32_t kBt = 2 * 16384;                // B [128 s][64 n] fp16 (u), 16 KB
constexpr uint32_t kXhBytes = 16384 + 8192;        // per stage: x [128 s][64 p] + H_c [64 n][64 p]
constexpr uint32_t kXh = kBt + 16384;              // x / H_c ring, 2 x 24 KB
constexpr uint32_t kZt = kXh + 2 * kXhBytes;       // z ring [128 t][64 p] bf16, 2 x 16 KB
constexpr uint32_t kAbuf = kZt + 2 * 16384;        // A [2][2 k-blocks][128 t][64 s] fp16, 2 x 32 KB
constexpr uint32_t kTcOutTiles = kAbuf + 2 * 32768;  // 176 KB
constexpr int kGroupThreads = 256;                 // threads of the operand / epilogue groups

// Every array read or written with 16-byte accesses (float4 loads and stores) is
// 16-byte aligned; the static_asserts below check it.
struct OutShared {
  // decay terms of the unit's heads (operand group)
  alignas(16) float cum2[2][kMaxHeadsPerCta][kQ];  // [unit parity] cumsum * log2(e) (also read by the epilogue)
  alignas(16) float dt[kMaxHeadsPerCta][kQ];
  alignas(16) float beta[kMaxHeadsPerCta][kQ];   // exp(cum_r - cum_s) dt_s, r = end of s's 32-token group
  alignas(16) float betad[kMaxHeadsPerCta][kQ];  // exp(cum_s0 - cum_s) dt_s, s0 = start of s's group
  // epilogue group
  alignas(16) float half_ss[2][kQ];              // per-token sums of squares of the two column halves
  alignas(16) float cbd[kQ];                     // C_t . B_t (fp32) of the unit's chunk and group
  alignas(16) uint8_t scs[2][kMaxHeadsPerCta][32];  // [unit parity] exponents s of H_c's row-pair scales 2^s
  alignas(16) float nw[kMaxHeadsPerCta][kHP];     // the unit's norm weights (epilogue group)
  int span_ok[kMaxHeadsPerCta][4];   // group's log2-decay span <= 60: factorise its diagonal
  float Dh[kMaxHeadsPerCta];
  uint64_t full_cb[2], b_free, c_free[2], full_xh[2], empty_xh[2], full_z[2], empty_z[2],
      a_ready[2], mma_done[2], mbar_cb, cb_free, t_free, y_free[kMaxHeadsPerCta], mma_final,
      e1_done[2];
  uint32_t tmem_holder;
};

static_assert(offsetof(OutShared, cum2) % 16 == 0 && offsetof(OutShared, dt) % 16 == 0 &&
                  offsetof(OutShared, beta) % 16 == 0 && offsetof(OutShared, betad) % 16 == 0 &&
                  offsetof(OutShared, cbd) % 16 == 0 &&
                  offsetof(OutShared, scs) % 16 == 0 && offsetof(OutShared, nw) % 16 == 0 &&
                  offsetof(OutShared, full_cb) % 8 == 0,
              "16-byte accessed shared arrays must be 16-byte aligned");
static_assert(kTcOutTiles % 1024 == 0, "OutShared starts 16-byte aligned");

struct OutMaps {
  CUtensorMap u;   // [b][L][conv_dim] fp16, box 64 ch x 128 tokens
  CUtensorMap z;   // [b][L][d_inner] bf16 (row stride ld_z), box 64 x 128
  CUtensorMap hc;  // [rows][64] fp16, box 64 x 64
  CUtensorMap u2;  // packed sequences: u and z as [L tokens][channels], the same boxes
  CUtensorMap z2;
};

// Release increment of a counter in global memory (gpu scope), and an acquire
// read of it.
__device__ __forceinline__ void red_release_add(unsigned *p, unsigned v) {
  asm volatile("red.release.gpu.global.add.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}
__device__ __forceinline__ unsigned ld_acquire(const unsigned *p) {
  unsigned v;
  asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}
// Waits (bounded) until *cnt >= target; false (and the error flag) if it never gets there.
__device__ __forceinline__ bool wait_count_bounded(const unsigned *cnt, unsigned target) {
  if (ld_acquire(cnt) >= target) return true;
  const unsigned long long t0 = globaltimer_ns();
  while (ld_acquire(cnt) < target) {
    if (globaltimer_ns() - t0 > kWaitLimitNs) {
      atomicOr(&g_tc_errors, kErrWaitTimeout);
      return false;
    }
  }
  return true;
}

// Barriers over one 256-thread group (id 1: operand group, id 2: epilogue group);
// the _and form also returns whether every thread of the group passed `v`.
__device__ __forceinline__ void group_sync(int id) {
  asm volatile("bar.sync %0, 256;" ::"r"(id) : "memory");
}
__device__ __forceinline__ bool group_all(int id, bool v) {
  int r;
  asm volatile("{\n .reg .pred p, q;\n setp.ne.s32 p, %2, 0;\n bar.red.and.pred q, %1, 256, p;\n"
               " selp.s32 %0, 1, 0, q;\n}"
               : "=r"(r)
               : "r"(id), "r"((int)v)
               : "memory");
  return r != 0;
}
__device__ __forceinline__ void st_global_v4(void *p, uint32_t a, uint32_t b, uint32_t c,
                                             uint32_t d) {
  asm volatile("st.global.v4.b32 [%0], {%1, %2, %3, %4};" ::"l"(p), "r"(a), "r"(b), "r"(c), "r"(d)
               : "memory");
}
// 32-byte store (one whole L2 sector), 32-byte aligned address
__device__ __forceinline__ void st_global_v8(void *p, const uint32_t (&v)[8]) {
  asm volatile("st.global.v8.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};" ::"l"(p), "r"(v[0]),
               "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7])
               : "memory");
}

// Unit n of CTA `cid` in a grid of P: (global chunk gc, group g, head block hb);
// key = gc G + g numbers the (chunk, group).  The group's hpg heads are split into
// nhb blocks as evenly as possible: the first hpg % nhb blocks take one head more.
// (Every index fits in 32 bits: the launch checks that the chunks times the
// heads do.)
struct OutUnit {
  int gc, key, g, hb;
  int lh0, nh;  // first head of the block within the group, and its heads
};
__device__ __forceinline__ OutUnit out_unit(const TcArgs &a, int P, int cid, int n) {
  const unsigned u = (unsigned)cid + (unsigned)n * (unsigned)P;
  const unsigned nhb = (unsigned)a.nhb, G = (unsigned)a.pr.G;
  OutUnit o;
  o.key = (int)(u / nhb);
  o.hb = (int)(u - (unsigned)o.key * nhb);
  o.gc = (int)((unsigned)o.key / G);
  o.g = o.key - o.gc * (int)G;
  const int hpg = a.pr.heads_per_group(), base = hpg / a.nhb, rem = hpg - base * a.nhb;
  o.lh0 = o.hb * base + min(o.hb, rem);
  o.nh = base + (o.hb < rem ? 1 : 0);
  return o;
}

// One 32-column group k of row t of the decay operand A_j (j = head), written as
// four 16-byte chunks at column kc (0 or 32) of the 64-wide k-block at `at`:
// zero above the diagonal group, factorised alpha_t beta_s below it, and on it
// either factorised (decay span within 2^60) or with direct exponentials.
__device__ __forceinline__ void build_a_group(const OutShared &sh, int par, int j, int k, int q,
                                              int t, uint32_t at, int kc, uint32_t tmem_cb) {
  const int s0 = 32 * k;
  if (k > q) {
#pragma unroll
    for (int qq = 0; qq < 4; ++qq) st_shared_v4(at + sw128_chunk(t, kc + 8 * qq), 0u, 0u, 0u, 0u);
    return;
  }
  float cb[32];
  tmem_ld32(tmem_cb + s0, cb);
  const float c2t = sh.cum2[par][j][t];
  if (k < q) {
    const float alpha = ex2_approx(c2t - sh.cum2[par][j][s0 + 31]);
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
    return;
  }
  const float Dh = sh.Dh[j];
  if (sh.span_ok[j][k]) {
    // diagonal group, decay span <= 2^60: alpha_t = exp(cum_t - cum_s0) and
    // betad_s = exp(cum_s0 - cum_s) dt_s stay within [2^-60, 2^60]
    const float alpha = ex2_approx(c2t - sh.cum2[par][j][s0]);
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
          if (s == t) vv = fmaf(sh.cbd[t], sh.dt[j][t], Dh);  // exp(0) = 1; fp32 C_t . B_t
          val[u] = (s <= t) ? vv : 0.0f;
        }
        w4[e] = pack_half2(val[0], val[1]);
      }
      st_shared_v4(at + sw128_chunk(t, kc + 8 * qq), w4[0], w4[1], w4[2], w4[3]);
    }
  } else {
    const float4 *c4 = reinterpret_cast<const float4 *>(&sh.cum2[par][j][s0]);
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
          if (s == t) vv = fmaf(sh.cbd[t], sh.dt[j][t], Dh);
          val[u] = (s <= t) ? vv : 0.0f;
        }
        w4[e] = pack_half2(val[0], val[1]);
      }
      st_shared_v4(at + sw128_chunk(t, kc + 8 * qq), w4[0], w4[1], w4[2], w4[3]);
    }
  }
}

// (18 warps: one SM sub-partition holds 5 of them, and 5 x 32 x 96 registers is what
// its quarter of the register file allows)
__global__ void __launch_bounds__(kWsThreads, 1)
    tc_chunk_out_kernel(TcArgs a, const __grid_constant__ OutMaps maps) {
  if (test_stall(&g_tc_stall, &g_tc_errors)) return;  // every CTA alike
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  const Problem &pr = a.pr;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const uint32_t base = (smem_u32(smem_raw) + 1023u) & ~1023u;
  OutShared &sh = *reinterpret_cast<OutShared *>(smem_raw + (base - smem_u32(smem_raw)) +
                                                 kTcOutTiles);
  const int cid = blockIdx.x, P = gridDim.x;
  const int hpg = pr.heads_per_group();
  const int64_t n_all = total_chunks(a) * pr.G * a.nhb;
  const int n_units = n_all > cid ? (int)((n_all - cid + P - 1) / P) : 0;

  if (warp == 0) tmem_alloc(&sh.tmem_holder, 512);
  if (tid == 0) {
    for (int k = 0; k < 2; ++k) {
      mbar_init(&sh.full_cb[k], 1);
      mbar_init(&sh.c_free[k], 1);
      mbar_init(&sh.full_xh[k], 1);
      mbar_init(&sh.empty_xh[k], 1);  // tcgen05.commit after the head's MMAs
      mbar_init(&sh.full_z[k], 1);
      mbar_init(&sh.empty_z[k], kGroupThreads);
      mbar_init(&sh.a_ready[k], kGroupThreads);
      mbar_init(&sh.mma_done[k], 1);
      mbar_init(&sh.e1_done[k], kGroupThreads);  // the epilogue is done with a parity's cum2 / scs
    }
    mbar_init(&sh.b_free, 1);
    mbar_init(&sh.mbar_cb, 1);
    mbar_init(&sh.mma_final, 1);
    mbar_init(&sh.cb_free, kGroupThreads);
    mbar_init(&sh.t_free, kGroupThreads);
    for (int j = 0; j < kMaxHeadsPerCta; ++j) mbar_init(&sh.y_free[j], kGroupThreads);
    fence_mbar_init();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  grid_dependency_wait();  // u, H_c, the scales, the dt rows and the zeroed counters are ready
  const uint32_t tmem = sh.tmem_holder;
  constexpr uint32_t kTmemY = 128;                     // y_j at columns 128 + 64 j

  // normalised bf16 output of head j of unit `un` by a thread of the epilogue group
  // (row t = 32 (warp % 4) + lane, columns 32 ((warp / 4) % 2) .. +31 of the head);
  // the head's TMEM columns go back to the MMA warp as soon as they are read
  auto output_head = [&](int h0, const ChunkPos &pos, int j, float inv) {
    const int q = warp & 3, eh = (warp >> 2) & 1, t = 32 * q + lane;
    const uint32_t lane_off = (uint32_t)(32 * q) << 16;
    const int h = h0 + j;
    const int64_t tok = pos.t0 + t;
    const bool t_valid = t < pos.nv;
    __nv_bfloat16 *yrow = a.y + tok * pr.d_inner + (int64_t)h * kHP + 32 * eh;
    float v32[32];
    tmem_ld32(tmem + lane_off + kTmemY + 64 * j + 32 * eh, v32);
    tc_fence_before();
    mbar_arrive(&sh.y_free[j]);
    if (!t_valid) return;
#pragma unroll
    for (int hh = 0; hh < 2; ++hh) {
      float *v = v32 + 16 * hh;
      if (pr.nbg) {
        const uint4 *zp = reinterpret_cast<const uint4 *>(a.z + tok * a.ld_z +
                                                          (int64_t)h * kHP + 32 * eh + 16 * hh);
#pragma unroll
        for (int qq = 0; qq < 2; ++qq) {
          const uint4 raw = M2_OK(zp + qq, 16, a.sp.z, &g_tc_errors) ? __ldg(zp + qq)
                                                                      : make_uint4(0, 0, 0, 0);
          const __nv_bfloat162 *h2 = reinterpret_cast<const __nv_bfloat162 *>(&raw);
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const float2 f = __bfloat1622float2(h2[i]);
            v[8 * qq + 2 * i] *= silu_fast(f.x);
            v[8 * qq + 2 * i + 1] *= silu_fast(f.y);
          }
        }
      }
      const float4 *nw4 = reinterpret_cast<const float4 *>(&sh.nw[j][32 * eh + 16 * hh]);
      uint32_t o[8];
#pragma unroll
      for (int qq = 0; qq < 2; ++qq) {
        const float4 wA = nw4[2 * qq], wB = nw4[2 * qq + 1];
        const float ww[8] = {wA.x, wA.y, wA.z, wA.w, wB.x, wB.y, wB.z, wB.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int i = 8 * qq + 2 * e;
          const __nv_bfloat162 b2 =
              __floats2bfloat162_rn(v[i] * inv * ww[2 * e], v[i + 1] * inv * ww[2 * e + 1]);
          o[4 * qq + e] = *reinterpret_cast<const uint32_t *>(&b2);
        }
      }
      __nv_bfloat16 *yp = yrow + 16 * hh;  // 16 columns = 32 bytes
      if (a.y32) {
        if (M2_OK(yp, 16, a.sp.y, &g_tc_errors) && M2_OK(yp + 8, 16, a.sp.y, &g_tc_errors))
          st_global_v8(yp, o);
      } else {
#pragma unroll
        for (int qq = 0; qq < 2; ++qq)
          if (M2_OK(yp + 8 * qq, 16, a.sp.y, &g_tc_errors))
            st_global_v4(yp + 8 * qq, o[4 * qq], o[4 * qq + 1], o[4 * qq + 2], o[4 * qq + 3]);
      }
    }
  };
  if (warp == 16) {
    // ---------------- producer
    if (lane == 0) {
      bool ok = true;
      int J = 0, ncb = 0, nxh = 0, nz = 0;  // copies issued into each ring
      // a [128 tokens][64 ch] tile of u or z for the unit at `pos`
      auto load_tok = [&](uint32_t dst, const CUtensorMap *m3, const CUtensorMap *m2, int ch,
                          const ChunkPos &pos, uint64_t *bar) {
        if (a.varlen) tma_load_2d(dst, m2, ch, (int)pos.t0, bar);
        else tma_load_3d(dst, m3, ch, pos.c * kQ, pos.seq, bar);
      };
      auto load_cb = [&](int n) {  // C and B tiles of unit n
        const OutUnit ou = out_unit(a, P, cid, n);
        const int64_t gc = ou.gc;
        const int g = ou.g;
        const ChunkPos pos = chunk_pos(a, gc);
        const int cbuf = n & 1;
        if (n >= 2) ok = ok && mbar_wait_bounded(&sh.c_free[cbuf], (uint32_t)(((n - 2) >> 1) & 1), &g_tc_errors);
        if (n >= 1) ok = ok && mbar_wait_bounded(&sh.b_free, (uint32_t)((n - 1) & 1), &g_tc_errors);
        if (!ok) return;
        mbar_arrive_expect_tx(&sh.full_cb[cbuf], 2 * 16384);
        load_tok(base + kCt0 + cbuf * 16384, &maps.u, &maps.u2,
                 (int)(pr.d_inner + (int64_t)(pr.G + g) * kNS), pos, &sh.full_cb[cbuf]);
        load_tok(base + kBt, &maps.u, &maps.u2, (int)(pr.d_inner + (int64_t)g * kNS), pos,
                 &sh.full_cb[cbuf]);
        ++ncb;
      };
      if (n_units > 0) load_cb(0);
      for (int n = 0; ok && n < n_units; ++n) {
        const OutUnit ou = out_unit(a, P, cid, n);
        const int64_t gc = ou.gc;
        const int nh = ou.nh;
        const ChunkPos pos = chunk_pos(a, gc);
        const int h0 = ou.g * hpg + ou.lh0;
        for (int j = 0; ok && j < nh; ++j, ++J) {
          const int h = h0 + j, sl = J & 1;
          if (J >= 2) ok = mbar_wait_bounded(&sh.empty_xh[sl], (uint32_t)(((J - 2) >> 1) & 1), &g_tc_errors);
          if (!ok) break;
          mbar_arrive_expect_tx(&sh.full_xh[sl], kXhBytes);
          load_tok(base + kXh + sl * kXhBytes, &maps.u, &maps.u2, h * kHP, pos, &sh.full_xh[sl]);
          tma_load_2d(base + kXh + sl * kXhBytes + 16384, &maps.hc, 0,
                      (int)((gc * pr.H + h) * kHP), &sh.full_xh[sl]);
          ++nxh;
          if (J >= 2) ok = mbar_wait_bounded(&sh.empty_z[sl], (uint32_t)(((J - 2) >> 1) & 1), &g_tc_errors);
          if (!ok) break;
          mbar_arrive_expect_tx(&sh.full_z[sl], 16384);
          load_tok(base + kZt + sl * 16384, &maps.z, &maps.z2, h * kHP, pos, &sh.full_z[sl]);
          ++nz;
          if (j == min(1, nh - 1) && n + 1 < n_units) load_cb(n + 1);
        }
      }
      // no copy may be in flight when the CTA exits: the last copies into each ring
      for (int k = max(0, ncb - 2); k < ncb; ++k)
        mbar_wait_bounded(&sh.full_cb[k & 1], (uint32_t)((k >> 1) & 1), &g_tc_errors);
      for (int k = max(0, nxh - 2); k < nxh; ++k)
        mbar_wait_bounded(&sh.full_xh[k & 1], (uint32_t)((k >> 1) & 1), &g_tc_errors);
      for (int k = max(0, nz - 2); k < nz; ++k)
        mbar_wait_bounded(&sh.full_z[k & 1], (uint32_t)((k >> 1) & 1), &g_tc_errors);
    }
  } else if (warp == 17) {
    // ---------------- MMA issuer
    if (lane == 0) {
      const uint32_t idesc_cb = umma_idesc_f16(128, 128);
      const uint32_t idesc_mn = umma_idesc_f16(128, 64) | (1u << 16);  // B operand MN-major
      int J = 0;
      bool ok = true;
      for (int n = 0; ok && n < n_units; ++n) {
        const int cbuf = n & 1;
        const uint32_t ct = base + kCt0 + cbuf * 16384;
        ok = mbar_wait_bounded(&sh.full_cb[cbuf], (uint32_t)((n >> 1) & 1), &g_tc_errors) &&
             (n == 0 || mbar_wait_bounded(&sh.cb_free, (uint32_t)((n - 1) & 1), &g_tc_errors));
        if (!ok) break;
        tc_fence_after();
        // CB = C B^T : M = 128 (t), N = 128 (s), K = 64 (n)
        for (int kin = 0; kin < 4; ++kin)
          umma_f16(tmem, umma_desc_sw128(ct + kin * 32), umma_desc_sw128(base + kBt + kin * 32),
                   idesc_cb, kin > 0 ? 1u : 0u);
        umma_commit(&sh.mbar_cb);
        umma_commit(&sh.b_free);
        const int nh = out_unit(a, P, cid, n).nh;
        for (int j = 0; j < nh; ++j, ++J) {
          const int sl = J & 1;
          ok = mbar_wait_bounded(&sh.a_ready[sl], (uint32_t)((J >> 1) & 1), &g_tc_errors) &&
               mbar_wait_bounded(&sh.full_xh[sl], (uint32_t)((J >> 1) & 1), &g_tc_errors) &&
               (n == 0 || mbar_wait_bounded(&sh.y_free[j], (uint32_t)((n - 1) & 1), &g_tc_errors));
          if (!ok) break;
          tc_fence_after();
          const uint32_t xt = base + kXh + sl * kXhBytes, ht = xt + 16384;
          const uint32_t ab = base + kAbuf + sl * 32768;
          // y_j = [CB o L o dt (+D)] x : K = 128 (x [s][p] MN-major)
          for (int ks = 0; ks < 8; ++ks)
            umma_f16(tmem + kTmemY + 64 * j, umma_desc_sw128(ab + (ks >> 2) * 16384 + (ks & 3) * 32),
                     umma_desc_sw128_mn(xt + ks * 2048, 16384), idesc_mn, ks > 0 ? 1u : 0u);
          // T = C H_c^T : K = 64 (n), H_c [n][p] MN-major; once the epilogue has read the
          // previous head's T
          if (J > 0 && !mbar_wait_bounded(&sh.t_free, (uint32_t)((J - 1) & 1), &g_tc_errors)) {
            ok = false;
            break;
          }
          tc_fence_after();
          for (int kin = 0; kin < 4; ++kin)
            umma_f16(tmem + kTmemT, umma_desc_sw128(ct + kin * 32),
                     umma_desc_sw128_mn(ht + kin * 2048, 8192), idesc_mn, kin > 0 ? 1u : 0u);
          umma_commit(&sh.mma_done[sl]);
          umma_commit(&sh.empty_xh[sl]);  // its x / H_c stage is free once they complete
        }
        if (ok) umma_commit(&sh.c_free[cbuf]);
      }
      // no MMA may be in flight when the CTA frees its tensor memory: one more commit
      // tracks every MMA this thread issued, whichever way the loop ended
      umma_commit(&sh.mma_final);
      mbar_wait_bounded(&sh.mma_final, 0, &g_tc_errors);
    }
  } else if (warp < 8) {
    // ---------------- decay operands
    const int q = warp & 3, blk = warp >> 2, t = 32 * q + lane;
    const uint32_t lane_off = (uint32_t)(32 * q) << 16;
    bool ok = true;
    int J = 0;
    for (int n = 0; ok && n < n_units; ++n) {
      const OutUnit ou = out_unit(a, P, cid, n);
      const int64_t gc = ou.gc;
      const int g = ou.g, nh = ou.nh;
      const int h0 = g * hpg + ou.lh0;
      const int par = n & 1;
      // the epilogue reads this parity's exp(cum) and scales of unit n - 2 until it is done
      // with that unit's gate pass
      if (n >= 2) {
        const bool got = mbar_wait_bounded(&sh.e1_done[par], (uint32_t)(((n - 2) >> 1) & 1), &g_tc_errors);
        ok = group_all(1, got);
        if (!ok) break;
      }
      // decay terms of head j = warp (from the per-chunk dt and cumsum rows)
      if (warp < nh) {
        const int j = warp;
        const int64_t row = gc * pr.H + h0 + j;
        const float4 *cup = reinterpret_cast<const float4 *>(a.cum + row * kQ) + lane;
        const float4 *dvp = reinterpret_cast<const float4 *>(a.dtv + row * kQ) + lane;
        const float4 z4 = make_float4(0.f, 0.f, 0.f, 0.f);
        const float4 cu = M2_OK(cup, 16, a.sp.cum, &g_tc_errors) ? *cup : z4;
        const float4 dv = M2_OK(dvp, 16, a.sp.dtv, &g_tc_errors) ? *dvp : z4;
        const float cum4[4] = {cu.x, cu.y, cu.z, cu.w}, dt4[4] = {dv.x, dv.y, dv.z, dv.w};
        float c2[4];
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          c2[k] = cum4[k] * kLog2e;
          sh.cum2[par][j][4 * lane + k] = c2[k];
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
        // for the epilogue: the exponents of H_c's row-pair scales (powers of two >= 1)
        const float *scp = a.hsc + row * 32 + lane;
        const float scv = M2_OK(scp, 4, a.sp.hsc, &g_tc_errors) ? *scp : 1.0f;
        sh.scs[par][j][lane] = (uint8_t)((__float_as_uint(scv) >> 23) - 127u);
        if (lane == 0)
          sh.Dh[j] = M2_OK(a.prm.D + h0 + j, 4, a.sp.D, &g_tc_errors) ? a.prm.D[h0 + j] : 0.0f;
      }
      if (warp == 7) {  // the unit's fp32 diagonal C_t . B_t
        const float4 *src = reinterpret_cast<const float4 *>(a.cbd + (gc * pr.G + g) * kQ) + lane;
        reinterpret_cast<float4 *>(sh.cbd)[lane] =
            M2_OK(src, 16, a.sp.cbd, &g_tc_errors) ? *src : make_float4(0.f, 0.f, 0.f, 0.f);
      }
      group_sync(1);
      for (int j = 0; j < nh; ++j, ++J) {
        const int sl = J & 1;
        if (j == 0) ok = mbar_wait_bounded(&sh.mbar_cb, (uint32_t)(n & 1), &g_tc_errors);
        // A buffer sl is free once the MMAs of head J - 2 (which read it) completed
        if (ok && J >= 2) ok = mbar_wait_bounded(&sh.mma_done[sl], (uint32_t)(((J - 2) >> 1) & 1), &g_tc_errors);
        ok = __all_sync(0xffffffffu, ok) != 0;
        if (!ok) break;
        tc_fence_after();
        const uint32_t at = base + kAbuf + sl * 32768 + blk * 16384;
        build_a_group(sh, par, j, 2 * blk, q, t, at, 0, tmem + lane_off);
        build_a_group(sh, par, j, 2 * blk + 1, q, t, at, 32, tmem + lane_off);
        fence_proxy_async_smem();
        tc_fence_before();
        mbar_arrive(&sh.a_ready[sl]);
      }
      // this unit's CB columns and decay terms are no longer read
      tc_fence_before();
      if (ok) mbar_arrive(&sh.cb_free);
      ok = group_all(1, ok);
    }

  } else {
    // ---------------- epilogue
    const int q = warp & 3, eh = (warp - 8) >> 2, t = 32 * q + lane, gt = tid - 256;
    const uint32_t lane_off = (uint32_t)(32 * q) << 16;
    bool ok = true;
    int J = 0;
    for (int n = 0; ok && n < n_units; ++n) {
      const OutUnit ou = out_unit(a, P, cid, n);
      const int nh = ou.nh;
      const int h0 = ou.g * hpg + ou.lh0;
      const int par = n & 1;
      float ss = 0.0f;
      for (int j = 0; j < nh; ++j, ++J) {
        const int sl = J & 1;
        ok = ok && mbar_wait_bounded(&sh.mma_done[sl], (uint32_t)((J >> 1) & 1), &g_tc_errors) &&
             mbar_wait_bounded(&sh.full_z[sl], (uint32_t)((J >> 1) & 1), &g_tc_errors);
        ok = __all_sync(0xffffffffu, ok) != 0;
        if (!ok) break;
        tc_fence_after();
        const float ec = ex2_approx(sh.cum2[par][j][t]);  // exp(cum_t)
        const uint32_t ycol = tmem + lane_off + kTmemY + 64 * j + 32 * eh;
        const uint32_t zt = base + kZt + sl * 16384;
        // this thread's 32 columns of C H_c^T first, together with the first 16 of
        // y_j, so that the shared accumulator can take the next head's product early
        float w32[32], v[16];
        tmem_ld32x16(tmem + lane_off + kTmemT + 32 * eh, w32, ycol, v);
        tc_fence_before();
        mbar_arrive(&sh.t_free);  // the C H_c^T columns may take the next head's product
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
          if (hh == 1) tmem_ld16(ycol + 16, v);
          const float *w = w32 + 16 * hh;
          // the scales 2^s of H_c's rows p (pairs) of these 16 columns, from their exponents
          const uint2 se = *reinterpret_cast<const uint2 *>(&sh.scs[par][j][16 * eh + 8 * hh]);
          float scp[8];
#pragma unroll
          for (int i = 0; i < 8; ++i)
            scp[i] = __uint_as_float((127u + (((i < 4 ? se.x : se.y) >> (8 * (i & 3))) & 0xFFu)) << 23);
#pragma unroll
          for (int i = 0; i < 16; ++i) v[i] = fmaf(ec * scp[i >> 1], w[i], v[i]);
          if (!pr.nbg) {
#pragma unroll
            for (int qq = 0; qq < 2; ++qq) {
              const uint4 raw = ld_shared_v4(zt + sw128_chunk(t, 32 * eh + 16 * hh + 8 * qq));
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
          for (int i = 0; i < 16; ++i) ss = fmaf(v[i], v[i], ss);
          tmem_st16_async(ycol + 16 * hh, v);
        }
        mbar_arrive(&sh.empty_z[sl]);
      }
      tmem_wait_st();  // the gated values are in TMEM before this thread reads them back
      mbar_arrive(&sh.e1_done[par]);
      // the unit's norm weights: loads issued now, stored to shared memory once the
      // exchange below has been waited for (their latency overlaps it)
      float nwv[2] = {0.0f, 0.0f};
#pragma unroll
      for (int r = 0; r < 2; ++r) {
        const int idx = gt + kGroupThreads * r;
        if (idx < nh * kHP) {
          const float *wp = a.prm.norm_w + (int64_t)(h0 + idx / kHP) * kHP + idx % kHP;
          nwv[r] = M2_OK(wp, 4, a.sp.norm_w, &g_tc_errors) ? __ldg(wp) : 0.0f;
        }
      }
      // the block's per-token sums into row hb of the (chunk, group)'s exchange slot
      sh.half_ss[eh][t] = ss;
      ok = group_all(2, ok);
      if (!ok) break;
      float *xslot = a.xpart + (int64_t)ou.key * a.nhb * kQ;
      unsigned *xcnt = a.xcnt + ou.key;
      if (gt < kQ) {
        float *dst = xslot + ou.hb * kQ + gt;
        if (M2_OK(dst, 4, a.sp.xpart, &g_tc_errors)) __stcg(dst, sh.half_ss[0][gt] + sh.half_ss[1][gt]);
      }
      group_sync(2);  // every row of the block is written before it is counted
      bool got = true;
      if (gt == 0 && M2_OK(xcnt, 4, a.sp.xcnt, &g_tc_errors)) {
        // (release: the rows the group wrote before the barrier are visible first)
        red_release_add(xcnt, 1u);
        got = wait_count_bounded(xcnt, (unsigned)a.nhb);
      }
      ok = group_all(2, got);
      if (!ok) break;
      float tot = 0.0f;  // blocks in order: the same sum in every block's CTA
      for (int r0 = 0; r0 < a.nhb; r0 += 16) {
        float pv[16];  // (loads issued together, added in order)
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          const float *src = xslot + (r0 + i) * kQ + t;
          pv[i] = (r0 + i < a.nhb && M2_OK(src, 4, a.sp.xpart, &g_tc_errors)) ? __ldcg(src) : 0.0f;
        }
#pragma unroll
        for (int i = 0; i < 16; ++i)
          if (r0 + i < a.nhb) tot += pv[i];
      }
      const float inv = rsqrtf(tot / (float)(hpg * kHP) + pr.eps);
#pragma unroll
      for (int r = 0; r < 2; ++r) {
        const int idx = gt + kGroupThreads * r;
        if (idx < nh * kHP) sh.nw[idx / kHP][idx % kHP] = nwv[r];
      }
      ok = group_all(2, ok);
      if (!ok) break;
      // normalised bf16 output, head by head; each head's TMEM columns go back to the
      // MMA warp (for the next unit) as soon as they are read.  Slots this unit
      // leaves empty (a smaller head block) are handed back too, so that every
      // slot's barrier completes once per unit
      const ChunkPos pos = chunk_pos(a, ou.gc);
      for (int j = 0; j < nh; ++j) output_head(h0, pos, j, inv);
      for (int j = nh; j < a.hpc; ++j) mbar_arrive(&sh.y_free[j]);
    }
  }
  __syncwarp();
  tc_fence_before();
  __syncthreads();
  if (warp == 0) tmem_dealloc(tmem, 512);
}


// Most head blocks per group the output kernel uses (blocks of 2 heads or more,
// unless a group has one head): the size of the exchange.
int out_max_blocks(int hpg) { return hpg <= 1 ? 1 : (hpg + 1) / 2; }

// Head blocks of the output kernel for hpg heads per group and `keys` (chunk,
// group) pairs on `sms` SMs: every block size h = 2 .. 5 (1 for a single head)
// gives nhb = ceil(hpg / h) blocks and a grid of the largest multiple of nhb that
// fits the SMs; the choice minimises the rounds of units times (heads per block +
// a per-unit cost of about 2.5 heads).  False if no block size fits (more than
// 5 x sms heads).
bool out_choose(int hpg, int64_t keys, int sms, int *hpc, int *nhb, int *grid) {
  int64_t best = -1;
  for (int h = std::min(hpg, 2); h <= kMaxHeadsPerCta; ++h) {
    const int nb = (hpg + h - 1) / h;
    if (nb > sms) continue;
    const int hh = (hpg + nb - 1) / nb;  // the largest block after evening out
    const int64_t units = keys * nb;
    const int64_t P = std::min<int64_t>((int64_t)(sms / nb) * nb, units);
    const int64_t rounds = (units + P - 1) / P;
    const int64_t score = rounds * (2 * hh + 5);
    if (best < 0 || score < best) {
      best = score;
      *hpc = hh;
      *nhb = nb;
      *grid = (int)P;
    }
  }
  return best >= 0;
}

struct TcWorkspace {
  float *S, *cum_end, *cum, *dtv, *hsc, *smax, *cbd, *xpart;
  unsigned *xcnt;
  __half *Hc, *u;
  int4 *vl_chunks;
  int *vl_chunk0;
  float *vl_h0max;
};

// Chunks the workspace holds: b * ceil(L / 128), or for packed sequences an
// upper bound on the sum of their chunk counts, ceil(L / 128) + b.
int64_t tc_chunk_cap(const Problem &pr, bool varlen) {
  return varlen ? ceil_div(pr.L, kQ) + pr.batch : pr.batch * ceil_div(pr.L, kQ);
}

// Carves the workspace (or, with base null, measures it).
size_t tc_carve(const Problem &pr, bool varlen, char *base, TcWorkspace *w) {
  const size_t cap = (size_t)tc_chunk_cap(pr, varlen);
  const size_t st = cap * pr.H * kHP * kNS;
  size_t off = 0;
  auto take = [&](size_t bytes) -> char * {
    char *p = base == nullptr ? nullptr : base + off;
    off += align_up(bytes, 256);
    return p;
  };
  TcWorkspace t;
  t.S = reinterpret_cast<float *>(take(st * 4));
  t.cum_end = reinterpret_cast<float *>(take(cap * pr.H * 4));
  t.cum = reinterpret_cast<float *>(take(cap * pr.H * kQ * 4));
  t.dtv = reinterpret_cast<float *>(take(cap * pr.H * kQ * 4));
  t.Hc = reinterpret_cast<__half *>(take(st * 2));
  t.hsc = reinterpret_cast<float *>(take(cap * pr.H * 32 * 4));
  t.smax = reinterpret_cast<float *>(take(cap * pr.H * 4));
  t.cbd = reinterpret_cast<float *>(take(cap * pr.G * kQ * 4));
  // output-kernel exchange: at most hpg head blocks per (chunk, group)
  t.xpart = reinterpret_cast<float *>(take(cap * pr.G * out_max_blocks(pr.heads_per_group()) * kQ * 4));
  t.xcnt = reinterpret_cast<unsigned *>(take(cap * pr.G * 4));
  t.vl_chunks = varlen ? reinterpret_cast<int4 *>(take(cap * 16)) : nullptr;
  t.vl_chunk0 = varlen ? reinterpret_cast<int *>(take((size_t)(pr.batch + 2) * 4)) : nullptr;
  t.vl_h0max = varlen ? reinterpret_cast<float *>(take((size_t)pr.batch * pr.H * 4)) : nullptr;
  const size_t tokens = varlen ? (size_t)pr.L : (size_t)(pr.batch * pr.L);
  t.u = reinterpret_cast<__half *>(take(tokens * pr.conv_dim * 2));
  if (w != nullptr) *w = t;
  return off;
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
// (each kernel that uses tensor memory also holds 1 KB of static shared memory; the
// chunk-state kernel's own static arrays take 12 KB more)
static_assert(kK1Smem + 14 * 1024 <= 227 * 1024 && kK3Smem + 1024 <= 227 * 1024,
              "shared memory per CTA");

}  // namespace

const char *const kPrefillTcStages[] = {"tc_chunk_state", "tc_state_pass", "tc_chunk_out"};
const int kPrefillTcStageCount = 3;

bool prefill_tc_supported(const Problem &pr, bool varlen) {
  const int64_t nch = ceil_div(pr.L, kQ), cap = tc_chunk_cap(pr, varlen);
  const int64_t pairs = (pr.heads_per_group() + 1) / 2;
  return pr.io == MAMBA2_BF16 && pr.P == kHP && pr.N == kNS && pr.K == 4 &&
         pr.heads_per_group() <= kMaxHeadsPerCta * 128 && pr.L > 0 &&
         (varlen || nch <= 65535) && pr.L < ((int64_t)1 << 31) &&
         pr.batch * pr.L < ((int64_t)1 << 31) && cap * pr.H * kHP < ((int64_t)1 << 31) &&
         cap * pr.G * (pairs + 1) < ((int64_t)1 << 31);
}

size_t prefill_tc_workspace(const Problem &pr, bool varlen) {
  return tc_carve(pr, varlen, nullptr, nullptr);
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
  a.y32 = (reinterpret_cast<uintptr_t>(pa.y) % 32) == 0;
  a.conv_in = static_cast<const __nv_bfloat16 *>(pa.conv_state);
  a.ssm_state = pa.ssm_state;
  a.states_in = pa.states_in;
  const bool varlen = pa.cu_seqlens != nullptr;
  a.nch = (int)ceil_div(pr.L, kQ);
  TcWorkspace w;
  tc_carve(pr, varlen, pa.ws, &w);
  a.varlen = varlen ? 1 : 0;
  a.vl_chunks = w.vl_chunks;
  a.vl_chunk0 = w.vl_chunk0;
  a.vl_h0max = varlen && pa.states_in ? w.vl_h0max : nullptr;
  a.cu_seqlens = pa.cu_seqlens;
  const int64_t cap = tc_chunk_cap(pr, varlen);    // chunks the workspace holds
  const int64_t tokens = varlen ? pr.L : pr.batch * pr.L;
  a.S = w.S;
  a.cum_end = w.cum_end;
  a.cum = w.cum;
  a.dtv = w.dtv;
  a.Hc = w.Hc;
  a.hsc = w.hsc;
  a.smax = w.smax;
  a.cbd = w.cbd;
  a.u = w.u;
  a.xpart = w.xpart;
  a.xcnt = w.xcnt;
  a.xkeys = cap * pr.G;
  {
    const int64_t bl = tokens, nq = cap, nrow = 1;  // chunk arrays: cap chunks
    const size_t st1 = (size_t)nrow * nq * pr.H * kHP * kNS;
    a.sp.xbc = span_of(a.xBC, (size_t)((bl - 1) * pa.ld_xbc + pr.conv_dim) * 2);
    a.sp.z = span_of(a.z, (size_t)((bl - 1) * pa.ld_z + pr.d_inner) * 2);
    a.sp.dt = span_of(a.dt_raw, (size_t)((bl - 1) * pa.ld_dt + pr.H) * 2);
    a.sp.y = span_of(a.y, (size_t)bl * pr.d_inner * 2);
    a.sp.conv = span_of(pa.conv_state, (size_t)pr.batch * pr.conv_dim * 4 * 2);
    a.sp.ssm = span_of(a.ssm_state, (size_t)pr.batch * pr.H * kHP * kNS * 4);
    a.sp.S = span_of(a.S, st1 * 4);
    a.sp.cum_end = span_of(a.cum_end, (size_t)nq * pr.H * 4);
    a.sp.cum = span_of(a.cum, (size_t)nq * pr.H * kQ * 4);
    a.sp.dtv = span_of(a.dtv, (size_t)nq * pr.H * kQ * 4);
    a.sp.Hc = span_of(a.Hc, st1 * 2);
    a.sp.hsc = span_of(a.hsc, (size_t)nq * pr.H * 32 * 4);
    a.sp.smax = span_of(a.smax, (size_t)nq * pr.H * 4);
    a.sp.cbd = span_of(a.cbd, (size_t)pr.G * nq * kQ * 4);
    a.sp.xpart = span_of(a.xpart, (size_t)nq * pr.G * out_max_blocks(pr.heads_per_group()) * kQ * 4);
    a.sp.xcnt = span_of(a.xcnt, (size_t)nq * pr.G * 4);
    a.sp.u = span_of(a.u, (size_t)bl * pr.conv_dim * 2);
    a.sp.conv_w = span_of(a.prm.conv_w, (size_t)pr.conv_dim * 4 * 4);
    a.sp.conv_b = span_of(a.prm.conv_b, (size_t)pr.conv_dim * 4);
    a.sp.dt_bias = span_of(a.prm.dt_bias, (size_t)pr.H * 4);
    a.sp.A = span_of(a.prm.A, (size_t)pr.H * 4);
    a.sp.D = span_of(a.prm.D, (size_t)pr.H * 4);
    a.sp.norm_w = span_of(a.prm.norm_w, (size_t)pr.d_inner * 4);
    a.sp.h0max = span_of(a.vl_h0max, (size_t)pr.batch * pr.H * 4);
  }
  const int hpg = pr.heads_per_group();
  cudaError_t e;
  if (first_use_in_context(0)) {  // attributes belong to the context: set them once in each
    e = cudaFuncSetAttribute(tc_chunk_state_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)kK1Smem);
    if (e != cudaSuccess) return e;
    e = cudaFuncSetAttribute(tc_chunk_out_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)kK3Smem);
    if (e != cudaSuccess) return e;
  }
  // the output kernel's head blocks and grid (one CTA per SM, all resident at once)
  int hpc = 1, nhb = 1, grid3 = 1;
  if (!out_choose(hpg, cap * (int64_t)pr.G, sm_count(), &hpc, &nhb, &grid3))
    return cudaErrorNotSupported;
  a.hpc = hpc;
  a.nhb = nhb;

  stage_mark(st, 0);
  if (varlen) {  // the chunks of the packed sequences
    const unsigned gp = 1u + (a.vl_h0max != nullptr ? (unsigned)(pr.batch * pr.H) : 0u);
    tc_varlen_prep_kernel<<<gp, kPrepThreads, 0, st>>>(pa.cu_seqlens, (int)pr.batch, pr.L, cap,
                                                       w.vl_chunks, w.vl_chunk0, pa.ssm_state,
                                                       w.vl_h0max, a.sp.ssm);
  }
  const int64_t n_items = cap * (int64_t)pr.G * ((hpg + 1) / 2 + 1);
  const unsigned g1 = (unsigned)std::min<int64_t>(n_items, sm_count());
  {
    NvtxRange r1("tc_chunk_state");
    K1Maps m1;
    std::memset(&m1, 0, sizeof(m1));
    const uint32_t bx[3] = {64, kRawRows, 1};
    if (varlen) {
      const uint64_t dx[2] = {(uint64_t)pr.conv_dim, (uint64_t)pr.L};
      const uint64_t sx[1] = {(uint64_t)pa.ld_xbc * 2};
      if (!make_map(&m1.xbc2, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, a.xBC, 2, dx, sx, bx))
        return cudaErrorInvalidValue;
    } else {
      const uint64_t dx[3] = {(uint64_t)pr.conv_dim, (uint64_t)pr.L, (uint64_t)pr.batch};
      const uint64_t sx[2] = {(uint64_t)pa.ld_xbc * 2, (uint64_t)pr.L * pa.ld_xbc * 2};
      if (!make_map(&m1.xbc, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, a.xBC, 3, dx, sx, bx))
        return cudaErrorInvalidValue;
    }
    tc_chunk_state_kernel<<<g1, kK1Threads, kK1Smem, st>>>(a, m1, (int)n_items);
  }
  stage_mark(st, 1);
  NvtxRange r2("tc_state_pass + tc_chunk_out");
  dim3 g2((unsigned)(pr.H * kPassBlocks + ceil_div(pr.conv_dim, kPassThreads)), (unsigned)pr.batch, 1);
  {
    // programmatic dependent launches: the state pass and the output kernel are
    // scheduled while their predecessor drains and wait for it on the device
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = g2;
    cfg.blockDim = dim3(kPassThreads, 1, 1);
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    e = cudaLaunchKernelEx(&cfg, tc_state_pass_kernel, a,
                           static_cast<__nv_bfloat16 *>(pa.conv_state));
    if (e != cudaSuccess) return e;
  }
  stage_mark(st, 2);
  {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)grid3, 1, 1);
    cfg.blockDim = dim3(kWsThreads, 1, 1);
    cfg.dynamicSmemBytes = kK3Smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    OutMaps maps;
    std::memset(&maps, 0, sizeof(maps));
    {
      const uint32_t bu[3] = {64, kQ, 1};
      const uint64_t dh[2] = {(uint64_t)kNS, (uint64_t)(cap * pr.H * kHP)};
      const uint64_t shc[1] = {(uint64_t)kNS * 2};
      const uint32_t bh[2] = {64, 64};
      if (!make_map(&maps.hc, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, a.Hc, 2, dh, shc, bh))
        return cudaErrorInvalidValue;
      if (varlen) {
        const uint64_t du[2] = {(uint64_t)pr.conv_dim, (uint64_t)pr.L};
        const uint64_t su[1] = {(uint64_t)pr.conv_dim * 2};
        const uint64_t dz[2] = {(uint64_t)pr.d_inner, (uint64_t)pr.L};
        const uint64_t sz[1] = {(uint64_t)pa.ld_z * 2};
        if (!make_map(&maps.u2, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, a.u, 2, du, su, bu) ||
            !make_map(&maps.z2, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, a.z, 2, dz, sz, bu))
          return cudaErrorInvalidValue;
      } else {
        const uint64_t du[3] = {(uint64_t)pr.conv_dim, (uint64_t)pr.L, (uint64_t)pr.batch};
        const uint64_t su[2] = {(uint64_t)pr.conv_dim * 2, (uint64_t)pr.L * pr.conv_dim * 2};
        const uint64_t dz[3] = {(uint64_t)pr.d_inner, (uint64_t)pr.L, (uint64_t)pr.batch};
        const uint64_t sz[2] = {(uint64_t)pa.ld_z * 2, (uint64_t)pr.L * pa.ld_z * 2};
        if (!make_map(&maps.u, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, a.u, 3, du, su, bu) ||
            !make_map(&maps.z, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, a.z, 3, dz, sz, bu))
          return cudaErrorInvalidValue;
      }
    }
    e = cudaLaunchKernelEx(&cfg, tc_chunk_out_kernel, a, maps);
    if (e != cudaSuccess) return e;
  }
  stage_mark(st, 3);
  return cudaGetLastError();
}

}  // namespace m2
