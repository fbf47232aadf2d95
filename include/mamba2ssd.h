/*
 * mamba2ssd.h -- C ABI of the B200 (sm_100a) Mamba-2 mixer core library
 * (libmamba2ssd.so).
 *
 * The mixer core is the middle of a Zamba2 Mamba2 layer, between in_proj and
 * out_proj ("Zamba2 hybrid architecture in Transformers", qwbw.cn, section 三
 * "Mamba2 Mixer", steps 2-4):
 *   1. causal depthwise conv1d (width d_conv = 4, with bias) + SiLU over the
 *      x | B | C channels (conv_dim = d_inner + 2 * ngroups * d_state);
 *   2. dt = softplus(dt_raw + dt_bias) per head;
 *   3. the selective state-space scan of the Mamba-2 (state-space duality)
 *      layer named on the state-spaces/mamba repository page (opendeer.net,
 *      "About the project"):
 *          h_t = exp(dt_t * A_h) * h_{t-1} + dt_t * x_t B_t^T     (h: [P, N])
 *          y_t = C_t h_t + D_h * x_t
 *      evaluated chunk by chunk for prefill and as a single-token update for
 *      decode (section 三 step 3);
 *   4. gated group RMSNorm: out = rmsnorm(y * silu(z)) * norm_w over groups
 *      of d_inner / ngroups channels, eps from the dims (section 三 step 4,
 *      section 五 rms_norm_eps = 1e-5); norm_before_gate = 1 selects
 *      rmsnorm(y) * norm_w * silu(z).
 * The conv state and SSM state that the pages keep in the model cache
 * (section 三) are caller-owned buffers passed to every call.
 *
 * Conventions shared by every entry point
 *  - All data pointers are DEVICE pointers of the current CUDA device, except
 *    `dims` and `params` themselves (host structs; the arrays they point to
 *    are device arrays).  The library never allocates device memory, never
 *    synchronises the stream and keeps no pointer after a call returns.
 *  - Work is enqueued on `stream` (a cudaStream_t passed as void*; NULL is
 *    the legacy default stream) and runs asynchronously: a return of
 *    MAMBA2_OK means the arguments were valid and the launches were enqueued.
 *  - Layouts are row-major.  Channel c of xBC is x for c < d_inner (head h,
 *    lane p at h*P + p), then B (ngroups * d_state, group-major), then C.
 *    Head h uses B/C group h / (nheads / ngroups).
 *  - Outputs must not alias inputs; the conv and SSM state buffers are read
 *    and then overwritten in place.
 *  - Errors are returned, never thrown; on any status other than MAMBA2_OK
 *    from argument validation nothing was enqueued.  MAMBA2_ERR_CUDA reports
 *    a launch error (cudaGetLastError) after enqueueing.
 */
#ifndef MAMBA2SSD_H
#define MAMBA2SSD_H

#include <stddef.h>
#include <stdint.h>

#if defined(_WIN32)
#define MAMBA2_API __declspec(dllexport)
#else
#define MAMBA2_API __attribute__((visibility("default")))
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  MAMBA2_OK = 0,
  MAMBA2_ERR_INVALID_ARG = -1, /* null pointer, bad size, stride or alignment */
  MAMBA2_ERR_UNSUPPORTED = -2, /* valid in principle, not built (e.g. d_conv != 4) */
  MAMBA2_ERR_WORKSPACE = -3,   /* workspace missing or smaller than required */
  MAMBA2_ERR_CUDA = -4         /* a CUDA launch or runtime call failed */
} mamba2_status;

typedef enum {
  MAMBA2_F32 = 0, /* fp32 inputs, outputs and conv state */
  MAMBA2_BF16 = 1 /* bf16 inputs, outputs and conv state */
} mamba2_dtype;

/* Problem sizes.  The SSM state is always fp32; `io_dtype` is the type of
 * xBC, z, dt_raw, y and the conv state. */
typedef struct {
  int64_t batch;            /* b >= 0 */
  int64_t seqlen;           /* L >= 0 (prefill); ignored by mamba2_ssd_step */
  int32_t nheads;           /* H >= 1, multiple of ngroups */
  int32_t headdim;          /* P: 16, 32 or 64 */
  int32_t dstate;           /* N: 16, 32, 64 or 128 */
  int32_t ngroups;          /* G >= 1: B/C groups, and the number of norm groups */
  int32_t d_conv;           /* conv width; must be 4 */
  int32_t chunk_size;       /* Q: 64, 128 or 256 (prefill only) */
  int32_t io_dtype;         /* mamba2_dtype */
  int32_t norm_before_gate; /* 0: rmsnorm(y * silu(z)) * w;  1: rmsnorm(y) * w * silu(z) */
  float norm_eps;           /* > 0, e.g. 1e-5 */
} mamba2_dims;

/* fp32 parameters (device arrays, read only). */
typedef struct {
  const float *conv_w;  /* [conv_dim, d_conv], 16-byte aligned: tap k multiplies the input
                          d_conv-1-k steps back */
  const float *conv_b;  /* [conv_dim] */
  const float *dt_bias; /* [nheads] */
  const float *A;       /* [nheads], A_h < 0 (callers holding A_log pass -exp(A_log)) */
  const float *D;       /* [nheads] */
  const float *norm_w;  /* [d_inner] */
} mamba2_params;

/* Human-readable name of a status code (static string). */
MAMBA2_API const char *mamba2_status_string(int status);

/* Library version as major * 10000 + minor * 100 + patch. */
MAMBA2_API int mamba2_version(void);

/* Bytes of device workspace that mamba2_conv_ssd_prefill needs for `dims`
 * (0 if dims are invalid).  The caller allocates it (256-byte aligned) and
 * may reuse it across calls that do not overlap on the GPU. */
MAMBA2_API size_t mamba2_prefill_workspace_size(const mamba2_dims *dims);

/* Prefill: run the whole mixer core over `seqlen` new tokens of each of the
 * `batch` sequences (qwbw.cn section 三 steps 2-4, chunked scan of step 3).
 *
 *  xBC     [b, L, conv_dim] io_dtype; token t of row bi starts at
 *          xBC + (bi * L + t) * xBC_row_stride elements, so it may point into
 *          a packed in_proj output.  Row stride >= conv_dim, multiple of 8;
 *          pointer 16-byte aligned.
 *  z       [b, L, d_inner] io_dtype, row stride >= d_inner, multiple of 8;
 *          16-byte aligned.  The gate.
 *  dt_raw  [b, L, nheads] io_dtype, row stride >= nheads (any alignment of
 *          the element type).
 *  y       [b, L, d_inner] io_dtype, contiguous, 16-byte aligned.  Output.
 *  conv_state  [b, conv_dim, d_conv] io_dtype, contiguous, or NULL.  When
 *          states_in != 0 it holds the d_conv raw xBC inputs before the first
 *          new token (oldest first) and supplies the conv's left context;
 *          otherwise that context is zero.  On return (if not NULL) it holds
 *          the last d_conv raw inputs of [old state | new tokens].
 *  ssm_state   [b, nheads, headdim, dstate] fp32, contiguous, or NULL.  When
 *          states_in != 0 it is the state h entering the first new token,
 *          otherwise the scan starts from zero.  On return (if not NULL) it
 *          holds the state after the last new token.
 *  states_in   0 or 1, as above.  States must be non-NULL when it is 1.
 *  workspace   device scratch of at least mamba2_prefill_workspace_size(dims)
 *          bytes, 256-byte aligned; contents on entry are ignored.
 *  stream  cudaStream_t as void*.
 * seqlen need not be a multiple of chunk_size.  seqlen == 0 copies or zeroes
 * the states and writes nothing else.
 * Range: bf16 I/O with headdim 64 and d_state 64 runs on the tensor cores with
 * fp16 operands, so the post-conv activations x, B, C and the products
 * x * dt * decay must stay below 2^15 in magnitude (larger values saturate);
 * inputs of normal magnitude (|xBC| up to about 1e4) are far inside that.
 * The carried SSM state has no such limit (its fp16 operand copy is scaled by
 * a power of two per chunk and head; the returned state is fp32). */
MAMBA2_API int mamba2_conv_ssd_prefill(const mamba2_dims *dims, const mamba2_params *params,
                                       const void *xBC, int64_t xBC_row_stride, const void *z,
                                       int64_t z_row_stride, const void *dt_raw,
                                       int64_t dt_row_stride, void *y, void *conv_state,
                                       float *ssm_state, int32_t states_in, void *workspace,
                                       size_t workspace_bytes, void *stream);

/* Bytes of DEVICE workspace that mamba2_conv_ssd_prefill_host needs for `dims`
 * (0 if dims are invalid): two staged input pieces, two output pieces, the
 * carried states and one piece's prefill workspace (about a quarter of the
 * whole-sequence input and output, for long sequences). */
MAMBA2_API size_t mamba2_prefill_host_workspace_size(const mamba2_dims *dims);

/* Prefill with every input and output in HOST memory: the same computation as
 * mamba2_conv_ssd_prefill (qwbw.cn section 三 steps 2-4) on host buffers, with
 * the copies overlapped with the work.  The sequence is cut into pieces of
 * whole chunks (a multiple of 256 tokens, about an eighth of L); piece i + 1 is
 * copied in and piece i - 1's y copied out while piece i runs, each piece
 * continuing from the states the previous one left (the chunked prefill of
 * section 三 step 3), so the result equals the one-call prefill up to rounding.
 *
 *  xBC, z, dt_raw  HOST, layout and row strides as for mamba2_conv_ssd_prefill
 *          (strides in elements, >= the widths; no alignment needed).
 *  y       HOST [b, L, d_inner] io_dtype, contiguous.  Output.
 *  conv_state, ssm_state  HOST or NULL, layouts as for mamba2_conv_ssd_prefill;
 *          read when states_in = 1, overwritten with the final states.
 *  workspace  DEVICE, >= mamba2_prefill_host_workspace_size(dims) bytes,
 *          256-byte aligned; contents on entry are ignored.
 *  stream  the caller's cudaStream_t (as void*): the call begins after the
 *          work already enqueued on it, and work enqueued on it afterwards
 *          begins after the call's last copy.  The call returns once its work
 *          is enqueued: synchronise the stream before reading y or the states.
 * Host buffers should be page-locked (cudaHostAlloc / cudaHostRegister): the
 * copies of pageable memory are correct but neither asynchronous nor
 * overlapped.  The call uses two streams and eight events of its own, made on
 * a host thread's first call on a device and kept for the thread's lifetime
 * (so it cannot be captured into a CUDA graph; calls from one thread are
 * ordered by the caller's stream as usual).  Stage events
 * (mamba2_record_stage_events) are not recorded.
 * Returns MAMBA2_OK, MAMBA2_ERR_INVALID_ARG (null pointer, stride below a
 * width, states_in without states), MAMBA2_ERR_UNSUPPORTED (as for
 * mamba2_conv_ssd_prefill), MAMBA2_ERR_WORKSPACE or MAMBA2_ERR_CUDA. */
MAMBA2_API int mamba2_conv_ssd_prefill_host(const mamba2_dims *dims,
                                            const mamba2_params *params, const void *xBC,
                                            int64_t xBC_row_stride, const void *z,
                                            int64_t z_row_stride, const void *dt_raw,
                                            int64_t dt_row_stride, void *y, void *conv_state,
                                            float *ssm_state, int32_t states_in,
                                            void *workspace, size_t workspace_bytes,
                                            void *stream);

/* Workspace bytes mamba2_conv_ssd_prefill_varlen needs for `dims` (batch =
 * number of sequences, seqlen = total tokens); 0 if the dims are invalid or
 * the call is not supported for them (see below). */
MAMBA2_API size_t mamba2_prefill_varlen_workspace_size(const mamba2_dims *dims);

/* Prefill of `batch` sequences of different lengths packed along the token
 * axis, in one call (the chunked prefill of "Zamba2 hybrid architecture in
 * Transformers", qwbw.cn, section 三 step 3, with a cache per sequence, for
 * requests of different lengths served together as in the time-to-first-token
 * scenario of the Zamba2-VL announcement, k7ail.com).  As
 * mamba2_conv_ssd_prefill, except:
 *  dims    batch = number of sequences, seqlen = L, the total token count.
 *  xBC, z, dt_raw, y  as above for one row of L tokens: sequence s owns tokens
 *          cu_seqlens[s] .. cu_seqlens[s + 1] - 1.  No chunk of the scan
 *          spans two sequences, and no conv reaches across them.
 *  cu_seqlens  device int32 [batch + 1], 4-byte aligned: 0, then the running
 *          token counts, last = seqlen (empty sequences allowed).  Offsets
 *          that break this are found on the device: the call then writes
 *          nothing and mamba2_device_errors reports bit 2.
 *  conv_state, ssm_state  per sequence ([batch, ...]), in and out as above;
 *          a sequence of fewer than d_conv tokens shifts its conv state.
 *  workspace   at least mamba2_prefill_varlen_workspace_size(dims) bytes.
 * Supported on the tensor-core path only: bf16 I/O, headdim 64, d_state 64,
 * at most 80 heads per group (MAMBA2_ERR_UNSUPPORTED otherwise).  The
 * sequences' chunks are laid out on the device (one small kernel), so the
 * host needs no copy of cu_seqlens. */
MAMBA2_API int mamba2_conv_ssd_prefill_varlen(
    const mamba2_dims *dims, const mamba2_params *params, const void *xBC,
    int64_t xBC_row_stride, const void *z, int64_t z_row_stride, const void *dt_raw,
    int64_t dt_row_stride, const int32_t *cu_seqlens, void *y, void *conv_state,
    float *ssm_state, int32_t states_in, void *workspace, size_t workspace_bytes, void *stream);

/* Decode: advance every sequence by one token (qwbw.cn section 三 step 3,
 * the single-token recurrent update used when the cache holds the states and
 * the new sequence length is 1).  The conv state is shifted left by one and
 * the new xBC column appended; the conv output is its dot product with the
 * taps; the SSM state takes one recurrence step; then D-skip and the gated
 * norm as in prefill.  dims->seqlen and dims->chunk_size are ignored.
 *
 *  xBC     [b, conv_dim] io_dtype, row (batch) stride >= conv_dim, multiple
 *          of 8, 16-byte aligned.
 *  z       [b, d_inner] io_dtype, row stride >= d_inner, multiple of 8,
 *          16-byte aligned.
 *  dt_raw  [b, nheads] io_dtype, row stride >= nheads.
 *  y       [b, d_inner] io_dtype, contiguous, 16-byte aligned.  Output.
 *  conv_state  [b, conv_dim, d_conv] io_dtype, contiguous, 16-byte aligned,
 *          updated in place.
 *  ssm_state   [b, nheads, headdim, dstate] fp32, contiguous, 16-byte
 *          aligned, updated in place.
 * Uses no workspace. */
MAMBA2_API int mamba2_ssd_step(const mamba2_dims *dims, const mamba2_params *params,
                               const void *xBC, int64_t xBC_row_stride, const void *z,
                               int64_t z_row_stride, const void *dt_raw, int64_t dt_row_stride,
                               void *y, void *conv_state, float *ssm_state, void *stream);

/* Device-side error flags (no counterpart on the pages).  Kernels that wait
 * for asynchronous copies give every wait a time limit (2 s); when one runs
 * out the kernel stops using the data, lets its own copies in flight land,
 * sets a flag and returns, leaving the context usable and the outputs of that
 * call undefined.  This call synchronises the current device, stores the
 * flags raised since the previous call in *flags (0 = none; bit 0 = a wait
 * ran out; bit 1 = the bounds-checked build skipped an access; bit 2 = a
 * packed-sequence prefill got invalid cu_seqlens) and clears them.  Returns MAMBA2_OK, MAMBA2_ERR_INVALID_ARG (flags
 * NULL) or MAMBA2_ERR_CUDA. */
MAMBA2_API int mamba2_device_errors(unsigned int *flags);

/* Test aid (no counterpart on the pages): makes the time limit of a kernel's
 * wait run out on purpose, without a fault.  While enabled (1) on the current
 * device, every kernel that waits for asynchronous work starts with a wait on
 * a barrier that nothing completes, limited to 20 ms; when it runs out the
 * kernel raises the flag that mamba2_device_errors reports (bit 0) and
 * returns before it has issued any copy, so the call's outputs are left
 * unwritten and the context stays usable.  0 restores normal operation.
 * Synchronises the device.  Returns MAMBA2_OK, MAMBA2_ERR_INVALID_ARG or
 * MAMBA2_ERR_CUDA. */
MAMBA2_API int mamba2_debug_stall_waits(int enable);

/* Size of the fixed device scratch array used by
 * mamba2_conv_ssd_prefill_noalloc (64 MiB). */
#define MAMBA2_STATIC_SCRATCH_BYTES (64u * 1024u * 1024u)

/* Prefill without a workspace argument, for callers that may not allocate
 * device memory (for example a plugin inside a runtime whose memory pool owns
 * every device allocation, or a latency-critical path that cannot afford
 * cudaMalloc's implicit synchronisation).  The pages have no counterpart of
 * this entry point.
 *
 * Same arguments, meaning and results as mamba2_conv_ssd_prefill, minus the
 * workspace: the scratch comes from one array of MAMBA2_STATIC_SCRATCH_BYTES
 * that the library holds in every GPU it is loaded on until the process
 * exits.  The caller still allocates inputs, outputs and states.
 *  - Problems whose mamba2_prefill_workspace_size exceeds
 *    MAMBA2_STATIC_SCRATCH_BYTES are rejected with MAMBA2_ERR_WORKSPACE and
 *    nothing is enqueued.
 *  - The first call in a device's context looks up the array's device
 *    address (with that device current), and so does the first call after
 *    that context was destroyed and re-created (cudaDeviceReset); make such a
 *    call before any stream capture.
 *  - Invalid dims return MAMBA2_ERR_INVALID_ARG / MAMBA2_ERR_UNSUPPORTED as
 *    for mamba2_conv_ssd_prefill, before the size check.
 *  - All calls share the one array: calls that may overlap on the GPU (other
 *    streams, other host threads using the same device) race on it and must
 *    be serialised by the caller.  No part of the array needs to start at
 *    zero, so leftover contents from an earlier call are harmless.
 *  - Allocates nothing: no cudaMalloc/cudaFree, no allocating library call. */
MAMBA2_API int mamba2_conv_ssd_prefill_noalloc(const mamba2_dims *dims,
                                               const mamba2_params *params, const void *xBC,
                                               int64_t xBC_row_stride, const void *z,
                                               int64_t z_row_stride, const void *dt_raw,
                                               int64_t dt_row_stride, void *y, void *conv_state,
                                               float *ssm_state, int32_t states_in,
                                               void *stream);

/* Workspace bytes mamba2_conv_ssd_prefill_backward needs for `dims` (0 if
 * the dims are invalid).  It holds the SSM state after every token:
 * batch * nheads * seqlen * headdim * dstate * 4 bytes of it (5.4 GB for one
 * 4096-token sequence of 80 heads of 64 x 64), plus O(batch * seqlen *
 * (conv_dim + nheads * dstate * 16)) bytes more. */
MAMBA2_API size_t mamba2_prefill_backward_workspace_size(const mamba2_dims *dims);

/* Backward pass of mamba2_conv_ssd_prefill, for training.  The pages give the
 * Zamba2 layers gradient checkpointing ("Zamba2 hybrid architecture in
 * Transformers", qwbw.cn, section 三): the forward is recomputed from the
 * layer's inputs inside this call (nothing of a forward call is needed) and
 * differentiated.  The gradients are those of
 *     sum(y * dy) + sum(h_L * d_ssm_state_out)
 * with respect to every input, parameter and initial state, y being the
 * prefill's output and h_L its final SSM state.
 *
 *  dims, params, xBC, z, dt_raw and their row strides: as for the prefill
 *          (the same validation; fixed-length rows, states_in given by the
 *          state pointers below).
 *  conv_state_in  [b, conv_dim, d_conv] io_dtype, contiguous, or NULL: the
 *          carried conv state the prefill started from (NULL: zero context).
 *  ssm_state_in   [b, nheads, headdim, dstate] fp32, contiguous, or NULL: the
 *          initial SSM state (NULL: zero).
 *  dy      [b, L, d_inner] io_dtype, contiguous: gradient of y.
 *  d_ssm_state_out [b, nheads, headdim, dstate] fp32 or NULL (zero): gradient
 *          of the returned final state.  (The final conv state's gradient is
 *          taken as zero.)
 * Outputs, overwritten (not accumulated):
 *  d_xBC   [b, L, conv_dim] io_dtype, contiguous.
 *  d_z     [b, L, d_inner] io_dtype, contiguous.
 *  d_dt_raw [b, L, nheads] io_dtype, contiguous.
 *  d_conv_w [conv_dim, d_conv], d_conv_b [conv_dim], d_dt_bias [nheads],
 *          d_A [nheads], d_D [nheads], d_norm_w [d_inner]: fp32.
 *  d_conv_state_in [b, conv_dim, d_conv] io_dtype or NULL (column 0, the
 *          oldest input, never reaches y: its gradient is zero).
 *  d_ssm_state_in  [b, nheads, headdim, dstate] fp32 or NULL.
 *  workspace  >= mamba2_prefill_backward_workspace_size(dims) bytes, 256-byte
 *          aligned.  stream: cudaStream_t as void*.
 * Runs in fp32 on the CUDA cores for every supported shape.  The parameter
 * gradients (sums over tokens) and the per-token sums over a head's state
 * rows behind d_xBC's B and C channels and d_dt_raw use atomic additions, so
 * those may differ in the last bits between runs.
 * Returns MAMBA2_OK, MAMBA2_ERR_INVALID_ARG (null or misaligned pointer, bad
 * stride), MAMBA2_ERR_UNSUPPORTED, MAMBA2_ERR_WORKSPACE or MAMBA2_ERR_CUDA. */
MAMBA2_API int mamba2_conv_ssd_prefill_backward(
    const mamba2_dims *dims, const mamba2_params *params, const void *xBC,
    int64_t xBC_row_stride, const void *z, int64_t z_row_stride, const void *dt_raw,
    int64_t dt_row_stride, const void *conv_state_in, const float *ssm_state_in, const void *dy,
    const float *d_ssm_state_out, void *d_xBC, void *d_z, void *d_dt_raw, float *d_conv_w,
    float *d_conv_b, float *d_dt_bias, float *d_A, float *d_D, float *d_norm_w,
    void *d_conv_state_in, float *d_ssm_state_in, void *workspace, size_t workspace_bytes,
    void *stream);

/* Profiling aid (no counterpart on the pages).  Arms the calling host thread
 * so that its NEXT call of mamba2_conv_ssd_prefill,
 * mamba2_conv_ssd_prefill_noalloc, mamba2_ssd_step or
 * mamba2_conv_ssd_prefill_backward records events[i]
 * (cudaEvent_t passed as void*, created by the caller) on the call's stream
 * just before the call's kernel stage i, and events[S] after
 * its last stage, S being the stage count that mamba2_stage_names reports.
 * Entries beyond n_events, and NULL entries, are not recorded, so a caller
 * can bracket a single stage.  The call disarms the thread when it returns,
 * whatever its status.  0 <= n_events <= 16.  Returns MAMBA2_OK or
 * MAMBA2_ERR_INVALID_ARG (bad count, or events NULL with n_events > 0). */
MAMBA2_API int mamba2_record_stage_events(void *const *events, int n_events);

/* Number of kernel stages a call of `kind` (0 = prefill, 1 = decode step,
 * 2 = prefill backward)
 * enqueues for `dims`, or MAMBA2_ERR_INVALID_ARG; writes up to max_names
 * static stage names to `names` (may be NULL).  A stage is one kernel launch
 * (a stage whose work is absent for a call, e.g. the conv-state write without
 * a conv state buffer, launches nothing but keeps its place). */
MAMBA2_API int mamba2_stage_names(int kind, const mamba2_dims *dims, const char **names,
                                  int max_names);

#ifdef __cplusplus
}
#endif

#endif /* MAMBA2SSD_H */
