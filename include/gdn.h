/*
 * gdn.h -- C ABI of the B200 (sm_100a) Gated DeltaNet token mixer.
 *
 * The mixer is the linear-attention layer that fills three of every four
 * layers of the Qwen3.5 / Qwen3-Next hybrid stack ("Qwen3.5", HF transformers
 * model doc, Usage tips: layer_types alternate three Gated DeltaNet layers
 * with one full-attention layer).  For each token it computes
 *
 *   1. y = causal depthwise conv1d (kernel 4, no bias) of the mixed q|k|v
 *      projection, then SiLU                 ("Qwen3.5 (Qwen3-Next)", API
 *      table: linear_conv_kernel_dim 4; "Qwen/Qwen3.5-9B", module tree:
 *      conv1d 8192x1x4, 32.8K parameters);
 *   2. q, k = per-head L2-normalised slices of y (q also times `scale`),
 *      v = the value slice;
 *   3. per value head: g = -exp(A_log) * softplus(a + dt_bias),
 *      alpha = exp(g), beta = sigmoid(b)     ("Qwen/Qwen3.5-9B", module tree:
 *      in_proj_a / in_proj_b 4096->32 and the direct parameters "32, 32");
 *   4. the gated delta rule, value head h reading key head h / (Hv/Hk):
 *         S_t = alpha_t S_{t-1} (I - beta_t k_t k_t^T) + beta_t v_t k_t^T,
 *         o_t = S_t q_t,     S in R^{dv x dk}
 *      ("Qwen (text & vision-language)", Architecture notes and Generation:
 *      conv1d + delta rule, with a conv state and a recurrent state carried
 *      per layer);
 *   5. out = o / sqrt(mean(o^2) + eps_norm) * norm_w * silu(z), one dv-wide
 *      norm_w shared by all heads    ("Qwen/Qwen3.5-9B", module tree: norm
 *      Qwen3_5RMSNormGated with 128 parameters).
 *
 * gdn_prefill runs steps 1-5 over variable-length packed sequences with the
 * chunked (WY / UT transform) form of step 4, which is algebraically equal to
 * the recurrence ("Qwen (text & vision-language)", Verified parity).
 * gdn_decode runs one token per sequence with the recurrent form on an fp32
 * state held in HBM and updated in place ("Qwen3.5", HF model doc, Usage
 * tips: the single-token recurrence is memory-bandwidth-bound).
 *
 * Conventions shared by every entry point
 *   - Pointers named "device" must point to device memory of the current
 *     CUDA device; the caller owns all memory.  The library allocates nothing
 *     and keeps no state between calls; calls on different streams are
 *     independent.
 *   - All work is enqueued asynchronously on `stream` (a cudaStream_t; NULL =
 *     the legacy default stream).  A call returns after launching.
 *   - Arguments are validated on the host before anything is launched; a
 *     failed check returns a negative gdn_status and launches nothing.
 *     Contents of device arrays (e.g. cu_seqlens) cannot be checked on the
 *     host; out-of-range offsets are clamped by the kernels so that no access
 *     leaves the buffers, but the results are then unspecified.
 *   - Layouts are row-major (C order).  "dtype" below is gdn_dtype `dtype`
 *     of the call: bf16 (GDN_BF16) or fp32 (GDN_F32).  States are always fp32.
 *   - Every device pointer must be 16-byte aligned.
 *   - Channel order of the mixed projection: [q heads | k heads | v heads],
 *     head-major within each block (q head i occupies channels i*dk ..
 *     i*dk+dk-1).  Value head h reads key head h / (Hv/Hk).
 *   - Conv taps: conv_w[c][3] multiplies the current token, conv_w[c][0] the
 *     token three steps back.  A conv history [.., Cc, 3] holds the last
 *     three raw (pre-conv) inputs per channel, oldest first.
 */
#ifndef GDN_B200_H
#define GDN_B200_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  GDN_OK = 0,
  GDN_ERR_NULL = -1,        /* a required pointer is NULL                       */
  GDN_ERR_DIMS = -2,        /* inconsistent or out-of-range sizes               */
  GDN_ERR_ALIGN = -3,       /* a pointer is not 16-byte aligned                 */
  GDN_ERR_UNSUPPORTED = -4, /* valid, but not a shape the library supports     */
  GDN_ERR_CUDA = -5,        /* a CUDA runtime/driver call failed (launch, ...)  */
  GDN_ERR_WORKSPACE = -6,   /* workspace missing or smaller than required       */
  GDN_ERR_ALIAS = -7,       /* buffers that must not overlap do overlap         */
  GDN_ERR_TIMEOUT = -8      /* a bounded wait inside a kernel gave up; reported
                               after the fact by gdn_device_error, since kernels
                               run asynchronously to the call that launched them */
} gdn_status;

/* Element types.  gdn_prefill / gdn_decode take GDN_F32 or GDN_BF16 inputs;
 * GDN_F16 is accepted only for the q, k, v of gdn_chunk_core (it is the type
 * gdn_prefill itself uses between its kernels for bf16 inputs). */
typedef enum { GDN_F32 = 0, GDN_BF16 = 1, GDN_F16 = 2 } gdn_dtype;

/* Implementation selector for the chunked core of gdn_prefill. */
typedef enum {
  GDN_IMPL_AUTO = 0,   /* tensor cores when supported (GDN_IMPL_TC_SPLIT when the
                          workspace holds its records, else GDN_IMPL_TC_FUSED;
                          for gdn_chunk_core GDN_IMPL_TC_FUSED only when given
                          its workspace, else GDN_IMPL_TC), CUDA cores
                          otherwise                                          */
  GDN_IMPL_SIMT = 1,   /* fp32 CUDA-core chunked kernel                       */
  GDN_IMPL_TC = 2,     /* tcgen05 tensor-core chunked core, one kernel per call
                          (bf16 inputs, fp16 operands, d = 128, chunk 64);
                          GDN_ERR_UNSUPPORTED otherwise                       */
  GDN_IMPL_TC_SPLIT = 3, /* the same tensor-core core as two kernels: the
                          state-independent key-side work of every (chunk,
                          head) first, over all SMs, then the per-head state
                          chain.  Needs gdn_prefill_workspace_size_n bytes
                          of workspace (GDN_ERR_WORKSPACE otherwise).         */
  GDN_IMPL_TC_FUSED = 4 /* the same tensor-core core as one persistent kernel
                          per SM: warps that do the key-side work of the next
                          chunk run beside the warps that carry the state, so
                          nothing passes through HBM between them; (sequence,
                          value head) chains are taken longest first.  Needs
                          only gdn_prefill_workspace_size bytes.            */
} gdn_impl;

/* Layer shape.  Supported: dk == dv in {32, 64, 128}; Hv % Hk == 0;
 * conv_k == 4.  scale multiplies q after its L2 norm (dk^-1/2 is usual);
 * eps_l2 is added to sum(x^2) inside the q/k L2 norm; eps_norm to mean(o^2)
 * inside the gated RMSNorm (1e-6 for the Qwen3.5 family). */
typedef struct {
  int Hk, Hv, dk, dv;
  int conv_k;
  float scale;
  float eps_l2;
  float eps_norm;
} gdn_dims;

/* ------------------------------------------------------------------ prefill
 * Packed varlen prefill: N sequences, sequence n occupying tokens
 * cu_seqlens[n] .. cu_seqlens[n+1]-1 of the packed token axis (T_tot tokens).
 * Cc = 2*Hk*dk + Hv*dv.
 */
typedef struct {
  const void* mixed_qkv;       /* device [T_tot, Cc]      dtype                     */
  const void* conv_w;          /* device [Cc, 4]          dtype                     */
  const void* a;               /* device [T_tot, Hv]      dtype                     */
  const void* b;               /* device [T_tot, Hv]      dtype                     */
  const float* A_log;          /* device [Hv]             fp32                      */
  const float* dt_bias;        /* device [Hv]             fp32                      */
  const void* z;               /* device [T_tot, Hv*dv]   dtype                     */
  const void* norm_w;          /* device [dv]             dtype                     */
  const int32_t* cu_seqlens;   /* device [N+1] int32, cu[0]=0, non-decreasing,
                                  cu[N]=T_tot; empty sequences are allowed        */
  int N;                       /* number of sequences (>= 1)                      */
  int T_tot;                   /* packed tokens (>= 0)                            */
  int chunk;                   /* chunk length: 16, 32 or 64                      */
  gdn_dtype dtype;
  gdn_impl impl;
  const float* initial_state;  /* device [N, Hv, dv, dk] fp32, or NULL for zeros  */
  float* final_state;          /* device [N, Hv, dv, dk] fp32, or NULL; may be the
                                  same pointer as initial_state (updated in place) */
  const void* conv_state_in;   /* device [N, Cc, 3] dtype, or NULL for zeros      */
  void* conv_state_out;        /* device [N, Cc, 3] dtype, or NULL; must not
                                  overlap conv_state_in                           */
  void* out;                   /* device [T_tot, Hv, dv] dtype                    */
  void* workspace;             /* device scratch, >= gdn_prefill_workspace_size  */
  size_t workspace_bytes;
  void* core_event_begin;      /* optional cudaEvent_t recorded on `stream` just
                                  before / after the chunked-core kernel (timing
                                  of that kernel alone); NULL to skip           */
  void* core_event_end;
  int segments;                /* two-kernel tensor-core path only: the number of
                                  segments each sequence's state chain is cut
                                  into and run in parallel (0 = chosen from the
                                  sizes and the SM count, 1 = one serial chain,
                                  2..8 = that many).  Other values, or more than 1
                                  when N*Hv > 64, return GDN_ERR_UNSUPPORTED.
                                  Every choice computes the same result up to
                                  rounding.                                      */
  int reuse_workspace;         /* 1: the workspace already holds what this call
                                  would compute before its state chains -- left
                                  there by gdn_prefill_state_map on the same
                                  dims, dtype, inputs (mixed_qkv, conv_w, a, b,
                                  A_log, dt_bias, cu_seqlens, conv_state_in, and
                                  z and norm_w, which that call must then have
                                  been given), N, T_tot and chunk -- so the conv
                                  and the key-side kernel are skipped and
                                  conv_state_out is not written.  Two-kernel
                                  tensor-core path only (GDN_ERR_UNSUPPORTED
                                  otherwise).  0: compute everything.  A
                                  context-parallel rank maps its part, folds the
                                  gathered maps into its start state and then
                                  runs its part from there without repeating the
                                  key-side work.                                  */
} gdn_prefill_args;

/* Bytes of device workspace gdn_prefill needs for these sizes (0 when the
 * sizes are invalid).  The workspace holds the normalised q, k, the values v
 * (fp16 for bf16 inputs, fp32 for fp32 inputs) and the gates of every token
 * between the two kernels of the call. */
size_t gdn_prefill_workspace_size(const gdn_dims* dims, int T_tot, gdn_dtype dtype);

/* Bytes of workspace that also holds the per-(chunk, value head) operand
 * records of the two-kernel tensor-core path (GDN_IMPL_TC_SPLIT): about
 * 82 KB per 64 tokens and value head, for N sequences of T_tot tokens in
 * total, plus, when N*Hv <= 64, 1.4 MB per (sequence, value head) for the
 * segment maps and start states of a segmented state chain (see
 * gdn_prefill_args.segments).  With at least this much, GDN_IMPL_AUTO takes
 * the two-kernel path where the tensor cores apply; with only
 * gdn_prefill_workspace_size bytes it takes the fused one.  0 when
 * the sizes are invalid. */
size_t gdn_prefill_workspace_size_n(const gdn_dims* dims, int N, int T_tot, gdn_dtype dtype);

/* Steps 1-5 over packed sequences.  Writes out, and final_state /
 * conv_state_out when given.  The workspace is overwritten. */
gdn_status gdn_prefill(const gdn_dims* dims, const gdn_prefill_args* args, void* stream);

/* The implementation gdn_prefill runs for these sizes when called with
 * `impl` (GDN_IMPL_AUTO resolved to a concrete one) and a workspace of
 * workspace_bytes bytes on the current device; negative gdn_status when that
 * call would be rejected for its sizes or impl. */
int gdn_prefill_resolve_impl(const gdn_dims* dims, int N, int T_tot, int chunk, gdn_dtype dtype,
                             gdn_impl impl, size_t workspace_bytes);

/* Number of segments the two-kernel tensor-core path cuts each sequence's
 * state chain into when gdn_prefill_args.segments is 0, for N sequences of
 * T_tot tokens in total on the current device (1: one serial chain per
 * (sequence, value head)).  With more than one segment the path launches
 * two more kernels: the segments' affine maps and the scan of their start
 * states.  0 when the sizes are invalid. */
int gdn_prefill_auto_segments(const gdn_dims* dims, int N, int T_tot);

/* ------------------------------------------------ context-parallel prefill
 * One long sequence cut into consecutive parts, e.g. one part per GPU (the
 * family is built for long contexts: "Qwen/Qwen3.5-9B", config table:
 * max_position_embeddings 262144; "Qwen3.5-397B-A17B", specification table:
 * context length 256K tokens).  Step 4 is linear in the state, so over a
 * part of the sequence the state after it is an affine function of the state
 * before it:
 *     S_after = S_before M + R,
 *     M = prod over the part's tokens, in order, of alpha_t (I - beta_t k_t k_t^T)
 *         (dk x dk),
 *     R = the state after the part when it starts from zero (dv x dk).
 * The parts' (M, R) are independent of one another; the start state of part
 * j is the fold S_j = (...((S_0 M_0 + R_0) M_1 + R_1) ...) M_{j-1} + R_{j-1}.
 * A context-parallel prefill therefore computes every part's map at once,
 * gathers the maps (an exchange of 2 * Hv * d * d * 4 bytes per part and
 * sequence), folds them, and runs gdn_prefill on each part from its start
 * state, with the last three raw inputs before the part as conv_state_in.
 *
 * gdn_prefill_state_map: (M, R) of every sequence of the call.
 *   map   device [N, Hv, 2, dv, dk] fp32, written: map[n][h][0] = M (dk x dk,
 *         dv = dk), map[n][h][1] = R.  Must not overlap the workspace.
 *   args  as for gdn_prefill; mixed_qkv, conv_w, a, b, A_log, dt_bias,
 *         cu_seqlens and conv_state_in are read, conv_state_out is written
 *         when given; initial_state, final_state and out are not used.
 *         z and norm_w are optional (both or neither when T_tot > 0, else
 *         GDN_ERR_NULL): with them the workspace is left ready for
 *         gdn_prefill with reuse_workspace = 1 on the same inputs.
 *         segments: 0 = chosen from the sizes, 1 = one serial chain, 2..7 =
 *         that many segments per sequence, composed in fp32 (more than 1
 *         only when N*Hv <= 64).
 *   Supported: bf16, dk = dv = 128, chunk 64 (the tensor-core shapes), with
 *   gdn_prefill_workspace_size_n bytes of workspace; GDN_ERR_UNSUPPORTED /
 *   GDN_ERR_WORKSPACE otherwise.  An empty sequence gives M = I, R = 0.
 *
 * gdn_state_fold: S_out = the fold of `count` consecutive maps from S_first.
 *   maps    device [count, N, Hv, 2, dv, dk] fp32 (e.g. the maps of parts
 *           0 .. count-1 gathered from their ranks, in part order)
 *   S_first device [N, Hv, dv, dk] fp32, or NULL for zeros
 *   S_out   device [N, Hv, dv, dk] fp32; may be S_first (in place), must not
 *           overlap maps.  count = 0 copies S_first (or zeros).
 *   Supported: dk = dv = 128.
 */
gdn_status gdn_prefill_state_map(const gdn_dims* dims, const gdn_prefill_args* args, float* map,
                                 void* stream);
gdn_status gdn_state_fold(const gdn_dims* dims, int N, int count, const float* maps,
                          const float* S_first, float* S_out, void* stream);

/* ------------------------------------------------ prefill without workspace
 * No counterpart on the pages: this is an addition of this library for
 * callers that cannot hand gdn_prefill a workspace -- e.g. an operator plugin
 * that receives only its input and output tensors and has no allocator to
 * ask for temporary device memory, or a runtime that has carved up all device
 * memory up front and allows no cudaMalloc (nor its implicit device
 * synchronisation) while serving.
 *
 * gdn_prefill_noalloc runs gdn_prefill with its workspace taken from one
 * fixed scratch array inside the library (GDN_NOALLOC_SCRATCH_BYTES of device
 * memory, held on every device that uses it until the process exits).  It
 * allocates nothing.
 *   - args->workspace and args->workspace_bytes are ignored; every other
 *     argument means what it means for gdn_prefill, with the same checks,
 *     except reuse_workspace, which must be 0 (GDN_ERR_UNSUPPORTED).
 *   - Returns GDN_ERR_WORKSPACE, launching nothing, when the workspace these
 *     sizes need (gdn_prefill_workspace_size) exceeds
 *     GDN_NOALLOC_SCRATCH_BYTES -- about 3200 tokens at 16 key / 16 value
 *     heads of width 128, bf16.
 *   - With impl GDN_IMPL_AUTO the call takes the path gdn_prefill would take
 *     with a workspace of GDN_NOALLOC_SCRATCH_BYTES: a batch whose two-kernel
 *     records (gdn_prefill_workspace_size_n) do not fit in the scratch runs
 *     on a path that needs none.
 *   - Under CUDA's lazy module loading (the default) the scratch's device
 *     memory is committed on the first call on each device.  A runtime that
 *     divides up device memory in advance should make one call (any size,
 *     e.g. one sequence of one token) before it does so.
 *   - The first call on a device looks up the scratch's device address
 *     (cudaGetSymbolAddress) and caches it with the id of the current CUDA
 *     context; a call in a new context (after cudaDeviceReset) looks it up
 *     again.  Make the first call on a device, and the first after a reset,
 *     outside any CUDA stream capture.  GDN_ERR_CUDA if the lookup fails.
 *   - All calls share the one scratch array, which keeps the previous call's
 *     contents (nothing in it needs to start at zero).  Calls whose work may
 *     overlap on the GPU -- on different streams, or from host threads that
 *     do not order their streams -- race on it and corrupt each other's
 *     results: issue them on one stream, or order them.
 */
#define GDN_NOALLOC_SCRATCH_BYTES (64u << 20)

gdn_status gdn_prefill_noalloc(const gdn_dims* dims, const gdn_prefill_args* args, void* stream);

/* ------------------------------------------------------------------- decode
 * One token for each of B independent sequences.  state and conv_state are
 * read and overwritten in place with the values after this token.
 *
 * The recurrent state is fp32 by default.  With state_dtype = GDN_BF16 it is
 * held in bf16 ([B, Hv, dv, dk], 2 bytes per entry), which halves the HBM
 * bytes of this bandwidth-bound step ("Qwen3.5", HF model doc, Usage tips: the
 * single-token recurrence is memory-bandwidth-bound): the step reads the bf16
 * state, computes in fp32 and writes the new state rounded to the nearest
 * bf16; out is computed from the unrounded fp32 state.
 */
typedef struct {
  const void* mixed_qkv;       /* device [B, Cc]          dtype                     */
  const void* conv_w;          /* device [Cc, 4]          dtype                     */
  const void* a;               /* device [B, Hv]          dtype                     */
  const void* b;               /* device [B, Hv]          dtype                     */
  const float* A_log;          /* device [Hv]             fp32                      */
  const float* dt_bias;        /* device [Hv]             fp32                      */
  const void* z;               /* device [B, Hv*dv]       dtype                     */
  const void* norm_w;          /* device [dv]             dtype                     */
  void* state;                 /* device [B, Hv, dv, dk]  state_dtype, in place     */
  void* conv_state;            /* device [B, Cc, 3]       dtype, in place           */
  void* out;                   /* device [B, Hv, dv]      dtype                     */
  int B;                       /* batch (>= 0)                                      */
  gdn_dtype dtype;
  gdn_dtype state_dtype;       /* GDN_F32 (0, the default) or GDN_BF16             */
  int T;                       /* tokens per sequence in this step: 1..8 (0 = 1).
                                  With T > 1 the token inputs are [B, T, ...]
                                  (mixed_qkv [B, T, Cc], a, b [B, T, Hv], z
                                  [B, T, Hv*dv]) and out is [B, T, Hv, dv]; the
                                  step equals T one-token steps (short
                                  multi-token decode, e.g. verifying drafted
                                  tokens), with the state read and written once.
                                  T > 8 returns GDN_ERR_UNSUPPORTED.             */
} gdn_decode_args;

gdn_status gdn_decode(const gdn_dims* dims, const gdn_decode_args* args, void* stream);

/* ------------------------------------------------ projections and the layer
 * The dense projections around the mixer ("Qwen/Qwen3.5-9B", module tree of a
 * Gated DeltaNet block: in_proj_qkv 4096->8192, in_proj_z 4096->4096,
 * in_proj_b and in_proj_a 4096->32, out_proj 4096->4096), on the tcgen05
 * tensor cores in bf16 with fp32 accumulation.
 *
 * gdn_linear: Y = X W^T for X [M, K] and W [N, K] (the [out, in] layout of the
 * layer's weights), bf16 in and out.  The N columns of Y are cut into
 * n_outputs consecutive ranges; range i (out_cols[i] columns) is stored to
 * out[i] as an [M, out_cols[i]] array with row stride out_ld[i], so one call
 * over the stacked input-projection weights writes mixed_qkv, z, b and a
 * directly.
 *   Supported: K a positive multiple of 64; every out_cols[i] a positive
 *   multiple of 8 with the ranges summing to N; ldx, ldw >= K and out_ld[i] >=
 *   out_cols[i], all multiples of 8 elements; every pointer 16-byte aligned.
 *   GDN_ERR_UNSUPPORTED / GDN_ERR_DIMS / GDN_ERR_ALIGN / GDN_ERR_NULL otherwise,
 *   before anything is launched.  M = 0 does nothing.  The caller owns every
 *   buffer; the call is asynchronous on `stream` and allocates nothing; columns
 *   of an output row past its range are not written.  A bounded wait of the
 *   kernel that gives up is reported by gdn_device_error.
 */
typedef struct {
  const void* x;               /* device [M, K] bf16, rows ldx elements apart   */
  const void* w;               /* device [N, K] bf16, rows ldw elements apart   */
  int M, N, K;
  int ldx, ldw;
  int n_outputs;               /* 1 .. 4                                        */
  void* out[4];                /* device bf16 [M, out_cols[i]], rows out_ld[i]  */
  int out_cols[4];
  int out_ld[4];
} gdn_linear_args;

gdn_status gdn_linear(const gdn_linear_args* args, void* stream);

/* gdn_layer_prefill: the layer on packed sequences, y = out_proj(mixer(
 * in_proj(hidden))).  The input projection is one gdn_linear over w_in, the
 * rows of in_proj_qkv, in_proj_z, in_proj_b and in_proj_a stacked in that
 * order ([Cc + Hv*dv + 2*Hv, d_model]); its outputs and the mixer output are
 * bf16 arrays in the workspace; the mixer is gdn_prefill with `impl` on the
 * rest of the workspace (AUTO: the two-kernel path when that rest holds its
 * records).  bf16 only; d_model and Hv*dv multiples of 64.
 * gdn_layer_workspace_size gives the bytes for both (0 for invalid sizes);
 * with gdn_layer_activation_bytes + gdn_prefill_workspace_size bytes the
 * mixer runs without records.  The other arguments mean what they mean for
 * gdn_prefill.  Errors: GDN_ERR_UNSUPPORTED for d_model or Hv*dv not a
 * multiple of 64 (or Hv not a multiple of 8), GDN_ERR_WORKSPACE for a
 * workspace smaller than the activations, GDN_ERR_NULL / GDN_ERR_ALIGN for
 * missing or misaligned buffers -- these before any launch -- and what
 * gdn_prefill returns for the mixer's arguments, which it checks after
 * in_proj has been queued (out_proj is then not launched).  Everything runs
 * in order on `stream`: in_proj, the mixer, out_proj. */
typedef struct {
  const void* hidden;          /* device [T_tot, d_model] bf16                   */
  const void* w_in;            /* device [Cc + Hv*dv + 2*Hv, d_model] bf16       */
  const void* w_out;           /* device [d_model, Hv*dv] bf16                   */
  void* y;                     /* device [T_tot, d_model] bf16                   */
  int d_model;
  const void* conv_w;          /* device [Cc, 4] bf16                            */
  const float* A_log;          /* device [Hv]                                    */
  const float* dt_bias;        /* device [Hv]                                    */
  const void* norm_w;          /* device [dv] bf16                               */
  const int32_t* cu_seqlens;   /* device [N+1]                                   */
  int N, T_tot, chunk;
  gdn_impl impl;
  const float* initial_state;  /* as in gdn_prefill_args                         */
  float* final_state;
  const void* conv_state_in;
  void* conv_state_out;
  void* workspace;
  size_t workspace_bytes;
} gdn_layer_args;

size_t gdn_layer_activation_bytes(const gdn_dims* dims, int d_model, int T_tot);
size_t gdn_layer_workspace_size(const gdn_dims* dims, int d_model, int N, int T_tot);
gdn_status gdn_layer_prefill(const gdn_dims* dims, const gdn_layer_args* args, void* stream);

/* --------------------------------------------------------------- core only
 * Step 4 alone, chunked form, on given q, k (already normalised/scaled), v,
 * log-decay g and beta.  It exists so that the exact invariants of the delta
 * rule can be checked on the GPU without the conv, L2 norm and gated norm.
 *   q, k  device [T_tot, Hk, dk] dtype;  v device [T_tot, Hv, dv] dtype
 *         (dtype GDN_F32, GDN_BF16 or GDN_F16; the tensor-core kernel takes
 *         GDN_F16)
 *   g, beta device [Hv, T_tot] fp32 (head-major)
 *   o     device [T_tot, Hv, dv] fp32 (the core output before the gated norm)
 *   initial_state / final_state as in gdn_prefill_args.
 */
typedef struct {
  const void* q;
  const void* k;
  const void* v;
  const float* g;
  const float* beta;
  const int32_t* cu_seqlens;
  int N, T_tot, chunk;
  gdn_dtype dtype;
  gdn_impl impl;
  const float* initial_state;
  float* final_state;
  float* o;
  void* workspace;             /* device scratch: gdn_core_workspace_size bytes for
                                  GDN_IMPL_TC_FUSED, gdn_core_workspace_size_split
                                  bytes for GDN_IMPL_TC_SPLIT (its records); may be
                                  NULL otherwise */
  size_t workspace_bytes;
} gdn_core_args;

/* Bytes of workspace gdn_chunk_core needs for N sequences (the chain queue of
 * GDN_IMPL_TC_FUSED). */
size_t gdn_core_workspace_size(int N);
/* Bytes for GDN_IMPL_TC_SPLIT (the two-kernel path's per-(chunk, head) records,
 * and at least gdn_core_workspace_size, so one buffer serves every path); 0
 * for invalid sizes.  With less, GDN_IMPL_TC_SPLIT returns GDN_ERR_WORKSPACE. */
size_t gdn_core_workspace_size_split(const gdn_dims* dims, int N, int T_tot);

gdn_status gdn_chunk_core(const gdn_dims* dims, const gdn_core_args* args, void* stream);

/* Error word of the kernels.  Their internal waits (on TMA copies, on
 * tensor-core completion, on the other CTA of a cluster, between the roles of
 * a warp-specialised kernel) are bounded; one that gives up records it here,
 * lets the copies and tensor-core work it started land (bounded again), frees
 * its TMEM and returns instead of hanging.  This call synchronises the current
 * device, stores GDN_ERR_TIMEOUT in *code if any wait gave up since the word
 * was last cleared (0 otherwise), and clears the word when clear != 0. */
gdn_status gdn_device_error(int* code, int clear);

/* Test of that failure path, with no counterpart on the pages: launches on
 * `stream` one warp that waits, through the same bounded wait the kernels
 * use, on an mbarrier nothing ever arrives at, gives up after limit_us
 * microseconds (1 .. 1000000; GDN_ERR_DIMS otherwise) and records the
 * timeout in the error word.  Nothing else is in flight in that kernel. */
gdn_status gdn_selftest_bounded_wait(int limit_us, void* stream);

/* Human-readable name of a status code (static storage). */
const char* gdn_status_string(gdn_status status);

/* Library version string, e.g. "gdn-b200 0.1". */
const char* gdn_version(void);

#ifdef __cplusplus
}
#endif

#endif /* GDN_B200_H */
