// Internal launch interfaces between the C-ABI layer (gdn_api.cu) and the
// kernels.  Nothing here is exported from the shared library.
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "gdn.h"
#include "gdn_common.cuh"

namespace gdn {

// conv_prep.cu
struct ConvPrepParams {
  const void* x;              // [T, Cc]
  const void* conv_w;         // [Cc, 4]
  const void* a;              // [T, Hv]
  const void* b;              // [T, Hv]
  const float* A_log;         // [Hv]
  const float* dt_bias;       // [Hv]
  const int32_t* cu_seqlens;  // [N+1]
  const void* conv_state_in;  // [N, Cc, 3] or null
  void* conv_state_out;       // [N, Cc, 3] or null
  void* q;                    // [T, Hk, d]  fp16 (bf16 inputs) or fp32
  void* k;                    // [T, Hk, d]
  void* v;                    // [T, Hv, d]
  // fp16 intermediates only: the rounding residuals of q and k,
  // q_lo = fp16(q - fp16(q)), so that q + q_lo carries about 22 significand
  // bits into the K K^T and Q K^T products (null: not written)
  void* q_lo;                 // [T, Hk, d]
  void* k_lo;                 // [T, Hk, d]
  float* g;                   // [Hv, T]
  float* beta;                // [Hv, T]
  int T, N, Hk, Hv, Cc;
  float scale, eps_l2;
  int tok_blocks;             // set by the launcher
};
cudaError_t launch_conv_prep(const ConvPrepParams& p, int d, gdn_dtype dt, cudaStream_t st);
int conv_error_word(int clear);  // host: read (and clear) the conv kernel's device error word

// Parameters of the chunked core (both implementations).
struct ChunkParams {
  const void* q;              // [T, Hk, d]
  const void* k;              // [T, Hk, d]
  const void* v;              // [T, Hv, d]
  // residuals of fp16 q and k (see ConvPrepParams), or null: the tensor-core
  // kernels then form K K^T and Q K^T from the fp16 values alone
  const void* q_lo;           // [T, Hk, d]
  const void* k_lo;           // [T, Hk, d]
  const float* g;             // [Hv, T]
  const float* beta;          // [Hv, T]
  const int32_t* cu_seqlens;  // [N+1]
  const float* S0;            // [N, Hv, d, d] or null
  float* S_out;               // [N, Hv, d, d] or null
  // gated-norm epilogue (when out != null)
  const void* z;              // [T, Hv*d]
  const void* norm_w;         // [d]
  void* out;                  // [T, Hv, d]
  float* o_raw;               // [T, Hv, d] fp32 core output (when out == null)
  int T, N, Hk, Hv, chunk;
  float eps_norm;
  uint8_t* rec;               // split tensor-core path: per-(chunk, head) operand records
  // split tensor-core path, segmented state chain (nseg > 1): each sequence's
  // chunks are cut into nseg segments; seg_mr holds the affine map (M, R) of
  // every segment but the last, [N][nseg-1][Hv][2][d][d], seg_start the state
  // at the start of every segment, [N][nseg][Hv][d][d] (both fp32)
  int nseg;
  float* seg_mr;
  float* seg_start;
  // state-map mode (map_out != null): no outputs; every one of the nseg
  // segments gets its map, in seg_mr as [N][nseg][Hv][2][d][d] (role 1 from a
  // zero state), and the maps of each (sequence, head), composed in segment
  // order, go to map_out [N][Hv][2][d][d].  With nseg == 1, seg_mr == map_out.
  float* map_out;
  // the workspace already holds q, k, v, the gates and the records (of a
  // state-map call on the same inputs): the key-side kernel is not launched
  int reuse_records;
};

// chunk_simt.cu: fp32 CUDA-core chunked core.  Supported (d, chunk) pairs:
// d in {32, 64} with chunk in {16, 32, 64}; d = 128 with chunk in {16, 32}.
bool chunk_simt_supported(int d, int chunk);
// dt_out: dtype of z / norm_w / out; dt_mid: dtype of q, k, v.
cudaError_t launch_chunk_simt(const ChunkParams& p, int d, gdn_dtype dt_out, gdn_dtype dt_mid,
                              cudaStream_t st);

// chunk_tc.cu: tcgen05 chunked core, fp16 operands (q, k, v of dtype
// dt_mid = GDN_F16), d = 128, chunk = 64.
bool chunk_tc_supported(int d, int chunk, gdn_dtype dt_mid);
cudaError_t launch_chunk_tc(const ChunkParams& p, cudaStream_t st);

// chunk_tc_split.cu: the same core as two kernels -- a key-side kernel over
// every (chunk, value head) writing operand records, then a per-head chain
// kernel.  Needs chunk_tc_split_record_bytes(...) of extra workspace.
size_t chunk_tc_split_record_bytes(int N, int T, int Hv);
// Segmented state chains: at most this many segments per sequence, and only
// while N * Hv <= kSegMaxChains; chunk_tc_split_seg_bytes is the workspace
// they take (0 beyond that bound).
constexpr int kSegMax = 8;
constexpr int kSegMaxChains = 64;
size_t chunk_tc_split_seg_bytes(int N, int Hv);
// Segments chosen for these sizes when the caller asks for none in particular.
int chunk_tc_split_auto_segments(int N, int T, int Hv);
cudaError_t launch_chunk_tc_split(const ChunkParams& p, cudaStream_t st);
int split_error_word(int clear);  // host: read (and clear) that path's device error word
// Segments of the state-map mode for N sequences of Hv heads (1 when the
// segment buffers do not exist for these sizes).
int chunk_tc_split_map_segments(int N, int Hv);

// chunk_fused.cu: the same core as one persistent warp-specialised kernel.
// `sched` is kFusedSchedBytes of workspace: the chain counter and the queue
// order of up to kFusedSortMax sequences, written by
// launch_chunk_fused_order, which must run first on the stream (it reads
// only cu_seqlens).
constexpr int kFusedSortMax = 1024;
constexpr size_t kFusedSchedBytes = (1 + kFusedSortMax) * sizeof(int);
cudaError_t launch_chunk_fused_order(const ChunkParams& p, int* sched, cudaStream_t st);
cudaError_t launch_chunk_fused(const ChunkParams& p, int* sched, cudaStream_t st);
int fused_error_word(int clear);  // host: read (and clear) that kernel's device error word

// Affine fold, d = 128: for every (sequence n, head h), the rows X (rows x d,
// fp32) start from x0 (zeros when null) and go through the maps s = 0 ..
// nmaps-1 in order, X <- X M_s, and rows r >= r_add also take row r - r_add
// of R_s.  With rows = d and r_add = 0, X is a state and the fold is the
// state after consecutive parts; with rows = 2d and r_add = d, X is a stacked
// map [M; R] and the fold composes maps.  out may be x0 (each row is read
// before it is written, by the same CTA).
struct FoldParams {
  const float* x0;        // rows of (n, h) at x0 + n * x0_n + h * x0_h, or null
  size_t x0_n, x0_h;
  const float* maps;      // map s of (n, h) at maps + s * map_s + n * map_n + h * 2 d d: M then R
  size_t map_s, map_n;
  int nmaps;
  int rows;               // d or 2 d
  int r_add;              // 0 or d
  float* out;             // [N][Hv][rows][d]
  int N, Hv;
};
cudaError_t launch_state_fold(const FoldParams& p, cudaStream_t st);

// linear_tc.cu: Y = X W^T in bf16 on the tensor cores (X [M, K], W [N, K],
// K a multiple of 64), the N columns of Y split into n_out consecutive ranges,
// range i stored to out[i] ([M, out_cols[i]], row stride out_ld[i]).
struct LinearParams {
  int M, N, K;
  int n_out;
  void* out[4];
  int out_cols[4];
  int out_ld[4];
  int tiles_m, tiles_n;  // set by the launcher
};
cudaError_t launch_linear_tc(const LinearParams& p, const void* x, int ldx, const void* w, int ldw,
                             cudaStream_t st);
int linear_error_word(int clear);

// decode.cu
struct DecodeParams {
  const void* x;              // [B, Cc]
  const void* conv_w;         // [Cc, 4]
  const void* a;              // [B, Hv]
  const void* b;              // [B, Hv]
  const float* A_log;
  const float* dt_bias;
  const void* z;              // [B, Hv*d]
  const void* norm_w;         // [d]
  void* state;                // [B, Hv, d, d] fp32 or bf16 (state_bf16)
  void* conv_state;           // [B, Cc, 3]
  void* out;                  // [B, Hv, d]
  int B, Hk, Hv, Cc;
  int T;                      // tokens per sequence in this step (1..8)
  float scale, eps_l2, eps_norm;
  bool state_bf16;
};
cudaError_t launch_decode(const DecodeParams& p, int d, gdn_dtype dt, cudaStream_t st);

}  // namespace gdn
