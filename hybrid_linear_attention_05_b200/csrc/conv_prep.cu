// Conv1d + SiLU + q/k L2 norm + gate preparation for gdn_prefill.
//
// The normalised q, k and the values are written as fp16 for bf16 inputs
// (fp32 for fp32 inputs): they are the tensor-core operands of the chunked
// core, and fp16 keeps three more significand bits than bf16 at the same size
// and MMA rate (all of them are bounded: |q|, |k| <= 1 after the norm).
//
// One thread handles 8 consecutive channels of one token: it reads the four
// conv inputs of those channels (the token and the three before it, or the
// sequence's conv history before its first token), applies the depthwise
// 4-tap conv and SiLU, and for q / k heads joins the other threads of its
// head in a shuffle reduction for the L2 norm.  The first thread of every
// value head also computes that head's gates g = -exp(A_log) softplus(a +
// dt_bias) and beta = sigmoid(b).  A second group of threads writes the conv
// tail (the last three raw inputs of every sequence).
//
// HBM traffic per token: the Cc-wide input row once (the three earlier rows
// it also reads are the previous tokens' rows, served from L1/L2), the
// Cc-wide normalised row once, and the gates.
#include "gdn_internal.h"

namespace gdn {

template <typename T, typename TM, int D>
__global__ void __launch_bounds__(256) conv_prep_kernel(ConvPrepParams p) {
  constexpr int TPS = D / 8;  // threads per head segment
  const int Cc = p.Cc;
  const int groups = Cc / 8;  // threads per token row
  const size_t gid = (size_t)blockIdx.x * blockDim.x + threadIdx.x;
  const size_t n_tok = (size_t)p.T * groups;
  const T* __restrict__ x = static_cast<const T*>(p.x);
  const T* __restrict__ hist_all = static_cast<const T*>(p.conv_state_in);
  const int lane = threadIdx.x & 31;
  const unsigned seg_mask = ((TPS == 32) ? 0xffffffffu : ((1u << TPS) - 1u)) << (lane & ~(TPS - 1));

  if (blockIdx.x < p.tok_blocks) {
    // ------------------------------------------------------ token threads
    const bool valid = gid < n_tok;
    const int t = valid ? (int)(gid / groups) : 0;
    const int cg = valid ? (int)(gid % groups) : 0;
    const int c0 = cg * 8;
    const int seg = c0 / D;
    const int n = seq_of_token(p.cu_seqlens, p.N, t);
    const int bos = clampi(__ldg(p.cu_seqlens + n), 0, p.T);
    const T* hist = hist_all ? hist_all + (size_t)n * Cc * 3 : nullptr;

    float w[8][4];
    {
      const T* wp = static_cast<const T*>(p.conv_w) + (size_t)c0 * 4;
      float tmp[8];
#pragma unroll
      for (int r = 0; r < 4; ++r) {
        load8(wp + r * 8, tmp);
#pragma unroll
        for (int i = 0; i < 8; ++i) w[(r * 8 + i) / 4][(r * 8 + i) % 4] = tmp[i];
      }
    }
    float y[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) y[i] = 0.0f;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int tau = t - 3 + j;
      float xv[8];
      if (tau >= bos) {
        load8(x + (size_t)tau * Cc + c0, xv);
      } else if (hist) {
        const int hidx = 3 - (bos - tau);  // 0..2, oldest first
#pragma unroll
        for (int i = 0; i < 8; ++i) xv[i] = ld_f(hist + (size_t)(c0 + i) * 3 + hidx);
      } else {
#pragma unroll
        for (int i = 0; i < 8; ++i) xv[i] = 0.0f;
      }
#pragma unroll
      for (int i = 0; i < 8; ++i) y[i] = fmaf(w[i][j], xv[i], y[i]);
    }
#pragma unroll
    for (int i = 0; i < 8; ++i) y[i] = silu_f(y[i]);

    const int two_hk = 2 * p.Hk;
    if (seg < two_hk) {
      float ss = 0.0f;
#pragma unroll
      for (int i = 0; i < 8; ++i) ss = fmaf(y[i], y[i], ss);
#pragma unroll
      for (int o = TPS / 2; o > 0; o >>= 1) ss += __shfl_xor_sync(seg_mask, ss, o, 32);
      const bool is_q = seg < p.Hk;
      const float r = rsqrtf(ss + p.eps_l2) * (is_q ? p.scale : 1.0f);
#pragma unroll
      for (int i = 0; i < 8; ++i) y[i] *= r;
      if (valid) {
        TM* dst = static_cast<TM*>(is_q ? p.q : p.k);
        const int col = c0 - (is_q ? 0 : p.Hk * D);
        store8(dst + (size_t)t * p.Hk * D + col, y);
      }
    } else if (valid) {
      const int col = c0 - two_hk * D;
      store8(static_cast<TM*>(p.v) + (size_t)t * p.Hv * D + col, y);
      if ((c0 % D) == 0) {
        const int h = seg - two_hk;
        const float av = ld_f(static_cast<const T*>(p.a) + (size_t)t * p.Hv + h);
        const float bv = ld_f(static_cast<const T*>(p.b) + (size_t)t * p.Hv + h);
        const float gg = -expf(__ldg(p.A_log + h)) * softplus_f(av + __ldg(p.dt_bias + h));
        p.g[(size_t)h * p.T + t] = gg;
        p.beta[(size_t)h * p.T + t] = sigmoid_f(bv);
      }
    }
  } else {
    // ------------------------------------------------------- tail threads
    if (p.conv_state_out == nullptr) return;
    const size_t tid = (size_t)(blockIdx.x - p.tok_blocks) * blockDim.x + threadIdx.x;
    if (tid >= (size_t)p.N * groups) return;
    const int n = (int)(tid / groups);
    const int c0 = (int)(tid % groups) * 8;
    const int bos = clampi(__ldg(p.cu_seqlens + n), 0, p.T);
    const int eos = clampi(__ldg(p.cu_seqlens + n + 1), bos, p.T);
    const int len = eos - bos;
    const T* hist = hist_all ? hist_all + (size_t)n * Cc * 3 : nullptr;
    T* dst = static_cast<T*>(p.conv_state_out) + (size_t)n * Cc * 3;
#pragma unroll
    for (int s = 0; s < 3; ++s) {
      const int idx = len - 3 + s;  // index into the sequence; < 0 -> history
      float xv[8];
      if (idx >= 0) {
        load8(x + (size_t)(bos + idx) * Cc + c0, xv);
      } else if (hist) {
#pragma unroll
        for (int i = 0; i < 8; ++i) xv[i] = ld_f(hist + (size_t)(c0 + i) * 3 + (3 + idx));
      } else {
#pragma unroll
        for (int i = 0; i < 8; ++i) xv[i] = 0.0f;
      }
#pragma unroll
      for (int i = 0; i < 8; ++i) st_f(dst + (size_t)(c0 + i) * 3 + s, xv[i]);
    }
  }
}

cudaError_t launch_conv_prep(const ConvPrepParams& p0, int d, gdn_dtype dt, cudaStream_t st) {
  ConvPrepParams p = p0;
  const int groups = p.Cc / 8;
  const size_t n_tok = (size_t)p.T * groups;
  const size_t n_tail = (size_t)p.N * groups;
  p.tok_blocks = (int)((n_tok + 255) / 256);
  const int tail_blocks = (int)((n_tail + 255) / 256);
  const int blocks = p.tok_blocks + tail_blocks;
  if (blocks == 0) return cudaSuccess;
#define GDN_CONV_CASE(T_, TM_, D_) conv_prep_kernel<T_, TM_, D_><<<blocks, 256, 0, st>>>(p)
  // bf16 inputs -> fp16 intermediates (3 more significand bits for the
  // tensor-core operands); fp32 inputs -> fp32 intermediates.
  if (dt == GDN_BF16) {
    if (d == 128) GDN_CONV_CASE(__nv_bfloat16, __half, 128);
    else if (d == 64) GDN_CONV_CASE(__nv_bfloat16, __half, 64);
    else GDN_CONV_CASE(__nv_bfloat16, __half, 32);
  } else {
    if (d == 128) GDN_CONV_CASE(float, float, 128);
    else if (d == 64) GDN_CONV_CASE(float, float, 64);
    else GDN_CONV_CASE(float, float, 32);
  }
#undef GDN_CONV_CASE
  return cudaGetLastError();
}

}  // namespace gdn
