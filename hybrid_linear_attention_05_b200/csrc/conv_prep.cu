// Conv1d + SiLU + q/k L2 norm + gate preparation for gdn_prefill.
//
// The normalised q, k and the values are written as fp16 for bf16 inputs
// (fp32 for fp32 inputs): they are the tensor-core operands of the chunked
// core, and fp16 keeps three more significand bits than bf16 at the same size
// and MMA rate (all of them are bounded: |q|, |k| <= 1 after the norm).
//
// One thread handles 8 consecutive channels of TPT consecutive tokens (all
// TPT input rows are requested before the first is used): it
// keeps the conv window of those channels in registers (the three previous
// inputs, or the sequence's conv history before its first token), applies
// the depthwise 4-tap conv and SiLU token by token, and for q / k heads joins
// the other threads of its head in a shuffle reduction for the L2 norm.  The first thread of every
// value head also computes that head's gates g = -exp(A_log) softplus(a +
// dt_bias) and beta = sigmoid(b).  A second group of threads writes the conv
// tail (the last three raw inputs of every sequence).
//
// HBM traffic per token: the Cc-wide input row once (the three rows before a
// thread's first token are the previous thread's rows, served from L2), the
// Cc-wide normalised row once, and the gates.
#include "gdn_internal.h"

namespace gdn {

constexpr int TPT = 8;  // consecutive tokens per thread (sliding conv window)

// Eight input elements kept as loaded (16 B of bf16, 32 B of fp32) until use,
// so that all TPT rows of a thread can be in flight at once.
template <typename T> struct Raw8;
template <> struct Raw8<__nv_bfloat16> {
  uint4 u;
  __device__ __forceinline__ void load(const __nv_bfloat16* p) { u = *reinterpret_cast<const uint4*>(p); }
  __device__ __forceinline__ void to_f(float* f) const {
    const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&u);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float2 t = __bfloat1622float2(h[i]);
      f[2 * i] = t.x;
      f[2 * i + 1] = t.y;
    }
  }
};
template <> struct Raw8<float> {
  float4 a, b;
  __device__ __forceinline__ void load(const float* p) {
    a = reinterpret_cast<const float4*>(p)[0];
    b = reinterpret_cast<const float4*>(p)[1];
  }
  __device__ __forceinline__ void to_f(float* f) const {
    f[0] = a.x; f[1] = a.y; f[2] = a.z; f[3] = a.w;
    f[4] = b.x; f[5] = b.y; f[6] = b.z; f[7] = b.w;
  }
};

template <typename T, typename TM, int D>
__global__ void __launch_bounds__(256) conv_prep_kernel(ConvPrepParams p) {
  constexpr int TPS = D / 8;  // threads per head segment
  const int Cc = p.Cc;
  const int groups = Cc / 8;  // threads per block of TPT tokens
  const size_t gid = (size_t)blockIdx.x * blockDim.x + threadIdx.x;
  const int n_blocks_tok = (p.T + TPT - 1) / TPT;
  const size_t n_tok = (size_t)n_blocks_tok * groups;
  const T* __restrict__ x = static_cast<const T*>(p.x);
  const T* __restrict__ hist_all = static_cast<const T*>(p.conv_state_in);
  const int lane = threadIdx.x & 31;
  const unsigned seg_mask = ((TPS == 32) ? 0xffffffffu : ((1u << TPS) - 1u)) << (lane & ~(TPS - 1));

  if (blockIdx.x < p.tok_blocks) {
    // ------------------------------------------------------ token threads
    // This thread: channels c0 .. c0+7 of tokens t0 .. t0+TPT-1.  Segments
    // (the TPS threads of one head) share t0, so their shuffles line up.
    const bool valid = gid < n_tok;
    const int tb = valid ? (int)(gid / groups) : 0;
    const int cg = valid ? (int)(gid % groups) : 0;
    const int c0 = cg * 8;
    const int seg = c0 / D;
    const int t0 = tb * TPT;
    const int two_hk = 2 * p.Hk;
    const bool is_qk = seg < two_hk;
    const bool is_q = seg < p.Hk;

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
    // the TPT new input rows, issued together
    Raw8<T> xr[TPT];
#pragma unroll
    for (int k = 0; k < TPT; ++k) {
      const int t = min(t0 + k, p.T - 1);
      xr[k].load(x + (size_t)t * Cc + c0);
    }
    // conv window before token t0 (positions t0-3 .. t0-1) of t0's sequence
    int n = seq_of_token(p.cu_seqlens, p.N, min(t0, p.T - 1));
    int bos = clampi(__ldg(p.cu_seqlens + n), 0, p.T);
    int eos = clampi(__ldg(p.cu_seqlens + n + 1), bos, p.T);
    float win[3][8];
#pragma unroll
    for (int j = 0; j < 3; ++j) {
      const int tau = t0 - 3 + j;
      if (tau >= bos) {
        load8(x + (size_t)tau * Cc + c0, win[j]);
      } else if (hist_all) {
        const T* hist = hist_all + (size_t)n * Cc * 3;
#pragma unroll
        for (int i = 0; i < 8; ++i) win[j][i] = ld_f(hist + (size_t)(c0 + i) * 3 + (3 - (bos - tau)));
      } else {
#pragma unroll
        for (int i = 0; i < 8; ++i) win[j][i] = 0.f;
      }
    }

#pragma unroll
    for (int k = 0; k < TPT; ++k) {
      const int t = t0 + k;
      if (t >= p.T) break;  // the whole segment shares t: no divergent shuffle
      if (t >= eos) {
        // first token of a later sequence: its window is that sequence's history
        while (n + 1 < p.N && t >= __ldg(p.cu_seqlens + n + 1)) ++n;
        bos = clampi(__ldg(p.cu_seqlens + n), 0, p.T);
        eos = clampi(__ldg(p.cu_seqlens + n + 1), bos, p.T);
        const T* hist = hist_all ? hist_all + (size_t)n * Cc * 3 : nullptr;
#pragma unroll
        for (int j = 0; j < 3; ++j)
#pragma unroll
          for (int i = 0; i < 8; ++i)
            win[j][i] = hist ? ld_f(hist + (size_t)(c0 + i) * 3 + j) : 0.f;
      }
      float xk[8], y[8];
      xr[k].to_f(xk);
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        float acc = w[i][0] * win[0][i];
        acc = fmaf(w[i][1], win[1][i], acc);
        acc = fmaf(w[i][2], win[2][i], acc);
        acc = fmaf(w[i][3], xk[i], acc);
        y[i] = silu_f(acc);
        win[0][i] = win[1][i];
        win[1][i] = win[2][i];
        win[2][i] = xk[i];
      }
      if (is_qk) {
        float ss = 0.0f;
#pragma unroll
        for (int i = 0; i < 8; ++i) ss = fmaf(y[i], y[i], ss);
#pragma unroll
        for (int o = TPS / 2; o > 0; o >>= 1) ss += __shfl_xor_sync(seg_mask, ss, o, 32);
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
          const int hh = seg - two_hk;
          const float av = ld_f(static_cast<const T*>(p.a) + (size_t)t * p.Hv + hh);
          const float bv = ld_f(static_cast<const T*>(p.b) + (size_t)t * p.Hv + hh);
          const float gg = -expf(__ldg(p.A_log + hh)) * softplus_f(av + __ldg(p.dt_bias + hh));
          p.g[(size_t)hh * p.T + t] = gg;
          p.beta[(size_t)hh * p.T + t] = sigmoid_f(bv);
        }
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
  const size_t n_tok = (size_t)((p.T + TPT - 1) / TPT) * groups;
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
