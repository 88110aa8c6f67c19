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
#include <string.h>

#include "gdn_internal.h"
#include "host_util.h"
#include "tc_ptx.cuh"

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

// Rounding residual of eight values stored as fp16: fp16(x - fp16(x)).
__device__ __forceinline__ void store_lo8(__half* p, const float* f) {
  float r[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) r[i] = f[i] - __half2float(__float2half_rn(f[i]));
  store8(p, r);
}
__device__ __forceinline__ void store_lo8(float*, const float*) {}  // fp32 intermediates: none

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
          void* lo = is_q ? p.q_lo : p.k_lo;
          if (lo) store_lo8(static_cast<TM*>(lo) + (size_t)t * p.Hk * D + col, y);
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

// ------------------------------------------------------------------------
// The bf16 / head-width-128 case (the shapes of the Qwen3.5 family), staged
// through shared memory by TMA.
//
// A tile is 64 tokens of one 128-channel head segment (q, k or v head).  One
// 2-D TMA box brings its 67 input rows -- the 64 tokens and the 3 before
// them, which the conv window needs; rows before token 0 read as zeros --
// into shared memory, 256 B per row.  Persistent CTAs of 128 threads walk
// the tiles with a two-buffer ring, so the next tile's box is in flight while
// this one is computed; the head's conv taps (1 KiB) arrive with each box.  Thread (tg = tid / 16, cg = tid % 16) takes channels
// 8 cg .. 8 cg + 7 of tokens 8 tg .. 8 tg + 7: the 16 threads of a token
// group hold one whole head and reduce the L2 norm with shuffles.  Window
// rows before a sequence's first token come from its conv history (or are
// zero), as in the generic kernel.  CTAs past the persistent ones write the
// conv tails.
constexpr int KT = 64;              // tokens per tile
constexpr int KR = KT + 3;          // rows per box
constexpr int KNT = 128;            // threads per CTA
constexpr uint32_t KW = KR * 256;   // the head's conv taps (128 x 4 bf16) follow the box
constexpr uint32_t KBUF = 18432;    // one box (67 x 256 B) and the taps (1 KiB), rounded up to 1 KiB
constexpr int KST = 2;               // boxes in flight per CTA
constexpr uint32_t KSMEM = KST * KBUF + 64 + 1024;
constexpr int KCTAS_PER_SM = 5;

__device__ int g_conv_error = 0;  // nonzero: a box of conv_tma_kernel never landed

__global__ void __launch_bounds__(KNT, KCTAS_PER_SM)
    conv_tma_kernel(const __grid_constant__ CUtensorMap tm_x, ConvPrepParams p, int n_tiles, int main_ctas) {
  constexpr int D = 128;
  extern __shared__ uint8_t conv_raw[];
  uint8_t* smem = conv_raw + ((1024u - (ptx::smem_u32(conv_raw) & 1023u)) & 1023u);
  const uint32_t sb = ptx::smem_u32(smem);
  const uint32_t bar0 = sb + KST * KBUF;
  const int tid = threadIdx.x;
  const int Cc = p.Cc;
  const int n_ct = Cc / D;  // head segments
  const __nv_bfloat16* __restrict__ x = static_cast<const __nv_bfloat16*>(p.x);
  const __nv_bfloat16* __restrict__ hist_all = static_cast<const __nv_bfloat16*>(p.conv_state_in);
  // the key-side kernel may be scheduled now; it waits for this grid to finish
  ptx::pdl_launch();

  if ((int)blockIdx.x >= main_ctas) {
    // ------------------------------------------------------ conv tails
    if (p.conv_state_out == nullptr) return;
    const int groups = Cc / 8;
    const size_t item = (size_t)(blockIdx.x - main_ctas) * KNT + tid;
    if (item >= (size_t)p.N * groups) return;
    const int n = (int)(item / groups);
    const int c0 = (int)(item % groups) * 8;
    const int bos = clampi(__ldg(p.cu_seqlens + n), 0, p.T);
    const int eos = clampi(__ldg(p.cu_seqlens + n + 1), bos, p.T);
    const int len = eos - bos;
    const __nv_bfloat16* hist = hist_all ? hist_all + (size_t)n * Cc * 3 : nullptr;
    __nv_bfloat16* dst = static_cast<__nv_bfloat16*>(p.conv_state_out) + (size_t)n * Cc * 3;
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
    return;
  }

  if (tid == 0) {
    for (int b = 0; b < KST; ++b) ptx::mbar_init(bar0 + 8 * b, 1);
    ptx::fence_mbar_init();
  }
  __syncthreads();
  auto issue = [&](int tile, int buf) {
    const int ct = tile % n_ct, tt = tile / n_ct;
    const uint32_t bar = bar0 + 8 * buf;
    ptx::mbar_arrive_expect_tx(bar, (uint32_t)(KR * 256 + 1024));
    ptx::tma_load_2d(sb + buf * KBUF, &tm_x, ct * D, tt * KT - 3, bar);
    ptx::bulk_load(sb + buf * KBUF + KW, static_cast<const __nv_bfloat16*>(p.conv_w) + (size_t)ct * D * 4, 1024, bar);
  };

  const int cg = tid & 15, tg = tid >> 4;
  const unsigned seg_mask = 0xffffu << (tid & 16);
  int tile = blockIdx.x;
  if (tid == 0)
    for (int b = 0; b < KST - 1; ++b)
      if (tile + b * main_ctas < n_tiles) issue(tile + b * main_ctas, b);
  for (int k = 0; tile < n_tiles; ++k, tile += main_ctas) {
    const int buf = k % KST;
    // refill the buffer the previous tile used (everyone passed the barrier after reading it)
    if (tid == 0 && tile + (KST - 1) * main_ctas < n_tiles) issue(tile + (KST - 1) * main_ctas, (k + KST - 1) % KST);
    const int ct = tile % n_ct, tt = tile / n_ct;
    const int c0 = ct * D + cg * 8;
    const int t0 = tt * KT + tg * 8;
    const bool is_qk = ct < 2 * p.Hk, is_q = ct < p.Hk;
    // gate inputs: in a value head's token group, thread cg < 8 takes token
    // t0 + cg; requested before the wait so that their latency overlaps it
    const int hh = ct - 2 * p.Hk;
    const int tgate = t0 + cg;
    const bool gates = !is_qk && cg < 8 && tgate < p.T;
    float av = 0.f, bv = 0.f;
    if (gates) {
      av = ld_f(static_cast<const __nv_bfloat16*>(p.a) + (size_t)tgate * p.Hv + hh);
      bv = ld_f(static_cast<const __nv_bfloat16*>(p.b) + (size_t)tgate * p.Hv + hh);
    }
    int n = seq_of_token(p.cu_seqlens, p.N, min(t0, p.T - 1));
    int bos = clampi(__ldg(p.cu_seqlens + n), 0, p.T);
    int eos = clampi(__ldg(p.cu_seqlens + n + 1), bos, p.T);
    // the box cannot fail to land; the bounded wait only keeps a broken
    // launch from spinning forever
    if (__syncthreads_or(!ptx::mbar_wait(bar0 + 8 * buf, (uint32_t)(k / KST) & 1u))) {
      if (tid == 0) {  // record it and let the boxes in flight land before leaving
        atomicExch(&g_conv_error, 1);
        for (int b = 0; b < KST; ++b)
          if (tile + b * main_ctas < n_tiles)
            ptx::mbar_wait(bar0 + 8 * ((k + b) % KST), (uint32_t)((k + b) / KST) & 1u, 100000000ull);
      }
      break;
    }
    const uint8_t* rows = smem + buf * KBUF + cg * 16;  // box row r of this thread at rows + 256 r
    // conv taps as channel pairs: wv[tap][pair] = (w[2 pair][tap], w[2 pair + 1][tap])
    float2 wv[4][4];
    {
      const __nv_bfloat16* wsm = reinterpret_cast<const __nv_bfloat16*>(smem + buf * KBUF + KW) + cg * 32;
      float tmp[32];
#pragma unroll
      for (int r = 0; r < 4; ++r) load8(wsm + r * 8, tmp + r * 8);
#pragma unroll
      for (int q = 0; q < 4; ++q)
#pragma unroll
        for (int tap = 0; tap < 4; ++tap) wv[tap][q] = make_float2(tmp[(2 * q) * 4 + tap], tmp[(2 * q + 1) * 4 + tap]);
    }
    auto row2 = [&](int r, float2* f) {  // eight bf16 of box row r as four channel pairs
      const uint4 u = *reinterpret_cast<const uint4*>(rows + 256 * r);
      const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&u);
#pragma unroll
      for (int q = 0; q < 4; ++q) f[q] = __bfloat1622float2(h[q]);
    };
    auto hist2 = [&](int j, float2* f) {  // conv history slot j of sequence n (zeros without one)
      const __nv_bfloat16* hist = hist_all ? hist_all + (size_t)n * Cc * 3 : nullptr;
#pragma unroll
      for (int q = 0; q < 4; ++q)
        f[q] = hist ? make_float2(ld_f(hist + (size_t)(c0 + 2 * q) * 3 + j), ld_f(hist + (size_t)(c0 + 2 * q + 1) * 3 + j))
                    : make_float2(0.f, 0.f);
    };
    float2 win[3][4];
#pragma unroll
    for (int j = 0; j < 3; ++j) {
      const int tau = t0 - 3 + j;
      if (tau >= bos) row2(tg * 8 + j, win[j]);
      else hist2(3 - (bos - tau), win[j]);
    }
    // conv of token t (box row kk + 3 of this thread's group), sliding the window
    auto conv = [&](int t, int kk, float2* y) {
      if (t >= eos) {
        // first token of a later sequence: its window is that sequence's history
        while (n + 1 < p.N && t >= __ldg(p.cu_seqlens + n + 1)) ++n;
        bos = clampi(__ldg(p.cu_seqlens + n), 0, p.T);
        eos = clampi(__ldg(p.cu_seqlens + n + 1), bos, p.T);
#pragma unroll
        for (int j = 0; j < 3; ++j) hist2(j, win[j]);
      }
      float2 xk[4];
      row2(tg * 8 + kk + 3, xk);
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        float2 acc = __fmul2_rn(wv[0][q], win[0][q]);
        acc = __ffma2_rn(wv[1][q], win[1][q], acc);
        acc = __ffma2_rn(wv[2][q], win[2][q], acc);
        acc = __ffma2_rn(wv[3][q], xk[q], acc);
        y[q] = acc;
        win[0][q] = win[1][q];
        win[1][q] = win[2][q];
        win[2][q] = xk[q];
      }
    };
    // y <- y sigmoid(y) = y / (1 + 2^(-y log2 e)), two channels per step
    auto silu2 = [&](float2* y) {
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const float2 m = __fmul2_rn(y[q], make_float2(-1.4426950408889634f, -1.4426950408889634f));
        float2 e;
        asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(e.x) : "f"(m.x));
        asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(e.y) : "f"(m.y));
        const float2 dd = __fadd2_rn(e, make_float2(1.f, 1.f));
        float2 r;
        asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(r.x) : "f"(dd.x));
        asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(r.y) : "f"(dd.y));
        y[q] = __fmul2_rn(y[q], r);
      }
    };
    auto sumsq = [&](const float2* y) {
      float2 a = __fmul2_rn(y[0], y[0]);
#pragma unroll
      for (int q = 1; q < 4; ++q) a = __ffma2_rn(y[q], y[q], a);
      return a.x + a.y;
    };
    void* const lo = is_qk ? (is_q ? p.q_lo : p.k_lo) : nullptr;
    auto store = [&](int t, const float2* y, float f) {
      uint4 u;
      __half2* h = reinterpret_cast<__half2*>(&u);
      float2 x[4];
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        x[q] = __fmul2_rn(y[q], make_float2(f, f));
        h[q] = __float22half2_rn(x[q]);
      }
      const size_t qk_off = (size_t)t * p.Hk * D + (c0 - (is_q ? 0 : p.Hk * D));
      __half* dst = is_qk ? static_cast<__half*>(is_q ? p.q : p.k) + qk_off
                          : static_cast<__half*>(p.v) + (size_t)t * p.Hv * D + (c0 - 2 * p.Hk * D);
      *reinterpret_cast<uint4*>(dst) = u;
      if (lo) {  // rounding residuals of q and k: x - fp16(x), itself rounded to fp16
        uint4 ul;
        __half2* hl = reinterpret_cast<__half2*>(&ul);
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const float2 xh = __half22float2(h[q]);
          hl[q] = __float22half2_rn(make_float2(x[q].x - xh.x, x[q].y - xh.y));
        }
        *reinterpret_cast<uint4*>(static_cast<__half*>(lo) + qk_off) = ul;
      }
    };
    // two tokens at a time, so that their reductions and MUFU work overlap
#pragma unroll
    for (int kk = 0; kk < 8; kk += 2) {
      const int t = t0 + kk;
      if (t >= p.T) break;  // the token group shares t: no divergent shuffle
      const bool has1 = t + 1 < p.T;
      float2 y0[4], y1[4];
      conv(t, kk, y0);
      conv(t + 1, kk + 1, y1);
      silu2(y0);
      silu2(y1);
      float f0 = 1.f, f1 = 1.f;
      if (is_qk) {
        float s0 = sumsq(y0), s1 = sumsq(y1);
#pragma unroll
        for (int o = 8; o > 0; o >>= 1) {
          s0 += __shfl_xor_sync(seg_mask, s0, o, 32);
          s1 += __shfl_xor_sync(seg_mask, s1, o, 32);
        }
        const float sc = is_q ? p.scale : 1.0f;
        f0 = rsqrtf(s0 + p.eps_l2) * sc;
        f1 = rsqrtf(s1 + p.eps_l2) * sc;
      }
      store(t, y0, f0);
      if (has1) store(t + 1, y1, f1);
    }
    if (gates) {  // gates of value head hh for token tgate
      const float eA = expf(__ldg(p.A_log + hh)), db = __ldg(p.dt_bias + hh);
      p.g[(size_t)hh * p.T + tgate] = -eA * softplus_f(av + db);
      p.beta[(size_t)hh * p.T + tgate] = sigmoid_f(bv);
    }
    __syncthreads();  // this buffer is read; the next iteration's prefetch may refill it
  }
}

bool make_conv_map(CUtensorMap* m, const void* x, int T, int Cc) {
  host::EncodeTiledFn fn = host::encode_tiled();
  if (!fn) return false;
  cuuint64_t dims[2] = {(cuuint64_t)Cc, (cuuint64_t)T};
  cuuint64_t strides[1] = {(cuuint64_t)Cc * 2};
  cuuint32_t box[2] = {128, (cuuint32_t)KR};
  cuuint32_t es[2] = {1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(x), dims, strides, box, es,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

cudaError_t launch_conv_tma(const ConvPrepParams& p, cudaStream_t st) {
  CUtensorMap m;
  memset(&m, 0, sizeof(m));
  if (!make_conv_map(&m, p.x, p.T, p.Cc)) return cudaErrorInvalidValue;
  const int n_tiles = ((p.T + KT - 1) / KT) * (p.Cc / 128);
  const int main_ctas = n_tiles < host::sm_count() * KCTAS_PER_SM ? n_tiles : host::sm_count() * KCTAS_PER_SM;
  const int tail_ctas = p.conv_state_out ? (int)(((size_t)p.N * (p.Cc / 8) + KNT - 1) / KNT) : 0;
  if (main_ctas + tail_ctas == 0) return cudaSuccess;
  cudaError_t e = cudaFuncSetAttribute(conv_tma_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)KSMEM);
  if (e != cudaSuccess) return e;
  conv_tma_kernel<<<main_ctas + tail_ctas, KNT, KSMEM, st>>>(m, p, n_tiles, main_ctas);
  return cudaGetLastError();
}

int conv_error_word(int clear) {
  int v = 0;
  if (cudaMemcpyFromSymbol(&v, g_conv_error, sizeof(int)) != cudaSuccess) return -1;
  if (clear && v != 0) {
    const int zero = 0;
    if (cudaMemcpyToSymbol(g_conv_error, &zero, sizeof(int)) != cudaSuccess) return -1;
  }
  return v;
}

cudaError_t launch_conv_prep(const ConvPrepParams& p0, int d, gdn_dtype dt, cudaStream_t st) {
  if (dt == GDN_BF16 && d == 128 && p0.T > 0) return launch_conv_tma(p0, st);
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
