// One decode step of the Gated DeltaNet mixer for a batch of sequences.
//
// One CTA per (sequence, key head) owns the G = Hv/Hk value heads that read
// that key head, so the conv-cache channels it updates in place (its q and k
// head, and its G value heads) belong to no other CTA.
//   1. conv over (cache[0..2], the new inputs) + SiLU for those channels,
//      cache shifted left with the new raw inputs appended;
//   2. L2 norm of q and k, gates alpha = exp(-exp(A_log) softplus(a+dt_bias)),
//      beta = sigmoid(b);
//   3. each state row S[r, :] (dk floats) is read once from HBM and written
//      once: u = S k, p = S q, delta = beta (v - alpha u),
//      S' = alpha S + delta k^T, o = alpha p + (k.q) delta   (= S' q);
//   4. gated RMSNorm of o with z.
// A step may carry T = 1..8 tokens per sequence (short multi-token decode,
// e.g. verifying drafted tokens): each state row then takes the T updates in
// turn while it is in registers, so the state is still read and written once.
// The state rows are spread over the warps with each lane holding a float4 of
// a row; row dot products are shuffle reductions over the lanes of the row.
// HBM traffic is dominated by the state: 2 * Hv * dk * dv * 4 bytes per
// token in fp32, half that with a bf16 state ("Qwen3.5", HF model doc, Usage
// tips: the single-token recurrence is memory-bandwidth-bound).  A bf16
// state is widened to fp32 on load and rounded to nearest on store; all
// arithmetic is fp32.
#include <type_traits>

#include "gdn_internal.h"

namespace gdn {

namespace {

// Four consecutive state entries (one lane's share of a row) in the state's
// storage type, widened to / narrowed from fp32.
template <typename S> struct State4;
template <> struct State4<float> {
  using Raw = float4;
  static __device__ __forceinline__ Raw load(const float* p) { return __ldcs(reinterpret_cast<const float4*>(p)); }
  static __device__ __forceinline__ float4 widen(Raw r) { return r; }
  static __device__ __forceinline__ void store(float* p, float4 v) { __stcs(reinterpret_cast<float4*>(p), v); }
};
template <> struct State4<__nv_bfloat16> {
  using Raw = uint2;
  static __device__ __forceinline__ Raw load(const __nv_bfloat16* p) { return __ldcs(reinterpret_cast<const uint2*>(p)); }
  static __device__ __forceinline__ float4 widen(Raw r) {
    const float2 a = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&r.x));
    const float2 b = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&r.y));
    return make_float4(a.x, a.y, b.x, b.y);
  }
  static __device__ __forceinline__ void store(__nv_bfloat16* p, float4 v) {
    uint2 r;
    *reinterpret_cast<__nv_bfloat162*>(&r.x) = __floats2bfloat162_rn(v.x, v.y);
    *reinterpret_cast<__nv_bfloat162*>(&r.y) = __floats2bfloat162_rn(v.z, v.w);
    __stcs(reinterpret_cast<uint2*>(p), r);
  }
};

// Row sums of RG rows at once: v[j] holds this lane's partial sum of row j,
// and the LPR lanes of a row group hold the rest.  A butterfly that trades
// half of the remaining rows at each of the first log2(RG) levels (the lane
// with the level's bit set keeps the upper half) and sums plainly at the
// others leaves every lane with the full sum of row (lane % LPR) / (LPR / RG).
// That takes RG - 1 + log2(LPR / RG) shuffles instead of RG log2(LPR)
// (9 instead of 40 for 8 rows over 32 lanes).
template <int RG, int LPR>
__device__ __forceinline__ float rows_sum_transposed(float (&v)[RG], int lane) {
#pragma unroll
  for (int lev = 0; (LPR >> (lev + 1)) > 0; ++lev) {
    const int o = LPR >> (lev + 1);
    const int c = RG >> lev;  // rows still held
    if (c > 1) {
      const bool up = (lane & o) != 0;
#pragma unroll
      for (int j = 0; j < c / 2; ++j) {
        const float send = up ? v[j] : v[j + c / 2];
        const float keep = up ? v[j + c / 2] : v[j];
        v[j] = keep + __shfl_xor_sync(0xffffffffu, send, o, 32);
      }
    } else {
      v[0] += __shfl_xor_sync(0xffffffffu, v[0], o, 32);
    }
  }
  return v[0];
}

template <typename T, typename SD, int D>
__global__ void __launch_bounds__(256) decode_kernel(DecodeParams p) {
  using SV = State4<SD>;
  constexpr int NT = 256, NW = NT / 32;
  constexpr int LPR = D / 4;            // lanes per state row
  constexpr int RPW = 32 / LPR;         // rows per warp per pass
  constexpr int ROWS_PER_WARP = D / NW; // rows of one head handled by a warp
  constexpr int PASSES = ROWS_PER_WARP / RPW;
  static_assert(PASSES >= 1, "decode layout");

  extern __shared__ float sm[];
  const int G = p.Hv / p.Hk;
  float* ys = sm;                 // [(2 + G) * D] q | k | v of this CTA
  float* os = ys + (2 + G) * D;   // [G * D] core outputs
  float* misc = os + G * D;       // [4 + 2G]: rq, rk, kq, -, alpha[G], beta[G]

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int b = blockIdx.x / p.Hk, kh = blockIdx.x % p.Hk;
  const int Cc = p.Cc;
  const int NC = (2 + G) * D;
  const T* xrow = static_cast<const T*>(p.x) + (size_t)b * Cc;
  T* cs = static_cast<T*>(p.conv_state) + (size_t)b * Cc * 3;
  const T* cw = static_cast<const T*>(p.conv_w);

  // The first value head's state rows are requested before anything else:
  // they do not depend on the conv, so their HBM latency overlaps steps 1-2.
  const int col = (lane % LPR) * 4;
  SD* const state = static_cast<SD*>(p.state);
  auto state_of = [&](int gi) { return state + ((size_t)b * p.Hv + kh * G + gi) * D * D; };
  auto row_of = [&](int s) { return warp * ROWS_PER_WARP + s * RPW + lane / LPR; };
  typename SV::Raw Sv[PASSES];
  {
    const SD* S0 = state_of(0);
#pragma unroll
    for (int s = 0; s < PASSES; ++s) Sv[s] = SV::load(S0 + (size_t)row_of(s) * D + col);
  }

  // 1. conv + SiLU, cache update in place (each channel read then written by one thread)
  for (int idx = tid; idx < NC; idx += NT) {
    int c;
    if (idx < D) c = kh * D + idx;
    else if (idx < 2 * D) c = p.Hk * D + kh * D + (idx - D);
    else c = 2 * p.Hk * D + kh * G * D + (idx - 2 * D);
    const float xn = ld_f(xrow + c);
    const float h0 = ld_f(cs + (size_t)c * 3 + 0);
    const float h1 = ld_f(cs + (size_t)c * 3 + 1);
    const float h2 = ld_f(cs + (size_t)c * 3 + 2);
    float y = ld_f(cw + (size_t)c * 4 + 0) * h0;
    y = fmaf(ld_f(cw + (size_t)c * 4 + 1), h1, y);
    y = fmaf(ld_f(cw + (size_t)c * 4 + 2), h2, y);
    y = fmaf(ld_f(cw + (size_t)c * 4 + 3), xn, y);
    ys[idx] = silu_f(y);
    st_f(cs + (size_t)c * 3 + 0, h1);
    st_f(cs + (size_t)c * 3 + 1, h2);
    st_f(cs + (size_t)c * 3 + 2, xn);
  }
  __syncthreads();
  // 2. norms and gates
  if (warp < 2) {
    float ss = 0.f;
    for (int i = lane; i < D; i += 32) { const float v = ys[warp * D + i]; ss = fmaf(v, v, ss); }
    ss = warp_sum(ss);
    if (lane == 0) misc[warp] = rsqrtf(ss + p.eps_l2) * (warp == 0 ? p.scale : 1.0f);
  } else if (warp == 2) {
    for (int gi = lane; gi < G; gi += 32) {
      const int h = kh * G + gi;
      const float av = ld_f(static_cast<const T*>(p.a) + (size_t)b * p.Hv + h);
      const float bv = ld_f(static_cast<const T*>(p.b) + (size_t)b * p.Hv + h);
      const float gg = -expf(__ldg(p.A_log + h)) * softplus_f(av + __ldg(p.dt_bias + h));
      misc[4 + gi] = expf(gg);
      misc[4 + G + gi] = sigmoid_f(bv);
    }
  }
  __syncthreads();
  for (int i = tid; i < 2 * D; i += NT) ys[i] *= misc[i < D ? 0 : 1];
  __syncthreads();
  if (warp == 0) {
    float kq = 0.f;
    for (int i = lane; i < D; i += 32) kq = fmaf(ys[i], ys[D + i], kq);
    kq = warp_sum(kq);
    if (lane == 0) misc[2] = kq;
  }
  __syncthreads();

  // 3. state stream; while head gi is updated, head gi + 1's rows are requested
  const float* qv = ys;
  const float* kv = ys + D;
  const float4 k4 = make_float4(kv[col], kv[col + 1], kv[col + 2], kv[col + 3]);
  const float4 q4 = make_float4(qv[col], qv[col + 1], qv[col + 2], qv[col + 3]);
  const float kq = misc[2];
  // the row sums of RG passes at a time are reduced together
  // (rows_sum_transposed): 8 for an fp32 state, 4 for a bf16 one (measured at
  // batch 256, 16/32 heads of width 128: 102 us against 106 us with each
  // row's sums reduced on their own and 130 us with 8)
  constexpr int RG = std::is_same<SD, float>::value ? (PASSES < 8 ? PASSES : 8) : (PASSES < 4 ? PASSES : 4);
  static_assert(RG <= LPR && PASSES % RG == 0, "decode layout");
  const int jr = (lane % LPR) / (LPR / RG);  // the pass of a group whose sums this lane ends with
  const int src0 = lane - lane % LPR;        // first lane of this lane's row group
  for (int gi = 0; gi < G; ++gi) {
    const int h = kh * G + gi;
    const float alpha = misc[4 + gi], beta = misc[4 + G + gi];
    SD* Sh = state + ((size_t)b * p.Hv + h) * D * D;
    const SD* Snext = gi + 1 < G ? state_of(gi + 1) : nullptr;
    const float* vv = ys + (2 + gi) * D;
#pragma unroll
    for (int s0 = 0; s0 < PASSES; s0 += RG) {
      float4 sv[RG];
      float u[RG], pp[RG];
#pragma unroll
      for (int j = 0; j < RG; ++j) {
        sv[j] = SV::widen(Sv[s0 + j]);
        u[j] = sv[j].x * k4.x + sv[j].y * k4.y + sv[j].z * k4.z + sv[j].w * k4.w;
        pp[j] = sv[j].x * q4.x + sv[j].y * q4.y + sv[j].z * q4.z + sv[j].w * q4.w;
      }
      const float us = rows_sum_transposed<RG, LPR>(u, lane);
      const float ps = rows_sum_transposed<RG, LPR>(pp, lane);
      const int r_me = row_of(s0 + jr);
      const float d_me = beta * (vv[r_me] - alpha * us);
      if ((lane % (LPR / RG)) == 0) os[gi * D + r_me] = fmaf(alpha, ps, kq * d_me);
#pragma unroll
      for (int j = 0; j < RG; ++j) {
        const int r = row_of(s0 + j);
        const float delta = RG == 1 ? d_me : __shfl_sync(0xffffffffu, d_me, src0 + j * (LPR / RG), 32);
        float4 sn;
        sn.x = fmaf(alpha, sv[j].x, delta * k4.x);
        sn.y = fmaf(alpha, sv[j].y, delta * k4.y);
        sn.z = fmaf(alpha, sv[j].z, delta * k4.z);
        sn.w = fmaf(alpha, sv[j].w, delta * k4.w);
        SV::store(Sh + (size_t)r * D + col, sn);
        if (Snext) Sv[s0 + j] = SV::load(Snext + (size_t)r * D + col);
      }
    }
  }
  __syncthreads();

  // 4. gated RMSNorm, one warp per value head
  for (int gi = warp; gi < G; gi += NW) {
    const int h = kh * G + gi;
    float ss = 0.f;
    for (int r = lane; r < D; r += 32) { const float o = os[gi * D + r]; ss = fmaf(o, o, ss); }
    ss = warp_sum(ss);
    const float inv = rsqrtf(ss / D + p.eps_norm);
    const T* zz = static_cast<const T*>(p.z) + ((size_t)b * p.Hv + h) * D;
    T* oo = static_cast<T*>(p.out) + ((size_t)b * p.Hv + h) * D;
    const T* ww = static_cast<const T*>(p.norm_w);
    for (int r = lane; r < D; r += 32)
      st_f(oo + r, os[gi * D + r] * inv * ld_f(ww + r) * silu_f(ld_f(zz + r)));
  }
}

// The same step for p.T = 2..8 tokens per sequence (short multi-token
// decode): each state row takes the T tokens' updates in turn while it is in
// registers, so the state is still read and written once per step.
template <typename T, typename SD, int D>
__global__ void __launch_bounds__(256, 3) decode_multi_kernel(DecodeParams p) {
  using SV = State4<SD>;
  constexpr int NT = 256, NW = NT / 32;
  constexpr int LPR = D / 4;            // lanes per state row
  constexpr int RPW = 32 / LPR;         // rows per warp per pass
  constexpr int ROWS_PER_WARP = D / NW; // rows of one head handled by a warp
  constexpr int PASSES = ROWS_PER_WARP / RPW;
  static_assert(PASSES >= 1, "decode layout");

  extern __shared__ float sm[];
  const int G = p.Hv / p.Hk;
  const int TK = p.T;             // tokens of every sequence in this step
  const int NC = (2 + G) * D;     // channels of this CTA
  const int MS = 4 + 2 * G;
  float* ys = sm;                 // [TK][NC] q | k | v of each token
  float* os = ys + TK * NC;       // [TK][G * D] core outputs
  float* misc = os + TK * G * D;  // [TK][MS]: rq, rk, kq, -, alpha[G], beta[G]

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int b = blockIdx.x / p.Hk, kh = blockIdx.x % p.Hk;
  const int Cc = p.Cc;
  const T* xb = static_cast<const T*>(p.x) + (size_t)b * TK * Cc;  // token t at xb + t Cc
  T* cs = static_cast<T*>(p.conv_state) + (size_t)b * Cc * 3;
  const T* cw = static_cast<const T*>(p.conv_w);

  // A thread's rows of a head are taken RG at a time (a "group"); the first
  // group is requested before anything else, each next one while the current
  // one is updated, so the state latency overlaps the conv and the updates.
  constexpr int RG = PASSES < 4 ? PASSES : 4;
  constexpr int NGH = PASSES / RG;  // groups per head
  static_assert(RG <= LPR, "decode layout");
  const int col = (lane % LPR) * 4;
  const int jr = (lane % LPR) / (LPR / RG);  // the row of a group whose sums this lane ends with
  const int src0 = lane - lane % LPR;        // first lane of this lane's row group
  SD* const state = static_cast<SD*>(p.state);
  auto row_of = [&](int s) { return warp * ROWS_PER_WARP + s * RPW + lane / LPR; };
  // group q: head q / NGH, passes (q % NGH) RG .. + RG - 1
  auto group_ptr = [&](int q, int j) {
    return state + ((size_t)b * p.Hv + kh * G + q / NGH) * D * D + (size_t)row_of((q % NGH) * RG + j) * D + col;
  };
  typename SV::Raw Sv[RG];
#pragma unroll
  for (int j = 0; j < RG; ++j) Sv[j] = SV::load(group_ptr(0, j));

  // 1. conv + SiLU over [cache, x_0 .. x_{TK-1}]; the cache keeps the last
  //    three raw inputs (each channel read then written by one thread)
  for (int idx = tid; idx < NC; idx += NT) {
    int c;
    if (idx < D) c = kh * D + idx;
    else if (idx < 2 * D) c = p.Hk * D + kh * D + (idx - D);
    else c = 2 * p.Hk * D + kh * G * D + (idx - 2 * D);
    const float w0 = ld_f(cw + (size_t)c * 4 + 0), w1 = ld_f(cw + (size_t)c * 4 + 1);
    const float w2 = ld_f(cw + (size_t)c * 4 + 2), w3 = ld_f(cw + (size_t)c * 4 + 3);
    float h0 = ld_f(cs + (size_t)c * 3 + 0);
    float h1 = ld_f(cs + (size_t)c * 3 + 1);
    float h2 = ld_f(cs + (size_t)c * 3 + 2);
    for (int t = 0; t < TK; ++t) {
      const float xn = ld_f(xb + (size_t)t * Cc + c);
      float y = w0 * h0;
      y = fmaf(w1, h1, y);
      y = fmaf(w2, h2, y);
      y = fmaf(w3, xn, y);
      ys[t * NC + idx] = silu_f(y);
      h0 = h1;
      h1 = h2;
      h2 = xn;
    }
    st_f(cs + (size_t)c * 3 + 0, h0);
    st_f(cs + (size_t)c * 3 + 1, h1);
    st_f(cs + (size_t)c * 3 + 2, h2);
  }
  __syncthreads();
  // 2. norms and gates of every token
  for (int job = warp; job < 2 * TK; job += NW) {  // the q (even) and k (odd) norms
    const int t = job >> 1, which = job & 1;
    const float* y = ys + t * NC + which * D;
    float ss = 0.f;
    for (int i = lane; i < D; i += 32) ss = fmaf(y[i], y[i], ss);
    ss = warp_sum(ss);
    if (lane == 0) misc[t * MS + which] = rsqrtf(ss + p.eps_l2) * (which == 0 ? p.scale : 1.0f);
  }
  for (int j = tid; j < TK * G; j += NT) {
    const int t = j / G, gi = j % G, h = kh * G + gi;
    const size_t row = (size_t)b * TK + t;
    const float av = ld_f(static_cast<const T*>(p.a) + row * p.Hv + h);
    const float bv = ld_f(static_cast<const T*>(p.b) + row * p.Hv + h);
    const float gg = -expf(__ldg(p.A_log + h)) * softplus_f(av + __ldg(p.dt_bias + h));
    misc[t * MS + 4 + gi] = expf(gg);
    misc[t * MS + 4 + G + gi] = sigmoid_f(bv);
  }
  __syncthreads();
  for (int i = tid; i < TK * 2 * D; i += NT) {
    const int t = i / (2 * D), j = i % (2 * D);
    ys[t * NC + j] *= misc[t * MS + (j < D ? 0 : 1)];
  }
  __syncthreads();
  for (int t = warp; t < TK; t += NW) {
    const float* q = ys + t * NC;
    float kq = 0.f;
    for (int i = lane; i < D; i += 32) kq = fmaf(q[i], q[D + i], kq);
    kq = warp_sum(kq);
    if (lane == 0) misc[t * MS + 2] = kq;
  }
  __syncthreads();

  // 3. state stream: a group of this thread's rows stays in registers while
  //    the TK tokens update it in turn; the rows of one token are
  //    independent, so their row reductions overlap.
  for (int q = 0; q < G * NGH; ++q) {
    const int gi = q / NGH;
    float4 sv[RG];
#pragma unroll
    for (int j = 0; j < RG; ++j) sv[j] = SV::widen(Sv[j]);
    if (q + 1 < G * NGH) {
#pragma unroll
      for (int j = 0; j < RG; ++j) Sv[j] = SV::load(group_ptr(q + 1, j));
    }
    for (int t = 0; t < TK; ++t) {
      const float* qt = ys + t * NC;
      const float4 q4 = *reinterpret_cast<const float4*>(qt + col);
      const float4 k4 = *reinterpret_cast<const float4*>(qt + D + col);
      const float alpha = misc[t * MS + 4 + gi], beta = misc[t * MS + 4 + G + gi], kq = misc[t * MS + 2];
      float u[RG], pp[RG];
#pragma unroll
      for (int j = 0; j < RG; ++j) {
        u[j] = sv[j].x * k4.x + sv[j].y * k4.y + sv[j].z * k4.z + sv[j].w * k4.w;
        pp[j] = sv[j].x * q4.x + sv[j].y * q4.y + sv[j].z * q4.z + sv[j].w * q4.w;
      }
      // this lane ends with u and p of its row jr of the group; delta and the
      // output of that row are formed there, delta goes back to the row's lanes
      const float us = rows_sum_transposed<RG, LPR>(u, lane);
      const float ps = rows_sum_transposed<RG, LPR>(pp, lane);
      const int r_me = row_of((q % NGH) * RG + jr);
      const float d_me = beta * (qt[(2 + gi) * D + r_me] - alpha * us);
      if ((lane % (LPR / RG)) == 0) os[(t * G + gi) * D + r_me] = fmaf(alpha, ps, kq * d_me);
#pragma unroll
      for (int j = 0; j < RG; ++j) {
        const float delta = RG == 1 ? d_me : __shfl_sync(0xffffffffu, d_me, src0 + j * (LPR / RG), 32);
        sv[j].x = fmaf(alpha, sv[j].x, delta * k4.x);
        sv[j].y = fmaf(alpha, sv[j].y, delta * k4.y);
        sv[j].z = fmaf(alpha, sv[j].z, delta * k4.z);
        sv[j].w = fmaf(alpha, sv[j].w, delta * k4.w);
      }
    }
#pragma unroll
    for (int j = 0; j < RG; ++j) SV::store(group_ptr(q, j), sv[j]);
  }
  __syncthreads();

  // 4. gated RMSNorm, one warp per (token, value head)
  for (int job = warp; job < TK * G; job += NW) {
    const int t = job / G, gi = job % G, h = kh * G + gi;
    const float* o = os + (t * G + gi) * D;
    float ss = 0.f;
    for (int r = lane; r < D; r += 32) ss = fmaf(o[r], o[r], ss);
    ss = warp_sum(ss);
    const float inv = rsqrtf(ss / D + p.eps_norm);
    const size_t row = ((size_t)b * TK + t) * p.Hv + h;
    const T* zz = static_cast<const T*>(p.z) + row * D;
    T* oo = static_cast<T*>(p.out) + row * D;
    const T* ww = static_cast<const T*>(p.norm_w);
    for (int r = lane; r < D; r += 32) st_f(oo + r, o[r] * inv * ld_f(ww + r) * silu_f(ld_f(zz + r)));
  }
}

template <typename T, typename SD, int D>
cudaError_t launch_ts(const DecodeParams& p, cudaStream_t st) {
  const int G = p.Hv / p.Hk;
  const size_t smem = (size_t)p.T * ((size_t)(2 + G) * D + (size_t)G * D + 4 + 2 * G) * sizeof(float);
  if (smem > 48 * 1024) {
    cudaError_t e = cudaFuncSetAttribute(p.T == 1 ? decode_kernel<T, SD, D> : decode_multi_kernel<T, SD, D>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
  }
  if (p.T == 1) decode_kernel<T, SD, D><<<p.B * p.Hk, 256, smem, st>>>(p);
  else decode_multi_kernel<T, SD, D><<<p.B * p.Hk, 256, smem, st>>>(p);
  return cudaGetLastError();
}
template <typename T, int D>
cudaError_t launch_t(const DecodeParams& p, cudaStream_t st) {
  return p.state_bf16 ? launch_ts<T, __nv_bfloat16, D>(p, st) : launch_ts<T, float, D>(p, st);
}

}  // namespace

cudaError_t launch_decode(const DecodeParams& p, int d, gdn_dtype dt, cudaStream_t st) {
  if (p.B == 0) return cudaSuccess;
  if (dt == GDN_BF16) {
    if (d == 128) return launch_t<__nv_bfloat16, 128>(p, st);
    if (d == 64) return launch_t<__nv_bfloat16, 64>(p, st);
    return launch_t<__nv_bfloat16, 32>(p, st);
  }
  if (d == 128) return launch_t<float, 128>(p, st);
  if (d == 64) return launch_t<float, 64>(p, st);
  return launch_t<float, 32>(p, st);
}

}  // namespace gdn
