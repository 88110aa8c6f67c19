// Chunked gated delta rule on CUDA cores, fp32 throughout.
//
// One CTA per (value head, sequence) walks the sequence chunk by chunk with
// the dv x dk state in shared memory.  Within a chunk of L <= C tokens, with
// gamma_i the cumulative log decay of the chunk:
//   A_ij = beta_i e^{gamma_i - gamma_j} k_i.k_j (i > j);  T = (I + A)^-1
//   W = T diag(beta e^gamma) K,  U = T diag(beta) V,  Vn = U - W S^T
//   O = diag(e^gamma) Q S^T + (Q K^T o causal decay) Vn
//   S <- e^{gamma_L} S + Vn^T diag(e^{gamma_L - gamma}) K
// and the gated RMSNorm of O is applied before the store.  This is the
// chunked (WY / UT transform) form of the recurrence; it is exact in real
// arithmetic ("Qwen (text & vision-language)", Verified parity).
//
// This kernel covers the shapes the tensor-core kernel does not (small heads,
// fp32 inputs, short chunks) and serves as an fp32 cross-check of it.
#include "gdn_internal.h"

namespace gdn {

namespace {

template <int D, int C>
struct SimtSmem {
  static constexpr int DP = D + 1;  // padded row strides (no bank conflicts on column walks)
  static constexpr int CP = C + 1;
  static constexpr size_t floats = (size_t)D * DP + 5 * (size_t)C * DP + 3 * (size_t)C * CP + 4 * C;
  static constexpr size_t bytes = floats * sizeof(float);
};

template <typename T, typename TM, int D, int C>
__global__ void __launch_bounds__(256) chunk_simt_kernel(ChunkParams p) {
  using SM = SimtSmem<D, C>;
  constexpr int DP = SM::DP, CP = SM::CP, NT = 256;
  extern __shared__ float smem[];
  float* S = smem;                 // [D][DP]   state, row = value channel
  float* Ks = S + D * DP;          // [C][DP]
  float* Qs = Ks + C * DP;         // [C][DP]
  float* Vs = Qs + C * DP;         // [C][DP]
  float* Ws = Vs + C * DP;         // [C][DP]   W, later O
  float* Us = Ws + C * DP;         // [C][DP]   U, later Vn
  float* Am = Us + C * DP;         // [C][CP]
  float* Tm = Am + C * CP;         // [C][CP]
  float* Pm = Tm + C * CP;         // [C][CP]
  float* gl = Pm + C * CP;         // [C] raw g
  float* gam = gl + C;             // [C] cumulative
  float* eg = gam + C;             // [C] e^gamma
  float* bet = eg + C;             // [C]

  const int tid = threadIdx.x;
  const int h = blockIdx.x, n = blockIdx.y;
  const int G = p.Hv / p.Hk;
  const int hk = h / G;
  const int bos = clampi(__ldg(p.cu_seqlens + n), 0, p.T);
  const int eos = clampi(__ldg(p.cu_seqlens + n + 1), bos, p.T);
  const TM* __restrict__ qg = static_cast<const TM*>(p.q);
  const TM* __restrict__ kg = static_cast<const TM*>(p.k);
  const TM* __restrict__ vg = static_cast<const TM*>(p.v);
  const size_t sbase = ((size_t)n * p.Hv + h) * D * D;

  for (int idx = tid; idx < D * D; idx += NT) {
    const int r = idx / D, l = idx % D;
    S[r * DP + l] = p.S0 ? p.S0[sbase + idx] : 0.0f;
  }

  for (int c0 = bos; c0 < eos; c0 += C) {
    const int L = min(C, eos - c0);
    __syncthreads();  // previous chunk done with every tile
    for (int idx = tid; idx < C * D; idx += NT) {
      const int i = idx / D, l = idx % D;
      float kv = 0.f, qv = 0.f, vv = 0.f;
      if (i < L) {
        const size_t t = (size_t)(c0 + i);
        kv = ld_f(kg + (t * p.Hk + hk) * D + l);
        qv = ld_f(qg + (t * p.Hk + hk) * D + l);
        vv = ld_f(vg + (t * p.Hv + h) * D + l);
        if (p.k_lo) {  // fp16 q, k plus their rounding residuals
          kv += ld_f(static_cast<const TM*>(p.k_lo) + (t * p.Hk + hk) * D + l);
          qv += ld_f(static_cast<const TM*>(p.q_lo) + (t * p.Hk + hk) * D + l);
        }
      }
      Ks[i * DP + l] = kv; Qs[i * DP + l] = qv; Vs[i * DP + l] = vv;
    }
    for (int i = tid; i < C; i += NT) {
      gl[i] = i < L ? __ldg(p.g + (size_t)h * p.T + c0 + i) : 0.f;
      bet[i] = i < L ? __ldg(p.beta + (size_t)h * p.T + c0 + i) : 0.f;
    }
    __syncthreads();
    if (tid == 0) {
      float run = 0.f;
      for (int i = 0; i < C; ++i) { run += gl[i]; gam[i] = run; }
    }
    __syncthreads();
    for (int i = tid; i < C; i += NT) eg[i] = expf(gam[i]);
    // A (strictly lower) and P = (Q K^T) o decay (lower incl. diagonal)
    for (int idx = tid; idx < C * C; idx += NT) {
      const int i = idx / C, j = idx % C;
      float a = 0.f, pq = 0.f;
      if (i < L && j <= i) {
        float kk = 0.f, qk = 0.f;
        for (int l = 0; l < D; ++l) {
          const float kj = Ks[j * DP + l];
          kk = fmaf(Ks[i * DP + l], kj, kk);
          qk = fmaf(Qs[i * DP + l], kj, qk);
        }
        const float dec = expf(gam[i] - gam[j]);
        if (j < i) a = bet[i] * dec * kk;
        pq = dec * qk;
      }
      Am[i * CP + j] = a;
      Pm[i * CP + j] = pq;
    }
    __syncthreads();
    // T = (I + A)^-1, one column per thread, forward substitution down the column
    if (tid < C) {
      const int m = tid;
      for (int i = 0; i < C; ++i) {
        float val = (i == m) ? 1.f : 0.f;
        for (int j = 0; j < i; ++j) val = fmaf(-Am[i * CP + j], Tm[j * CP + m], val);
        Tm[i * CP + m] = (i < m) ? 0.f : val;
      }
    }
    __syncthreads();
    // W = T diag(beta e^gamma) K ; U = T diag(beta) V
    for (int idx = tid; idx < C * D; idx += NT) {
      const int i = idx / D, l = idx % D;
      float w = 0.f, u = 0.f;
      for (int j = 0; j <= i; ++j) {
        const float tij = Tm[i * CP + j] * bet[j];
        w = fmaf(tij * eg[j], Ks[j * DP + l], w);
        u = fmaf(tij, Vs[j * DP + l], u);
      }
      Ws[i * DP + l] = w;
      Us[i * DP + l] = u;
    }
    __syncthreads();
    // Vn = U - W S^T
    for (int idx = tid; idx < C * D; idx += NT) {
      const int i = idx / D, r = idx % D;
      float acc = Us[i * DP + r];
      for (int l = 0; l < D; ++l) acc = fmaf(-Ws[i * DP + l], S[r * DP + l], acc);
      Us[i * DP + r] = acc;
    }
    __syncthreads();
    // O = diag(e^gamma) Q S^T + P Vn   (into Ws)
    for (int idx = tid; idx < C * D; idx += NT) {
      const int i = idx / D, r = idx % D;
      float qs = 0.f;
      for (int l = 0; l < D; ++l) qs = fmaf(Qs[i * DP + l], S[r * DP + l], qs);
      float acc = eg[i] * qs;
      for (int j = 0; j <= i; ++j) acc = fmaf(Pm[i * CP + j], Us[j * DP + r], acc);
      Ws[i * DP + r] = acc;
    }
    __syncthreads();
    // S <- e^{gamma_L} S + Vn^T diag(e^{gamma_L - gamma}) K
    {
      const float gL = gam[L - 1];
      const float egL = expf(gL);
      for (int idx = tid; idx < D * D; idx += NT) {
        const int r = idx / D, l = idx % D;
        float acc = egL * S[r * DP + l];
        for (int i = 0; i < L; ++i) acc = fmaf(Us[i * DP + r] * expf(gL - gam[i]), Ks[i * DP + l], acc);
        S[r * DP + l] = acc;
      }
    }
    // epilogue: gated RMSNorm (or the raw core output), one warp per token
    {
      const int warp = tid >> 5, lane = tid & 31;
      for (int i = warp; i < L; i += NT / 32) {
        const size_t t = (size_t)(c0 + i);
        const size_t ob = (t * p.Hv + h) * D;
        if (p.out) {
          float ss = 0.f;
          for (int r = lane; r < D; r += 32) { const float o = Ws[i * DP + r]; ss = fmaf(o, o, ss); }
          ss = warp_sum(ss);
          const float inv = rsqrtf(ss / D + p.eps_norm);
          const T* zz = static_cast<const T*>(p.z) + ob;
          const T* ww = static_cast<const T*>(p.norm_w);
          T* oo = static_cast<T*>(p.out) + ob;
          for (int r = lane; r < D; r += 32)
            st_f(oo + r, Ws[i * DP + r] * inv * ld_f(ww + r) * silu_f(ld_f(zz + r)));
        } else {
          for (int r = lane; r < D; r += 32) p.o_raw[ob + r] = Ws[i * DP + r];
        }
      }
    }
  }
  __syncthreads();
  if (p.S_out) {
    for (int idx = tid; idx < D * D; idx += NT) {
      const int r = idx / D, l = idx % D;
      p.S_out[sbase + idx] = S[r * DP + l];
    }
  }
}

template <typename T, typename TM, int D, int C>
cudaError_t launch_one(const ChunkParams& p, cudaStream_t st) {
  const size_t smem = SimtSmem<D, C>::bytes;
  cudaError_t e = cudaFuncSetAttribute(chunk_simt_kernel<T, TM, D, C>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  dim3 grid(p.Hv, p.N);
  chunk_simt_kernel<T, TM, D, C><<<grid, 256, smem, st>>>(p);
  return cudaGetLastError();
}

template <typename T, typename TM, int D>
cudaError_t launch_d(const ChunkParams& p, cudaStream_t st) {
  switch (p.chunk) {
    case 16: return launch_one<T, TM, D, 16>(p, st);
    case 32: return launch_one<T, TM, D, 32>(p, st);
    default: break;
  }
  if constexpr (D <= 64) {
    if (p.chunk == 64) return launch_one<T, TM, D, 64>(p, st);
  }
  return cudaErrorInvalidValue;
}

template <typename T, typename TM>
cudaError_t launch_tm(const ChunkParams& p, int d, cudaStream_t st) {
  if (d == 128) return launch_d<T, TM, 128>(p, st);
  if (d == 64) return launch_d<T, TM, 64>(p, st);
  return launch_d<T, TM, 32>(p, st);
}

}  // namespace

bool chunk_simt_supported(int d, int chunk) {
  if (d == 32 || d == 64) return chunk == 16 || chunk == 32 || chunk == 64;
  if (d == 128) return chunk == 16 || chunk == 32;
  return false;
}

cudaError_t launch_chunk_simt(const ChunkParams& p, int d, gdn_dtype dt_out, gdn_dtype dt_mid,
                              cudaStream_t st) {
  if (p.N == 0 || p.Hv == 0) return cudaSuccess;
  if (dt_out == GDN_BF16) {
    if (dt_mid == GDN_F16) return launch_tm<__nv_bfloat16, __half>(p, d, st);
    if (dt_mid == GDN_BF16) return launch_tm<__nv_bfloat16, __nv_bfloat16>(p, d, st);
    return launch_tm<__nv_bfloat16, float>(p, d, st);
  }
  if (dt_mid == GDN_F16) return launch_tm<float, __half>(p, d, st);
  if (dt_mid == GDN_BF16) return launch_tm<float, __nv_bfloat16>(p, d, st);
  return launch_tm<float, float>(p, d, st);
}

}  // namespace gdn
