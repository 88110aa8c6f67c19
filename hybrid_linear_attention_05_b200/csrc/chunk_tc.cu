// Chunked gated delta rule on the sm_100a tensor cores (tcgen05 + TMEM + TMA).
//
// One CTA (128 threads, one per TMEM lane) per (value head h, sequence n)
// walks the sequence in chunks of C = 64 tokens; the fp32 state S (dv x dk =
// 128 x 128) lives in TMEM for the whole sequence.  Per chunk, with gamma the
// cumulative log decay inside the chunk, everything is written transposed so
// that every product has M = 128 rows (dv, dk, or the stacked [K; Q] rows):
//
//   D1 = [K; Q] K^T                      (128 x 64)  -> A = beta e^{gamma_i-gamma_j} K K^T
//                                                       P = (Q K^T) o causal decay
//   T  = (I + A)^-1                      CUDA cores, fp32, blocked 16 x 16
//   D2 = V^T (T diag beta)^T             = U^T       (dv x 64)
//   D3 = K^T (T diag(beta e^gamma))^T    = W^T       (dk x 64)
//   D2 += S (-W^T)                       = Vn^T      (new values, dv x 64)
//   D4 = S Q^T                                       (dv x 64)
//   S  = e^{gamma_L} S + (Vn^T diag(e^{gamma_L-gamma})) K     (dv x dk, in TMEM)
//   D5 = Vn^T P^T                                    (dv x 64)
//   O^T = D4 diag(e^gamma) + D5, then the gated RMSNorm over dv per token.
//
// This is the chunked (WY / UT transform) form of the recurrence, exact in
// real arithmetic ("Qwen (text & vision-language)", Verified parity: chunked
// and recurrent Gated DeltaNet agree up to floating-point accumulation).
// Operands are fp16 in 128-byte-swizzled shared memory (TMA for q, k, v;
// CUDA cores for the derived operands), accumulators fp32 in TMEM.  No TMA
// multicast is used.
#include <cuda.h>

#include "gdn_internal.h"
#include "tc_ptx.cuh"

namespace gdn {

__device__ int g_tc_error = 0;  // nonzero: a bounded wait in a kernel gave up

namespace {

using namespace ptx;

constexpr int C = 64;
constexpr int D = 128;
constexpr int NT = 128;

// shared memory layout, byte offsets from a 1024-aligned base
constexpr uint32_t OFF_KQ0 = 0;       // [K;Q] tile, stage 0: two dk halves x 128 rows x 128 B
constexpr uint32_t OFF_KQ1 = 32768;   //                stage 1
constexpr uint32_t OFF_V0 = 65536;    // V tile, stage 0: two dv halves x 64 rows x 128 B; later -W^T
constexpr uint32_t OFF_V1 = 81920;    //          stage 1
constexpr uint32_t OFF_S = 98304;     // S (fp16), K-major A operand: two dk halves x 128 rows
constexpr uint32_t OFF_P = 131072;    // P (fp16), 64 rows x 128 B
constexpr uint32_t OFF_TB = 139264;   // T diag(beta); with OFF_TBE later holds Vn^T (16 KiB)
constexpr uint32_t OFF_TBE = 147456;  // T diag(beta e^gamma)
constexpr uint32_t OFF_VTS = 155648;  // Vn^T diag(e^{gamma_L - gamma}), 128 rows x 128 B
constexpr uint32_t OFF_AF = 172032;   // fp32 A [64][65]; the epilogue reuses AF..TF as O [64][128]
constexpr uint32_t OFF_TF = OFF_AF + 64 * 65 * 4;
constexpr uint32_t OFF_RS = OFF_TF + 64 * 65 * 4;
constexpr uint32_t OFF_MISC = OFF_RS + 3 * 256 * 4;  // gamma, e^gamma, beta, scan scratch
constexpr uint32_t OFF_BAR = OFF_MISC + 3 * 64 * 4 + 64;
constexpr uint32_t SMEM_USED = OFF_BAR + 64;
constexpr uint32_t SMEM_BYTES = SMEM_USED + 1024;  // + alignment slack
static_assert(OFF_AF + 64 * 128 * 4 <= OFF_MISC, "epilogue staging overlaps misc");
static_assert(SMEM_BYTES <= 232448, "shared memory");

// TMEM columns (fp32 accumulators, 128 lanes each)
constexpr uint32_t TM_D1 = 0, TM_D2 = 64, TM_D3 = 128, TM_D4 = 192, TM_S = 256, TM_D5 = 384;
constexpr uint32_t TM_COLS = 512;

constexpr uint32_t TILE_BYTES = 64 * 128;           // one 64 x 64 fp16 TMA box
constexpr uint32_t STAGE_TX = 6 * TILE_BYTES;       // K, Q (2 halves each), V (2 halves)

__device__ __forceinline__ void st_half8(uint8_t* base, uint32_t off, const float* f) {
  uint4 u;
  __half2* h = reinterpret_cast<__half2*>(&u);
#pragma unroll
  for (int i = 0; i < 4; ++i) h[i] = __floats2half2_rn(f[2 * i], f[2 * i + 1]);
  *reinterpret_cast<uint4*>(base + off) = u;
}

// T = (I + A)^-1 for the strictly lower triangular 64 x 64 A (row stride 65).
// Diagonal 16 x 16 blocks by forward substitution (one column per thread),
// then block rows r = 1..3:  T_rc = -T_rr * sum_{k=c}^{r-1} A_rk T_kc.
__device__ __forceinline__ void solve_unit_lower(const float* Af, float* Tf, float* Rs, int tid) {
  if (tid < 64) {
    const int b = tid >> 4, m = tid & 15;
    float x[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      float acc = (i == m) ? 1.f : 0.f;
#pragma unroll
      for (int j = 0; j < i; ++j) acc = fmaf(-Af[(16 * b + i) * 65 + 16 * b + j], x[j], acc);
      x[i] = acc;
    }
#pragma unroll
    for (int i = 0; i < 16; ++i) Tf[(16 * b + i) * 65 + 16 * b + m] = x[i];
  } else {
    // blocks above the diagonal are zero
    for (int e = tid - 64; e < 6 * 256; e += 64) {
      const int blk = e >> 8, w = e & 255, i = w >> 4, m = w & 15;
      const int r = blk < 3 ? 0 : (blk < 5 ? 1 : 2);
      const int c = blk < 3 ? blk + 1 : (blk < 5 ? blk - 1 : 3);
      Tf[(16 * r + i) * 65 + 16 * c + m] = 0.f;
    }
  }
  __syncthreads();
  for (int r = 1; r < 4; ++r) {
    for (int e = tid; e < r * 256; e += NT) {
      const int c = e >> 8, i = (e >> 4) & 15, m = e & 15;
      float acc = 0.f;
      for (int k = c; k < r; ++k) {
#pragma unroll
        for (int j = 0; j < 16; ++j)
          acc = fmaf(Af[(16 * r + i) * 65 + 16 * k + j], Tf[(16 * k + j) * 65 + 16 * c + m], acc);
      }
      Rs[e] = acc;
    }
    __syncthreads();
    for (int e = tid; e < r * 256; e += NT) {
      const int c = e >> 8, i = (e >> 4) & 15, m = e & 15;
      float acc = 0.f;
#pragma unroll
      for (int j = 0; j < 16; ++j)
        acc = fmaf(Tf[(16 * r + i) * 65 + 16 * r + j], Rs[c * 256 + j * 16 + m], acc);
      Tf[(16 * r + i) * 65 + 16 * c + m] = -acc;
    }
    __syncthreads();
  }
}

__global__ void __launch_bounds__(NT, 1)
    chunk_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                    const __grid_constant__ CUtensorMap tm_v, ChunkParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  const uint32_t sb = smem_u32(smem);
  float* Af = reinterpret_cast<float*>(smem + OFF_AF);
  float* Tf = reinterpret_cast<float*>(smem + OFF_TF);
  float* Rs = reinterpret_cast<float*>(smem + OFF_RS);
  float* Os = reinterpret_cast<float*>(smem + OFF_AF);
  float* gam = reinterpret_cast<float*>(smem + OFF_MISC);
  float* eg = gam + 64;
  float* bet = eg + 64;
  float* scan = bet + 64;
  const uint32_t bar_load0 = sb + OFF_BAR, bar_mma = sb + OFF_BAR + 16;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + OFF_BAR + 32);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int h = blockIdx.x, n = blockIdx.y;
  const int hk = h / (p.Hv / p.Hk);
  const int bos = clampi(__ldg(p.cu_seqlens + n), 0, p.T);
  const int eos = clampi(__ldg(p.cu_seqlens + n + 1), bos, p.T);
  const int nchunks = (eos - bos + C - 1) / C;
  const size_t sbase = ((size_t)n * p.Hv + h) * D * D;

  if (nchunks == 0) {  // empty sequence: the state passes through
    if (p.S_out)
      for (int idx = tid; idx < D * D; idx += NT) p.S_out[sbase + idx] = p.S0 ? p.S0[sbase + idx] : 0.f;
    return;
  }

  if (tid == 0) {
    mbar_init(bar_load0, 1);
    mbar_init(bar_load0 + 8, 1);
    mbar_init(bar_mma, 1);
    fence_mbar_init();
  }
  if (warp == 0) {
    tmem_alloc(smem_u32(tmem_slot), TM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t lane_base = tmem + ((uint32_t)(warp * 32) << 16);  // this warp's TMEM lanes

  auto issue_loads = [&](int cc, int s) {
    const int row = bos + cc * C;
    const uint32_t bar = bar_load0 + 8 * s;
    const uint32_t kq = sb + (s ? OFF_KQ1 : OFF_KQ0);
    const uint32_t vv = sb + (s ? OFF_V1 : OFF_V0);
    mbar_arrive_expect_tx(bar, STAGE_TX);
    tma_load_2d(kq, &tm_k, hk * D, row, bar);
    tma_load_2d(kq + 16384, &tm_k, hk * D + 64, row, bar);
    tma_load_2d(kq + 8192, &tm_q, hk * D, row, bar);
    tma_load_2d(kq + 16384 + 8192, &tm_q, hk * D + 64, row, bar);
    tma_load_2d(vv, &tm_v, h * D, row, bar);
    tma_load_2d(vv + 8192, &tm_v, h * D + 64, row, bar);
  };
  if (tid == 0) issue_loads(0, 0);

  // initial state -> TMEM (row v = tid)
  {
    float r[32];
#pragma unroll
    for (int piece = 0; piece < 4; ++piece) {
#pragma unroll
      for (int j = 0; j < 32; j += 4) {
        float4 f = p.S0 ? *reinterpret_cast<const float4*>(p.S0 + sbase + (size_t)tid * D + piece * 32 + j)
                        : make_float4(0.f, 0.f, 0.f, 0.f);
        r[j] = f.x; r[j + 1] = f.y; r[j + 2] = f.z; r[j + 3] = f.w;
      }
      tmem_st32(lane_base + TM_S + piece * 32, r);
    }
    tmem_wait_st();
  }

  uint32_t mma_phase = 0;
  bool ok = true;
  int c = 0;
  for (; c < nchunks; ++c) {
    const int s = c & 1;
    const int c0 = bos + c * C;
    const int L = min(C, eos - c0);
    const uint32_t kq = sb + (s ? OFF_KQ1 : OFF_KQ0);
    const uint32_t vv = sb + (s ? OFF_V1 : OFF_V0);
    uint8_t* wt_ptr = smem + (s ? OFF_V1 : OFF_V0);  // -W^T reuses the consumed V tile

    if (tid == 0 && c + 1 < nchunks) issue_loads(c + 1, s ^ 1);

    // ---- gates of the chunk: gamma = cumulative g, e^gamma, beta
    float gv = 0.f, bv = 0.f;
    if (tid < 64) {
      if (tid < L) {
        gv = __ldg(p.g + (size_t)h * p.T + c0 + tid);
        bv = __ldg(p.beta + (size_t)h * p.T + c0 + tid);
      }
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const float t = __shfl_up_sync(0xffffffffu, gv, o);
        if (lane >= o) gv += t;
      }
      if (tid == 31) scan[0] = gv;
    }
    __syncthreads();
    if (tid < 64) {
      if (tid >= 32) gv += scan[0];
      gam[tid] = gv;
      eg[tid] = __expf(gv);
      bet[tid] = bv;
    }

    // ---- D1 = [K; Q] K^T
    ok = mbar_wait(bar_load0 + 8 * s, (uint32_t)(c >> 1) & 1u);
    if (__syncthreads_or(!ok)) break;
    if (tid == 0) {
      tc_fence_after();
      constexpr uint32_t id = idesc_f16(128, 64, false, false);
#pragma unroll
      for (int kk = 0; kk < 8; ++kk) {
        const uint32_t off = (kk >> 2) * 16384 + (kk & 3) * 32;
        mma_f16(tmem + TM_D1, sdesc_sw128(kq + off, 16, 1024), sdesc_sw128(kq + off, 16, 1024), id,
                kk > 0);
      }
      mma_commit(bar_mma);
    }
    ok = mbar_wait(bar_mma, mma_phase);
    mma_phase ^= 1;
    if (__syncthreads_or(!ok)) break;
    tc_fence_after();

    // ---- A (rows 0..63) and P (rows 64..127)
    {
      float x[64];
      tmem_ld32(lane_base + TM_D1, x);
      tmem_ld32(lane_base + TM_D1 + 32, x + 32);
      if (tid < 64) {
        const int i = tid;
        const float gi = gam[i], bi = bet[i];
#pragma unroll
        for (int j = 0; j < 64; ++j)
          Af[i * 65 + j] = (j < i && i < L) ? bi * __expf(gi - gam[j]) * x[j] : 0.f;
      } else {
        const int i = tid - 64;
        const float gi = gam[i];
        uint8_t* P = smem + OFF_P;
#pragma unroll
        for (int q = 0; q < 8; ++q) {
          float f[8];
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            const int j = q * 8 + e;
            f[e] = (j <= i && i < L) ? __expf(gi - gam[j]) * x[j] : 0.f;
          }
          st_half8(P, swz(i, q), f);
        }
      }
    }
    __syncthreads();

    // ---- T = (I + A)^-1, then the B operands T diag(beta) and T diag(beta e^gamma)
    solve_unit_lower(Af, Tf, Rs, tid);
    {
      const int i = tid >> 1, hf = tid & 1;
      uint8_t* Tb = smem + OFF_TB;
      uint8_t* Tbe = smem + OFF_TBE;
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        float fb[8], fe[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          const int j = hf * 32 + q * 8 + e;
          const float t = Tf[i * 65 + j] * bet[j];
          fb[e] = t;
          fe[e] = t * eg[j];
        }
        st_half8(Tb, swz(i, hf * 4 + q), fb);
        st_half8(Tbe, swz(i, hf * 4 + q), fe);
      }
    }
    fence_proxy_async();
    tc_fence_before();
    __syncthreads();

    // ---- D2 = V^T Tb^T (= U^T), D3 = K^T Tbe^T (= W^T)
    if (tid == 0) {
      tc_fence_after();
      constexpr uint32_t id = idesc_f16(128, 64, true, false);
#pragma unroll
      for (int kk = 0; kk < 4; ++kk) {
        mma_f16(tmem + TM_D2, sdesc_sw128(vv + kk * 2048, 8192, 1024),
                sdesc_sw128(sb + OFF_TB + kk * 32, 16, 1024), id, kk > 0);
      }
#pragma unroll
      for (int kk = 0; kk < 4; ++kk) {
        mma_f16(tmem + TM_D3, sdesc_sw128(kq + kk * 2048, 16384, 1024),
                sdesc_sw128(sb + OFF_TBE + kk * 32, 16, 1024), id, kk > 0);
      }
      mma_commit(bar_mma);
    }

    // ---- meanwhile: S -> fp16 operand, and S *= e^{gamma_L} in TMEM
    {
      const float egL = eg[L - 1];
      uint8_t* Sb = smem + OFF_S;
#pragma unroll
      for (int piece = 0; piece < 4; ++piece) {
        float r[32];
        tmem_ld32(lane_base + TM_S + piece * 32, r);
        uint8_t* half_base = Sb + (piece >> 1) * 16384;
#pragma unroll
        for (int q = 0; q < 4; ++q) st_half8(half_base, swz(tid, (piece & 1) * 4 + q), r + q * 8);
#pragma unroll
        for (int j = 0; j < 32; ++j) r[j] *= egL;
        tmem_st32(lane_base + TM_S + piece * 32, r);
      }
      tmem_wait_st();
    }
    fence_proxy_async();
    ok = mbar_wait(bar_mma, mma_phase);
    mma_phase ^= 1;
    if (__syncthreads_or(!ok)) break;
    tc_fence_after();

    // ---- -W^T as the MN-major B operand (row l = tid, 64 tokens)
    {
      float x[64];
      tmem_ld32(lane_base + TM_D3, x);
      tmem_ld32(lane_base + TM_D3 + 32, x + 32);
#pragma unroll
      for (int j = 0; j < 64; ++j) x[j] = -x[j];
#pragma unroll
      for (int q = 0; q < 8; ++q) st_half8(wt_ptr, swz(tid, q), x + q * 8);
    }
    fence_proxy_async();
    tc_fence_before();
    __syncthreads();

    // ---- D2 += S (-W^T)  (= Vn^T),  D4 = S Q^T
    if (tid == 0) {
      tc_fence_after();
      constexpr uint32_t id_w = idesc_f16(128, 64, false, true);
      constexpr uint32_t id_q = idesc_f16(128, 64, false, false);
      const uint32_t wt = smem_u32(wt_ptr);
#pragma unroll
      for (int kk = 0; kk < 8; ++kk) {
        const uint32_t aoff = (kk >> 2) * 16384 + (kk & 3) * 32;
        mma_f16(tmem + TM_D2, sdesc_sw128(sb + OFF_S + aoff, 16, 1024),
                sdesc_sw128(wt + kk * 2048, 16384, 1024), id_w, 1);
      }
#pragma unroll
      for (int kk = 0; kk < 8; ++kk) {
        const uint32_t aoff = (kk >> 2) * 16384 + (kk & 3) * 32;
        mma_f16(tmem + TM_D4, sdesc_sw128(sb + OFF_S + aoff, 16, 1024),
                sdesc_sw128(kq + aoff + 8192, 16, 1024), id_q, kk > 0);
      }
      mma_commit(bar_mma);
    }
    ok = mbar_wait(bar_mma, mma_phase);
    mma_phase ^= 1;
    if (__syncthreads_or(!ok)) break;
    tc_fence_after();

    // ---- Vn^T rows: plain (A of D5) and decayed to the chunk end (A of the state update)
    {
      float x[64];
      tmem_ld32(lane_base + TM_D2, x);
      tmem_ld32(lane_base + TM_D2 + 32, x + 32);
      const float gL = gam[L - 1];
      uint8_t* Vt = smem + OFF_TB;
      uint8_t* Vts = smem + OFF_VTS;
#pragma unroll
      for (int q = 0; q < 8; ++q) {
        float f[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          const int i = q * 8 + e;
          f[e] = i < L ? x[i] * __expf(gL - gam[i]) : 0.f;
        }
        st_half8(Vt, swz(tid, q), x + q * 8);
        st_half8(Vts, swz(tid, q), f);
      }
    }
    fence_proxy_async();
    tc_fence_before();
    __syncthreads();

    // ---- S += Vts K,  D5 = Vn^T P^T
    if (tid == 0) {
      tc_fence_after();
      constexpr uint32_t id_s = idesc_f16(128, 128, false, true);
      constexpr uint32_t id_p = idesc_f16(128, 64, false, false);
#pragma unroll
      for (int kk = 0; kk < 4; ++kk) {
        mma_f16(tmem + TM_S, sdesc_sw128(sb + OFF_VTS + kk * 32, 16, 1024),
                sdesc_sw128(kq + kk * 2048, 16384, 1024), id_s, 1);
      }
#pragma unroll
      for (int kk = 0; kk < 4; ++kk) {
        mma_f16(tmem + TM_D5, sdesc_sw128(sb + OFF_TB + kk * 32, 16, 1024),
                sdesc_sw128(sb + OFF_P + kk * 32, 16, 1024), id_p, kk > 0);
      }
      mma_commit(bar_mma);
    }
    ok = mbar_wait(bar_mma, mma_phase);
    mma_phase ^= 1;
    if (__syncthreads_or(!ok)) break;
    tc_fence_after();

    // ---- epilogue: O^T = D4 diag(e^gamma) + D5, transposed through shared memory
    {
      float a4[32], a5[32];
#pragma unroll
      for (int half = 0; half < 2; ++half) {
        tmem_ld32(lane_base + TM_D4 + half * 32, a4);
        tmem_ld32(lane_base + TM_D5 + half * 32, a5);
#pragma unroll
        for (int j = 0; j < 32; ++j) {
          const int i = half * 32 + j;
          Os[i * D + tid] = fmaf(eg[i], a4[j], a5[j]);
        }
      }
    }
    __syncthreads();
    for (int i = warp; i < L; i += NT / 32) {
      const size_t ob = ((size_t)(c0 + i) * p.Hv + h) * D;
      float o[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) o[u] = Os[i * D + lane + 32 * u];
      if (p.out) {
        float ss = o[0] * o[0] + o[1] * o[1] + o[2] * o[2] + o[3] * o[3];
        ss = warp_sum(ss);
        const float inv = rsqrtf(ss * (1.0f / D) + p.eps_norm);
        const __nv_bfloat16* zz = static_cast<const __nv_bfloat16*>(p.z) + ob;
        const __nv_bfloat16* ww = static_cast<const __nv_bfloat16*>(p.norm_w);
        __nv_bfloat16* oo = static_cast<__nv_bfloat16*>(p.out) + ob;
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const int v = lane + 32 * u;
          oo[v] = __float2bfloat16_rn(o[u] * inv * __bfloat162float(ww[v]) *
                                      silu_f(__bfloat162float(zz[v])));
        }
      } else {
#pragma unroll
        for (int u = 0; u < 4; ++u) p.o_raw[ob + lane + 32 * u] = o[u];
      }
    }
    __syncthreads();
  }

  if (!ok) {
    // A wait gave up: record it, let the copies this CTA issued land (bounded),
    // release TMEM and leave.
    if (tid == 0) {
      atomicExch(&g_tc_error, 1);
      mbar_wait(bar_load0 + 8 * (c & 1), (uint32_t)(c >> 1) & 1u, 100000000ull);
      if (c + 1 < nchunks) mbar_wait(bar_load0 + 8 * ((c + 1) & 1), (uint32_t)((c + 1) >> 1) & 1u, 100000000ull);
    }
  } else if (p.S_out) {
    float r[32];
#pragma unroll
    for (int piece = 0; piece < 4; ++piece) {
      tmem_ld32(lane_base + TM_S + piece * 32, r);
#pragma unroll
      for (int j = 0; j < 32; j += 4)
        *reinterpret_cast<float4*>(p.S_out + sbase + (size_t)tid * D + piece * 32 + j) =
            make_float4(r[j], r[j + 1], r[j + 2], r[j + 3]);
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, TM_COLS);
  }
}

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  if (!fn) {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(ptr);
  }
  return fn;
}

// Tensor map over a row-major fp16 [rows, cols] array, 64 x 64 boxes,
// 128-byte swizzle; rows past the end read as zeros.
bool make_map(CUtensorMap* m, const void* base, uint64_t rows, uint64_t cols) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {cols, rows};
  cuuint64_t strides[1] = {cols * 2};
  cuuint32_t box[2] = {64, 64};
  cuuint32_t es[2] = {1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, const_cast<void*>(base), dims, strides, box, es,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

bool chunk_tc_supported(int d, int chunk, gdn_dtype dt_mid) {
  return d == D && chunk == C && dt_mid == GDN_F16;
}

cudaError_t launch_chunk_tc(const ChunkParams& p, cudaStream_t st) {
  if (p.N == 0 || p.Hv == 0) return cudaSuccess;
  CUtensorMap mq, mk, mv;
  memset(&mq, 0, sizeof(mq));
  memset(&mk, 0, sizeof(mk));
  memset(&mv, 0, sizeof(mv));
  if (p.T > 0) {
    if (!make_map(&mq, p.q, (uint64_t)p.T, (uint64_t)p.Hk * D) ||
        !make_map(&mk, p.k, (uint64_t)p.T, (uint64_t)p.Hk * D) ||
        !make_map(&mv, p.v, (uint64_t)p.T, (uint64_t)p.Hv * D))
      return cudaErrorInvalidValue;
  }
  cudaError_t e = cudaFuncSetAttribute(chunk_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)SMEM_BYTES);
  if (e != cudaSuccess) return e;
  dim3 grid(p.Hv, p.N);
  chunk_tc_kernel<<<grid, NT, SMEM_BYTES, st>>>(mq, mk, mv, p);
  return cudaGetLastError();
}

}  // namespace gdn

extern "C" gdn_status gdn_device_error(int* code, int clear) {
  if (!code) return GDN_ERR_NULL;
  if (cudaDeviceSynchronize() != cudaSuccess) return GDN_ERR_CUDA;
  int v = 0;
  if (cudaMemcpyFromSymbol(&v, gdn::g_tc_error, sizeof(int)) != cudaSuccess) return GDN_ERR_CUDA;
  *code = v;
  if (clear && v != 0) {
    const int zero = 0;
    if (cudaMemcpyToSymbol(gdn::g_tc_error, &zero, sizeof(int)) != cudaSuccess) return GDN_ERR_CUDA;
  }
  return GDN_OK;
}
