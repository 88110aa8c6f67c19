// Chunked gated delta rule on the tensor cores, as two kernels.
//
// The single-kernel path (chunk_tc.cu) runs everything for one (value head,
// sequence) on one SM, so a batch with few heads x sequences leaves most SMs
// idle, and every chunk pays the key-side work (which does not depend on the
// state) inside the serial state chain.  Here that work moves out:
//
//  1. chunk_keys_kernel, one CTA per (chunk, value head), on every SM:
//       D1 = [K; Q] K^T  ->  A = beta e^{gamma_i-gamma_j} K K^T,  P = (Q K^T) o decay
//       T  = (I + A)^-1                (CUDA cores, fp32)
//       D3 = K^T (T diag(beta e^gamma))^T = W^T
//     and writes one record per (chunk, head): fp16 images of -W^T, of
//     T diag(beta) and of P, laid out exactly as the tensor cores read them
//     from shared memory (128-byte swizzle), plus e^{gamma_i} and
//     e^{gamma_L - gamma_i}.
//  2. chunk_chain_kernel, one CTA per (value head, sequence), walks the
//     chunks with the fp32 state in TMEM.  Each chunk's record arrives in
//     shared memory by one bulk copy, next to the TMA tiles of K, Q, V:
//       D2  = V^T (T diag beta)^T + S (-W^T)   = Vn^T
//       D4  = S Q^T
//       S   = e^{gamma_L} S + (Vn^T diag(e^{gamma_L-gamma})) K
//       D5  = Vn^T P^T
//       O^T = D4 diag(e^gamma) + D5, then the gated RMSNorm per token.
// The algebra is the chunked (WY / UT transform) form of the recurrence, exact
// in real arithmetic ("Qwen (text & vision-language)", Verified parity).
// No TMA multicast is used.
#include <cuda.h>

#include "gdn_internal.h"
#include "tc_chunk_common.cuh"
#include "tc_ptx.cuh"

namespace gdn {

__device__ int g_split_error = 0;  // nonzero: a bounded wait in a kernel of this file gave up

#ifdef GDN_PHASE_TIMING
// Development aid (off by default): SM cycles spent by chain-kernel thread 0
// in each phase of the chunk loop, summed over all CTAs.
__device__ unsigned long long g_split_phase[16];
#define GDN_SPLIT_PHASE(k)                                              \
  do {                                                                  \
    if (tid == 0) {                                                     \
      const long long t_ = clock64();                                   \
      atomicAdd(&g_split_phase[k], (unsigned long long)(t_ - t_prev));  \
      t_prev = t_;                                                      \
    }                                                                   \
  } while (0)
#else
#define GDN_SPLIT_PHASE(k) \
  do {                     \
  } while (0)
#endif

namespace {

using namespace ptx;
using namespace tcc;

constexpr int C = 64;
constexpr int D = 128;
constexpr uint32_t TILE = 64 * 128;  // one 64 x 64 16-bit box

// ---- record written by the key-side kernel for one (chunk, value head)
constexpr uint32_t R_WT = 0;       // -W^T: MN-major B image, 128 rows (dk) x 128 B (64 tokens)
constexpr uint32_t R_TB = 16384;   // T diag(beta): K-major B image, 64 rows (i) x 128 B (j)
constexpr uint32_t R_P = 24576;    // P: K-major B image, 64 rows (i) x 128 B (j)
constexpr uint32_t R_VEC = 32768;  // fp32 e^{gamma_i} [64], then e^{gamma_L - gamma_i} [64]
constexpr uint32_t REC = 33280;

// Record slot of chunk c of sequence n is slot_start(n) + c; slot_start is
// strictly increasing in n and the slots of different chunks never collide.
__device__ __forceinline__ int slot_start(const int32_t* cu, int n, int T) {
  return clampi(__ldg(cu + n), 0, T) / C + n;
}

// ===================================================== key-side kernel
constexpr int NTA = 256;
constexpr uint32_t A_KQ = 0;                     // [K;Q] tile: two dk halves x 128 rows x 128 B
constexpr uint32_t A_TBE = 32768;                // T diag(beta e^gamma), fp16 K-major image
constexpr uint32_t A_AF = 40960;                 // fp32 A [64][AS]
constexpr uint32_t A_TF = A_AF + 64 * AS * 4;    // fp32 T [64][AS]; before it the decay table E
constexpr uint32_t A_X = A_TF + 64 * AS * 4;     // fp32 scratch of the inverse, 1024 floats
constexpr uint32_t A_MISC = A_X + 4096;          // gamma, e^gamma, beta, scan
constexpr uint32_t A_BAR = A_MISC + 3 * 256 + 64;
constexpr uint32_t A_SMEM = A_BAR + 64 + 1024;   // + alignment slack
constexpr uint32_t A_TM_D1 = 0, A_TM_D3 = 64, A_TM_COLS = 128;
static_assert(2 * A_SMEM <= 232448, "two key-side CTAs per SM");

__global__ void __launch_bounds__(NTA, 2)
    chunk_keys_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                      ChunkParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  const uint32_t sb = smem_u32(smem);
  float* Af = reinterpret_cast<float*>(smem + A_AF);
  float* Tf = reinterpret_cast<float*>(smem + A_TF);
  float* Ef = Tf;
  float* Xs = reinterpret_cast<float*>(smem + A_X);
  float* gam = reinterpret_cast<float*>(smem + A_MISC);
  float* eg = gam + 64;
  float* bet = eg + 64;
  float* scan = bet + 64;
  const uint32_t bar_load = sb + A_BAR, bar_m1 = sb + A_BAR + 8, bar_w = sb + A_BAR + 16;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + A_BAR + 24);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int wg = tid >> 7, tl = tid & 127;
  const int g = blockIdx.x, h = blockIdx.y;
  // the sequence whose chunk owns this slot
  int lo = 0, hi = p.N - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (slot_start(p.cu_seqlens, mid, p.T) <= g) lo = mid; else hi = mid - 1;
  }
  const int n = lo;
  const int bos = clampi(__ldg(p.cu_seqlens + n), 0, p.T);
  const int eos = clampi(__ldg(p.cu_seqlens + n + 1), bos, p.T);
  const int c = g - slot_start(p.cu_seqlens, n, p.T);
  if (c < 0 || c >= (eos - bos + C - 1) / C) return;  // slot without a chunk
  const int c0 = bos + c * C;
  const int L = min(C, eos - c0);
  const int hk = h / (p.Hv / p.Hk);
  uint8_t* rec = p.rec + ((size_t)g * p.Hv + h) * REC;

  if (tid == 0) {
    mbar_init(bar_load, 1);
    mbar_init(bar_m1, 1);
    mbar_init(bar_w, 1);
    fence_mbar_init();
  }
  if (warp == 0) {
    tmem_alloc(smem_u32(tmem_slot), A_TM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t lane_base = tmem + ((uint32_t)((warp & 3) * 32) << 16);

  if (tid == 0) {
    mbar_arrive_expect_tx(bar_load, 4 * TILE);
    tma_load_2d(sb + A_KQ, &tm_k, hk * D, c0, bar_load);
    tma_load_2d(sb + A_KQ + 16384, &tm_k, hk * D + 64, c0, bar_load);
    tma_load_2d(sb + A_KQ + 8192, &tm_q, hk * D, c0, bar_load);
    tma_load_2d(sb + A_KQ + 16384 + 8192, &tm_q, hk * D + 64, c0, bar_load);
  }
  // gates of the chunk: gamma = cumulative g, e^gamma, beta
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

  bool ok = mbar_wait(bar_load, 0);
  if (!__syncthreads_or(!ok)) {
    if (tid == 0) {  // D1 = [K; Q] K^T
      tc_fence_after();
      constexpr uint32_t id = idesc_f16(128, 64, false, false);
      const uint64_t dkq = sdesc_sw128(sb + A_KQ, 16, 1024);
#pragma unroll
      for (int kk = 0; kk < 8; ++kk) {
        const uint32_t off = (kk >> 2) * 16384 + (kk & 3) * 32;
        mma_f16(tmem + A_TM_D1, sdesc_add(dkq, off), sdesc_add(dkq, off), id, kk > 0);
      }
      mma_commit(bar_m1);
    }
    // meanwhile: the decay table E[i][j] = e^{gamma_i - gamma_j} (j <= i) and the record's vectors
    for (int e = tid; e < 64 * 64; e += NTA) {
      const int i = e >> 6, j = e & 63;
      if (j <= i) Ef[i * ES + j] = __expf(gam[i] - gam[j]);
    }
    if (tid < 64) {
      float* vec = reinterpret_cast<float*>(rec + R_VEC);
      vec[tid] = eg[tid];
      vec[64 + tid] = __expf(gam[L - 1] - gam[tid]);
    }
    ok = mbar_wait(bar_m1, 0);
  }
  if (!__syncthreads_or(!ok)) {
    tc_fence_after();
    // A (rows 0..63) and P (rows 64..127); this thread: columns wg*32 .. wg*32+31
    {
      float x[32];
      tmem_ld32(lane_base + A_TM_D1 + wg * 32, x);
      if (tl < 64) {
        const int i = tl;
        const float bi = i < L ? bet[i] : 0.f;
#pragma unroll
        for (int e4 = 0; e4 < 32; e4 += 4) {
          float4 v;
          float* vf = reinterpret_cast<float*>(&v);
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            const int j = wg * 32 + e4 + u;
            vf[u] = j < i ? bi * Ef[i * ES + j] * x[e4 + u] : 0.f;
          }
          *reinterpret_cast<float4*>(Af + i * AS + wg * 32 + e4) = v;
        }
      } else {
        const int i = tl - 64;
        const float keep = i < L ? 1.f : 0.f;
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          float f[8];
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            const int j = wg * 32 + q * 8 + e;
            f[e] = j <= i ? keep * Ef[i * ES + j] * x[q * 8 + e] : 0.f;
          }
          st_half8(rec + R_P, swz(i, wg * 4 + q), f);
        }
      }
    }
    __syncthreads();
    solve_unit_lower<NTA>(Af, Tf, Xs, tid);
    // T diag(beta) -> record, T diag(beta e^gamma) -> shared memory (B of W^T)
    {
      const int i = tid >> 2, qt = tid & 3;
#pragma unroll
      for (int q = 0; q < 2; ++q) {
        float fb[8], fe[8];
#pragma unroll
        for (int e4 = 0; e4 < 8; e4 += 4) {
          const int j0 = qt * 16 + q * 8 + e4;
          const float4 t4 = *reinterpret_cast<const float4*>(Tf + i * AS + j0);
          const float tv[4] = {t4.x, t4.y, t4.z, t4.w};
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            const float t = tv[u] * bet[j0 + u];
            fb[e4 + u] = t;
            fe[e4 + u] = t * eg[j0 + u];
          }
        }
        st_half8(rec + R_TB, swz(i, qt * 2 + q), fb);
        st_half8(smem + A_TBE, swz(i, qt * 2 + q), fe);
      }
    }
    fence_proxy_async();
    tc_fence_before();
    __syncthreads();
    if (tid == 0) {  // D3 = K^T Tbe^T = W^T
      tc_fence_after();
      constexpr uint32_t id = idesc_f16(128, 64, true, false);
      const uint64_t dk = sdesc_sw128(sb + A_KQ, 16384, 1024), dt = sdesc_sw128(sb + A_TBE, 16, 1024);
#pragma unroll
      for (int kk = 0; kk < 4; ++kk)
        mma_f16(tmem + A_TM_D3, sdesc_add(dk, kk * 2048), sdesc_add(dt, kk * 32), id, kk > 0);
      mma_commit(bar_w);
    }
    ok = mbar_wait(bar_w, 0);
  }
  if (!__syncthreads_or(!ok)) {
    tc_fence_after();
    // -W^T -> record (row l = tl, tokens wg*32 .. wg*32+31)
    float x[32];
    tmem_ld32(lane_base + A_TM_D3 + wg * 32, x);
#pragma unroll
    for (int j = 0; j < 32; ++j) x[j] = -x[j];
#pragma unroll
    for (int q = 0; q < 4; ++q) st_half8(rec + R_WT, swz(tl, wg * 4 + q), x + q * 8);
  } else if (tid == 0) {
    atomicExch(&g_split_error, 1);
    mbar_wait(bar_load, 0, 100000000ull);
    mbar_wait(bar_w, 0, 100000000ull);
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, A_TM_COLS);
  }
}

// ========================================================= chain kernel
constexpr int NTB = 512;
constexpr int CW = 16;                            // columns of a 64-wide accumulator per warpgroup
constexpr int SW = 32;                            // columns of the state per warpgroup
constexpr uint32_t B_KQ = 0;                      // per stage: [K;Q] tile (32 KiB)
constexpr uint32_t B_V = 32768;                   //            V tile (16 KiB), later Vn^T decayed
constexpr uint32_t B_REC = 49152;                 //            record; its -W^T image later Vn^T
constexpr uint32_t B_STAGE = 83968;               // 82 KiB per stage
constexpr uint32_t B_Z = 2 * B_STAGE;             // z tile, then the output tile
constexpr uint32_t B_S16 = B_Z + 16384;           // fp16 state (K-major A operand, two dk halves)
constexpr uint32_t B_MISC = B_S16 + 32768;        // per-token sum of squares
constexpr uint32_t B_BAR = B_MISC + 512;
constexpr uint32_t B_SMEM = B_BAR + 64 + 1024;
static_assert(B_REC + REC <= B_STAGE, "record fits its stage");
static_assert(B_SMEM <= 232448, "shared memory");
constexpr uint32_t B_TM_S = 0, B_TM_D2 = 128, B_TM_D4 = 192, B_TM_D5 = 256, B_TM_COLS = 512;

__global__ void __launch_bounds__(NTB, 1)
    chunk_chain_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                       const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_z,
                       ChunkParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  const uint32_t sb = smem_u32(smem);
  __nv_bfloat16* Zs = reinterpret_cast<__nv_bfloat16*>(smem + B_Z);
  float* ss = reinterpret_cast<float*>(smem + B_MISC);
  const uint32_t bar_load0 = sb + B_BAR, bar_z = sb + B_BAR + 16, bar_v = sb + B_BAR + 24,
                 bar_o = sb + B_BAR + 32;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + B_BAR + 40);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int wg = tid >> 7, tl = tid & 127;
  const int h = blockIdx.x, n = blockIdx.y;
  const int hk = h / (p.Hv / p.Hk);
  const int bos = clampi(__ldg(p.cu_seqlens + n), 0, p.T);
  const int eos = clampi(__ldg(p.cu_seqlens + n + 1), bos, p.T);
  const int nchunks = (eos - bos + C - 1) / C;
  const size_t sbase = ((size_t)n * p.Hv + h) * D * D;
  const bool norm_out = p.out != nullptr;

  if (nchunks == 0) {  // empty sequence: the state passes through
    if (p.S_out)
      for (int idx = tid; idx < D * D; idx += NTB) p.S_out[sbase + idx] = p.S0 ? p.S0[sbase + idx] : 0.f;
    return;
  }
  const int slot0 = slot_start(p.cu_seqlens, n, p.T);

  if (tid == 0) {
    mbar_init(bar_load0, 1);
    mbar_init(bar_load0 + 8, 1);
    mbar_init(bar_z, 1);
    mbar_init(bar_v, 1);
    mbar_init(bar_o, 1);
    fence_mbar_init();
  }
  if (warp == 0) {
    tmem_alloc(smem_u32(tmem_slot), B_TM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t lane_base = tmem + ((uint32_t)((warp & 3) * 32) << 16);

  auto issue_loads = [&](int cc, int s) {
    const int row = bos + cc * C;
    const uint32_t bar = bar_load0 + 8 * s;
    const uint32_t st = sb + s * B_STAGE;
    mbar_arrive_expect_tx(bar, 6 * TILE + REC);
    tma_load_2d(st + B_KQ, &tm_k, hk * D, row, bar);
    tma_load_2d(st + B_KQ + 16384, &tm_k, hk * D + 64, row, bar);
    tma_load_2d(st + B_KQ + 8192, &tm_q, hk * D, row, bar);
    tma_load_2d(st + B_KQ + 16384 + 8192, &tm_q, hk * D + 64, row, bar);
    tma_load_2d(st + B_V, &tm_v, h * D, row, bar);
    tma_load_2d(st + B_V + 8192, &tm_v, h * D + 64, row, bar);
    bulk_load(st + B_REC, p.rec + ((size_t)(slot0 + cc) * p.Hv + h) * REC, REC, bar);
  };
  constexpr int LOADER = 32;  // one lane of warp 1 issues the copies (thread 0 issues the MMAs)
  if (tid == LOADER) issue_loads(0, 0);
  const float w_norm = norm_out ? __bfloat162float(static_cast<const __nv_bfloat16*>(p.norm_w)[tl]) : 0.f;

  // initial state -> TMEM (row tl, columns wg*SW .. wg*SW+SW-1)
  {
    float r[32];
    const int col = wg * SW;
#pragma unroll
    for (int j = 0; j < 32; j += 4) {
      float4 f = p.S0 ? *reinterpret_cast<const float4*>(p.S0 + sbase + (size_t)tl * D + col + j)
                      : make_float4(0.f, 0.f, 0.f, 0.f);
      r[j] = f.x; r[j + 1] = f.y; r[j + 2] = f.z; r[j + 3] = f.w;
    }
    tmem_st32(lane_base + B_TM_S + col, r);
    tmem_wait_st();
  }

  bool ok = true;
  int c = 0;
#ifdef GDN_PHASE_TIMING
  long long t_prev = clock64();
#endif
  for (; c < nchunks; ++c) {
    const int s = c & 1;
    const int c0 = bos + c * C;
    const int L = min(C, eos - c0);
    const uint32_t par = (uint32_t)c & 1u;
    const uint32_t st = sb + s * B_STAGE;
    uint8_t* stp = smem + s * B_STAGE;
    const float* vec = reinterpret_cast<const float*>(stp + B_REC + R_VEC);  // e^gamma, decay to end

    if (tid == LOADER) {
      if (c + 1 < nchunks) issue_loads(c + 1, s ^ 1);
      if (norm_out) {
        mbar_arrive_expect_tx(bar_z, 2 * TILE);
        tma_load_2d(sb + B_Z, &tm_z, h * D, c0, bar_z);
        tma_load_2d(sb + B_Z + TILE, &tm_z, h * D + 64, c0, bar_z);
      }
    }
    if (tid < 64) ss[tid] = 0.f;
    ok = mbar_wait(bar_load0 + 8 * s, (uint32_t)(c >> 1) & 1u);
    if (__syncthreads_or(!ok)) break;
    GDN_SPLIT_PHASE(0);

    // D2 = V^T (T diag beta)^T  (= U^T); needs no state
    if (tid == 0) {
      tc_fence_after();
      constexpr uint32_t id = idesc_f16(128, 64, true, false);
      const uint64_t dv = sdesc_sw128(st + B_V, 8192, 1024), dt = sdesc_sw128(st + B_REC + R_TB, 16, 1024);
#pragma unroll
      for (int kk = 0; kk < 4; ++kk)
        mma_f16(tmem + B_TM_D2, sdesc_add(dv, kk * 2048), sdesc_add(dt, kk * 32), id, kk > 0);
    }
    // meanwhile: state -> fp16 operand, then S *= e^{gamma_L} in TMEM
    {
      const float egL = vec[L - 1];
      uint8_t* half_base = smem + B_S16 + (wg >> 1) * 16384;
      const int col = wg * SW;
      float r[32];
      tmem_ld32(lane_base + B_TM_S + col, r);
#pragma unroll
      for (int q = 0; q < 4; ++q) st_half8(half_base, swz(tl, (wg & 1) * 4 + q), r + q * 8);
#pragma unroll
      for (int j = 0; j < 32; ++j) r[j] *= egL;
      tmem_st32(lane_base + B_TM_S + col, r);
      tmem_wait_st();
    }
    fence_proxy_async();
    tc_fence_before();
    __syncthreads();

    // D2 += S (-W^T)  (= Vn^T), committed alone; then D4 = S Q^T
    GDN_SPLIT_PHASE(1);
    if (tid == 0) {
      tc_fence_after();
      constexpr uint32_t id_w = idesc_f16(128, 64, false, true);
      constexpr uint32_t id_q = idesc_f16(128, 64, false, false);
      const uint64_t ds = sdesc_sw128(sb + B_S16, 16, 1024);
      const uint64_t dw = sdesc_sw128(st + B_REC + R_WT, 16384, 1024);
      const uint64_t dq = sdesc_sw128(st + B_KQ + 8192, 16, 1024);
#pragma unroll
      for (int kk = 0; kk < 8; ++kk) {
        const uint32_t aoff = (kk >> 2) * 16384 + (kk & 3) * 32;
        mma_f16(tmem + B_TM_D2, sdesc_add(ds, aoff), sdesc_add(dw, kk * 2048), id_w, 1);
      }
      mma_commit(bar_v);
#pragma unroll
      for (int kk = 0; kk < 8; ++kk) {
        const uint32_t aoff = (kk >> 2) * 16384 + (kk & 3) * 32;
        mma_f16(tmem + B_TM_D4, sdesc_add(ds, aoff), sdesc_add(dq, aoff), id_q, kk > 0);
      }
    }
    ok = mbar_wait(bar_v, par);
    if (__syncthreads_or(!ok)) break;
    tc_fence_after();
    GDN_SPLIT_PHASE(2);

    // Vn^T rows: plain (A of D5, over the consumed -W^T image) and decayed to the chunk end
    // (A of the state update, over the consumed V tile)
    {
      float x[CW];
      tmem_ld16(lane_base + B_TM_D2 + wg * CW, x);
#pragma unroll
      for (int q = 0; q < CW / 8; ++q) {
        float f[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          const int i = wg * CW + q * 8 + e;
          f[e] = i < L ? x[q * 8 + e] * vec[64 + i] : 0.f;
        }
        st_half8(stp + B_REC + R_WT, swz(tl, wg * (CW / 8) + q), x + q * 8);
        st_half8(stp + B_V, swz(tl, wg * (CW / 8) + q), f);
      }
    }
    fence_proxy_async();
    tc_fence_before();
    __syncthreads();

    // S += Vts K,  D5 = Vn^T P^T
    GDN_SPLIT_PHASE(3);
    if (tid == 0) {
      tc_fence_after();
      constexpr uint32_t id_s = idesc_f16(128, 128, false, true);
      constexpr uint32_t id_p = idesc_f16(128, 64, false, false);
      const uint64_t dvs = sdesc_sw128(st + B_V, 16, 1024), dk = sdesc_sw128(st + B_KQ, 16384, 1024);
      const uint64_t dvt = sdesc_sw128(st + B_REC + R_WT, 16, 1024), dp = sdesc_sw128(st + B_REC + R_P, 16, 1024);
#pragma unroll
      for (int kk = 0; kk < 4; ++kk)
        mma_f16(tmem + B_TM_S, sdesc_add(dvs, kk * 32), sdesc_add(dk, kk * 2048), id_s, 1);
#pragma unroll
      for (int kk = 0; kk < 4; ++kk)
        mma_f16(tmem + B_TM_D5, sdesc_add(dvt, kk * 32), sdesc_add(dp, kk * 32), id_p, kk > 0);
      mma_commit(bar_o);
    }
    // meanwhile: w * silu(z) for this thread's outputs (column tl, tokens wg*CW ..)
    float zw[CW];
    if (norm_out) {
      ok = mbar_wait(bar_z, par);
      const __nv_bfloat16* zcol = Zs + (tl >> 6) * (TILE / 2) + (tl & 63);
#pragma unroll
      for (int j = 0; j < CW; ++j) zw[j] = w_norm * silu_tanh(__bfloat162float(zcol[(wg * CW + j) * 64]));
    }
    ok = mbar_wait(bar_o, par) && ok;
    if (__syncthreads_or(!ok)) break;
    tc_fence_after();
    GDN_SPLIT_PHASE(4);

    // epilogue: O^T = D4 diag(e^gamma) + D5 for tokens wg*CW .. wg*CW+CW-1
    float o[CW];
    {
      float a5[CW];
      tmem_ld16(lane_base + B_TM_D4 + wg * CW, o);
      tmem_ld16(lane_base + B_TM_D5 + wg * CW, a5);
#pragma unroll
      for (int j = 0; j < CW; ++j) o[j] = fmaf(vec[wg * CW + j], o[j], a5[j]);
    }
    if (norm_out) {
      // sum over v of o^2 per token: each lane holds one v; fold the 16 token
      // values across the warp's 32 lanes, then one shared atomic per token
      float a[CW];
#pragma unroll
      for (int j = 0; j < CW; ++j) a[j] = o[j] * o[j];
#pragma unroll
      for (int off = 16, cnt = CW; off >= 2; off >>= 1, cnt >>= 1) {
        const bool upper = (lane & off) != 0;
#pragma unroll
        for (int i = 0; i < cnt / 2; ++i) {
          const float send = upper ? a[i] : a[i + cnt / 2];
          const float keep = upper ? a[i + cnt / 2] : a[i];
          a[i] = keep + __shfl_xor_sync(0xffffffffu, send, off);
        }
      }
      a[0] += __shfl_xor_sync(0xffffffffu, a[0], 1);
      const int t = ((lane >> 4) & 1) * 8 + ((lane >> 3) & 1) * 4 + ((lane >> 2) & 1) * 2 + ((lane >> 1) & 1);
      if ((lane & 1) == 0) atomicAdd(&ss[wg * CW + t], a[0]);
      __syncthreads();
      if (tid < 64) ss[tid] = rsqrtf(ss[tid] * (1.0f / D) + p.eps_norm);  // now 1 / rms
      __syncthreads();
    GDN_SPLIT_PHASE(5);
      // gated output, written over the z tile (each element read, then written, by one thread)
      __nv_bfloat16* zcol = Zs + (tl >> 6) * (TILE / 2) + (tl & 63);
#pragma unroll
      for (int j = 0; j < CW; ++j) {
        const int i = wg * CW + j;
        zcol[i * 64] = __float2bfloat16_rn(o[j] * ss[i] * zw[j]);
      }
      fence_proxy_async();  // the next chunk's z tile lands here through TMA
      __syncthreads();
      uint8_t* obase = reinterpret_cast<uint8_t*>(p.out) + ((size_t)c0 * p.Hv + h) * D * 2;
      const size_t ostride = (size_t)p.Hv * D * 2;
#pragma unroll
      for (int k = 0; k < 1024 / NTB; ++k) {
        const int e = tid + NTB * k, row = e >> 4, c16 = e & 15;
        if (row < L) {
          const uint4 val = *reinterpret_cast<const uint4*>(smem + B_Z + (c16 >> 3) * TILE + row * 128 +
                                                           (c16 & 7) * 16);
          *reinterpret_cast<uint4*>(obase + row * ostride + c16 * 16) = val;
        }
      }
    } else {
      float* ocol = p.o_raw + ((size_t)c0 * p.Hv + h) * D + tl;
      const size_t ostride = (size_t)p.Hv * D;
#pragma unroll
      for (int j = 0; j < CW; ++j) {
        const int i = wg * CW + j;
        if (i < L) ocol[i * ostride] = o[j];
      }
    }
    __syncthreads();
    GDN_SPLIT_PHASE(6);
  }

  if (!ok) {
    if (tid == 0) {
      atomicExch(&g_split_error, 1);
      mbar_wait(bar_load0 + 8 * (c & 1), (uint32_t)(c >> 1) & 1u, 100000000ull);
      if (c + 1 < nchunks)
        mbar_wait(bar_load0 + 8 * ((c + 1) & 1), (uint32_t)((c + 1) >> 1) & 1u, 100000000ull);
      if (norm_out) mbar_wait(bar_z, (uint32_t)c & 1u, 100000000ull);
      mbar_wait(bar_o, (uint32_t)c & 1u, 100000000ull);
    }
  } else if (p.S_out) {
    float r[32];
    const int col = wg * SW;
    tmem_ld32(lane_base + B_TM_S + col, r);
#pragma unroll
    for (int j = 0; j < 32; j += 4)
      *reinterpret_cast<float4*>(p.S_out + sbase + (size_t)tl * D + col + j) =
          make_float4(r[j], r[j + 1], r[j + 2], r[j + 3]);
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, B_TM_COLS);
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

// Tensor map over a row-major 16-bit [rows, cols] array with 64 x 64 boxes;
// rows past the end read as zeros.
bool make_map(CUtensorMap* m, const void* base, uint64_t rows, uint64_t cols,
              CUtensorMapDataType dt, CUtensorMapSwizzle sw) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {cols, rows};
  cuuint64_t strides[1] = {cols * 2};
  cuuint32_t box[2] = {64, 64};
  cuuint32_t es[2] = {1, 1};
  return fn(m, dt, 2, const_cast<void*>(base), dims, strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE,
            sw, CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

size_t record_slots(int N, int T) { return (size_t)(T / C) + (size_t)N + 1; }

}  // namespace

size_t chunk_tc_split_record_bytes(int N, int T, int Hv) {
  return record_slots(N, T) * (size_t)Hv * REC;
}

cudaError_t launch_chunk_tc_split(const ChunkParams& p, cudaStream_t st) {
  if (p.N == 0 || p.Hv == 0) return cudaSuccess;
  if (!p.rec) return cudaErrorInvalidValue;
  CUtensorMap mq, mk, mv, mz;
  memset(&mq, 0, sizeof(mq));
  memset(&mk, 0, sizeof(mk));
  memset(&mv, 0, sizeof(mv));
  memset(&mz, 0, sizeof(mz));
  if (p.T > 0) {
    const CUtensorMapDataType f16 = CU_TENSOR_MAP_DATA_TYPE_FLOAT16;
    const CUtensorMapSwizzle sw = CU_TENSOR_MAP_SWIZZLE_128B;
    if (!make_map(&mq, p.q, (uint64_t)p.T, (uint64_t)p.Hk * D, f16, sw) ||
        !make_map(&mk, p.k, (uint64_t)p.T, (uint64_t)p.Hk * D, f16, sw) ||
        !make_map(&mv, p.v, (uint64_t)p.T, (uint64_t)p.Hv * D, f16, sw))
      return cudaErrorInvalidValue;
    if (p.out && !make_map(&mz, p.z, (uint64_t)p.T, (uint64_t)p.Hv * D,
                           CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, CU_TENSOR_MAP_SWIZZLE_NONE))
      return cudaErrorInvalidValue;
    cudaError_t e = cudaFuncSetAttribute(chunk_keys_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)A_SMEM);
    if (e != cudaSuccess) return e;
    dim3 ga((unsigned)record_slots(p.N, p.T), p.Hv);
    chunk_keys_kernel<<<ga, NTA, A_SMEM, st>>>(mq, mk, p);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  cudaError_t e = cudaFuncSetAttribute(chunk_chain_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)B_SMEM);
  if (e != cudaSuccess) return e;
  dim3 gb(p.Hv, p.N);
  chunk_chain_kernel<<<gb, NTB, B_SMEM, st>>>(mq, mk, mv, mz, p);
  return cudaGetLastError();
}

#ifdef GDN_PHASE_TIMING
extern "C" int gdn_debug_phase_cycles_split(unsigned long long* out, int clear) {
  cudaDeviceSynchronize();
  if (cudaMemcpyFromSymbol(out, g_split_phase, sizeof(unsigned long long) * 16) != cudaSuccess) return -1;
  if (clear) {
    unsigned long long z[16] = {0};
    cudaMemcpyToSymbol(g_split_phase, z, sizeof(z));
  }
  return 0;
}
#endif

int split_error_word(int clear) {
  int v = 0;
  if (cudaMemcpyFromSymbol(&v, g_split_error, sizeof(int)) != cudaSuccess) return -1;
  if (clear && v != 0) {
    const int zero = 0;
    cudaMemcpyToSymbol(g_split_error, &zero, sizeof(int));
  }
  return v;
}

}  // namespace gdn
