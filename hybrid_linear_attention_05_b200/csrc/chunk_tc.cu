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
#include "tc_chunk_common.cuh"
#include "tc_ptx.cuh"

namespace gdn {

__device__ int g_tc_error = 0;  // nonzero: a bounded wait in a kernel gave up

namespace {

using namespace ptx;
using namespace tcc;

constexpr int C = 64;
constexpr int D = 128;
constexpr int NT = 512;   // four warpgroups; each TMEM lane (row) is split by columns between them
constexpr int NW = NT / 32;
constexpr int NWG = NT / 128;
constexpr int CW = 64 / NWG;   // columns of a 64-wide accumulator per warpgroup (16)
constexpr int SW = 128 / NWG;  // columns of the 128-wide state per warpgroup (32)
static_assert(CW == 16 && SW == 32, "column split assumes four warpgroups");

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
constexpr uint32_t OFF_Z = 172032;    // z tile (bf16, two dv halves x 64 tokens x 128 B); then the output tile
constexpr uint32_t OFF_AF = 188416;   // fp32 A [64][AS]; the epilogue reuses AF..TF as O [64][128]
constexpr uint32_t OFF_TF = OFF_AF + 64 * AS * 4;     // fp32 T [64][AS]; before it, the decay table E
constexpr uint32_t OFF_RS = OFF_TF + 64 * AS * 4;     // fp32 scratch of the inverse, 1024 floats
constexpr uint32_t OFF_MISC = OFF_RS + 1024 * 4;      // gamma, e^gamma, beta, rms, e^{gamma_L - gamma}, scan
constexpr uint32_t OFF_BAR = OFF_MISC + 5 * 64 * 4 + 64;
constexpr uint32_t SMEM_USED = OFF_BAR + 80;
constexpr uint32_t SMEM_BYTES = SMEM_USED + 1024;  // + alignment slack
static_assert(OFF_AF + 64 * 128 * 4 <= OFF_RS, "epilogue staging overlaps the scratch");
static_assert(SMEM_BYTES <= 232448, "shared memory");

// TMEM columns (fp32 accumulators, 128 lanes each)
constexpr uint32_t TM_D1 = 0, TM_D2 = 64, TM_D3 = 128, TM_D4 = 192, TM_S = 256, TM_D5 = 384;
constexpr uint32_t TM_COLS = 512;

constexpr uint32_t TILE_BYTES = 64 * 128;           // one 64 x 64 16-bit TMA box
constexpr uint32_t STAGE_TX = 6 * TILE_BYTES;       // K, Q (2 halves each), V (2 halves)

__global__ void __launch_bounds__(NT, 1)
    chunk_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                    const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_z,
                    const __grid_constant__ CUtensorMap tm_ql, const __grid_constant__ CUtensorMap tm_kl,
                    ChunkParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  const uint32_t sb = smem_u32(smem);
  float* Af = reinterpret_cast<float*>(smem + OFF_AF);
  float* Tf = reinterpret_cast<float*>(smem + OFF_TF);
  float* Ef = Tf;  // decay table e^{gamma_i - gamma_j}, [64][ES], alive before the inverse
  float* Xs = reinterpret_cast<float*>(smem + OFF_RS);
  float* Os = reinterpret_cast<float*>(smem + OFF_AF);
  __nv_bfloat16* Zs = reinterpret_cast<__nv_bfloat16*>(smem + OFF_Z);
  float* gam = reinterpret_cast<float*>(smem + OFF_MISC);
  float* eg = gam + 64;
  float* bet = eg + 64;
  float* rms = bet + 64;
  float* decL = rms + 64;
  float* scan = decL + 64;
  // mbarriers: TMA stages 0/1, z tile, and one per tensor-core commit point
  const uint32_t bar_load0 = sb + OFF_BAR, bar_z = sb + OFF_BAR + 16;
  const uint32_t bar_m1 = sb + OFF_BAR + 24, bar_w = sb + OFF_BAR + 32, bar_v = sb + OFF_BAR + 40,
                 bar_o = sb + OFF_BAR + 48;
  const uint32_t bar_lo = sb + OFF_BAR + 56;  // the chunk's [K_lo; Q_lo] tiles
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + OFF_BAR + 64);
  // With the rounding residuals of q and k, D1 also takes [K_lo; Q_lo] K^T and
  // [K; Q] K_lo^T.  Their dk halves (laid out like [K; Q]) land in OFF_TB (the
  // TB and TBE tiles) and OFF_VTS at the top of each chunk: the previous
  // chunk's last MMAs, which read those regions, have completed by then.
  const bool has_lo = p.k_lo != nullptr;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int wg = tid >> 7;     // warpgroup: which column quarter of a TMEM row this thread handles
  const int tl = tid & 127;    // TMEM lane (row) of this thread
  const int h = blockIdx.x, n = blockIdx.y;
  const int hk = h / (p.Hv / p.Hk);
  const int bos = clampi(__ldg(p.cu_seqlens + n), 0, p.T);
  const int eos = clampi(__ldg(p.cu_seqlens + n + 1), bos, p.T);
  const int nchunks = (eos - bos + C - 1) / C;
  const size_t sbase = ((size_t)n * p.Hv + h) * D * D;
  const bool norm_out = p.out != nullptr;

  if (nchunks == 0) {  // empty sequence: the state passes through
    if (p.S_out)
      for (int idx = tid; idx < D * D; idx += NT) p.S_out[sbase + idx] = p.S0 ? p.S0[sbase + idx] : 0.f;
    return;
  }

  if (tid == 0) {
    mbar_init(bar_load0, 1);
    mbar_init(bar_load0 + 8, 1);
    mbar_init(bar_z, 1);
    mbar_init(bar_m1, 1);
    mbar_init(bar_w, 1);
    mbar_init(bar_v, 1);
    mbar_init(bar_o, 1);
    mbar_init(bar_lo, 1);
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
  const uint32_t lane_base = tmem + ((uint32_t)((warp & 3) * 32) << 16);  // this warp's TMEM lanes

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

  // gates are fetched one chunk ahead (threads 0..63, one token each)
  float g_next = 0.f, b_next = 0.f;
  auto load_gates = [&](int cc) {
    const int t0 = bos + cc * C;
    const int Lc = min(C, eos - t0);
    g_next = tid < Lc ? __ldg(p.g + (size_t)h * p.T + t0 + tid) : 0.f;
    b_next = tid < Lc ? __ldg(p.beta + (size_t)h * p.T + t0 + tid) : 0.f;
  };
  if (tid < 64) load_gates(0);
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
    tmem_st32(lane_base + TM_S + col, r);
    tmem_wait_st();
  }

  bool ok = true;
  int c = 0;
  for (; c < nchunks; ++c) {
    const int s = c & 1;
    const int c0 = bos + c * C;
    const int L = min(C, eos - c0);
    const uint32_t kq = sb + (s ? OFF_KQ1 : OFF_KQ0);
    const uint32_t vv = sb + (s ? OFF_V1 : OFF_V0);
    uint8_t* wt_ptr = smem + (s ? OFF_V1 : OFF_V0);  // -W^T reuses the consumed V tile

    if (tid == 0) {
      if (has_lo) {
        mbar_arrive_expect_tx(bar_lo, 4 * TILE_BYTES);
        tma_load_2d(sb + OFF_TB, &tm_kl, hk * D, c0, bar_lo);
        tma_load_2d(sb + OFF_VTS, &tm_kl, hk * D + 64, c0, bar_lo);
        tma_load_2d(sb + OFF_TB + 8192, &tm_ql, hk * D, c0, bar_lo);
        tma_load_2d(sb + OFF_VTS + 8192, &tm_ql, hk * D + 64, c0, bar_lo);
      }
      if (c + 1 < nchunks) issue_loads(c + 1, s ^ 1);
      if (norm_out) {
        mbar_arrive_expect_tx(bar_z, 2 * TILE_BYTES);
        tma_load_2d(sb + OFF_Z, &tm_z, h * D, c0, bar_z);
        tma_load_2d(sb + OFF_Z + TILE_BYTES, &tm_z, h * D + 64, c0, bar_z);
      }
    }

    // ---- gates of the chunk: gamma = cumulative g, e^gamma, beta
    float gv = g_next, bv = b_next;
    if (tid < 64) {
      if (c + 1 < nchunks) load_gates(c + 1);
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
    const uint32_t par = (uint32_t)c & 1u;  // phase parity of the once-per-chunk barriers
    ok = mbar_wait(bar_load0 + 8 * s, (uint32_t)(c >> 1) & 1u);
    if (has_lo) ok = mbar_wait(bar_lo, par) && ok;
    if (__syncthreads_or(!ok)) break;
    if (tid == 0) {
      tc_fence_after();
      constexpr uint32_t id = idesc_f16(128, 64, false, false);
      const uint32_t lo_half[2] = {sb + OFF_TB, sb + OFF_VTS};
#pragma unroll
      for (int kk = 0; kk < 8; ++kk) {
        const uint32_t off = (kk >> 2) * 16384 + (kk & 3) * 32;
        const uint64_t dh = sdesc_sw128(kq + off, 16, 1024);
        mma_f16(tmem + TM_D1, dh, dh, id, kk > 0);
        if (has_lo) {
          const uint64_t lw = sdesc_sw128(lo_half[kk >> 2] + (kk & 3) * 32, 16, 1024);
          mma_f16(tmem + TM_D1, lw, dh, id, 1);
          mma_f16(tmem + TM_D1, dh, lw, id, 1);
        }
      }
      mma_commit(bar_m1);
    }
    // meanwhile: decay table E[i][j] = e^{gamma_i - gamma_j} (j <= i), e^{gamma_L - gamma_i},
    // and the state: fp16 copy for this chunk's products, then S *= e^{gamma_L} in TMEM
    {
#pragma unroll 4
      for (int e = tid; e < 64 * 64; e += NT) {
        const int i = e >> 6, j = e & 63;
        if (j <= i) Ef[i * ES + j] = __expf(gam[i] - gam[j]);
      }
      if (tid < 64) decL[tid] = __expf(gam[L - 1] - gam[tid]);
      const float egL = eg[L - 1];
      uint8_t* half_base = smem + OFF_S + (wg >> 1) * 16384;  // dk half holding columns wg*SW..
      {
        const int col = wg * SW;
        float r[32];
        tmem_ld32(lane_base + TM_S + col, r);
#pragma unroll
        for (int q = 0; q < 4; ++q) st_half8(half_base, swz(tl, (wg & 1) * 4 + q), r + q * 8);
#pragma unroll
        for (int j = 0; j < 32; ++j) r[j] *= egL;
        tmem_st32(lane_base + TM_S + col, r);
      }
      tmem_wait_st();
      fence_proxy_async();
    }
    ok = mbar_wait(bar_m1, par);
    if (__syncthreads_or(!ok)) break;
    tc_fence_after();

    // ---- A (rows 0..63) and P (rows 64..127); this thread: columns wg*CW .. wg*CW+CW-1
    {
      float x[CW];
      tmem_ld16(lane_base + TM_D1 + wg * CW, x);
      if (tl < 64) {
        const int i = tl;
        const float bi = i < L ? bet[i] : 0.f;
#pragma unroll
        for (int e4 = 0; e4 < CW; e4 += 4) {
          float4 v;
          float* vf = reinterpret_cast<float*>(&v);
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            const int j = wg * CW + e4 + u;
            vf[u] = j < i ? bi * Ef[i * ES + j] * x[e4 + u] : 0.f;
          }
          *reinterpret_cast<float4*>(Af + i * AS + wg * CW + e4) = v;
        }
      } else {
        const int i = tl - 64;
        const float keep = i < L ? 1.f : 0.f;
        uint8_t* P = smem + OFF_P;
#pragma unroll
        for (int q = 0; q < CW / 8; ++q) {
          float f[8];
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            const int j = wg * CW + q * 8 + e;
            f[e] = j <= i ? keep * Ef[i * ES + j] * x[q * 8 + e] : 0.f;
          }
          st_half8(P, swz(i, wg * (CW / 8) + q), f);
        }
      }
    }
    __syncthreads();

    // ---- T = (I + A)^-1, then the B operands T diag(beta) and T diag(beta e^gamma)
    solve_unit_lower<NT>(Af, Tf, Xs, tid);
    {
      const int i = tid >> 3, qt = tid & 7;  // row i, 8 columns (one 16-byte chunk) per thread
      uint8_t* Tb = smem + OFF_TB;
      uint8_t* Tbe = smem + OFF_TBE;
      {
        float fb[8], fe[8];
#pragma unroll
        for (int e4 = 0; e4 < 8; e4 += 4) {
          const int j0 = qt * 8 + e4;
          const float4 t4 = *reinterpret_cast<const float4*>(Tf + i * AS + j0);
          const float tv[4] = {t4.x, t4.y, t4.z, t4.w};
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            const float t = tv[u] * bet[j0 + u];
            fb[e4 + u] = t;
            fe[e4 + u] = t * eg[j0 + u];
          }
        }
        st_half8(Tb, swz(i, qt), fb);
        st_half8(Tbe, swz(i, qt), fe);
      }
    }
    fence_proxy_async();
    tc_fence_before();
    __syncthreads();

    // ---- D3 = K^T Tbe^T (= W^T), committed alone; then D2 = V^T Tb^T (= U^T), which the
    //      in-order tensor pipe finishes before the D2 accumulation below
    if (tid == 0) {
      tc_fence_after();
      constexpr uint32_t id = idesc_f16(128, 64, true, false);
#pragma unroll
      for (int kk = 0; kk < 4; ++kk) {
        mma_f16(tmem + TM_D3, sdesc_sw128(kq + kk * 2048, 16384, 1024),
                sdesc_sw128(sb + OFF_TBE + kk * 32, 16, 1024), id, kk > 0);
      }
      mma_commit(bar_w);
#pragma unroll
      for (int kk = 0; kk < 4; ++kk) {
        mma_f16(tmem + TM_D2, sdesc_sw128(vv + kk * 2048, 8192, 1024),
                sdesc_sw128(sb + OFF_TB + kk * 32, 16, 1024), id, kk > 0);
      }
    }
    ok = mbar_wait(bar_w, par);
    if (__syncthreads_or(!ok)) break;
    tc_fence_after();

    // ---- -W^T as the MN-major B operand (row l = tl, tokens wg*CW .. wg*CW+CW-1)
    {
      float x[CW];
      tmem_ld16(lane_base + TM_D3 + wg * CW, x);
#pragma unroll
      for (int j = 0; j < CW; ++j) x[j] = -x[j];
#pragma unroll
      for (int q = 0; q < CW / 8; ++q) st_half8(wt_ptr, swz(tl, wg * (CW / 8) + q), x + q * 8);
    }
    fence_proxy_async();
    tc_fence_before();
    __syncthreads();

    // ---- D2 += S (-W^T)  (= Vn^T), committed alone; then D4 = S Q^T
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
      mma_commit(bar_v);
#pragma unroll
      for (int kk = 0; kk < 8; ++kk) {
        const uint32_t aoff = (kk >> 2) * 16384 + (kk & 3) * 32;
        mma_f16(tmem + TM_D4, sdesc_sw128(sb + OFF_S + aoff, 16, 1024),
                sdesc_sw128(kq + aoff + 8192, 16, 1024), id_q, kk > 0);
      }
    }
    ok = mbar_wait(bar_v, par);
    if (__syncthreads_or(!ok)) break;
    tc_fence_after();

    // ---- Vn^T rows: plain (A of D5) and decayed to the chunk end (A of the state update)
    {
      float x[CW];
      tmem_ld16(lane_base + TM_D2 + wg * CW, x);
      uint8_t* Vt = smem + OFF_TB;
      uint8_t* Vts = smem + OFF_VTS;
#pragma unroll
      for (int q = 0; q < CW / 8; ++q) {
        float f[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          const int i = wg * CW + q * 8 + e;
          f[e] = i < L ? x[q * 8 + e] * decL[i] : 0.f;
        }
        st_half8(Vt, swz(tl, wg * (CW / 8) + q), x + q * 8);
        st_half8(Vts, swz(tl, wg * (CW / 8) + q), f);
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
      mma_commit(bar_o);
    }
    // meanwhile: w * silu(z) for this thread's outputs (column tl, tokens wg*CW .. wg*CW+CW-1)
    float zw[CW];
    if (norm_out) {
      ok = mbar_wait(bar_z, par);
      const __nv_bfloat16* zcol = Zs + (tl >> 6) * (TILE_BYTES / 2) + (tl & 63);
#pragma unroll
      for (int j = 0; j < CW; ++j) zw[j] = w_norm * silu_tanh(__bfloat162float(zcol[(wg * CW + j) * 64]));
    }
    ok = mbar_wait(bar_o, par) && ok;
    if (__syncthreads_or(!ok)) break;
    tc_fence_after();

    // ---- epilogue: O^T = D4 diag(e^gamma) + D5 for tokens wg*CW .. +CW-1, staged as O [token][v]
    float o[CW];
    {
      float a5[CW];
      tmem_ld16(lane_base + TM_D4 + wg * CW, o);
      tmem_ld16(lane_base + TM_D5 + wg * CW, a5);
#pragma unroll
      for (int j = 0; j < CW; ++j) {
        const int i = wg * CW + j;
        o[j] = fmaf(eg[i], o[j], a5[j]);
        Os[i * D + tl] = o[j];
      }
    }
    __syncthreads();
    if (norm_out) {
      // 1 / rms per token: warp w reduces tokens TPW*w .. TPW*w+TPW-1
      constexpr int TPW = 64 / NW;
      float ss[TPW];
#pragma unroll
      for (int t = 0; t < TPW; ++t) {
        const float* row = Os + (TPW * warp + t) * D;
        const float o0 = row[lane], o1 = row[lane + 32], o2 = row[lane + 64], o3 = row[lane + 96];
        ss[t] = o0 * o0 + o1 * o1 + o2 * o2 + o3 * o3;
      }
#pragma unroll
      for (int t = 0; t < TPW; ++t) ss[t] = warp_sum(ss[t]);
#pragma unroll
      for (int t = 0; t < TPW; ++t)
        if (lane == t) rms[TPW * warp + t] = rsqrtf(ss[t] * (1.0f / D) + p.eps_norm);
      __syncthreads();
      // gated output, written over the z tile (each element read, then written, by one thread)
      __nv_bfloat16* zcol = Zs + (tl >> 6) * (TILE_BYTES / 2) + (tl & 63);
#pragma unroll
      for (int j = 0; j < CW; ++j) {
        const int i = wg * CW + j;
        zcol[i * 64] = __float2bfloat16_rn(o[j] * rms[i] * zw[j]);
      }
      fence_proxy_async();  // the next chunk's z tile lands here through TMA
      __syncthreads();
      // rows 0..L-1 of the tile -> out, 16 bytes per thread and pass
      uint8_t* obase = reinterpret_cast<uint8_t*>(p.out) + ((size_t)c0 * p.Hv + h) * D * 2;
      const size_t ostride = (size_t)p.Hv * D * 2;
#pragma unroll
      for (int k = 0; k < 1024 / NT; ++k) {
        const int e = tid + NT * k, row = e >> 4, c16 = e & 15;
        if (row < L) {
          const uint4 val = *reinterpret_cast<const uint4*>(smem + OFF_Z + (c16 >> 3) * TILE_BYTES +
                                                           row * 128 + (c16 & 7) * 16);
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
  }

  if (!ok) {
    // A wait gave up: record it, let the copies this CTA issued land (bounded),
    // release TMEM and leave.
    if (tid == 0) {
      atomicExch(&g_tc_error, 1);
      mbar_wait(bar_load0 + 8 * (c & 1), (uint32_t)(c >> 1) & 1u, 100000000ull);
      if (c + 1 < nchunks)
        mbar_wait(bar_load0 + 8 * ((c + 1) & 1), (uint32_t)((c + 1) >> 1) & 1u, 100000000ull);
      if (norm_out) mbar_wait(bar_z, (uint32_t)c & 1u, 100000000ull);
      if (has_lo) mbar_wait(bar_lo, (uint32_t)c & 1u, 100000000ull);
      mbar_wait(bar_o, (uint32_t)c & 1u, 100000000ull);  // tensor-core work of this chunk
    }
  } else if (p.S_out) {
    float r[32];
    const int col = wg * SW;
    tmem_ld32(lane_base + TM_S + col, r);
#pragma unroll
    for (int j = 0; j < 32; j += 4)
      *reinterpret_cast<float4*>(p.S_out + sbase + (size_t)tl * D + col + j) =
          make_float4(r[j], r[j + 1], r[j + 2], r[j + 3]);
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

}  // namespace

bool chunk_tc_supported(int d, int chunk, gdn_dtype dt_mid) {
  return d == D && chunk == C && dt_mid == GDN_F16;
}

cudaError_t launch_chunk_tc(const ChunkParams& p, cudaStream_t st) {
  if (p.N == 0 || p.Hv == 0) return cudaSuccess;
  CUtensorMap mq, mk, mv, mz, mql, mkl;
  memset(&mq, 0, sizeof(mq));
  memset(&mk, 0, sizeof(mk));
  memset(&mv, 0, sizeof(mv));
  memset(&mz, 0, sizeof(mz));
  memset(&mql, 0, sizeof(mql));
  memset(&mkl, 0, sizeof(mkl));
  if ((p.q_lo == nullptr) != (p.k_lo == nullptr)) return cudaErrorInvalidValue;
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
    if (p.k_lo && (!make_map(&mql, p.q_lo, (uint64_t)p.T, (uint64_t)p.Hk * D, f16, sw) ||
                   !make_map(&mkl, p.k_lo, (uint64_t)p.T, (uint64_t)p.Hk * D, f16, sw)))
      return cudaErrorInvalidValue;
  }
  cudaError_t e = cudaFuncSetAttribute(chunk_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)SMEM_BYTES);
  if (e != cudaSuccess) return e;
  dim3 grid(p.Hv, p.N);
  chunk_tc_kernel<<<grid, NT, SMEM_BYTES, st>>>(mq, mk, mv, mz, mql, mkl, p);
  return cudaGetLastError();
}

}  // namespace gdn

extern "C" gdn_status gdn_device_error(int* code, int clear) {
  if (!code) return GDN_ERR_NULL;
  if (cudaDeviceSynchronize() != cudaSuccess) return GDN_ERR_CUDA;
  int v = 0;
  if (cudaMemcpyFromSymbol(&v, gdn::g_tc_error, sizeof(int)) != cudaSuccess) return GDN_ERR_CUDA;
  if (clear && v != 0) {
    const int zero = 0;
    if (cudaMemcpyToSymbol(gdn::g_tc_error, &zero, sizeof(int)) != cudaSuccess) return GDN_ERR_CUDA;
  }
  const int v2 = gdn::split_error_word(clear);
  if (v2 < 0) return GDN_ERR_CUDA;
  const int v3 = gdn::conv_error_word(clear);
  if (v3 < 0) return GDN_ERR_CUDA;
  const int v4 = gdn::fused_error_word(clear);
  if (v4 < 0) return GDN_ERR_CUDA;
  const int v5 = gdn::linear_error_word(clear);
  if (v5 < 0) return GDN_ERR_CUDA;
  *code = (v | v2 | v3 | v4 | v5) != 0 ? GDN_ERR_TIMEOUT : 0;
  return GDN_OK;
}

namespace gdn {
namespace {
// One warp waits on an mbarrier that nothing arrives at, through the bounded
// wait of the tensor-core kernels, and records that it gave up.
__global__ void selftest_wait_kernel(uint64_t limit_ns) {
  __shared__ __align__(8) uint64_t bar;
  const uint32_t b = ptx::smem_u32(&bar);
  if (threadIdx.x == 0) {
    ptx::mbar_init(b, 1);
    ptx::fence_mbar_init();
  }
  __syncwarp();
  const bool ok = ptx::mbar_wait(b, 0, limit_ns);
  if (!__any_sync(0xffffffffu, ok) && threadIdx.x == 0) atomicExch(&g_tc_error, 1);
}
}  // namespace
}  // namespace gdn

extern "C" gdn_status gdn_selftest_bounded_wait(int limit_us, void* stream) {
  if (limit_us < 1 || limit_us > 1000000) return GDN_ERR_DIMS;
  gdn::selftest_wait_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>((uint64_t)limit_us * 1000ull);
  return cudaGetLastError() == cudaSuccess ? GDN_OK : GDN_ERR_CUDA;
}
