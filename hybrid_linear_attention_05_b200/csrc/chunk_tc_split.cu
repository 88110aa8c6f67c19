// Chunked gated delta rule on the tensor cores, as two kernels.
//
// The single-kernel path (chunk_tc.cu) runs everything for one (value head,
// sequence) on one SM: a batch with few heads x sequences leaves most SMs
// idle, and each chunk pays the key-side work (which does not depend on the
// state) inside the serial state chain.  Here the chain keeps only what needs
// the state.  With Tb = T diag(beta), Tbe = T diag(beta e^gamma), W = Tbe K
// and U = Tb V, the new values and the chunk output are
//     Vn = U - W S0^T,
//     O  = Qt S0^T + Pt V,   Qt = diag(e^gamma) Q - P W,   Pt = P Tb,
// so one M = 128 accumulator [-W; Qt] S0^T plus [U; Pt V] holds both.
//
//  1. chunk_keys_kernel, one unit per (chunk, value head), persistent CTAs:
//       D1 = [K; Q] K^T              ->  A = beta e^{gamma_i-gamma_j} K K^T,  P
//       T  = (I + A)^-1              (CUDA cores, fp32)
//       D2 = [Tb; P] [Tb | Tbe]      ->  Pt = P Tb,  Ph = P Tbe
//       D3 = [Tbe; Ph] K             =   [W; P W],   Qt = E Q - P W in fp32
//                                                  (E = diag(e^gamma))
//       D4 = [Tb; Pt] V              =   [U; Pt V]
//     and writes one record per (chunk, head): fp16 images of [-W; Qt] (the
//     A operand of the chain, 128-byte swizzle) and of [U; Pt V] (swizzled
//     rows, split into 64-column value blocks), then e^{gamma_L - gamma_i}
//     and e^{gamma_L}.
//  2. chunk_chain_kernel walks the chunks of one (value head, sequence) with
//     the fp32 state slice S^T[dk][v] in TMEM.  The value columns are split
//     over a cluster of CL CTAs (each state row evolves on its own); only the
//     gated RMSNorm needs whole rows, and the CTAs swap per-token sums of
//     squares through distributed shared memory.  One thread streams the K
//     tile and the record into a ring of stages.  Per chunk:
//       D   = [-W; Qt] S0^T                      (tensor cores)
//       Vn  = D[0:64] + U,   O = D[64:128] + Pt V
//       S^T = e^{gamma_L} S^T + K^T (diag(e^{gamma_L-gamma}) Vn)
//     Four warpgroups carry the state; a fifth (the output group) takes the
//     O rows of each chunk as soon as its MMAs complete, adds Pt V, swaps
//     per-token sums of squares with the other CTA and writes the gated
//     output from the w * silu(z) tile that the key-side kernel left in the
//     record, while the state moves on to the next chunks.
//  3. Segmented chains (few heads x sequences): one serial chain per (value
//     head, sequence) leaves most SMs idle and takes one chain step per chunk.
//     Each chunk maps the state affinely, S -> S M_c + R_c with
//       M_c = e^{gamma_L} I - W^T diag(e^{gamma_L - gamma}) K,
//       R_c = U^T diag(e^{gamma_L - gamma}) K,
//     so the chunks are cut into segments and chunk_chain_kernel<D, true> runs
//     every segment but the last at once, twice: from S = I with U = 0 (which
//     leaves the segment's M) and from S = 0 (its R).  seg_scan_kernel then
//     walks the segments, S_start(s+1) = S_start(s) M_s + R_s in fp32, and the
//     output chains run all segments at once from their start states.
//  4. State-map mode (gdn_prefill_state_map, for context-parallel prefill):
//     the transfer chains run every segment, both maps of segment 0 too and
//     R from a zero state, and state_fold_kernel composes the segments' maps
//     in order into the map of the whole sequence; no output chain runs.
//     state_fold_kernel also folds gathered maps into a start state
//     (gdn_state_fold).
// The algebra is the chunked (WY / UT transform) form of the recurrence, exact
// in real arithmetic ("Qwen (text & vision-language)", Verified parity).
// No TMA multicast is used.
#include <cuda.h>
#include <math.h>

#include "gdn_internal.h"
#include "host_util.h"
#include "tc_chunk_common.cuh"
#include "tc_ptx.cuh"

namespace gdn {

__device__ int g_split_error = 0;  // nonzero: a bounded wait in a kernel of this file gave up

namespace {

using namespace ptx;
using namespace tcc;

constexpr int C = 64;
constexpr int D = 128;
constexpr uint32_t TILE = 64 * 128;  // one 64 x 64 16-bit box

// ---- record written by the key-side kernel for one (chunk, value head)
constexpr uint32_t R_WQ = 0;       // [-W; Qt]: K-major image, 128 rows x 128 dk (two 16 KiB dk atoms)
constexpr uint32_t R_UO = 32768;   // [U; Pt V]: 128 rows x 128 v as two 16 KiB swizzled value blocks
constexpr uint32_t R_ZW = 65536;   // w * silu(z) in fp16: two 8 KiB value blocks, 64 rows x 128 B, swizzled
constexpr uint32_t R_VEC = 81920;  // fp32 e^{gamma_L - gamma_i} [64] (0 past the chunk), e^{gamma_L}
constexpr uint32_t REC = 82432;

// Record slot of chunk c of sequence n is slot_start(n) + c; slot_start is
// strictly increasing in n and the slots of different chunks never collide.
__device__ __forceinline__ int slot_start(const int32_t* cu, int n, int T) {
  return clampi(__ldg(cu + n), 0, T) / C + n;
}
// First chunk of segment s when nch chunks are cut into P segments.
__device__ __forceinline__ int seg_lo(int nch, int s, int P) { return (int)(((long long)nch * s) / P); }

// ===================================================== key-side kernel
constexpr int NTA = 256;
constexpr uint32_t A_KQ = 0;                     // [K;Q] tile: two dk halves x 128 rows x 128 B
constexpr uint32_t A_TBP = 32768;                // [Tb; P], later [Tb; Pt]: K-major, 128 rows x 64
constexpr uint32_t A_V = 49152;                  // V tile: two 64-column halves x 64 rows
constexpr uint32_t A_AW = 65536;                 // [Tbe; Ph] (16 KiB K atom), then [-W; Qt] (32 KiB)
constexpr uint32_t A_AF = A_AW;                  // fp32 A [64][AS] (dead before A_AW is written)
constexpr uint32_t A_TF = A_AF + 64 * AS * 4;    // fp32 T [64][AS]; before it the decay table E
constexpr uint32_t A_X = A_TF + 64 * AS * 4;     // fp32 scratch of the inverse, 1024 floats
constexpr uint32_t A_MISC = A_X + 4096;          // gamma, e^gamma, beta, scan, norm weights
constexpr uint32_t A_BAR = A_MISC + 3 * 256 + 64 + 512;
constexpr uint32_t A_SMEM = A_BAR + 64 + 1024;   // + alignment slack
constexpr uint32_t A_TM_D1 = 0, A_TM_D3 = 0, A_TM_D2 = 128, A_TM_D4 = 128, A_TM_COLS = 256;
static_assert(A_AW + 32768 <= A_MISC, "AW image inside the dead fp32 scratch");
static_assert(2 * A_SMEM <= 232448, "two key-side CTAs per SM");

// Where a unit (chunk slot g, value head h) of the key-side kernel lies: its
// sequence's chunk c0 .. c0 + L - 1.  Units run heads fastest and chunk slots
// from the last down, so that the records the chains read first are the most
// recently written (in L2).  Returns false for a slot without a chunk.
struct KeyUnit {
  int g, h, c0, L;
};
__device__ __forceinline__ bool key_unit(const ChunkParams& p, int slots, int u, KeyUnit& k) {
  k.h = u % p.Hv;
  k.g = slots - 1 - u / p.Hv;
  int lo = 0, hi = p.N - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (slot_start(p.cu_seqlens, mid, p.T) <= k.g) lo = mid; else hi = mid - 1;
  }
  const int bos = clampi(__ldg(p.cu_seqlens + lo), 0, p.T);
  const int eos = clampi(__ldg(p.cu_seqlens + lo + 1), bos, p.T);
  const int c = k.g - slot_start(p.cu_seqlens, lo, p.T);
  if (c < 0 || c >= (eos - bos + C - 1) / C) return false;
  k.c0 = bos + c * C;
  k.L = min(C, eos - k.c0);
  return true;
}
// The first unit with a chunk at or after u in this CTA's stride (u >= units: none).
__device__ __forceinline__ int next_key_unit(const ChunkParams& p, int slots, int u, KeyUnit& k) {
  const int units = slots * p.Hv;
  for (; u < units; u += (int)gridDim.x)
    if (key_unit(p, slots, u, k)) return u;
  return units;
}

// Persistent: each CTA walks the units u = blockIdx.x + k gridDim.x.  While a
// unit's MMAs run, the next unit's place and gates are looked up, so that
// only its operand copies stand between two units.
__global__ void __launch_bounds__(NTA, 2)
    chunk_keys_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                      const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_ql,
                      const __grid_constant__ CUtensorMap tm_kl, ChunkParams p, int slots) {
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
  float* wsm = scan + 16;  // norm weights, fp32 [128]
  const uint32_t bar_load = sb + A_BAR, bar_m1 = sb + A_BAR + 8, bar_m2 = sb + A_BAR + 16,
                 bar_m3 = sb + A_BAR + 24;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + A_BAR + 32);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int wg = tid >> 7, tl = tid & 127;
  pdl_launch();
  const int units = slots * p.Hv;
  const bool gated = p.z != nullptr;  // w * silu(z) into the record (the gated norm's factor)
  // With the rounding residuals of q and k, D1 also takes [K_lo; Q_lo] K^T
  // and [K; Q] K_lo^T; their tiles ([K_lo; Q_lo] dk halves, laid out like
  // [K; Q]) land in A_TBP and A_AF, which nothing uses before D1 completes.
  const bool has_lo = p.k_lo != nullptr;

  if (tid == 0) {
    mbar_init(bar_load, 1);
    mbar_init(bar_m1, 1);
    mbar_init(bar_m2, 1);
    mbar_init(bar_m3, 1);
    fence_mbar_init();
  }
  if (warp == 0) {
    tmem_alloc(smem_u32(tmem_slot), A_TM_COLS);
    tmem_relinquish();
  }
  if (gated && tid < D) wsm[tid] = __bfloat162float(static_cast<const __nv_bfloat16*>(p.norm_w)[tid]);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t lane_base = tmem + ((uint32_t)((warp & 3) * 32) << 16);
  pdl_wait();  // q, k, v and the gates come from the conv kernel

  KeyUnit cur{}, nxt{};
  int u = next_key_unit(p, slots, (int)blockIdx.x, cur);
  // gates of the unit about to start (thread i < 64: token i of its chunk)
  float gv_n = 0.f, bv_n = 0.f;
  if (u < units && tid < cur.L) {
    gv_n = __ldg(p.g + (size_t)cur.h * p.T + cur.c0 + tid);
    bv_n = __ldg(p.beta + (size_t)cur.h * p.T + cur.c0 + tid);
  }
  // barrier phases completed so far (one per unit each), and what thread 0
  // has started in the current unit (to let it land on a failure)
  uint32_t par = 0;
  bool started_load = false, started_m1 = false, started_m2 = false, started_m3 = false;
  bool failed = false;
  while (u < units) {
    const int h = cur.h, g = cur.g, c0 = cur.c0, L = cur.L;
    const int hk = h / (p.Hv / p.Hk);
    uint8_t* rec = p.rec + ((size_t)g * p.Hv + h) * REC;
    started_load = started_m1 = started_m2 = started_m3 = false;

    // z of the chunk for the gated norm: thread tid takes the 16-byte chunks
    // e = tid + 256 k of the 64 x 128 tile, row e / 16, value chunk e % 16
    uint4 zv[4];
    if (gated) {
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const int e = tid + NTA * k, r = e >> 4, ch = e & 15;
        zv[k] = r < L ? __ldg(reinterpret_cast<const uint4*>(static_cast<const __nv_bfloat16*>(p.z) +
                                                             (size_t)(c0 + r) * p.Hv * D + h * D + ch * 8))
                      : make_uint4(0u, 0u, 0u, 0u);
      }
    }
    if (tid == 0) {
      mbar_arrive_expect_tx(bar_load, (has_lo ? 10 : 6) * TILE);
      tma_load_2d(sb + A_KQ, &tm_k, hk * D, c0, bar_load);
      tma_load_2d(sb + A_KQ + 16384, &tm_k, hk * D + 64, c0, bar_load);
      tma_load_2d(sb + A_KQ + 8192, &tm_q, hk * D, c0, bar_load);
      tma_load_2d(sb + A_KQ + 16384 + 8192, &tm_q, hk * D + 64, c0, bar_load);
      tma_load_2d(sb + A_V, &tm_v, h * D, c0, bar_load);
      tma_load_2d(sb + A_V + TILE, &tm_v, h * D + 64, c0, bar_load);
      if (has_lo) {
        tma_load_2d(sb + A_TBP, &tm_kl, hk * D, c0, bar_load);
        tma_load_2d(sb + A_AF, &tm_kl, hk * D + 64, c0, bar_load);
        tma_load_2d(sb + A_TBP + 8192, &tm_ql, hk * D, c0, bar_load);
        tma_load_2d(sb + A_AF + 8192, &tm_ql, hk * D + 64, c0, bar_load);
      }
      started_load = true;
    }
    // gates of the chunk: gamma = cumulative g, e^gamma, beta (0 past the chunk)
    float gv = gv_n, bv = bv_n;
    if (tid < 64) {
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
    // the next unit's place and gates, while this one's copies and MMAs run
    const int u_next = next_key_unit(p, slots, u + (int)gridDim.x, nxt);
    gv_n = 0.f;
    bv_n = 0.f;
    if (u_next < units && tid < nxt.L) {
      gv_n = __ldg(p.g + (size_t)nxt.h * p.T + nxt.c0 + tid);
      bv_n = __ldg(p.beta + (size_t)nxt.h * p.T + nxt.c0 + tid);
    }

    __syncthreads();
    // while the operands are copied: the decay table E[i][j] = e^{gamma_i -
    // gamma_j} (j <= i; this thread: column j = tid % 64, rows 16 (tid / 64)
    // .. +15), the record's vectors, and w * silu(z) straight into the record
    // in the chain's tile layout (value block ch / 8, row r, swizzled chunk;
    // a warp's stores fill whole 128-byte lines)
    {
      const int j = tid & 63, i0 = (tid >> 6) * 16;
      const float gj = gam[j];
#pragma unroll
      for (int u2 = 0; u2 < 16; ++u2) {
        const int i = i0 + u2;
        if (j <= i) Ef[i * ES + j] = __expf(gam[i] - gj);
      }
    }
    if (tid < 64) {
      float* vec = reinterpret_cast<float*>(rec + R_VEC);
      vec[tid] = tid < L ? __expf(gam[L - 1] - gam[tid]) : 0.f;
      if (tid == 0) vec[64] = eg[L - 1];
    }
    if (gated) {
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const int e = tid + NTA * k, r = e >> 4, ch = e & 15;
        const __nv_bfloat162* z2 = reinterpret_cast<const __nv_bfloat162*>(&zv[k]);
        uint4 res;
        __half2* r2 = reinterpret_cast<__half2*>(&res);
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const float2 zf = __bfloat1622float2(z2[q]);
          r2[q] = __floats2half2_rn(wsm[ch * 8 + 2 * q] * silu_tanh(zf.x), wsm[ch * 8 + 2 * q + 1] * silu_tanh(zf.y));
        }
        *reinterpret_cast<uint4*>(rec + R_ZW + (ch >> 3) * 8192 + swz(r, ch & 7)) = res;
      }
    }

    bool ok = mbar_wait(bar_load, par);
    if (!__syncthreads_or(!ok)) {
      if (tid == 0) {  // D1 = [K; Q] K^T (+ [K_lo; Q_lo] K^T + [K; Q] K_lo^T)
        tc_fence_after();
        constexpr uint32_t id = idesc_f16(128, 64, false, false);
        const uint64_t dkq = sdesc_sw128(sb + A_KQ, 16, 1024);
        const uint64_t dlo[2] = {sdesc_sw128(sb + A_TBP, 16, 1024), sdesc_sw128(sb + A_AF, 16, 1024)};
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const uint32_t off = (kk >> 2) * 16384 + (kk & 3) * 32;
          const uint64_t dh = sdesc_add(dkq, off);
          mma_f16(tmem + A_TM_D1, dh, dh, id, kk > 0);
          if (has_lo) {
            const uint64_t lw = sdesc_add(dlo[kk >> 2], (kk & 3) * 32);
            mma_f16(tmem + A_TM_D1, lw, dh, id, 1);
            mma_f16(tmem + A_TM_D1, dh, lw, id, 1);
          }
        }
        mma_commit(bar_m1);
        started_m1 = true;
      }
      ok = mbar_wait(bar_m1, par);
    }
    if (!__syncthreads_or(!ok)) {
      tc_fence_after();
      // A (rows 0..63) -> fp32; P (rows 64..127) -> fp16 rows 64..127 of [Tb; P].
      // This thread: row tl, columns wg*32 .. wg*32+31.
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
            for (int q = 0; q < 4; ++q) {
              const int j = wg * 32 + e4 + q;
              vf[q] = j < i ? bi * Ef[i * ES + j] * x[e4 + q] : 0.f;
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
            st_half8(smem + A_TBP, swz(tl, wg * 4 + q), f);
          }
        }
      }
      __syncthreads();
      solve_unit_lower<NTA>(Af, Tf, Xs, tid);
      // this thread's 16 entries of T, row i = tid / 4, columns (tid % 4) * 16 ..
      const int i = tid >> 2, qt = tid & 3;
      float tv[16];
#pragma unroll
      for (int e4 = 0; e4 < 16; e4 += 4) {
        const float4 t4 = *reinterpret_cast<const float4*>(Tf + i * AS + qt * 16 + e4);
        tv[e4] = t4.x; tv[e4 + 1] = t4.y; tv[e4 + 2] = t4.z; tv[e4 + 3] = t4.w;
      }
      __syncthreads();  // the fp32 scratch is dead from here: the AW image goes over it
#pragma unroll
      for (int q = 0; q < 2; ++q) {
        float fb[8], fe[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          const int j = qt * 16 + q * 8 + e;
          fb[e] = tv[q * 8 + e] * bet[j];
          fe[e] = fb[e] * eg[j];
        }
        st_half8(smem + A_TBP, swz(i, qt * 2 + q), fb);  // Tb: A rows 0..63 and B block 0 of D2
        st_half8(smem + A_AW, swz(i, qt * 2 + q), fe);   // Tbe: AW rows 0..63 and B block 1 of D2
      }
      fence_proxy_async();
      tc_fence_before();
      __syncthreads();
      if (tid == 0) {  // D2 = [Tb; P] [Tb | Tbe]
        tc_fence_after();
        constexpr uint32_t id = idesc_f16(128, 128, false, true);
        const uint64_t da = sdesc_sw128(sb + A_TBP, 16, 1024);
        const uint64_t db = sdesc_sw128(sb + A_TBP, A_AW - A_TBP, 1024);
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
          mma_f16(tmem + A_TM_D2, sdesc_add(da, kk * 32), sdesc_add(db, kk * 2048), id, kk > 0);
        mma_commit(bar_m2);
        started_m2 = true;
      }
      ok = mbar_wait(bar_m2, par);
    }
    if (!__syncthreads_or(!ok)) {
      tc_fence_after();
      // rows 64..127 of D2: Pt (columns 0..63) over P in [Tb; P], Ph (64..127) -> AW rows 64..127
      if (tl >= 64) {
        float x[32];
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
          tmem_ld32(lane_base + A_TM_D2 + wg * 64 + hh * 32, x);
          uint8_t* dst = smem + (wg == 0 ? A_TBP : A_AW);
#pragma unroll
          for (int q = 0; q < 4; ++q) st_half8(dst, swz(tl, hh * 4 + q), x + q * 8);
        }
      }
      fence_proxy_async();
      tc_fence_before();
      __syncthreads();
      if (tid == 0) {
        tc_fence_after();
        // D3 = [Tbe; Ph] K = [W; P W]  (Qt = E Q - P W is completed at extraction)
        constexpr uint32_t id = idesc_f16(128, 128, false, true);
        const uint64_t da = sdesc_sw128(sb + A_AW, 16, 1024);
        const uint64_t db = sdesc_sw128(sb + A_KQ, 16384, 1024);
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
          mma_f16(tmem + A_TM_D3, sdesc_add(da, kk * 32), sdesc_add(db, kk * 2048), id, kk > 0);
        // D4 = [Tb; Pt] V = [U; Pt V]
        const uint64_t dt = sdesc_sw128(sb + A_TBP, 16, 1024);
        const uint64_t dv = sdesc_sw128(sb + A_V, TILE, 1024);
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
          mma_f16(tmem + A_TM_D4, sdesc_add(dt, kk * 32), sdesc_add(dv, kk * 2048), id, kk > 0);
        mma_commit(bar_m3);
        started_m3 = true;
      }
      ok = mbar_wait(bar_m3, par);
    }
    if (!__syncthreads_or(!ok)) {
      tc_fence_after();
      // The record is assembled in shared memory regions the MMAs no longer
      // read: [-W; Qt] over AW, [U; Pt V] over [K; Q] (w * silu(z) went
      // straight to global memory at the start of the unit).
      // Row tl: [-W; Qt] dk atom wg and [U; Pt V] value block wg.  Each
      // warpgroup's part leaves by bulk copy as soon as that warpgroup has
      // written it (a named barrier per warpgroup), overlapping the rest.
      const bool wg_lead = tl == 0;
      // rows 64.. take e^{gamma_i} q_i (fp32, from the Q rows of [K; Q]; 0 past the chunk)
      const float eq = tl >= 64 && tl - 64 < L ? eg[tl - 64] : 0.f;
      float x[32];
#pragma unroll
      for (int hh = 0; hh < 2; ++hh) {
        tmem_ld32(lane_base + A_TM_D3 + wg * 64 + hh * 32, x);
#pragma unroll
        for (int j = 0; j < 32; ++j) x[j] = -x[j];
        if (tl >= 64) {
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            const uint4 u4 = *reinterpret_cast<const uint4*>(smem + A_KQ + wg * 16384 + swz(tl, hh * 4 + q));
            const __half2* h2 = reinterpret_cast<const __half2*>(&u4);
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const float2 f = __half22float2(h2[e]);
              x[q * 8 + 2 * e] = fmaf(eq, f.x, x[q * 8 + 2 * e]);
              x[q * 8 + 2 * e + 1] = fmaf(eq, f.y, x[q * 8 + 2 * e + 1]);
            }
          }
        }
#pragma unroll
        for (int q = 0; q < 4; ++q) st_half8(smem + A_AW + wg * 16384, swz(tl, hh * 4 + q), x + q * 8);
      }
      fence_proxy_async();
      bar_named(1 + wg, 128);
      if (wg_lead) bulk_store(rec + R_WQ + wg * 16384, sb + A_AW + wg * 16384, 16384);
#pragma unroll
      for (int hh = 0; hh < 2; ++hh) {
        tmem_ld32(lane_base + A_TM_D4 + wg * 64 + hh * 32, x);
#pragma unroll
        for (int q = 0; q < 4; ++q) st_half8(smem + A_KQ + wg * 16384, swz(tl, hh * 4 + q), x + q * 8);
      }
      fence_proxy_async();
      bar_named(1 + wg, 128);
      if (wg_lead) {
        bulk_store(rec + R_UO + wg * 16384, sb + A_KQ + wg * 16384, 16384);
        bulk_commit();
      }
      if (wg_lead) bulk_wait_read();  // shared memory stays valid until the copies have read it
    }
    // End of the unit: its copies have read shared memory and its TMEM has
    // been read; the next unit's copies and MMAs may overwrite both.
    fence_proxy_async();
    tc_fence_before();
    failed = __syncthreads_or(!ok);
    tc_fence_after();
    if (failed) break;
    par ^= 1u;
    u = u_next;
    cur = nxt;
  }
  if (failed && tid == 0) {
    // let every copy and MMA this thread started in the unit land (bounded)
    atomicExch(&g_split_error, 1);
    if (started_load) mbar_wait(bar_load, par, 100000000ull);
    if (started_m1) mbar_wait(bar_m1, par, 100000000ull);
    if (started_m2) mbar_wait(bar_m2, par, 100000000ull);
    if (started_m3) mbar_wait(bar_m3, par, 100000000ull);
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, A_TM_COLS);
  }
}

// ========================================================= chain kernel
// VS value columns per CTA; CL = 128 / VS CTAs (one cluster) per (head, sequence).
template <int VS>
struct ChainCfg {
  static constexpr int CL = D / VS;
  static constexpr int NA = VS / 64;                  // 64-wide value blocks
  static constexpr int CW = VS / 4;                   // state columns per main warpgroup
  static constexpr int NST = VS == 64 ? 3 : 2;        // stages in the ring
  static constexpr uint32_t S_K = 0;                  // per stage: K tile (two dk halves, 16 KiB)
  static constexpr uint32_t S_WQ = 16384;             //   [-W; Qt] (32 KiB)
  static constexpr uint32_t S_UO = 49152;             //   this CTA's blocks of [U; Pt V]
  static constexpr uint32_t S_VEC = S_UO + NA * 16384;
  static constexpr uint32_t STAGE = (S_VEC + 512 + 1023) / 1024 * 1024;
  static constexpr uint32_t S16 = NST * STAGE;        // fp16 S0^T (NA x 16 KiB); then decayed Vn (NA x 8 KiB)
  static constexpr uint32_t ZT = S16 + NA * 16384;    // w * silu(z) of a chunk, then its output (NA x 8 KiB)
  static constexpr uint32_t SSP = ZT + NA * 8192;     // this CTA's per-token half-row sums of squares [2][64]
  static constexpr uint32_t XB = SSP + 512;           // the other CTA's half-row sums [2 buffers][2][64]
  static constexpr uint32_t BAR = XB + 1024;
  static constexpr uint32_t SMEM = BAR + 256 + 1024;
  static constexpr uint32_t TM_S = 0, TM_D = VS;      // state, then two [Vn; O] accumulators
  static constexpr uint32_t TM_COLS = 3 * VS <= 256 ? 256 : 512;
  static_assert(SMEM <= 232448, "shared memory");
};
// Warps 0..15: the state chain (four warpgroups; TMEM lane quarter = warp % 4).
// Warps 16..23: the output group; warps 18, 19, 22 and 23 reach TMEM lanes
// 64..127, where the O rows are: two threads per token row, half the
// columns each.
constexpr int NCW = 512;
constexpr int NOG = 256;
constexpr int NTB = NCW + NOG;
constexpr int BAR_COMPUTE = 1;  // named barrier of the state-chain threads
constexpr int BAR_OG = 2;       // the output group
constexpr int BAR_VN = 3;       // the 256 state-chain threads that own new-value rows

template <int CW>
__device__ __forceinline__ void tmem_ldw(uint32_t taddr, float* v) {
  if constexpr (CW == 16) tmem_ld16(taddr, v); else tmem_ld32(taddr, v);
}
template <int CW>
__device__ __forceinline__ void tmem_stw(uint32_t taddr, const float* v) {
  if constexpr (CW == 16) tmem_st16(taddr, v); else tmem_st32(taddr, v);
}
// x[0..8) += eight fp16 values at base + off
__device__ __forceinline__ void add_half8(const uint8_t* base, uint32_t off, float* x) {
  const uint4 u = *reinterpret_cast<const uint4*>(base + off);
  const __half2* h2 = reinterpret_cast<const __half2*>(&u);
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    const float2 f = __half22float2(h2[e]);
    x[2 * e] += f.x;
    x[2 * e + 1] += f.y;
  }
}

// XFER = false: the output chain of one segment (the whole sequence when
// p.nseg == 1) of one (value head, sequence), CL CTAs over the value columns.
// XFER = true: the affine map of one segment that is not the last, one CTA
// per role: role 0 runs the chain from S = I with U = 0 and leaves M, role 1
// from S = 0 and leaves R; neither writes outputs (no output group).
template <int VS, bool XFER>
__global__ void __launch_bounds__(XFER ? NCW : NTB, 1)
    chunk_chain_kernel(const __grid_constant__ CUtensorMap tm_k, ChunkParams p) {
  using G = ChainCfg<VS>;
  constexpr int CL = G::CL, NA = G::NA, CW = G::CW, NST = G::NST;
  static_assert(!XFER || CL == 1, "a transfer chain owns whole state rows");
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  const uint32_t sb = smem_u32(smem);
  float* xb = reinterpret_cast<float*>(smem + G::XB);
  float* ssp = reinterpret_cast<float*>(smem + G::SSP);
  // bar_a[b], bar_s[b], bar_x[b], bar_dfree[b] follow accumulator buffer b = chunk & 1: the state
  // chain cannot finish chunk c + 2 in buffer b before the output group released
  // chunk c, so nobody waits on these barriers more than one phase late
  const uint32_t bar_full = sb + G::BAR, bar_free = bar_full + 8 * NST, bar_a = bar_free + 8 * NST,
                 bar_s = bar_a + 16, bar_x = bar_s + 16, bar_dfree = bar_x + 16;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + G::BAR + 8 * (2 * NST + 8));

  const int tid = threadIdx.x, warp = tid >> 5;
  const int wg = tid >> 7, tl = tid & 127;
  pdl_launch();
  const int P = p.nseg;
  const int h = XFER ? (int)blockIdx.x >> 1 : (int)blockIdx.x / CL;
  const int vs = XFER ? 0 : (int)blockIdx.x % CL;
  const int role = XFER ? (int)blockIdx.x & 1 : 1;  // 0: the map M (from S = I, U = 0)
  // transfer chains: the maps of segments 0 .. P-2, or of all P in state-map mode
  const bool map_all = XFER && p.map_out != nullptr;
  const int NM = XFER ? (map_all ? P : P - 1) : P;
  const int n = (int)blockIdx.y / NM;
  const int sg = (int)blockIdx.y % NM;
  const int hk = h / (p.Hv / p.Hk);
  const int bos0 = clampi(__ldg(p.cu_seqlens + n), 0, p.T);
  const int eos = clampi(__ldg(p.cu_seqlens + n + 1), bos0, p.T);
  const int nch_all = (eos - bos0 + C - 1) / C;
  const int cb = seg_lo(nch_all, sg, P);
  const int nchunks = seg_lo(nch_all, sg + 1, P) - cb;  // chunks of this segment
  const int bos = bos0 + cb * C;                          // its first token
  const size_t hd = (size_t)D * D;
  const size_t slice = (size_t)vs * VS * D;  // first state row of this CTA's slice
  const size_t nh = (size_t)n * p.Hv + h;
  // the state this CTA starts from (null: zero; transfer chains build theirs)
  // and where its last state goes (null: nowhere)
  // (the R chain of segment 0 starts from S0 itself, so it leaves the state
  // at the start of segment 1 and segment 0 needs no map M)
  auto start_state = [&]() -> const float* {
    if (XFER) return sg == 0 && p.S0 && !map_all ? p.S0 + nh * hd + slice : nullptr;
    if (P == 1) return p.S0 ? p.S0 + nh * hd + slice : nullptr;
    return p.seg_start + (((size_t)n * P + sg) * p.Hv + h) * hd + slice;
  };
  auto final_state = [&]() -> float* {
    if (XFER) return p.seg_mr + ((((size_t)n * NM + sg) * p.Hv + h) * 2 + role) * hd;
    return sg == P - 1 && p.S_out ? p.S_out + nh * hd + slice : nullptr;
  };
  const bool norm_out = !XFER && p.out != nullptr;
  const bool want_u = !XFER || role == 1;  // the chain adds U to its new values

  if (XFER && sg == 0 && role == 0 && !map_all) return;  // segment 0's map M is not needed
  if (nchunks == 0) {
    // empty segment; the last one is empty only for an empty sequence, whose
    // state passes through (every CTA of the cluster returns here).  In
    // state-map mode an empty segment's map is the identity: M = I, R = 0.
    pdl_wait();
    const float* Sin = start_state();
    float* Sfin = final_state();
    if (!XFER && Sfin)
      for (int idx = tid; idx < VS * D; idx += NTB) Sfin[idx] = Sin ? Sin[idx] : 0.f;
    if (map_all)
      for (int idx = tid; idx < D * D; idx += NCW) Sfin[idx] = role == 0 && idx / D == idx % D ? 1.f : 0.f;
    return;
  }
  const int slot0 = slot_start(p.cu_seqlens, n, p.T) + cb;

  if (tid == 0) {
    for (int k = 0; k < NST; ++k) {
      mbar_init(bar_full + 8 * k, 1);
      mbar_init(bar_free + 8 * k, XFER ? 1 : 1 + 128);  // the state-update MMAs (and the 128 O-row threads)
    }
    mbar_init(bar_a, 1);
    mbar_init(bar_a + 8, 1);
    mbar_init(bar_s, 1);
    mbar_init(bar_s + 8, 1);
    mbar_init(bar_x, 1);
    mbar_init(bar_x + 8, 1);
    mbar_init(bar_dfree, 128);
    mbar_init(bar_dfree + 8, 128);
    fence_mbar_init();
  }
  if (warp == 0) {
    tmem_alloc(smem_u32(tmem_slot), G::TM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  if constexpr (CL > 1) cluster_sync();  // the other CTA's barriers exist before anyone arrives on them
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t lane_base = tmem + ((uint32_t)((warp & 3) * 32) << 16);
  pdl_wait();  // the records, k and the start states come from the kernels before

  // thread LOADER streams K and the records: chunks 0 .. NST-1 up front, then
  // chunk c - 1 + NST once chunk c - 1 has released its stage
  constexpr int LOADER = 32;
  auto issue_loads = [&](int cc) {
    const int s = cc % NST;
    const int row = bos + cc * C;
    const uint32_t bar = bar_full + 8 * s, st = sb + s * G::STAGE;
    const uint8_t* rec = p.rec + ((size_t)(slot0 + cc) * p.Hv + h) * REC;
    if constexpr (XFER) {
      // only the -W rows (the first 64 of each dk atom) and the U rows (the
      // first 64 of each value block); the MMA rows they leave stale are never read
      mbar_arrive_expect_tx(bar, 2 * TILE + 16384 + (want_u ? 16384 : 0) + 512);
      tma_load_2d(st + G::S_K, &tm_k, hk * D, row, bar);
      tma_load_2d(st + G::S_K + TILE, &tm_k, hk * D + 64, row, bar);
      bulk_load(st + G::S_WQ, rec + R_WQ, 8192, bar);
      bulk_load(st + G::S_WQ + 16384, rec + R_WQ + 16384, 8192, bar);
      if (want_u) {
        bulk_load(st + G::S_UO, rec + R_UO, 8192, bar);
        bulk_load(st + G::S_UO + 16384, rec + R_UO + 16384, 8192, bar);
      }
      bulk_load(st + G::S_VEC, rec + R_VEC, 512, bar);
    } else {
      mbar_arrive_expect_tx(bar, 2 * TILE + 32768 + NA * 16384 + 512);
      tma_load_2d(st + G::S_K, &tm_k, hk * D, row, bar);
      tma_load_2d(st + G::S_K + TILE, &tm_k, hk * D + 64, row, bar);
      bulk_load(st + G::S_WQ, rec + R_WQ, 32768, bar);
      bulk_load(st + G::S_UO, rec + R_UO + vs * NA * 16384, NA * 16384, bar);
      bulk_load(st + G::S_VEC, rec + R_VEC, 512, bar);
    }
  };
  if (tid == LOADER)
    for (int cc = 0; cc < NST && cc < nchunks; ++cc) issue_loads(cc);

  if (XFER || warp < NCW / 32) {
    // ============================================ state chain (warps 0..15)
    const int col = wg * CW;                            // this thread's state columns in the slice
    const uint32_t blk = (uint32_t)(col >> 6) * 16384;  // their 64-column block in S16 / [U; Pt V]
    const int ch0 = (col & 63) >> 3;                    // their first 16-byte chunk in a block row
    {  // initial state: S^T[dk = tl][v] = S_start[v][dk]; I for the map M
      const float* Sin = start_state();
      float r[CW];
#pragma unroll
      for (int j = 0; j < CW; ++j)
        r[j] = XFER && role == 0 ? (col + j == tl ? 1.f : 0.f) : (Sin ? Sin[(size_t)(col + j) * D + tl] : 0.f);
      tmem_stw<CW>(lane_base + G::TM_S + col, r);
      tmem_wait_st();
    }
    bool ok = true, bad = false;
    int c = 0;
    for (; c < nchunks; ++c) {
      const int s = c % NST, b = c & 1;
      uint8_t* stp = smem + s * G::STAGE;
      const uint32_t st = sb + s * G::STAGE;
      const float* vec = reinterpret_cast<const float*>(stp + G::S_VEC);
      ok = mbar_wait(bar_full + 8 * s, (uint32_t)(c / NST) & 1u) && ok;
      if (c > 0) ok = mbar_wait(bar_s + 8 * (b ^ 1), (uint32_t)((c - 1) >> 1) & 1u) && ok;
      tc_fence_after();
      // the stage of chunk c - 1 is free once its output rows have also read it:
      // refill it now if they have, else after the barrier below
      bool loads_due = tid == LOADER && c >= 1 && c - 1 + NST < nchunks;
      if (loads_due && mbar_try_wait(bar_free + 8 * ((c - 1) % NST), (uint32_t)((c - 1) / NST) & 1u)) {
        issue_loads(c - 1 + NST);
        loads_due = false;
      }
      {  // state -> fp16 operand, then S *= e^{gamma_L} in TMEM
        const float egL = vec[64];
        float r[CW];
        tmem_ldw<CW>(lane_base + G::TM_S + col, r);
#pragma unroll
        for (int q = 0; q < CW / 8; ++q) st_half8(smem + G::S16 + blk, swz(tl, ch0 + q), r + q * 8);
#pragma unroll
        for (int j = 0; j < CW; ++j) r[j] *= egL;
        tmem_stw<CW>(lane_base + G::TM_S + col, r);
        tmem_wait_st();
      }
      fence_proxy_async();
      tc_fence_before();
      if (bar_named_or(BAR_COMPUTE, NCW, !ok)) { bad = true; break; }
      if (loads_due) {
        // the state MMAs of chunk c-1 are done; its O rows were read right after them
        const int cc = c - 1 + NST;
        if (mbar_wait(bar_free + 8 * (cc % NST), (uint32_t)(cc / NST - 1) & 1u))
          issue_loads(cc);
        else
          ok = false;
      }
      if (warp == 0) {  // D = [-W; Qt] S0^T (descriptors warp-uniform, one lane issues)
        tc_fence_after();
        // D[b] was last read by the output group for chunk c - 2
        bool go = ok;
        if (!XFER && c >= 2) go = mbar_wait(bar_dfree + 8 * b, (uint32_t)((c >> 1) - 1) & 1u) && go;
        tc_fence_after();
        constexpr uint32_t id = idesc_f16(128, VS, false, true);
        const uint64_t da = sdesc_sw128(st + G::S_WQ, 16, 1024);
        const uint64_t db = sdesc_sw128(sb + G::S16, 16384, 1024);
        if (go && elect_one()) {
#pragma unroll
          for (int kk = 0; kk < 8; ++kk)
            mma_f16(tmem + G::TM_D + b * VS, sdesc_add(da, (kk >> 2) * 16384 + (kk & 3) * 32),
                    sdesc_add(db, kk * 2048), id, kk > 0);
          mma_commit(bar_a + 8 * b);
        }
        __syncwarp();
        ok = go;
      }
      if (tl < 64) {
        // Vn = D + U, decayed to the chunk end -> B operand of the state update (over S16)
        ok = mbar_wait(bar_a + 8 * b, (uint32_t)(c >> 1) & 1u) && ok;
        tc_fence_after();
        float x[CW];
        tmem_ldw<CW>(lane_base + G::TM_D + b * VS + col, x);
        if (want_u) {
#pragma unroll
          for (int q = 0; q < CW / 8; ++q) add_half8(stp + G::S_UO + blk, swz(tl, ch0 + q), x + q * 8);
        }
        const float dec = vec[tl];
#pragma unroll
        for (int j = 0; j < CW; ++j) x[j] *= dec;
#pragma unroll
        for (int q = 0; q < CW / 8; ++q) st_half8(smem + G::S16 + (blk >> 1), swz(tl, ch0 + q), x + q * 8);
        fence_proxy_async();
        tc_fence_before();
        ok = !bar_named_or(BAR_VN, 256, !ok);
        if (warp == 0 && ok) {  // S^T += K^T Vts; with the O-row threads' arrivals the stage is free
          tc_fence_after();
          constexpr uint32_t id = idesc_f16(128, VS, true, true);
          const uint64_t da = sdesc_sw128(st + G::S_K, TILE, 1024);
          const uint64_t db = sdesc_sw128(sb + G::S16, TILE, 1024);
          if (elect_one()) {
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
              mma_f16(tmem + G::TM_S, sdesc_add(da, kk * 2048), sdesc_add(db, kk * 2048), id, 1);
            mma_commit(bar_s + 8 * b);
            mma_commit(bar_free + 8 * s);
          }
          __syncwarp();
        }
      }
    }
    if (!bad) {
      const bool okk = mbar_wait(bar_s + 8 * ((nchunks - 1) & 1), (uint32_t)((nchunks - 1) >> 1) & 1u);
      tc_fence_after();
      float* Sfin = final_state();
      if (!okk) {
        atomicExch(&g_split_error, 1);
      } else if (Sfin) {
        float r[CW];
        tmem_ldw<CW>(lane_base + G::TM_S + col, r);
#pragma unroll
        for (int j = 0; j < CW; ++j) Sfin[(size_t)(col + j) * D + tl] = r[j];
      }
    } else if (tid == 0) {
      // let the copies and MMAs in flight finish before the CTA leaves
      atomicExch(&g_split_error, 1);
      for (int k = 0; k < NST && c + k < nchunks; ++k)
        mbar_wait(bar_full + 8 * ((c + k) % NST), (uint32_t)((c + k) / NST) & 1u, 100000000ull);
      if (c > 0) mbar_wait(bar_s + 8 * ((c - 1) & 1), (uint32_t)((c - 1) >> 1) & 1u, 100000000ull);
    }
  } else if constexpr (!XFER) {
    // ========================================== output group (warps 16..23)
    // Thread og owns the 16-byte chunks (og + NOG k) * 16 of the w * silu(z)
    // tile for the copies in and the output stores; the O-row threads (warps
    // 18, 19, 22, 23) own half of token row t each.
    const int og = tid - NCW;
    const bool orow = (warp & 3) >= 2;
    const int t = (og & 127) - 64;       // token row (O-row threads)
    const int half = og >> 7;            // which half of the columns
    constexpr int HV = VS / 2;
    const int hc = half * HV;
    constexpr int ZK = NA * 8192 / 16 / NOG;
    auto z_copy = [&](int cc) {
      const uint8_t* src = p.rec + ((size_t)(slot0 + cc) * p.Hv + h) * REC + R_ZW + vs * NA * 8192;
#pragma unroll
      for (int k = 0; k < ZK; ++k) {
        const uint32_t pos = (uint32_t)(og + NOG * k) * 16;
        cp_async16(sb + G::ZT + pos, src + pos, 16u);
      }
      cp_async_commit();
    };
    if (norm_out) z_copy(0);
    bool ok = true;
    for (int c = 0; c < nchunks; ++c) {
      const int s = c % NST, b = c & 1;
      const int c0 = bos + c * C, L = min(C, eos - c0);
      const uint8_t* stp = smem + s * G::STAGE;
      const uint32_t dcol = G::TM_D + b * VS;
      float ss = 0.f;
      if (orow) {
        // O = D + Pt V, back into TMEM, and its sum of squares over this CTA's columns
        ok = mbar_wait(bar_full + 8 * s, (uint32_t)(c / NST) & 1u) && ok;  // the stage's copies are seen here too
        ok = mbar_wait(bar_a + 8 * b, (uint32_t)(c >> 1) & 1u) && ok;
        tc_fence_after();
#pragma unroll 1
        for (int j0 = hc; j0 < hc + HV; j0 += 32) {
          float o[32];
          tmem_ld32(lane_base + dcol + j0, o);
#pragma unroll
          for (int q = 0; q < 4; ++q)
            add_half8(stp + G::S_UO + (j0 >> 6) * 16384, swz(64 + t, ((j0 & 63) >> 3) + q), o + q * 8);
#pragma unroll
          for (int j = 0; j < 32; ++j) ss = fmaf(o[j], o[j], ss);
          tmem_st32(lane_base + dcol + j0, o);
          tmem_wait_st();
        }
        mbar_arrive(bar_free + 8 * s);  // Pt V read
        if (norm_out) {
          ssp[half * 64 + t] = ss;
          if constexpr (CL > 1) {
            const uint32_t peer = (uint32_t)(vs ^ 1);
            st_async_f32(mapa_shared(sb + G::XB + (uint32_t)((b * 2 + half) * 64 + t) * 4, peer), ss,
                         mapa_shared(bar_x + 8 * b, peer));
            if (og == 64) mbar_arrive_expect_tx(bar_x + 8 * b, 128 * 4);  // the other CTA's sums of this chunk
          }
        }
      }
      if (norm_out) {
        cp_async_wait_all();
        bar_named(BAR_OG, NOG);  // the chunk's w * silu(z) tile is complete
        if (orow) {
          ss = ssp[t] + ssp[64 + t];
          if constexpr (CL > 1) {
            ok = mbar_wait_cluster(bar_x + 8 * b, (uint32_t)(c >> 1) & 1u) && ok;
            ss += xb[(b * 2) * 64 + t] + xb[(b * 2 + 1) * 64 + t];
          }
          const float ri = rsqrtf(ss * (1.0f / D) + p.eps_norm);
#pragma unroll 1
          for (int j0 = hc; j0 < hc + HV; j0 += 32) {
            float o[32];
            tmem_ld32(lane_base + dcol + j0, o);
#pragma unroll
            for (int q = 0; q < 4; ++q) {
              uint4* zq = reinterpret_cast<uint4*>(smem + G::ZT + (j0 >> 6) * 8192 + swz(t, ((j0 & 63) >> 3) + q));
              const uint4 zv = *zq;
              const __half2* z2 = reinterpret_cast<const __half2*>(&zv);
              uint4 res;
              __nv_bfloat162* r2 = reinterpret_cast<__nv_bfloat162*>(&res);
#pragma unroll
              for (int e = 0; e < 4; ++e) {
                const float2 zf = __half22float2(z2[e]);
                r2[e] = __floats2bfloat162_rn(o[q * 8 + 2 * e] * ri * zf.x, o[q * 8 + 2 * e + 1] * ri * zf.y);
              }
              *zq = res;  // the output over its own w * silu(z)
            }
          }
          tc_fence_before();
          mbar_arrive(bar_dfree + 8 * b);  // D[b] read for the last time
        }
        if (bar_named_or(BAR_OG, NOG, !ok)) { ok = false; break; }  // the output tile is complete
        uint8_t* obase = reinterpret_cast<uint8_t*>(p.out) + ((size_t)c0 * p.Hv * D + h * D + vs * VS) * 2;
#pragma unroll
        for (int k = 0; k < ZK; ++k) {
          const uint32_t pos = (uint32_t)(og + NOG * k) * 16;
          const int r = (pos & 8191) >> 7, chn = (int)(pos >> 13) * 8 + ((int)((pos >> 4) & 7) ^ (r & 7));
          if (r < L)
            *reinterpret_cast<uint4*>(obase + ((size_t)r * p.Hv * D + chn * 8) * 2) =
                *reinterpret_cast<const uint4*>(smem + G::ZT + pos);
        }
        // the next chunk's w * silu(z) over the chunks this thread just stored
        if (c + 1 < nchunks) z_copy(c + 1);
      } else {
        if (orow) {
#pragma unroll 1
          for (int j0 = hc; j0 < hc + HV; j0 += 32) {
            float o[32];
            tmem_ld32(lane_base + dcol + j0, o);
            if (t < L) {
              float* dst = p.o_raw + (size_t)(c0 + t) * p.Hv * D + h * D + vs * VS + j0;
#pragma unroll
              for (int q = 0; q < 8; ++q)
                *reinterpret_cast<float4*>(dst + q * 4) = make_float4(o[4 * q], o[4 * q + 1], o[4 * q + 2], o[4 * q + 3]);
            }
          }
          tc_fence_before();
          mbar_arrive(bar_dfree + 8 * b);
        }
        if (bar_named_or(BAR_OG, NOG, !ok)) { ok = false; break; }
      }
    }
    if (!ok) atomicExch(&g_split_error, 1);
    if (norm_out) cp_async_wait_all();
  }
  tc_fence_before();
  __syncthreads();
  if constexpr (CL > 1) cluster_sync();  // no CTA leaves while the other may still write to it
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, G::TM_COLS);
  }
}

// ========================================================== segment scan
// Start states of the segments of one (value head, sequence), SR state rows
// per CTA, in fp32 on the CUDA cores: S_start(0) = S0 (or 0), then
// S_start(s+1) = S_start(s) M_s + R_s for every segment s but the last (an
// empty segment maps the state to itself).  The CTA keeps its rows
// transposed in shared memory (sT[i][r]) and each M_s in a double buffer
// filled by bulk copies one segment ahead; every map and R slice it will
// read is requested into L2 at the start.  The product is split over the
// contraction index: warp w takes i in [32 (w / 4), 32 (w / 4) + 32) and,
// with lane l, the 4 x 4 output tile rows 4 (l / 8) .. +3, columns
// 4 (8 (w % 4) + l % 8) .. +3 (per i a warp reads 64 contiguous bytes of sT
// and 128 of M: one wavefront each); the four partial tiles are summed
// through shared memory by the threads of warps 0..3, which own the rows.
constexpr int SR = 16;                  // state rows per CTA
constexpr int SCAN_KS = 4;              // contraction slices
constexpr int SCAN_POS = SR * 8;        // 4 x 4 output tiles per slice
constexpr int SCAN_THREADS = SCAN_POS * SCAN_KS;
constexpr uint32_t SCAN_SMEM = (2 * D * D + D * SR + SCAN_KS * 16 * SCAN_POS) * 4 + 16 + 128;
__global__ void __launch_bounds__(SCAN_THREADS) seg_scan_kernel(ChunkParams p) {
  extern __shared__ uint8_t scan_raw[];
  float* Mb = reinterpret_cast<float*>(scan_raw + ((128u - (smem_u32(scan_raw) & 127u)) & 127u));
  float* sT = Mb + 2 * D * D;   // [D][SR]
  float* red = sT + D * SR;     // [SCAN_KS][16][SCAN_POS] partial tiles
  const uint32_t mbar = smem_u32(red + SCAN_KS * 16 * SCAN_POS);  // two mbarriers, one per M buffer
  pdl_launch();
  const int P = p.nseg;
  const int h = blockIdx.x / (D / SR), r0 = (blockIdx.x % (D / SR)) * SR;
  const int n = blockIdx.y;
  const int tid = threadIdx.x, w = tid >> 5, l = tid & 31;
  const int ks = w >> 2, pos = tid & (SCAN_POS - 1);
  const bool owner = ks == 0;  // warps 0..3 own the rows
  const int rr = (l >> 3) * 4, cc = ((w & 3) * 8 + (l & 7)) * 4;  // this thread's tile within the CTA's rows
  const size_t hd = (size_t)D * D;
  const size_t nh = (size_t)n * p.Hv + h;
  const int bos = clampi(__ldg(p.cu_seqlens + n), 0, p.T);
  const int eos = clampi(__ldg(p.cu_seqlens + n + 1), bos, p.T);
  const int nch = (eos - bos + C - 1) / C;
  auto nonempty = [&](int sg) { return seg_lo(nch, sg + 1, P) > seg_lo(nch, sg, P); };
  auto map_of = [&](int sg) { return p.seg_mr + ((((size_t)n * (P - 1) + sg) * p.Hv + h) * 2) * hd; };
  // next non-empty segment at or after sg that has a map M (1 <= sg < P - 1;
  // segment 0 has none: its R slot holds the state at the start of segment 1), or P - 1
  auto next_map = [&](int sg) {
    if (sg < 1) sg = 1;
    while (sg < P - 1 && !nonempty(sg)) ++sg;
    return sg;
  };
  auto prefetch = [&](int sg, int buf) {  // thread 0: M_sg into buffer buf
    const float* M = map_of(sg);
    const uint32_t dst = smem_u32(Mb + buf * D * D), bar = mbar + 8 * buf;
    mbar_arrive_expect_tx(bar, D * D * 4);
#pragma unroll
    for (int q = 0; q < 4; ++q) bulk_load(dst + q * (D * D), M + q * (D * D / 4), D * D, bar);
  };
  if (tid == 0) {
    mbar_init(mbar, 1);
    mbar_init(mbar + 8, 1);
    fence_mbar_init();
  }
  pdl_wait();  // the maps come from the transfer chains
  if (tid < P - 1 && nonempty(tid)) {  // every map and R slice this CTA will read, into L2
    if (tid > 0) bulk_prefetch_l2(map_of(tid), D * D * 4);
    bulk_prefetch_l2(map_of(tid) + hd + (size_t)r0 * D, SR * D * 4);
  }
  __syncthreads();
  int sg_next = next_map(0);
  int j = 0;  // maps applied so far: map j sits in buffer j & 1, that buffer's use j >> 1
  if (tid == 0 && sg_next < P - 1) prefetch(sg_next, 0);

  // owners: the state tile; everyone: partial products.  Column pairs as
  // float2 for the packed fp32x2 FMA: acc[r][0] = columns cc, cc+1; acc[r][1] = cc+2, cc+3
  float2 acc[4][2];
  if (owner) {
    const float* S0 = p.S0 ? p.S0 + nh * hd : nullptr;
#pragma unroll
    for (int r = 0; r < 4; ++r) {
      const float4 v = S0 ? *reinterpret_cast<const float4*>(S0 + (size_t)(r0 + rr + r) * D + cc)
                          : make_float4(0.f, 0.f, 0.f, 0.f);
      acc[r][0] = make_float2(v.x, v.y);
      acc[r][1] = make_float2(v.z, v.w);
    }
  }
  for (int sg = 0;; ++sg) {
    if (owner) {
      float* dst = p.seg_start + (((size_t)n * P + sg) * p.Hv + h) * hd;
#pragma unroll
      for (int r = 0; r < 4; ++r)
        *reinterpret_cast<float4*>(dst + (size_t)(r0 + rr + r) * D + cc) =
            make_float4(acc[r][0].x, acc[r][0].y, acc[r][1].x, acc[r][1].y);
    }
    if (sg + 1 >= P) break;
    if (sg == 0) {  // segment 0: its R is the next start state (or, if it is empty, S0 passes)
      if (owner && nonempty(0)) {
        const float* R = map_of(0) + hd;
#pragma unroll
        for (int r = 0; r < 4; ++r) {
          const float4 v = __ldg(reinterpret_cast<const float4*>(R + (size_t)(r0 + rr + r) * D + cc));
          acc[r][0] = make_float2(v.x, v.y);
          acc[r][1] = make_float2(v.z, v.w);
        }
      }
      continue;
    }
    if (sg != sg_next) continue;  // empty segment: the state passes through
    // this segment's map: S <- S M + R (R is added by the owners after the
    // products, so its loads overlap them)
    float4 rv[4];
    if (owner) {
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        const int hc = c >> 1;
        *reinterpret_cast<float4*>(sT + (cc + c) * SR + rr) =
            (c & 1) ? make_float4(acc[0][hc].y, acc[1][hc].y, acc[2][hc].y, acc[3][hc].y)
                    : make_float4(acc[0][hc].x, acc[1][hc].x, acc[2][hc].x, acc[3][hc].x);
      }
      const float* R = map_of(sg) + hd;
#pragma unroll
      for (int r = 0; r < 4; ++r) rv[r] = __ldg(reinterpret_cast<const float4*>(R + (size_t)(r0 + rr + r) * D + cc));
    }
#pragma unroll
    for (int r = 0; r < 4; ++r) acc[r][0] = acc[r][1] = make_float2(0.f, 0.f);
    const int buf = j & 1;
    const uint32_t par = (uint32_t)(j >> 1) & 1u;
    if (__syncthreads_or(!mbar_wait(mbar + 8 * buf, par))) {
      // sT is complete but this segment's M never landed: record it, let the copy finish, stop
      if (tid == 0) {
        atomicExch(&g_split_error, 1);
        mbar_wait(mbar + 8 * buf, par, 100000000ull);
      }
      break;
    }
    sg_next = next_map(sg + 1);
    if (tid == 0 && sg_next < P - 1) prefetch(sg_next, buf ^ 1);
    const float* M = Mb + buf * D * D;
#pragma unroll 8
    for (int i = ks * (D / SCAN_KS); i < (ks + 1) * (D / SCAN_KS); ++i) {
      const float4 s4 = *reinterpret_cast<const float4*>(sT + i * SR + rr);
      const float4 m4 = *reinterpret_cast<const float4*>(M + i * D + cc);
      const float sv[4] = {s4.x, s4.y, s4.z, s4.w};
      const float2 m01 = make_float2(m4.x, m4.y), m23 = make_float2(m4.z, m4.w);
#pragma unroll
      for (int r = 0; r < 4; ++r) {
        const float2 s2 = make_float2(sv[r], sv[r]);
        acc[r][0] = __ffma2_rn(s2, m01, acc[r][0]);
        acc[r][1] = __ffma2_rn(s2, m23, acc[r][1]);
      }
    }
    if (!owner) {
#pragma unroll
      for (int r = 0; r < 4; ++r)
#pragma unroll
        for (int c = 0; c < 4; ++c)
          red[((ks * 16) + r * 4 + c) * SCAN_POS + pos] = (c & 1) ? acc[r][c >> 1].y : acc[r][c >> 1].x;
    }
    __syncthreads();  // partial tiles written; everyone is done with sT and this buffer
    if (owner) {
#pragma unroll
      for (int r = 0; r < 4; ++r) {
        const float rvr[4] = {rv[r].x, rv[r].y, rv[r].z, rv[r].w};
        float v[4];
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          v[c] = ((c & 1) ? acc[r][c >> 1].y : acc[r][c >> 1].x) + rvr[c];
#pragma unroll
          for (int k2 = 1; k2 < SCAN_KS; ++k2) v[c] += red[((k2 * 16) + r * 4 + c) * SCAN_POS + pos];
        }
        acc[r][0] = make_float2(v[0], v[1]);
        acc[r][1] = make_float2(v[2], v[3]);
      }
    }
    ++j;
    // the owners' reads of `red` end before its next write: two barriers
    // (the one above sT's completion and the one after the products) lie between
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

// ========================================================== affine fold
// X <- X M_s (+ R_s on rows >= r_add) for s = 0 .. nmaps-1, in fp32 on the
// CUDA cores, SR rows of one (sequence, head) per CTA (the products split as
// in seg_scan_kernel: four contraction slices, 4 x 4 output tiles, slice 0
// owning the rows).  M_s arrives by bulk copies into a double buffer one map
// ahead.  Used to compose the segment maps of the state-map mode and to fold
// the maps of consecutive parts of a sequence into a start state.
constexpr int FOLD_KS = 4;
constexpr int FOLD_POS = SR * 8;
constexpr int FOLD_THREADS = FOLD_POS * FOLD_KS;
constexpr uint32_t FOLD_SMEM = (2 * D * D + D * SR + (FOLD_KS - 1) * 16 * FOLD_POS) * 4 + 16 + 128;
__global__ void __launch_bounds__(FOLD_THREADS) state_fold_kernel(FoldParams p) {
  extern __shared__ uint8_t fold_raw[];
  float* Mb = reinterpret_cast<float*>(fold_raw + ((128u - (smem_u32(fold_raw) & 127u)) & 127u));
  float* sT = Mb + 2 * D * D;  // [D][SR]: this CTA's rows, transposed
  float* red = sT + D * SR;    // [FOLD_KS - 1][16][FOLD_POS]: partial tiles of slices 1..
  const uint32_t mbar = smem_u32(red + (FOLD_KS - 1) * 16 * FOLD_POS);
  pdl_launch();
  const int per = p.rows / SR;
  const int h = (int)blockIdx.x / per, r0 = ((int)blockIdx.x % per) * SR;
  const int n = (int)blockIdx.y;
  const int tid = threadIdx.x, w = tid >> 5, l = tid & 31;
  const int ks = w >> 2, pos = tid & (FOLD_POS - 1);
  const bool owner = ks == 0;
  const int rr = (l >> 3) * 4, cc = ((w & 3) * 8 + (l & 7)) * 4;
  const size_t dd = (size_t)D * D;
  const bool add_r = r0 >= p.r_add;  // a CTA's rows lie on one side of r_add (a multiple of SR)
  auto map_of = [&](int s) { return p.maps + (size_t)s * p.map_s + (size_t)n * p.map_n + (size_t)h * 2 * dd; };
  auto prefetch = [&](int s, int buf) {  // thread 0: M_s into buffer buf
    const float* M = map_of(s);
    const uint32_t dst = smem_u32(Mb + buf * D * D), bar = mbar + 8 * buf;
    mbar_arrive_expect_tx(bar, D * D * 4);
#pragma unroll
    for (int q = 0; q < 4; ++q) bulk_load(dst + q * (D * D), M + q * (D * D / 4), D * D, bar);
  };
  if (tid == 0) {
    mbar_init(mbar, 1);
    mbar_init(mbar + 8, 1);
    fence_mbar_init();
  }
  pdl_wait();  // the maps may come from the kernel before
  if (tid < p.nmaps) {  // every map (and R slice) this CTA reads, into L2
    bulk_prefetch_l2(map_of(tid), D * D * 4);
    if (add_r) bulk_prefetch_l2(map_of(tid) + dd + (size_t)(r0 - p.r_add) * D, SR * D * 4);
  }
  __syncthreads();
  if (tid == 0 && p.nmaps > 0) prefetch(0, 0);
  float2 acc[4][2];
  if (owner) {
    const float* X0 = p.x0 ? p.x0 + (size_t)n * p.x0_n + (size_t)h * p.x0_h : nullptr;
#pragma unroll
    for (int r = 0; r < 4; ++r) {
      const float4 v = X0 ? *reinterpret_cast<const float4*>(X0 + (size_t)(r0 + rr + r) * D + cc)
                          : make_float4(0.f, 0.f, 0.f, 0.f);
      acc[r][0] = make_float2(v.x, v.y);
      acc[r][1] = make_float2(v.z, v.w);
    }
  }
  bool ok = true;
  for (int s = 0; s < p.nmaps; ++s) {
    float4 rv[4];
    if (owner) {
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        const int hc = c >> 1;
        *reinterpret_cast<float4*>(sT + (cc + c) * SR + rr) =
            (c & 1) ? make_float4(acc[0][hc].y, acc[1][hc].y, acc[2][hc].y, acc[3][hc].y)
                    : make_float4(acc[0][hc].x, acc[1][hc].x, acc[2][hc].x, acc[3][hc].x);
      }
      const float* R = map_of(s) + dd + (size_t)(r0 - p.r_add) * D;
#pragma unroll
      for (int r = 0; r < 4; ++r)
        rv[r] = add_r ? __ldg(reinterpret_cast<const float4*>(R + (size_t)(rr + r) * D + cc))
                      : make_float4(0.f, 0.f, 0.f, 0.f);
    }
#pragma unroll
    for (int r = 0; r < 4; ++r) acc[r][0] = acc[r][1] = make_float2(0.f, 0.f);
    const int buf = s & 1;
    const uint32_t par = (uint32_t)(s >> 1) & 1u;
    if (__syncthreads_or(!mbar_wait(mbar + 8 * buf, par))) {
      if (tid == 0) {  // the copy never landed: record it, let it finish, stop
        atomicExch(&g_split_error, 1);
        mbar_wait(mbar + 8 * buf, par, 100000000ull);
      }
      ok = false;
      break;
    }
    if (tid == 0 && s + 1 < p.nmaps) prefetch(s + 1, buf ^ 1);
    const float* M = Mb + buf * D * D;
#pragma unroll 8
    for (int i = ks * (D / FOLD_KS); i < (ks + 1) * (D / FOLD_KS); ++i) {
      const float4 s4 = *reinterpret_cast<const float4*>(sT + i * SR + rr);
      const float4 m4 = *reinterpret_cast<const float4*>(M + i * D + cc);
      const float sv[4] = {s4.x, s4.y, s4.z, s4.w};
      const float2 m01 = make_float2(m4.x, m4.y), m23 = make_float2(m4.z, m4.w);
#pragma unroll
      for (int r = 0; r < 4; ++r) {
        const float2 s2 = make_float2(sv[r], sv[r]);
        acc[r][0] = __ffma2_rn(s2, m01, acc[r][0]);
        acc[r][1] = __ffma2_rn(s2, m23, acc[r][1]);
      }
    }
    if (!owner) {
#pragma unroll
      for (int r = 0; r < 4; ++r)
#pragma unroll
        for (int c = 0; c < 4; ++c)
          red[(((ks - 1) * 16) + r * 4 + c) * FOLD_POS + pos] = (c & 1) ? acc[r][c >> 1].y : acc[r][c >> 1].x;
    }
    __syncthreads();  // partial tiles written; sT and this buffer are free again
    if (owner) {
#pragma unroll
      for (int r = 0; r < 4; ++r) {
        const float rvr[4] = {rv[r].x, rv[r].y, rv[r].z, rv[r].w};
        float v[4];
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          v[c] = ((c & 1) ? acc[r][c >> 1].y : acc[r][c >> 1].x) + rvr[c];
#pragma unroll
          for (int k2 = 1; k2 < FOLD_KS; ++k2) v[c] += red[(((k2 - 1) * 16) + r * 4 + c) * FOLD_POS + pos];
        }
        acc[r][0] = make_float2(v[0], v[1]);
        acc[r][1] = make_float2(v[2], v[3]);
      }
    }
  }
  if (owner && ok) {
    float* dst = p.out + ((size_t)n * p.Hv + h) * p.rows * D;
#pragma unroll
    for (int r = 0; r < 4; ++r)
      *reinterpret_cast<float4*>(dst + (size_t)(r0 + rr + r) * D + cc) =
          make_float4(acc[r][0].x, acc[r][0].y, acc[r][1].x, acc[r][1].y);
  }
}

}  // namespace

size_t chunk_tc_split_record_bytes(int N, int T, int Hv) {
  return record_slots(N, T) * (size_t)Hv * REC;
}

size_t chunk_tc_split_seg_bytes(int N, int Hv) {
  if ((long)N * Hv > kSegMaxChains) return 0;
  // seg_mr [N][kSegMax-1][Hv][2][D][D] then seg_start [N][kSegMax][Hv][D][D]
  return (size_t)N * Hv * (2 * (kSegMax - 1) + kSegMax) * D * D * sizeof(float);
}

namespace {

int sm_count() {
  static int count = 0;
  if (count == 0) {
    int dev = 0, v = 0;
    if (cudaGetDevice(&dev) == cudaSuccess &&
        cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev) == cudaSuccess && v > 0)
      count = v;
    else
      return 148;
  }
  return count;
}

// Launch the chains: the output chains of every segment (XFER = false), or
// the transfer chains of every segment but the last (XFER = true, VS = D).
template <int VS, bool XFER>
cudaError_t launch_chain(const CUtensorMap& mk, const ChunkParams& p, cudaStream_t st) {
  using G = ChainCfg<VS>;
  cudaError_t e = cudaFuncSetAttribute(chunk_chain_kernel<VS, XFER>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)G::SMEM);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg;
  memset(&cfg, 0, sizeof(cfg));
  cfg.gridDim = XFER ? dim3((unsigned)(2 * p.Hv), (unsigned)(p.N * (p.map_out ? p.nseg : p.nseg - 1)), 1)
                     : dim3((unsigned)(G::CL * p.Hv), (unsigned)(p.N * p.nseg), 1);
  cfg.blockDim = dim3(XFER ? NCW : NTB, 1, 1);
  cfg.dynamicSmemBytes = G::SMEM;
  cfg.stream = st;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = G::CL;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;  // see pdl_wait
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  return cudaLaunchKernelEx(&cfg, chunk_chain_kernel<VS, XFER>, mk, p);
}

}  // namespace

cudaError_t launch_chunk_tc_split(const ChunkParams& p0, cudaStream_t st) {
  if (p0.N == 0 || p0.Hv == 0) return cudaSuccess;
  ChunkParams p = p0;
  if (p.nseg < 1) p.nseg = 1;
  if (!p.rec) return cudaErrorInvalidValue;
  CUtensorMap mq, mk, mv, mql, mkl;
  memset(&mq, 0, sizeof(mq));
  memset(&mk, 0, sizeof(mk));
  memset(&mv, 0, sizeof(mv));
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
    if (p.k_lo && (!make_map(&mql, p.q_lo, (uint64_t)p.T, (uint64_t)p.Hk * D, f16, sw) ||
                   !make_map(&mkl, p.k_lo, (uint64_t)p.T, (uint64_t)p.Hk * D, f16, sw)))
      return cudaErrorInvalidValue;
  }
  if (p.T > 0 && !p.reuse_records) {
    cudaError_t e = cudaFuncSetAttribute(chunk_keys_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)A_SMEM);
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t cfg;
    memset(&cfg, 0, sizeof(cfg));
    // persistent: two CTAs per SM (shared memory, registers and TMEM allow two)
    const int slots = (int)record_slots(p.N, p.T);
    const long long units = (long long)slots * p.Hv;
    const int ctas = (int)(units < 2LL * host::sm_count() ? units : 2LL * host::sm_count());
    cfg.gridDim = dim3((unsigned)ctas, 1, 1);
    cfg.blockDim = dim3(NTA, 1, 1);
    cfg.dynamicSmemBytes = A_SMEM;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;  // see pdl_wait
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    e = cudaLaunchKernelEx(&cfg, chunk_keys_kernel, mq, mk, mv, mql, mkl, p, slots);
    if (e != cudaSuccess) return e;
  }
  const int P = p.nseg;
  if (p.map_out) {
    // state-map mode: the maps of all P segments, then their composition
    if (!p.seg_mr || P > kSegMax - 1 || (P == 1 && p.seg_mr != p.map_out)) return cudaErrorInvalidValue;
    cudaError_t e = launch_chain<D, true>(mk, p, st);
    if (e != cudaSuccess || P == 1) return e;
    const size_t dd = (size_t)D * D;
    FoldParams f{};
    f.x0 = p.seg_mr;  // segment 0's [M; R]
    f.x0_n = (size_t)P * p.Hv * 2 * dd;
    f.x0_h = 2 * dd;
    f.maps = p.seg_mr + (size_t)p.Hv * 2 * dd;  // segments 1 .. P-1
    f.map_s = (size_t)p.Hv * 2 * dd;
    f.map_n = (size_t)P * p.Hv * 2 * dd;
    f.nmaps = P - 1;
    f.rows = 2 * D;
    f.r_add = D;
    f.out = p.map_out;
    f.N = p.N;
    f.Hv = p.Hv;
    return launch_state_fold(f, st);
  }
  if (P > 1) {
    if (!p.seg_mr || !p.seg_start || P > kSegMax) return cudaErrorInvalidValue;
    cudaError_t e = launch_chain<D, true>(mk, p, st);
    if (e != cudaSuccess) return e;
    e = cudaFuncSetAttribute(seg_scan_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)SCAN_SMEM);
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t cfg;
    memset(&cfg, 0, sizeof(cfg));
    cfg.gridDim = dim3((unsigned)(p.Hv * (D / SR)), (unsigned)p.N, 1);
    cfg.blockDim = dim3(SCAN_THREADS, 1, 1);
    cfg.dynamicSmemBytes = SCAN_SMEM;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;  // see pdl_wait
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    e = cudaLaunchKernelEx(&cfg, seg_scan_kernel, p);
    if (e != cudaSuccess) return e;
  }
  // Half-width value slices (two CTAs per chain) while that still fits the
  // machine in one wave; otherwise one CTA per chain.
  const long ctas = (long)p.Hv * p.N * P;
  if (2 * ctas <= sm_count()) return launch_chain<64, false>(mk, p, st);
  return launch_chain<128, false>(mk, p, st);
}

// Segments per sequence for the chain: the count that minimises an estimate
// of the serial chain steps -- ceil(chunks / P) steps for the transfer chains
// (per wave of them: 2 (P - 1) - 1 CTAs per chain, segment 0 needing no map)
// plus as many for the output chains, about two per scan step (P - 2) and two
// for the extra launches -- among those whose output chains fit the SMs in
// one wave.  One serial chain takes `chunks` steps.
cudaError_t launch_state_fold(const FoldParams& p, cudaStream_t st) {
  if (p.N == 0 || p.Hv == 0) return cudaSuccess;
  if (p.rows != D && p.rows != 2 * D) return cudaErrorInvalidValue;
  if (p.r_add != 0 && p.r_add != D) return cudaErrorInvalidValue;
  if (p.nmaps < 0 || (p.nmaps > 0 && !p.maps) || !p.out) return cudaErrorInvalidValue;
  cudaError_t e = cudaFuncSetAttribute(state_fold_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)FOLD_SMEM);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg;
  memset(&cfg, 0, sizeof(cfg));
  cfg.gridDim = dim3((unsigned)(p.Hv * (p.rows / SR)), (unsigned)p.N, 1);
  cfg.blockDim = dim3(FOLD_THREADS, 1, 1);
  cfg.dynamicSmemBytes = FOLD_SMEM;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;  // see pdl_wait
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, state_fold_kernel, p);
}

// State-map mode: as many segments as fill the SMs with the transfer chains
// (both roles of every segment) in one wave.
int chunk_tc_split_map_segments(int N, int Hv) {
  const long chains = (long)N * Hv;
  if (N <= 0 || chains > kSegMaxChains) return 1;
  const long P = sm_count() / (2 * chains);
  return (int)(P < 1 ? 1 : P > kSegMax - 1 ? kSegMax - 1 : P);
}

int chunk_tc_split_auto_segments(int N, int T, int Hv) {
  const long chains = (long)N * Hv;
  if (N <= 0 || chains > kSegMaxChains) return 1;
  const int sms = sm_count();
  const double nch = (double)T / C / N;  // chunks per sequence, on average
  int best = 1;
  double best_cost = nch;
  for (int P = 3; P <= kSegMax; ++P) {
    if (chains * P > sms) break;
    const double seg = ceil(nch / P);
    const double waves = ceil((double)chains * (2 * (P - 1) - 1) / sms);
    const double out_step = 2 * chains * P <= sms ? 1.0 : 1.15;  // whole-row chains are a little slower
    const double cost = seg * waves + seg * out_step + 2.0 * (P - 2) + 2.0;
    if (cost < best_cost) {
      best_cost = cost;
      best = P;
    }
  }
  return best;
}

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
