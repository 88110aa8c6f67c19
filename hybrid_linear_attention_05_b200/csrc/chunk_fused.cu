// Chunked gated delta rule on the tensor cores in one persistent,
// warp-specialised kernel: the key-side work of chunk c + 1 runs on the same
// SM as the state chain of chunk c, so nothing passes through HBM between
// them.
//
// The algebra is the regrouped chunked (WY / UT transform) form of the
// recurrence that the two-kernel path uses ("Qwen (text & vision-language)",
// Verified parity: chunked and recurrent Gated DeltaNet agree up to
// floating-point accumulation).  With T = (I + A)^-1, Tb = T diag(beta),
// Tbe = T diag(beta e^gamma), W = Tbe K, U = Tb V, P = (Q K^T) o causal decay,
// Pt = P Tb and Ph = P Tbe:
//     Vn = U - W S0^T,   O = Qt S0^T + Pt V,   Qt = diag(e^gamma) Q - Ph K,
//     S^T = e^{gamma_L} S0^T + K^T diag(e^{gamma_L - gamma}) Vn.
//
// One CTA per SM walks (sequence, value head) chains taken from a queue that
// holds the longest sequences first.  Roles:
//   producer warp   takes the next chain from the queue, fills a stage (one of
//                   two): the chunk's K, Q tiles and their rounding residuals
//                   by TMA, its gates, and where it is;
//   key side        (8 warps) per chunk: D1 = [K;Q] K^T (with the residual
//                   cross terms), the decay table, A and P, T = (I + A)^-1 on
//                   CUDA cores, D2 = [Tb; P] [Tb | -Tbe] (Pt and -Ph),
//                   D3 = [-Tbe 0; -Ph E] [K; Q] = [-W; Qt] into the stage as the
//                   chain's A operand, and D4 = [Tb; Pt] V = [U; Pt V] straight
//                   into the chain's TMEM accumulator of that stage;
//   chain           (8 warps) holds S^T[dk][v] in TMEM for the whole chain:
//                   per chunk the fp16 image of S^T, D += [-W; Qt] S0^T
//                   (so D = [Vn; O]), the decayed Vn as the B operand of
//                   S^T += K^T Vn_d; the warps that reach TMEM lanes 64..127
//                   take O and write the gated RMSNorm output.
// No TMA multicast is used.
#include <cuda.h>
#include <string.h>

#include "gdn_internal.h"
#include "host_util.h"
#include "tc_chunk_common.cuh"
#include "tc_ptx.cuh"

namespace gdn {

__device__ int g_fused_error = 0;  // nonzero: a bounded wait in the fused kernel gave up

namespace {

using namespace ptx;
using namespace tcc;

constexpr int C = 64;
constexpr int D = 128;
constexpr uint32_t TILE = 64 * 128;  // one 64 x 64 16-bit box

// ---- roles
constexpr int NK = 256;                   // key side: warps 0..7
constexpr int NCH = 256;                  // chain: warps 8..15
constexpr int PROD_WARP = 16;             // producer
constexpr int NTHREADS = NK + NCH + 32;
constexpr int BAR_K = 1, BAR_C = 2, BAR_VN = 3, BAR_O = 4;  // named barriers

// ---- shared memory (byte offsets from a 1024-aligned base)
// A stage: [K; Q] (two dk halves of 16 KiB, each 64 K rows then 64 Q rows of
// 128 B, 128-byte swizzle); then a 32 KiB region that holds the residual
// tiles [K_lo; Q_lo] for D1, then the V tile (two 64-column halves of 64
// rows) for D4, then [-W; Qt] (two dk atoms of 128 rows) for the chain; then
// the stage's bookkeeping.
constexpr uint32_t ST_KQ = 0;
constexpr uint32_t ST_LOV = 32768;
constexpr uint32_t ST_META = 65536;
constexpr uint32_t STAGE = 66560;
struct StageMeta {
  float decL[64];    // e^{gamma_L - gamma_i}, 0 past the chunk        (key side)
  float egL;         // e^{gamma_L}                                     (key side)
  int n, h, c0, L;   // sequence, value head, first token, tokens     (producer)
  int flags;         // 1: first chunk of its chain, 2: last, 4: no more work
  int pad[2];
  float g[64];       // log decay, 0 past the chunk                    (producer)
  float beta[64];
};
static_assert(sizeof(StageMeta) <= STAGE - ST_META, "stage bookkeeping");
constexpr int F_FIRST = 1, F_LAST = 2, F_DONE = 4;

constexpr uint32_t OFF_TBP = 2 * STAGE;              // [Tb; P], later [Tb; Pt]: K-major 128 rows x 64
constexpr uint32_t OFF_AW = OFF_TBP + 16384;         // [-Tbe 0; -Ph E]: two 16 KiB K atoms
constexpr uint32_t OFF_AF = OFF_AW;                  // fp32 A [64][AS] (dead before AW is written)
constexpr uint32_t OFF_TF = OFF_AF + 64 * AS * 4;    // fp32 T [64][AS]; before it the decay table E
constexpr uint32_t OFF_X = OFF_TF + 64 * AS * 4;     // fp32 scratch of the inverse
constexpr uint32_t OFF_S16 = OFF_X + 4096;           // fp16 S^T image (two 64-column value blocks); then Vn_d
constexpr uint32_t OFF_MISC = OFF_S16 + 32768;
constexpr uint32_t M_GAM = 0, M_EG = 256, M_BET = 512, M_SCAN = 768, M_W = 832, M_SSP = 1344,
                   M_ABORT = 2368, M_BAR = 2432, M_ISSUED = 2432 + 8 * 16, M_TMEM = M_ISSUED + 4 * 16;
constexpr uint32_t SMEM_USED = OFF_MISC + M_TMEM + 16;
constexpr uint32_t SMEM_BYTES = SMEM_USED + 1024;
static_assert(OFF_AW % 1024 == 0 && OFF_TBP % 1024 == 0 && OFF_S16 % 1024 == 0, "swizzled tiles");
static_assert(OFF_AW + 32768 <= OFF_S16, "AW inside the dead fp32 scratch");
static_assert(SMEM_BYTES <= 232448, "shared memory");

// ---- TMEM columns
constexpr uint32_t TM_S = 0;      // S^T [dk lanes][v columns], fp32
constexpr uint32_t TM_D = 128;    // the chain's [Vn; O] accumulator
constexpr uint32_t TM_D1 = 256;   // D1 of each stage (64 columns each), issued ahead by the producer
constexpr uint32_t TM_KEY = 384;  // D2, D3 of the key side
constexpr uint32_t TM_COLS = 512;

// mbarriers (8 bytes each, from M_BAR).  issued[i] counts the phases of
// barrier i that a copy or a tensor-core commit was started for, so that
// the CTA can let them all land before it frees TMEM and leaves.
enum { B_FULL = 0, B_VFULL = 2, B_READY = 4, B_FREE = 6, B_K1 = 8, B_K2 = 10, B_K3 = 11, B_D = 12,
       B_S = 13, B_DFREE = 14, NBARS = 15 };

// Bounded wait that also gives up when another role has given up.
__device__ __forceinline__ bool wait_bar(uint32_t bar, uint32_t parity, volatile int* abort_flag,
                                         uint64_t limit_ns = 2000000000ull) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = globaltimer_ns();
  while (true) {
    if (mbar_try_wait(bar, parity)) return true;
    if (*abort_flag) return false;
    if (globaltimer_ns() - t0 > limit_ns) {
      *abort_flag = 1;
      atomicExch(&g_fused_error, 1);
      return false;
    }
  }
}

struct FusedArgs {
  ChunkParams p;
  const int* order;  // [N] sequences by decreasing length (or null: index order)
  int* queue;        // chain counter, zero at launch
};

__global__ void __launch_bounds__(NTHREADS, 1)
    chunk_fused_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                       const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_ql,
                       const __grid_constant__ CUtensorMap tm_kl, const FusedArgs fa) {
  const ChunkParams& p = fa.p;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  const uint32_t sb = smem_u32(smem);
  uint8_t* misc = smem + OFF_MISC;
  float* gam = reinterpret_cast<float*>(misc + M_GAM);
  float* eg = reinterpret_cast<float*>(misc + M_EG);
  float* bet = reinterpret_cast<float*>(misc + M_BET);
  float* scan = reinterpret_cast<float*>(misc + M_SCAN);
  float* wsm = reinterpret_cast<float*>(misc + M_W);
  float* ssp = reinterpret_cast<float*>(misc + M_SSP);  // [2 parities][2 halves][64 tokens]
  volatile int* abort_flag = reinterpret_cast<volatile int*>(misc + M_ABORT);
  int* issued = reinterpret_cast<int*>(misc + M_ISSUED);
  const uint32_t bars = sb + OFF_MISC + M_BAR;
  auto bar = [&](int i) { return bars + 8u * (uint32_t)i; };
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(misc + M_TMEM);
  auto meta = [&](int s) { return reinterpret_cast<StageMeta*>(smem + s * STAGE + ST_META); };

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const bool has_lo = p.k_lo != nullptr;
  const int G = p.Hv / p.Hk;

  if (tid == 0) {
    for (int s = 0; s < 2; ++s) {
      mbar_init(bar(B_FULL + s), 32);       // the producer warp's lanes (lane 0 with the TMA bytes)
      mbar_init(bar(B_VFULL + s), 1);
      mbar_init(bar(B_READY + s), 1);
      mbar_init(bar(B_FREE + s), 1);        // the chain's MMAs of the stage's chunk have completed
      mbar_init(bar(B_K1 + s), 1);
    }
    mbar_init(bar(B_D), 1);
    mbar_init(bar(B_DFREE), 2);             // the chain's new-value and O-row threads read D
    mbar_init(bar(B_K2), 1);
    mbar_init(bar(B_K3), 1);
    mbar_init(bar(B_S), 1);
    *abort_flag = 0;
    for (int i = 0; i < NBARS; ++i) issued[i] = 0;
    fence_mbar_init();
  }
  if (tid < D) wsm[tid] = p.out ? __bfloat162float(static_cast<const __nv_bfloat16*>(p.norm_w)[tid]) : 0.f;
  if (warp == 0) {
    tmem_alloc(smem_u32(tmem_slot), TM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  pdl_wait();  // q, k, v, their residuals and the gates come from the conv kernel

  if (warp == PROD_WARP) {
    // =================================================== producer warp
    int ci = 0;        // chunks published by this CTA
    bool ok = true;
    const int nchains = p.N * p.Hv;
    while (ok) {
      int idx = 0;
      if (lane == 0) idx = atomicAdd(fa.queue, 1);
      idx = __shfl_sync(0xffffffffu, idx, 0);
      const bool more = idx < nchains;
      int n = 0, h = 0, bos = 0, eos = 0, nch = 1;
      if (more) {
        const int r = idx / p.Hv;
        h = idx - r * p.Hv;
        n = fa.order ? clampi(__ldg(fa.order + r), 0, p.N - 1) : r;
        bos = clampi(__ldg(p.cu_seqlens + n), 0, p.T);
        eos = clampi(__ldg(p.cu_seqlens + n + 1), bos, p.T);
        nch = (eos - bos + C - 1) / C;
        if (nch == 0) {  // empty sequence: its state passes through
          if (p.S_out) {
            const size_t base = ((size_t)n * p.Hv + h) * D * D;
            for (int e = lane; e < D * D; e += 32) p.S_out[base + e] = p.S0 ? p.S0[base + e] : 0.f;
          }
          continue;
        }
      }
      const int hk = h / G;
      for (int cc = 0; cc < nch && ok; ++cc, ++ci) {
        const int s = ci & 1;
        if (ci >= 2) {
          bool w = true;
          if (lane == 0) w = wait_bar(bar(B_FREE + s), (uint32_t)((ci >> 1) - 1) & 1u, abort_flag);
          ok = __shfl_sync(0xffffffffu, (int)w, 0) != 0;
        }
        if (!ok) break;
        StageMeta* m = meta(s);
        const int c0 = bos + cc * C, L = more ? min(C, eos - c0) : 0;
        if (more) {
          for (int e = lane; e < C; e += 32) {
            m->g[e] = e < L ? __ldg(p.g + (size_t)h * p.T + c0 + e) : 0.f;
            m->beta[e] = e < L ? __ldg(p.beta + (size_t)h * p.T + c0 + e) : 0.f;
          }
        }
        if (lane == 0) {
          m->n = n; m->h = h; m->c0 = c0; m->L = L;
          m->flags = more ? ((cc == 0 ? F_FIRST : 0) | (cc == nch - 1 ? F_LAST : 0)) : F_DONE;
        }
        __syncwarp();
        if (lane == 0) issued[B_FULL + s]++;
        if (lane == 0 && more) {
          const uint32_t st = sb + s * STAGE;
          mbar_arrive_expect_tx(bar(B_FULL + s), (has_lo ? 8 : 4) * TILE);
          tma_load_2d(st + ST_KQ, &tm_k, hk * D, c0, bar(B_FULL + s));
          tma_load_2d(st + ST_KQ + 16384, &tm_k, hk * D + 64, c0, bar(B_FULL + s));
          tma_load_2d(st + ST_KQ + 8192, &tm_q, hk * D, c0, bar(B_FULL + s));
          tma_load_2d(st + ST_KQ + 16384 + 8192, &tm_q, hk * D + 64, c0, bar(B_FULL + s));
          if (has_lo) {
            tma_load_2d(st + ST_LOV, &tm_kl, hk * D, c0, bar(B_FULL + s));
            tma_load_2d(st + ST_LOV + 16384, &tm_kl, hk * D + 64, c0, bar(B_FULL + s));
            tma_load_2d(st + ST_LOV + 8192, &tm_ql, hk * D, c0, bar(B_FULL + s));
            tma_load_2d(st + ST_LOV + 16384 + 8192, &tm_ql, hk * D + 64, c0, bar(B_FULL + s));
          }
        } else {
          mbar_arrive(bar(B_FULL + s));
        }
        if (more) {
          // D1 = [K; Q] K^T (+ [K_lo; Q_lo] K^T + [K; Q] K_lo^T) into this stage's
          // D1 columns as soon as the tiles land (the key side took the previous
          // D1 of the stage before the chain released it), then the V tile over
          // the residual tiles D1 has read
          bool w = true;
          if (lane == 0) {
            const uint32_t ph = (uint32_t)(ci >> 1) & 1u;
            const uint32_t st = sb + s * STAGE;
            w = wait_bar(bar(B_FULL + s), ph, abort_flag);
            if (w) {
              tc_fence_after();
              constexpr uint32_t id = idesc_f16(128, 64, false, false);
              const uint64_t dkq = sdesc_sw128(st + ST_KQ, 16, 1024);
              const uint64_t dlo = sdesc_sw128(st + ST_LOV, 16, 1024);
#pragma unroll
              for (int kk = 0; kk < 8; ++kk) {
                const uint32_t off = (kk >> 2) * 16384 + (kk & 3) * 32;
                const uint64_t dh = sdesc_add(dkq, off);
                mma_f16(tmem + TM_D1 + s * 64, dh, dh, id, kk > 0);
                if (has_lo) {
                  const uint64_t dl = sdesc_add(dlo, off);
                  mma_f16(tmem + TM_D1 + s * 64, dl, dh, id, 1);
                  mma_f16(tmem + TM_D1 + s * 64, dh, dl, id, 1);
                }
              }
              mma_commit(bar(B_K1 + s));
              issued[B_K1 + s]++;
              w = wait_bar(bar(B_K1 + s), ph, abort_flag);
            }
            if (w) {
              mbar_arrive_expect_tx(bar(B_VFULL + s), 2 * TILE);
              tma_load_2d(st + ST_LOV, &tm_v, h * D, c0, bar(B_VFULL + s));
              tma_load_2d(st + ST_LOV + TILE, &tm_v, h * D + 64, c0, bar(B_VFULL + s));
              issued[B_VFULL + s]++;
            }
          }
          ok = __shfl_sync(0xffffffffu, (int)w, 0) != 0;
        }
      }
      if (!more) break;
    }
  } else if (warp < NK / 32) {
    // ======================================================== key side
    // Every wait result is folded into `ok`; once anything has failed no more
    // copies or MMAs are started, and the role leaves its loop only at the
    // agreement point at the top of a chunk, all threads together.
    const int kt = tid, wg = kt >> 7, tl = kt & 127;
    const uint32_t lane_base = tmem + ((uint32_t)((warp & 3) * 32) << 16);
    float* Af = reinterpret_cast<float*>(smem + OFF_AF);
    float* Tf = reinterpret_cast<float*>(smem + OFF_TF);
    float* Xs = reinterpret_cast<float*>(smem + OFF_X);
    bool ok = true;
    for (int ci = 0;; ++ci) {
      const int s = ci & 1;
      const uint32_t ph = (uint32_t)(ci >> 1) & 1u;  // phase of the per-stage barriers
      const uint32_t pk = (uint32_t)ci & 1u;         // phase of the once-per-chunk barriers
      ok = wait_bar(bar(B_FULL + s), ph, abort_flag) && ok;
      StageMeta* m = meta(s);
      const bool done = ok && (m->flags & F_DONE);
      if (bar_named_or(BAR_K, NK, !ok || done)) {
        if (done && kt == 0) mbar_arrive(bar(B_READY + s));  // tell the chain
        break;
      }
      const int L = m->L;
      const uint32_t st = sb + s * STAGE;
      // gates: gamma = cumulative g, e^gamma, beta
      float gv = 0.f, bv = 0.f;
      if (kt < 64) {
        gv = m->g[kt];
        bv = m->beta[kt];
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const float t = __shfl_up_sync(0xffffffffu, gv, o);
          if (lane >= o) gv += t;
        }
        if (kt == 31) scan[0] = gv;
      }
      role_sync<NK, BAR_K>();
      if (kt < 64) {
        if (kt >= 32) gv += scan[0];
        gam[kt] = gv;
        eg[kt] = __expf(gv);
        bet[kt] = bv;
      }
      role_sync<NK, BAR_K>();  // gamma is in shared memory
      if (kt < 64) m->decL[kt] = kt < L ? __expf(gam[L - 1] - gam[kt]) : 0.f;
      if (kt == 0) m->egL = eg[L - 1];
      ok = wait_bar(bar(B_K1 + s), ph, abort_flag) && ok;  // D1, issued by the producer
      tc_fence_after();
      // A (rows 0..63) -> fp32; P (rows 64..127) -> fp16 rows 64..127 of [Tb; P].
      // This thread: row tl, columns wg*32 .. wg*32+31.
      // the decay factors e^{gamma_i - gamma_j} (j <= i) are formed here, from
      // the row's gamma_i and the columns' gamma_j (clamped so that the masked
      // entries j > i never overflow)
      {
        float x[32];
        tmem_ld32(lane_base + TM_D1 + s * 64 + wg * 32, x);
        const int i = tl & 63;
        const float gi = gam[i];
        if (tl < 64) {
          const float bi = i < L ? bet[i] : 0.f;
#pragma unroll
          for (int e4 = 0; e4 < 32; e4 += 4) {
            const float4 g4 = *reinterpret_cast<const float4*>(gam + wg * 32 + e4);
            const float gj[4] = {g4.x, g4.y, g4.z, g4.w};
            float4 v;
            float* vf = reinterpret_cast<float*>(&v);
#pragma unroll
            for (int u = 0; u < 4; ++u) {
              const int j = wg * 32 + e4 + u;
              vf[u] = j < i ? bi * __expf(fminf(gi - gj[u], 0.f)) * x[e4 + u] : 0.f;
            }
            *reinterpret_cast<float4*>(Af + i * AS + wg * 32 + e4) = v;
          }
        } else {
          const float keep = i < L ? 1.f : 0.f;
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            const float4 ga = *reinterpret_cast<const float4*>(gam + wg * 32 + q * 8);
            const float4 gb = *reinterpret_cast<const float4*>(gam + wg * 32 + q * 8 + 4);
            const float gj[8] = {ga.x, ga.y, ga.z, ga.w, gb.x, gb.y, gb.z, gb.w};
            float f[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) {
              const int j = wg * 32 + q * 8 + e;
              f[e] = j <= i ? keep * __expf(fminf(gi - gj[e], 0.f)) * x[q * 8 + e] : 0.f;
            }
            st_half8(smem + OFF_TBP, swz(tl, wg * 4 + q), f);
          }
        }
      }
      role_sync<NK, BAR_K>();
      solve_unit_lower<NK, BAR_K>(Af, Tf, Xs, kt);
      {
        // this thread's 16 entries of T, row i = kt / 4, columns (kt % 4) * 16 ..
        const int i = kt >> 2, qt = kt & 3;
        float tv[16];
#pragma unroll
        for (int e4 = 0; e4 < 16; e4 += 4) {
          const float4 t4 = *reinterpret_cast<const float4*>(Tf + i * AS + qt * 16 + e4);
          tv[e4] = t4.x; tv[e4 + 1] = t4.y; tv[e4 + 2] = t4.z; tv[e4 + 3] = t4.w;
        }
        role_sync<NK, BAR_K>();  // the fp32 scratch is dead from here: AW goes over it
#pragma unroll
        for (int q = 0; q < 2; ++q) {
          float fb[8], fe[8];
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            const int j = qt * 16 + q * 8 + e;
            fb[e] = tv[q * 8 + e] * bet[j];
            fe[e] = -fb[e] * eg[j];
          }
          st_half8(smem + OFF_TBP, swz(i, qt * 2 + q), fb);  // Tb: A rows 0..63 and B block 0 of D2
          st_half8(smem + OFF_AW, swz(i, qt * 2 + q), fe);   // -Tbe: AW rows 0..63 and B block 1 of D2
        }
      }
      fence_proxy_async();
      tc_fence_before();
      role_sync<NK, BAR_K>();
      if (kt == 0 && ok) {  // D2 = [Tb; P] [Tb | -Tbe]
        tc_fence_after();
        constexpr uint32_t id = idesc_f16(128, 128, false, true);
        const uint64_t da = sdesc_sw128(sb + OFF_TBP, 16, 1024);
        const uint64_t db = sdesc_sw128(sb + OFF_TBP, OFF_AW - OFF_TBP, 1024);
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
          mma_f16(tmem + TM_KEY, sdesc_add(da, kk * 32), sdesc_add(db, kk * 2048), id, kk > 0);
        mma_commit(bar(B_K2));
        issued[B_K2]++;
      }
      ok = wait_bar(bar(B_K2), pk, abort_flag) && ok;
      tc_fence_after();
      // rows 64..127 of D2: Pt (columns 0..63) over P in [Tb; P], -Ph (64..127) -> AW rows 64..127
      if (tl >= 64) {
        float x[32];
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
          tmem_ld32(lane_base + TM_KEY + wg * 64 + hh * 32, x);
          uint8_t* dst = smem + (wg == 0 ? OFF_TBP : OFF_AW);
#pragma unroll
          for (int q = 0; q < 4; ++q) st_half8(dst, swz(tl, hh * 4 + q), x + q * 8);
        }
      }
      fence_proxy_async();
      tc_fence_before();
      role_sync<NK, BAR_K>();
      if (kt == 0) {
        ok = wait_bar(bar(B_VFULL + s), ph, abort_flag) && ok;
        // the chain has read its accumulator for the previous chunk
        if (ci > 0) ok = wait_bar(bar(B_DFREE), (uint32_t)(ci - 1) & 1u, abort_flag) && ok;
        if (ok) {
          tc_fence_after();
          // D3 = [-Tbe; -Ph] K = [-W; -Ph K]; the diagonal term e^gamma Q of Qt
          // is added on the CUDA cores as D3 is read
          constexpr uint32_t id = idesc_f16(128, 128, false, true);
          const uint64_t da = sdesc_sw128(sb + OFF_AW, 16, 1024);
          const uint64_t db = sdesc_sw128(st + ST_KQ, 16384, 1024);
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            mma_f16(tmem + TM_KEY, sdesc_add(da, kk * 32), sdesc_add(db, kk * 2048), id, kk > 0);
          // D4 = [Tb; Pt] V = [U; Pt V], the start of the chain's accumulator
          const uint64_t dt = sdesc_sw128(sb + OFF_TBP, 16, 1024);
          const uint64_t dv = sdesc_sw128(st + ST_LOV, TILE, 1024);
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            mma_f16(tmem + TM_D, sdesc_add(dt, kk * 32), sdesc_add(dv, kk * 2048), id, kk > 0);
          mma_commit(bar(B_K3));
          issued[B_K3]++;
        }
      }
      ok = wait_bar(bar(B_K3), pk, abort_flag) && ok;
      tc_fence_after();
      // [-W; Qt] -> fp16 K-major A operand of the chain, over V: row tl, dk atom
      // wg; the Qt rows (tl >= 64, token i = tl - 64) add e^{gamma_i} Q[i]
      {
        const int i = tl - 64;
        const float egi = (tl >= 64 && i < L) ? eg[i] : 0.f;
        const uint8_t* qrow = smem + s * STAGE + ST_KQ + wg * 16384;
        float x[32];
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
          tmem_ld32(lane_base + TM_KEY + wg * 64 + hh * 32, x);
          if (tl >= 64) {
#pragma unroll
            for (int q = 0; q < 4; ++q) {
              const uint4 u = *reinterpret_cast<const uint4*>(qrow + swz(tl, hh * 4 + q));
              const __half2* h2 = reinterpret_cast<const __half2*>(&u);
#pragma unroll
              for (int e = 0; e < 4; ++e) {
                const float2 f = __half22float2(h2[e]);
                x[q * 8 + 2 * e] = fmaf(egi, f.x, x[q * 8 + 2 * e]);
                x[q * 8 + 2 * e + 1] = fmaf(egi, f.y, x[q * 8 + 2 * e + 1]);
              }
            }
          }
#pragma unroll
          for (int q = 0; q < 4; ++q) st_half8(smem + s * STAGE + ST_LOV + wg * 16384, swz(tl, hh * 4 + q), x + q * 8);
        }
      }
      fence_proxy_async();
      tc_fence_before();
      role_sync<NK, BAR_K>();
      if (kt == 0 && ok) mbar_arrive(bar(B_READY + s));
    }
  } else {
    // ============================================================ chain
    // Same discipline as the key side: results of waits fold into `ok`, no
    // MMA is started once anything failed, and the role leaves only at the
    // agreement point at the top of a chunk.
    const int ct = tid - NK;                 // 0..255
    const int cw = warp - NK / 32;           // chain warp 0..7
    const int quarter = warp & 3;            // TMEM lanes 32 quarter ..
    const int half = cw >> 2;                // value columns half*64 ..
    const int tl = quarter * 32 + lane;      // TMEM lane (dk row of the state; token row of D)
    const uint32_t lane_base = tmem + ((uint32_t)(quarter * 32) << 16);
    const bool vn_role = quarter < 2;        // lanes 0..63: new values; 64..127: outputs
    const bool norm_out = p.out != nullptr;
    bool ok = true;
    for (int ci = 0;; ++ci) {
      const int s = ci & 1;
      const uint32_t ph = (uint32_t)(ci >> 1) & 1u;
      const uint32_t pk = (uint32_t)ci & 1u;
      ok = wait_bar(bar(B_READY + s), ph, abort_flag) && ok;
      StageMeta* m = meta(s);
      const int flags = ok ? m->flags : F_DONE;
      if (bar_named_or(BAR_C, NCH, !ok || (flags & F_DONE))) break;
      const int n = m->n, h = m->h, c0 = m->c0, L = m->L;
      const size_t sbase = ((size_t)n * p.Hv + h) * D * D;
      const float egL = m->egL;
      const uint32_t st = sb + s * STAGE;
      // ---- the state's fp16 image for this chunk's products, then S^T *= e^{gamma_L}
      {
        uint8_t* img = smem + OFF_S16 + half * 16384;
        float r[32];
        if (flags & F_FIRST) {
          // a new chain: S^T[dk = tl][v] = S0[v][dk] (the last chain's state
          // update was waited for at its last chunk)
#pragma unroll
          for (int hh = 0; hh < 2; ++hh) {
            const int col = half * 64 + hh * 32;
#pragma unroll
            for (int j = 0; j < 32; ++j) r[j] = p.S0 ? p.S0[sbase + (size_t)(col + j) * D + tl] : 0.f;
#pragma unroll
            for (int q = 0; q < 4; ++q) st_half8(img, swz(tl, hh * 4 + q), r + q * 8);
#pragma unroll
            for (int j = 0; j < 32; ++j) r[j] *= egL;
            tmem_st32(lane_base + TM_S + col, r);
          }
        } else {
          ok = wait_bar(bar(B_S), pk ^ 1u, abort_flag) && ok;  // the previous chunk's state update
          tc_fence_after();
#pragma unroll
          for (int hh = 0; hh < 2; ++hh) {
            const int col = half * 64 + hh * 32;
            tmem_ld32(lane_base + TM_S + col, r);
#pragma unroll
            for (int q = 0; q < 4; ++q) st_half8(img, swz(tl, hh * 4 + q), r + q * 8);
#pragma unroll
            for (int j = 0; j < 32; ++j) r[j] *= egL;
            tmem_st32(lane_base + TM_S + col, r);
          }
        }
        tmem_wait_st();
      }
      fence_proxy_async();
      tc_fence_before();
      ok = !bar_named_or(BAR_C, NCH, !ok);
      if (ct == 0 && ok) {  // D += [-W; Qt] S0^T: D = [Vn; O]
        tc_fence_after();
        constexpr uint32_t id = idesc_f16(128, 128, false, true);
        const uint64_t da = sdesc_sw128(st + ST_LOV, 16, 1024);
        const uint64_t db = sdesc_sw128(sb + OFF_S16, 16384, 1024);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          mma_f16(tmem + TM_D, sdesc_add(da, (kk >> 2) * 16384 + (kk & 3) * 32),
                  sdesc_add(db, kk * 2048), id, 1);
        mma_commit(bar(B_D));
        issued[B_D]++;
      }
      ok = wait_bar(bar(B_D), pk, abort_flag) && ok;
      tc_fence_after();
      if (vn_role) {
        // Vn decayed to the chunk end -> B operand of the state update (over the image)
        const float dec = m->decL[tl];
        float x[32];
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
          tmem_ld32(lane_base + TM_D + half * 64 + hh * 32, x);
#pragma unroll
          for (int j = 0; j < 32; ++j) x[j] *= dec;
#pragma unroll
          for (int q = 0; q < 4; ++q) st_half8(smem + OFF_S16 + half * 8192, swz(tl, hh * 4 + q), x + q * 8);
        }
        fence_proxy_async();
        tc_fence_before();
        ok = !bar_named_or(BAR_VN, 128, !ok);
        if (ct == 0 && ok) mbar_arrive(bar(B_DFREE));  // the new-value rows of D are read
        if (ct == 0 && ok) {  // S^T += K^T Vn_d; then the stage is free
          tc_fence_after();
          constexpr uint32_t id = idesc_f16(128, 128, true, true);
          const uint64_t da = sdesc_sw128(st + ST_KQ, 16384, 1024);
          const uint64_t db = sdesc_sw128(sb + OFF_S16, 8192, 1024);
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            mma_f16(tmem + TM_S, sdesc_add(da, kk * 2048), sdesc_add(db, kk * 2048), id, 1);
          mma_commit(bar(B_S));
          mma_commit(bar(B_FREE + s));
          issued[B_S]++;
        }
      } else {
        // O rows: token t = tl - 64, this thread's 64 value columns
        const int t = tl - 64;
        float o[64];
        tmem_ld32(lane_base + TM_D + half * 64, o);
        tmem_ld32(lane_base + TM_D + half * 64 + 32, o + 32);
        float ss = 0.f;
#pragma unroll
        for (int j = 0; j < 64; ++j) ss = fmaf(o[j], o[j], ss);
        float* sp = ssp + (ci & 1) * 128;
        sp[half * 64 + t] = ss;
        tc_fence_before();
        ok = !bar_named_or(BAR_O, 128, !ok);  // both halves' sums are in; D's O rows are read
        if (ct == 64 && ok) mbar_arrive(bar(B_DFREE));  // the O rows of D are read
        if (t < L && ok) {
          if (norm_out) {
            const float ri = rsqrtf((sp[t] + sp[64 + t]) * (1.0f / D) + p.eps_norm);
            const size_t row = ((size_t)(c0 + t) * p.Hv + h) * D + half * 64;
            const __nv_bfloat16* zr = static_cast<const __nv_bfloat16*>(p.z) + row;
            __nv_bfloat16* orow = static_cast<__nv_bfloat16*>(p.out) + row;
#pragma unroll
            for (int g8 = 0; g8 < 8; ++g8) {
              const uint4 zv = __ldg(reinterpret_cast<const uint4*>(zr + g8 * 8));
              const __nv_bfloat162* z2 = reinterpret_cast<const __nv_bfloat162*>(&zv);
              uint4 res;
              __nv_bfloat162* r2 = reinterpret_cast<__nv_bfloat162*>(&res);
#pragma unroll
              for (int e = 0; e < 4; ++e) {
                const float2 zf = __bfloat1622float2(z2[e]);
                const int j = g8 * 8 + 2 * e;
                const float w0 = wsm[half * 64 + j], w1 = wsm[half * 64 + j + 1];
                r2[e] = __floats2bfloat162_rn(o[j] * ri * w0 * silu_tanh(zf.x),
                                              o[j + 1] * ri * w1 * silu_tanh(zf.y));
              }
              *reinterpret_cast<uint4*>(orow + g8 * 8) = res;
            }
          } else {
            float* dst = p.o_raw + ((size_t)(c0 + t) * p.Hv + h) * D + half * 64;
#pragma unroll
            for (int q = 0; q < 16; ++q)
              *reinterpret_cast<float4*>(dst + q * 4) =
                  make_float4(o[4 * q], o[4 * q + 1], o[4 * q + 2], o[4 * q + 3]);
          }
        }
      }
      if (flags & F_LAST) {
        // the chain's final state
        ok = wait_bar(bar(B_S), pk, abort_flag) && ok;
        tc_fence_after();
        if (p.S_out && ok) {
#pragma unroll
          for (int hh = 0; hh < 2; ++hh) {
            const int col = half * 64 + hh * 32;
            float r[32];
            tmem_ld32(lane_base + TM_S + col, r);
#pragma unroll
            for (int j = 0; j < 32; ++j) p.S_out[sbase + (size_t)(col + j) * D + tl] = r[j];
          }
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    // every copy and tensor-core commit started by this CTA has landed
    // before TMEM is freed (at once unless a wait above gave up)
    if (lane == 0) {
      for (int i = 0; i < NBARS; ++i)
        if (issued[i] > 0 && i != B_FREE && i != B_FREE + 1 && i != B_READY && i != B_READY + 1 &&
            i != B_DFREE)
          mbar_wait(bar(i), (uint32_t)(issued[i] - 1) & 1u, 100000000ull);
    }
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, TM_COLS);
  }
}

// Queue order: sequences by decreasing length (ties by index), so that the
// longest chains start first; the chain counter starts at zero.  Beyond
// kFusedSortMax sequences the queue keeps index order.
__global__ void __launch_bounds__(kFusedSortMax) fused_order_kernel(const int32_t* cu, int N, int T, int* sched) {
  __shared__ int len[kFusedSortMax];
  const int tid = threadIdx.x;
  if (tid == 0) sched[0] = 0;
  int* order = sched + 1;
  if (N > kFusedSortMax) return;
  for (int i = tid; i < N; i += blockDim.x) {
    const int b = clampi(cu[i], 0, T);
    len[i] = clampi(cu[i + 1], b, T) - b;
  }
  __syncthreads();
  for (int i = tid; i < N; i += blockDim.x) {
    const int li = len[i];
    int rank = 0;
    for (int j = 0; j < N; ++j) rank += (len[j] > li || (len[j] == li && j < i)) ? 1 : 0;
    order[rank] = i;
  }
}

bool make_map(CUtensorMap* m, const void* base, uint64_t rows, uint64_t cols) {
  host::EncodeTiledFn fn = host::encode_tiled();
  if (!fn) return false;
  cuuint64_t dims[2] = {cols, rows};
  cuuint64_t strides[1] = {cols * 2};
  cuuint32_t box[2] = {64, 64};
  cuuint32_t es[2] = {1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, const_cast<void*>(base), dims, strides, box, es,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

cudaError_t launch_chunk_fused_order(const ChunkParams& p, int* sched, cudaStream_t st) {
  if (p.N == 0) return cudaSuccess;
  fused_order_kernel<<<1, kFusedSortMax, 0, st>>>(p.cu_seqlens, p.N, p.T, sched);
  return cudaGetLastError();
}

cudaError_t launch_chunk_fused(const ChunkParams& p, int* sched, cudaStream_t st) {
  if (p.N == 0 || p.Hv == 0) return cudaSuccess;
  if ((p.q_lo == nullptr) != (p.k_lo == nullptr) || !sched) return cudaErrorInvalidValue;
  CUtensorMap mq, mk, mv, mql, mkl;
  memset(&mq, 0, sizeof(mq));
  memset(&mk, 0, sizeof(mk));
  memset(&mv, 0, sizeof(mv));
  memset(&mql, 0, sizeof(mql));
  memset(&mkl, 0, sizeof(mkl));
  if (p.T > 0) {
    if (!make_map(&mq, p.q, (uint64_t)p.T, (uint64_t)p.Hk * D) ||
        !make_map(&mk, p.k, (uint64_t)p.T, (uint64_t)p.Hk * D) ||
        !make_map(&mv, p.v, (uint64_t)p.T, (uint64_t)p.Hv * D))
      return cudaErrorInvalidValue;
    if (p.k_lo && (!make_map(&mql, p.q_lo, (uint64_t)p.T, (uint64_t)p.Hk * D) ||
                   !make_map(&mkl, p.k_lo, (uint64_t)p.T, (uint64_t)p.Hk * D)))
      return cudaErrorInvalidValue;
  }
  cudaError_t e = cudaFuncSetAttribute(chunk_fused_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)SMEM_BYTES);
  if (e != cudaSuccess) return e;
  const long chains = (long)p.N * p.Hv;
  const int ctas = (int)(chains < host::sm_count() ? chains : host::sm_count());
  FusedArgs fa;
  fa.p = p;
  fa.order = p.N <= kFusedSortMax ? sched + 1 : nullptr;
  fa.queue = sched;
  cudaLaunchConfig_t cfg;
  memset(&cfg, 0, sizeof(cfg));
  cfg.gridDim = dim3((unsigned)ctas, 1, 1);
  cfg.blockDim = dim3(NTHREADS, 1, 1);
  cfg.dynamicSmemBytes = SMEM_BYTES;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;  // see pdl_wait
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, chunk_fused_kernel, mq, mk, mv, mql, mkl, fa);
}

int fused_error_word(int clear) {
  int v = 0;
  if (cudaMemcpyFromSymbol(&v, g_fused_error, sizeof(int)) != cudaSuccess) return -1;
  if (clear && v != 0) {
    const int zero = 0;
    if (cudaMemcpyToSymbol(g_fused_error, &zero, sizeof(int)) != cudaSuccess) return -1;
  }
  return v;
}

}  // namespace gdn
