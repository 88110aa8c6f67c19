// The dense projections around the mixer on the tensor cores: Y = X W^T with
// X [M, K] and W [N, K] in bf16 (W in the [out, in] layout of the layer's
// weights), fp32 accumulation in TMEM, bf16 results.  The layer applies four
// input projections to the hidden states -- in_proj_qkv, in_proj_z,
// in_proj_b, in_proj_a -- and out_proj to the gated-norm output
// ("Qwen/Qwen3.5-9B", module tree of a Gated DeltaNet block).  The input
// projections run as one product over their stacked weights; the epilogue
// routes consecutive column ranges of Y to separate outputs, so the mixer's
// inputs mixed_qkv, z, a and b are written where gdn_prefill reads them.
//
// One persistent CTA per SM walks 128 x 256 output tiles (in groups of row
// blocks, see tile_origin):
//   warp 0      streams 128 x 64 X tiles and 256 x 64 W tiles by TMA (128-byte
//               swizzle, no multicast) into a ring of four stages;
//   warp 1      issues the tcgen05 MMAs (M = 128, N = 256, K = 16) of a tile
//               into one of two TMEM accumulators and releases each stage when
//               its MMAs complete;
//   warps 2..5  read the other accumulator (one TMEM lane quarter each),
//               round to bf16 and store, while the next tile accumulates.
// Every wait is bounded; a wait that gives up records it in the error word.
#include <cuda.h>
#include <string.h>

#include "gdn_internal.h"
#include "host_util.h"
#include "tc_ptx.cuh"

namespace gdn {

__device__ int g_linear_error = 0;  // nonzero: a bounded wait of the projection kernel gave up

namespace {

using namespace ptx;

constexpr int BM = 128, BN = 256, BK = 64;
constexpr int NSTAGE = 4;
constexpr uint32_t A_BYTES = BM * BK * 2;             // 16 KiB
constexpr uint32_t B_BYTES = BN * BK * 2;             // 32 KiB
constexpr uint32_t STAGE_BYTES = A_BYTES + B_BYTES;
constexpr uint32_t OFF_BAR = NSTAGE * STAGE_BYTES;    // full[4], empty[4], acc_full[2], acc_empty[2]
constexpr uint32_t OFF_TMEM = OFF_BAR + 12 * 8;
constexpr uint32_t SMEM_BYTES = OFF_TMEM + 16 + 1024;
constexpr int NTHREADS = 192;
constexpr uint32_t TM_COLS = 512;                     // two 256-column fp32 accumulators
static_assert(SMEM_BYTES <= 232448, "shared memory");

// Instruction descriptor of tcgen05.mma kind::f16 with bf16 A and B (both
// K-major) and an fp32 accumulator.
__host__ __device__ constexpr uint32_t idesc_bf16(int M, int N) {
  return (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}

// Output tile of a tile index.  Tiles run down a group of kGroupRows row
// blocks before moving one column block on, so the CTAs working at one time
// share a few X row blocks and a few W column blocks in L2 and each W tile is
// read from DRAM about once per group instead of once per row block.
constexpr int kGroupRows = 16;
__device__ __forceinline__ void tile_origin(int tile, const LinearParams& p, int& m0, int& n0) {
  const int per_group = kGroupRows * p.tiles_n;
  const int g = tile / per_group, r = tile - g * per_group;
  const int rows = min(kGroupRows, p.tiles_m - g * kGroupRows);
  m0 = (g * kGroupRows + r % rows) * BM;
  n0 = (r / rows) * BN;
}

__device__ __forceinline__ bool wait_lin(uint32_t bar, uint32_t parity) {
  if (mbar_wait(bar, parity)) return true;
  atomicExch(&g_linear_error, 1);
  return false;
}

__global__ void __launch_bounds__(NTHREADS, 1)
    linear_tc_kernel(const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_w,
                     const LinearParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  const uint32_t sb = smem_u32(smem);
  const uint32_t full = sb + OFF_BAR, empty = full + 8 * NSTAGE, acc_full = empty + 8 * NSTAGE,
                 acc_empty = acc_full + 16;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + OFF_TMEM);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

  if (tid == 0) {
    for (int s = 0; s < NSTAGE; ++s) {
      mbar_init(full + 8 * s, 1);
      mbar_init(empty + 8 * s, 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(acc_full + 8 * b, 1);
      mbar_init(acc_empty + 8 * b, 128);  // every epilogue thread
    }
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
  pdl_wait();  // X may come from the kernel launched before this one

  const int n_tiles = p.tiles_m * p.tiles_n;
  const int kiters = p.K / BK;
  // A failed wait stops the role; the others then give up at their own
  // bounded waits.  Before TMEM is freed, thread 0 lets every copy and MMA this
  // CTA started land (bounded again).
  int issued_loads = 0;
  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      int it = 0;
      bool ok = true;
      for (int tile = blockIdx.x; tile < n_tiles && ok; tile += gridDim.x) {
        int m0, n0;
        tile_origin(tile, p, m0, n0);
        for (int k = 0; k < kiters; ++k, ++it) {
          const int s = it % NSTAGE;
          if (it >= NSTAGE && !(ok = wait_lin(empty + 8 * s, (uint32_t)((it / NSTAGE) - 1) & 1u))) break;
          const uint32_t st = sb + s * STAGE_BYTES;
          mbar_arrive_expect_tx(full + 8 * s, STAGE_BYTES);
          tma_load_2d(st, &tm_x, k * BK, m0, full + 8 * s);
          tma_load_2d(st + A_BYTES, &tm_w, k * BK, n0, full + 8 * s);
          ++issued_loads;
        }
      }
      // the last copies land before the CTA may leave
      for (int k = 1; k <= NSTAGE && it - k >= 0 && issued_loads > 0; ++k)
        mbar_wait(full + 8 * ((it - k) % NSTAGE), (uint32_t)((it - k) / NSTAGE) & 1u, 100000000ull);
    }
  } else if (warp == 1) {
    // ----------------------------------------------------------------- MMA
    if (lane == 0) {
      int it = 0, tc = 0;
      bool ok = true;
      constexpr uint32_t id = idesc_bf16(BM, BN);
      for (int tile = blockIdx.x; tile < n_tiles && ok; tile += gridDim.x, ++tc) {
        const int b = tc & 1;
        if (tc >= 2 && !(ok = wait_lin(acc_empty + 8 * b, (uint32_t)((tc >> 1) - 1) & 1u))) break;
        tc_fence_after();
        for (int k = 0; k < kiters; ++k, ++it) {
          const int s = it % NSTAGE;
          if (!(ok = wait_lin(full + 8 * s, (uint32_t)(it / NSTAGE) & 1u))) break;
          tc_fence_after();
          const uint32_t st = sb + s * STAGE_BYTES;
          const uint64_t da = sdesc_sw128(st, 16, 1024);
          const uint64_t db = sdesc_sw128(st + A_BYTES, 16, 1024);
#pragma unroll
          for (int kk = 0; kk < BK / 16; ++kk)
            mma_f16(tmem + b * BN, sdesc_add(da, kk * 32), sdesc_add(db, kk * 32), id, (k | kk) != 0);
          mma_commit(empty + 8 * s);  // the stage is free once these MMAs have read it
        }
        if (!ok) break;
        mma_commit(acc_full + 8 * b);
      }
      if (it > 0)  // every MMA this thread issued has completed before the CTA may leave
        mbar_wait(empty + 8 * ((it - 1) % NSTAGE), (uint32_t)((it - 1) / NSTAGE) & 1u, 100000000ull);
    }
  } else {
    // ------------------------------------------------------------ epilogue
    const int q = warp & 3;  // TMEM lane quarter: tile rows 32 q .. 32 q + 31
    const uint32_t lane_base = tmem + ((uint32_t)(q * 32) << 16);
    int tc = 0;
    for (int tile = blockIdx.x; tile < n_tiles; tile += gridDim.x, ++tc) {
      const int b = tc & 1;
      int m0, n0;
      tile_origin(tile, p, m0, n0);
      // the whole warp leaves together: tcgen05.ld below is warp-collective
      if (!__all_sync(0xffffffffu, wait_lin(acc_full + 8 * b, (uint32_t)(tc >> 1) & 1u))) break;
      tc_fence_after();
      const int row = m0 + q * 32 + lane;
#pragma unroll 1
      for (int c = 0; c < BN / 32; ++c) {
        float v[32];
        tmem_ld32(lane_base + b * BN + c * 32, v);
        const int col0 = n0 + c * 32;
        if (row < p.M && col0 < p.N) {
#pragma unroll
          for (int g = 0; g < 4; ++g) {
            const int col = col0 + g * 8;
            if (col >= p.N) break;
            // the output range holding columns col .. col + 7 (ranges are multiples of 8)
            int o = 0, base = 0;
            while (o + 1 < p.n_out && col >= base + p.out_cols[o]) base += p.out_cols[o++];
            uint4 u;
            __nv_bfloat162* h = reinterpret_cast<__nv_bfloat162*>(&u);
#pragma unroll
            for (int e = 0; e < 4; ++e) h[e] = __floats2bfloat162_rn(v[g * 8 + 2 * e], v[g * 8 + 2 * e + 1]);
            __nv_bfloat16* dst = static_cast<__nv_bfloat16*>(p.out[o]) + (size_t)row * p.out_ld[o] + (col - base);
            *reinterpret_cast<uint4*>(dst) = u;
          }
        }
      }
      tc_fence_before();
      mbar_arrive(acc_empty + 8 * b);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, TM_COLS);
  }
}

bool make_map(CUtensorMap* m, const void* base, uint64_t rows, uint64_t cols, uint64_t ld, uint32_t box_rows) {
  host::EncodeTiledFn fn = host::encode_tiled();
  if (!fn) return false;
  cuuint64_t dims[2] = {cols, rows};
  cuuint64_t strides[1] = {ld * 2};
  cuuint32_t box[2] = {(cuuint32_t)BK, box_rows};
  cuuint32_t es[2] = {1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, es,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

cudaError_t launch_linear_tc(const LinearParams& p0, const void* x, int ldx, const void* w, int ldw,
                             cudaStream_t st) {
  if (p0.M == 0) return cudaSuccess;
  LinearParams p = p0;
  p.tiles_m = (p.M + BM - 1) / BM;
  p.tiles_n = (p.N + BN - 1) / BN;
  CUtensorMap mx, mw;
  memset(&mx, 0, sizeof(mx));
  memset(&mw, 0, sizeof(mw));
  if (!make_map(&mx, x, (uint64_t)p.M, (uint64_t)p.K, (uint64_t)ldx, BM) ||
      !make_map(&mw, w, (uint64_t)p.N, (uint64_t)p.K, (uint64_t)ldw, BN))
    return cudaErrorInvalidValue;
  cudaError_t e = cudaFuncSetAttribute(linear_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)SMEM_BYTES);
  if (e != cudaSuccess) return e;
  const int tiles = p.tiles_m * p.tiles_n;
  const int ctas = tiles < host::sm_count() ? tiles : host::sm_count();
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
  return cudaLaunchKernelEx(&cfg, linear_tc_kernel, mx, mw, p);
}

int linear_error_word(int clear) {
  int v = 0;
  if (cudaMemcpyFromSymbol(&v, g_linear_error, sizeof(int)) != cudaSuccess) return -1;
  if (clear && v != 0) {
    const int zero = 0;
    if (cudaMemcpyToSymbol(g_linear_error, &zero, sizeof(int)) != cudaSuccess) return -1;
  }
  return v;
}

}  // namespace gdn
