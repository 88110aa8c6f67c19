// Pieces shared by the tensor-core chunked kernels (chunk_tc.cu, chunk_tc_split.cu).
#pragma once

#include <cuda_fp16.h>
#include <stdint.h>

namespace gdn {
namespace tcc {

constexpr int AS = 68;  // row stride (floats) of the fp32 A and T matrices: 16-byte aligned rows
constexpr int ES = 65;  // row stride of the decay table E (conflict-free row walks)

// Eight floats -> eight fp16 values -> one 16-byte store at base + off.
__device__ __forceinline__ void st_half8(uint8_t* base, uint32_t off, const float* f) {
  uint4 u;
  __half2* h = reinterpret_cast<__half2*>(&u);
#pragma unroll
  for (int i = 0; i < 4; ++i) h[i] = __floats2half2_rn(f[2 * i], f[2 * i + 1]);
  *reinterpret_cast<uint4*>(base + off) = u;
}

// Barrier over the NT threads that run a shared step: the whole CTA
// (BAR == 0), or named barrier BAR when those threads are one role of a
// larger CTA.
template <int NT, int BAR>
__device__ __forceinline__ void role_sync() {
  if constexpr (BAR == 0)
    __syncthreads();
  else
    asm volatile("bar.sync %0, %1;" ::"n"(BAR), "n"(NT) : "memory");
}

// Tf := (I + A)^-1 for the strictly lower triangular 64 x 64 A (fp32, row
// stride AS), by recursive doubling of the block size:
//   16 x 16 diagonal blocks by forward substitution (one column per thread);
//   32 x 32: T_{r,r-1} = -T_rr A_{r,r-1} T_{r-1,r-1} for the 16-blocks (1,0), (3,2);
//   64 x 64: T_{LL}   = -T_bb A_{LL} T_tt for the lower-left 32-block.
// Every product step gives each thread independent accumulators.
template <int NT, int BAR = 0>
__device__ __forceinline__ void solve_unit_lower(const float* Af, float* Tf, float* X, int tid) {
  constexpr int NW = NT / 32;
  const int warp = tid >> 5, lane = tid & 31;
  if (tid < 64) {
    const int b = tid >> 4, m = tid & 15;
    float x[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      float a0 = (i == m) ? 1.f : 0.f, a1 = 0.f;
#pragma unroll
      for (int j = 0; j < i; j += 2) {
        a0 = fmaf(-Af[(16 * b + i) * AS + 16 * b + j], x[j], a0);
        if (j + 1 < i) a1 = fmaf(-Af[(16 * b + i) * AS + 16 * b + j + 1], x[j + 1], a1);
      }
      x[i] = a0 + a1;
    }
#pragma unroll
    for (int i = 0; i < 16; ++i) Tf[(16 * b + i) * AS + 16 * b + m] = x[i];
  } else {
    // 16-blocks above the diagonal are zero
    for (int e = tid - 64; e < 6 * 256; e += NT - 64) {
      const int blk = e >> 8, w = e & 255, i = w >> 4, m = w & 15;
      const int r = blk < 3 ? 0 : (blk < 5 ? 1 : 2);
      const int c = blk < 3 ? blk + 1 : (blk < 5 ? blk - 1 : 3);
      Tf[(16 * r + i) * AS + 16 * c + m] = 0.f;
    }
  }
  role_sync<NT, BAR>();
  // 32 x 32 diagonal blocks: element e = tid + NT k -> 16-block (r, r-1), r = 1 or 3
  constexpr int K1 = 512 / NT;
  {
    float acc[K1];
#pragma unroll
    for (int k = 0; k < K1; ++k) acc[k] = 0.f;
#pragma unroll
    for (int j = 0; j < 16; ++j) {
#pragma unroll
      for (int k = 0; k < K1; ++k) {
        const int e = tid + NT * k, r = (e >> 8) ? 3 : 1, i = (e >> 4) & 15, m = e & 15;
        acc[k] = fmaf(Af[(16 * r + i) * AS + 16 * (r - 1) + j],
                      Tf[(16 * (r - 1) + j) * AS + 16 * (r - 1) + m], acc[k]);
      }
    }
#pragma unroll
    for (int k = 0; k < K1; ++k) X[tid + NT * k] = acc[k];
  }
  role_sync<NT, BAR>();
  {
    float acc[K1];
#pragma unroll
    for (int k = 0; k < K1; ++k) acc[k] = 0.f;
#pragma unroll
    for (int j = 0; j < 16; ++j) {
#pragma unroll
      for (int k = 0; k < K1; ++k) {
        const int e = tid + NT * k, blk = e >> 8, r = blk ? 3 : 1, i = (e >> 4) & 15, m = e & 15;
        acc[k] = fmaf(Tf[(16 * r + i) * AS + 16 * r + j], X[blk * 256 + j * 16 + m], acc[k]);
      }
    }
#pragma unroll
    for (int k = 0; k < K1; ++k) {
      const int e = tid + NT * k, r = (e >> 8) ? 3 : 1, i = (e >> 4) & 15, m = e & 15;
      Tf[(16 * r + i) * AS + 16 * (r - 1) + m] = -acc[k];
    }
  }
  role_sync<NT, BAR>();
  // 64 x 64: rows 32 + warp + NW k of the lower-left block, column `lane`
  constexpr int K2 = 32 / NW;
  {
    float acc[K2];
#pragma unroll
    for (int k = 0; k < K2; ++k) acc[k] = 0.f;
#pragma unroll 2
    for (int j = 0; j < 32; j += 4) {
      float t[4];
#pragma unroll
      for (int q = 0; q < 4; ++q) t[q] = Tf[(j + q) * AS + lane];
#pragma unroll
      for (int k = 0; k < K2; ++k) {
        const float4 a4 = *reinterpret_cast<const float4*>(Af + (32 + warp + NW * k) * AS + j);
        acc[k] = fmaf(a4.x, t[0], fmaf(a4.y, t[1], fmaf(a4.z, t[2], fmaf(a4.w, t[3], acc[k]))));
      }
    }
#pragma unroll
    for (int k = 0; k < K2; ++k) X[(warp + NW * k) * 32 + lane] = acc[k];
  }
  role_sync<NT, BAR>();
  {
    float acc[K2];
#pragma unroll
    for (int k = 0; k < K2; ++k) acc[k] = 0.f;
#pragma unroll 2
    for (int j = 0; j < 32; j += 4) {
      float x[4];
#pragma unroll
      for (int q = 0; q < 4; ++q) x[q] = X[(j + q) * 32 + lane];
#pragma unroll
      for (int k = 0; k < K2; ++k) {
        const float4 t4 = *reinterpret_cast<const float4*>(Tf + (32 + warp + NW * k) * AS + 32 + j);
        acc[k] = fmaf(t4.x, x[0], fmaf(t4.y, x[1], fmaf(t4.z, x[2], fmaf(t4.w, x[3], acc[k]))));
      }
    }
#pragma unroll
    for (int k = 0; k < K2; ++k) Tf[(32 + warp + NW * k) * AS + lane] = -acc[k];
  }
  role_sync<NT, BAR>();
}


}  // namespace tcc
}  // namespace gdn
