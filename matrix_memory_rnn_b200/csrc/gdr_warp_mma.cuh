// gdr_warp_mma.cuh -- warp-level tf32 tensor-core products on fp32 tiles (mma.sync
// m16n8k8, fp32 accumulate), used by the reverse mode and the mLSTM kernels: a warp
// computes a 16 x 32 output tile from two accessor functions A(m, k) and B(k, n).  With
// kSplit each operand is split into tf32 high and low parts and three products are
// accumulated (hi*hi + hi*lo + lo*hi), which keeps fp32 accuracy for fp32 inputs.
#pragma once

#include "gdr_tc_common.cuh"

namespace gdr {
namespace wmma_tf32 {

using tc::mma_tf32_16x8x8;
using tc::to_tf32;

// Warp tile: 16 rows x 32 columns (four m16n8 MMA tiles), acc[i][e] at
// row r0 + g + 8 (e >> 1), column c0 + 8 i + 2 t + (e & 1)  (lane = 4 g + t).
template <bool kSplit>
__device__ __forceinline__ void split_tf32(float x, uint32_t &hi, uint32_t &lo) {
  hi = to_tf32(x);
  lo = kSplit ? to_tf32(x - __uint_as_float(hi)) : 0u;
}

// An operand value that tf32 holds exactly (a widened bf16: 8 exponent bits, 7 mantissa
// bits), so it enters the MMA as it is, with no rounding step and no low part.
struct Tf32Exact {
  float x;
};
__device__ __forceinline__ Tf32Exact tf32_exact(__nv_bfloat16 v) { return {__bfloat162float(v)}; }
__device__ __forceinline__ float tf32_exact(float v) { return v; }
template <bool kSplit>
__device__ __forceinline__ void split_tf32(Tf32Exact v, uint32_t &hi, uint32_t &lo) {
  hi = __float_as_uint(v.x);
  lo = 0u;
}

// acc += A[r0 .. r0+16, k0 .. k1) B[k0 .. k1, c0 .. c0+32); A(m, k), B(k, n) accessors
// returning float (rounded to tf32 here) or Tf32Exact.
template <bool kSplit, class FA, class FB>
__device__ __forceinline__ void mma_seg(float (&acc)[4][4], int r0, int c0, int k0, int k1,
                                        const FA &A, const FB &B, int lane) {
  const int g = lane >> 2, t = lane & 3;
  for (int k = k0; k < k1; k += 8) {
    uint32_t ah[4], al[4];
    split_tf32<kSplit>(A(r0 + g, k + t), ah[0], al[0]);
    split_tf32<kSplit>(A(r0 + g + 8, k + t), ah[1], al[1]);
    split_tf32<kSplit>(A(r0 + g, k + t + 4), ah[2], al[2]);
    split_tf32<kSplit>(A(r0 + g + 8, k + t + 4), ah[3], al[3]);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      uint32_t bh0, bl0, bh1, bl1;
      split_tf32<kSplit>(B(k + t, c0 + 8 * i + g), bh0, bl0);
      split_tf32<kSplit>(B(k + t + 4, c0 + 8 * i + g), bh1, bl1);
      if (kSplit) {
        mma_tf32_16x8x8(acc[i], al[0], al[1], al[2], al[3], bh0, bh1);
        mma_tf32_16x8x8(acc[i], ah[0], ah[1], ah[2], ah[3], bl0, bl1);
      }
      mma_tf32_16x8x8(acc[i], ah[0], ah[1], ah[2], ah[3], bh0, bh1);
    }
  }
}

// acc += A[r0 .. r0+16, k0 .. k1) Bt[c0 .. c0+32, k0 .. k1)^T for bf16 tiles in shared
// memory, A and Bt row-major with row strides lda, ldb (elements; rows 16-byte aligned):
// m16n8k16 bf16 MMAs fed by ldmatrix, the same accumulator layout as mma_seg.  A product
// of two bf16 values is exact in fp32, so this equals the tf32 product of the same tiles.
// k1 - k0 a multiple of 16.
__device__ __forceinline__ void mma_bf16_abt(float (&acc)[4][4], const __nv_bfloat16 *A, int lda,
                                             const __nv_bfloat16 *Bt, int ldb, int r0, int c0, int k0,
                                             int k1, int lane) {
  // ldmatrix x4 row addresses: A, the 16 x 16 block as (rows 0-7 | 8-15) x (k 0-7 | 8-15);
  // Bt, two 8-column tiles as (tile i, k 0-7), (tile i, k 8-15), (tile i+1, k 0-7), ...
  const uint32_t a_addr = sm100::smem_u32(A + (size_t)(r0 + (lane & 15)) * lda + k0 + (lane >> 4) * 8);
  const int mat = lane >> 3;
  const uint32_t b_addr = sm100::smem_u32(Bt + (size_t)(c0 + 8 * (mat >> 1) + (lane & 7)) * ldb + k0 +
                                          8 * (mat & 1));
  const uint32_t b_tiles = 16u * (uint32_t)ldb * 2u;   // bytes between tile pairs (16 rows)
  for (int k = 0; k < k1 - k0; k += 16) {
    uint32_t a[4], b[2][4];
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
                 : "=r"(a[0]), "=r"(a[1]), "=r"(a[2]), "=r"(a[3])
                 : "r"(a_addr + 2u * k));
#pragma unroll
    for (int p = 0; p < 2; ++p)
      asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
                   : "=r"(b[p][0]), "=r"(b[p][1]), "=r"(b[p][2]), "=r"(b[p][3])
                   : "r"(b_addr + p * b_tiles + 2u * k));
#pragma unroll
    for (int i = 0; i < 4; ++i)
      asm volatile(
          "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
          "{%8,%9}, {%0,%1,%2,%3};"
          : "+f"(acc[i][0]), "+f"(acc[i][1]), "+f"(acc[i][2]), "+f"(acc[i][3])
          : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b[i >> 1][2 * (i & 1)]),
            "r"(b[i >> 1][2 * (i & 1) + 1]));
  }
}

__device__ __forceinline__ void zero_acc(float (&acc)[4][4]) {
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int e = 0; e < 4; ++e) acc[i][e] = 0.f;
}

template <class F>
__device__ __forceinline__ void for_acc(const float (&acc)[4][4], int r0, int c0, int lane,
                                        const F &f) {
  const int g = lane >> 2, t = lane & 3;
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int e = 0; e < 4; ++e) f(r0 + g + 8 * (e >> 1), c0 + 8 * i + 2 * t + (e & 1), acc[i][e]);
}

}  // namespace wmma_tf32
}  // namespace gdr
