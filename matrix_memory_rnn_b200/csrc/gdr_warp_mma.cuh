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

// acc += A[r0 .. r0+16, k0 .. k1) B[k0 .. k1, c0 .. c0+32); A(m, k), B(k, n) accessors.
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
