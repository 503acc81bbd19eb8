// gdr_tc_common.cuh -- pieces shared by the tensor-core forward kernels
// (gdr_fwd_tc.cu, gdr_fwd_tc_split.cu): sizes, bf16 packing, the bounded MMA
// wait, and the fp32 blocked inverse of the chunk's unit lower-triangular T.
#pragma once

#include "gdr_internal.cuh"
#include "gdr_sm100.cuh"

namespace gdr {
namespace tc {

using namespace sm100;

constexpr int kC = 64;
constexpr int kDK = 128;
constexpr int kThreads = 256;
constexpr float kMaxChunkDecay = 80.f;        // nats
constexpr uint64_t kWaitLimitNs = 2000000000ull;
constexpr uint32_t kTmemCols = 256;

__device__ __forceinline__ uint4 ld16(const __nv_bfloat16 *p) {
  return __ldg(reinterpret_cast<const uint4 *>(p));
}

__device__ __forceinline__ void unpack8(const uint4 &u, float (&f)[8]) {
  const __nv_bfloat162 *h = reinterpret_cast<const __nv_bfloat162 *>(&u);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float2 x = __bfloat1622float2(h[i]);
    f[2 * i] = x.x;
    f[2 * i + 1] = x.y;
  }
}

__device__ __forceinline__ uint32_t pack2(float a, float b) {
  __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
  return *reinterpret_cast<uint32_t *>(&h);
}

__device__ __forceinline__ uint4 pack8(const float *f) {
  return make_uint4(pack2(f[0], f[1]), pack2(f[2], f[3]), pack2(f[4], f[5]), pack2(f[6], f[7]));
}

__device__ __forceinline__ void st_smem16(uint8_t *base, uint32_t off, const uint4 &v) {
  *reinterpret_cast<uint4 *>(base + off) = v;
}

// Bounded wait for the MMA group committed to `bar`: thread 0 polls the
// mbarrier, then a CTA barrier passes the completion on (and makes every thread
// take the same branch).  Returns false, with the shared abort flag set, when the
// wait ran out.
__device__ __forceinline__ bool wait_mma(uint64_t *bar, uint32_t &phase, volatile int *abort) {
  if (threadIdx.x == 0 && *abort == 0 && !mbar_wait_bounded(bar, phase, kWaitLimitNs)) *abort = 1;
  phase ^= 1u;
  __syncthreads();
  tc_fence_after();
  return *abort == 0;
}

// T^-1 for the unit lower-triangular T = I + L (L strictly lower, fp32; element
// (r, s) of L at Lm[IxL::at(r, s)], of T^-1 at Ti[IxT::at(r, s)]), by blocks (eq. (11) of the Muir page): the four 16 x 16 diagonal blocks by
// forward substitution, then two merge levels X21 = -T_R^-1 (L_RL T_L^-1).  Writes
// all of Ti (zeros above the diagonal); overwrites the merged L_RL blocks of Lm
// with the products L_RL T_L^-1.  All 256 threads; ends with a CTA barrier.
template <class IxL, class IxT>
__device__ void invert_unit_lower(float *Lm, float *Ti, int tid) {
  if (tid < 64) {
    const int blk = tid >> 4, c = tid & 15, o = 16 * blk;
    float x[16];
#pragma unroll
    for (int t = 0; t < 16; ++t) {
      float acc = (t == c) ? 1.f : 0.f;
#pragma unroll
      for (int s = 0; s < t; ++s) acc -= Lm[IxL::at(o + t, o + s)] * x[s];
      x[t] = acc;
    }
#pragma unroll
    for (int t = 0; t < 16; ++t) Ti[IxT::at(o + t, o + c)] = x[t];
  } else {
    // zero the strictly-upper blocks the merge products read
    for (int i = tid - 64; i < 32 * 32 + 2 * 16 * 16; i += kThreads - 64) {
      int r, c;
      if (i < 1024) { r = i >> 5; c = 32 + (i & 31); }
      else { const int k = i - 1024, p = k >> 8; r = 32 * p + ((k >> 4) & 15); c = 32 * p + 16 + (k & 15); }
      Ti[IxT::at(r, c)] = 0.f;
    }
  }
  __syncthreads();
  // level 1: pairs (blocks 0,1) and (2,3).  Thread: pair p, row i, columns 2jq, 2jq+1.
  {
    const int p = tid >> 7, i = (tid >> 3) & 15, j = 2 * (tid & 7), o = 32 * p;
    float w0 = 0.f, w1 = 0.f;
#pragma unroll
    for (int k = 0; k < 16; ++k) {
      const float l = Lm[IxL::at(o + 16 + i, o + k)];
      const float2 t = *reinterpret_cast<const float2 *>(Ti + IxT::at(o + k, o + j));
      w0 += l * t.x;
      w1 += l * t.y;
    }
    __syncthreads();
    *reinterpret_cast<float2 *>(Lm + IxL::at(o + 16 + i, o + j)) = make_float2(w0, w1);
    __syncthreads();
    float x0 = 0.f, x1 = 0.f;
#pragma unroll
    for (int k = 0; k < 16; ++k) {
      const float t = Ti[IxT::at(o + 16 + i, o + 16 + k)];
      const float2 w = *reinterpret_cast<const float2 *>(Lm + IxL::at(o + 16 + k, o + j));
      x0 += t * w.x;
      x1 += t * w.y;
    }
    *reinterpret_cast<float2 *>(Ti + IxT::at(o + 16 + i, o + j)) = make_float2(-x0, -x1);
  }
  __syncthreads();
  // level 2: rows 32..63 x columns 0..31.  Thread: row i, columns 4jq .. 4jq+3.
  {
    const int i = tid >> 3, j = 4 * (tid & 7);
    float4 w = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
    for (int k = 0; k < 32; ++k) {
      const float l = Lm[IxL::at(32 + i, k)];
      const float4 t = *reinterpret_cast<const float4 *>(Ti + IxT::at(k, j));
      w.x += l * t.x; w.y += l * t.y; w.z += l * t.z; w.w += l * t.w;
    }
    __syncthreads();
    *reinterpret_cast<float4 *>(Lm + IxL::at(32 + i, j)) = w;
    __syncthreads();
    float4 x = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
    for (int k = 0; k < 32; ++k) {
      const float t = Ti[IxT::at(32 + i, 32 + k)];
      const float4 v = *reinterpret_cast<const float4 *>(Lm + IxL::at(32 + k, j));
      x.x += t * v.x; x.y += t * v.y; x.z += t * v.z; x.w += t * v.w;
    }
    *reinterpret_cast<float4 *>(Ti + IxT::at(32 + i, j)) = make_float4(-x.x, -x.y, -x.z, -x.w);
  }
  __syncthreads();
}


// Row-major C x C fp32 storage for invert_unit_lower: padded rows (68 floats, 16-byte
// aligned, conflict-free column writes) or exactly 64 floats with the 16-byte
// groups of row r XOR-permuted by (r & 15) (same properties, no padding).
struct PaddedIdx {
  static constexpr int kBytes = kC * (kC + 4) * 4;
  static __device__ __forceinline__ int at(int r, int s) { return r * (kC + 4) + s; }
};
struct SwizzledIdx {
  static constexpr int kBytes = kC * kC * 4;
  static __device__ __forceinline__ int at(int r, int s) {
    return r * kC + ((((s >> 2) ^ (r & 15))) << 2) + (s & 3);
  }
};

}  // namespace tc
}  // namespace gdr
