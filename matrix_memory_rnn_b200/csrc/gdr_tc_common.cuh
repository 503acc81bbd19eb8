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


// fp32 -> tf32 (round to nearest, ties away), as the operand of mma.sync .tf32.
__device__ __forceinline__ uint32_t to_tf32(float x) {
  uint32_t r;
  asm("cvt.rna.tf32.f32 %0, %1;" : "=r"(r) : "f"(x));
  return r;
}

// d += a (16 x 8, row-major) * b (8 x 8), tf32 operands, fp32 accumulate; warp-wide.
// Fragments (lane = 4 g + t): a0 (g, t) a1 (g+8, t) a2 (g, t+4) a3 (g+8, t+4);
// b0 (k = t, n = g) b1 (k = t+4, n = g); d0 (g, 2t) d1 (g, 2t+1) d2 (g+8, 2t) d3 (g+8, 2t+1).
__device__ __forceinline__ void mma_tf32_16x8x8(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                                uint32_t a3, uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k8.row.col.f32.tf32.tf32.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
      "{%8,%9}, {%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// One 16 x 8 tile of D = A B with A (16 x K) at rows r0.., columns k0.. of X (index
// IxA) and B (K x 8) at rows kb.., columns n0.. of Y (index IxB); K a multiple of 8.
template <class IxA, class IxB, int K>
__device__ __forceinline__ void tile_16x8(float (&d)[4], const float *X, int r0, int k0,
                                          const float *Y, int kb, int n0, int lane) {
  const int g = lane >> 2, t = lane & 3;
#pragma unroll
  for (int ks = 0; ks < K; ks += 8) {
    mma_tf32_16x8x8(d, to_tf32(X[IxA::at(r0 + g, k0 + ks + t)]), to_tf32(X[IxA::at(r0 + g + 8, k0 + ks + t)]),
                    to_tf32(X[IxA::at(r0 + g, k0 + ks + t + 4)]),
                    to_tf32(X[IxA::at(r0 + g + 8, k0 + ks + t + 4)]),
                    to_tf32(Y[IxB::at(kb + ks + t, n0 + g)]), to_tf32(Y[IxB::at(kb + ks + t + 4, n0 + g)]));
  }
}

// Stores a 16 x 8 tile (times `sign`) at rows r0.., columns n0.. of Z (index IxZ).
template <class IxZ>
__device__ __forceinline__ void store_16x8(const float (&d)[4], float sign, float *Z, int r0, int n0,
                                           int lane) {
  const int g = lane >> 2, t = lane & 3;
  *reinterpret_cast<float2 *>(Z + IxZ::at(r0 + g, n0 + 2 * t)) = make_float2(sign * d[0], sign * d[1]);
  *reinterpret_cast<float2 *>(Z + IxZ::at(r0 + g + 8, n0 + 2 * t)) = make_float2(sign * d[2], sign * d[3]);
}

// T^-1 for T = I + L as invert_unit_lower (same blocks, same merge order), for a
// CTA of NT threads, with the merge products X21 = -T_R^-1 (L_RL T_L^-1) on the
// tensor cores as warp-level tf32 MMAs (16 x 8 tiles, fp32 accumulate): the
// diagonal 16 x 16 blocks stay fp32 forward substitution.  Ends with a CTA barrier.
// Barrier policies for the helpers below: the whole CTA, or a named barrier shared
// by one group of N threads (warp-specialised kernels).
struct CtaSync {
  static __device__ __forceinline__ void sync() { __syncthreads(); }
};
template <int ID, int N>
struct GroupSync {
  static __device__ __forceinline__ void sync() {
    asm volatile("bar.sync %0, %1;" ::"n"(ID), "n"(N) : "memory");
  }
  // Barrier that also returns, to every thread of the group, the OR of `v` over it.
  static __device__ __forceinline__ bool sync_or(bool v) {
    uint32_t r;
    asm volatile(
        "{\n\t.reg .pred pi, po;\n\t"
        "setp.ne.u32 pi, %1, 0;\n\t"
        "bar.red.or.pred po, %2, %3, pi;\n\t"
        "selp.u32 %0, 1, 0, po;\n\t}"
        : "=r"(r)
        : "r"(v ? 1u : 0u), "n"(ID), "n"(N)
        : "memory");
    return r != 0;
  }
};

// Step 1: the eight 8 x 8 diagonal blocks by forward substitution (64 threads), then each
// 16 x 16 block's lower-left 8 x 8 by the merge X21 = -T_R^-1 (L_RL T_L^-1) (one thread per
// entry).  Needs NT >= 256.
template <class IxL, class IxT, int NT, class Sync = CtaSync>
__device__ void invert_diag_blocks8(float *Lm, float *Ti, int tid) {
  static_assert(NT >= 256, "one thread per entry of the four 8 x 8 merges");
  if (tid < 64) {
    const int o = 8 * (tid >> 3), c = tid & 7;
    float x[8];
#pragma unroll
    for (int t = 0; t < 8; ++t) {
      float acc = (t == c) ? 1.f : 0.f;
#pragma unroll
      for (int s = 0; s < t; ++s) acc -= Lm[IxL::at(o + t, o + s)] * x[s];
      x[t] = acc;
    }
#pragma unroll
    for (int t = 0; t < 8; ++t) Ti[IxT::at(o + t, o + c)] = x[t];
  } else if (tid < 64 + 128) {
    // zeros: the upper-right 8 x 8 of each 16 x 16 block (2 entries per thread) and
    // the upper 16 x 16 blocks of the two 32 x 32 blocks (4 entries per thread)
    const int u = tid - 64;
    {
      const int p = u >> 5, r = (u >> 2) & 7, c = 2 * (u & 3);
      Ti[IxT::at(16 * p + r, 16 * p + 8 + c)] = 0.f;
      Ti[IxT::at(16 * p + r, 16 * p + 8 + c + 1)] = 0.f;
    }
    const int k = u * 4, q = k >> 8, r = 32 * q + ((k >> 4) & 15), c = 32 * q + 16 + (k & 15);
#pragma unroll
    for (int e = 0; e < 4; ++e) Ti[IxT::at(r, c + e)] = 0.f;
  }
  Sync::sync();
  {
    const int p = (tid >> 6) & 3, r = (tid >> 3) & 7, c = tid & 7, o = 16 * p;
    float w = 0.f;
    if (tid < 256) {
#pragma unroll
      for (int k = 0; k < 8; ++k) w += Lm[IxL::at(o + 8 + r, o + k)] * Ti[IxT::at(o + k, o + c)];
    }
    Sync::sync();
    if (tid < 256) Lm[IxL::at(o + 8 + r, o + c)] = w;
    Sync::sync();
    if (tid < 256) {
      float x = 0.f;
#pragma unroll
      for (int k = 0; k < 8; ++k) x += Ti[IxT::at(o + 8 + r, o + 8 + k)] * Lm[IxL::at(o + 8 + k, o + c)];
      Ti[IxT::at(o + 8 + r, o + c)] = -x;
    }
  }
  Sync::sync();
}

// Step 2: the two merge levels on the tensor cores.
template <class IxL, class IxT, int NT, class Sync = CtaSync>
__device__ void invert_merge_levels(float *Lm, float *Ti, int tid) {
  static_assert(NT >= 256, "level 2 uses eight warps");
  const int warp = tid >> 5, lane = tid & 31;
  // level 1: pair q (blocks 2q, 2q+1), column tile nt: W = L_RL T_L^-1, X = -T_R^-1 W
  const int q1 = warp >> 1, nt1 = warp & 1, o1 = 32 * q1;
  float w1[4] = {0.f, 0.f, 0.f, 0.f};
  if (warp < 4) tile_16x8<IxL, IxT, 16>(w1, Lm, o1 + 16, o1, Ti, o1, o1 + 8 * nt1, lane);
  Sync::sync();
  if (warp < 4) store_16x8<IxL>(w1, 1.f, Lm, o1 + 16, o1 + 8 * nt1, lane);
  Sync::sync();
  if (warp < 4) {
    float x[4] = {0.f, 0.f, 0.f, 0.f};
    tile_16x8<IxT, IxL, 16>(x, Ti, o1 + 16, o1 + 16, Lm, o1 + 16, o1 + 8 * nt1, lane);
    store_16x8<IxT>(x, -1.f, Ti, o1 + 16, o1 + 8 * nt1, lane);
  }
  Sync::sync();
  // level 2: rows 32..63 x columns 0..31; row tile mt, column tile nt
  const int mt = warp >> 2, nt2 = warp & 3;
  float w2[4] = {0.f, 0.f, 0.f, 0.f};
  if (warp < 8) tile_16x8<IxL, IxT, 32>(w2, Lm, 32 + 16 * mt, 0, Ti, 0, 8 * nt2, lane);
  Sync::sync();
  if (warp < 8) store_16x8<IxL>(w2, 1.f, Lm, 32 + 16 * mt, 8 * nt2, lane);
  Sync::sync();
  if (warp < 8) {
    float x[4] = {0.f, 0.f, 0.f, 0.f};
    tile_16x8<IxT, IxL, 32>(x, Ti, 32 + 16 * mt, 32, Lm, 32, 8 * nt2, lane);
    store_16x8<IxT>(x, -1.f, Ti, 32 + 16 * mt, 8 * nt2, lane);
  }
  Sync::sync();
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
