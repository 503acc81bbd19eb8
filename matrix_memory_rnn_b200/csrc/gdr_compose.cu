// gdr_compose.cu -- S_out = M S_in + Q per head: the affine exit-state map of a sequence
// segment applied to its entry state ("Muir ...", section 4.2 eq. (10), extended from a
// chunk to any run of chunks).  One 128-thread CTA per (head, 32 value columns); the
// product is a warp-level tf32 MMA with the three-product split, so fp32 states keep fp32
// accuracy.  Operands are read from global memory (small, L2-resident).
#include "gdr_internal.cuh"
#include "gdr_warp_mma.cuh"

namespace gdr {
namespace {

using wmma_tf32::for_acc;
using wmma_tf32::mma_seg;
using wmma_tf32::zero_acc;

constexpr int kThreads = 128;

// dk >= 16 and dv >= 32: 16 x 32 warp tiles over (dk rows) x (32 columns); dv = 16 uses
// the scalar path below.
__global__ void __launch_bounds__(kThreads) compose_mma_kernel(float *S_out, const float *M,
                                                               const float *S_in, const float *Q,
                                                               int dk, int dv) {
  const size_t bh = blockIdx.y;
  const int c0 = 32 * blockIdx.x, warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const float *Mh = M + bh * dk * dk;
  const float *Sh = S_in ? S_in + bh * dk * dv : nullptr;
  const float *Qh = Q ? Q + bh * dk * dv : nullptr;
  float *Oh = S_out + bh * dk * dv;
  for (int wt = warp; wt < dk / 16; wt += kThreads / 32) {
    const int r0 = 16 * wt;
    float acc[4][4];
    zero_acc(acc);
    if (Sh)
      mma_seg<true>(acc, r0, c0, 0, dk, [&](int m, int kk) { return __ldg(Mh + (size_t)m * dk + kk); },
                    [&](int kk, int nn) { return __ldg(Sh + (size_t)kk * dv + nn); }, lane);
    for_acc(acc, r0, c0, lane, [&](int r, int c, float x) {
      const size_t i = (size_t)r * dv + c;
      Oh[i] = x + (Qh ? Qh[i] : 0.f);
    });
  }
}

__global__ void __launch_bounds__(kThreads) compose_scalar_kernel(float *S_out, const float *M,
                                                                  const float *S_in, const float *Q,
                                                                  int dk, int dv) {
  const size_t bh = blockIdx.x;
  for (int i = threadIdx.x; i < dk * dv; i += kThreads) {
    const int r = i / dv, c = i % dv;
    double acc = 0.0;
    if (S_in)
      for (int kk = 0; kk < dk; ++kk)
        acc += (double)M[bh * dk * dk + (size_t)r * dk + kk] * S_in[bh * dk * dv + (size_t)kk * dv + c];
    S_out[bh * dk * dv + i] = (float)acc + (Q ? Q[bh * dk * dv + i] : 0.f);
  }
}

}  // namespace

cudaError_t launch_state_compose(float *S_out, const float *M, const float *S_in, const float *Q,
                                 int BH, int dk, int dv, cudaStream_t stream) {
  if (BH == 0) return cudaSuccess;
  if (dv >= 32)
    compose_mma_kernel<<<dim3(dv / 32, BH), kThreads, 0, stream>>>(S_out, M, S_in, Q, dk, dv);
  else
    compose_scalar_kernel<<<BH, kThreads, 0, stream>>>(S_out, M, S_in, Q, dk, dv);
  return cudaGetLastError();
}

}  // namespace gdr
