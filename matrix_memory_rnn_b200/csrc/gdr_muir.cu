// gdr_muir.cu -- the Muir token mixer's prologue and epilogue ("Muir: Linear Attention
// with Sensitivity-Allocated Gating and Matched-Filter Readout", section 2.1 and section
// 4.1, eqs. (8)-(9)): SiLU and per-head l2-normalisation of q and k, SiLU of v, the gate
// activations, the gain-modulated query, and the per-head RMSNorm (.) SiLU(g) readout.
// One warp per (token, head): the l2 norms and the RMS are warp reductions.
#include "gdr_internal.cuh"

namespace gdr {
namespace {

constexpr int kWarpsPerBlock = 8;

__device__ __forceinline__ float silu_f(float x) { return x / (1.f + expf(-x)); }
__device__ __forceinline__ float sigmoid_f(float x) { return 1.f / (1.f + expf(-x)); }
__device__ __forceinline__ float softplus_f(float x) { return x > 20.f ? x : log1pf(expf(x)); }

__device__ __forceinline__ float warp_sum(float x) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
  return x;
}

__device__ __forceinline__ void st_out(float *p, size_t i, float x) { p[i] = x; }
__device__ __forceinline__ void st_out(__nv_bfloat16 *p, size_t i, float x) { p[i] = __float2bfloat16_rn(x); }

// Up to 4 channels per lane (d <= 128).
template <typename Tin>
__global__ void __launch_bounds__(32 * kWarpsPerBlock) muir_prologue_kernel(
    MuirParams m, Tin *qh, Tin *kh, Tin *vh, Tin *bo, Tin *wo, float *lw) {
  const size_t tok = (size_t)blockIdx.x * kWarpsPerBlock + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (tok >= (size_t)m.B * m.T * m.H) return;
  const int h = (int)(tok % m.H), dk = m.dk, dv = m.dv;
  const Tin *q = static_cast<const Tin *>(m.q), *k = static_cast<const Tin *>(m.k);
  const Tin *v = static_cast<const Tin *>(m.v), *zf = static_cast<const Tin *>(m.zf);
  const Tin *zb = static_cast<const Tin *>(m.zb), *zw = static_cast<const Tin *>(m.zw);
  const Tin *zq = static_cast<const Tin *>(m.zq);
  const size_t ik = tok * dk, iv = tok * dv;
  float xq[4], xk[4], sq = 0.f, sk = 0.f;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int j = lane + 32 * i;
    xq[i] = xk[i] = 0.f;
    if (j < dk) {
      xq[i] = silu_f(ld_in(q, ik + j));
      xk[i] = silu_f(ld_in(k, ik + j));
    }
    sq += xq[i] * xq[i];
    sk += xk[i] * xk[i];
  }
  const float nq = fmaxf(sqrtf(warp_sum(sq)), 1e-12f), nk = fmaxf(sqrtf(warp_sum(sk)), 1e-12f);
  const float rate = expf(m.a_log[h]);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int j = lane + 32 * i;
    if (j >= dk) break;
    const float gs = m.gamma_stat ? m.gamma_stat[(size_t)h * dk + j] : 1.f;
    st_out(qh, ik + j, gs * 2.f * sigmoid_f(ld_in(zq, ik + j)) * xq[i] / nq);
    st_out(kh, ik + j, xk[i] / nk);
    st_out(bo, ik + j, 2.f * sigmoid_f(ld_in(zb, ik + j)));
    lw[ik + j] = -rate * softplus_f(ld_in(zf, ik + j));
  }
  for (int c = lane; c < dv; c += 32) {
    st_out(vh, iv + c, silu_f(ld_in(v, iv + c)));
    st_out(wo, iv + c, sigmoid_f(ld_in(zw, iv + c)));
  }
}

template <typename Tin>
__global__ void __launch_bounds__(32 * kWarpsPerBlock) muir_epilogue_kernel(MuirParams m,
                                                                            const float *o,
                                                                            float *y) {
  const size_t tok = (size_t)blockIdx.x * kWarpsPerBlock + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (tok >= (size_t)m.B * m.T * m.H) return;
  const int dv = m.dv;
  const Tin *zg = static_cast<const Tin *>(m.zg);
  const size_t iv = tok * dv;
  float x[4], ss = 0.f;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int c = lane + 32 * i;
    x[i] = c < dv ? o[iv + c] : 0.f;
    ss += x[i] * x[i];
  }
  const float inv = rsqrtf(warp_sum(ss) / dv + m.rms_eps);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int c = lane + 32 * i;
    if (c >= dv) break;
    const float rho = m.rms_weight ? m.rms_weight[c] : 1.f;
    y[iv + c] = rho * x[i] * inv * silu_f(ld_in(zg, iv + c));
  }
}

}  // namespace

cudaError_t launch_muir_prologue(const MuirParams &m, gdr_dtype dtype, void *qh, void *kh,
                                 void *vh, void *b, void *w, float *log_w, cudaStream_t stream) {
  const size_t n = (size_t)m.B * m.T * m.H;
  if (n == 0) return cudaSuccess;
  const unsigned grid = (unsigned)((n + kWarpsPerBlock - 1) / kWarpsPerBlock);
  if (dtype == GDR_BF16)
    muir_prologue_kernel<__nv_bfloat16><<<grid, 32 * kWarpsPerBlock, 0, stream>>>(
        m, static_cast<__nv_bfloat16 *>(qh), static_cast<__nv_bfloat16 *>(kh),
        static_cast<__nv_bfloat16 *>(vh), static_cast<__nv_bfloat16 *>(b),
        static_cast<__nv_bfloat16 *>(w), log_w);
  else
    muir_prologue_kernel<float><<<grid, 32 * kWarpsPerBlock, 0, stream>>>(
        m, static_cast<float *>(qh), static_cast<float *>(kh), static_cast<float *>(vh),
        static_cast<float *>(b), static_cast<float *>(w), log_w);
  return cudaGetLastError();
}

cudaError_t launch_muir_epilogue(const MuirParams &m, gdr_dtype dtype, const float *o, float *y,
                                 cudaStream_t stream) {
  const size_t n = (size_t)m.B * m.T * m.H;
  if (n == 0) return cudaSuccess;
  const unsigned grid = (unsigned)((n + kWarpsPerBlock - 1) / kWarpsPerBlock);
  if (dtype == GDR_BF16)
    muir_epilogue_kernel<__nv_bfloat16><<<grid, 32 * kWarpsPerBlock, 0, stream>>>(m, o, y);
  else
    muir_epilogue_kernel<float><<<grid, 32 * kWarpsPerBlock, 0, stream>>>(m, o, y);
  return cudaGetLastError();
}

}  // namespace gdr
