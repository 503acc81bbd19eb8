// gdr_muir.cu -- the Muir token mixer's prologue and epilogue ("Muir: Linear Attention
// with Sensitivity-Allocated Gating and Matched-Filter Readout", section 2.1 and section
// 4.1, eqs. (8)-(9)): SiLU and per-head l2-normalisation of q and k, SiLU of v, the gate
// activations, the gain-modulated query, and the per-head RMSNorm (.) SiLU(g) readout.
// One warp per (token, head): the l2 norms and the RMS are warp reductions.
#include "gdr_internal.cuh"

namespace gdr {
namespace {

constexpr int kWarpsPerBlock = 8;

// The activations use the hardware exponential, logarithm and approximate division (a few
// ulp, below the rounding of the stored activations); the exponential's argument is clamped
// so that 1 + e^-x stays finite, and softplus switches to its asymptotes where 1 + e^x rounds.
__device__ __forceinline__ float sigmoid_f(float x) {
  return __fdividef(1.f, 1.f + __expf(-fmaxf(x, -80.f)));
}
__device__ __forceinline__ float silu_f(float x) { return x * sigmoid_f(x); }
__device__ __forceinline__ float softplus_f(float x) {
  return x > 15.f ? x : (x < -15.f ? __expf(x) : __logf(1.f + __expf(x)));
}

__device__ __forceinline__ float warp_sum(float x) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
  return x;
}

// Four consecutive elements: 8-byte (bf16) or 16-byte (fp32) accesses.
__device__ __forceinline__ void ld4(const __nv_bfloat16 *p, size_t i, float (&f)[4]) {
  const uint2 u = __ldg(reinterpret_cast<const uint2 *>(p + i));
  const __nv_bfloat162 *h = reinterpret_cast<const __nv_bfloat162 *>(&u);
  const float2 a = __bfloat1622float2(h[0]), b = __bfloat1622float2(h[1]);
  f[0] = a.x; f[1] = a.y; f[2] = b.x; f[3] = b.y;
}
__device__ __forceinline__ void ld4(const float *p, size_t i, float (&f)[4]) {
  const float4 a = __ldg(reinterpret_cast<const float4 *>(p + i));
  f[0] = a.x; f[1] = a.y; f[2] = a.z; f[3] = a.w;
}
__device__ __forceinline__ void st4(__nv_bfloat16 *p, size_t i, const float (&f)[4]) {
  __nv_bfloat162 h[2] = {__floats2bfloat162_rn(f[0], f[1]), __floats2bfloat162_rn(f[2], f[3])};
  *reinterpret_cast<uint2 *>(p + i) = *reinterpret_cast<const uint2 *>(h);
}
__device__ __forceinline__ void st4(float *p, size_t i, const float (&f)[4]) {
  *reinterpret_cast<float4 *>(p + i) = make_float4(f[0], f[1], f[2], f[3]);
}

// One warp per (token, head); lane l holds channels 4l .. 4l + 3 (d <= 128).
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
  const size_t ik = tok * dk + 4 * lane, iv = tok * dv + 4 * lane;
  const bool onk = 4 * lane < dk, onv = 4 * lane < dv;
  float xq[4] = {0.f, 0.f, 0.f, 0.f}, xk[4] = {0.f, 0.f, 0.f, 0.f};
  float f4[4], b4[4], g4[4];
  if (onk) {
    ld4(q, ik, xq);
    ld4(k, ik, xk);
    ld4(zf, ik, f4);
    ld4(zb, ik, b4);
    ld4(zq, ik, g4);
  }
  float sq = 0.f, sk = 0.f;
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    xq[e] = silu_f(xq[e]);
    xk[e] = silu_f(xk[e]);
    sq += xq[e] * xq[e];
    sk += xk[e] * xk[e];
  }
  const float nq = rsqrtf(fmaxf(warp_sum(sq), 1e-24f)), nk = rsqrtf(fmaxf(warp_sum(sk), 1e-24f));
  if (onk) {
    const float rate = __expf(m.a_log[h]);
    float gs[4] = {1.f, 1.f, 1.f, 1.f}, oq[4], ok[4], ob[4], ol[4];
    if (m.gamma_stat) ld4(m.gamma_stat, (size_t)h * dk + 4 * lane, gs);
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      oq[e] = gs[e] * 2.f * sigmoid_f(g4[e]) * xq[e] * nq;
      ok[e] = xk[e] * nk;
      ob[e] = 2.f * sigmoid_f(b4[e]);
      ol[e] = -rate * softplus_f(f4[e]);
    }
    st4(qh, ik, oq);
    st4(kh, ik, ok);
    st4(bo, ik, ob);
    st4(lw, ik, ol);
  }
  if (onv) {
    float x[4], w[4];
    ld4(v, iv, x);
    ld4(zw, iv, w);
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      x[e] = silu_f(x[e]);
      w[e] = sigmoid_f(w[e]);
    }
    st4(vh, iv, x);
    st4(wo, iv, w);
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
  const size_t iv = tok * dv + 4 * lane;
  const bool on = 4 * lane < dv;
  float x[4] = {0.f, 0.f, 0.f, 0.f}, g[4];
  if (on) {
    ld4(o, iv, x);
    ld4(zg, iv, g);
  }
  const float inv = rsqrtf(warp_sum(x[0] * x[0] + x[1] * x[1] + x[2] * x[2] + x[3] * x[3]) / dv +
                           m.rms_eps);
  if (on) {
    float rho[4] = {1.f, 1.f, 1.f, 1.f}, out[4];
    if (m.rms_weight) ld4(m.rms_weight, 4 * lane, rho);
#pragma unroll
    for (int e = 0; e < 4; ++e) out[e] = rho[e] * x[e] * inv * silu_f(g[e]);
    st4(y, iv, out);
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
