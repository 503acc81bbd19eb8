// gdr_mlstm.cu -- xLSTM's mLSTM cell with the log-domain stabilizer ("Exponential gates
// and matrix memory: xLSTM and RWKV-7", section 13.4 and the solution to Exercise 13.6),
// chunkwise.
//
// The stabilizer is a running maximum of the log-weights of everything the memory holds:
// unrolled, m_t = max(F_t + m_0, max_{s<=t} (F_t - F_s + i~_s)) with F the cumulative
// log forget gate.  Inside a chunk (local cumulative A_t, carried state C, n, m) that is
//   m_t = A_t + max(m, P_t),   P_t = max_{s<=t} (i~_s - A_s)   (a prefix maximum),
// and every weight of the readout and of the carried state is an exponential of a
// non-positive argument:
//   w_ts = e^{A_t - A_s + i~_s - m_t} (s <= t),   g_t = e^{A_t + m - m_t},
//   num_t = sum_s w_ts (q_t . k_s) v_s + g_t C q_t,   den_t = sum_s w_ts (q_t . k_s) + g_t n . q_t,
//   h_t = num_t / max(|den_t|, e^{-m_t}),
//   C <- g_L C + sum_s w_Ls v_s k_s^T,   n <- g_L n + sum_s w_Ls k_s,   m <- m_L.
// One CTA per (b, h, 64 value columns) walks the chunks of its sequence with the state
// slice in shared memory; Q K^T, P V + diag(g) Q C, and the state update K^T diag(w_L) V
// are warp-level tf32 MMAs (three products for fp32 inputs).  Tokens past T are padding
// with log f = 0 and i~ = -inf (no write, no decay).
#include <math.h>

#include "gdr_internal.cuh"
#include "gdr_warp_mma.cuh"

namespace gdr {
namespace {

using wmma_tf32::for_acc;
using wmma_tf32::mma_seg;
using wmma_tf32::zero_acc;

constexpr int kL = 64;          // chunk
constexpr int kNV = 64;         // value columns per CTA
constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;
constexpr int kLDL = kL + 4;
constexpr int kLDN = kNV + 4;

// Shared memory: fp32 arrays (offsets in floats), then the q, k, v tiles at the input's
// element type (offsets in bytes from `tiles`): bf16 inputs keep their exact values in
// half the space, and are widened as they are read.
struct MlstmSmem {
  int LDK, LDV;  // row strides of the q / k and v tiles, in elements (16-byte rows)
  size_t P, C, n, A, lf, ib, m, g, den, mcar, tiles, Q, K, V, bytes;
  __host__ __device__ MlstmSmem(int dk, int esize) {
    const int pad = 16 / esize;
    LDK = dk + pad;
    LDV = kNV + pad;
    size_t off = 0;
    P = off; off += (size_t)kL * kLDL;
    C = off; off += (size_t)dk * kLDN;
    n = off; off += dk;
    A = off; off += kL;
    lf = off; off += kL;
    ib = off; off += kL;
    m = off; off += kL;
    g = off; off += kL;
    den = off; off += kL;
    mcar = off; off += 4;
    tiles = off * 4;
    Q = 0;
    K = Q + (size_t)kL * LDK * esize;
    V = K + (size_t)kL * LDK * esize;
    bytes = tiles + V + (size_t)kL * LDV * esize;
  }
};
__device__ __forceinline__ float widen1(float x) { return x; }
__device__ __forceinline__ float widen1(__nv_bfloat16 x) { return __bfloat162float(x); }

// 16-byte pieces of the chunk's q, k (64 x dk) and v slice (64 x 64) held in registers:
// the next chunk is loaded while the current one is computed.  kE = elements per piece.
template <typename Tin, int kDK>
struct ChunkRegs {
  static constexpr int kE = 16 / sizeof(Tin);
  static constexpr int kQK = kL * kDK / kE / kThreads;   // pieces per thread of q (and of k)
  static constexpr int kV = kL * kNV / kE / kThreads;
  uint4 q[kQK], k[kQK], v[kV];
  float lf, ib;
};
template <typename Tin, bool kSplit, int kDK>
__global__ void __launch_bounds__(kThreads, kSplit ? 1 : 2) mlstm_kernel(gdr_mlstm_args a) {
  extern __shared__ float sm[];
  constexpr int dk = kDK;
  const int dv = a.dv, T = a.T, H = a.H;
  const MlstmSmem L(dk, sizeof(Tin));
  const int LDK = L.LDK, LDV = L.LDV;
  const int c0 = blockIdx.x * kNV, h = blockIdx.y, b = blockIdx.z;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  float *P = sm + L.P, *C = sm + L.C, *nn = sm + L.n;
  float *A = sm + L.A, *lf = sm + L.lf, *ib = sm + L.ib, *mt = sm + L.m, *gt = sm + L.g;
  float *den = sm + L.den;
  float *mcar = sm + L.mcar;   // the carried running max
  uint8_t *tiles = reinterpret_cast<uint8_t *>(sm) + L.tiles;
  Tin *Qs = reinterpret_cast<Tin *>(tiles + L.Q), *Ks = reinterpret_cast<Tin *>(tiles + L.K);
  Tin *Vs = reinterpret_cast<Tin *>(tiles + L.V);
  auto Q = [&](int r, int c) { return widen1(Qs[r * LDK + c]); };
  auto K = [&](int r, int c) { return widen1(Ks[r * LDK + c]); };
  auto V = [&](int r, int c) { return widen1(Vs[r * LDV + c]); };
  const Tin *q = static_cast<const Tin *>(a.q), *k = static_cast<const Tin *>(a.k);
  const Tin *v = static_cast<const Tin *>(a.v);
  const size_t bh = (size_t)b * H + h;

  for (int i = tid; i < dk * kNV; i += kThreads) {
    const int j = i / kNV, c = i % kNV;
    C[j * kLDN + c] = a.C0 ? a.C0[bh * dk * dv + (size_t)j * dv + c0 + c] : 0.f;
  }
  for (int j = tid; j < dk; j += kThreads) nn[j] = a.n0 ? a.n0[bh * dk + j] : 0.f;
  if (tid == 0) *mcar = a.m0 ? a.m0[bh] : -INFINITY;

  // ---- chunk loads (padding: q = k = v = 0, log f = 0, i~ = -inf), one chunk ahead
  using R = ChunkRegs<Tin, kDK>;
  R rg;
  const int gq = dk / R::kE;                 // pieces per row of q / k
  const int nq = kL * gq / kThreads;         // pieces per thread (d_k = 64: half of kQK)
  auto fetch = [&](int t0) {
#pragma unroll
    for (int u = 0; u < R::kQK; ++u) {
      if (u >= nq) break;
      const int i = tid + u * kThreads, t = i / gq, j = (i % gq) * R::kE;
      const size_t ik = (((size_t)b * T + t0 + t) * H + h) * dk + j;
      const bool in = t0 + t < T;
      rg.q[u] = in ? __ldg(reinterpret_cast<const uint4 *>(q + ik)) : make_uint4(0u, 0u, 0u, 0u);
      rg.k[u] = in ? __ldg(reinterpret_cast<const uint4 *>(k + ik)) : make_uint4(0u, 0u, 0u, 0u);
    }
#pragma unroll
    for (int u = 0; u < R::kV; ++u) {
      const int i = tid + u * kThreads, t = i / (kNV / R::kE), c = (i % (kNV / R::kE)) * R::kE;
      const bool in = t0 + t < T;
      rg.v[u] = in ? __ldg(reinterpret_cast<const uint4 *>(v + (((size_t)b * T + t0 + t) * H + h) * dv + c0 + c))
                   : make_uint4(0u, 0u, 0u, 0u);
    }
    if (tid < kL) {
      const bool in = t0 + tid < T;
      const size_t ts = ((size_t)b * T + t0 + tid) * H + h;
      rg.lf = in ? __ldg(a.f_pre + ts) : 0.f;
      rg.ib = in ? __ldg(a.i_pre + ts) : -INFINITY;
    }
  };
  auto commit = [&](int n) {
#pragma unroll
    for (int u = 0; u < R::kQK; ++u) {
      if (u >= nq) break;
      const int i = tid + u * kThreads, t = i / gq, j = (i % gq) * R::kE;
      *reinterpret_cast<uint4 *>(Qs + t * LDK + j) = rg.q[u];
      *reinterpret_cast<uint4 *>(Ks + t * LDK + j) = rg.k[u];
    }
#pragma unroll
    for (int u = 0; u < R::kV; ++u) {
      const int i = tid + u * kThreads, t = i / (kNV / R::kE), c = (i % (kNV / R::kE)) * R::kE;
      *reinterpret_cast<uint4 *>(Vs + t * LDV + c) = rg.v[u];
    }
    if (tid < kL) {
      const float x = rg.lf;   // log sigmoid; padding keeps log f = 0
      lf[tid] = tid < n ? (x >= 0.f ? -log1pf(expf(-x)) : x - log1pf(expf(x))) : 0.f;
      ib[tid] = rg.ib;
    }
  };
  fetch(0);

  for (int t0 = 0; t0 < T; t0 += kL) {
    const int n = min(kL, T - t0);
    __syncthreads();   // the previous chunk is done with every buffer
    commit(n);
    if (t0 + kL < T) fetch(t0 + kL);
    __syncthreads();
    // ---- A (inclusive prefix of log f), the prefix max of i~ - A, m_t and g_t (warp 0)
    if (warp == 0) {
      float a0 = lf[lane], a1 = lf[lane + 32];
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const float x0 = __shfl_up_sync(0xffffffffu, a0, o), x1 = __shfl_up_sync(0xffffffffu, a1, o);
        if (lane >= o) {
          a0 += x0;
          a1 += x1;
        }
      }
      a1 += __shfl_sync(0xffffffffu, a0, 31);
      float p0 = ib[lane] - a0, p1 = ib[lane + 32] - a1;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const float x0 = __shfl_up_sync(0xffffffffu, p0, o), x1 = __shfl_up_sync(0xffffffffu, p1, o);
        if (lane >= o) {
          p0 = fmaxf(p0, x0);
          p1 = fmaxf(p1, x1);
        }
      }
      p1 = fmaxf(p1, __shfl_sync(0xffffffffu, p0, 31));
      const float mc = *mcar;
      const float m0 = a0 + fmaxf(mc, p0), m1 = a1 + fmaxf(mc, p1);
      A[lane] = a0;
      A[lane + 32] = a1;
      mt[lane] = m0;
      mt[lane + 32] = m1;
      gt[lane] = expf(a0 + mc - m0);      // 0 for an empty memory (mc = -inf)
      gt[lane + 32] = expf(a1 + mc - m1);
    }
    __syncthreads();
    // ---- P = (Q K^T) (.) w, w_ts = e^{A_t - A_s + i~_s - m_t} (s <= t)
    {
      const int r0 = 16 * (warp >> 1), cc0 = 32 * (warp & 1);
      float acc[4][4];
      zero_acc(acc);
      mma_seg<kSplit>(acc, r0, cc0, 0, dk, [&](int m, int kk) { return Q(m, kk); },
                      [&](int kk, int nn2) { return K(nn2, kk); }, lane);
      for_acc(acc, r0, cc0, lane, [&](int t, int s, float x) {
        P[t * kLDL + s] = s <= t ? x * expf(A[t] - A[s] + ib[s] - mt[t]) : 0.f;
      });
    }
    __syncthreads();
    // ---- den_t = sum_s P_ts + g_t n . q_t (4 threads per row)
    {
      const int t = tid >> 2, part = tid & 3;
      float s = 0.f;
      for (int u = part; u < kL; u += 4) s += P[t * kLDL + u];
      for (int j = part; j < dk; j += 4) s += gt[t] * nn[j] * Q(t, j);
      s += __shfl_xor_sync(0xffffffffu, s, 1);
      s += __shfl_xor_sync(0xffffffffu, s, 2);
      if (part == 0) den[t] = s;
    }
    __syncthreads();
    // ---- h = (P V + diag(g) Q C) / max(|den|, e^{-m})
    {
      const int r0 = 16 * (warp >> 1), cc0 = 32 * (warp & 1);
      float acc[4][4];
      zero_acc(acc);
      mma_seg<kSplit>(acc, r0, cc0, 0, kL, [&](int m, int kk) { return P[m * kLDL + kk]; },
                      [&](int kk, int nn2) { return V(kk, nn2); }, lane);
      mma_seg<kSplit>(acc, r0, cc0, 0, dk, [&](int m, int kk) { return gt[m] * Q(m, kk); },
                      [&](int kk, int nn2) { return C[kk * kLDN + nn2]; }, lane);
      for_acc(acc, r0, cc0, lane, [&](int t, int c, float x) {
        if (t < n)
          a.h[(((size_t)b * T + t0 + t) * H + h) * dv + c0 + c] =
              x / fmaxf(fabsf(den[t]), expf(-mt[t]));
      });
    }
    __syncthreads();   // C and n are read above; they change below
    // ---- state: C <- g_L C + K^T diag(w_L) V, n <- g_L n + K^T w_L, m <- m_L
    {
      const float mL = mt[kL - 1], gL = gt[kL - 1];
      float *wl = den;   // den is read above: w_Ls = e^{A_L - A_s + i~_s - m_L} in its place
      if (tid < kL) wl[tid] = expf(A[kL - 1] - A[tid] + ib[tid] - mL);
      __syncthreads();
      auto wL = [&](int s) { return wl[s]; };
      for (int wt = warp; wt < dk / 8; wt += kWarps) {
        const int r0 = 16 * (wt >> 1), cc0 = 32 * (wt & 1);
        float acc[4][4];
        zero_acc(acc);
        mma_seg<kSplit>(acc, r0, cc0, 0, kL, [&](int m, int s) { return K(s, m) * wL(s); },
                        [&](int s, int nn2) { return V(s, nn2); }, lane);
        for_acc(acc, r0, cc0, lane, [&](int j, int c, float x) {
          C[j * kLDN + c] = gL * C[j * kLDN + c] + x;
        });
      }
      for (int j = tid; j < dk; j += kThreads) {
        float s = 0.f;
        for (int u = 0; u < kL; ++u) s += wL(u) * K(u, j);
        nn[j] = gL * nn[j] + s;
      }
      __syncthreads();
      if (tid == 0) *mcar = mL;
    }
  }
  __syncthreads();
  if (a.C_T)
    for (int i = tid; i < dk * kNV; i += kThreads) {
      const int j = i / kNV, c = i % kNV;
      a.C_T[bh * dk * dv + (size_t)j * dv + c0 + c] = C[j * kLDN + c];
    }
  if (blockIdx.x == 0) {
    if (a.n_T)
      for (int j = tid; j < dk; j += kThreads) a.n_T[bh * dk + j] = nn[j];
    if (a.m_T && tid == 0) a.m_T[bh] = *mcar;
  }
}

template <typename Tin, bool kSplit, int kDK>
cudaError_t launch_typed(const gdr_mlstm_args &a, cudaStream_t stream) {
  const size_t smem = MlstmSmem(kDK, sizeof(Tin)).bytes;
  cudaError_t e = cudaFuncSetAttribute(mlstm_kernel<Tin, kSplit, kDK>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  mlstm_kernel<Tin, kSplit, kDK><<<dim3(a.dv / kNV, a.H, a.B), kThreads, smem, stream>>>(a);
  return cudaGetLastError();
}

__global__ void fill_kernel(float *p, size_t n, float x) {
  for (size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (size_t)gridDim.x * blockDim.x)
    p[i] = x;
}

}  // namespace

cudaError_t fill_f32(float *p, size_t n, float x, cudaStream_t stream) {
  if (n == 0) return cudaSuccess;
  fill_kernel<<<(unsigned)((n + 255) / 256 < 1024 ? (n + 255) / 256 : 1024), 256, 0, stream>>>(p, n, x);
  return cudaGetLastError();
}

cudaError_t launch_mlstm(const gdr_mlstm_args &a, cudaStream_t stream) {
  if (a.dtype == GDR_BF16)
    return a.dk == 64 ? launch_typed<__nv_bfloat16, false, 64>(a, stream)
                      : launch_typed<__nv_bfloat16, false, 128>(a, stream);
  return a.dk == 64 ? launch_typed<float, true, 64>(a, stream) : launch_typed<float, true, 128>(a, stream);
}

}  // namespace gdr
