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
// slice in shared memory.  Q K^T takes bf16 MMAs for bf16 inputs (exact products) and
// tf32 otherwise; P V, Q C and the state update K^T diag(w_L) V are tf32 (three products
// for fp32 inputs).  Tokens past T are padding with log f = 0 and i~ = -inf (no write, no
// decay).
#include <math.h>

#include <type_traits>

#include "gdr_internal.cuh"
#include "gdr_warp_mma.cuh"

namespace gdr {
namespace {

using wmma_tf32::for_acc;
using wmma_tf32::mma_bf16_abt;
using wmma_tf32::mma_seg;
using wmma_tf32::tf32_exact;
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

// Views of one CTA's shared memory.
template <typename Tin>
struct Views {
  float *P, *C, *nn, *A, *lf, *ib, *mt, *gt, *den, *mcar;
  Tin *Qs, *Ks, *Vs;
  int LDK, LDV;
  __device__ Views(float *sm, const MlstmSmem &L) {
    P = sm + L.P; C = sm + L.C; nn = sm + L.n; A = sm + L.A; lf = sm + L.lf; ib = sm + L.ib;
    mt = sm + L.m; gt = sm + L.g; den = sm + L.den; mcar = sm + L.mcar;
    uint8_t *tiles = reinterpret_cast<uint8_t *>(sm) + L.tiles;
    Qs = reinterpret_cast<Tin *>(tiles + L.Q);
    Ks = reinterpret_cast<Tin *>(tiles + L.K);
    Vs = reinterpret_cast<Tin *>(tiles + L.V);
    LDK = L.LDK;
    LDV = L.LDV;
  }
  __device__ float Q(int r, int c) const { return widen(Qs[r * LDK + c]); }
  __device__ float K(int r, int c) const { return widen(Ks[r * LDK + c]); }
  // the tiles as MMA operands (a bf16 value is exact in tf32)
  __device__ auto Qx(int r, int c) const { return tf32_exact(Qs[r * LDK + c]); }
  __device__ auto Kx(int r, int c) const { return tf32_exact(Ks[r * LDK + c]); }
  __device__ auto Vx(int r, int c) const { return tf32_exact(Vs[r * LDV + c]); }
  static __device__ float widen(float x) { return x; }
  static __device__ float widen(__nv_bfloat16 x) { return __bfloat162float(x); }
};

__device__ __forceinline__ float log_sigmoid(float x) {
  return x >= 0.f ? -log1pf(expf(-x)) : x - log1pf(expf(x));
}

// Warp 0: A (inclusive prefix of log f), the prefix max of i~ - A, m_t and g_t, from the
// carried running max mc.
__device__ __forceinline__ void scan_chunk(const float *lf, const float *ib, float mc, float *A,
                                           float *mt, float *gt, int lane) {
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
  const float m0 = a0 + fmaxf(mc, p0), m1 = a1 + fmaxf(mc, p1);
  A[lane] = a0;
  A[lane + 32] = a1;
  mt[lane] = m0;
  mt[lane + 32] = m1;
  gt[lane] = expf(a0 + mc - m0);      // 0 for an empty memory (mc = -inf)
  gt[lane + 32] = expf(a1 + mc - m1);
}

// The chunk's readout h for value columns [c0, c0 + 64) from the scanned gates and the
// state in shared memory; every thread calls it after a barrier that follows the scan.
// Rows t >= n are not stored.
template <typename Tin, bool kSplit, int kDK>
__device__ __forceinline__ void readout(const Views<Tin> &s, float *hout, size_t hstride, int n) {
  constexpr int dk = kDK;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int r0 = 16 * (warp >> 1), cc0 = 32 * (warp & 1), g = lane >> 2, tq = lane & 3;
  // ---- P = (Q K^T) (.) w, w_ts = e^{A_t - A_s + i~_s - m_t} (s <= t)
  {
    float acc[4][4];
    zero_acc(acc);
    if constexpr (std::is_same<Tin, __nv_bfloat16>::value)
      mma_bf16_abt(acc, s.Qs, s.LDK, s.Ks, s.LDK, r0, cc0, 0, dk, lane);
    else
      mma_seg<kSplit>(acc, r0, cc0, 0, dk, [&](int m, int kk) { return s.Qx(m, kk); },
                      [&](int kk, int nn2) { return s.Kx(nn2, kk); }, lane);
    for_acc(acc, r0, cc0, lane, [&](int t, int j, float x) {
      s.P[t * kLDL + j] = j <= t ? x * __expf(s.A[t] - s.A[j] + s.ib[j] - s.mt[t]) : 0.f;
    });
  }
  __syncthreads();
  // ---- 1 / max(|den_t|, e^{-m_t}), den_t = sum_s P_ts + g_t n . q_t (4 threads per row)
  {
    const int t = tid >> 2, part = tid & 3;
    float sp = 0.f, sq = 0.f;
    for (int u = part; u < kL; u += 4) sp += s.P[t * kLDL + u];
    for (int j = part; j < dk; j += 4) sq += s.nn[j] * s.Q(t, j);
    float acc = sp + s.gt[t] * sq;
    acc += __shfl_xor_sync(0xffffffffu, acc, 1);
    acc += __shfl_xor_sync(0xffffffffu, acc, 2);
    if (part == 0) s.den[t] = 1.f / fmaxf(fabsf(acc), expf(-s.mt[t]));
  }
  __syncthreads();
  // ---- h = (P V + diag(g) Q C) / max(|den|, e^{-m}); P V and Q C in two accumulators
  {
    float pv[4][4], qc[4][4];
    zero_acc(pv);
    zero_acc(qc);
    mma_seg<kSplit>(pv, r0, cc0, 0, kL, [&](int m, int kk) { return s.P[m * kLDL + kk]; },
                    [&](int kk, int nn2) { return s.Vx(kk, nn2); }, lane);
    mma_seg<kSplit>(qc, r0, cc0, 0, dk, [&](int m, int kk) { return s.Qx(m, kk); },
                    [&](int kk, int nn2) { return s.C[kk * kLDN + nn2]; }, lane);
#pragma unroll
    for (int hf = 0; hf < 2; ++hf) {   // rows r0 + g and r0 + g + 8
      const int t = r0 + g + 8 * hf;
      if (t >= n) continue;
      const float gg = s.gt[t], rd = s.den[t];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const float x0 = fmaf(gg, qc[i][2 * hf], pv[i][2 * hf]) * rd;
        const float x1 = fmaf(gg, qc[i][2 * hf + 1], pv[i][2 * hf + 1]) * rd;
        *reinterpret_cast<float2 *>(hout + t * hstride + cc0 + 8 * i + 2 * tq) = make_float2(x0, x1);
      }
    }
  }
}

// C <- g_L C + K^T diag(w_L) V, n <- g_L n + K^T w_L, m <- m_L; every thread calls it after
// a barrier that follows every read of C, n and den.
template <typename Tin, bool kSplit, int kDK>
__device__ __forceinline__ void update_state(const Views<Tin> &s) {
  constexpr int dk = kDK;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const float mL = s.mt[kL - 1], gL = s.gt[kL - 1];
  float *wl = s.den;   // den is read: w_Ls = e^{A_L - A_s + i~_s - m_L} in its place
  if (tid < kL) wl[tid] = expf(s.A[kL - 1] - s.A[tid] + s.ib[tid] - mL);
  __syncthreads();
  for (int wt = warp; wt < dk / 8; wt += kWarps) {
    const int r0 = 16 * (wt >> 1), cc0 = 32 * (wt & 1);
    float acc[4][4];
    zero_acc(acc);
    mma_seg<kSplit>(acc, r0, cc0, 0, kL, [&](int m, int j) { return s.K(j, m) * wl[j]; },
                    [&](int j, int nn2) { return s.Vx(j, nn2); }, lane);
    for_acc(acc, r0, cc0, lane, [&](int j, int c, float x) {
      s.C[j * kLDN + c] = gL * s.C[j * kLDN + c] + x;
    });
  }
  {   // kThreads / dk adjacent lanes per key channel
    constexpr int kP = kThreads / kDK;
    const int j = tid / kP, part = tid % kP;
    float acc = 0.f;
    for (int u = part; u < kL; u += kP) acc += wl[u] * s.K(u, j);
#pragma unroll
    for (int o = 1; o < kP; o <<= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
    if (part == 0) s.nn[j] = gL * s.nn[j] + acc;
  }
  __syncthreads();
  if (tid == 0) *s.mcar = mL;
}

// 16-byte pieces of the chunk's q, k (64 x dk) and v slice (64 x 64) held in registers:
// the next chunk is loaded while the current one is computed.  kE = elements per piece.
template <typename Tin, int kDK>
struct ChunkRegs {
  static constexpr int kE = 16 / sizeof(Tin);
  static constexpr int kQK = kL * kDK / kE / kThreads;   // pieces per thread of q (and of k)
  static constexpr int kV = kL * kNV / kE / kThreads;
  uint4 q[kQK], k[kQK], v[kV];
  float lf, ib;

  __device__ void fetch(const gdr_mlstm_args &a, int b, int h, int c0, int t0) {
    const Tin *q_ = static_cast<const Tin *>(a.q), *k_ = static_cast<const Tin *>(a.k);
    const Tin *v_ = static_cast<const Tin *>(a.v);
    const int tid = threadIdx.x, T = a.T, H = a.H, gq = kDK / kE;
#pragma unroll
    for (int u = 0; u < kQK; ++u) {
      const int i = tid + u * kThreads, t = i / gq, j = (i % gq) * kE;
      const size_t ik = (((size_t)b * T + t0 + t) * H + h) * kDK + j;
      const bool in = t0 + t < T;
      q[u] = in ? __ldg(reinterpret_cast<const uint4 *>(q_ + ik)) : make_uint4(0u, 0u, 0u, 0u);
      k[u] = in ? __ldg(reinterpret_cast<const uint4 *>(k_ + ik)) : make_uint4(0u, 0u, 0u, 0u);
    }
#pragma unroll
    for (int u = 0; u < kV; ++u) {
      const int i = tid + u * kThreads, t = i / (kNV / kE), c = (i % (kNV / kE)) * kE;
      const bool in = t0 + t < T;
      v[u] = in ? __ldg(reinterpret_cast<const uint4 *>(v_ + (((size_t)b * T + t0 + t) * H + h) * a.dv + c0 + c))
                : make_uint4(0u, 0u, 0u, 0u);
    }
    if (tid < kL) {
      const bool in = t0 + tid < T;
      const size_t ts = ((size_t)b * T + t0 + tid) * H + h;
      lf = in ? __ldg(a.f_pre + ts) : 0.f;
      ib = in ? __ldg(a.i_pre + ts) : -INFINITY;
    }
  }
  __device__ void commit(const Views<Tin> &s, int n) const {
    const int tid = threadIdx.x, gq = kDK / kE;
#pragma unroll
    for (int u = 0; u < kQK; ++u) {
      const int i = tid + u * kThreads, t = i / gq, j = (i % gq) * kE;
      *reinterpret_cast<uint4 *>(s.Qs + t * s.LDK + j) = q[u];
      *reinterpret_cast<uint4 *>(s.Ks + t * s.LDK + j) = k[u];
    }
#pragma unroll
    for (int u = 0; u < kV; ++u) {
      const int i = tid + u * kThreads, t = i / (kNV / kE), c = (i % (kNV / kE)) * kE;
      *reinterpret_cast<uint4 *>(s.Vs + t * s.LDV + c) = v[u];
    }
    if (tid < kL) {
      s.lf[tid] = tid < n ? log_sigmoid(lf) : 0.f;   // padding keeps log f = 0
      s.ib[tid] = ib;
    }
  }
};

// The state a CTA starts from: C0's 64 columns (or zeros), n0, m0 (or an empty memory).
template <typename Tin, int kDK>
__device__ __forceinline__ void load_initial_state(const Views<Tin> &s, const gdr_mlstm_args &a,
                                                   size_t bh, int c0) {
  const int tid = threadIdx.x, dv = a.dv;
  for (int i = tid; i < kDK * kNV; i += kThreads) {
    const int j = i / kNV, c = i % kNV;
    s.C[j * kLDN + c] = a.C0 ? a.C0[bh * kDK * dv + (size_t)j * dv + c0 + c] : 0.f;
  }
  for (int j = tid; j < kDK; j += kThreads) s.nn[j] = a.n0 ? a.n0[bh * kDK + j] : 0.f;
  if (tid == 0) *s.mcar = a.m0 ? a.m0[bh] : -INFINITY;
}

// The final state (C_T's 64 columns; n_T, m_T from the first column block).
template <typename Tin, int kDK>
__device__ __forceinline__ void store_final_state(const Views<Tin> &s, const gdr_mlstm_args &a,
                                                  size_t bh, int c0) {
  const int tid = threadIdx.x, dv = a.dv;
  if (a.C_T)
    for (int i = tid; i < kDK * kNV; i += kThreads) {
      const int j = i / kNV, c = i % kNV;
      a.C_T[bh * kDK * dv + (size_t)j * dv + c0 + c] = s.C[j * kLDN + c];
    }
  if (blockIdx.x == 0) {
    if (a.n_T)
      for (int j = tid; j < kDK; j += kThreads) a.n_T[bh * kDK + j] = s.nn[j];
    if (a.m_T && tid == 0) a.m_T[bh] = *s.mcar;
  }
}

// One CTA per (b, h, 64 value columns): readout and state update, chunk after chunk.
template <typename Tin, bool kSplit, int kDK>
__global__ void __launch_bounds__(kThreads, kSplit ? 1 : 2) mlstm_kernel(gdr_mlstm_args a) {
  extern __shared__ float sm[];
  const Views<Tin> s(sm, MlstmSmem(kDK, sizeof(Tin)));
  const int c0 = blockIdx.x * kNV, h = blockIdx.y, b = blockIdx.z;
  const int T = a.T, H = a.H, dv = a.dv, warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const size_t bh = (size_t)b * H + h;
  load_initial_state<Tin, kDK>(s, a, bh, c0);

  ChunkRegs<Tin, kDK> rg;
  rg.fetch(a, b, h, c0, 0);
  for (int t0 = 0; t0 < T; t0 += kL) {
    const int n = min(kL, T - t0);
    __syncthreads();   // the previous chunk is done with every buffer
    rg.commit(s, n);
    if (t0 + kL < T) rg.fetch(a, b, h, c0, t0 + kL);
    __syncthreads();
    if (warp == 0) scan_chunk(s.lf, s.ib, *s.mcar, s.A, s.mt, s.gt, lane);
    __syncthreads();
    readout<Tin, kSplit, kDK>(s, a.h + (((size_t)b * T + t0) * H + h) * dv + c0, (size_t)H * dv, n);
    __syncthreads();   // C and n are read above; they change below
    update_state<Tin, kSplit, kDK>(s);
  }
  __syncthreads();
  store_final_state<Tin, kDK>(s, a, bh, c0);
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
  if (mlstm_tc_supported(a)) return launch_mlstm_tc(a, stream);   // tcgen05 kernel (gdr_mlstm_tc.cu)
  if (a.dtype == GDR_BF16)
    return a.dk == 64 ? launch_typed<__nv_bfloat16, false, 64>(a, stream)
                      : launch_typed<__nv_bfloat16, false, 128>(a, stream);
  return a.dk == 64 ? launch_typed<float, true, 64>(a, stream) : launch_typed<float, true, 128>(a, stream);
}

}  // namespace gdr
