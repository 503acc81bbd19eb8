// gdr_bwd.cu -- reverse mode of the chunkwise forward (all forms; d_k, d_v in {64, 128}).
//
// The chunkwise forward ("Muir: Linear Attention with Sensitivity-Allocated Gating
// and Matched-Filter Readout", section 2.2, and section 4.2 eq. (10) for outputs and
// end state affine in the chunk's start state), generalized to a separate erase key
// z, in the storage orientation (S[j][c]: key j, value c).  One chunk of n <= 32
// tokens (rows t, s = 0..31, zero-padded past n) starting from state S:
//
//   lam[m]  = sum_{r < m} log w_r  (m = 0..32)       pi = exp(lam[32])
//   U~_t = u_t e^{lam[t]}   Q~_t = q_t e^{lam[t+1]}   K~_s = k_s e^{lam[32]-lam[s+1]}  (Z~ alike)
//   A   = stril(sum_j u_t z_s e^{lam[t]-lam[s+1]})    B  = stril(.. k_s ..)
//   M_z = tril(sum_j q_t z_s e^{lam[t+1]-lam[s+1]})   M_k = tril(.. k_s ..)
//   T = I + A,  E = T^-1 (U~ S + B V),   O = Q~ S + M_k V - M_z E
//   S_end = Diag(pi) S + K~^T V - Z~^T E
//
// With W = T^-1 U~, N = T^-1 B and X = Q~ - M_z W the end state and the outputs are
// affine in S:  S_end = Diag(pi) S - Z~^T (W S) + (K~ - N^T Z~)^T V,  O = X S + (..) V,
// so the adjoint of the start state is  dS = Diag(pi) dS_end - W^T (Z~ dS_end) + X^T dO.
// Both maps act on each value column separately.  Reverse mode, for one chunk given S
// and dS_end (= the adjoint of S_end):
//
//   dE  = -Z~ dS_end - M_z^T dO          dR = T^-T dE
//   dV  =  K~ dS_end + M_k^T dO + B^T dR
//   dM_k = tril(dO V^T)   dM_z = -tril(dO E^T)   dA = -stril(dR E^T)   dB = stril(dR V^T)
//   dq_t = e^{lam[t+1]} (dO S^T + dM_k K' + dM_z Z')_t          K'_s = k_s e^{-lam[s+1]}
//   du_t = e^{lam[t]}   (dR S^T + dA Z' + dB K')_t              (Z' alike)
//   dk_s = e^{-lam[s+1]} (e^{lam[32]} (V dS_end^T) + dB^T U~ + dM_k^T Q~)_s
//   dz_s = e^{-lam[s+1]} (-e^{lam[32]} (E dS_end^T) + dA^T U~ + dM_z^T Q~)_s
//
// The factors e^{-lam} are at most e^80: a chunk in which some channel decays by more
// than 80 nats forms the decayed products from the exact pairwise exponentials instead
// (the same bound and fallback as the forward kernels).  The gradient of the log-decays
// stays inside the chunk: lam enters the chunk through Q~, U~, K', Z' (rows t) and, at
// m = 32, through S_end, which is e^{lam[32]} times a quantity free of lam[32]; so with
// D_t = q dq - k dk - z dz + u du (the form's effective q, k, z, u)
//   dlog_w_t = sum_{r = t}^{31} D_r - u_t du_t + diag(S_end^T dS_end),
// and for GDN-2 (u = alpha b k) the direct dependence of u on log alpha_t adds back
// u_t du_t.  (Summed over the chunks this is the telescoped sequence-wide form, but no
// error accumulates along the sequence.)
//
// Kernels: bwd_prep (per chunk: W, Z~, K~ - N^T Z~, X, pi), bwd_chain (per (b, h) and
// 64 value columns: the forward chain storing every chunk-start state and the final
// state, then the adjoint chain storing every dS_end; the next chunk's records are
// loaded into registers while the current one is applied) and bwd_grads (per chunk:
// every token gradient).  Products run as warp-level tf32 MMAs with fp32 accumulate,
// every operand in shared memory (S and dS_end staged in slabs); bf16 inputs take one
// tf32 product, fp32 inputs three (hi*hi + hi*lo + lo*hi), which keeps fp32 accuracy.
#include "gdr_internal.cuh"
#include "gdr_tc_common.cuh"
#include "gdr_warp_mma.cuh"

namespace gdr {
namespace {

using tc::kMaxChunkDecay;
using wmma_tf32::for_acc;
using wmma_tf32::mma_seg;
using wmma_tf32::zero_acc;

constexpr int kC = kBwdChunk;    // 32
constexpr int kLDC = kC + 4;     // row stride of the C x C matrices
constexpr int kThreads = 256;    // prep and grads kernels
constexpr int kWarps = kThreads / 32;
constexpr int kNC = 64;          // value columns per chain CTA
constexpr int kChainThreads = 256;
constexpr int kLDN = kNC + 4;
constexpr int kSlab = 16;        // value columns of S / dS_end staged per step (grads)
constexpr int kLDS = kSlab + 4;

// Eight consecutive elements (16-byte aligned) widened to fp32.
__device__ __forceinline__ void ld8(const __nv_bfloat16 *p, size_t i, float (&f)[8]) {
  tc::unpack8(__ldg(reinterpret_cast<const uint4 *>(p + i)), f);
}
__device__ __forceinline__ void ld8(const float *p, size_t i, float (&f)[8]) {
  const float4 a = __ldg(reinterpret_cast<const float4 *>(p + i));
  const float4 b = __ldg(reinterpret_cast<const float4 *>(p + i + 4));
  f[0] = a.x; f[1] = a.y; f[2] = a.z; f[3] = a.w;
  f[4] = b.x; f[5] = b.y; f[6] = b.z; f[7] = b.w;
}
__device__ __forceinline__ void st8(float *p, const float (&f)[8]) {
  *reinterpret_cast<float4 *>(p) = make_float4(f[0], f[1], f[2], f[3]);
  *reinterpret_cast<float4 *>(p + 4) = make_float4(f[4], f[5], f[6], f[7]);
}

// Register-held copy of up to N float4 per thread of a rows x cols fp32 block: the
// next slab is loaded while the current one is used, then stored to shared memory.
template <int N>
struct Prefetch {
  float4 x[N];
  __device__ __forceinline__ void load(const float *src, size_t gs, int rows, int cols) {
    const int c4 = cols / 4, n = rows * c4;
#pragma unroll
    for (int u = 0; u < N; ++u) {
      const int i = threadIdx.x + u * blockDim.x;
      if (i < n) x[u] = __ldg(reinterpret_cast<const float4 *>(src + (size_t)(i / c4) * gs + 4 * (i % c4)));
    }
  }
  __device__ __forceinline__ void store(float *dst, int ls, int rows, int cols, const float *rs) const {
    const int c4 = cols / 4, n = rows * c4;
#pragma unroll
    for (int u = 0; u < N; ++u) {
      const int i = threadIdx.x + u * blockDim.x;
      if (i < n) {
        const int r = i / c4, c = 4 * (i % c4);
        float4 y = x[u];
        if (rs) {
          const float f = rs[r];
          y.x *= f; y.y *= f; y.z *= f; y.w *= f;
        }
        *reinterpret_cast<float4 *>(dst + r * ls + c) = y;
      }
    }
  }
};

// ---------------------------------------------------------------------------
// Shared-memory layout of the per-chunk kernels (floats).  Row strides dk + 4 and
// dv + 4 keep the MMA fragment loads conflict-free.
// ---------------------------------------------------------------------------
struct ChunkSmem {
  int LDK, LDV;
  size_t lam, Q, K, U, Z, V, dO, E, dR, Tmp, A, Bm, Mk, Mz, Ti, dA, dBm, dMk, dMz, pi, dc, flag,
      total;
  __host__ __device__ ChunkSmem(int dk, int dv, bool grads) {
    LDK = dk + 4;
    LDV = dv + 4;
    const size_t tk = (size_t)kC * LDK, tv = (size_t)kC * LDV, cc = (size_t)kC * kLDC;
    size_t off = 0;
    lam = off; off += (size_t)(kC + 1) * LDK;
    Q = off; off += tk;
    K = off; off += tk;
    U = off; off += tk;
    Z = off; off += tk;
    // A, B, M_z, T^-1, M_k contiguous: dead by the token-gradient phase, where they
    // hold the staged slabs of S and dS_end (2 x dk x kLDS floats <= 5 C x kLDC)
    A = off; off += cc;
    Bm = off; off += cc;
    Mz = off; off += cc;
    Ti = off; off += cc;
    if (grads) {
      Mk = off; off += cc;
      V = off; off += tv;
      dO = off; off += tv;
      E = off; off += tv;
      dR = off; off += tv;
      Tmp = off; off += (tk > tv ? tk : tv);
      dA = off; off += cc;
      dBm = off; off += cc;
      dMk = off; off += cc;
      dMz = off; off += cc;
    } else {
      Tmp = U;  // W replaces U~ once it is formed
      V = dO = E = dR = Mk = dA = dBm = dMk = dMz = 0;
    }
    pi = off; off += dk;
    dc = off; off += kC;
    flag = off; off += dk;   // grads: diag(S_end^T dS_end)
    total = off;
  }
};

// Loads one chunk (rows past n zero), forms lam and pi, decides the exact path and,
// on the pivot path, scales Q -> Q~, U -> U~, K -> K', Z -> Z' in place.  With
// `grads` also loads V (GDN-2: wg (.) v) and dO.  Returns the exact-path flag.
template <typename Tin, int kDK, int kDV>
__device__ bool load_chunk(const BwdParams &p, const ChunkSmem &L, float *sm, int b, int h,
                           int t0, int n, bool grads) {
  constexpr int dk = kDK, dv = kDV;
  const int T = p.T, H = p.H, LDK = L.LDK, LDV = L.LDV;
  const int tid = threadIdx.x;
  const Tin *q = static_cast<const Tin *>(p.q), *k = static_cast<const Tin *>(p.k);
  const Tin *v = static_cast<const Tin *>(p.v), *e1 = static_cast<const Tin *>(p.e1);
  const Tin *e2 = static_cast<const Tin *>(p.e2);
  float *lam = sm + L.lam, *Q = sm + L.Q, *K = sm + L.K, *U = sm + L.U, *Z = sm + L.Z;
  const int gk = dk / 8;
  for (int i = tid; i < kC * gk; i += blockDim.x) {
    const int t = i / gk, j0 = 8 * (i % gk);
    float qq[8], kk[8], lw[8], u[8], z[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) qq[e] = kk[e] = lw[e] = u[e] = z[e] = 0.f;
    if (t < n) {
      const size_t tok = ((size_t)b * T + t0 + t) * H + h;
      const size_t ik = tok * dk + j0;
      ld8(p.log_w, ik, lw);
      ld8(q, ik, qq);
      ld8(k, ik, kk);
      switch (p.form) {
        case GDR_FORM_GENERAL:
          ld8(e1, ik, u);
          ld8(e2, ik, z);
          break;
        case GDR_FORM_GDN2:
          ld8(e1, ik, u);
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            u[e] *= __expf(lw[e]) * kk[e];
            z[e] = kk[e];
          }
          break;
        case GDR_FORM_RWKV7: {
          const float cc = ld_in(e2, tok);
          ld8(e1, ik, z);
#pragma unroll
          for (int e = 0; e < 8; ++e) u[e] = cc * z[e];
          break;
        }
        default:
          break;
      }
    }
    st8(lam + (t + 1) * LDK + j0, lw);
    st8(Q + t * LDK + j0, qq);
    st8(K + t * LDK + j0, kk);
    st8(U + t * LDK + j0, u);
    st8(Z + t * LDK + j0, z);
  }
  if (grads) {
    float *V = sm + L.V, *dO = sm + L.dO;
    const bool gated = p.form == GDR_FORM_GDN2 && e2 != nullptr;
    const int gv = dv / 8;
    for (int i = tid; i < kC * gv; i += blockDim.x) {
      const int t = i / gv, c0 = 8 * (i % gv);
      float x[8], g[8];
#pragma unroll
      for (int e = 0; e < 8; ++e) x[e] = g[e] = 0.f;
      if (t < n) {
        const size_t iv = (((size_t)b * T + t0 + t) * H + h) * dv + c0;
        ld8(v, iv, x);
        if (gated) {
          float wg[8];
          ld8(e2, iv, wg);
#pragma unroll
          for (int e = 0; e < 8; ++e) x[e] *= wg[e];
        }
        ld8(p.dO, iv, g);
      }
      st8(V + t * LDV + c0, x);
      st8(dO + t * LDV + c0, g);
    }
    if (tid < kC) sm[L.dc + tid] = 0.f;
  }
  __syncthreads();
  bool strong = false;
  for (int j = tid; j < dk; j += blockDim.x) {
    float acc = 0.f;
    lam[j] = 0.f;
    for (int t = 1; t <= kC; ++t) {
      acc += lam[t * LDK + j];
      lam[t * LDK + j] = acc;
    }
    sm[L.pi + j] = __expf(acc);
    strong |= acc < -kMaxChunkDecay;
  }
  const bool exact = __syncthreads_or(strong) != 0;
  if (!exact) {
    for (int i = tid; i < kC * dk; i += blockDim.x) {
      const int t = i / dk, j = i % dk;
      const float l0 = lam[t * LDK + j], l1 = lam[(t + 1) * LDK + j];
      Q[t * LDK + j] *= __expf(l1);
      U[t * LDK + j] *= __expf(l0);
      const float g = __expf(-l1);
      K[t * LDK + j] *= g;
      Z[t * LDK + j] *= g;
    }
  }
  __syncthreads();
  return exact;
}

// The chunk's C x C matrices A, B (strictly lower), M_z and, with `with_mk`, M_k
// (lower, diagonal included).  Ends with a CTA barrier.
template <bool kSplit, int dk>
__device__ void chunk_matrices(const ChunkSmem &L, float *sm, bool exact, bool with_mk) {
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31, LDK = L.LDK;
  const float *lam = sm + L.lam, *Q = sm + L.Q, *K = sm + L.K, *U = sm + L.U, *Z = sm + L.Z;
  if (!exact) {
    // product p: 0 A = U~ Z'^T, 1 B = U~ K'^T, 2 M_z = Q~ Z'^T, 3 M_k = Q~ K'^T
    const int np = with_mk ? 4 : 3;
    for (int wt = warp; wt < 2 * np; wt += kWarps) {
      const int pr = wt >> 1, r0 = 16 * (wt & 1);
      const float *X = pr < 2 ? U : Q;
      const float *Y = (pr & 1) ? K : Z;
      float *out = sm + (pr == 0 ? L.A : pr == 1 ? L.Bm : pr == 2 ? L.Mz : L.Mk);
      float acc[4][4];
      zero_acc(acc);
      mma_seg<kSplit>(acc, r0, 0, 0, dk, [&](int m, int kk) { return X[m * LDK + kk]; },
                      [&](int kk, int nn) { return Y[nn * LDK + kk]; }, lane);
      const bool strict = pr < 2;
      for_acc(acc, r0, 0, lane, [&](int r, int c, float x) {
        out[r * kLDC + c] = (c < r || (!strict && c == r)) ? x : 0.f;
      });
    }
  } else {
    for (int i = tid; i < kC * kC; i += blockDim.x) {
      const int t = i / kC, s = i % kC;
      float a = 0.f, bm = 0.f, mz = 0.f, mk = 0.f;
      if (s <= t) {
        const float *lt = lam + t * LDK, *lt1 = lam + (t + 1) * LDK, *ls1 = lam + (s + 1) * LDK;
        for (int j = 0; j < dk; ++j) {
          const float ks = K[s * LDK + j], zs = Z[s * LDK + j];
          const float dq = __expf(lt1[j] - ls1[j]) * Q[t * LDK + j];
          mz += dq * zs;
          mk += dq * ks;
          if (s < t) {
            const float du = __expf(lt[j] - ls1[j]) * U[t * LDK + j];
            a += du * zs;
            bm += du * ks;
          }
        }
      }
      sm[L.A + t * kLDC + s] = a;
      sm[L.Bm + t * kLDC + s] = bm;
      sm[L.Mz + t * kLDC + s] = mz;
      if (with_mk) sm[L.Mk + t * kLDC + s] = mk;
    }
  }
  __syncthreads();
}

// Ti = (I + A)^-1 by forward substitution, 8 lanes per column.  Ends with a barrier.
__device__ void invert_unit_lower32(const float *A, float *Ti) {
  const int tid = threadIdx.x, s = tid >> 3, r = tid & 7;
  for (int t = 0; t < kC; ++t) {
    float acc = 0.f;
    for (int m = s + r; m < t; m += 8) acc += A[t * kLDC + m] * Ti[m * kLDC + s];
    acc += __shfl_xor_sync(0xffffffffu, acc, 1);
    acc += __shfl_xor_sync(0xffffffffu, acc, 2);
    acc += __shfl_xor_sync(0xffffffffu, acc, 4);
    if (r == 0) Ti[t * kLDC + s] = t < s ? 0.f : (t == s ? 1.f : -acc);
    __syncwarp();
  }
  __syncthreads();
}

// Decayed key / query / erase vectors from the chunk tiles: pivot path (scaled tiles)
// or exact path (raw tiles times one exponential).
struct Decayed {
  const float *lam, *pi;
  int LDK;
  bool exact;
  // U~_t = u_t e^{lam[t]}
  __device__ __forceinline__ float ut(const float *U, int t, int j) const {
    return exact ? U[t * LDK + j] * __expf(lam[t * LDK + j]) : U[t * LDK + j];
  }
  // Q~_t = q_t e^{lam[t+1]}
  __device__ __forceinline__ float qt(const float *Q, int t, int j) const {
    return exact ? Q[t * LDK + j] * __expf(lam[(t + 1) * LDK + j]) : Q[t * LDK + j];
  }
  // K~_s = k_s e^{lam[32] - lam[s+1]} (pivot tile holds K' = k e^{-lam[s+1]})
  __device__ __forceinline__ float end(const float *K, int s, int j) const {
    return exact ? K[s * LDK + j] * __expf(lam[kC * LDK + j] - lam[(s + 1) * LDK + j])
                 : K[s * LDK + j] * pi[j];
  }
};

// ---------------------------------------------------------------------------
// bwd_prep: per chunk W = T^-1 U~, Z~, K~ - N^T Z~ (N = T^-1 B), X = Q~ - M_z W, pi.
// Record layout [W | Z~ | K~ - N^T Z~ | X] (32 x dk each, row-major) then pi [dk].
// ---------------------------------------------------------------------------
template <typename Tin, bool kSplit, int kDK, int kDV>
__global__ void __launch_bounds__(kThreads, kSplit ? 1 : 2) bwd_prep_kernel(BwdParams p) {
  extern __shared__ float sm[];
  constexpr int dk = kDK;
  const ChunkSmem L(kDK, kDV, false);
  const int c = blockIdx.x, h = blockIdx.y, b = blockIdx.z, LDK = L.LDK;
  const int t0 = c * kC, n = min(kC, p.T - t0);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const bool exact = load_chunk<Tin, kDK, kDV>(p, L, sm, b, h, t0, n, false);
  chunk_matrices<kSplit, kDK>(L, sm, exact, false);
  invert_unit_lower32(sm + L.A, sm + L.Ti);

  const size_t cid = ((size_t)b * p.H + h) * p.nc + c;
  float *rec = p.rec + cid * (4 * kC * dk + dk);
  const Decayed D{sm + L.lam, sm + L.pi, LDK, exact};
  const float *Ti = sm + L.Ti, *U = sm + L.U, *Bm = sm + L.Bm;
  float *W = sm + L.Tmp, *Nm = sm + L.A;  // W over U~, N over A (both dead once read)
  // W = Ti U~ (record and shared copy) and N = Ti B: every warp computes its tiles,
  // then, after a barrier, stores them over the operands
  const int ntn = dk / 32, ntiles = 2 * ntn + 2;
  float acc[2][4][4];
  for (int u = 0; u < 2; ++u) {
    const int wt = warp + u * kWarps;
    zero_acc(acc[u]);
    if (wt < 2 * ntn) {
      const int r0 = 16 * (wt / ntn), c0 = 32 * (wt % ntn);
      // the exact and pivot paths as separate loops, so that the operand is a plain load
      // on the pivot path
      auto ti = [&](int m, int kk) { return Ti[m * kLDC + kk]; };
      if (exact)
        mma_seg<kSplit>(acc[u], r0, c0, 0, kC, ti, [&](int kk, int nn) { return D.ut(U, kk, nn); }, lane);
      else
        mma_seg<kSplit>(acc[u], r0, c0, 0, kC, ti, [&](int kk, int nn) { return U[kk * LDK + nn]; }, lane);
    } else if (wt < ntiles) {
      const int r0 = 16 * (wt - 2 * ntn);
      mma_seg<kSplit>(acc[u], r0, 0, 0, kC, [&](int m, int kk) { return Ti[m * kLDC + kk]; },
                      [&](int kk, int nn) { return Bm[kk * kLDC + nn]; }, lane);
    }
  }
  __syncthreads();
  for (int u = 0; u < 2; ++u) {
    const int wt = warp + u * kWarps;
    if (wt < 2 * ntn) {
      const int r0 = 16 * (wt / ntn), c0 = 32 * (wt % ntn);
      for_acc(acc[u], r0, c0, lane, [&](int r, int cc, float x) {
        W[r * LDK + cc] = x;
        rec[r * dk + cc] = x;
      });
    } else if (wt < ntiles) {
      const int r0 = 16 * (wt - 2 * ntn);
      for_acc(acc[u], r0, 0, lane, [&](int r, int cc, float x) { Nm[r * kLDC + cc] = x; });
    }
  }
  __syncthreads();
  // K~ - N^T Z~ and X = Q~ - M_z W; Z~ and pi
  const float *Z = sm + L.Z, *K = sm + L.K, *Q = sm + L.Q, *Mz = sm + L.Mz;
  for (int wt = warp; wt < 4 * ntn; wt += kWarps) {
    const int which = wt / (2 * ntn), w2 = wt % (2 * ntn);
    const int r0 = 16 * (w2 / ntn), c0 = 32 * (w2 % ntn);
    float acc[4][4];
    zero_acc(acc);
    if (which == 0) {
      auto nt = [&](int m, int kk) { return Nm[kk * kLDC + m]; };
      if (exact)
        mma_seg<kSplit>(acc, r0, c0, 0, kC, nt, [&](int kk, int nn) { return D.end(Z, kk, nn); }, lane);
      else
        mma_seg<kSplit>(acc, r0, c0, 0, kC, nt, [&](int kk, int nn) { return Z[kk * LDK + nn] * D.pi[nn]; },
                        lane);
      for_acc(acc, r0, c0, lane, [&](int r, int cc, float x) {
        rec[2 * kC * dk + r * dk + cc] = D.end(K, r, cc) - x;
      });
    } else {
      mma_seg<kSplit>(acc, r0, c0, 0, kC, [&](int m, int kk) { return Mz[m * kLDC + kk]; },
                      [&](int kk, int nn) { return W[kk * LDK + nn]; }, lane);
      for_acc(acc, r0, c0, lane, [&](int r, int cc, float x) {
        rec[3 * kC * dk + r * dk + cc] = D.qt(Q, r, cc) - x;
      });
    }
  }
  for (int i = tid; i < kC * dk; i += kThreads) {
    const int t = i / dk, j = i % dk;
    rec[kC * dk + i] = D.end(Z, t, j);
  }
  for (int j = tid; j < dk; j += kThreads) rec[4 * kC * dk + j] = sm[L.pi + j];
}

// ---------------------------------------------------------------------------
// bwd_chain: one CTA per (64 value columns, h, b).  Forward chain (stores every
// chunk-start state and, as entry nc, the final state), then the adjoint chain
// (stores every dS_end; ends with dS0).  Chunk c + 1's records and V / dO slice are
// loaded into registers while chunk c is applied.
// ---------------------------------------------------------------------------
struct ChainSmem {
  int LDK;
  size_t S, Rw, Rz, Rk, Vs, Av, pi, total;
  __host__ __device__ explicit ChainSmem(int dk) {
    LDK = dk + 4;
    size_t off = 0;
    S = off; off += (size_t)dk * kLDN;
    Rw = off; off += (size_t)kC * LDK;
    Rz = off; off += (size_t)kC * LDK;
    Rk = off; off += (size_t)kC * LDK;
    Vs = off; off += (size_t)kC * kLDN;
    Av = off; off += (size_t)kC * kLDN;
    pi = off; off += dk;
    total = off;
  }
};

// Registers of one chunk's prefetch: three record tiles (32 x dk, float4 per thread
// slot), the 32 x 64 V or dO slice (8 values per thread) and pi.
template <int kMaxDK>
struct ChainRegs {
  static constexpr int kRec = kC * kMaxDK / 4 / kChainThreads;  // float4 per tile
  float4 r[3][kRec];
  float x[8];
  float4 pi4;
};

template <typename Tin, bool kSplit, int kDK>
__global__ void __launch_bounds__(kChainThreads, 1) bwd_chain_kernel(BwdParams p) {
  extern __shared__ float sm[];
  constexpr int dk = kDK;
  const int dv = p.dv, T = p.T, H = p.H, nc = p.nc;
  const ChainSmem L(dk);
  const int LDK = L.LDK;
  const int c0 = blockIdx.x * kNC, h = blockIdx.y, b = blockIdx.z;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  constexpr int nw = kChainThreads / 32;
  float *S = sm + L.S, *Rw = sm + L.Rw, *Rz = sm + L.Rz, *Rk = sm + L.Rk, *Vs = sm + L.Vs;
  float *Av = sm + L.Av, *pi = sm + L.pi;
  const Tin *v = static_cast<const Tin *>(p.v), *e2 = static_cast<const Tin *>(p.e2);
  const size_t bh = (size_t)b * H + h, sbase = bh * dk * dv;
  const size_t rec_floats = 4 * (size_t)kC * dk + dk;
  const bool gated = p.form == GDR_FORM_GDN2 && e2 != nullptr;
  ChainRegs<dk> R;
  const int xt = tid >> 3, xc = 8 * (tid & 7);   // this thread's V / dO slot: row, 8 columns

  // prefetch chunk c: W, Z~, third tile (2: K~ - N^T Z~, 3: X), pi, and V (fwd) or dO
  auto fetch = [&](int c, int third, bool fwd) {
    const float4 *rec = reinterpret_cast<const float4 *>(p.rec + (bh * nc + c) * rec_floats);
    constexpr int q4 = kC * dk / 4;
#pragma unroll
    for (int u = 0; u < ChainRegs<dk>::kRec; ++u) {
      const int i = tid + u * kChainThreads;
      R.r[0][u] = __ldg(rec + i);
      R.r[1][u] = __ldg(rec + q4 + i);
      R.r[2][u] = __ldg(rec + third * q4 + i);
    }
    if (tid < dk / 4) R.pi4 = __ldg(rec + 4 * q4 + tid);
    const int t0 = c * kC;
#pragma unroll
    for (int e = 0; e < 8; ++e) R.x[e] = 0.f;
    if (t0 + xt < T) {
      const size_t iv = (((size_t)b * T + t0 + xt) * H + h) * dv + c0 + xc;
      if (fwd) {
        ld8(v, iv, R.x);
        if (gated) {
          float wg[8];
          ld8(e2, iv, wg);
#pragma unroll
          for (int e = 0; e < 8; ++e) R.x[e] *= wg[e];
        }
      } else {
        ld8(p.dO, iv, R.x);
      }
    }
  };
  auto commit = [&]() {
#pragma unroll
    for (int u = 0; u < ChainRegs<dk>::kRec; ++u) {
      const int i = 4 * (tid + u * kChainThreads), t = i / dk, j = i % dk;
      *reinterpret_cast<float4 *>(Rw + t * LDK + j) = R.r[0][u];
      *reinterpret_cast<float4 *>(Rz + t * LDK + j) = R.r[1][u];
      *reinterpret_cast<float4 *>(Rk + t * LDK + j) = R.r[2][u];
    }
    if (tid < dk / 4) *reinterpret_cast<float4 *>(pi + 4 * tid) = R.pi4;
    st8(Vs + xt * kLDN + xc, R.x);
  };
  // one chunk: Av = P S (P = W forward, Z~ adjoint); S = Diag(pi) S - M1^T Av + M2^T X
  auto apply = [&](const float *P, const float *M1, const float *M2) {
    if (warp < 4) {
      const int r0 = 16 * (warp >> 1), cc0 = 32 * (warp & 1);
      float acc[4][4];
      zero_acc(acc);
      mma_seg<kSplit>(acc, r0, cc0, 0, dk, [&](int m, int kk) { return P[m * LDK + kk]; },
                      [&](int kk, int nn) { return S[kk * kLDN + nn]; }, lane);
      for_acc(acc, r0, cc0, lane, [&](int r, int cc, float x) { Av[r * kLDN + cc] = x; });
    }
    __syncthreads();
    for (int wt = warp; wt < dk / 8; wt += nw) {
      const int r0 = 16 * (wt >> 1), cc0 = 32 * (wt & 1);
      float acc[4][4];
      zero_acc(acc);
      mma_seg<kSplit>(acc, r0, cc0, 0, kC, [&](int m, int kk) { return -M1[kk * LDK + m]; },
                      [&](int kk, int nn) { return Av[kk * kLDN + nn]; }, lane);
      mma_seg<kSplit>(acc, r0, cc0, 0, kC, [&](int m, int kk) { return M2[kk * LDK + m]; },
                      [&](int kk, int nn) { return Vs[kk * kLDN + nn]; }, lane);
      for_acc(acc, r0, cc0, lane, [&](int r, int cc, float x) {
        S[r * kLDN + cc] = pi[r] * S[r * kLDN + cc] + x;
      });
    }
  };
  auto store_state = [&](float *dst) {
    for (int i = tid; i < dk * kNC / 4; i += kChainThreads) {
      const int j = (4 * i) / kNC, cc = (4 * i) % kNC;
      *reinterpret_cast<float4 *>(dst + (size_t)j * dv + c0 + cc) =
          *reinterpret_cast<const float4 *>(S + j * kLDN + cc);
    }
  };
  auto load_state = [&](const float *src) {
    for (int i = tid; i < dk * kNC / 4; i += kChainThreads) {
      const int j = (4 * i) / kNC, cc = (4 * i) % kNC;
      *reinterpret_cast<float4 *>(S + j * kLDN + cc) =
          src ? __ldg(reinterpret_cast<const float4 *>(src + (size_t)j * dv + c0 + cc))
              : make_float4(0.f, 0.f, 0.f, 0.f);
    }
  };

  // ---- forward chain
  load_state(p.S0 ? p.S0 + sbase : nullptr);
  fetch(0, 2, true);
  for (int c = 0; c < nc; ++c) {
    __syncthreads();
    commit();
    store_state(p.states + (bh * (nc + 1) + c) * dk * dv);
    if (c + 1 < nc) fetch(c + 1, 2, true);
    __syncthreads();
    apply(Rw, Rz, Rk);
  }
  __syncthreads();
  store_state(p.states + (bh * (nc + 1) + nc) * dk * dv);

  // ---- adjoint chain
  load_state(p.dS_T ? p.dS_T + sbase : nullptr);
  fetch(nc - 1, 3, false);
  for (int c = nc - 1; c >= 0; --c) {
    __syncthreads();
    commit();
    store_state(p.adj + (bh * nc + c) * dk * dv);
    if (c > 0) fetch(c - 1, 3, false);
    __syncthreads();
    apply(Rz, Rw, Rk);
  }
  __syncthreads();
  if (p.gS0) store_state(p.gS0 + sbase);
}

// ---------------------------------------------------------------------------
// bwd_grads: one CTA per (chunk, h, b).  Every token gradient of the chunk and the
// chunk's log-decay gradients.  S and dS_end are staged into shared memory in slabs.
// ---------------------------------------------------------------------------
template <typename Tin, bool kSplit, int kDK, int kDV>
__global__ void __launch_bounds__(kThreads, 1) bwd_grads_kernel(BwdParams p) {
  extern __shared__ float sm[];
  constexpr int dk = kDK, dv = kDV;
  const ChunkSmem L(kDK, kDV, true);
  const int c = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int T = p.T, H = p.H, LDK = L.LDK, LDV = L.LDV;
  const int t0 = c * kC, n = min(kC, T - t0);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const size_t bh = (size_t)b * H + h, cid = bh * p.nc + c;
  const float *S = p.states + (bh * (p.nc + 1) + c) * dk * dv;       // chunk-start state
  const float *Send = S + (size_t)dk * dv;                             // chunk-end state
  const float *G = p.adj + cid * dk * dv;                              // its adjoint

  const bool exact = load_chunk<Tin, kDK, kDV>(p, L, sm, b, h, t0, n, true);
  // S's first 32 rows, in flight while the chunk matrices and T^-1 are formed
  Prefetch<4> pfS;
  pfS.load(S, dv, kC, dv);
  chunk_matrices<kSplit, kDK>(L, sm, exact, true);
  invert_unit_lower32(sm + L.A, sm + L.Ti);

  const float *lam = sm + L.lam, *pi = sm + L.pi;
  const float *Q = sm + L.Q, *K = sm + L.K, *U = sm + L.U, *Z = sm + L.Z;
  const float *V = sm + L.V, *dO = sm + L.dO;
  float *E = sm + L.E, *dR = sm + L.dR, *Tmp = sm + L.Tmp;
  const float *Bm = sm + L.Bm, *Mk = sm + L.Mk, *Mz = sm + L.Mz, *Ti = sm + L.Ti;
  float *dA = sm + L.dA, *dBm = sm + L.dBm, *dMk = sm + L.dMk, *dMz = sm + L.dMz;
  float *xcv = sm + L.flag;
  float *Lloc = sm + L.A;   // per-token local decay-gradient term, after the slab loop
  const Decayed D{lam, pi, LDK, exact};
  const int nvt = dv / 32, nkt = dk / 32;
  const float *gscale = exact ? nullptr : pi;   // dS_end rows scaled by pi on the pivot path
  // this warp's 16 x 32 tile of a 32 x dv output (dv <= 128: at most one per warp)
  const bool vt_own = warp < 2 * nvt;
  const int vr0 = 16 * (warp / max(nvt, 1)), vc0 = 32 * (warp % max(nvt, 1));

  // R = U~ S + B V (into Tmp): S staged 32 rows at a time into dR (free until dR)
  {
    float acc[4][4];
    zero_acc(acc);
    Prefetch<4> &pf = pfS;
    for (int kk0 = 0; kk0 < dk; kk0 += kC) {
      pf.store(dR, LDV, kC, dv, nullptr);
      __syncthreads();
      if (kk0 + kC < dk) pf.load(S + (size_t)(kk0 + kC) * dv, dv, kC, dv);
      if (vt_own) {
        auto st = [&](int kk, int nn) { return dR[kk * LDV + nn]; };
        if (exact)
          mma_seg<kSplit>(acc, vr0, vc0, 0, kC, [&](int m, int kk) { return D.ut(U, m, kk0 + kk); }, st, lane);
        else
          mma_seg<kSplit>(acc, vr0, vc0, 0, kC, [&](int m, int kk) { return U[m * LDK + kk0 + kk]; }, st, lane);
      }
      __syncthreads();
    }
    if (vt_own) {
      mma_seg<kSplit>(acc, vr0, vc0, 0, kC, [&](int m, int kk) { return Bm[m * kLDC + kk]; },
                      [&](int kk, int nn) { return V[kk * LDV + nn]; }, lane);
      for_acc(acc, vr0, vc0, lane, [&](int r, int cc, float x) { Tmp[r * LDV + cc] = x; });
    }
  }
  // dS_end's first 32 rows, in flight during E = T^-1 R
  Prefetch<4> pfG;
  pfG.load(G, dv, kC, dv);
  __syncthreads();
  // E = T^-1 R
  if (vt_own) {
    float acc[4][4];
    zero_acc(acc);
    mma_seg<kSplit>(acc, vr0, vc0, 0, kC, [&](int m, int kk) { return Ti[m * kLDC + kk]; },
                    [&](int kk, int nn) { return Tmp[kk * LDV + nn]; }, lane);
    for_acc(acc, vr0, vc0, lane, [&](int r, int cc, float x) { E[r * LDV + cc] = x; });
  }
  __syncthreads();
  // dE = -(Z~ dS_end + M_z^T dO) (into Tmp) and the K~ dS_end part of dV (kept in
  // registers): dS_end staged into dR once for both
  float accv[4][4];
  zero_acc(accv);
  {
    float acc[4][4];
    zero_acc(acc);
    Prefetch<4> &pf = pfG;
    for (int kk0 = 0; kk0 < dk; kk0 += kC) {
      pf.store(dR, LDV, kC, dv, gscale ? gscale + kk0 : nullptr);
      __syncthreads();
      if (kk0 + kC < dk) pf.load(G + (size_t)(kk0 + kC) * dv, dv, kC, dv);
      if (vt_own) {
        auto gs = [&](int kk, int nn) { return dR[kk * LDV + nn]; };
        if (exact) {
          mma_seg<kSplit>(acc, vr0, vc0, 0, kC, [&](int m, int kk) { return D.end(Z, m, kk0 + kk); }, gs, lane);
          mma_seg<kSplit>(accv, vr0, vc0, 0, kC, [&](int m, int kk) { return D.end(K, m, kk0 + kk); }, gs, lane);
        } else {
          mma_seg<kSplit>(acc, vr0, vc0, 0, kC, [&](int m, int kk) { return Z[m * LDK + kk0 + kk]; }, gs, lane);
          mma_seg<kSplit>(accv, vr0, vc0, 0, kC, [&](int m, int kk) { return K[m * LDK + kk0 + kk]; }, gs, lane);
        }
      }
      __syncthreads();
    }
    if (vt_own) {
      mma_seg<kSplit>(acc, vr0, vc0, 0, kC, [&](int m, int kk) { return Mz[kk * kLDC + m]; },
                      [&](int kk, int nn) { return dO[kk * LDV + nn]; }, lane);
      for_acc(acc, vr0, vc0, lane, [&](int r, int cc, float x) { Tmp[r * LDV + cc] = -x; });
    }
  }
  __syncthreads();
  // dR = T^-T dE
  if (vt_own) {
    float acc[4][4];
    zero_acc(acc);
    mma_seg<kSplit>(acc, vr0, vc0, 0, kC, [&](int m, int kk) { return Ti[kk * kLDC + m]; },
                    [&](int kk, int nn) { return Tmp[kk * LDV + nn]; }, lane);
    for_acc(acc, vr0, vc0, lane, [&](int r, int cc, float x) { dR[r * LDV + cc] = x; });
  }
  __syncthreads();
  // the first slabs of S^T and dS_end^T for the token gradients, in flight during dV and
  // the C x C gradients: kDepth slabs ahead (two where the registers allow)
  constexpr int kDepth = kSplit ? 1 : 2;
  Prefetch<2> pS[kDepth], pG[kDepth];
#pragma unroll
  for (int d = 0; d < kDepth; ++d)
    if (d * kSlab < dv) {
      pS[d].load(S + d * kSlab, dv, dk, kSlab);
      pG[d].load(G + d * kSlab, dv, dk, kSlab);
    }
  // dV = K~ dS_end (above) + M_k^T dO + B^T dR (written out)
  {
    const Tin *v = static_cast<const Tin *>(p.v), *e2 = static_cast<const Tin *>(p.e2);
    const bool gated = p.form == GDR_FORM_GDN2 && e2 != nullptr;
    float acc[4][4];
    if (vt_own) {
      mma_seg<kSplit>(accv, vr0, vc0, 0, kC, [&](int m, int kk) { return Mk[kk * kLDC + m]; },
                      [&](int kk, int nn) { return dO[kk * LDV + nn]; }, lane);
      mma_seg<kSplit>(accv, vr0, vc0, 0, kC, [&](int m, int kk) { return Bm[kk * kLDC + m]; },
                      [&](int kk, int nn) { return dR[kk * LDV + nn]; }, lane);
      // the write-gate and value entries of this thread's 16 outputs, loaded together
      const int g = lane >> 2, tq = lane & 3;
      float pw[4][4], pv[4][4];
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int r = vr0 + g + 8 * (e >> 1), cc = vc0 + 8 * i + 2 * tq + (e & 1);
          const size_t iv = (((size_t)b * T + t0 + r) * H + h) * dv + cc;
          const bool in = gated && r < n;
          pw[i][e] = in ? ld_in(e2, iv) : 0.f;
          pv[i][e] = in ? ld_in(v, iv) : 0.f;
        }
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int r = vr0 + g + 8 * (e >> 1), cc = vc0 + 8 * i + 2 * tq + (e & 1);
          if (r >= n) continue;
          const size_t iv = (((size_t)b * T + t0 + r) * H + h) * dv + cc;
          const float x = accv[i][e];
          if (gated) {
            p.gv[iv] = x * pw[i][e];
            p.ge2[iv] = x * pv[i][e];
          } else {
            p.gv[iv] = x;
          }
        }
    }
    // 0 dM_k = tril(dO V^T), 1 dM_z = -tril(dO E^T), 2 dA = -stril(dR E^T), 3 dB = stril(dR V^T)
    {
      const int pr = warp >> 1, r0 = 16 * (warp & 1);
      const float *X = pr < 2 ? dO : dR;
      const float *Y = (pr == 0 || pr == 3) ? V : E;
      float *out = pr == 0 ? dMk : pr == 1 ? dMz : pr == 2 ? dA : dBm;
      const float sign = (pr == 1 || pr == 2) ? -1.f : 1.f;
      const bool strict = pr >= 2;
      zero_acc(acc);
      mma_seg<kSplit>(acc, r0, 0, 0, dv, [&](int m, int kk) { return X[m * LDV + kk]; },
                      [&](int kk, int nn) { return Y[nn * LDV + kk]; }, lane);
      for_acc(acc, r0, 0, lane, [&](int r, int cc, float x) {
        out[r * kLDC + cc] = (cc < r || (!strict && cc == r)) ? sign * x : 0.f;
      });
    }
  }
  __syncthreads();
  // Token gradients dq, du, dk, dz; decay-gradient terms D into Tmp.  S^T and dS_end^T
  // are staged kSlab value columns at a time into the dead A .. M_k block.
  {
    const Tin *e1 = static_cast<const Tin *>(p.e1), *e2 = static_cast<const Tin *>(p.e2);
    float *slS = sm + L.A, *slG = slS + (size_t)dk * kLDS;
    const bool own = warp < 2 * nkt;
    const int r0 = 16 * (warp / nkt), c0 = 32 * (warp % nkt);
    float aq[4][4], au[4][4], ak[4][4], az[4][4];
    zero_acc(aq);
    zero_acc(au);
    zero_acc(ak);
    zero_acc(az);
    constexpr int kUnroll = kDepth > 1 ? kDV / kSlab : 1;   // two buffers alternate statically
#pragma unroll kUnroll
    for (int it = 0; it < dv / kSlab; ++it) {
      const int cs = it * kSlab, q = it % kDepth;
      pS[q].store(slS, kLDS, dk, kSlab, nullptr);
      pG[q].store(slG, kLDS, dk, kSlab, gscale);
      __syncthreads();
      if (cs + kDepth * kSlab < dv) {
        pS[q].load(S + cs + kDepth * kSlab, dv, dk, kSlab);
        pG[q].load(G + cs + kDepth * kSlab, dv, dk, kSlab);
      }
      if (own) {
        auto St = [&](int kk, int nn) { return slS[nn * kLDS + kk]; };
        auto Gt = [&](int kk, int nn) { return slG[nn * kLDS + kk]; };
        mma_seg<kSplit>(aq, r0, c0, 0, kSlab, [&](int m, int kk) { return dO[m * LDV + cs + kk]; }, St, lane);
        mma_seg<kSplit>(au, r0, c0, 0, kSlab, [&](int m, int kk) { return dR[m * LDV + cs + kk]; }, St, lane);
        mma_seg<kSplit>(ak, r0, c0, 0, kSlab, [&](int m, int kk) { return V[m * LDV + cs + kk]; }, Gt, lane);
        mma_seg<kSplit>(az, r0, c0, 0, kSlab, [&](int m, int kk) { return -E[m * LDV + cs + kk]; }, Gt, lane);
      }
      __syncthreads();
    }
    if (own) {
      if (!exact) {
        auto tile = [&](const float *X) { return [=](int kk, int nn) { return X[kk * LDK + nn]; }; };
        mma_seg<kSplit>(aq, r0, c0, 0, kC, [&](int m, int kk) { return dMk[m * kLDC + kk]; }, tile(K), lane);
        mma_seg<kSplit>(aq, r0, c0, 0, kC, [&](int m, int kk) { return dMz[m * kLDC + kk]; }, tile(Z), lane);
        mma_seg<kSplit>(au, r0, c0, 0, kC, [&](int m, int kk) { return dA[m * kLDC + kk]; }, tile(Z), lane);
        mma_seg<kSplit>(au, r0, c0, 0, kC, [&](int m, int kk) { return dBm[m * kLDC + kk]; }, tile(K), lane);
        mma_seg<kSplit>(ak, r0, c0, 0, kC, [&](int m, int kk) { return dBm[kk * kLDC + m]; }, tile(U), lane);
        mma_seg<kSplit>(ak, r0, c0, 0, kC, [&](int m, int kk) { return dMk[kk * kLDC + m]; }, tile(Q), lane);
        mma_seg<kSplit>(az, r0, c0, 0, kC, [&](int m, int kk) { return dA[kk * kLDC + m]; }, tile(U), lane);
        mma_seg<kSplit>(az, r0, c0, 0, kC, [&](int m, int kk) { return dMz[kk * kLDC + m]; }, tile(Q), lane);
      }
      const int g = lane >> 2, tq = lane & 3;
      // the form's inputs of this thread's 16 outputs (GDN-2's erase gate b, RWKV-7's c),
      // loaded together ahead of the loop
      float pre[4][4];
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int t = r0 + g + 8 * (e >> 1), j = c0 + 8 * i + 2 * tq + (e & 1);
          const size_t tok = ((size_t)b * T + t0 + t) * H + h;
          pre[i][e] = t >= n ? 0.f
                      : p.form == GDR_FORM_GDN2  ? ld_in(e1, tok * dk + j)
                      : p.form == GDR_FORM_RWKV7 ? ld_in(e2, tok)
                                                 : 0.f;
        }
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int t = r0 + g + 8 * (e >> 1), j = c0 + 8 * i + 2 * tq + (e & 1);
          const float l0 = lam[t * LDK + j], l1 = lam[(t + 1) * LDK + j];
          float dq, du, dkk, dz;
          if (!exact) {
            const float f = __expf(-l1);
            dq = aq[i][e] * __expf(l1);
            du = au[i][e] * __expf(l0);
            dkk = ak[i][e] * f;
            dz = az[i][e] * f;
          } else {
            const float f = __expf(lam[kC * LDK + j] - l1);
            dq = aq[i][e] * __expf(l1);
            du = au[i][e] * __expf(l0);
            dkk = ak[i][e] * f;
            dz = az[i][e] * f;
            for (int s = 0; s <= t; ++s) {
              const float x = __expf(l1 - lam[(s + 1) * LDK + j]);
              dq += (dMk[t * kLDC + s] * K[s * LDK + j] + dMz[t * kLDC + s] * Z[s * LDK + j]) * x;
              if (s < t) {
                const float y = __expf(l0 - lam[(s + 1) * LDK + j]);
                du += (dA[t * kLDC + s] * Z[s * LDK + j] + dBm[t * kLDC + s] * K[s * LDK + j]) * y;
              }
            }
            for (int r = t; r < kC; ++r) {
              const float x = __expf(lam[(r + 1) * LDK + j] - l1);
              dkk += dMk[r * kLDC + t] * Q[r * LDK + j] * x;
              dz += dMz[r * kLDC + t] * Q[r * LDK + j] * x;
              if (r > t) {
                const float y = __expf(lam[r * LDK + j] - l1);
                dkk += dBm[r * kLDC + t] * U[r * LDK + j] * y;
                dz += dA[r * kLDC + t] * U[r * LDK + j] * y;
              }
            }
          }
          if (t >= n) {
            Tmp[t * LDK + j] = 0.f;
            Lloc[t * LDK + j] = 0.f;
            continue;
          }
          const size_t tok = ((size_t)b * T + t0 + t) * H + h;
          const size_t ik = tok * dk + j;
          // the form's effective q, k, u, z from the tiles (pivot path: undo the scaling)
          const float fq = exact ? 1.f : __expf(-l1), fk = exact ? 1.f : __expf(l1);
          const float fu = exact ? 1.f : __expf(-l0);
          const float qr = Q[t * LDK + j] * fq, kr = K[t * LDK + j] * fk;
          const float z = Z[t * LDK + j] * fk, u = U[t * LDK + j] * fu;
          const float w = __expf(l1 - l0);
          Tmp[t * LDK + j] = qr * dq - kr * dkk - z * dz + u * du;
          float lw_local = -u * du;
          p.gq[ik] = dq;
          switch (p.form) {
            case GDR_FORM_GENERAL:
              p.gk[ik] = dkk;
              p.ge1[ik] = du;
              p.ge2[ik] = dz;
              break;
            case GDR_FORM_GDN2: {
              const float bb = pre[i][e];
              p.gk[ik] = dkk + dz + du * w * bb;
              p.ge1[ik] = du * w * kr;
              lw_local = 0.f;
              break;
            }
            case GDR_FORM_RWKV7: {
              p.gk[ik] = dkk;
              p.ge1[ik] = pre[i][e] * du + dz;
              atomicAdd(sm + L.dc + t, du * z);   // z = a
              break;
            }
            default:
              p.gk[ik] = dkk;
              break;
          }
          Lloc[t * LDK + j] = lw_local;
        }
    }
  }
  // diag(S_end^T dS_end): kThreads / dk threads per key channel
  {
    const int per = kThreads / dk, j = tid / per, part = tid % per, span = dv / per;
    const float *se = Send + (size_t)j * dv + part * span, *ge = G + (size_t)j * dv + part * span;
    float acc = 0.f;
    for (int cc = 0; cc < span; cc += 16) {   // span is a multiple of 16
      float4 a[4], g4[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        a[u] = __ldg(reinterpret_cast<const float4 *>(se + cc + 4 * u));
        g4[u] = __ldg(reinterpret_cast<const float4 *>(ge + cc + 4 * u));
      }
#pragma unroll
      for (int u = 0; u < 4; ++u)
        acc += a[u].x * g4[u].x + a[u].y * g4[u].y + a[u].z * g4[u].z + a[u].w * g4[u].w;
    }
    for (int o = per / 2; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
    if (part == 0) xcv[j] = acc;
  }
  __syncthreads();
  // dlog_w_t = sum_{r >= t in the chunk} D_r + (local term written above) + diag(S_end^T dS_end)
  for (int j = tid; j < dk; j += kThreads) {
    float run = xcv[j];
    for (int t = kC - 1; t >= 0; --t) {
      run += Tmp[t * LDK + j];
      if (t < n) p.glw[(((size_t)b * T + t0 + t) * H + h) * dk + j] = run + Lloc[t * LDK + j];
    }
  }
  if (p.form == GDR_FORM_RWKV7 && tid < n) p.ge2[((size_t)b * T + t0 + tid) * H + h] = sm[L.dc + tid];
}

size_t align256(size_t x) { return (x + 255) & ~(size_t)255; }

struct WsLayout {
  size_t rec, states, adj, total;
  WsLayout(int B, int H, int T, int dk, int dv) {
    const size_t nc = (size_t)(T + kC - 1) / kC, bh = (size_t)B * H;
    size_t off = kStatusBytes;
    rec = off; off = align256(off + bh * nc * (4 * (size_t)kC * dk + dk) * 4);
    states = off; off = align256(off + bh * (nc + 1) * (size_t)dk * dv * 4);
    adj = off; off = align256(off + bh * nc * (size_t)dk * dv * 4);
    total = off;
  }
};

template <typename Tin, bool kSplit, int kDK>
cudaError_t launch_chain(const BwdParams &p, cudaStream_t stream) {
  const ChainSmem Lc(kDK);
  const size_t sc = Lc.total * 4;
  cudaError_t e = cudaFuncSetAttribute(bwd_chain_kernel<Tin, kSplit, kDK>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sc);
  if (e != cudaSuccess) return e;
  bwd_chain_kernel<Tin, kSplit, kDK><<<dim3(p.dv / kNC, p.H, p.B), kChainThreads, sc, stream>>>(p);
  return cudaSuccess;
}

template <typename Tin, bool kSplit, int kDK, int kDV>
cudaError_t launch_sized(const BwdParams &p, cudaStream_t stream) {
  const ChunkSmem Lp(kDK, kDV, false), Lg(kDK, kDV, true);
  const size_t sp = Lp.total * 4, sg = Lg.total * 4;
  cudaError_t e;
  if ((e = cudaFuncSetAttribute(bwd_prep_kernel<Tin, kSplit, kDK, kDV>,
                                cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sp)) != cudaSuccess)
    return e;
  if ((e = cudaFuncSetAttribute(bwd_grads_kernel<Tin, kSplit, kDK, kDV>,
                                cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sg)) != cudaSuccess)
    return e;
  const dim3 chunks(p.nc, p.H, p.B);
  bwd_prep_kernel<Tin, kSplit, kDK, kDV><<<chunks, kThreads, sp, stream>>>(p);
  if ((e = launch_chain<Tin, kSplit, kDK>(p, stream)) != cudaSuccess) return e;
  bwd_grads_kernel<Tin, kSplit, kDK, kDV><<<chunks, kThreads, sg, stream>>>(p);
  return cudaGetLastError();
}

template <typename Tin, bool kSplit>
cudaError_t launch_typed(const BwdParams &p, cudaStream_t stream) {
  if (p.dk == 64)
    return p.dv == 64 ? launch_sized<Tin, kSplit, 64, 64>(p, stream)
                      : launch_sized<Tin, kSplit, 64, 128>(p, stream);
  return p.dv == 64 ? launch_sized<Tin, kSplit, 128, 64>(p, stream)
                    : launch_sized<Tin, kSplit, 128, 128>(p, stream);
}

}  // namespace

bool backward_supported(int dk, int dv) {
  return (dk == 64 || dk == 128) && (dv == 64 || dv == 128);
}

size_t backward_workspace_bytes(int form, int B, int H, int T, int dk, int dv) {
  (void)form;
  return WsLayout(B, H, T, dk, dv).total;
}

cudaError_t launch_backward(const BwdParams &p_in, gdr_dtype dtype, void *workspace,
                            cudaStream_t stream) {
  BwdParams p = p_in;
  const WsLayout W(p.B, p.H, p.T, p.dk, p.dv);
  uint8_t *ws = static_cast<uint8_t *>(workspace);
  p.rec = reinterpret_cast<float *>(ws + W.rec);
  p.states = reinterpret_cast<float *>(ws + W.states);
  p.adj = reinterpret_cast<float *>(ws + W.adj);
  p.nc = (p.T + kC - 1) / kC;
  return dtype == GDR_BF16 ? launch_typed<__nv_bfloat16, false>(p, stream)
                           : launch_typed<float, true>(p, stream);
}

}  // namespace gdr
