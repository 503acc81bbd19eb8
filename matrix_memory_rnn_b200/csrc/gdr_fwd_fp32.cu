// gdr_fwd_fp32.cu -- chunkwise forward, fp32 CUDA-core kernel (all forms).
//
// Chunkwise form: "Muir: Linear Attention with Sensitivity-Allocated Gating and
// Matched-Filter Readout", section 2.2 (effective write, unit lower-triangular
// system, S_C and O as matrix products) and section 4.2 eq. (10), generalized to a
// separate erase key z.  In the storage orientation (S[j][c]: key j, value c), for
// one chunk of n tokens (t, s = 0..n-1) starting from state S:
//
//   Lam[m]      = sum_{r < m} log w_r                 (m = 0..n, <= 0, fp32)
//   A[t][s]     = sum_j u_tj z_sj exp(Lam[t]_j - Lam[s+1]_j)      (s < t)
//   Bm[t][s]    = sum_j u_tj k_sj exp(Lam[t]_j - Lam[s+1]_j)      (s < t)
//   Mk[t][s]    = sum_j q_tj k_sj exp(Lam[t+1]_j - Lam[s+1]_j)    (s <= t)
//   Mz[t][s]    = sum_j q_tj z_sj exp(Lam[t+1]_j - Lam[s+1]_j)    (s <= t)
//   (I + A) E   = P + Bm V,   P[t][c] = sum_j u_tj exp(Lam[t]_j) S[j][c]
//   O[t][c]     = sum_j q_tj exp(Lam[t+1]_j) S[j][c] + sum_{s<=t} (Mk[t][s] V[s][c] - Mz[t][s] E[s][c])
//   S'[j][c]    = exp(Lam[n]_j) S[j][c] + sum_s exp(Lam[n]_j - Lam[s+1]_j)(k_sj V[s][c] - z_sj E[s][c])
//
// E holds the erase reads e_t = S_{t-1} u_t.  Every exponent is a difference
// Lam[later] - Lam[earlier] <= 0, so no factor exceeds 1 and nothing overflows
// (section 4.2, the log-space decays behind boundary-pivoted splitting).
// For GDN-2 (z = k, u = alpha b k) this reduces exactly to section 2.2 with
// A = Bm = L_strict and V~ = V - E.
//
// This kernel evaluates every product in fp32 on the CUDA cores.  When no channel
// decays by more than 80 nats over the chunk, each pair's decay e^{Lam[a] - Lam[b]} (a
// the later index) splits as e^{Lam[a] - P} e^{P - Lam[b]} with P the channel's Lam at
// the chunk's middle, every factor in [e^-80, e^80]: q and u take the first factor, k
// and z the second, in place, and the pairwise products become plain dot products (one
// exponential per element instead of up to three per pair and channel).  A chunk that
// decays more takes the exact pairwise decay (one exp per pair and channel).  It is the
// accurate path (fp32 inputs) and the reference kernel for the tensor-core path.  One CTA per
// (b, h, slice of NV value columns), looping over the chunks; the chunk is held
// in shared memory, so the kernel caps its chunk at 64 tokens and at
// 4096 / dk tokens (32 at dk = 128); the result does not depend on the chunk
// length beyond rounding.
#include "gdr_internal.cuh"

namespace gdr {
namespace {

constexpr int kThreads = 512;
constexpr float kMaxSpan = 80.f;   // nats of decay over a chunk for the pivot path

__host__ __device__ inline int fp32_chunk(int dk, int chunk) {
  int c = chunk < 64 ? chunk : 64;
  const int cap = 4096 / dk;
  return c < cap ? c : cap;
}
__host__ __device__ inline int fp32_nv(int dv) { return dv < 32 ? dv : 32; }

struct Smem {
  int LD;  // padded row stride of the d_k-wide arrays (dk + 1: conflict-free columns)
  int C, NV, dk;
  size_t lam, q, k, u, z, v, e, r, A, Bm, Mk, Mz, S, fac, flag, total;  // float offsets
  __host__ __device__ Smem(int dk_, int dv, int chunk) {
    dk = dk_;
    LD = dk + 1;
    C = fp32_chunk(dk, chunk);
    NV = fp32_nv(dv);
    size_t off = 0;
    lam = off; off += (size_t)(C + 1) * LD;
    q = off; off += (size_t)C * LD;
    k = off; off += (size_t)C * LD;
    u = off; off += (size_t)C * LD;
    z = off; off += (size_t)C * LD;
    v = off; off += (size_t)C * NV;
    e = off; off += (size_t)C * NV;
    r = off; off += (size_t)C * NV;
    A = off; off += (size_t)C * C;
    Bm = off; off += (size_t)C * C;
    Mk = off; off += (size_t)C * C;
    Mz = off; off += (size_t)C * C;
    S = off; off += (size_t)dk * NV;
    fac = off; off += (size_t)3 * dk;   // pivot path: e^P, e^(Lam[n] - P), e^Lam[n] per channel
    flag = off; off += 4;               // int: this chunk takes the exact pairwise path
    total = off;
  }
};

template <typename Tin>
__global__ void __launch_bounds__(kThreads) fwd_fp32_kernel(FwdParams p) {
  extern __shared__ float sm[];
  const Smem L(p.dk, p.dv, p.chunk);
  const int dk = p.dk, dv = p.dv, T = p.T, H = p.H, LD = L.LD, NV = L.NV, C = L.C;
  const int c0 = blockIdx.x * NV, h = blockIdx.y, b = blockIdx.z;
  const int tid = threadIdx.x;
  const bool has_erase = p.form != GDR_FORM_GLA;
  float *lam = sm + L.lam, *Q = sm + L.q, *K = sm + L.k, *U = sm + L.u, *Z = sm + L.z;
  float *V = sm + L.v, *E = sm + L.e, *R = sm + L.r;
  float *A = sm + L.A, *Bm = sm + L.Bm, *Mk = sm + L.Mk, *Mz = sm + L.Mz, *S = sm + L.S;
  float *fac = sm + L.fac;
  volatile int *sflag = reinterpret_cast<volatile int *>(sm + L.flag);
  const Tin *q = static_cast<const Tin *>(p.q), *k = static_cast<const Tin *>(p.k);
  const Tin *v = static_cast<const Tin *>(p.v), *e1 = static_cast<const Tin *>(p.e1);
  const Tin *e2 = static_cast<const Tin *>(p.e2);

  // Initial state slice S[j][c], c in [c0, c0 + NV).
  const size_t sbase = ((size_t)b * H + h) * dk * dv;
  for (int i = tid; i < dk * NV; i += kThreads) {
    const int j = i / NV, c = i % NV;
    S[i] = p.S0 ? p.S0[sbase + (size_t)j * dv + c0 + c] : 0.f;
  }

  for (int t0 = 0; t0 < T; t0 += C) {
    const int n = min(C, T - t0);
    __syncthreads();  // previous chunk done with every buffer

    // 1. chunk inputs; log w goes to lam[t + 1] and is prefix-summed below.
    for (int i = tid; i < n * dk; i += kThreads) {
      const int t = i / dk, j = i % dk;
      const size_t tok = ((size_t)b * T + t0 + t) * H + h;
      const size_t ik = tok * dk + j;
      const float lw = __ldg(p.log_w + ik);
      float u, z;
      erase_pair(p.form, k, e1, e2, ik, tok, __expf(lw), u, z);
      lam[(t + 1) * LD + j] = lw;
      Q[t * LD + j] = ld_in(q, ik);
      K[t * LD + j] = ld_in(k, ik);
      U[t * LD + j] = u;
      Z[t * LD + j] = z;
    }
    for (int i = tid; i < n * NV; i += kThreads) {
      const int t = i / NV, c = i % NV;
      const size_t iv = (((size_t)b * T + t0 + t) * H + h) * dv + c0 + c;
      float x = ld_in(v, iv);
      if (p.form == GDR_FORM_GDN2 && e2 != nullptr) x *= ld_in(e2, iv);
      V[t * NV + c] = x;
    }
    __syncthreads();

    // 2. cumulative log-decay (one thread per channel); a channel that decays by more
    //    than 80 nats over the chunk sends the chunk to the exact pairwise path
    if (tid == 0) *sflag = 0;
    __syncthreads();
    for (int j = tid; j < dk; j += kThreads) {
      float acc = 0.f;
      lam[j] = 0.f;
      for (int t = 1; t <= n; ++t) {
        acc += lam[t * LD + j];
        lam[t * LD + j] = acc;
      }
      if (!(acc >= -kMaxSpan)) *sflag = 1;   // (NaN too)
    }
    __syncthreads();
    const bool exact = *sflag != 0;

    // 2b. pivot path: q_t *= e^(Lam[t+1] - P), u_t *= e^(Lam[t] - P), k_s, z_s *= e^(P - Lam[s+1])
    //     in place, P = Lam[n/2] per channel; then the three per-channel factors the later
    //     steps use in place of their exponentials of Lam
    if (!exact) {
      const int pv = n / 2;
      for (int i = tid; i < n * dk; i += kThreads) {
        const int t = i / dk, j = i % dk;
        const float P = lam[pv * LD + j], l1 = lam[(t + 1) * LD + j];
        Q[t * LD + j] *= expf(l1 - P);
        K[t * LD + j] *= expf(P - l1);
        if (has_erase) {
          U[t * LD + j] *= expf(lam[t * LD + j] - P);
          Z[t * LD + j] *= expf(P - l1);
        }
      }
      for (int j = tid; j < dk; j += kThreads) {
        const float P = lam[pv * LD + j], ln = lam[n * LD + j];
        fac[j] = expf(P);
        fac[dk + j] = expf(ln - P);
        fac[2 * dk + j] = expf(ln);
      }
      __syncthreads();
    }

    // 3. pairwise decay-weighted products
    for (int i = tid; i < n * n; i += kThreads) {
      const int t = i / n, s = i % n;
      float a = 0.f, bm = 0.f, mk = 0.f, mz = 0.f;
      if (s <= t && !exact) {   // the decays are in the scaled rows
        const float *qt = Q + t * LD, *ut = U + t * LD, *ks = K + s * LD, *zs = Z + s * LD;
        for (int j = 0; j < dk; ++j) {
          mk += qt[j] * ks[j];
          if (has_erase) {
            mz += qt[j] * zs[j];
            if (s < t) {
              a += ut[j] * zs[j];
              bm += ut[j] * ks[j];
            }
          }
        }
      } else if (s <= t) {
        const float *lt = lam + t * LD, *lt1 = lam + (t + 1) * LD, *ls1 = lam + (s + 1) * LD;
        const float *qt = Q + t * LD, *ut = U + t * LD, *ks = K + s * LD, *zs = Z + s * LD;
        for (int j = 0; j < dk; ++j) {
          const float dq = __expf(lt1[j] - ls1[j]);
          mk += qt[j] * dq * ks[j];
          if (has_erase) {
            mz += qt[j] * dq * zs[j];
            if (s < t) {
              const float du = __expf(lt[j] - ls1[j]);
              a += ut[j] * du * zs[j];
              bm += ut[j] * du * ks[j];
            }
          }
        }
      }
      A[i] = a;
      Bm[i] = bm;
      Mk[i] = mk;
      Mz[i] = mz;
    }
    __syncthreads();

    if (has_erase) {
      // 4. right-hand side R = P + Bm V
      for (int i = tid; i < n * NV; i += kThreads) {
        const int t = i / NV, c = i % NV;
        float acc = 0.f;
        const float *lt = lam + t * LD, *ut = U + t * LD;
        if (exact)
          for (int j = 0; j < dk; ++j) acc += ut[j] * __expf(lt[j]) * S[j * NV + c];
        else   // u_t e^(Lam[t] - P) e^P
          for (int j = 0; j < dk; ++j) acc += ut[j] * fac[j] * S[j * NV + c];
        for (int s = 0; s < t; ++s) acc += Bm[t * n + s] * V[s * NV + c];
        R[i] = acc;
      }
      __syncthreads();

      // 5. forward substitution (I + A) E = R; 8 lanes per column share the dot product
      {
        const int c = tid / 8, r = tid % 8;
        for (int cc = c; cc < NV; cc += kThreads / 8) {
          for (int t = 0; t < n; ++t) {
            float acc = 0.f;
            for (int s = r; s < t; s += 8) acc += A[t * n + s] * E[s * NV + cc];
            acc += __shfl_xor_sync(0xffffffffu, acc, 1);
            acc += __shfl_xor_sync(0xffffffffu, acc, 2);
            acc += __shfl_xor_sync(0xffffffffu, acc, 4);
            if (r == 0) E[t * NV + cc] = R[t * NV + cc] - acc;
            __syncwarp();
          }
        }
      }
      __syncthreads();
    }

    // 6. outputs
    for (int i = tid; i < n * NV; i += kThreads) {
      const int t = i / NV, c = i % NV;
      float acc = 0.f;
      const float *lt1 = lam + (t + 1) * LD, *qt = Q + t * LD;
      if (exact)
        for (int j = 0; j < dk; ++j) acc += qt[j] * __expf(lt1[j]) * S[j * NV + c];
      else   // q_t e^(Lam[t+1] - P) e^P
        for (int j = 0; j < dk; ++j) acc += qt[j] * fac[j] * S[j * NV + c];
      for (int s = 0; s <= t; ++s) {
        acc += Mk[t * n + s] * V[s * NV + c];
        if (has_erase) acc -= Mz[t * n + s] * E[s * NV + c];
      }
      p.o[(((size_t)b * T + t0 + t) * H + h) * dv + c0 + c] = acc;
    }
    // decayed keys k~_s = exp(Lam[n] - Lam[s+1]) k_s, z~_s likewise (in place)
    __syncthreads();
    for (int i = tid; i < n * dk; i += kThreads) {
      const int s = i / dk, j = i % dk;
      // (pivot path: k_s e^(P - Lam[s+1]) e^(Lam[n] - P))
      const float d = exact ? __expf(lam[n * LD + j] - lam[(s + 1) * LD + j]) : fac[dk + j];
      K[s * LD + j] *= d;
      Z[s * LD + j] *= d;
    }
    __syncthreads();

    // 7. state update
    for (int i = tid; i < dk * NV; i += kThreads) {
      const int j = i / NV, c = i % NV;
      float acc = (exact ? __expf(lam[n * LD + j]) : fac[2 * dk + j]) * S[i];
      for (int s = 0; s < n; ++s) {
        acc += K[s * LD + j] * V[s * NV + c];
        if (has_erase) acc -= Z[s * LD + j] * E[s * NV + c];
      }
      S[i] = acc;
    }
  }
  __syncthreads();
  if (p.S_T)
    for (int i = tid; i < dk * NV; i += kThreads) {
      const int j = i / NV, c = i % NV;
      p.S_T[sbase + (size_t)j * dv + c0 + c] = S[i];
    }
}

}  // namespace

bool forward_fp32_supported(int dk, int dv) {
  return (dk == 16 || dk == 32 || dk == 64 || dk == 128) &&
         (dv == 16 || dv == 32 || dv == 64 || dv == 128);
}

size_t forward_fp32_smem_bytes(int dk, int dv, int chunk) {
  return Smem(dk, dv, chunk).total * sizeof(float);
}

cudaError_t launch_forward_fp32(const FwdParams &p, gdr_dtype dtype, cudaStream_t stream) {
  const Smem L(p.dk, p.dv, p.chunk);
  const size_t smem = L.total * sizeof(float);
  dim3 grid(p.dv / L.NV, p.H, p.B);
  if (dtype == GDR_BF16) {
    cudaError_t e = cudaFuncSetAttribute(fwd_fp32_kernel<__nv_bfloat16>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    fwd_fp32_kernel<__nv_bfloat16><<<grid, kThreads, smem, stream>>>(p);
  } else {
    cudaError_t e = cudaFuncSetAttribute(fwd_fp32_kernel<float>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    fwd_fp32_kernel<float><<<grid, kThreads, smem, stream>>>(p);
  }
  return cudaGetLastError();
}

}  // namespace gdr
