// gdr_fwd_recur.cu -- the forward as the token recurrence itself, for problems whose
// chunkwise kernels would leave most of the GPU idle.
//
// "Muir: Linear Attention with Sensitivity-Allocated Gating and Matched-Filter
// Readout", section 2.1 eq. (1) and section 4.2 eq. (8); "Exponential gates and
// matrix memory: xLSTM and RWKV-7", section 13.3.  In the storage orientation (state
// S[j][c], key channel j, value channel c), token by token:
//
//   e[c] = sum_j S[j][c] u[j],   p[c] = sum_j S[j][c] w[j] q[j]     (old state)
//   o[c] = p[c] - e[c] <z, q> + v[c] <k, q>                          (the updated state's readout)
//   S[j][c] <- S[j][c] w[j] - z[j] e[c] + k[j] v[c]
//
// Each value column of S evolves on its own, so one warp carries one column (lane
// holds R = d_k / 32 key rows, in fp32 registers) and a token costs it one two-value
// warp reduction and a few fused multiply-adds.  A CTA holds kCols columns of one
// head; its warps stage the head's token vectors (u, z, w, w q, k and the two dots
// <z, q>, <k, q>, formed once per token for the CTA) in shared memory, a block of eight
// tokens at a time, loading the next block's inputs into registers before the current
// block's recurrence so that their latency overlaps it.  (Blocks of 32 tokens measured
// 5 % faster on the smallest problems and 15-20 % slower on large ones: the extra
// registers halve the CTAs an SM holds.)  The chunkwise kernels parallelise a
// sequence over its chunks; with only a few heads and short sequences that parallelism
// is not there, and this kernel's latency per token (one reduction) is far below
// theirs per chunk divided by the chunk length.
#include "gdr_internal.cuh"

namespace gdr {
namespace {

constexpr int kCols = 8;                  // value columns (= warps) per CTA
constexpr int kRThreads = 32 * kCols;

template <int DK>
struct RecurShape {
  static constexpr int R = DK >= 32 ? DK / 32 : 1;   // key rows per lane
  static constexpr int LANES = DK / R;               // lanes holding rows (16 at d_k = 16)
  static constexpr int TB = kCols;                   // tokens per staged block (one per warp)
  static constexpr int TPW = TB / kCols;             // of which each warp stages
  // shared memory (floats): [2][TB][u, z, w, w q, k][DK], [2][TB][2] dots, [2][TB][kCols] v
  static constexpr int SV = 0, SDOT = SV + 2 * TB * 5 * DK, SVV = SDOT + 2 * TB * 2;
  static constexpr size_t BYTES = (size_t)(SVV + 2 * TB * kCols) * 4;
};

// The inputs of one token for this lane's key rows, as loaded.
template <int R>
struct TokRegs {
  float lw[R], q[R], k[R], e1[R], e2[R];
  float v = 0.f, e2s = 0.f;   // lanes < kCols: v of column c0 + lane (times GDN-2's write gate);
                              // e2s: RWKV-7's c
};

// R consecutive floats of shared memory (R = 1, 2 or 4; 4 R-byte aligned)
template <int R>
__device__ __forceinline__ void lds_r(const float *src, float (&d)[R]) {
  if constexpr (R == 4) {
    const float4 x = *reinterpret_cast<const float4 *>(src);
    d[0] = x.x; d[1] = x.y; d[2] = x.z; d[3] = x.w;
  } else if constexpr (R == 2) {
    const float2 x = *reinterpret_cast<const float2 *>(src);
    d[0] = x.x; d[1] = x.y;
  } else {
    d[0] = src[0];
  }
}

template <int DK, typename Tin>
__global__ void __launch_bounds__(kRThreads) fwd_recur_kernel(FwdParams p) {
  using Sh = RecurShape<DK>;
  constexpr int R = Sh::R, kTB = Sh::TB, TPW = Sh::TPW;
  extern __shared__ __align__(16) float rsm[];
  auto sv = reinterpret_cast<float (*)[kTB][5][DK]>(rsm + Sh::SV);      // [buffer][token][vec][j]
  auto sdot = reinterpret_cast<float (*)[kTB][2]>(rsm + Sh::SDOT);      // <z, q>, <k, q>
  auto svv = reinterpret_cast<float (*)[kTB][kCols]>(rsm + Sh::SVV);    // v (x write gate)

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int c0 = blockIdx.x * kCols, c = c0 + warp;
  const int h = blockIdx.y, b = blockIdx.z;
  const int T = p.T, H = p.H, dv = p.dv;
  const gdr_form form = p.form;
  const bool lact = lane < Sh::LANES;            // lane holds key rows j0 .. j0 + R - 1
  const int j0 = lane * R;
  const Tin *q = static_cast<const Tin *>(p.q), *k = static_cast<const Tin *>(p.k);
  const Tin *v = static_cast<const Tin *>(p.v);
  const Tin *e1 = static_cast<const Tin *>(p.e1), *e2 = static_cast<const Tin *>(p.e2);
  const size_t bh = (size_t)b * H + h;

  // this warp's token of a block: inputs into registers (tokens past T are skipped)
  auto fetch = [&](int t, TokRegs<R> &x) {
    if (t >= T) return;
    const size_t tok = ((size_t)b * T + t) * H + h;
    if (lact) {
#pragma unroll
      for (int r = 0; r < R; ++r) {
        const size_t ik = tok * DK + j0 + r;
        x.lw[r] = __ldg(p.log_w + ik);
        x.q[r] = ld_in(q, ik);
        x.k[r] = ld_in(k, ik);
        x.e1[r] = (form == GDR_FORM_GLA) ? 0.f : ld_in(e1, ik);
        x.e2[r] = (form == GDR_FORM_GENERAL) ? ld_in(e2, ik) : 0.f;
      }
    }
    x.e2s = (form == GDR_FORM_RWKV7) ? ld_in(e2, tok) : 0.f;
    if (lane < kCols && c0 + lane < dv) {
      const size_t iv = tok * dv + c0 + lane;
      x.v = ld_in(v, iv);
      if (form == GDR_FORM_GDN2 && e2 != nullptr) x.v *= ld_in(e2, iv);
    }
  };
  // the staged vectors of that token, row `slot` of the block (the decay exponentiated
  // once per token for the CTA)
  auto stage = [&](int t, int slot, const TokRegs<R> &x, int buf) {
    if (t >= T) return;
    float zq = 0.f, kq = 0.f;
    if (lact) {
#pragma unroll
      for (int r = 0; r < R; ++r) {
        const float wj = __expf(x.lw[r]);
        float u, z;
        switch (form) {
          case GDR_FORM_GENERAL: u = x.e1[r]; z = x.e2[r]; break;
          case GDR_FORM_GDN2: u = wj * x.e1[r] * x.k[r]; z = x.k[r]; break;
          case GDR_FORM_RWKV7: u = x.e2s * x.e1[r]; z = x.e1[r]; break;
          default: u = 0.f; z = 0.f; break;
        }
        float *dst = &sv[buf][slot][0][j0 + r];
        dst[0 * DK] = u;
        dst[1 * DK] = z;
        dst[2 * DK] = wj;
        dst[3 * DK] = wj * x.q[r];
        dst[4 * DK] = x.k[r];
        zq = fmaf(z, x.q[r], zq);
        kq = fmaf(x.k[r], x.q[r], kq);
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      zq += __shfl_xor_sync(0xffffffffu, zq, o);
      kq += __shfl_xor_sync(0xffffffffu, kq, o);
    }
    if (lane == 0) {
      sdot[buf][slot][0] = zq;
      sdot[buf][slot][1] = kq;
    }
    if (lane < kCols) svv[buf][slot][lane] = x.v;
  };

  // this warp's column of the state: rows j0 .. j0 + R - 1
  float s[R];
  const size_t sbase = bh * DK * dv + c;
  const bool col = c < dv;
#pragma unroll
  for (int r = 0; r < R; ++r) s[r] = (p.S0 && col && lact) ? __ldg(p.S0 + sbase + (size_t)(j0 + r) * dv) : 0.f;

  const int nblk = (T + kTB - 1) / kTB;
  {
    TokRegs<R> x[TPW];
#pragma unroll
    for (int m = 0; m < TPW; ++m) fetch(kCols * m + warp, x[m]);
#pragma unroll
    for (int m = 0; m < TPW; ++m) stage(kCols * m + warp, kCols * m + warp, x[m], 0);
  }
  __syncthreads();
  // one token of the recurrence from block buffer `buf`, row i
  auto step = [&](int buf, int i, int t) {
    const float *vec = &sv[buf][i][0][0];
    float pe = 0.f, pp = 0.f;
    float u[R], z[R], w[R], wq[R], kk[R];
    if (lact) {
      lds_r<R>(vec + 0 * DK + j0, u);
      lds_r<R>(vec + 1 * DK + j0, z);
      lds_r<R>(vec + 2 * DK + j0, w);
      lds_r<R>(vec + 3 * DK + j0, wq);
      lds_r<R>(vec + 4 * DK + j0, kk);
#pragma unroll
      for (int r = 0; r < R; ++r) {
        pe = fmaf(s[r], u[r], pe);
        pp = fmaf(s[r], wq[r], pp);
      }
    } else {
#pragma unroll
      for (int r = 0; r < R; ++r) u[r] = z[r] = w[r] = wq[r] = kk[r] = 0.f;
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      pe += __shfl_xor_sync(0xffffffffu, pe, o);
      pp += __shfl_xor_sync(0xffffffffu, pp, o);
    }
    const float vc = svv[buf][i][warp];
    if (lane == 0 && col) {
      const size_t tok = ((size_t)b * T + t) * H + h;
      p.o[tok * dv + c] = pp - pe * sdot[buf][i][0] + vc * sdot[buf][i][1];
    }
#pragma unroll
    for (int r = 0; r < R; ++r) s[r] = fmaf(kk[r], vc, fmaf(s[r], w[r], -z[r] * pe));
  };
  for (int blk = 0; blk < nblk; ++blk) {
    const int buf = blk & 1, tb0 = blk * kTB;
    TokRegs<R> x[TPW];
    const bool more = blk + 1 < nblk;
    if (more) {   // lands while this block's recurrence runs
#pragma unroll
      for (int m = 0; m < TPW; ++m) fetch(tb0 + kTB + kCols * m + warp, x[m]);
    }
    const int n = min(kTB, T - tb0);
    for (int i = 0; i < n; ++i) step(buf, i, tb0 + i);
    if (more) {
#pragma unroll
      for (int m = 0; m < TPW; ++m) stage(tb0 + kTB + kCols * m + warp, kCols * m + warp, x[m], buf ^ 1);
    }
    __syncthreads();
  }
  if (p.S_T && col && lact) {
#pragma unroll
    for (int r = 0; r < R; ++r) p.S_T[sbase + (size_t)(j0 + r) * dv] = s[r];
  }
}

template <int DK, typename Tin>
cudaError_t launch_typed(const FwdParams &p, cudaStream_t stream) {
  using Sh = RecurShape<DK>;
  const dim3 grid((p.dv + kCols - 1) / kCols, p.H, p.B);
  cudaError_t e = cudaFuncSetAttribute(fwd_recur_kernel<DK, Tin>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)Sh::BYTES);
  if (e != cudaSuccess) return e;
  fwd_recur_kernel<DK, Tin><<<grid, kRThreads, Sh::BYTES, stream>>>(p);
  return cudaGetLastError();
}

template <int DK>
cudaError_t launch_dk(const FwdParams &p, gdr_dtype dtype, cudaStream_t stream) {
  return dtype == GDR_BF16 ? launch_typed<DK, __nv_bfloat16>(p, stream) : launch_typed<DK, float>(p, stream);
}

}  // namespace

bool forward_recur_supported(int dk, int dv) {
  return (dk == 16 || dk == 32 || dk == 64 || dk == 128) && dv >= 1;
}

cudaError_t launch_forward_recur(const FwdParams &p, gdr_dtype dtype, cudaStream_t stream) {
  switch (p.dk) {
    case 16: return launch_dk<16>(p, dtype, stream);
    case 32: return launch_dk<32>(p, dtype, stream);
    case 64: return launch_dk<64>(p, dtype, stream);
    case 128: return launch_dk<128>(p, dtype, stream);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace gdr
