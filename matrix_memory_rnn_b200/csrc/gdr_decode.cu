// gdr_decode.cu -- one recurrent step (decode) of the generalized delta rule.
//
// "Muir: Linear Attention with Sensitivity-Allocated Gating and Matched-Filter
// Readout", section 2.1 eq. (1) and section 4.2 eq. (8); "Exponential gates and
// matrix memory: xLSTM and RWKV-7", section 13.3.  In the storage orientation
// (state S[j][c], key channel j, value channel c):
//
//   e[c] = sum_j S[j][c] u[j]                 (old state)
//   p[c] = sum_j S[j][c] w[j] q[j]            (old state, same pass)
//   o[c] = p[c] - e[c] <z, q> + v[c] <k, q>   (= readout of the updated state)
//   S[j][c] <- S[j][c] w[j] - z[j] e[c] + k[j] v[c]
//
// The step is bound by HBM: it streams the fp32 state in and out once
// (2 * dk * dv * 4 bytes per head).  Two kernels: a persistent, cp.async-pipelined
// one for d_k = d_v = 128 (below), and the general one: one CTA per (b, h); each thread keeps RPT
// rows x 4 columns of the state in registers between the read and the write, so
// the state is read exactly once.  A warp reads whole rows (float4 per lane,
// 512 contiguous bytes at dv = 128); the reduction over rows runs across warps
// through shared memory.  Loads and stores use the streaming cache hints: the
// state (1 GiB at B=256, H=32, d=128) is far larger than L2 and is not reused
// within a step.
#include "gdr_internal.cuh"
#include "gdr_sm100.cuh"

namespace gdr {
namespace {

using sm100::cp_async16;
using sm100::cp_async_commit;
using sm100::cp_async_wait;

template <int DK, int DV>
struct DecodeShape {
  static constexpr int TC = DV / 4;                             // threads along columns
  static constexpr int NT = (TC * DK < 256) ? TC * DK : 256;    // threads per CTA
  static constexpr int RG = NT / TC;                            // row groups
  static constexpr int RPT = DK / RG;                           // rows per thread
  static_assert(RG * RPT == DK, "row split");
};

template <int DK, int DV, typename Tin>
__global__ void __launch_bounds__(DecodeShape<DK, DV>::NT)
decode_step_kernel(gdr_form form, const Tin *__restrict__ q, const Tin *__restrict__ k,
                   const Tin *__restrict__ v, const float *__restrict__ log_w,
                   const Tin *__restrict__ e1, const Tin *__restrict__ e2,
                   float *__restrict__ S, float *__restrict__ o) {
  using Sh = DecodeShape<DK, DV>;
  constexpr int TC = Sh::TC, RG = Sh::RG, RPT = Sh::RPT;
  __shared__ float s_u[DK], s_z[DK], s_w[DK], s_wq[DK], s_k[DK];
  __shared__ float s_v[DV];
  __shared__ __align__(16) float s_red[2][RG][DV];
  __shared__ float s_dot[2];

  const int bh = blockIdx.x;           // b * H + h
  const int tid = threadIdx.x;
  const int cg = tid % TC;             // columns 4cg .. 4cg+3
  const int rg = tid / TC;             // rows rg, rg + RG, ...

  // Issue the state loads first: they are the long-latency part.
  float *Sbh = S + (size_t)bh * DK * DV;
  float4 s[RPT];
#pragma unroll
  for (int i = 0; i < RPT; ++i)
    s[i] = __ldcs(reinterpret_cast<const float4 *>(Sbh + (size_t)(i * RG + rg) * DV) + cg);

  // Token vectors (fp32 in shared memory).
  const size_t base_k = (size_t)bh * DK, base_v = (size_t)bh * DV;
  for (int j = tid; j < DK; j += Sh::NT) {
    const float wj = __expf(__ldg(log_w + base_k + j));
    float u, z;
    erase_pair(form, k, e1, e2, base_k + j, (size_t)bh, wj, u, z);
    const float qj = ld_in(q, base_k + j);
    s_u[j] = u;
    s_z[j] = z;
    s_w[j] = wj;
    s_wq[j] = wj * qj;
    s_k[j] = ld_in(k, base_k + j);
  }
  for (int c = tid; c < DV; c += Sh::NT) {
    float vc = ld_in(v, base_v + c);
    if (form == GDR_FORM_GDN2 && e2 != nullptr) vc *= ld_in(e2, base_v + c);
    s_v[c] = vc;
  }
  __syncthreads();

  // <z, q> and <k, q> (warp 0, shuffle reduction).  q_j = wq_j / w_j is avoided:
  // read q again instead.
  if (tid < 32) {
    float zq = 0.f, kq = 0.f;
    for (int j = tid; j < DK; j += 32) {
      const float qj = ld_in(q, base_k + j);
      zq += s_z[j] * qj;
      kq += s_k[j] * qj;
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
      zq += __shfl_xor_sync(0xffffffffu, zq, off);
      kq += __shfl_xor_sync(0xffffffffu, kq, off);
    }
    if (tid == 0) {
      s_dot[0] = zq;
      s_dot[1] = kq;
    }
  }

  // Partial reductions over this thread's rows.
  float4 pe = make_float4(0.f, 0.f, 0.f, 0.f), pp = pe;
#pragma unroll
  for (int i = 0; i < RPT; ++i) {
    const int j = i * RG + rg;
    const float uj = s_u[j], wqj = s_wq[j];
    pe.x += s[i].x * uj; pe.y += s[i].y * uj; pe.z += s[i].z * uj; pe.w += s[i].w * uj;
    pp.x += s[i].x * wqj; pp.y += s[i].y * wqj; pp.z += s[i].z * wqj; pp.w += s[i].w * wqj;
  }
  reinterpret_cast<float4 *>(&s_red[0][rg][0])[cg] = pe;
  reinterpret_cast<float4 *>(&s_red[1][rg][0])[cg] = pp;
  __syncthreads();

  float4 e = make_float4(0.f, 0.f, 0.f, 0.f), p = e;
#pragma unroll 8
  for (int r = 0; r < RG; ++r) {
    const float4 a = reinterpret_cast<const float4 *>(&s_red[0][r][0])[cg];
    const float4 b = reinterpret_cast<const float4 *>(&s_red[1][r][0])[cg];
    e.x += a.x; e.y += a.y; e.z += a.z; e.w += a.w;
    p.x += b.x; p.y += b.y; p.z += b.z; p.w += b.w;
  }
  const float4 vv = reinterpret_cast<const float4 *>(s_v)[cg];

  if (rg == 0) {
    const float zq = s_dot[0], kq = s_dot[1];
    float4 oc;
    oc.x = p.x - e.x * zq + vv.x * kq;
    oc.y = p.y - e.y * zq + vv.y * kq;
    oc.z = p.z - e.z * zq + vv.z * kq;
    oc.w = p.w - e.w * zq + vv.w * kq;
    __stcs(reinterpret_cast<float4 *>(o + base_v) + cg, oc);
  }

#pragma unroll
  for (int i = 0; i < RPT; ++i) {
    const int j = i * RG + rg;
    const float wj = s_w[j], zj = s_z[j], kj = s_k[j];
    float4 n;
    n.x = s[i].x * wj - zj * e.x + kj * vv.x;
    n.y = s[i].y * wj - zj * e.y + kj * vv.y;
    n.z = s[i].z * wj - zj * e.z + kj * vv.z;
    n.w = s[i].w * wj - zj * e.w + kj * vv.w;
    __stcs(reinterpret_cast<float4 *>(Sbh + (size_t)j * DV) + cg, n);
  }
}

// ---------------------------------------------------------------------------
// Persistent, pipelined variant (d_k = d_v = 128; general, GDN-2 and GLA forms).
// One CTA per SM loops over heads.  Each thread copies, with 16-byte cp.async
// into a 3-stage shared-memory ring, exactly the state rows it will read, two
// heads ahead; the 112 threads with the lowest index also copy the head's
// token vectors.  A thread waits only for its own copies (cp.async.wait_group)
// and the CTA then meets at a barrier, so no wait depends on another CTA.
// While head i is reduced and written back from registers, heads i+1 and i+2
// are in flight: about 130 KB per SM, enough to cover HBM latency.
template <typename Tin>
struct PipeShape {
  static constexpr int DK = 128, DV = 128, NST = 3, NT = 256;
  static constexpr int TC = DV / 4, RG = NT / TC, RPT = DK / RG;   // 32, 8, 16
  static constexpr int SZ = sizeof(Tin);
  // stage layout (bytes): state | q | k | e1 | e2 | v | log_w
  static constexpr int OFF_Q = DK * DV * 4;
  static constexpr int OFF_K = OFF_Q + DK * SZ;
  static constexpr int OFF_E1 = OFF_K + DK * SZ;
  static constexpr int OFF_E2 = OFF_E1 + DK * SZ;                  // d_v (GDN-2) or d_k (general)
  static constexpr int OFF_V = OFF_E2 + DV * SZ;
  static constexpr int OFF_LW = OFF_V + DV * SZ;
  static constexpr int STAGE = OFF_LW + DK * 4;
  static constexpr int TOK_UNITS = (STAGE - OFF_Q) / 16;
  static constexpr int SMEM = NST * STAGE + 2 * RG * DV * 4 + 6 * DK * 4 + 64;
  static_assert(TOK_UNITS <= NT, "token vectors: one 16-byte copy per thread");
};

template <typename Tin>
__device__ __forceinline__ void pipe_issue(uint8_t *stage, int bh, int tid, gdr_form form,
                                           const Tin *q, const Tin *k, const Tin *v,
                                           const float *log_w, const Tin *e1, const Tin *e2,
                                           const float *S) {
  using P = PipeShape<Tin>;
  const int cg = tid % P::TC, rg = tid / P::TC;
  const float *Sbh = S + (size_t)bh * P::DK * P::DV;
#pragma unroll
  for (int i = 0; i < P::RPT; ++i) {
    const int row = i * P::RG + rg;
    cp_async16(stage + (row * P::DV + 4 * cg) * 4, Sbh + (size_t)row * P::DV + 4 * cg);
  }
  if (tid < P::TOK_UNITS) {
    const int off = P::OFF_Q + 16 * tid;
    const uint8_t *src = nullptr;
    const size_t bk = (size_t)bh * P::DK * P::SZ, bv = (size_t)bh * P::DV * P::SZ;
    if (off < P::OFF_K) src = reinterpret_cast<const uint8_t *>(q) + bk + (off - P::OFF_Q);
    else if (off < P::OFF_E1) src = reinterpret_cast<const uint8_t *>(k) + bk + (off - P::OFF_K);
    else if (off < P::OFF_E2) src = e1 ? reinterpret_cast<const uint8_t *>(e1) + bk + (off - P::OFF_E1) : nullptr;
    else if (off < P::OFF_V) src = e2 ? reinterpret_cast<const uint8_t *>(e2) +
                                            (form == GDR_FORM_GDN2 ? bv : bk) + (off - P::OFF_E2)
                                      : nullptr;
    else if (off < P::OFF_LW) src = reinterpret_cast<const uint8_t *>(v) + bv + (off - P::OFF_V);
    else src = reinterpret_cast<const uint8_t *>(log_w) + (size_t)bh * P::DK * 4 + (off - P::OFF_LW);
    if (src) cp_async16(stage + off, src);
  }
}

template <typename Tin>
__device__ __forceinline__ float tok(const uint8_t *stage, int off, int i) {
  return (sizeof(Tin) == 2) ? __bfloat162float(reinterpret_cast<const __nv_bfloat16 *>(stage + off)[i])
                            : reinterpret_cast<const float *>(stage + off)[i];
}

template <typename Tin>
__global__ void __launch_bounds__(256, 1)
decode_pipe_kernel(gdr_form form, int nbh, const Tin *__restrict__ q, const Tin *__restrict__ k,
                   const Tin *__restrict__ v, const float *__restrict__ log_w,
                   const Tin *__restrict__ e1, const Tin *__restrict__ e2, float *__restrict__ S,
                   float *__restrict__ o) {
  using P = PipeShape<Tin>;
  constexpr int DK = P::DK, DV = P::DV, RG = P::RG, RPT = P::RPT, NST = P::NST;
  extern __shared__ __align__(16) uint8_t smem[];
  float *s_red = reinterpret_cast<float *>(smem + NST * P::STAGE);      // [2][RG][DV]
  float *s_u = s_red + 2 * RG * DV, *s_z = s_u + DK, *s_w = s_z + DK, *s_wq = s_w + DK,
        *s_k = s_wq + DK, *s_v = s_k + DK;
  float *s_dot = s_v + DV;
  const int tid = threadIdx.x, cg = tid % P::TC, rg = tid / P::TC;
  const bool has_e2 = e2 != nullptr;

  // prologue: heads 0 and 1 of this CTA
  for (int s = 0; s < NST - 1; ++s) {
    const int bh = blockIdx.x + s * gridDim.x;
    if (bh < nbh) pipe_issue(smem + s * P::STAGE, bh, tid, form, q, k, v, log_w, e1, e2, S);
    cp_async_commit();
  }
  for (int i = 0;; ++i) {
    const int bh = blockIdx.x + i * gridDim.x;
    if (bh >= nbh) break;
    {  // refill the stage the previous head used, with head i + 2
      const int nb = bh + (NST - 1) * gridDim.x;
      if (nb < nbh)
        pipe_issue(smem + ((i + NST - 1) % NST) * P::STAGE, nb, tid, form, q, k, v, log_w, e1, e2, S);
      cp_async_commit();
    }
    cp_async_wait<NST - 1>();          // this thread's copies of head i have landed
    __syncthreads();
    const uint8_t *st = smem + (i % NST) * P::STAGE;

    // token vectors (fp32 in shared memory)
    if (tid < DK) {
      const int j = tid;
      const float wj = __expf(reinterpret_cast<const float *>(st + P::OFF_LW)[j]);
      const float kj = tok<Tin>(st, P::OFF_K, j);
      float u = 0.f, z = 0.f;
      if (form == GDR_FORM_GENERAL) {
        u = tok<Tin>(st, P::OFF_E1, j);
        z = tok<Tin>(st, P::OFF_E2, j);
      } else if (form == GDR_FORM_GDN2) {
        u = wj * tok<Tin>(st, P::OFF_E1, j) * kj;
        z = kj;
      }
      s_u[j] = u;
      s_z[j] = z;
      s_w[j] = wj;
      s_wq[j] = wj * tok<Tin>(st, P::OFF_Q, j);
      s_k[j] = kj;
    } else if (tid - DK < DV) {
      const int c = tid - DK;
      float vc = tok<Tin>(st, P::OFF_V, c);
      if (form == GDR_FORM_GDN2 && has_e2) vc *= tok<Tin>(st, P::OFF_E2, c);
      s_v[c] = vc;
    }
    __syncthreads();
    if (tid < 32) {
      float zq = 0.f, kq = 0.f;
      for (int j = tid; j < DK; j += 32) {
        const float qj = tok<Tin>(st, P::OFF_Q, j);
        zq += s_z[j] * qj;
        kq += s_k[j] * qj;
      }
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) {
        zq += __shfl_xor_sync(0xffffffffu, zq, off);
        kq += __shfl_xor_sync(0xffffffffu, kq, off);
      }
      if (tid == 0) {
        s_dot[0] = zq;
        s_dot[1] = kq;
      }
    }
    // this thread's rows (the rows it copied itself)
    float4 sr[RPT];
    float4 pe = make_float4(0.f, 0.f, 0.f, 0.f), pp = pe;
#pragma unroll
    for (int r = 0; r < RPT; ++r) {
      const int j = r * RG + rg;
      sr[r] = reinterpret_cast<const float4 *>(st)[(j * DV) / 4 + cg];
      const float uj = s_u[j], wqj = s_wq[j];
      pe.x += sr[r].x * uj; pe.y += sr[r].y * uj; pe.z += sr[r].z * uj; pe.w += sr[r].w * uj;
      pp.x += sr[r].x * wqj; pp.y += sr[r].y * wqj; pp.z += sr[r].z * wqj; pp.w += sr[r].w * wqj;
    }
    reinterpret_cast<float4 *>(s_red + rg * DV)[cg] = pe;
    reinterpret_cast<float4 *>(s_red + (RG + rg) * DV)[cg] = pp;
    __syncthreads();
    float4 e = make_float4(0.f, 0.f, 0.f, 0.f), pq = e;
#pragma unroll
    for (int r = 0; r < RG; ++r) {
      const float4 a4 = reinterpret_cast<const float4 *>(s_red + r * DV)[cg];
      const float4 b4 = reinterpret_cast<const float4 *>(s_red + (RG + r) * DV)[cg];
      e.x += a4.x; e.y += a4.y; e.z += a4.z; e.w += a4.w;
      pq.x += b4.x; pq.y += b4.y; pq.z += b4.z; pq.w += b4.w;
    }
    const float4 vv = reinterpret_cast<const float4 *>(s_v)[cg];
    if (rg == 0) {
      const float zq = s_dot[0], kq = s_dot[1];
      __stcs(reinterpret_cast<float4 *>(o + (size_t)bh * DV) + cg,
             make_float4(pq.x - e.x * zq + vv.x * kq, pq.y - e.y * zq + vv.y * kq,
                         pq.z - e.z * zq + vv.z * kq, pq.w - e.w * zq + vv.w * kq));
    }
    float *Sbh = S + (size_t)bh * DK * DV;
#pragma unroll
    for (int r = 0; r < RPT; ++r) {
      const int j = r * RG + rg;
      const float wj = s_w[j], zj = s_z[j], kj = s_k[j];
      __stcs(reinterpret_cast<float4 *>(Sbh + (size_t)j * DV) + cg,
             make_float4(sr[r].x * wj - zj * e.x + kj * vv.x, sr[r].y * wj - zj * e.y + kj * vv.y,
                         sr[r].z * wj - zj * e.z + kj * vv.z, sr[r].w * wj - zj * e.w + kj * vv.w));
    }
  }
  cp_async_wait<0>();
}

template <typename Tin>
cudaError_t launch_pipe(const gdr_step_args &a, cudaStream_t stream) {
  using P = PipeShape<Tin>;
  const int nbh = a.B * a.H;
  if (nbh == 0) return cudaSuccess;
  int dev = 0, sms = 148;
  if (cudaGetDevice(&dev) == cudaSuccess)
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  cudaError_t e = cudaFuncSetAttribute(decode_pipe_kernel<Tin>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, P::SMEM);
  if (e != cudaSuccess) return e;
  const int grid = nbh < sms ? nbh : sms;
  decode_pipe_kernel<Tin><<<grid, P::NT, P::SMEM, stream>>>(
      a.form, nbh, static_cast<const Tin *>(a.q), static_cast<const Tin *>(a.k),
      static_cast<const Tin *>(a.v), a.log_w, static_cast<const Tin *>(a.e1),
      static_cast<const Tin *>(a.e2), a.S, a.o);
  return cudaGetLastError();
}

template <int DK, int DV, typename Tin>
cudaError_t launch_t(const gdr_step_args &a, cudaStream_t stream) {
  const int nbh = a.B * a.H;
  if (nbh == 0) return cudaSuccess;
  decode_step_kernel<DK, DV, Tin><<<nbh, DecodeShape<DK, DV>::NT, 0, stream>>>(
      a.form, static_cast<const Tin *>(a.q), static_cast<const Tin *>(a.k),
      static_cast<const Tin *>(a.v), a.log_w, static_cast<const Tin *>(a.e1),
      static_cast<const Tin *>(a.e2), a.S, a.o);
  return cudaGetLastError();
}

template <int DK, typename Tin>
cudaError_t dispatch_dv(const gdr_step_args &a, cudaStream_t s) {
  switch (a.dv) {
    case 16: return launch_t<DK, 16, Tin>(a, s);
    case 32: return launch_t<DK, 32, Tin>(a, s);
    case 64: return launch_t<DK, 64, Tin>(a, s);
    case 128: return launch_t<DK, 128, Tin>(a, s);
  }
  return cudaErrorInvalidValue;
}

template <typename Tin>
cudaError_t dispatch_dk(const gdr_step_args &a, cudaStream_t s) {
  switch (a.dk) {
    case 16: return dispatch_dv<16, Tin>(a, s);
    case 32: return dispatch_dv<32, Tin>(a, s);
    case 64: return dispatch_dv<64, Tin>(a, s);
    case 128: return dispatch_dv<128, Tin>(a, s);
  }
  return cudaErrorInvalidValue;
}

}  // namespace

cudaError_t launch_decode(const gdr_step_args &a, cudaStream_t stream) {
  // the pipelined kernel covers d_k = d_v = 128 outside the RWKV-7 form (whose
  // per-head scalar coefficient is not a 16-byte copy)
  if (a.dk == 128 && a.dv == 128 && a.form != GDR_FORM_RWKV7)
    return a.dtype == GDR_BF16 ? launch_pipe<__nv_bfloat16>(a, stream)
                               : launch_pipe<float>(a, stream);
  return a.dtype == GDR_BF16 ? dispatch_dk<__nv_bfloat16>(a, stream)
                             : dispatch_dk<float>(a, stream);
}

}  // namespace gdr
