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
// (2 * dk * dv * 4 bytes per head).  One CTA per (b, h); each thread keeps RPT
// rows x 4 columns of the state in registers between the read and the write, so
// the state is read exactly once.  A warp reads whole rows (float4 per lane,
// 512 contiguous bytes at dv = 128); the reduction over rows runs across warps
// through shared memory.  Loads and stores use the streaming cache hints: the
// state (1 GiB at B=256, H=32, d=128) is far larger than L2 and is not reused
// within a step.
#include "gdr_internal.cuh"

namespace gdr {
namespace {

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
  return a.dtype == GDR_BF16 ? dispatch_dk<__nv_bfloat16>(a, stream)
                             : dispatch_dk<float>(a, stream);
}

}  // namespace gdr
