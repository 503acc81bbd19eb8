// gdr_fwd_tc.cu -- chunkwise forward on the sm_100a tensor cores (tcgen05 + TMEM).
//
// Chunkwise algorithm: "Muir: Linear Attention with Sensitivity-Allocated Gating
// and Matched-Filter Readout", section 2.2 and section 4.2.  GDN-2 form, bf16
// inputs, d_k = d_v = 128, chunk C = 64.  Storage orientation S[j][c] (key j,
// value c), row vectors.  For one chunk of n <= C tokens starting from S0:
//
//   Lam_t      = sum_{r <= t} log alpha_r                        (fp32, <= 0)
//   pi_t       = exp(Lam_t),  k^_t = b_t (.) k_t,  v^_t = wg_t (.) v_t
//   f_t        = exp(Lam_t - Lam_1) <= 1,   g_s = exp(Lam_1 - Lam_s) >= 1
//   L[t][s]    = <k^_t (.) f_t, k_s (.) g_s>   (s < t)   = <k^_t, pi_{t,s} (.) k_s>
//   M[t][s]    = <q_t  (.) f_t, k_s (.) g_s>   (s <= t)  = <q_t,  pi_{t,s} (.) k_s>
//   T          = I + L,   U = T^-1 V^,   Y = T^-1 K^_pi = (T^-1 (K^ (.) f)) Diag(alpha_1)
//   V~         = U - Y S0
//   S_C        = Diag(pi_n) S0 + K~^T V~,     K~_s = exp(Lam_n - Lam_s) (.) k_s
//   O          = Q_pi S0 + M V~
//
// The decay split.  The pages evaluate the relative decays pi_{t,s} with
// boundary pivots so that no factor exceeds 1 (section 4.2).  On this chip the
// whole C x C product is one tensor-core MMA, so the kernel uses a single pivot,
// the chunk's first token: the row factor f_t <= 1 and the column factor
// g_s >= 1.  g_s is bounded by exp(80) whenever the chunk's log-decay after its
// first token, Lam_1 - Lam_n, stays below 80 in every channel, which keeps every
// operand a normal fp32/bf16 number; the kernel checks the bound per chunk and,
// for a chunk that exceeds it, forms L and M on the CUDA cores from the exact
// pairwise decays exp(Lam_t - Lam_s) instead.  Nothing is divided and no
// exponent is ever positive beyond 80.  (Pivoting at the first token also makes
// the chunk's first diagonal products exact: f_1 = g_1 = 1.)
//
// Mapping to the hardware.  One CTA per (b, h, 64-column value slice); 256
// threads; each chunk runs as five tcgen05 MMA groups (bf16 operands in 128-byte
// swizzled shared-memory tiles, fp32 accumulators in 256 TMEM columns) separated
// by CUDA-core phases:
//   MMA1  [K^ f; Q f] (128 x 128) x (K g)^T (128 x 64)         -> L, M
//   fp32  T^-1 by blocked inversion (16 x 16 diagonal blocks, two merge levels)
//   MMA2  T^-1 x [V^ | K^ f]                                    -> U, Y Diag(1/alpha_1)
//   MMA3  Y x S0,  Q_pi x S0                                     -> Y S0, O partial
//   MMA4  K~^T x V~,  M x V~                                     -> S_C increment, O
// The fp32 state slice lives in registers (thread = key channel, 32 columns);
// its bf16 copy in shared memory is the B operand of MMA3.
#include "gdr_tc_common.cuh"

// Phase hooks for an external timing harness; empty in the library build.
#ifndef GDR_PHASE
#define GDR_PHASE(i)
#endif

namespace gdr {
namespace {


using namespace tc;
using Ix = PaddedIdx;

template <int NV>
struct TcSmem {
  static constexpr uint32_t A_LM = 0;                          // [K_pi; Q_pi]  2C x DK bf16
  static constexpr uint32_t B_LM = A_LM + 2 * kC * kDK * 2;     // K / pi        C x DK
  static constexpr uint32_t KT = B_LM + kC * kDK * 2;           // K~            C x DK
  static constexpr uint32_t VH = KT + kC * kDK * 2;             // V^            C x NV
  static constexpr uint32_t TINV = VH + kC * NV * 2;            // T^-1          C x C
  static constexpr uint32_t MM = TINV + kC * kC * 2;            // M             C x C
  static constexpr uint32_t YY = MM + kC * kC * 2;              // Y             C x DK
  static constexpr uint32_t VT = YY + kC * kDK * 2;             // V~            C x NV
  static constexpr uint32_t S0B = VT + kC * NV * 2;             // bf16 S0       DK x NV
  static constexpr uint32_t QP = S0B + kDK * NV * 2;            // Q_pi          C x DK
  static constexpr uint32_t LAM = QP + kC * kDK * 2;            // fp32 Lambda   C x DK
  static constexpr uint32_t LF = LAM + kC * kDK * 4;            // fp32 L        (padded rows)
  static constexpr uint32_t TI = LF + Ix::kBytes;               // fp32 T^-1     (padded rows)
  static constexpr uint32_t PIN = TI + Ix::kBytes;              // fp32 exp(Lam_n) DK
  static constexpr uint32_t A1 = PIN + kDK * 4;                 // fp32 alpha_1 = exp(Lam_1) DK
  static constexpr uint32_t ED = A1 + kDK * 4;                  // fp32 exp(Lam_n - Lam_1) DK
  static constexpr uint32_t TOT = ED + kDK * 4;                 // fp32 first-half log-decay DK
  static constexpr uint32_t MISC = TOT + kDK * 4;               // mbarrier, TMEM slot, flags
  static constexpr uint32_t TOTAL = MISC + 64;
  static constexpr uint32_t ALLOC = TOTAL + 1024;               // + alignment slack
  static_assert(A_LM % 1024 == 0 && B_LM % 1024 == 0 && KT % 1024 == 0 && VH % 1024 == 0 &&
                    TINV % 1024 == 0 && MM % 1024 == 0 && YY % 1024 == 0 && VT % 1024 == 0 &&
                    S0B % 1024 == 0 && QP % 1024 == 0,
                "MMA tiles must be 1024-byte aligned");
};

template <int NV>
__global__ void __launch_bounds__(kThreads, 1) fwd_tc_gdn2_kernel(FwdParams p) {
  static_assert(NV == 64, "this kernel is written for 64-column value slices");
  using SL = TcSmem<NV>;
  constexpr int HALF = NV / 2;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  uint8_t *smem = smem_raw + (((raw + 1023u) & ~1023u) - raw);
  const uint32_t sb = smem_u32(smem);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int qd = warp & 3, hf = warp >> 2;         // TMEM lane quarter, column half
  const int c0 = blockIdx.x * NV, h = blockIdx.y, b = blockIdx.z;
  const int T = p.T, H = p.H;

  float *sLam = reinterpret_cast<float *>(smem + SL::LAM);
  float *sL = reinterpret_cast<float *>(smem + SL::LF);
  float *sTi = reinterpret_cast<float *>(smem + SL::TI);
  float *sPiN = reinterpret_cast<float *>(smem + SL::PIN);
  float *sA1 = reinterpret_cast<float *>(smem + SL::A1);
  float *sED = reinterpret_cast<float *>(smem + SL::ED);
  float *sTot = reinterpret_cast<float *>(smem + SL::TOT);
  uint64_t *mbar = reinterpret_cast<uint64_t *>(smem + SL::MISC);
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + SL::MISC + 8);
  volatile int *sflag = reinterpret_cast<volatile int *>(smem + SL::MISC + 16);  // [0] exact, [1] abort

  const __nv_bfloat16 *gq = static_cast<const __nv_bfloat16 *>(p.q);
  const __nv_bfloat16 *gk = static_cast<const __nv_bfloat16 *>(p.k);
  const __nv_bfloat16 *gv = static_cast<const __nv_bfloat16 *>(p.v);
  const __nv_bfloat16 *gb = static_cast<const __nv_bfloat16 *>(p.e1);
  const __nv_bfloat16 *gw = static_cast<const __nv_bfloat16 *>(p.e2);

  if (warp == 0) {
    tmem_alloc(tmem_slot, kTmemCols);
    tmem_relinquish();
  }
  if (tid == 0) {
    mbar_init(mbar, 1);
    fence_mbar_init();
    sflag[0] = 0;
    sflag[1] = 0;
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  uint32_t phase = 0;

  // TMEM columns: [0,64) L|M, later Y S0, later the S_C increment; [64,64+NV) U;
  // [64+NV, 192+NV) Y, later O.
  const uint32_t tLM = tmem, tD1 = tmem, tDS = tmem;
  const uint32_t tU = tmem + 64, tY = tmem + 64 + NV, tDO = tmem + 64 + NV;
  const uint32_t lane_q = (uint32_t)(32 * qd) << 16;

  // fp32 state: this thread owns key channel jrow, value columns [hf*HALF, hf*HALF + HALF)
  const int jrow = 32 * qd + lane;
  const size_t s_off = (((size_t)b * H + h) * kDK + jrow) * kDK + c0 + hf * HALF;
  float st[HALF];
#pragma unroll
  for (int i = 0; i < HALF; i += 4) {
    float4 x = p.S0 ? __ldg(reinterpret_cast<const float4 *>(p.S0 + s_off + i))
                    : make_float4(0.f, 0.f, 0.f, 0.f);
    st[i] = x.x; st[i + 1] = x.y; st[i + 2] = x.z; st[i + 3] = x.w;
  }
#pragma unroll
  for (int i = 0; i < HALF; i += 8)
    st_smem16(smem, SL::S0B + sw128_offset(jrow, hf * HALF + i, kDK * 128), pack8(st + i));
  fence_proxy_async_smem();
  __syncthreads();

  bool ok = true;
  for (int t0 = 0; t0 < T && ok; t0 += kC) {
    const int n = min(kC, T - t0);

    // ---- every global read of the chunk is issued first, before any use
    // log w: thread (channel jc, half hh) holds tokens [32 hh, 32 hh + 32)
    const int jc = tid & (kDK - 1), hh = tid >> 7;
    float lw[32];
#pragma unroll
    for (int t = 0; t < 32; ++t) {
      const int tt = 32 * hh + t;
      lw[t] = (tt < n) ? __ldg(p.log_w + (((size_t)b * T + t0 + tt) * H + h) * kDK + jc) : 0.f;
    }
    // operand inputs: items (t, 8-channel group g), 4 per thread
    uint4 rk[4], rb[4], rq[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int it = tid + u * kThreads, t = it >> 4, g = it & 15;
      if (t < n) {
        const size_t off = (((size_t)b * T + t0 + t) * H + h) * kDK + 8 * g;
        rk[u] = ld16(gk + off);
        rb[u] = ld16(gb + off);
        rq[u] = ld16(gq + off);
      } else {
        rk[u] = rb[u] = rq[u] = make_uint4(0u, 0u, 0u, 0u);
      }
    }
    // value inputs: items (t, g < NV / 8), 2 per thread
    constexpr int kVItems = kC * (NV / 8) / kThreads;
    uint4 rv[kVItems], rw[kVItems];
#pragma unroll
    for (int u = 0; u < kVItems; ++u) {
      const int it = tid + u * kThreads, t = it / (NV / 8), g = it % (NV / 8);
      if (t < n) {
        const size_t off = (((size_t)b * T + t0 + t) * H + h) * kDK + c0 + 8 * g;
        rv[u] = ld16(gv + off);
        rw[u] = gw ? ld16(gw + off) : make_uint4(0x3F803F80u, 0x3F803F80u, 0x3F803F80u, 0x3F803F80u);
      } else {
        rv[u] = rw[u] = make_uint4(0u, 0u, 0u, 0u);
      }
    }

    // ---- V^ = wg (.) v (needs no decay)
#pragma unroll
    for (int u = 0; u < kVItems; ++u) {
      const int it = tid + u * kThreads, t = it / (NV / 8), g = it % (NV / 8);
      float v8[8], w8[8];
      unpack8(rv[u], v8);
      unpack8(rw[u], w8);
#pragma unroll
      for (int e = 0; e < 8; ++e) v8[e] *= w8[e];
      st_smem16(smem, SL::VH + sw128_offset(t, 8 * g, kC * 128), pack8(v8));
    }

    // ---- P0: cumulative log-decay Lam_t (two halves of the chunk, then joined)
    {
      float acc = 0.f;
#pragma unroll
      for (int t = 0; t < 32; ++t) {
        acc += lw[t];
        lw[t] = acc;
      }
      if (hh == 0) {
#pragma unroll
        for (int t = 0; t < 32; ++t) sLam[t * kDK + jc] = lw[t];
        sTot[jc] = acc;
      }
      __syncthreads();
      if (hh == 1) {
        const float base = sTot[jc], lam1 = sLam[jc];
#pragma unroll
        for (int t = 0; t < 32; ++t) sLam[(32 + t) * kDK + jc] = base + lw[t];
        const float lamn = base + acc;
        sPiN[jc] = __expf(lamn);
        sA1[jc] = __expf(lam1);
        sED[jc] = __expf(lamn - lam1);
        if (lam1 - lamn > kMaxChunkDecay) sflag[0] = 1;
      }
      __syncthreads();
    }
    const bool exact = sflag[0] != 0;

    GDR_PHASE(0);
    // ---- P1: operand tiles [K^ f; Q f], K g, K~, Q_pi
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int it = tid + u * kThreads, t = it >> 4, g = it & 15, j0 = 8 * g;
      float k8[8], b8[8], q8[8];
      unpack8(rk[u], k8);
      unpack8(rb[u], b8);
      unpack8(rq[u], q8);
      const float4 *lp = reinterpret_cast<const float4 *>(sLam + t * kDK + j0);
      const float4 *l1p = reinterpret_cast<const float4 *>(sLam + j0);
      const float4 *ln = reinterpret_cast<const float4 *>(sLam + (kC - 1) * kDK + j0);
      const float4 l0 = lp[0], l1 = lp[1], f0 = l1p[0], f1 = l1p[1], n0 = ln[0], n1 = ln[1];
      const float lam[8] = {l0.x, l0.y, l0.z, l0.w, l1.x, l1.y, l1.z, l1.w};
      const float lam1[8] = {f0.x, f0.y, f0.z, f0.w, f1.x, f1.y, f1.z, f1.w};
      const float lamn[8] = {n0.x, n0.y, n0.z, n0.w, n1.x, n1.y, n1.z, n1.w};
      float a1[8], a2[8], bl[8], kt[8], qp[8];
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        const float f = __expf(lam[e] - lam1[e]);
        a1[e] = b8[e] * k8[e] * f;
        a2[e] = q8[e] * f;
        qp[e] = a2[e] * sA1[j0 + e];
        if (!exact) {
          bl[e] = k8[e] * __expf(lam1[e] - lam[e]);
          kt[e] = bl[e] * sED[j0 + e];
        } else {
          bl[e] = 0.f;
          kt[e] = k8[e] * __expf(lamn[e] - lam[e]);
        }
      }
      st_smem16(smem, SL::A_LM + sw128_offset(t, j0, 2 * kC * 128), pack8(a1));
      st_smem16(smem, SL::A_LM + sw128_offset(kC + t, j0, 2 * kC * 128), pack8(a2));
      st_smem16(smem, SL::B_LM + sw128_offset(t, j0, kC * 128), pack8(bl));
      st_smem16(smem, SL::KT + sw128_offset(t, j0, kC * 128), pack8(kt));
      st_smem16(smem, SL::QP + sw128_offset(t, j0, kC * 128), pack8(qp));
    }
    fence_proxy_async_smem();
    __syncthreads();

    GDR_PHASE(1);
    // ---- MMA1: [K^ f; Q f] (M = 128) x (K g)^T (N = C), K = DK
    if (tid == 0) {
      tc_fence_after();
      constexpr uint32_t id = idesc_bf16_f32(128, kC, false, false);
#pragma unroll
      for (int s = 0; s < kDK / 16; ++s) {
        const uint64_t ad = sdesc_sw128(sb + SL::A_LM + (s >> 2) * (2 * kC * 128) + (s & 3) * 32, 16, 1024);
        const uint64_t bd = sdesc_sw128(sb + SL::B_LM + (s >> 2) * (kC * 128) + (s & 3) * 32, 16, 1024);
        mma_bf16(tLM, ad, bd, id, s > 0);
      }
      if (!(p.debug & kDebugSkipHandoff)) mma_commit(mbar);   // (withheld in the fault test)
    }
    if (!(ok = wait_mma(mbar, phase, sflag + 1))) break;

    GDR_PHASE(2);
    // ---- L (fp32, strictly lower) and M (bf16, lower incl. diagonal) out of TMEM
    if (!exact) {
      float x[32];
      tmem_ld_32x32b_x32(tLM + lane_q + 32 * hf, x);
      tmem_ld_wait();
      const int r = 32 * qd + lane;
      if (r < kC) {
#pragma unroll
        for (int i = 0; i < 32; ++i) x[i] = (32 * hf + i < r) ? x[i] : 0.f;
#pragma unroll
        for (int i = 0; i < 32; i += 4)
          *reinterpret_cast<float4 *>(sL + Ix::at(r, 32 * hf + i)) =
              make_float4(x[i], x[i + 1], x[i + 2], x[i + 3]);
      } else {
        const int t = r - kC;
#pragma unroll
        for (int i = 0; i < 32; ++i) x[i] = (32 * hf + i <= t) ? x[i] : 0.f;
#pragma unroll
        for (int i = 0; i < 32; i += 8)
          st_smem16(smem, SL::MM + sw128_offset(t, 32 * hf + i, kC * 128), pack8(x + i));
      }
      tc_fence_before();
    } else {
      // exact pairwise decays on the CUDA cores (chunks whose decay exceeds the bound)
      for (int it = tid; it < kC * kC; it += kThreads) {
        const int t = it / kC, s = it % kC;
        float l = 0.f, m = 0.f;
        if (s <= t && t < n) {
          const size_t ot = (((size_t)b * T + t0 + t) * H + h) * kDK;
          const size_t os = (((size_t)b * T + t0 + s) * H + h) * kDK;
          for (int j = 0; j < kDK; ++j) {
            const float d = __expf(sLam[t * kDK + j] - sLam[s * kDK + j]);
            const float ks = __bfloat162float(gk[os + j]);
            m += __bfloat162float(gq[ot + j]) * d * ks;
            l += __bfloat162float(gb[ot + j]) * __bfloat162float(gk[ot + j]) * d * ks;
          }
        }
        sL[Ix::at(t, s)] = (s < t) ? l : 0.f;
        *reinterpret_cast<__nv_bfloat16 *>(smem + SL::MM + sw128_offset(t, s, kC * 128)) =
            __float2bfloat16_rn(m);
      }
    }
    __syncthreads();

    GDR_PHASE(3);
    // ---- T^-1 (fp32), then bf16 copy as the A operand of MMA2
    invert_unit_lower<Ix, Ix>(sL, sTi, tid);
    for (int it = tid; it < kC * (kC / 8); it += kThreads) {
      const int t = it >> 3, g = it & 7;
      const float4 y0 = *reinterpret_cast<const float4 *>(sTi + Ix::at(t, 8 * g));
      const float4 y1 = *reinterpret_cast<const float4 *>(sTi + Ix::at(t, 8 * g + 4));
      float x[8] = {y0.x, y0.y, y0.z, y0.w, y1.x, y1.y, y1.z, y1.w};
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        const int s = 8 * g + e;
        x[e] = (s < t) ? x[e] : (s == t ? 1.f : 0.f);
      }
      st_smem16(smem, SL::TINV + sw128_offset(t, 8 * g, kC * 128), pack8(x));
    }
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();

    GDR_PHASE(4);
    // ---- MMA2: U = T^-1 V^ (N = NV), Y Diag(1/alpha_1) = T^-1 (K^ f) (N = DK); K = C
    if (tid == 0) {
      tc_fence_after();
      constexpr uint32_t idu = idesc_bf16_f32(64, NV, false, true);
      constexpr uint32_t idy = idesc_bf16_f32(64, kDK, false, true);
#pragma unroll
      for (int s = 0; s < kC / 16; ++s) {
        const uint64_t ad = sdesc_sw128(sb + SL::TINV + s * 32, 16, 1024);
        const uint64_t bu = sdesc_sw128(sb + SL::VH + s * 2048, kC * 128, 1024);
        const uint64_t by = sdesc_sw128(sb + SL::A_LM + s * 2048, 2 * kC * 128, 1024);
        mma_bf16(tU, ad, bu, idu, s > 0);
        mma_bf16(tY, ad, by, idy, s > 0);
      }
      mma_commit(mbar);
    }
    if (!(ok = wait_mma(mbar, phase, sflag + 1))) break;

    GDR_PHASE(5);
    // ---- Y = (T^-1 (K^ f)) Diag(alpha_1) -> bf16 (K-major, rows = tokens);
    //      M = 64 accumulators hold row 16 qd + lane
    {
      float y[32];
#pragma unroll
      for (int part = 0; part < 2; ++part) {
        tmem_ld_32x32b_x32(tY + lane_q + 64 * hf + 32 * part, y);
        tmem_ld_wait();
        if (lane < 16) {
          const int t = 16 * qd + lane;
#pragma unroll
          for (int i = 0; i < 32; ++i) y[i] *= sA1[64 * hf + 32 * part + i];
#pragma unroll
          for (int i = 0; i < 32; i += 8)
            st_smem16(smem, SL::YY + sw128_offset(t, 64 * hf + 32 * part + i, kC * 128),
                      pack8(y + i));
        }
      }
    }
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();

    GDR_PHASE(6);
    // ---- MMA3: Y S0 and Q_pi S0 (K = DK)
    if (tid == 0) {
      tc_fence_after();
      constexpr uint32_t id = idesc_bf16_f32(64, NV, false, true);
#pragma unroll
      for (int s = 0; s < kDK / 16; ++s) {
        const uint64_t ay = sdesc_sw128(sb + SL::YY + (s >> 2) * (kC * 128) + (s & 3) * 32, 16, 1024);
        const uint64_t aq = sdesc_sw128(sb + SL::QP + (s >> 2) * (kC * 128) + (s & 3) * 32, 16, 1024);
        const uint64_t bs = sdesc_sw128(sb + SL::S0B + s * 2048, kDK * 128, 1024);
        mma_bf16(tD1, ay, bs, id, s > 0);
        mma_bf16(tDO, aq, bs, id, s > 0);
      }
      mma_commit(mbar);
    }
    if (!(ok = wait_mma(mbar, phase, sflag + 1))) break;

    GDR_PHASE(7);
    // ---- V~ = U - Y S0 -> bf16 (rows = tokens)
    {
      float u[32], d[32];
      tmem_ld_32x32b_x32(tU + lane_q + hf * HALF, u);
      tmem_ld_32x32b_x32(tD1 + lane_q + hf * HALF, d);
      tmem_ld_wait();
      if (lane < 16) {
        const int t = 16 * qd + lane;
#pragma unroll
        for (int i = 0; i < 32; ++i) u[i] = (t < n) ? u[i] - d[i] : 0.f;
#pragma unroll
        for (int i = 0; i < 32; i += 8)
          st_smem16(smem, SL::VT + sw128_offset(t, hf * HALF + i, kC * 128), pack8(u + i));
      }
    }
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();

    GDR_PHASE(8);
    // ---- MMA4: K~^T V~ (M = DK) and O += M V~ (M = C); K = C
    if (tid == 0) {
      tc_fence_after();
      constexpr uint32_t ids = idesc_bf16_f32(128, NV, true, true);
      constexpr uint32_t ido = idesc_bf16_f32(64, NV, false, true);
#pragma unroll
      for (int s = 0; s < kC / 16; ++s) {
        const uint64_t ak = sdesc_sw128(sb + SL::KT + s * 2048, kC * 128, 1024);
        const uint64_t bv = sdesc_sw128(sb + SL::VT + s * 2048, kC * 128, 1024);
        const uint64_t am = sdesc_sw128(sb + SL::MM + s * 32, 16, 1024);
        mma_bf16(tDS, ak, bv, ids, s > 0);
        mma_bf16(tDO, am, bv, ido, 1);
      }
      mma_commit(mbar);
    }
    if (!(ok = wait_mma(mbar, phase, sflag + 1))) break;

    GDR_PHASE(9);
    // ---- state update (fp32) and outputs
    {
      float d[32];
      tmem_ld_32x32b_x32(tDS + lane_q + hf * HALF, d);
      tmem_ld_wait();
      const float pn = sPiN[jrow];
#pragma unroll
      for (int i = 0; i < HALF; ++i) st[i] = pn * st[i] + d[i];
#pragma unroll
      for (int i = 0; i < HALF; i += 8)
        st_smem16(smem, SL::S0B + sw128_offset(jrow, hf * HALF + i, kDK * 128), pack8(st + i));
      float o[32];
      tmem_ld_32x32b_x32(tDO + lane_q + hf * HALF, o);
      tmem_ld_wait();
      if (lane < 16) {
        const int t = 16 * qd + lane;
        if (t < n) {
          float4 *dst = reinterpret_cast<float4 *>(
              p.o + (((size_t)b * T + t0 + t) * H + h) * kDK + c0 + hf * HALF);
#pragma unroll
          for (int i = 0; i < HALF; i += 4) dst[i / 4] = make_float4(o[i], o[i + 1], o[i + 2], o[i + 3]);
        }
      }
    }
    if (tid == 0) sflag[0] = 0;
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
    GDR_PHASE(10);
  }

  if (ok && p.S_T) {
#pragma unroll
    for (int i = 0; i < HALF; i += 4)
      *reinterpret_cast<float4 *>(p.S_T + s_off + i) = make_float4(st[i], st[i + 1], st[i + 2], st[i + 3]);
  }
  if (!ok) {
    // A tensor-core group did not complete in time: report it, give the
    // in-flight group one more bounded wait, then release TMEM.
    if (tid == 0) {
      if (p.status) atomicExch(p.status, (uint32_t)GDR_ERR_TIMEOUT);
      mbar_wait_bounded(mbar, phase ^ 1u, kWaitLimitNs);   // wait_mma advanced `phase` past it
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

}  // namespace

// The tensor-core kernels evaluate the chunkwise form with C = 64; a requested chunk
// of 128 is served with two 64-token chunks (the result depends on the chunk length
// only through rounding).  Smaller requested chunks go to the fp32 kernel.
bool forward_tc_supported(const FwdParams &p, gdr_dtype dtype) {
  return p.form == GDR_FORM_GDN2 && dtype == GDR_BF16 && p.dk == kDK && p.dv == kDK &&
         (p.chunk == kC || p.chunk == 2 * kC);
}

cudaError_t launch_forward_tc(const FwdParams &p, cudaStream_t stream) {
  constexpr int NV = 64;
  const size_t smem = TcSmem<NV>::ALLOC;
  cudaError_t e = cudaFuncSetAttribute(fwd_tc_gdn2_kernel<NV>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  dim3 grid(p.dv / NV, p.H, p.B);
  fwd_tc_gdn2_kernel<NV><<<grid, kThreads, smem, stream>>>(p);
  return cudaGetLastError();
}

}  // namespace gdr
