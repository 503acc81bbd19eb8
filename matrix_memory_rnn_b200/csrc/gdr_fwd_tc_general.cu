// gdr_fwd_tc_general.cu -- chunked forward of the generalized delta rule on the
// tensor cores at d_k = d_v = 64 (bf16 inputs, chunks of C = 64 tokens), written for
// the two-stream form and serving every form through its mapping:
// GDR_FORM_GENERAL (u, z given), GDR_FORM_RWKV7 (u = c a, z = a), GDR_FORM_GDN2
// (u = alpha (.) b (.) k, z = k, written value wg (.) v) and GDR_FORM_GLA (u = z = 0).
//
// "Exponential gates and matrix memory: xLSTM and RWKV-7", section 13.3 (the
// generalized delta rule; the erase reads the undecayed state S_{t-1}), evaluated
// in the chunkwise form of "Muir: Linear Attention with Sensitivity-Allocated
// Gating and Matched-Filter Readout", sections 2.2 and 4.2, generalized to a
// separate erase key z (two write streams).  In the storage orientation (state
// d_k x d_v, row vectors) and with Lam_t the cumulative log-decay of the chunk
// through token t (Lam_{-1} = 0), for tokens t, s of one chunk with initial state S0:
//   A[t,s]   = <u_t e^{Lam_{t-1}-Lam_s}, z_s>,  B[t,s] = <u_t e^{Lam_{t-1}-Lam_s}, k_s>  (s < t)
//   M_z[t,s] = <q_t e^{Lam_t-Lam_s}, z_s>,      M_k[t,s] = <q_t e^{Lam_t-Lam_s}, k_s>    (s <= t)
//   (I + A) E = U_pi S0 + B V       (row t of E: the erase read e_t = u_t^T S_{t-1})
//   O   = Q_pi S0 + M_k V - M_z E,   S_C = Diag(pi_C) S0 + K~^T V - Z~^T E
// with U_pi = u (.) e^{Lam_{t-1}}, Q_pi = q (.) e^{Lam_t}, K~ = k (.) e^{Lam_C - Lam_s},
// Z~ likewise.  With T = I + A, Y_u = T^-1 U_pi and W = T^-1 (B V), E = Y_u S0 + W,
// and writing V~ = -E = (-W) - Y_u S0:
//   S_C = Diag(pi_C) S0 + K~^T V + Z~^T V~,   O = Q_pi S0 + M_k V + M_z V~
// -- the carry of the single-stream kernels plus the two S0-free terms K~^T V and
// M_k V.
//
// One CTA of 256 threads per (b, h) walks its chunks in order (fused: the
// sequences are many and short in the workloads this serves); shared-memory
// slots are reused across the chunk's phases so that two CTAs share an SM.  Per chunk, five
// tcgen05 MMA groups with bf16 operands in 128-byte-swizzled shared memory and
// fp32 accumulators in TMEM, CUDA-core phases in between:
//   MMA1   [U f'; Q f] (M = 128) x [Z g; K g]^T (N = 128), K = d_k   -> A, B, M_z, M_k
//   MMA-BV B V (M = 64), and K~^T V into the state accumulator        (overlaps T^-1)
//   MMA2   T^-1 [U_pi | B V] (M = 64, N = 128)                        -> Y_u, W
//   MMA3   [Q_pi; Y_u] S0' (M = 128), and M_k V into the output accumulator
//   MMA4   state += Z~^T V~, output += M_z V~
// The decay is split at the chunk's first token (f = e^{Lam_t - Lam_0} <= 1,
// g = e^{Lam_0 - Lam_s} <= e^{80}); a chunk whose log-decay exceeds 80 in some
// channel forms A, B, M_z, M_k from the exact pairwise decays instead.  T^-1 is
// the blocked fp32 inverse shared with the single-stream kernels.
#include <cuda.h>
#include <cudaTypedefs.h>

#include <cstring>
#include <mutex>

#include "gdr_tc_common.cuh"

// Phase marks of the timing build (thread 0, cycles summed over CTAs and chunks into
// g_general_cycles); empty in libgdr.so.
#ifdef GDR_PHASE_TIMING
namespace gdr {
__device__ unsigned long long g_general_cycles[16];
}
#define GT_INIT                                                                     \
  long long gt_a_[16] = {0};                                                        \
  long long gt_l_ = 0;
#define GT_MARK(i)                                                                  \
  do {                                                                              \
    if (threadIdx.x == 0) {                                                         \
      const long long n_ = clock64();                                               \
      if (gt_l_) gt_a_[i] += n_ - gt_l_;                                            \
      gt_l_ = n_;                                                                   \
    }                                                                               \
  } while (0)
#define GT_FINI                                                                     \
  if (threadIdx.x == 0)                                                             \
    for (int i_ = 0; i_ < 16; ++i_) atomicAdd(&gdr::g_general_cycles[i_], (unsigned long long)gt_a_[i_]);
#else
#define GT_INIT
#define GT_MARK(i)
#define GT_FINI
#endif

namespace gdr {
namespace {

using namespace tc;
using Ix = SwizzledIdx;
constexpr int kD = 64;                      // d_k = d_v
constexpr int kGT = 256;                    // threads per CTA
constexpr uint32_t kTile = kC * kD * 2;     // one 64 x 64 bf16 tile in the sw128 layout (8 KB)

// Shared memory: thirteen 8 KB slots (bf16 64 x 64 tiles in the sw128 layout, rows =
// tokens unless stated) from a 1024-aligned base, reused as the chunk goes on, so two
// CTAs fit on an SM:
//   slot 0      v (TMA)                                   -> next chunk's v after MMA3
//   slot 1      S0' [j][c], bf16 copy of the state (B operand of MMA3)
//   slot 2      U_pi                        } B operand of MMA2: two atoms, U_pi first
//   slot 3      K~ [s][j] (MN-major A; slot 4 is its junk atom)
//   slot 4      Z~ [s][j] (MN-major A; slot 5 is its junk atom)
//   slots 5-6   u | q (TMA) -> [U f'; Q f] in place (MMA1 A) -> fp32 T^-1 (or, on the
//               exact path, Lam first) -> -W (5), V~ (6)
//   slots 7-8   z | k (TMA) -> [Z g; K g] in place (MMA1 B) -> fp32 A -> bf16 T^-1 (7),
//               B V (8)                     } second atom of MMA2's B operand
//   slots 9-10  log w (TMA, fp32 row-major) -> Lam - Lam_0 -> M_k (9), M_z (10)
//   slots 11-12 [Q_pi; B] -> [Q_pi; Y_u] (MMA3 A)
struct GenSmem {
  static constexpr uint32_t V = 0 * kTile;
  static constexpr uint32_t S0B = 1 * kTile;
  static constexpr uint32_t UP = 2 * kTile;
  static constexpr uint32_t KT = 3 * kTile;
  static constexpr uint32_t ZT = 4 * kTile;
  static constexpr uint32_t A1 = 5 * kTile;        // [U f'; Q f]: u lands in the first half, q in the second
  static constexpr uint32_t B1 = 7 * kTile;        // [Z g; K g]: z lands in the first half, k in the second
  static constexpr uint32_t LW = 9 * kTile;        // log w (16 KB)
  static constexpr uint32_t QY = 11 * kTile;       // [Q_pi; B then Y_u]
  static constexpr uint32_t UW = A1;               // -W
  static constexpr uint32_t VT = A1 + kTile;       // V~ (B operand of MMA4)
  static constexpr uint32_t TI = B1;               // bf16 T^-1 (A operand of MMA2)
  static constexpr uint32_t BV = B1 + kTile;       // B V
  static constexpr uint32_t MK = LW;               // M_k [t][s] (K-major; M_z is its junk rows)
  static constexpr uint32_t MZ = LW + kTile;       // M_z [t][s] (K-major; Q_pi is its junk rows)
  static constexpr uint32_t BB = QY + kTile;       // B [t][s] (K-major A of B V)
  static constexpr uint32_t PI = 13 * kTile;       // fp32 pi_C per channel
  static constexpr uint32_t A1V = PI + kD * 4;     // fp32 alpha_0 = e^{Lam_0} per channel
  static constexpr uint32_t DN = A1V + kD * 4;     // fp32 Lam_63 - Lam_0 per channel
  static constexpr uint32_t QT = DN + kD * 4;      // fp32 [4][d] quarter sums of log w
  static constexpr uint32_t CS = QT + 4 * kD * 4;  // fp32 RWKV-7 c per token
  static constexpr uint32_t MISC = CS + kC * 4;    // barriers, TMEM slot, flags
  static constexpr uint32_t ALLOC = MISC + 128 + 1024;
  static_assert(ALLOC <= 113 * 1024, "two CTAs per SM");
  static_assert(Ix::kBytes <= 2 * kTile, "fp32 64 x 64 must fit a 16 KB region");
  static_assert(BV > UP, "MMA2's B operand: the B V atom follows the U_pi atom");
};

struct GenMisc {
  static constexpr uint32_t IN1 = 0;    // uint64_t q, k, e1, e2, log w landed
  static constexpr uint32_t IN2 = 8;    // uint64_t v landed
  static constexpr uint32_t MB = 16;    // uint64_t MMA completion
  static constexpr uint32_t SLOT = 24;  // uint32_t TMEM base
  static constexpr uint32_t ABORT = 28; // int
  static constexpr uint32_t EXACT = 32; // int
};

// TMEM columns (256 allocated): MMA1 [0, 128); B V [128, 192); state accumulator
// [192, 256); MMA2 [0, 128) after MMA1 is read; MMA3 [0, 64); output extra [128, 192)
// after B V is read.
constexpr uint32_t kT_D1 = 0, kT_BV = 128, kT_DS = 192, kT_M2 = 0, kT_D3 = 0, kT_DO = 128;

struct GenMaps {
  CUtensorMap q, k, v, e1, e2, lw;
  CUtensorMap o;   // stores: boxes of 32 fp32 columns x 32 tokens, 128-byte swizzle
};

// Which tiles a form stages: e1 (u, a or the erase gate b) in the first half of the
// MMA1 A operand, e2 (z, or GDN-2's write gate) in the first half of its B operand.
template <int kForm>
__device__ __forceinline__ bool form_has_e1() { return kForm != GDR_FORM_GLA; }
template <int kForm>
__device__ __forceinline__ bool form_has_e2(bool has_wg) {
  return kForm == GDR_FORM_GENERAL || (kForm == GDR_FORM_GDN2 && has_wg);
}

template <int kForm>
__device__ __forceinline__ void load_in1(uint8_t *smem, const GenMaps &m, uint64_t *bar, int b, int h,
                                         int t0, bool has_wg) {
  using SL = GenSmem;
  const bool e1 = form_has_e1<kForm>(), e2 = form_has_e2<kForm>(has_wg);
  mbar_arrive_expect_tx(bar, (2u + (e1 ? 1u : 0u) + (e2 ? 1u : 0u)) * kTile + kC * kD * 4u);
  if (e1) tma_load_4d(smem + SL::A1, &m.e1, 0, h, t0, b, bar);
  tma_load_4d(smem + SL::A1 + kTile, &m.q, 0, h, t0, b, bar);
  if (e2) tma_load_4d(smem + SL::B1, &m.e2, 0, h, t0, b, bar);
  tma_load_4d(smem + SL::B1 + kTile, &m.k, 0, h, t0, b, bar);
  tma_load_4d(smem + SL::LW, &m.lw, 0, h, t0, b, bar);
}

__device__ __forceinline__ void load_in2(uint8_t *smem, const GenMaps &m, uint64_t *bar, int b, int h,
                                         int t0) {
  mbar_arrive_expect_tx(bar, kTile);
  tma_load_4d(smem + GenSmem::V, &m.v, 0, h, t0, b, bar);
}

// Cumulative log-decay of one chunk, Lam_t - Lam_0 in place in `lw` (row-major
// [t][d] fp32; rows past the sequence are zero).  Thread = (channel, token quarter).
// Also per channel: alpha_0 = e^{Lam_0}, dn = Lam_63 - Lam_0, pi_C = e^{Lam_63}, and
// the exact-path flag when dn < -80.  Ends with a CTA barrier.
__device__ __forceinline__ void chunk_scan(float *lw, float *sQT, float *sA1, float *sDN,
                                           float *sPI, volatile int *sexact, int tid) {
  const int ch = tid & (kD - 1), qt = tid >> 6;
  float x[16];
  float acc = 0.f;
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    acc += lw[(16 * qt + i) * kD + ch];
    x[i] = acc;
  }
  sQT[qt * kD + ch] = acc;
  __syncthreads();
  float excl = 0.f, all = 0.f;
#pragma unroll
  for (int q4 = 0; q4 < 4; ++q4) {
    const float v = sQT[q4 * kD + ch];
    all += v;
    excl += (q4 < qt) ? v : 0.f;
  }
  if (qt == 0) sA1[ch] = x[0];             // Lam_0 (token 0), replaced by alpha_0 below
  __syncthreads();
  const float lam0 = sA1[ch];
  const float shift = excl - lam0;
#pragma unroll
  for (int i = 0; i < 16; ++i) lw[(16 * qt + i) * kD + ch] = x[i] + shift;
  __syncthreads();
  if (qt == 0) {
    const float dn = all - lam0;
    sDN[ch] = dn;
    sA1[ch] = __expf(lam0);
    sPI[ch] = __expf(all);
    if (dn < -kMaxChunkDecay) *sexact = 1;
  }
  __syncthreads();
}

template <int kForm>
__global__ void __launch_bounds__(kGT, 2)
    tc_general_kernel(FwdParams p, const __grid_constant__ GenMaps maps) {
  constexpr bool kRwkv = kForm == GDR_FORM_RWKV7;
  using SL = GenSmem;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  uint8_t *smem = smem_raw + (((raw + 1023u) & ~1023u) - raw);
  const uint32_t sb = smem_u32(smem);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int qd = warp & 3, hf = warp >> 2;
  const int h = blockIdx.x, b = blockIdx.y;
  const int T = p.T, H = p.H, nch = (T + kC - 1) / kC;

  uint8_t *misc = smem + SL::MISC;
  uint64_t *in1 = reinterpret_cast<uint64_t *>(misc + GenMisc::IN1);
  uint64_t *in2 = reinterpret_cast<uint64_t *>(misc + GenMisc::IN2);
  uint64_t *mbar = reinterpret_cast<uint64_t *>(misc + GenMisc::MB);
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(misc + GenMisc::SLOT);
  volatile int *sabort = reinterpret_cast<volatile int *>(misc + GenMisc::ABORT);
  volatile int *sexact = reinterpret_cast<volatile int *>(misc + GenMisc::EXACT);
  float *sLW = reinterpret_cast<float *>(smem + SL::LW);
  float *sA = reinterpret_cast<float *>(smem + SL::B1);
  float *sTi = reinterpret_cast<float *>(smem + SL::A1);
  float *sPI = reinterpret_cast<float *>(smem + SL::PI);
  float *sA1 = reinterpret_cast<float *>(smem + SL::A1V);
  float *sDN = reinterpret_cast<float *>(smem + SL::DN);
  float *sQT = reinterpret_cast<float *>(smem + SL::QT);
  float *sC = reinterpret_cast<float *>(smem + SL::CS);
  const __nv_bfloat16 *gq = static_cast<const __nv_bfloat16 *>(p.q);
  const __nv_bfloat16 *gk = static_cast<const __nv_bfloat16 *>(p.k);
  const __nv_bfloat16 *ge1 = static_cast<const __nv_bfloat16 *>(p.e1);
  const __nv_bfloat16 *ge2 = static_cast<const __nv_bfloat16 *>(p.e2);   // z, RWKV-7 c [B][T][H], or wg
  const bool has_wg = kForm == GDR_FORM_GDN2 && p.e2 != nullptr;

  if (warp == 0) {
    tmem_alloc(tmem_slot, kTmemCols);
    tmem_relinquish();
  }
  if (tid == 0) {
    mbar_init(in1, 1);
    mbar_init(in2, 1);
    mbar_init(mbar, 1);
    fence_mbar_init();
    *sabort = 0;
    if (nch > 0) {
      load_in1<kForm>(smem, maps, in1, b, h, 0, has_wg);
      load_in2(smem, maps, in2, b, h, 0);
    }
  }
  // RWKV-7 c of the first chunk (lanes of warp 0, two tokens each)
  float cnext[2] = {0.f, 0.f};
  if (kRwkv && warp == 0) {
#pragma unroll
    for (int i = 0; i < 2; ++i) {
      const int t = 2 * lane + i;
      cnext[i] = t < T ? __bfloat162float(ge2[((size_t)b * T + t) * H + h]) : 0.f;
    }
  }

  // fp32 state on warps with qd < 2: key channel jrow, value columns [32 hf, 32 hf + 32)
  const int jrow = 32 * qd + lane;
  const bool owner = qd < 2;
  const size_t s_off = (((size_t)b * H + h) * kD + jrow) * kD + 32 * hf;
  float st[32];
#pragma unroll
  for (int i = 0; i < 32; ++i) st[i] = 0.f;
  if (owner && p.S0) {
#pragma unroll
    for (int i = 0; i < 32; i += 4) {
      const float4 x = __ldg(reinterpret_cast<const float4 *>(p.S0 + s_off + i));
      st[i] = x.x; st[i + 1] = x.y; st[i + 2] = x.z; st[i + 3] = x.w;
    }
  }
  if (owner) {
#pragma unroll
    for (int i = 0; i < 32; i += 8)
      st_smem16(smem, SL::S0B + sw128_offset(jrow, 32 * hf + i, kC * 128), pack8(st + i));
  }
  fence_proxy_async_smem();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = __shfl_sync(0xffffffffu, *tmem_slot, 0);
  const uint32_t lane_q = (uint32_t)(32 * qd) << 16;

  uint32_t phase = 0;
  // thread 0's counts: MMA groups committed, input loads issued / waited for
  uint32_t issued_mma = 0, in1_iss = nch > 0 ? 1u : 0u, in2_iss = in1_iss, in1_done = 0, in2_done = 0;
  bool ok = true;
  GT_INIT
  for (int c = 0; c < nch; ++c) {
    const int t0 = c * kC, n = min(kC, T - t0);
    GT_MARK(0);
    // ---- this chunk's inputs have landed; the previous chunk's o stores have read the
    //      staging that this chunk's operand tiles overwrite
    if (tid == 0) bulk_wait_read<0>();
    if (tid == 0 && !*sabort) {
      if (mbar_wait_bounded(in1, c & 1, kWaitLimitNs)) ++in1_done;
      else *sabort = 1;
      if (!*sabort && mbar_wait_bounded(in2, c & 1, kWaitLimitNs)) ++in2_done;
      else *sabort = 1;
      *sexact = 0;
    }
    if (kRwkv && warp == 0) {
      sC[2 * lane] = cnext[0];
      sC[2 * lane + 1] = cnext[1];
    }
    __syncthreads();
    if (!(ok = *sabort == 0)) break;
    GT_MARK(1);

    // ---- cumulative log-decay in place (slots 9-10)
    chunk_scan(sLW, sQT, sA1, sDN, sPI, sexact, tid);
    const bool exact = *sexact != 0;
    GT_MARK(2);

    // ---- operand tiles.  Thread = (channel group g of 8, token pair tp); each input
    //      element is read and its outputs written at the same swizzled offset, so the
    //      pivot-split MMA1 operands replace u, q, z, k in place:
    //        U f' (f' = e^{lam_{t-1}}, row 0 zero), Q f (f = e^{lam_t}), Z g, K g (g = e^{-lam_s});
    //      and the direct (<= 1) tiles go to their own slots:
    //        Q_pi = Q f alpha_0, U_pi = U f' alpha_0 (row 0: u_0), K~, Z~ = (k, z) e^{dn - lam_s}.
    {
      const int g = tid & 7, tp = tid >> 3, j0 = 8 * g;
      float dn[8], a0[8];
      {
        const float4 d0 = *reinterpret_cast<const float4 *>(sDN + j0);
        const float4 d1 = *reinterpret_cast<const float4 *>(sDN + j0 + 4);
        const float4 x0 = *reinterpret_cast<const float4 *>(sA1 + j0);
        const float4 x1 = *reinterpret_cast<const float4 *>(sA1 + j0 + 4);
        dn[0] = d0.x; dn[1] = d0.y; dn[2] = d0.z; dn[3] = d0.w;
        dn[4] = d1.x; dn[5] = d1.y; dn[6] = d1.z; dn[7] = d1.w;
        a0[0] = x0.x; a0[1] = x0.y; a0[2] = x0.z; a0[3] = x0.w;
        a0[4] = x1.x; a0[5] = x1.y; a0[6] = x1.z; a0[7] = x1.w;
      }
      // pivot path: e^{dn} per channel, so that K~'s e^{dn - lam} = e^{dn} e^{-lam} reuses
      // the e^{-lam} of K g; e^{lam} of the thread's first token is the second's f'
      float edn[8], elam_prev[8];
#pragma unroll
      for (int e = 0; e < 8; ++e) edn[e] = exact ? 0.f : __expf(dn[e]);
#pragma unroll
      for (int i = 0; i < 2; ++i) {
        const int t = 2 * tp + i;
        const uint32_t o = sw128_offset(t, j0, kC * 128);
        float lam[8], fp[8], q8[8], k8[8], u8[8], z8[8], x[8];
        {
          const float4 l0 = *reinterpret_cast<const float4 *>(sLW + t * kD + j0);
          const float4 l1 = *reinterpret_cast<const float4 *>(sLW + t * kD + j0 + 4);
          lam[0] = l0.x; lam[1] = l0.y; lam[2] = l0.z; lam[3] = l0.w;
          lam[4] = l1.x; lam[5] = l1.y; lam[6] = l1.z; lam[7] = l1.w;
        }
        // fp: lam_{t-1} (GDN-2 first takes its own decay alpha_t = e^{lam_t - lam_{t-1}}
        // from it, alpha_0 = e^{Lam_0}), then f' = e^{lam_{t-1}} (row 0: unused, 0)
        float at[8];
        if (t > 0) {
          const float4 m0 = *reinterpret_cast<const float4 *>(sLW + (t - 1) * kD + j0);
          const float4 m1 = *reinterpret_cast<const float4 *>(sLW + (t - 1) * kD + j0 + 4);
          fp[0] = m0.x; fp[1] = m0.y; fp[2] = m0.z; fp[3] = m0.w;
          fp[4] = m1.x; fp[5] = m1.y; fp[6] = m1.z; fp[7] = m1.w;
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            if (kForm == GDR_FORM_GDN2) at[e] = __expf(lam[e] - fp[e]);
            fp[e] = (i == 1 && !exact) ? elam_prev[e] : __expf(fp[e]);
          }
        } else {
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            if (kForm == GDR_FORM_GDN2) at[e] = a0[e];
            fp[e] = 0.f;
          }
        }
        unpack8(*reinterpret_cast<const uint4 *>(smem + SL::A1 + kTile + o), q8);
        unpack8(*reinterpret_cast<const uint4 *>(smem + SL::B1 + kTile + o), k8);
        if (kForm == GDR_FORM_GLA) {
#pragma unroll
          for (int e = 0; e < 8; ++e) u8[e] = z8[e] = 0.f;
        } else {
          unpack8(*reinterpret_cast<const uint4 *>(smem + SL::A1 + o), u8);
        }
        if (kForm == GDR_FORM_RWKV7) {
          const float ct = sC[t];
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            z8[e] = u8[e];        // z = a
            u8[e] *= ct;          // u = c a
          }
        } else if (kForm == GDR_FORM_GENERAL) {
          unpack8(*reinterpret_cast<const uint4 *>(smem + SL::B1 + o), z8);
        } else if (kForm == GDR_FORM_GDN2) {
          // u = alpha_t b k with alpha_t = e^{Lam_t - Lam_{t-1}} (alpha_0 = e^{Lam_0}), z = k;
          // the written value wg (.) v replaces v in place
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            u8[e] = at[e] * u8[e] * k8[e];
            z8[e] = k8[e];
          }
          if (has_wg) {
            float w8[8], v8[8];
            unpack8(*reinterpret_cast<const uint4 *>(smem + SL::B1 + o), w8);
            unpack8(*reinterpret_cast<const uint4 *>(smem + SL::V + o), v8);
#pragma unroll
            for (int e = 0; e < 8; ++e) v8[e] *= w8[e];
            st_smem16(smem, SL::V + o, pack8(v8));
          }
        }
        // U f' (in place over u) and U_pi
#pragma unroll
        for (int e = 0; e < 8; ++e) x[e] = u8[e] * fp[e];
        st_smem16(smem, SL::A1 + o, pack8(x));
#pragma unroll
        for (int e = 0; e < 8; ++e) x[e] = (t > 0) ? x[e] * a0[e] : u8[e];
        st_smem16(smem, SL::UP + o, pack8(x));
        // Q f (in place over q) and Q_pi
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          elam_prev[e] = __expf(lam[e]);
          x[e] = q8[e] * elam_prev[e];
        }
        st_smem16(smem, SL::A1 + kTile + o, pack8(x));
#pragma unroll
        for (int e = 0; e < 8; ++e) x[e] *= a0[e];
        st_smem16(smem, SL::QY + o, pack8(x));
        // K~, Z~ (direct: e^{Lam_63 - Lam_t} <= 1, as e^{dn} e^{-lam} on the pivot path, where
        // both factors lie in [e^-80, e^80]) and Z g, K g (pivot split; zero on the exact path)
        float eml[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) eml[e] = exact ? 0.f : __expf(-lam[e]);
#pragma unroll
        for (int e = 0; e < 8; ++e) fp[e] = exact ? __expf(dn[e] - lam[e]) : edn[e] * eml[e];
#pragma unroll
        for (int e = 0; e < 8; ++e) x[e] = k8[e] * fp[e];
        st_smem16(smem, SL::KT + o, pack8(x));
#pragma unroll
        for (int e = 0; e < 8; ++e) x[e] = z8[e] * fp[e];
        st_smem16(smem, SL::ZT + o, pack8(x));
#pragma unroll
        for (int e = 0; e < 8; ++e) fp[e] = eml[e];
#pragma unroll
        for (int e = 0; e < 8; ++e) x[e] = z8[e] * fp[e];
        st_smem16(smem, SL::B1 + o, pack8(x));
#pragma unroll
        for (int e = 0; e < 8; ++e) x[e] = k8[e] * fp[e];
        st_smem16(smem, SL::B1 + kTile + o, pack8(x));
      }
    }
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
    GT_MARK(3);

    // ---- MMA1: [U f'; Q f] (M = 128) x [Z g; K g]^T (N = 128), K = d_k
    if (warp == 0) {
      tc_fence_after();
      constexpr uint32_t id = idesc_bf16_f32(128, 128, false, false);
#pragma unroll
      for (int s = 0; s < kD / 16; ++s) {
        const uint64_t ad = sdesc_sw128(sb + SL::A1 + s * 32, 16, 1024);
        const uint64_t bd = sdesc_sw128(sb + SL::B1 + s * 32, 16, 1024);
        mma_bf16_warp(tmem + kT_D1, ad, bd, id, s > 0);
      }
      mma_commit_warp(mbar);
      if (lane == 0) ++issued_mma;
    }
    if (!(ok = wait_mma(mbar, phase, sabort))) break;
    GT_MARK(4);

    // ---- A (fp32, strictly lower -> over the MMA1 B operand), B (bf16, below Q_pi),
    //      M_k, M_z (bf16, over log w).  Row r = 32 qd + lane: r < 64 the U rows
    //      (t = r), else the Q rows (t = r - 64); hf = 0: the Z columns, 1: the K columns.
    if (!exact) {
      const int r = 32 * qd + lane, t = r & 63;
      float x[32], y[32];
      tmem_ld_32x32b_x32(tmem + kT_D1 + lane_q + 64 * hf, x);
      tmem_ld_32x32b_x32(tmem + kT_D1 + lane_q + 64 * hf + 32, y);
      tmem_ld_wait();
      GT_MARK(14);
      const bool urow = r < kC;
      // columns below lim are kept (strictly lower for A and B, lower with the diagonal for
      // M_z and M_k); one compare per element against a per-lane limit (a nested
      // condition per element here was measured at several times the cost)
      const int lim = urow ? t : t + 1;
#pragma unroll
      for (int i = 0; i < 32; ++i) {
        x[i] = i < lim ? x[i] : 0.f;
        y[i] = 32 + i < lim ? y[i] : 0.f;
      }
      if (urow && hf == 0) {
#pragma unroll
        for (int i = 0; i < 32; i += 4) {
          *reinterpret_cast<float4 *>(sA + Ix::at(t, i)) = make_float4(x[i], x[i + 1], x[i + 2], x[i + 3]);
          *reinterpret_cast<float4 *>(sA + Ix::at(t, 32 + i)) = make_float4(y[i], y[i + 1], y[i + 2], y[i + 3]);
        }
      } else {
        const uint32_t dst = urow ? SL::BB : (hf == 0 ? SL::MZ : SL::MK);
#pragma unroll
        for (int i = 0; i < 32; i += 8) {
          st_smem16(smem, dst + sw128_offset(t, i, kC * 128), pack8(x + i));
          st_smem16(smem, dst + sw128_offset(t, 32 + i, kC * 128), pack8(y + i));
        }
      }
    } else {
      // exact pairwise decays (a chunk whose log-decay exceeds the pivot bound): Lam
      // again from global log w into the dead MMA1 A operand, inputs from global
      float *lam = sTi;
      {
        const int ch = tid & (kD - 1), qt = tid >> 6;
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          const int t = 16 * qt + i;
          lam[t * kD + ch] = t < n ? __ldg(p.log_w + (((size_t)b * T + t0 + t) * H + h) * kD + ch) : 0.f;
        }
        __syncthreads();
        float x[16];
        float acc = 0.f;
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          acc += lam[(16 * qt + i) * kD + ch];
          x[i] = acc;
        }
        sQT[qt * kD + ch] = acc;
        __syncthreads();
        float excl = 0.f;
#pragma unroll
        for (int q4 = 0; q4 < 4; ++q4) excl += (q4 < qt) ? sQT[q4 * kD + ch] : 0.f;
#pragma unroll
        for (int i = 0; i < 16; ++i) lam[(16 * qt + i) * kD + ch] = x[i] + excl;   // Lam_t
        __syncthreads();
      }
      auto tok = [&](int t) { return (((size_t)b * T + t0 + t) * H + h) * kD; };
      for (int it = tid; it < kC * kC; it += kGT) {
        const int t = it / kC, s = it % kC;
        float av = 0.f, bv = 0.f, mz = 0.f, mk = 0.f;
        if (s <= t && t < n) {
          const size_t ot = tok(t), os = tok(s);
          const float ct = kRwkv ? sC[t] : 1.f;
          for (int j = 0; j < kD; ++j) {
            const float ls = lam[s * kD + j], lt = lam[t * kD + j];
            const float ks = __bfloat162float(gk[os + j]);
            // the form's erase key z_s and erase vector u_t
            float zs = 0.f, ut = 0.f;
            if (kForm == GDR_FORM_GENERAL) {
              zs = __bfloat162float(ge2[os + j]);
              ut = __bfloat162float(ge1[ot + j]);
            } else if (kForm == GDR_FORM_RWKV7) {
              zs = __bfloat162float(ge1[os + j]);
              ut = __bfloat162float(ge1[ot + j]) * ct;
            } else if (kForm == GDR_FORM_GDN2) {
              zs = ks;
              ut = __expf(__ldg(p.log_w + ot + j)) * __bfloat162float(ge1[ot + j]) *
                   __bfloat162float(gk[ot + j]);
            }
            const float dq = __expf(lt - ls) * __bfloat162float(gq[ot + j]);
            mz += dq * zs;
            mk += dq * ks;
            if (s < t) {
              const float du = __expf(lam[(t - 1) * kD + j] - ls) * ut;
              av += du * zs;
              bv += du * ks;
            }
          }
        }
        sA[Ix::at(t, s)] = (s < t) ? av : 0.f;
        *reinterpret_cast<__nv_bfloat16 *>(smem + SL::BB + sw128_offset(t, s, kC * 128)) =
            __float2bfloat16_rn(s < t ? bv : 0.f);
        *reinterpret_cast<__nv_bfloat16 *>(smem + SL::MZ + sw128_offset(t, s, kC * 128)) =
            __float2bfloat16_rn(mz);
        *reinterpret_cast<__nv_bfloat16 *>(smem + SL::MK + sw128_offset(t, s, kC * 128)) =
            __float2bfloat16_rn(mk);
      }
    }
    GT_MARK(15);
    if (kRwkv && warp == 0 && c + 1 < nch) {
#pragma unroll
      for (int i = 0; i < 2; ++i) {
        const int t = t0 + kC + 2 * lane + i;
        cnext[i] = t < T ? __bfloat162float(ge2[((size_t)b * T + t) * H + h]) : 0.f;
      }
    }
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();

    GT_MARK(5);
    // ---- MMA-BV: B V (M = 64) -> TMEM; state accumulator = K~^T V ([K~ | *], M = 128).
    //      They run while T^-1 is formed.
    if (warp == 0) {
      tc_fence_after();
      constexpr uint32_t idb = idesc_bf16_f32(64, kD, false, true);
      constexpr uint32_t ids = idesc_bf16_f32(128, kD, true, true);
#pragma unroll
      for (int s = 0; s < kC / 16; ++s) {
        const uint64_t ab = sdesc_sw128(sb + SL::BB + s * 32, 16, 1024);
        const uint64_t bvd = sdesc_sw128(sb + SL::V + s * 2048, kTile, 1024);
        const uint64_t ak = sdesc_sw128(sb + SL::KT + s * 2048, kTile, 1024);
        mma_bf16_warp(tmem + kT_BV, ab, bvd, idb, s > 0);
        mma_bf16_warp(tmem + kT_DS, ak, bvd, ids, s > 0);
      }
      mma_commit_warp(mbar);
      if (lane == 0) ++issued_mma;
    }
    // ---- T^-1 (fp32 over the dead MMA1 A operand), bf16 copy over the dead fp32 A
    invert_diag_blocks8<Ix, Ix, kGT>(sA, sTi, tid);
    invert_merge_levels<Ix, Ix, kGT>(sA, sTi, tid);
#pragma unroll
    for (int u = 0; u < 2; ++u) {
      const int it = tid + u * kGT, t = it >> 3, gg = it & 7;
      const float4 y0 = *reinterpret_cast<const float4 *>(sTi + Ix::at(t, 8 * gg));
      const float4 y1 = *reinterpret_cast<const float4 *>(sTi + Ix::at(t, 8 * gg + 4));
      float x[8] = {y0.x, y0.y, y0.z, y0.w, y1.x, y1.y, y1.z, y1.w};
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        const int s = 8 * gg + e;
        x[e] = (s < t) ? x[e] : (s == t ? 1.f : 0.f);
      }
      st_smem16(smem, SL::TI + sw128_offset(t, 8 * gg, kC * 128), pack8(x));
    }
    if (!(ok = wait_mma(mbar, phase, sabort))) break;    // B V and K~^T V
    GT_MARK(6);

    // ---- B V (M = 64 accumulator: row 16 qd + r at lane 32 qd + r) -> bf16 tile
    if (hf == 0) {
      float x[32];
      tmem_ld_16x32bx2_x32_split32(tmem + kT_BV + lane_q, x);
      tmem_ld_wait();
      const int t = 16 * qd + (lane & 15), col = 32 * (lane >> 4);
#pragma unroll
      for (int i = 0; i < 32; i += 8) st_smem16(smem, SL::BV + sw128_offset(t, col + i, kC * 128), pack8(x + i));
    }
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();

    GT_MARK(7);
    // ---- MMA2: [Y_u | W] = T^-1 [U_pi | B V] (M = 64, N = 128), K = C
    if (warp == 0) {
      tc_fence_after();
      constexpr uint32_t id = idesc_bf16_f32(64, 128, false, true);
#pragma unroll
      for (int s = 0; s < kC / 16; ++s) {
        const uint64_t ad = sdesc_sw128(sb + SL::TI + s * 32, 16, 1024);
        const uint64_t bd = sdesc_sw128(sb + SL::UP + s * 2048, SL::BV - SL::UP, 1024);
        mma_bf16_warp(tmem + kT_M2, ad, bd, id, s > 0);
      }
      mma_commit_warp(mbar);
      if (lane == 0) ++issued_mma;
    }
    if (!(ok = wait_mma(mbar, phase, sabort))) break;
    GT_MARK(8);

    // ---- Y_u -> rows 64..127 of [Q_pi; Y_u]; -W -> its tile.  hf 0: Y_u columns, 1: W columns
    {
      float x[32];
      tmem_ld_16x32bx2_x32_split32(tmem + kT_M2 + lane_q + 64 * hf, x);
      tmem_ld_wait();
      const int t = 16 * qd + (lane & 15), col = 32 * (lane >> 4);
      if (hf == 0) {
#pragma unroll
        for (int i = 0; i < 32; i += 8)
          st_smem16(smem, SL::QY + kTile + sw128_offset(t, col + i, kC * 128), pack8(x + i));
      } else {
#pragma unroll
        for (int i = 0; i < 32; ++i) x[i] = -x[i];
#pragma unroll
        for (int i = 0; i < 32; i += 8)
          st_smem16(smem, SL::UW + sw128_offset(t, col + i, kC * 128), pack8(x + i));
      }
    }
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();

    GT_MARK(9);
    // ---- MMA3: [Q_pi; Y_u] S0' (M = 128), K = d_k; output extra = [M_k; *] V (M = 128), K = C
    if (warp == 0) {
      tc_fence_after();
      constexpr uint32_t id = idesc_bf16_f32(128, kD, false, true);
#pragma unroll
      for (int s = 0; s < kD / 16; ++s) {
        const uint64_t ad = sdesc_sw128(sb + SL::QY + s * 32, 16, 1024);
        const uint64_t bd = sdesc_sw128(sb + SL::S0B + s * 2048, kTile, 1024);
        mma_bf16_warp(tmem + kT_D3, ad, bd, id, s > 0);
      }
#pragma unroll
      for (int s = 0; s < kC / 16; ++s) {
        const uint64_t ad = sdesc_sw128(sb + SL::MK + s * 32, 16, 1024);
        const uint64_t bd = sdesc_sw128(sb + SL::V + s * 2048, kTile, 1024);
        mma_bf16_warp(tmem + kT_DO, ad, bd, id, s > 0);
      }
      mma_commit_warp(mbar);
      if (lane == 0) ++issued_mma;
    }
    if (!(ok = wait_mma(mbar, phase, sabort))) break;
    GT_MARK(10);
    // ---- v is consumed: load the next chunk's
    if (tid == 0 && c + 1 < nch) {
      fence_proxy_async_smem();
      load_in2(smem, maps, in2, b, h, t0 + kC);
      ++in2_iss;
    }

    // ---- V~ = -W - Y_u S0 -> bf16 (rows = tokens), on the warps owning lanes 64..127
    if (qd >= 2) {
      const int t = 32 * (qd - 2) + lane;
      float d[32];
      tmem_ld_32x32b_x32(tmem + kT_D3 + lane_q + 32 * hf, d);
      tmem_ld_wait();
#pragma unroll
      for (int i = 0; i < 32; i += 8) {
        float w8[8];
        unpack8(*reinterpret_cast<const uint4 *>(smem + SL::UW + sw128_offset(t, 32 * hf + i, kC * 128)), w8);
#pragma unroll
        for (int e = 0; e < 8; ++e) w8[e] = (t < n) ? w8[e] - d[i + e] : 0.f;
        st_smem16(smem, SL::VT + sw128_offset(t, 32 * hf + i, kC * 128), pack8(w8));
      }
    }
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();

    GT_MARK(11);
    // ---- MMA4: state acc += [Z~ | *]^T V~ (M = 128); output extra += [M_z; *] V~ (M = 128)
    if (warp == 0) {
      tc_fence_after();
      constexpr uint32_t ids = idesc_bf16_f32(128, kD, true, true);
      constexpr uint32_t ido = idesc_bf16_f32(128, kD, false, true);
#pragma unroll
      for (int s = 0; s < kC / 16; ++s) {
        const uint64_t az = sdesc_sw128(sb + SL::ZT + s * 2048, kTile, 1024);
        const uint64_t bv = sdesc_sw128(sb + SL::VT + s * 2048, kTile, 1024);
        const uint64_t am = sdesc_sw128(sb + SL::MZ + s * 32, 16, 1024);
        mma_bf16_warp(tmem + kT_DS, az, bv, ids, 1);
        mma_bf16_warp(tmem + kT_DO, am, bv, ido, 1);
      }
      mma_commit_warp(mbar);
      if (lane == 0) ++issued_mma;
    }
    if (!(ok = wait_mma(mbar, phase, sabort))) break;
    GT_MARK(12);
    // ---- u, q, z, k, log w are consumed (and their slots' later tenants): load the next chunk's
    if (tid == 0 && c + 1 < nch) {
      fence_proxy_async_smem();
      load_in1<kForm>(smem, maps, in1, b, h, t0 + kC, has_wg);
      ++in1_iss;
    }

    // ---- state update and output (warps owning lanes 0..63: key rows / token rows)
    if (owner) {
      float d[32];
      tmem_ld_32x32b_x32(tmem + kT_DS + lane_q + 32 * hf, d);
      tmem_ld_wait();
      const float pn = sPI[jrow];
#pragma unroll
      for (int i = 0; i < 32; ++i) {
        st[i] = pn * st[i] + d[i];
        d[i] = st[i];
      }
#pragma unroll
      for (int i = 0; i < 32; i += 8)
        st_smem16(smem, SL::S0B + sw128_offset(jrow, 32 * hf + i, kC * 128), pack8(d + i));
      float o1[32];
      tmem_ld_32x32b_x32(tmem + kT_D3 + lane_q + 32 * hf, o1);
      tmem_ld_32x32b_x32(tmem + kT_DO + lane_q + 32 * hf, d);
      tmem_ld_wait();
      // o staged over [Q_pi; Y_u] (read by MMA3, rewritten only by the next chunk's
      // operand tiles) as four boxes of 32 tokens x 32 columns, 128-byte swizzled, for
      // thread 0's TMA stores after the barrier below; rows past T are clipped by the copy
      uint8_t *box = smem + SL::QY + ((2 * qd + hf) << 12);
#pragma unroll
      for (int i = 0; i < 32; i += 4)
        *reinterpret_cast<float4 *>(box + lane * 128 + (((i >> 2) ^ (lane & 7)) << 4)) =
            make_float4(o1[i] + d[i], o1[i + 1] + d[i + 1], o1[i + 2] + d[i + 2], o1[i + 3] + d[i + 3]);
    }
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
    if (tid == 0) {   // this chunk's o: four TMA stores from the staging
#pragma unroll
      for (int bx = 0; bx < 4; ++bx) {
        const int tok = t0 + 32 * (bx >> 1);
        if (tok < T) tma_store_4d(&maps.o, smem + SL::QY + (bx << 12), 32 * (bx & 1), h, tok, b);
      }
      bulk_commit();
    }
    GT_MARK(13);
  }
  GT_FINI
  if (tid == 0) bulk_wait<0>();   // o's stores complete before the CTA exits

  if (ok && owner && p.S_T) {
#pragma unroll
    for (int i = 0; i < 32; i += 4)
      *reinterpret_cast<float4 *>(p.S_T + s_off + i) = make_float4(st[i], st[i + 1], st[i + 2], st[i + 3]);
  }
  __syncthreads();
  if (!ok && tid == 0) {
    if (p.status) atomicExch(p.status, (uint32_t)GDR_ERR_TIMEOUT);
    // an MMA group or input loads may still be in flight: let them land (bounded)
    if (issued_mma > 0) mbar_wait_bounded(mbar, (issued_mma - 1) & 1, kWaitLimitNs);
    if (in1_iss > in1_done) mbar_wait_bounded(in1, in1_done & 1, kWaitLimitNs);
    if (in2_iss > in2_done) mbar_wait_bounded(in2, in2_done & 1, kWaitLimitNs);
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

PFN_cuTensorMapEncodeTiled_v12000 gen_map_encoder() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void *ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
  });
  return fn;
}

// [B][T][H][64] tensor as a 4-D map (channel, head, token, batch), one 64 x 64 box per
// chunk of one head: bf16 with the 128-byte swizzle (the MMA tile layout), fp32 row-major.
bool encode_gen_map(CUtensorMap *m, const void *base, bool bf16, const FwdParams &p) {
  PFN_cuTensorMapEncodeTiled_v12000 enc = gen_map_encoder();
  if (!enc) return false;
  const int elem = bf16 ? 2 : 4;
  const cuuint64_t dims[4] = {(cuuint64_t)kD, (cuuint64_t)p.H, (cuuint64_t)p.T, (cuuint64_t)p.B};
  const cuuint64_t strides[3] = {(cuuint64_t)kD * elem, (cuuint64_t)p.H * kD * elem,
                                 (cuuint64_t)p.T * p.H * kD * elem};
  const cuuint32_t box[4] = {(cuuint32_t)kD, 1, (cuuint32_t)kC, 1};
  const cuuint32_t estr[4] = {1, 1, 1, 1};
  return enc(m, bf16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4,
             const_cast<void *>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
             bf16 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_NONE,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// The output o [B][T][H][64] fp32 as a 4-D map for the TMA stores: boxes of 32 columns x 32
// tokens (128 bytes per row) with the 128-byte swizzle.
bool encode_out_map(CUtensorMap *m, void *base, const FwdParams &p) {
  PFN_cuTensorMapEncodeTiled_v12000 enc = gen_map_encoder();
  if (!enc) return false;
  const cuuint64_t dims[4] = {(cuuint64_t)kD, (cuuint64_t)p.H, (cuuint64_t)p.T, (cuuint64_t)p.B};
  const cuuint64_t strides[3] = {(cuuint64_t)kD * 4, (cuuint64_t)p.H * kD * 4,
                                 (cuuint64_t)p.T * p.H * kD * 4};
  const cuuint32_t box[4] = {32, 1, 32, 1};
  const cuuint32_t estr[4] = {1, 1, 1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, base, dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

bool forward_tc_general_supported(const FwdParams &p, gdr_dtype dtype) {
  return dtype == GDR_BF16 && p.dk == kD && p.dv == kD && (p.chunk == kC || p.chunk == 2 * kC);
}

cudaError_t launch_forward_tc_general(const FwdParams &p, cudaStream_t stream) {
  GenMaps maps;
  memset(&maps, 0, sizeof(maps));
  // e1: u, a or b (not GLA); e2: z (general) or the optional write gate (GDN-2)
  const bool e1 = p.form != GDR_FORM_GLA;
  const bool e2 = p.form == GDR_FORM_GENERAL || (p.form == GDR_FORM_GDN2 && p.e2);
  if (!encode_gen_map(&maps.q, p.q, true, p) || !encode_gen_map(&maps.k, p.k, true, p) ||
      !encode_gen_map(&maps.v, p.v, true, p) || (e1 && !encode_gen_map(&maps.e1, p.e1, true, p)) ||
      (e2 && !encode_gen_map(&maps.e2, p.e2, true, p)) ||
      !encode_gen_map(&maps.lw, p.log_w, false, p) || !encode_out_map(&maps.o, p.o, p))
    return cudaErrorInvalidValue;
  void (*kern)(FwdParams, const GenMaps) = nullptr;
  switch (p.form) {
    case GDR_FORM_GENERAL: kern = tc_general_kernel<GDR_FORM_GENERAL>; break;
    case GDR_FORM_RWKV7: kern = tc_general_kernel<GDR_FORM_RWKV7>; break;
    case GDR_FORM_GDN2: kern = tc_general_kernel<GDR_FORM_GDN2>; break;
    default: kern = tc_general_kernel<GDR_FORM_GLA>; break;
  }
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)GenSmem::ALLOC);
  if (e != cudaSuccess) return e;
  dim3 grid(p.H, p.B);
  kern<<<grid, kGT, GenSmem::ALLOC, stream>>>(p, maps);
  return cudaGetLastError();
}

}  // namespace gdr

#ifdef GDR_PHASE_TIMING
// Timing build only: copies the two-stream kernel's per-phase cycle sums ([16], thread 0 of
// every CTA, every chunk) to host memory, then clears them.  Returns 0 or a CUDA error.
extern "C" int gdr_general_timing_read(unsigned long long *cycles) {
  cudaError_t e = cudaDeviceSynchronize();
  if (e == cudaSuccess) e = cudaMemcpyFromSymbol(cycles, gdr::g_general_cycles, sizeof(gdr::g_general_cycles));
  static const unsigned long long z[16] = {};
  if (e == cudaSuccess) e = cudaMemcpyToSymbol(gdr::g_general_cycles, z, sizeof(z));
  return (int)e;
}
#endif
