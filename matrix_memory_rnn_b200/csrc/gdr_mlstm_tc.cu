// gdr_mlstm_tc.cu -- xLSTM's mLSTM cell on the fifth-generation tensor cores (bf16 inputs,
// d_k = 64 or 128, d_v a multiple of 64): "Exponential gates and matrix memory: xLSTM and
// RWKV-7", section 13.4 and the solution to Exercise 13.6.
//
// The stabilized cell, chunk by chunk (64 tokens), with A_t the cumulative log forget gate
// inside the chunk and (C, n, m) carried: the chunk-local stabilizer
//     mloc_t = A_t + max_{s <= t} (i~_s - A_s)
// makes every intra-chunk weight w~_ts = e^{A_t - A_s + i~_s - mloc_t} <= 1 independent of
// the carried m, and the carried m enters only through per-token scalars:
//     m_t = max(A_t + m, mloc_t),   r_t = e^{mloc_t - m_t},   g_t = e^{A_t + m - m_t}
//     h_t = (r_t [P~ V]_t + g_t [Q C]_t) / max(|r_t [P~ 1]_t + g_t n . q_t|, e^{-m_t})
//     C <- g_L C + r_L K~^T V,   n <- g_L n + r_L K~^T 1,   m <- m_L
// with P~ = (Q K^T) (.) w~ (s <= t) and K~_s = k_s e^{A_L - A_s + i~_s - mloc_L}.  (The same
// numbers as the cell's unrolled form; every exponent is <= 0.)  So the only sequential
// dependence between chunks is the elementwise update of C, n and m; the four products of a
// chunk run on tcgen05 with fp32 accumulators in TMEM:
//     S = [Q; K] K^T (rows 0..63 used)          [Q C | Q n] = [Q; K] [C | n]
//     [P~ V | P~ 1] = [P~; 0] [V | 1]           [K~^T V | K~^T 1] = K~^T [V | 1]
// The extra column (an all-ones column after V, and n after C, N = 64 + 16) gives the row
// sums and n . q in the same products.  The state is an MMA operand as the bf16 pair
// (bf16(C), bf16(C - bf16(C))), and likewise n: [Q C | Q n] is one product of Q with
// [C_hi | C_lo | n_hi n_lo] (N = 144), whose column pairs the readout adds.  With bf16 alone,
// tokens whose q_t . n_t nearly cancels (after a dominant input gate) lose their relative
// accuracy in the quotient h_t.
//
// One CTA of 256 threads per (b, h, 64 value columns), two warp groups working side by side
// on a chunk:
//   P~ / h warps (0, 1, 4, 5: TMEM lanes 0..63, i.e. the chunk's tokens): the weights w~
//     while the tensor cores form S, then P~, [P~ V | P~ 1] (issued by warp 1), h (staged in
//     shared memory, written by TMA stores), and the state update of key channels 0..63;
//   K~ warps (2, 3, 6, 7): S and [Q C | Q n] (issued by warp 3 at the chunk's start), the
//     next chunk's tile loads (warp 6), diag(f) [V | 1] and K^T diag(f) [V | 1] =
//     [K~^T V | K~^T 1] (issued by warp 2), the next chunk's gates and their scan (warp 7:
//     A, mloc and i~ - A, which do not depend on the carried m), and the state update of key
//     channels 64..127 (with d_k = 64 these rows are padding).
// Every thread carries m and forms its own r_t, g_t, g_L, r_L from the scanned arrays.  The
// next chunk's q, k and value slice arrive by TMA (128-byte swizzle, straight into the MMA
// tiles) and its gates by 4-byte cp.async while the current chunk is computed.  Every wait is
// bounded (2 s); one that runs out ends the CTA and writes GDR_ERR_TIMEOUT to the caller's
// status word.
#include <math.h>
#include <stdlib.h>
#include <string.h>

#include "gdr_tc_common.cuh"
#include "gdr_tma_host.cuh"

// Phase marks of the timing build: thread 0 (a P~ / h warp) and thread 224 (the K~ warp that
// scans the gates) sum
// the cycles between consecutive marks, over CTAs and chunks, into [2][16]; empty in
// libgdr.so.
#ifdef GDR_PHASE_TIMING
namespace gdr {
__device__ unsigned long long g_mlstm_cycles[2][16];
}
#define MT_INIT                                                                     \
  long long mt_a_[16] = {0};                                                        \
  long long mt_l_ = 0;
#define MT_MARK(i)                                                                  \
  do {                                                                              \
    if (threadIdx.x == 0 || threadIdx.x == 224) {                                   \
      const long long n_ = clock64();                                               \
      if (mt_l_) mt_a_[i] += n_ - mt_l_;                                            \
      mt_l_ = n_;                                                                   \
    }                                                                               \
  } while (0)
#define MT_FINI                                                                     \
  if (threadIdx.x == 0 || threadIdx.x == 224)                                       \
    for (int i_ = 0; i_ < 16; ++i_)                                                 \
      atomicAdd(&gdr::g_mlstm_cycles[threadIdx.x == 224][i_], (unsigned long long)mt_a_[i_]);
#else
#define MT_INIT
#define MT_MARK(i)
#define MT_FINI
#endif

namespace gdr {
namespace {

using namespace tc;

constexpr int kMNV = 64;          // value columns per CTA
constexpr int kMThreads = 256;

// Shared memory (bytes) for D key channels.  Per buffer (two, by chunk parity): the [Q; K]
// tile (128 rows: q's 64 tokens then k's, D channels, sw128 in 64-channel blocks of 16 KB), the value
// slice V (64 tokens x 64 columns, sw128) followed by the constant "ones" block (column 0
// = 1, the rest 0) so that [V | 1] is one MN-major operand of 128 columns, and the raw
// gates.  Then P~ (64 x 64, K-major A operand, with 8 KB of padding as the unused rows
// 64..127), diag(f) [V | 1] (64 tokens x (64 + 64), the B operand of K^T diag(f) [V | 1]; column 0
// of its second block holds f, the rest of that block stays 0), the state operand (bf16, D
// key channels x (64 + 64 + 64): bf16(C), then C - bf16(C) rounded to bf16, then a block whose
// columns 0 and 1 hold n's bf16 value and its remainder), the h staging
// (per chunk parity, four warps' 32 tokens x 32 fp32 columns, 128-byte swizzled for the TMA
// stores), the scan's per-token arrays (two chunks) and the barriers.
template <int D>   // key channels: 64 or 128
struct MSmemT {
  static_assert(D == 64 || D == 128, "d_k in {64, 128}");
  static constexpr int NB = D / 64;                           // 64-channel blocks of [Q; K]
  static constexpr uint32_t QK = 0;
  static constexpr uint32_t V = QK + NB * 128 * 128;          // NB x 16 KB
  static constexpr uint32_t ONES = V + 64 * 128;              // 8 KB after V
  static constexpr uint32_t GATES = ONES + 64 * 128;          // f~[64], i~[64] fp32
  static constexpr uint32_t BUF = GATES + 1024;
  static constexpr uint32_t PT = 2 * BUF;                     // P~ (8 KB) + 8 KB padding
  static constexpr uint32_t VS = PT + 16384;                  // diag(f) [V | 1]: two blocks of 8 KB
  static constexpr uint32_t CB = VS + 16384;                  // [C_hi | C_lo | n]: three blocks
  static constexpr uint32_t CBLK = D * 128;                   // bytes per block (D rows)
  static constexpr uint32_t HST = CB + 3 * CBLK;              // h staging: [2][4 warps] 4 KB
  static constexpr uint32_t ARR = HST + 32768;                // fp32 A, mloc, D [64], two chunks
  static constexpr uint32_t MISC = ARR + 6 * 256;
  static constexpr uint32_t ALLOC = MISC + 128 + 1024;
  static_assert(BUF % 1024 == 0 && PT % 1024 == 0 && VS % 1024 == 0 && CB % 1024 == 0 &&
                    HST % 1024 == 0,
                "MMA tiles and swizzled TMA boxes 1024-aligned");
  static_assert(ALLOC <= 227 * 1024, "shared memory");
};
struct MMisc {
  static constexpr uint32_t BAR1 = 0, BAR2 = 8, BAR3 = 16, BAR4 = 24, FULL = 32, SLOT = 48;  // FULL [2]
};

// Tensor maps of q, k, v (loads: boxes of 64 channels x 64 tokens) and of h (stores: boxes
// of 32 fp32 columns x 32 tokens), all with the 128-byte swizzle.
struct MMaps {
  CUtensorMap q, k, v, h;
};
// TMEM columns: S 64, [Q C_hi | Q C_lo | Q n_hi, Q n_lo] 144, [P~ V | P~ 1] 80,
// [K~^T V | K~^T 1] 80.
constexpr uint32_t kColS = 0, kColQC = 64, kColH = 208, kColDS = 288, kMTmemCols = 512;

// 2^x by the PTX instruction ex2.approx.ftz.f32 (an approximation; 2^-inf = 0).  The
// weights it forms are rounded to bf16 next.
__device__ __forceinline__ float ex2_approx(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ float log_sigmoid_f(float x) {
  return x >= 0.f ? -log1pf(expf(-x)) : x - log1pf(expf(x));
}

// Thread 192: the TMA copies of chunk t0's q and k (the D/64 64-channel blocks of each, into
// rows 0..63 and 64..127 of the [Q; K] tile) and of the value slice, completing on `full`;
// tokens past T arrive as zeros.
template <int D>
__device__ __forceinline__ void load_tiles(uint8_t *buf, const MMaps &m, uint64_t *full, int b, int h,
                                           int c0, int t0) {
  using SM = MSmemT<D>;
  mbar_arrive_expect_tx(full, SM::NB * 128 * 128 + 64 * 128);
#pragma unroll
  for (int blk = 0; blk < SM::NB; ++blk) {
    tma_load_4d(buf + SM::QK + blk * 16384, &m.q, 64 * blk, h, t0, b, full);
    tma_load_4d(buf + SM::QK + blk * 16384 + 8192, &m.k, 64 * blk, h, t0, b, full);
  }
  tma_load_4d(buf + SM::V, &m.v, c0, h, t0, b, full);
}

// Warp 0: the chunk's 128 gate values (f~ then i~, 4 bytes each; [B][T][H], so consecutive
// tokens are H apart) by cp.async, one group; tokens past T as zeros.
template <int D>
__device__ __forceinline__ void load_gates(uint8_t *buf, const gdr_mlstm_args &a, int b, int h, int t0) {
  using SM = MSmemT<D>;
  const int T = a.T, H = a.H, lane = threadIdx.x & 31;
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const int g = j >> 1, t = lane + 32 * (j & 1);
    const bool in = t0 + t < T;
    const float *src = (g == 0 ? a.f_pre : a.i_pre) + ((size_t)b * T + (in ? t0 + t : 0)) * H + h;
    const uint32_t dst = smem_u32(buf + SM::GATES + (g * 64 + t) * 4);
    asm volatile("cp.async.ca.shared.global [%0], [%1], 4, %2;" ::"r"(dst), "l"(src), "r"(in ? 4 : 0)
                 : "memory");
  }
  cp_async_commit();
}

// One warp: the part of a chunk's scan that does not depend on the carried m, for a chunk
// with n valid tokens, into the per-token arrays `arr` (A[64], mloc[64], D[64]):
//     A_t = sum_{s <= t} log f_s,   D_s = i~_s - A_s,   mloc_t = A_t + max_{s <= t} D_s
// Padding tokens add log f = 0 and D = -inf, so they change neither A nor mloc.
__device__ __forceinline__ void scan_gates(const float *gf, int n, float *arr) {
  const int lane = threadIdx.x & 31;
  float lf[2], pm[2], ib[2];
#pragma unroll
  for (int e = 0; e < 2; ++e) {
    const int t = lane + 32 * e;
    lf[e] = t < n ? log_sigmoid_f(gf[t]) : 0.f;
    ib[e] = t < n ? gf[64 + t] : -INFINITY;
  }
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
#pragma unroll
    for (int e = 0; e < 2; ++e) {
      const float x = __shfl_up_sync(0xffffffffu, lf[e], o);
      if (lane >= o) lf[e] += x;
    }
  }
  lf[1] += __shfl_sync(0xffffffffu, lf[0], 31);
#pragma unroll
  for (int e = 0; e < 2; ++e) {
    pm[e] = ib[e] - lf[e];
    arr[128 + lane + 32 * e] = pm[e];
  }
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
#pragma unroll
    for (int e = 0; e < 2; ++e) {
      const float x = __shfl_up_sync(0xffffffffu, pm[e], o);
      if (lane >= o) pm[e] = fmaxf(pm[e], x);
    }
  }
  pm[1] = fmaxf(pm[1], __shfl_sync(0xffffffffu, pm[0], 31));
#pragma unroll
  for (int e = 0; e < 2; ++e) {
    arr[lane + 32 * e] = lf[e];
    arr[64 + lane + 32 * e] = lf[e] + pm[e];
  }
}

// Named barriers of the two warp groups: the P~ / h warps (0, 1, 4, 5: TMEM lanes 0..63)
// and the K~ warps (2, 3, 6, 7).
using PSync = GroupSync<1, 128>;
using KSync = GroupSync<2, 128>;

template <int D>
__global__ void __launch_bounds__(kMThreads, 1)
    mlstm_tc_kernel(gdr_mlstm_args a, const __grid_constant__ MMaps maps, uint32_t debug) {
  using SM = MSmemT<D>;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  uint8_t *smem = smem_raw + (((raw + 1023u) & ~1023u) - raw);
  const uint32_t sb = smem_u32(smem);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int qd = warp & 3, hf = warp >> 2;
  const bool pw = qd < 2;   // a P~ / h warp (TMEM lanes 0..63); else a K~ warp
  const int slice = blockIdx.x, c0 = slice * kMNV, h = blockIdx.y, b = blockIdx.z;
  const int T = a.T, H = a.H, dv = a.dv, nch = (T + 63) / 64;
  const size_t bh = (size_t)b * H + h;

  uint8_t *misc = smem + SM::MISC;
  uint64_t *bar1 = reinterpret_cast<uint64_t *>(misc + MMisc::BAR1);   // S
  uint64_t *bar2 = reinterpret_cast<uint64_t *>(misc + MMisc::BAR2);   // [P~ V | P~ 1]
  uint64_t *bar3 = reinterpret_cast<uint64_t *>(misc + MMisc::BAR3);   // [K~^T V | K~^T 1]
  uint64_t *bar4 = reinterpret_cast<uint64_t *>(misc + MMisc::BAR4);   // [Q C | Q n]
  uint64_t *full = reinterpret_cast<uint64_t *>(misc + MMisc::FULL);
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(misc + MMisc::SLOT);
  float *arr0 = reinterpret_cast<float *>(smem + SM::ARR);   // A, mloc, D of even chunks; odd at +192

  if (warp == 0) {
    tmem_alloc(tmem_slot, kMTmemCols);
    tmem_relinquish();
  }
  if (tid == 192) {   // the thread that arms `full` for the first tile loads below
    mbar_init(bar1, 1);
    mbar_init(bar2, 1);
    mbar_init(bar3, 1);
    mbar_init(bar4, 1);
    mbar_init(full, 1);
    mbar_init(full + 1, 1);
    fence_mbar_init();
  }
  // constants: the ones blocks (column 0 = 1) and the padding rows of P~; [C | n]'s n block
  for (int i = tid; i < 2 * 64 * 8; i += kMThreads) {
    const int bi = i >> 9, r = (i >> 3) & 63, ch = i & 7;
    uint4 x = make_uint4(0u, 0u, 0u, 0u);
    if (ch == (r & 7)) x.x = 0x3F80u;          // bf16 1.0 in the chunk that holds column 0
    *reinterpret_cast<uint4 *>(smem + bi * SM::BUF + SM::ONES + r * 128 + ch * 16) = x;
  }
  for (int i = tid; i < 8192 / 16; i += kMThreads)
    *reinterpret_cast<uint4 *>(smem + SM::PT + 8192 + i * 16) = make_uint4(0u, 0u, 0u, 0u);
  for (int i = tid; i < (int)SM::CBLK / 16; i += kMThreads)   // the n block: columns 2..63 stay 0
    *reinterpret_cast<uint4 *>(smem + SM::CB + 2 * SM::CBLK + i * 16) = make_uint4(0u, 0u, 0u, 0u);
  for (int i = tid; i < 8192 / 16; i += kMThreads)   // diag(f) 1: only column 0 changes per chunk
    *reinterpret_cast<uint4 *>(smem + SM::VS + 8192 + i * 16) = make_uint4(0u, 0u, 0u, 0u);

  // fp32 state: key channel jrow, value columns [hf*32, hf*32 + 32) of the slice; n_j on hf 0.
  // Every thread carries m (mc) itself: the same arithmetic on the same values everywhere.
  // With D = 64 the rows 64..127 (warps of quarters 2 and 3) are padding: [K~^T V | K~^T 1]
  // stays an M = 128 product, one key channel per TMEM lane, whose upper half reads the
  // ones block behind V and is never loaded, stored or used.
  const int jrow = 32 * qd + lane;
  const bool jreal = jrow < D;
  float st[32];
  float nj = 0.f, mc = a.m0 ? a.m0[bh] : -INFINITY;
  {
    const float *C0 = a.C0 && jreal ? a.C0 + bh * D * dv + (size_t)jrow * dv + c0 + hf * 32 : nullptr;
#pragma unroll
    for (int i = 0; i < 32; i += 4) {
      const float4 x = C0 ? __ldg(reinterpret_cast<const float4 *>(C0 + i)) : make_float4(0.f, 0.f, 0.f, 0.f);
      st[i] = x.x; st[i + 1] = x.y; st[i + 2] = x.z; st[i + 3] = x.w;
    }
    if (hf == 0 && a.n0 && jreal) nj = a.n0[bh * D + jrow];
  }
  // The MMA operand of the state, row jrow, this thread's 32 columns: bf16(C) (columns 0..63),
  // C - bf16(C) in bf16 (64..127), and n's pair in columns 128 and 129.  The pair carries about
  // 16 significant bits, so that Q C and Q n keep their relative accuracy where q_t . n is
  // small against |q_t| |n| (one dominant input gate); bf16 alone loses it there.
  auto store_state_bf16 = [&]() {
    if (!jreal) return;
#pragma unroll
    for (int i = 0; i < 32; i += 8) {
      const uint4 hi = pack8(st + i);
      float hv[8], lo[8];
      unpack8(hi, hv);
#pragma unroll
      for (int e = 0; e < 8; ++e) lo[e] = st[i + e] - hv[e];
      st_smem16(smem, SM::CB + sw128_offset(jrow, hf * 32 + i, SM::CBLK), hi);
      st_smem16(smem, SM::CB + sw128_offset(jrow, 64 + hf * 32 + i, SM::CBLK), pack8(lo));
    }
    if (hf == 0) {
      const __nv_bfloat16 nh = __float2bfloat16_rn(nj);
      *reinterpret_cast<__nv_bfloat162 *>(smem + SM::CB + sw128_offset(jrow, 128, SM::CBLK)) =
          __halves2bfloat162(nh, __float2bfloat16_rn(nj - __bfloat162float(nh)));
    }
  };
  store_state_bf16();
  fence_proxy_async_smem();   // the constant blocks and [C | n] are read by the tensor cores

  // Thread 192 (warp 6, a K~ warp) requests the tiles and counts the chunks whose tiles it
  // requested and saw land; warp 7 loads the gates (one cp.async group per chunk) and scans
  // them a chunk ahead.
  int loads_issued = 0, loads_seen = 0;
  if (tid == 192) {
    load_tiles<D>(smem, maps, full, b, h, c0, 0);
    loads_issued = 1;
  }
  if (warp == 7) {
    load_gates<D>(smem, a, b, h, 0);
    cp_async_wait<0>();
    __syncwarp();
    scan_gates(reinterpret_cast<const float *>(smem + SM::GATES), min(64, T), arr0);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = __shfl_sync(0xffffffffu, *tmem_slot, 0);
  const uint32_t lane_q = (uint32_t)(32 * qd) << 16;

  // the state update of this thread's row and columns, C <- g_L C + r_L K~^T V and n
  // likewise, once [K~^T V | K~^T 1] has landed; then m <- m_L
  auto update_state = [&](const float *arr) {
    float d[32], dn[1];
    tmem_ld_32x32b_x32(tmem + kColDS + lane_q + hf * 32, d);
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x1.b32 {%0}, [%1];"
                 : "=r"(*reinterpret_cast<uint32_t *>(dn)) : "r"(tmem + kColDS + lane_q + 64));
    const float aL = arr[63], mlL = arr[64 + 63], mL = fmaxf(aL + mc, mlL);
    const float gL = expf(aL + mc - mL), rL = expf(mlL - mL);
    tmem_ld_wait();
#pragma unroll
    for (int i = 0; i < 32; ++i) st[i] = fmaf(gL, st[i], rL * d[i]);
    if (hf == 0) nj = fmaf(gL, nj, rL * dn[0]);
    store_state_bf16();
    mc = mL;
  };
  auto mma_wait = [&](uint64_t *bar, uint32_t par, bool &fail) {
    if (!mbar_wait_bounded(bar, par, kWaitLimitNs)) fail = true;
  };

  bool fail = false;      // one of this thread's bounded waits ran out
  bool ok = true;         // the same for every thread: no wait ran out
  int committed = 0;      // chunks whose MMA groups were all issued
  MT_INIT

  for (int c = 0; c < nch; ++c) {
    const int t0 = c * 64, n = min(64, T - t0), bi = c & 1;
    uint8_t *buf = smem + bi * SM::BUF;
    const uint32_t bb = sb + bi * SM::BUF;
    const uint32_t par = (uint32_t)(c & 1);   // each MMA barrier completes once per chunk
    const float *arr = arr0 + 192 * bi;       // this chunk's A, mloc, D (scanned a chunk ahead)
    MT_MARK(0);
    // ---- chunk c's tiles have landed (thread 192 polls, bounded); its gates are scanned
    if (tid == 192) {
      if (mbar_wait_bounded(full + bi, (uint32_t)((c >> 1) & 1), kWaitLimitNs)) ++loads_seen;
      else fail = true;
    }
    if (__syncthreads_or(fail)) {
      ok = false;
      break;
    }
    MT_MARK(1);
    // ---- MMA group 1 (warp 3): S = [Q; K] K^T, then [Q; K] [C_hi | C_lo | n_hi n_lo]
    if (warp == 3) {
      tc_fence_after();
      constexpr uint32_t id_s = idesc_bf16_f32(128, 64, false, false);
      constexpr uint32_t id_qc = idesc_bf16_f32(128, 144, false, true);
#pragma unroll
      for (int s = 0; s < D / 16; ++s) {
        const uint64_t aq = sdesc_sw128(bb + SM::QK + (s >> 2) * 16384 + (s & 3) * 32, 16, 1024);
        const uint64_t bk = sdesc_sw128(bb + SM::QK + 64 * 128 + (s >> 2) * 16384 + (s & 3) * 32, 16, 1024);
        mma_bf16_warp(tmem + kColS, aq, bk, id_s, s > 0);
      }
      mma_commit_warp(bar1);
#pragma unroll
      for (int s = 0; s < D / 16; ++s) {
        const uint64_t aq = sdesc_sw128(bb + SM::QK + (s >> 2) * 16384 + (s & 3) * 32, 16, 1024);
        const uint64_t bc = sdesc_sw128(sb + SM::CB + s * 2048, SM::CBLK, 1024);
        mma_bf16_warp(tmem + kColQC, aq, bc, id_qc, s > 0);
      }
      mma_commit_warp(bar4);
    }
    // ---- the next chunk's loads, into the other buffer (chunk c - 1 is done with it)
    if (c + 1 < nch) {
      if (tid == 192) {
        load_tiles<D>(smem + (bi ^ 1) * SM::BUF, maps, full + (bi ^ 1), b, h, c0, t0 + 64);
        ++loads_issued;
      }
      if (warp == 7) load_gates<D>(smem + (bi ^ 1) * SM::BUF, a, b, h, t0 + 64);
    }
    if (pw) {
      // ---- P~ = S (.) w~ for row t = 32 qd + lane, columns [32 hf, 32 hf + 32), with
      //      w~_ts = e^{(A_t - mloc_t) + D_s} for s <= t.  The weights are formed while the
      //      tensor cores compute S; the warp reads D_s as 16-byte broadcasts (32 scalar reads
      //      per thread, or 32 shuffles, were measured several times slower).
      //      Warp 4 (tokens 0..31, keys 32..63) lies wholly above the diagonal: zeros.
      const int t = 32 * qd + lane;
      const bool upper = qd == 0 && hf == 1;   // warp-uniform
      float w[32];
      if (upper) {
#pragma unroll
        for (int i = 0; i < 32; ++i) w[i] = 0.f;
      } else {
        constexpr float kLog2e = 1.4426950408889634f;
        const float rowv2 = (arr[t] - arr[64 + t]) * kLog2e;
        const float4 *dcol = reinterpret_cast<const float4 *>(arr + 128 + hf * 32);
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          const float4 d4 = dcol[j];
          const float dd[4] = {d4.x, d4.y, d4.z, d4.w};
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const int i = 4 * j + e;
            w[i] = hf * 32 + i <= t ? ex2_approx(fmaf(dd[e], kLog2e, rowv2)) : 0.f;
          }
        }
      }
      MT_MARK(2);
      mma_wait(bar1, par, fail);
      __syncwarp();   // the warp-wide tcgen05.ld below wants the warp converged
      tc_fence_after();
      MT_MARK(3);
      if (!upper) {
        float x[32];
        tmem_ld_32x32b_x32(tmem + kColS + lane_q + hf * 32, x);
        tmem_ld_wait();
#pragma unroll
        for (int i = 0; i < 32; ++i) w[i] *= x[i];
      }
      MT_MARK(4);
#pragma unroll
      for (int i = 0; i < 32; i += 8)
        st_smem16(smem, SM::PT + sw128_offset(t, hf * 32 + i, 8192), pack8(w + i));
      fence_proxy_async_smem();
      PSync::sync();
      MT_MARK(5);
      // ---- MMA 2a (warp 1): [P~ V | P~ 1] = [P~; 0] [V | 1]
      if (warp == 1) {
        tc_fence_after();
        constexpr uint32_t id_h = idesc_bf16_f32(128, 80, false, true);
#pragma unroll
        for (int s = 0; s < 4; ++s) {
          const uint64_t ap = sdesc_sw128(sb + SM::PT + s * 32, 16, 1024);
          const uint64_t bv = sdesc_sw128(bb + SM::V + s * 2048, 8192, 1024);
          mma_bf16_warp(tmem + kColH, ap, bv, id_h, s > 0);
        }
        if (!(debug & kDebugSkipHandoff)) mma_commit_warp(bar2);   // (withheld in the fault test)
      }
      // ---- h_t = (r_t [P~ V]_t + g_t [Q C]_t) / max(|r_t [P~ 1]_t + g_t [Q n]_t|, e^{-m_t})
      //      with m_t = max(A_t + m, mloc_t), r_t = e^{mloc_t - m_t}, g_t = e^{A_t + m - m_t}
      const float at = arr[t], mlt = arr[64 + t], mt = fmaxf(at + mc, mlt);
      const float r = expf(mlt - mt), g = expf(at + mc - mt), floor_t = expf(-mt);
      MT_MARK(6);
      mma_wait(bar2, par, fail);
      mma_wait(bar4, par, fail);
      __syncwarp();
      tc_fence_after();
      MT_MARK(7);
      {
        float hv[32], qc[32], ql[32], hx[1], qx[2];
        tmem_ld_32x32b_x32(tmem + kColH + lane_q + hf * 32, hv);
        tmem_ld_32x32b_x32(tmem + kColQC + lane_q + hf * 32, qc);
        tmem_ld_32x32b_x32(tmem + kColQC + lane_q + 64 + hf * 32, ql);
        asm volatile("tcgen05.ld.sync.aligned.32x32b.x1.b32 {%0}, [%1];"
                     : "=r"(*reinterpret_cast<uint32_t *>(hx)) : "r"(tmem + kColH + lane_q + 64));
        asm volatile("tcgen05.ld.sync.aligned.32x32b.x2.b32 {%0, %1}, [%2];"
                     : "=r"(*reinterpret_cast<uint32_t *>(qx)), "=r"(*reinterpret_cast<uint32_t *>(qx + 1))
                     : "r"(tmem + kColQC + lane_q + 128));
        tmem_ld_wait();
#pragma unroll
        for (int i = 0; i < 32; ++i) qc[i] += ql[i];
        // staged in this warp's 4 KB box (row = lane, 128-byte swizzle), then one TMA store
        // of 32 tokens x 32 columns; rows past T are clipped by the copy.  The box of chunk
        // c - 2 must have been read out first (lane 0's bulk groups, two in flight at most).
        uint8_t *hst = smem + SM::HST + ((bi * 4 + (warp & 1) + 2 * hf) << 12);
        if (lane == 0) bulk_wait_read<1>();
        __syncwarp();
        const float rd = 1.f / fmaxf(fabsf(fmaf(r, hx[0], g * (qx[0] + qx[1]))), floor_t);
#pragma unroll
        for (int i = 0; i < 32; i += 4)
          *reinterpret_cast<float4 *>(hst + lane * 128 + (((i >> 2) ^ (lane & 7)) << 4)) =
              make_float4(fmaf(r, hv[i], g * qc[i]) * rd, fmaf(r, hv[i + 1], g * qc[i + 1]) * rd,
                          fmaf(r, hv[i + 2], g * qc[i + 2]) * rd, fmaf(r, hv[i + 3], g * qc[i + 3]) * rd);
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0 && t0 + 32 * qd < T) {
          tma_store_4d(&maps.h, hst, c0 + hf * 32, h, t0 + 32 * qd, b);
          bulk_commit();
        }
      }
      MT_MARK(8);
      // ---- the state update of key channels 0..63
      mma_wait(bar3, par, fail);
      __syncwarp();
      tc_fence_after();
      MT_MARK(9);
      update_state(arr);
      MT_MARK(10);
    } else {
      // ---- diag(f) [V | 1] with f_s = e^{A_L - mloc_L + D_s} (token s, 32 value columns), so
      //      that K~^T [V | 1] = K^T (diag(f) [V | 1]) reads K in place from the [Q; K] tile
      const int u = ((warp & 1) << 5) + ((warp >> 2) << 6) + lane;   // 0..127 over warps 2, 3, 6, 7
      const int s = u & 63, ch = u >> 6;
      const float f = __expf(arr[63] - arr[64 + 63] + arr[128 + s]);
#pragma unroll
      for (int i = 0; i < 32; i += 8) {
        float v8[8];
        unpack8(*reinterpret_cast<const uint4 *>(buf + SM::V + sw128_offset(s, ch * 32 + i, 8192)), v8);
#pragma unroll
        for (int e = 0; e < 8; ++e) v8[e] *= f;
        st_smem16(smem, SM::VS + sw128_offset(s, ch * 32 + i, 8192), pack8(v8));
      }
      if (ch == 0)
        *reinterpret_cast<__nv_bfloat16 *>(smem + SM::VS + sw128_offset(s, 64, 8192)) = __float2bfloat16_rn(f);
      fence_proxy_async_smem();
      MT_MARK(2);
      KSync::sync();
      MT_MARK(3);
      // ---- MMA 2b (warp 2): [K~^T V | K~^T 1] = K^T (diag(f) [V | 1]); K^T is the MN-major
      //      view of the k rows of the [Q; K] tile (its two 64-channel blocks 16 KB apart)
      if (warp == 2) {
        tc_fence_after();
        constexpr uint32_t id_ds = idesc_bf16_f32(128, 80, true, true);
#pragma unroll
        for (int s4 = 0; s4 < 4; ++s4) {
          const uint64_t ak = sdesc_sw128(bb + SM::QK + 64 * 128 + s4 * 2048, 16384, 1024);
          const uint64_t bv = sdesc_sw128(sb + SM::VS + s4 * 2048, 8192, 1024);
          mma_bf16_warp(tmem + kColDS, ak, bv, id_ds, s4 > 0);
        }
        mma_commit_warp(bar3);
      }
      MT_MARK(4);
      // ---- the next chunk's carry-free scan (warp 7; its gates were requested at the
      //      chunk's start)
      if (warp == 7 && c + 1 < nch) {
        cp_async_wait<0>();
        __syncwarp();
        scan_gates(reinterpret_cast<const float *>(smem + (bi ^ 1) * SM::BUF + SM::GATES),
                   min(64, T - t0 - 64), arr0 + 192 * (bi ^ 1));
      }
      MT_MARK(5);
      // ---- the state update of key channels 64..127, once [Q C | Q n] has read [C | n]
      mma_wait(bar4, par, fail);
      mma_wait(bar3, par, fail);
      __syncwarp();
      tc_fence_after();
      MT_MARK(6);
      update_state(arr);
      MT_MARK(10);
    }
    committed = c + 1;
    fence_proxy_async_smem();   // [C | n] is read by the next chunk's group 1
    tc_fence_before();
    MT_MARK(11);
    if (__syncthreads_or(fail)) {
      ok = false;
      break;
    }
    MT_MARK(12);
  }
  MT_FINI
  if (pw && lane == 0) bulk_wait<0>();   // h's stores complete before the CTA exits

  // ---- the final state
  if (ok) {
    if (a.C_T && jreal) {
      float *dst = a.C_T + bh * D * dv + (size_t)jrow * dv + c0 + hf * 32;
#pragma unroll
      for (int i = 0; i < 32; i += 4)
        *reinterpret_cast<float4 *>(dst + i) = make_float4(st[i], st[i + 1], st[i + 2], st[i + 3]);
    }
    if (slice == 0) {
      if (a.n_T && hf == 0 && jreal) a.n_T[bh * D + jrow] = nj;
      if (a.m_T && tid == 0) a.m_T[bh] = mc;
    }
  } else if (tid == 192) {   // the issuing thread of the tile loads
    if (a.status) *reinterpret_cast<volatile uint32_t *>(a.status) = (uint32_t)GDR_ERR_TIMEOUT;
    // let what is still in flight land before the CTA exits: the last chunk's MMA groups
    // and the tile loads requested but not seen (each buffer's loads land in order)
    if (committed > 0) {
      const uint32_t p = (uint32_t)((committed - 1) & 1);
      mbar_wait_bounded(bar1, p, kWaitLimitNs);
      mbar_wait_bounded(bar2, p, kWaitLimitNs);
      mbar_wait_bounded(bar3, p, kWaitLimitNs);
      mbar_wait_bounded(bar4, p, kWaitLimitNs);
    }
    for (int j = loads_seen; j < loads_issued; ++j)
      if (!mbar_wait_bounded(full + (j & 1), (uint32_t)((j >> 1) & 1), kWaitLimitNs)) break;
  }
  cp_async_wait<0>();
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, kMTmemCols);
  }
}

}  // namespace

bool mlstm_tc_supported(const gdr_mlstm_args &a) {
  return a.dtype == GDR_BF16 && (a.dk == 64 || a.dk == 128) && a.dv % kMNV == 0;
}

#ifdef GDR_PHASE_TIMING
// Timing build only: copies the mLSTM kernel's per-phase cycle sums ([2][16]: thread 0's,
// then thread 224's) to host memory, then clears them.  Returns 0 or a CUDA error.
extern "C" int gdr_mlstm_timing_read(unsigned long long *cycles) {
  cudaError_t e = cudaDeviceSynchronize();
  if (e == cudaSuccess) e = cudaMemcpyFromSymbol(cycles, g_mlstm_cycles, sizeof(g_mlstm_cycles));
  static const unsigned long long z[32] = {};
  if (e == cudaSuccess) e = cudaMemcpyToSymbol(g_mlstm_cycles, z, sizeof(z));
  return (int)e;
}
#endif

template <int D>
cudaError_t launch_mlstm_tc_d(const gdr_mlstm_args &a, cudaStream_t stream) {
  MMaps maps;
  const CUtensorMapDataType bf = CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
  const CUtensorMapSwizzle sw = CU_TENSOR_MAP_SWIZZLE_128B;
  if (!tma::encode_input_map(&maps.q, a.q, bf, 2, 64, 64, sw, a.H, a.T, a.B, D) ||
      !tma::encode_input_map(&maps.k, a.k, bf, 2, 64, 64, sw, a.H, a.T, a.B, D) ||
      !tma::encode_input_map(&maps.v, a.v, bf, 2, 64, 64, sw, a.H, a.T, a.B, a.dv) ||
      !tma::encode_input_map(&maps.h, a.h, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, 32, 32, sw, a.H,
                             a.T, a.B, a.dv))
    return cudaErrorInvalidValue;
  using SM = MSmemT<D>;
  cudaError_t e = cudaFuncSetAttribute(mlstm_tc_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)SM::ALLOC);
  if (e != cudaSuccess) return e;
  const char *fault = getenv("GDR_DEBUG_FAULT");
  const uint32_t debug = (fault && strcmp(fault, "skip_handoff") == 0) ? kDebugSkipHandoff : 0u;
  mlstm_tc_kernel<D><<<dim3(a.dv / kMNV, a.H, a.B), kMThreads, SM::ALLOC, stream>>>(a, maps, debug);
  return cudaGetLastError();
}

cudaError_t launch_mlstm_tc(const gdr_mlstm_args &a, cudaStream_t stream) {
  if (!mlstm_tc_supported(a)) return cudaErrorInvalidValue;
  return a.dk == 64 ? launch_mlstm_tc_d<64>(a, stream) : launch_mlstm_tc_d<128>(a, stream);
}

}  // namespace gdr
