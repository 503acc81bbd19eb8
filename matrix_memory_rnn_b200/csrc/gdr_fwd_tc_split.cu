// gdr_fwd_tc_split.cu -- chunked forward on the tensor cores as two kernels.
//
// Same algorithm and numerics as gdr_fwd_tc.cu ("Muir: Linear Attention with
// Sensitivity-Allocated Gating and Matched-Filter Readout", section 2.2 and
// section 4.2; GDN-2 form, bf16 inputs, d_k = d_v = 128, C = 64), split where the
// chunkwise form itself splits:
//
//  * prep: everything that does not depend on the chunk's initial state S0 --
//    the cumulative log-decay, the decay-weighted products L and M (one tcgen05
//    MMA), T^-1 (fp32 8 x 8 diagonal blocks and 16 x 16 merge, tf32 warp-MMA
//    merges at 32 and 64), U = T^-1 V^ and
//    Y = T^-1 K^_pi (one tcgen05 MMA group), and the operand tiles Q_pi and K~.
//    Chunks are independent: a persistent grid of one 512-thread CTA per SM walks
//    them as a two-stage pipeline of warp groups (scan, element-wise phase and
//    MMA1 on one chunk while L readout, T^-1 and MMA2 run on the previous one);
//    inputs arrive by TMA, the bf16 ones straight into the MMA tiles.  Each chunk's result is a
//    record of bf16 MMA tiles, already in the 128-byte-swizzled shared-memory
//    layout, in the workspace.
//  * chain: the inter-chunk state carry and the outputs, sequential over chunks
//    for each (b, h, 64-column value slice):
//        V~ = U - Y S0,   S_C = Diag(pi_n) S0 + K~^T V~,   O = Q_pi S0 + M V~.
//    Records are fetched with bulk (TMA) copies three chunks ahead into a ring of
//    three buffers, so every chunk step is two MMA groups and two short CUDA-core
//    phases.
//
// The workspace holds one record (74752 bytes) per (b, h, chunk) after a
// 1024-byte header whose first word is the device status word.
#include <cuda.h>
#include <cudaTypedefs.h>

#include <cstring>
#include <mutex>
#include <type_traits>

#include "gdr_phase_timing.cuh"
#include "gdr_tc_common.cuh"
#include "gdr_tma_host.cuh"

// Phase hooks: filled by gdr_phase_timing.cuh in the timing build, empty in libgdr.so.
#ifndef GDR_PREP_PHASE
#define GDR_PREP_PHASE(i)
#endif
#ifndef GDR_CHAIN_PHASE
#define GDR_CHAIN_PHASE(i)
#endif
#ifndef GDR_PHASE_INIT
#define GDR_PHASE_INIT
#define GDR_PHASE_FINI(slot)
#endif
#ifndef GDR_MMA_DECL
#define GDR_MMA_DECL(slot)
#define GDR_MMA_BEGIN()
#define GDR_MMA_END(g, tbar)
#define GDR_MMA_FINI(slot)
#endif

namespace gdr {
namespace {

using namespace tc;
using Ix = SwizzledIdx;

// One chunk's record: bf16 tiles in the sw128 layout (64-column blocks of C*128 B).
struct Rec {
  static constexpr uint32_t QY = 0;                     // [Q_pi; Y] 2C x DK (K-major A of one
                                                        //   M = 2C MMA with S0): rows 0..C-1
                                                        //   Q_pi, rows C..2C-1 Y
  static constexpr uint32_t KT = QY + 2 * kC * kDK * 2;  // K~      C x DK  (MN-major A of K~^T V~)
  static constexpr uint32_t MM = KT + kC * kDK * 2;     // M       C x C   (K-major A of M V~)
  static constexpr uint32_t U = MM + kC * kC * 2;       // U       C x DV  (rows = tokens)
  static constexpr uint32_t PI = U + kC * kDK * 2;      // exp(Lam_n), DK fp32
  static constexpr uint32_t BYTES = PI + 1024;
  static constexpr uint32_t FRONT = U;                  // QY | KT | MM, copied as one block
  static constexpr uint32_t QY_STRIDE = 2 * kC * 128;   // bytes between QY's 64-column blocks
  static_assert(QY % 1024 == 0 && KT % 1024 == 0 && MM % 1024 == 0 && U % 1024 == 0 &&
                    PI % 1024 == 0 && BYTES % 1024 == 0,
                "record tiles must stay 1024-byte aligned");
};

// Where a chunk that takes the exact path parks Lam_t - Lam_1 (token t, DK fp32):
// the record's Y rows (two 8 KB pieces) and its U tile, all written only at the end.
__device__ __forceinline__ uint32_t park_row(int t) {
  return t < 16   ? Rec::QY + kC * 128 + t * kDK * 4
         : t < 32 ? Rec::QY + Rec::QY_STRIDE + kC * 128 + (t - 16) * kDK * 4
                  : Rec::U + (t - 32) * kDK * 4;
}
constexpr size_t kHeaderBytes = 1024;
// Sequences of at least this many chunks, whose chain CTAs fill at most a third of the
// SMs, run prep and chain in one cooperative launch.
constexpr int kFusedMinChunks = 32;

__host__ __device__ inline int num_chunks(int T) { return (T + kC - 1) / kC; }

// ============================================================== prep kernel
// Persistent: one CTA of 512 threads per SM walks the chunks (b, h, c) with a
// stride of gridDim.x, as a two-stage pipeline of warp groups over two chunk
// buffers:
//   front (warps 8..15): log-decay scan, operand tiles and MMA1 of chunk j;
//   back  (warps 0..7):  L / M readout, T^-1, MMA2 and U / Y readout of chunk j - 1.
// Inputs arrive by TMA: k, b, q, v straight into the chunk buffer's MMA tiles
// (128-byte swizzle, the tcgen05 operand layout), where the element-wise phase
// turns them into K g, K^ f, Q f, V^ in place; wg into one of two staging tiles,
// log w into a staging area that the scan releases as soon as it has read it.
// The back group loads chunk j + 2's tiles as soon as MMA2 of chunk j has
// released its buffer.
constexpr int kPrepThreads = 512;
constexpr int kGroup = 256;                    // threads per warp group
using FrontSync = GroupSync<1, kGroup>;
using BackSync = GroupSync<2, kGroup>;

// fp32 64 x 64 T^-1 in the Q rows of the [K^ f; Q f] tile once MMA1 has read them:
// those rows are two 8 KB pieces (one per 64-column atom), rows 0..31 in the
// first and 32..63 in the second; 16-byte groups XOR-permuted by (r & 15).
struct QRowsIdx {
  static __device__ __forceinline__ int at(int r, int s) {
    return (r < 32 ? kC * 32 : kC * 96) + (r & 31) * kC + ((((s >> 2) ^ (r & 15))) << 2) + (s & 3);
  }
};

struct PrepSmem {
  // chunk buffer (x2): tiles in the sw128 layout, 64-column blocks
  static constexpr uint32_t A_LM = 0;                         // [K^ f; Q f] 2C x DK (b, q land here);
                                                              //   Q rows then hold fp32 T^-1
  static constexpr uint32_t B_LM = A_LM + 2 * kC * kDK * 2;   // K g  C x DK (k lands here); then
                                                              //   fp32 L; then bf16 T^-1 (first 8 KB)
  static constexpr uint32_t VH = B_LM + kC * kDK * 2;         // V^ = wg (.) v (v lands here)
  static constexpr uint32_t BUF = VH + kC * kDK * 2;          // 64 KB per buffer
  static constexpr uint32_t SW = 2 * BUF;                     // write gate x2 (sw128, offsets as v)
  static constexpr uint32_t SLW = SW + 2 * kC * kDK * 2;      // log w, row-major fp32
  static constexpr uint32_t BT = SLW + kC * kDK * 4;          // fp32 [16][DK] block sums -> prefixes
  static constexpr uint32_t TOT = BT + 16 * kDK * 4;          // fp32 Lam_n per channel
  static constexpr uint32_t L1 = TOT + kDK * 4;               // fp32 Lam_1 per channel
  static constexpr uint32_t A1 = L1 + kDK * 4;                // fp32 [4][DK] alpha_1, by chunk & 3
  static constexpr uint32_t NRM = A1 + 4 * kDK * 4;           // fp32 [2][2][C] Muir 1/|q|, 1/|k|
  static constexpr uint32_t MISC = NRM + 4 * kC * 4;
  static constexpr uint32_t ALLOC = MISC + 256 + 1024;
  static_assert(BUF % 1024 == 0 && SW % 1024 == 0, "MMA tiles 1024-aligned");
  static_assert(Ix::kBytes <= kC * kDK * 2, "fp32 L must fit the reused bf16 tile");
  static_assert(ALLOC <= 227 * 1024, "shared memory");
};

struct PrepMisc {             // byte offsets inside PrepSmem::MISC
  static constexpr uint32_t BFULL = 0;      // uint64_t [2] chunk-buffer tiles landed
  static constexpr uint32_t WFULL = 16;     // uint64_t [2] write-gate staging landed
  static constexpr uint32_t LFULL = 32;     // uint64_t     log-w staging landed
  static constexpr uint32_t READY = 40;     // uint64_t [2] front -> back: operand tiles written
  static constexpr uint32_t BAR1 = 56;      // uint64_t [2] MMA1 done, per buffer
  static constexpr uint32_t BAR2 = 72;      // uint64_t     MMA2 done
  static constexpr uint32_t SLOT = 80;      // uint32_t     TMEM base
  static constexpr uint32_t ABORT = 84;     // int          a bounded wait ran out
  static constexpr uint32_t EXACT = 112;    // int [4]      chunk j takes the exact path (entry j & 3)
  static constexpr uint32_t QREADY = 96;    // uint64_t [2] Muir: back -> front: the q tile activated
  static constexpr uint32_t CNT = 128;      // uint32_t [16] issued / completed counts (drain)
  static constexpr uint32_t TBAR = 192;     // uint64_t [2] timing build: MMA1 / MMA2 group timing
};
enum {
  kBIss0, kBIss1, kBDone0, kBDone1, kWIss0, kWIss1, kWDone0, kWDone1,
  kLIss, kLDone, kM1Iss0, kM1Iss1, kM1Done0, kM1Done1, kM2Iss, kNCnt
};

// Tensor maps of the prep inputs, each 4-D (channel, head, token, batch).  k, b, q,
// v, wg: bf16 boxes of 64 channels x 64 tokens with the 128-byte swizzle (one
// 64-column block of an MMA tile); log w: fp32 box of 128 channels x 64 tokens,
// row-major.  Tokens past T read as 0.
struct PrepMaps {
  CUtensorMap k, b, q, v, wg, lw;
};

// One thread: the chunk buffer's tile loads (k, b, q, v) for chunk (b, h, t0); GLA
// (has_b false) has no erase gate and skips b.
__device__ __forceinline__ void load_tiles(uint8_t *buf, const PrepMaps &m, uint64_t *bar, int b,
                                           int h, int t0, bool has_b) {
  using SL = PrepSmem;
  mbar_arrive_expect_tx(bar, (has_b ? 4u : 3u) * kC * kDK * 2);
#pragma unroll
  for (int blk = 0; blk < 2; ++blk) {
    tma_load_4d(buf + SL::B_LM + blk * (kC * 128), &m.k, 64 * blk, h, t0, b, bar);
    if (has_b)
      tma_load_4d(buf + SL::A_LM + blk * (2 * kC * 128), &m.b, 64 * blk, h, t0, b, bar);
    tma_load_4d(buf + SL::A_LM + blk * (2 * kC * 128) + kC * 128, &m.q, 64 * blk, h, t0, b, bar);
    tma_load_4d(buf + SL::VH + blk * (kC * 128), &m.v, 64 * blk, h, t0, b, bar);
  }
}

// One thread: the write gate of chunk (b, h, t0) into staging tile `sw`.
__device__ __forceinline__ void load_gate(uint8_t *sw, const PrepMaps &m, uint64_t *bar, int b, int h,
                                          int t0) {
  mbar_arrive_expect_tx(bar, kC * kDK * 2u);
  tma_load_4d(sw, &m.wg, 0, h, t0, b, bar);
  tma_load_4d(sw + kC * 128, &m.wg, 64, h, t0, b, bar);
}

// One thread: log w of chunk (b, h, t0) into the log-w staging area (fp32; for the
// Muir mixer the decay logits z_f, bf16).
template <bool kMuir>
__device__ __forceinline__ void load_logw(uint8_t *slw, const PrepMaps &m, uint64_t *bar, int b, int h,
                                          int t0) {
  mbar_arrive_expect_tx(bar, kC * kDK * (kMuir ? 2u : 4u));
  tma_load_4d(slw, &m.lw, 0, h, t0, b, bar);
}

// One thread of a group polls `bar` for `parity` (bounded; gives up at once when the
// CTA is aborting), then the group meets at a barrier that ORs every thread's view
// of the abort flag, so the whole group takes the same branch even while the other
// group sets the flag.  Returns false (for the whole group) when the CTA aborts.
template <class Sync>
__device__ __forceinline__ bool group_wait(uint64_t *bar, uint32_t parity, volatile int *abort,
                                           bool poller) {
  bool failed = *abort != 0;
  if (poller && !failed) {
    bool done = mbar_try_wait(bar, parity);
    if (!done) {
      const uint64_t t0 = globaltimer_ns();
      while (!(done = mbar_try_wait(bar, parity)) && *abort == 0) {
        if (globaltimer_ns() - t0 > kWaitLimitNs) break;
      }
    }
    if (!done) {
      *abort = 1;
      failed = true;
    }
  }
  return !Sync::sync_or(failed);
}

// The Muir mixer's activations on the tiles as loaded ("Muir ...", section 2.1 and
// section 4.1): SiLU, the head's l2 norm (the 16 lanes holding one token's 128
// channels reduce with shuffles), the readout gain and the gates.  Seven of these per
// element ride on a kernel that is issue- and latency-bound, so they use the hardware's
// special-function unit directly: sigma(x) = (1 + tanh(x / 2)) / 2 with its tanh (one
// operation where an exponential and a reciprocal take two; absolute error about 2.5e-4,
// and every result is rounded to bf16 next), and its exponential and logarithm for
// softplus, which switches to its asymptotes where 1 + e^x would round.
__device__ __forceinline__ float tanh_approx(float x) {
  float y;
  asm("tanh.approx.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
__device__ __forceinline__ float sigmoid_f(float x) { return fmaf(0.5f, tanh_approx(0.5f * x), 0.5f); }
__device__ __forceinline__ float silu_f(float x) { return x * sigmoid_f(x); }
__device__ __forceinline__ float softplus_f(float x) {
  return x > 15.f ? x : (x < -15.f ? __expf(x) : __logf(1.f + __expf(x)));
}
__device__ __forceinline__ float inv_norm16(const float (&x)[8]) {
  float s = 0.f;
#pragma unroll
  for (int e = 0; e < 8; ++e) s += x[e] * x[e];
#pragma unroll
  for (int o = 1; o < 16; o <<= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
  return rsqrtf(fmaxf(s, 1e-24f));
}

// The chunks one prep CTA walks: items pid, pid + nprep, pid + 2 nprep, ...; item i is
// chunk c of sequence bh, numbered sequence-major (i = bh * nch + c) or, when chain CTAs
// consume the records while they are made, chunk-major (i = c * BH + bh).
struct PrepWork {
  int pid, nprep, BH;
  bool chunk_major;
};

// Publishes a finished record (release at GPU scope; the writers fenced their stores).
__device__ __forceinline__ void publish(uint32_t *flag) {
  __threadfence();
  asm volatile("st.release.gpu.global.u32 [%0], %1;" ::"l"(flag), "r"(1u) : "memory");
}

template <bool kMuir>
__device__ __forceinline__ void prep_body(const FwdParams &p, uint8_t *records, const PrepMaps &maps,
                                          const PrepWork W, uint32_t *flags) {
  using SL = PrepSmem;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  uint8_t *smem = smem_raw + (((raw + 1023u) & ~1023u) - raw);
  const uint32_t sb = smem_u32(smem);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const bool front = tid >= kGroup;
  const int gt = tid & (kGroup - 1);                      // index within the group
  const int qd = warp & 3, cpart = (warp >> 2) & 1;       // TMEM lane quarter, column half
  const int T = p.T, H = p.H, nch = num_chunks(T);
  const int items = p.B * H * nch;
  const int nloc = items > W.pid ? (items - 1 - W.pid) / W.nprep + 1 : 0;
  GDR_PHASE_INIT

  uint8_t *misc = smem + SL::MISC;
  uint64_t *bfull = reinterpret_cast<uint64_t *>(misc + PrepMisc::BFULL);
  uint64_t *wfull = reinterpret_cast<uint64_t *>(misc + PrepMisc::WFULL);
  uint64_t *lfull = reinterpret_cast<uint64_t *>(misc + PrepMisc::LFULL);
  uint64_t *ready = reinterpret_cast<uint64_t *>(misc + PrepMisc::READY);
  uint64_t *qready = reinterpret_cast<uint64_t *>(misc + PrepMisc::QREADY);
  uint64_t *bar1 = reinterpret_cast<uint64_t *>(misc + PrepMisc::BAR1);
  uint64_t *bar2 = reinterpret_cast<uint64_t *>(misc + PrepMisc::BAR2);
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(misc + PrepMisc::SLOT);
  volatile int *sabort = reinterpret_cast<volatile int *>(misc + PrepMisc::ABORT);
  volatile int *sexact = reinterpret_cast<volatile int *>(misc + PrepMisc::EXACT);
  uint32_t *cnt = reinterpret_cast<uint32_t *>(misc + PrepMisc::CNT);
  const float *sLW = reinterpret_cast<const float *>(smem + SL::SLW);
  float *sBT = reinterpret_cast<float *>(smem + SL::BT);
  float *sTOT = reinterpret_cast<float *>(smem + SL::TOT);
  float *sL1 = reinterpret_cast<float *>(smem + SL::L1);
  float *sA1 = reinterpret_cast<float *>(smem + SL::A1);
  const __nv_bfloat16 *gq = static_cast<const __nv_bfloat16 *>(p.q);
  const __nv_bfloat16 *gk = static_cast<const __nv_bfloat16 *>(p.k);
  const __nv_bfloat16 *gb = static_cast<const __nv_bfloat16 *>(p.e1);
  // GDN-2 (erase gate b, optional write gate) or GLA (u = 0: no b, no write gate)
  const bool has_b = p.form == GDR_FORM_GDN2;
  const bool has_wg = has_b && p.e2 != nullptr;
  // Which group forms V^ from v and the write gate: only MMA2 (back group) reads it.  The
  // plain gate product is cheap and stays in the front group; the Muir activations
  // (SiLU(v) sigmoid(z_w)) go to the back group, which otherwise waits on the front.
  const bool wg_front = has_wg && !kMuir, wg_back = has_wg && kMuir;
  float *sNRM = reinterpret_cast<float *>(smem + SL::NRM);   // [buffer][q, k][token]
  const __nv_bfloat16 *gzq = static_cast<const __nv_bfloat16 *>(p.zq);
  auto item_of = [&](int j) { return W.pid + j * W.nprep; };
  auto c_of = [&](int it) { return W.chunk_major ? it / W.BH : it % nch; };
  auto bh_of = [&](int it) { return W.chunk_major ? it % W.BH : it / nch; };
  auto rec_of = [&](int it) { return records + (size_t)(bh_of(it) * nch + c_of(it)) * Rec::BYTES; };
  uint64_t *tbar = reinterpret_cast<uint64_t *>(misc + PrepMisc::TBAR);
  GDR_MMA_DECL(1)
  (void)tbar;

  if (warp == 0) {
    tmem_alloc(tmem_slot, 2 * kTmemCols);
    tmem_relinquish();
  }
  if (tid == 0) {
    for (int i = 0; i < 2; ++i) {
      mbar_init(bfull + i, 1);
      mbar_init(wfull + i, 1);
      mbar_init(ready + i, 1);
      mbar_init(qready + i, 1);
      mbar_init(bar1 + i, 1);
      sexact[i] = 0;
      sexact[i + 2] = 0;
    }
    mbar_init(lfull, 1);
    mbar_init(bar2, 1);
#ifdef GDR_PHASE_TIMING
    mbar_init(tbar, 1);
    mbar_init(tbar + 1, 1);
#endif
    fence_mbar_init();
    *sabort = 0;
    for (int i = 0; i < kNCnt; ++i) cnt[i] = 0;
    for (int j = 0; j < 2 && j < nloc; ++j) {
      const int it = item_of(j), c = c_of(it), bh = bh_of(it);
      load_tiles(smem + j * SL::BUF, maps, bfull + j, bh / H, bh % H, c * kC, has_b);
      ++cnt[kBIss0 + j];
      if (has_wg) {
        load_gate(smem + SL::SW + j * (kC * kDK * 2), maps, wfull + j, bh / H, bh % H, c * kC);
        ++cnt[kWIss0 + j];
      }
      if (j == 0) {
        load_logw<kMuir>(smem + SL::SLW, maps, lfull, bh / H, bh % H, c * kC);
        ++cnt[kLIss];
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = __shfl_sync(0xffffffffu, *tmem_slot, 0);
  const uint32_t tD1 = tmem + 2 * kDK;                    // L | M accumulators, 64 columns x 2

  if (front) {
    // =========================================================== front group
    const bool poller = gt == 0;
    const int g = gt & 15, tb = gt >> 4, j0 = 8 * g;      // 8 channels x 4 tokens per thread
    for (int j = 0; j < nloc; ++j) {
      const int item = item_of(j), bi = j & 1;
      uint8_t *buf = smem + bi * SL::BUF;
      uint8_t *rec = rec_of(item);
      float *a1s = sA1 + (j & 3) * kDK;
      GDR_PREP_PHASE(0);
      // Muir: the head's a_log, loaded now so that its latency overlaps the waits
      const float a_log = kMuir ? __ldg(p.a_log + bh_of(item) % H) : 0.f;

      // chunk j's log w, tiles and write gate have landed.  Muir: the scan (softplus of
      // z_f) needs only the log-w staging, so the tiles and the back group's activation of
      // the q tile are waited for after it, while it runs.  The exact-path flag and a1s
      // are per chunk (entry j & 3): the back group is done with chunk j - 4's by now.
      if (poller) sexact[j & 3] = 0;
      if (!group_wait<FrontSync>(lfull, j & 1, sabort, poller)) break;
      if (!kMuir && !group_wait<FrontSync>(bfull + bi, (j >> 1) & 1, sabort, poller)) break;
      if (wg_front && !group_wait<FrontSync>(wfull + bi, (j >> 1) & 1, sabort, poller)) break;
      if (poller) {
        cnt[kLDone] = j + 1;
        if (!kMuir) cnt[kBDone0 + bi] += 1;
        if (wg_front) cnt[kWDone0 + bi] += 1;
      }
      GDR_PREP_PHASE(1);

      // ---- cumulative log-decay in registers: prefix over the thread's 4 tokens,
      //      then the exclusive prefix over the 16 token blocks (one thread per channel)
      float lam[4][8];
      if constexpr (kMuir) {
        // log alpha = -exp(a_log[h]) softplus(z_f); tokens past T keep the state (log alpha
        // = 0), as the zero-filled log w of the plain path does
        const float rate = __expf(a_log);
        const int tpad = T - c_of(item) * kC;
        const __nv_bfloat16 *zl = reinterpret_cast<const __nv_bfloat16 *>(smem + SL::SLW);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          unpack8(*reinterpret_cast<const uint4 *>(zl + (4 * tb + i) * kDK + j0), lam[i]);
          const bool real = 4 * tb + i < tpad;
#pragma unroll
          for (int e = 0; e < 8; ++e) lam[i][e] = real ? -rate * softplus_f(lam[i][e]) : 0.f;
        }
      } else {
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const float4 x0 = *reinterpret_cast<const float4 *>(sLW + (4 * tb + i) * kDK + j0);
          const float4 x1 = *reinterpret_cast<const float4 *>(sLW + (4 * tb + i) * kDK + j0 + 4);
          lam[i][0] = x0.x; lam[i][1] = x0.y; lam[i][2] = x0.z; lam[i][3] = x0.w;
          lam[i][4] = x1.x; lam[i][5] = x1.y; lam[i][6] = x1.z; lam[i][7] = x1.w;
        }
      }
      GDR_PREP_PHASE(5);
      {
        float tot[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          float acc = 0.f;
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            acc += lam[i][e];
            lam[i][e] = acc;
          }
          tot[e] = acc;
        }
        float4 *bt = reinterpret_cast<float4 *>(sBT + tb * kDK + j0);
        bt[0] = make_float4(tot[0], tot[1], tot[2], tot[3]);
        bt[1] = make_float4(tot[4], tot[5], tot[6], tot[7]);
        if (tb == 0) {
          float4 *l1 = reinterpret_cast<float4 *>(sL1 + j0);
          l1[0] = make_float4(lam[0][0], lam[0][1], lam[0][2], lam[0][3]);
          l1[1] = make_float4(lam[0][4], lam[0][5], lam[0][6], lam[0][7]);
        }
      }
      FrontSync::sync();
      GDR_PREP_PHASE(6);
      // the log-w staging has been read: load the next chunk's
      if (gt == 32 && j + 1 < nloc) {
        fence_proxy_async_smem();
        const int it = item_of(j + 1), cn = c_of(it), bhn = bh_of(it);
        load_logw<kMuir>(smem + SL::SLW, maps, lfull, bhn / H, bhn % H, cn * kC);
        cnt[kLIss] = j + 2;
      }
      if (gt < kDK) {
        float run = 0.f;
#pragma unroll
        for (int r = 0; r < 16; ++r) {
          const float v = sBT[r * kDK + gt];
          sBT[r * kDK + gt] = run;
          run += v;
        }
        sTOT[gt] = run;
      }
      FrontSync::sync();
      GDR_PREP_PHASE(7);
      // lam[i][e] becomes Lam_t - Lam_1 (the pivot at the chunk's first token)
      float dn[8], ed[8];
      {
        const float4 e0 = *reinterpret_cast<const float4 *>(sBT + tb * kDK + j0);
        const float4 e1 = *reinterpret_cast<const float4 *>(sBT + tb * kDK + j0 + 4);
        const float4 a0 = *reinterpret_cast<const float4 *>(sTOT + j0);
        const float4 a4 = *reinterpret_cast<const float4 *>(sTOT + j0 + 4);
        const float4 f0 = *reinterpret_cast<const float4 *>(sL1 + j0);
        const float4 f4 = *reinterpret_cast<const float4 *>(sL1 + j0 + 4);
        const float excl[8] = {e0.x, e0.y, e0.z, e0.w, e1.x, e1.y, e1.z, e1.w};
        const float all[8] = {a0.x, a0.y, a0.z, a0.w, a4.x, a4.y, a4.z, a4.w};
        const float l1[8] = {f0.x, f0.y, f0.z, f0.w, f4.x, f4.y, f4.z, f4.w};
        bool over = false;
#pragma unroll
        for (int e = 0; e < 8; ++e) {
#pragma unroll
          for (int i = 0; i < 4; ++i) lam[i][e] += excl[e] - l1[e];
          dn[e] = all[e] - l1[e];
          ed[e] = __expf(dn[e]);
          over |= dn[e] < -kMaxChunkDecay;
        }
        if (over) sexact[j & 3] = 1;
        if (tb == 0) {
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            a1s[j0 + e] = __expf(l1[e]);
            reinterpret_cast<float *>(rec + Rec::PI)[j0 + e] = __expf(all[e]);
          }
        }
      }
      FrontSync::sync();
      if constexpr (kMuir) {
        if (!group_wait<FrontSync>(bfull + bi, (j >> 1) & 1, sabort, poller)) break;
        if (!group_wait<FrontSync>(qready + bi, (j >> 1) & 1, sabort, poller)) break;
        if (poller) cnt[kBDone0 + bi] += 1;
      }
      const bool exact = sexact[j & 3] != 0;
      GDR_PREP_PHASE(2);

      // ---- operand tiles, in place: k -> K g, b -> K^ f, q -> Q f; Q_pi, K~ to the
      //      record (the exact path also parks Lam_t - Lam_1 there)
      {
        float a1[8];
        {
          const float4 a0 = *reinterpret_cast<const float4 *>(a1s + j0);
          const float4 a4 = *reinterpret_cast<const float4 *>(a1s + j0 + 4);
          a1[0] = a0.x; a1[1] = a0.y; a1[2] = a0.z; a1[3] = a0.w;
          a1[4] = a4.x; a1[5] = a4.y; a1[6] = a4.z; a1[7] = a4.w;
        }
        auto operands = [&](auto exact_path) {
          constexpr bool kExact = decltype(exact_path)::value;
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const int t = 4 * tb + i;
            const uint32_t ok_ = sw128_offset(t, j0, kC * 128);
            const uint32_t ob = SL::A_LM + sw128_offset(t, j0, 2 * kC * 128);
            const uint32_t oq = SL::A_LM + sw128_offset(kC + t, j0, 2 * kC * 128);
            float k8[8], b8[8], q8[8];
            unpack8(*reinterpret_cast<const uint4 *>(buf + SL::B_LM + ok_), k8);
            if (has_b) {
              unpack8(*reinterpret_cast<const uint4 *>(buf + ob), b8);
            } else {
#pragma unroll
              for (int e = 0; e < 8; ++e) b8[e] = 0.f;
            }
            unpack8(*reinterpret_cast<const uint4 *>(buf + oq), q8);
            if constexpr (kMuir) {
              // k = l2norm(silu(k)), b = 2 sigmoid(z_b); the q tile already holds q^ (the
              // back group's activate_q)
#pragma unroll
              for (int e = 0; e < 8; ++e) {
                k8[e] = silu_f(k8[e]);
                b8[e] = 2.f * sigmoid_f(b8[e]);
              }
              const float nk = inv_norm16(k8);
#pragma unroll
              for (int e = 0; e < 8; ++e) k8[e] *= nk;
              if (g == 0) sNRM[bi * 2 * kC + kC + t] = nk;
            }
            float av[8], aq[8], bl[8], kt[8], qp[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) {
              const float f = __expf(lam[i][e]);
              av[e] = b8[e] * k8[e] * f;
              aq[e] = q8[e] * f;
              qp[e] = aq[e] * a1[e];
              if (!kExact) {
                bl[e] = k8[e] * __expf(-lam[i][e]);
                kt[e] = bl[e] * ed[e];
              } else if (dn[e] >= -kMaxChunkDecay) {
                kt[e] = k8[e] * __expf(-lam[i][e]) * ed[e];
                bl[e] = 0.f;     // the exact path forms L and M without K g
              } else {
                kt[e] = k8[e] * __expf(dn[e] - lam[i][e]);
                bl[e] = 0.f;
              }
            }
            st_smem16(buf, ob, pack8(av));
            st_smem16(buf, oq, pack8(aq));
            st_smem16(buf, SL::B_LM + ok_, pack8(bl));
            *reinterpret_cast<uint4 *>(rec + Rec::QY + sw128_offset(t, j0, Rec::QY_STRIDE)) = pack8(qp);
            *reinterpret_cast<uint4 *>(rec + Rec::KT + ok_) = pack8(kt);
            if (kExact) {
              float4 *dst = reinterpret_cast<float4 *>(rec + park_row(t)) + g * 2;
              dst[0] = make_float4(lam[i][0], lam[i][1], lam[i][2], lam[i][3]);
              dst[1] = make_float4(lam[i][4], lam[i][5], lam[i][6], lam[i][7]);
            }
          }
        };
        if (!exact) operands(std::false_type{});
        else operands(std::true_type{});
      }
      // ---- V^ = wg (.) v in place (wg staged at the same swizzled offsets)
      if (wg_front) {
        const uint8_t *sw = smem + SL::SW + bi * (kC * kDK * 2);
#pragma unroll
        for (int u = 0; u < kC * 16 / kGroup; ++u) {
          const uint32_t off = (uint32_t)(gt + u * kGroup) * 16;
          float v8[8], w8[8];
          unpack8(*reinterpret_cast<const uint4 *>(buf + SL::VH + off), v8);
          unpack8(*reinterpret_cast<const uint4 *>(sw + off), w8);
#pragma unroll
          for (int e = 0; e < 8; ++e) v8[e] *= w8[e];
          st_smem16(buf, SL::VH + off, pack8(v8));
        }
      }
      if (flags) __threadfence();      // this thread's record stores, before the back group publishes
      fence_proxy_async_smem();
      FrontSync::sync();
      GDR_PREP_PHASE(3);

      // ---- the write-gate staging tile is read: load chunk j + 2's; MMA1 on this chunk
      if (gt == 32 && wg_front && j + 2 < nloc) {
        fence_proxy_async_smem();
        const int it = item_of(j + 2), cn = c_of(it), bhn = bh_of(it);
        load_gate(smem + SL::SW + bi * (kC * kDK * 2), maps, wfull + bi, bhn / H, bhn % H, cn * kC);
        cnt[kWIss0 + bi] += 1;
      }
      if (warp == 8) {
        // MMA1: [K^ f; Q f] (M = 128) x (K g)^T (N = C), K = DK  -> L, M
        tc_fence_after();
        const uint32_t bb = sb + bi * SL::BUF;
        constexpr uint32_t id = idesc_bf16_f32(128, kC, false, false);
        GDR_MMA_BEGIN()
#pragma unroll
        for (int s = 0; s < kDK / 16; ++s) {
          const uint64_t ad = sdesc_sw128(bb + SL::A_LM + (s >> 2) * (2 * kC * 128) + (s & 3) * 32, 16, 1024);
          const uint64_t bd = sdesc_sw128(bb + SL::B_LM + (s >> 2) * (kC * 128) + (s & 3) * 32, 16, 1024);
          mma_bf16_warp(tD1 + 64 * bi, ad, bd, id, s > 0);
        }
        mma_commit_warp(bar1 + bi);
        GDR_MMA_END(0, tbar);
        if (lane == 0) cnt[kM1Iss0 + bi] += 1;
      }
      // hand the chunk to the back group (the fault-injection hook withholds it)
      if (poller && !(p.debug & kDebugSkipHandoff)) mbar_arrive(ready + bi);
      GDR_PREP_PHASE(4);
    }
  } else {
    // =========================================================== back group
    const bool poller = gt == 0;
    // Muir: q^ = gamma_stat 2 sigmoid(z_q) l2norm(silu(q)) in place in chunk jq's q tile,
    // once its tiles have landed; then the front group may form Q f from it.  The back
    // group does this for chunk j + 2 after its own chunk j, in time it would otherwise
    // spend waiting for the front group.  Its z_q rows are read from global memory by
    // prefetch_q as soon as the chunk's tiles are requested, so that their latency
    // overlaps the U/Y readout instead of following the wait for the tiles.  Returns
    // false when the CTA aborts.
    uint4 zq_raw[4];
    auto prefetch_q = [&](int jq) {
      const int g = gt & 15, tb = gt >> 4, j0 = 8 * g;
      const int it = item_of(jq), bh = bh_of(it), hh = bh % H, t0 = c_of(it) * kC;
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int tt = t0 + 4 * tb + i;
        zq_raw[i] = tt < T ? ld16(gzq + (((size_t)(bh / H) * T + tt) * H + hh) * kDK + j0)
                           : make_uint4(0u, 0u, 0u, 0u);
      }
    };
    auto activate_q = [&](int jq) -> bool {
      const int bq = jq & 1;
      const int g = gt & 15, tb = gt >> 4, j0 = 8 * g;
      const int it = item_of(jq), bh = bh_of(it), hh = bh % H;
      float gs8[8];    // the head's static gain, requested before the wait for the tiles
      if (p.gamma_stat) {
        const float4 a = __ldg(reinterpret_cast<const float4 *>(p.gamma_stat + hh * kDK + j0));
        const float4 c = __ldg(reinterpret_cast<const float4 *>(p.gamma_stat + hh * kDK + j0 + 4));
        gs8[0] = a.x; gs8[1] = a.y; gs8[2] = a.z; gs8[3] = a.w;
        gs8[4] = c.x; gs8[5] = c.y; gs8[6] = c.z; gs8[7] = c.w;
      } else {
#pragma unroll
        for (int e = 0; e < 8; ++e) gs8[e] = 1.f;
      }
      if (!group_wait<BackSync>(bfull + bq, (jq >> 1) & 1, sabort, poller)) return false;
      uint8_t *qb = smem + bq * SL::BUF;
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int t = 4 * tb + i;
        const uint32_t oq = SL::A_LM + sw128_offset(kC + t, j0, 2 * kC * 128);
        float q8[8], zq8[8];
        unpack8(*reinterpret_cast<const uint4 *>(qb + oq), q8);
        unpack8(zq_raw[i], zq8);
#pragma unroll
        for (int e = 0; e < 8; ++e) q8[e] = silu_f(q8[e]);
        const float nq = inv_norm16(q8);
#pragma unroll
        for (int e = 0; e < 8; ++e) q8[e] *= nq * gs8[e] * 2.f * sigmoid_f(zq8[e]);
        st_smem16(qb, oq, pack8(q8));
        if (g == 0) sNRM[bq * 2 * kC + t] = nq;
      }
      BackSync::sync();
      if (poller) mbar_arrive(qready + bq);
      return true;
    };
    bool live = true;
    if constexpr (kMuir)
      for (int jq = 0; jq < 2 && jq < nloc && live; ++jq) {
        prefetch_q(jq);
        live = activate_q(jq);
      }
    for (int j = 0; j < nloc && live; ++j) {
      const int item = item_of(j), c = c_of(item), bh = bh_of(item), h = bh % H, b = bh / H;
      const int t0 = c * kC, n = min(kC, T - t0), bi = j & 1;
      uint8_t *buf = smem + bi * SL::BUF;
      float *sL = reinterpret_cast<float *>(buf + SL::B_LM);
      float *sTi = reinterpret_cast<float *>(buf + SL::A_LM);
      uint8_t *rec = rec_of(item);
      const float *a1s = sA1 + (j & 3) * kDK;
      auto tok_off = [&](int t) { return (((size_t)b * T + t0 + t) * H + h) * kDK; };
      GDR_PREP_PHASE(8);
      if (!group_wait<BackSync>(ready + bi, (j >> 1) & 1, sabort, poller)) break;
      // ---- Muir: V^ = SiLU(v) sigmoid(z_w) in place while MMA1 runs (v's tile landed
      //      before the hand-off; the gate staging tile is waited for here)
      if (wg_back) {
        if (!group_wait<BackSync>(wfull + bi, (j >> 1) & 1, sabort, poller)) break;
        if (poller) cnt[kWDone0 + bi] += 1;
        const uint8_t *sw = smem + SL::SW + bi * (kC * kDK * 2);
#pragma unroll
        for (int u = 0; u < kC * 16 / kGroup; ++u) {
          const uint32_t off = (uint32_t)(gt + u * kGroup) * 16;
          float v8[8], w8[8];
          unpack8(*reinterpret_cast<const uint4 *>(buf + SL::VH + off), v8);
          unpack8(*reinterpret_cast<const uint4 *>(sw + off), w8);
#pragma unroll
          for (int e = 0; e < 8; ++e) v8[e] = silu_f(v8[e]) * sigmoid_f(w8[e]);
          st_smem16(buf, SL::VH + off, pack8(v8));
        }
        fence_proxy_async_smem();   // MMA2 reads V^ after the barriers below
      }
      if (!group_wait<BackSync>(bar1 + bi, (j >> 1) & 1, sabort, poller)) break;
      if (poller) cnt[kM1Done0 + bi] += 1;
      tc_fence_after();
      const bool exact = sexact[j & 3] != 0;
      GDR_PREP_PHASE(9);

      // ---- L (fp32, strictly lower; over the dead K g tile) and M (bf16 -> record)
      if (!exact) {
        float x[32];
        tmem_ld_32x32b_x32(tD1 + 64 * bi + ((uint32_t)(32 * qd) << 16) + 32 * cpart, x);
        tmem_ld_wait();
        const int r = 32 * qd + lane, col = 32 * cpart;
        if (r < kC) {
#pragma unroll
          for (int i = 0; i < 32; ++i) x[i] = (col + i < r) ? x[i] : 0.f;
#pragma unroll
          for (int i = 0; i < 32; i += 4)
            *reinterpret_cast<float4 *>(sL + Ix::at(r, col + i)) = make_float4(x[i], x[i + 1], x[i + 2], x[i + 3]);
        } else {
          const int t = r - kC;
#pragma unroll
          for (int i = 0; i < 32; ++i) x[i] = (col + i <= t) ? x[i] : 0.f;
#pragma unroll
          for (int i = 0; i < 32; i += 8)
            *reinterpret_cast<uint4 *>(rec + Rec::MM + sw128_offset(t, col + i, kC * 128)) = pack8(x + i);
        }
      } else {
        // exact pairwise decays (a chunk whose log-decay exceeds the pivot bound)
        for (int it = gt; it < kC * kC; it += kGroup) {
          const int t = it / kC, s = it % kC;
          float l = 0.f, m = 0.f;
          if (s <= t && t < n) {
            const float *lt = reinterpret_cast<const float *>(rec + park_row(t));
            const float *ls = reinterpret_cast<const float *>(rec + park_row(s));
            const size_t ot = tok_off(t), os = tok_off(s);
            for (int jj = 0; jj < kDK; ++jj) {
              const float d = __expf(__ldcg(lt + jj) - __ldcg(ls + jj));
              float ks = __bfloat162float(gk[os + jj]), kt = __bfloat162float(gk[ot + jj]);
              float qt = __bfloat162float(gq[ot + jj]), bt = has_b ? __bfloat162float(gb[ot + jj]) : 0.f;
              if constexpr (kMuir) {   // the activations of the front group's operand tiles
                const float *nrm = sNRM + bi * 2 * kC;
                const float gs = p.gamma_stat ? __ldg(p.gamma_stat + h * kDK + jj) : 1.f;
                ks = silu_f(ks) * nrm[kC + s];
                kt = silu_f(kt) * nrm[kC + t];
                qt = silu_f(qt) * nrm[t] * gs * 2.f * sigmoid_f(__bfloat162float(gzq[ot + jj]));
                bt = 2.f * sigmoid_f(bt);
              }
              m += qt * d * ks;
              if (has_b) l += bt * kt * d * ks;
            }
          }
          sL[Ix::at(t, s)] = (s < t) ? l : 0.f;
          *reinterpret_cast<__nv_bfloat16 *>(rec + Rec::MM + sw128_offset(t, s, kC * 128)) =
              __float2bfloat16_rn(m);
        }
      }
      tc_fence_before();
      BackSync::sync();
      GDR_PREP_PHASE(10);
      // Muir: every back thread has read the gate staging tile: chunk j + 2's into it
      if (wg_back && gt == 32 && j + 2 < nloc) {
        fence_proxy_async_smem();
        const int it = item_of(j + 2), cn = c_of(it), bhn = bh_of(it);
        load_gate(smem + SL::SW + bi * (kC * kDK * 2), maps, wfull + bi, bhn / H, bhn % H, cn * kC);
        cnt[kWIss0 + bi] += 1;
      }

      // ---- T^-1 (fp32, into the dead Q rows of A_LM), bf16 copy (into the dead L tile)
      invert_diag_blocks8<Ix, QRowsIdx, kGroup, BackSync>(sL, sTi, gt);
      invert_merge_levels<Ix, QRowsIdx, kGroup, BackSync>(sL, sTi, gt);
#pragma unroll
      for (int u = 0; u < 2; ++u) {
        const int it = gt + u * kGroup, t = it >> 3, gg = it & 7;
        const float4 y0 = *reinterpret_cast<const float4 *>(sTi + QRowsIdx::at(t, 8 * gg));
        const float4 y1 = *reinterpret_cast<const float4 *>(sTi + QRowsIdx::at(t, 8 * gg + 4));
        float x[8] = {y0.x, y0.y, y0.z, y0.w, y1.x, y1.y, y1.z, y1.w};
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          const int s = 8 * gg + e;
          x[e] = (s < t) ? x[e] : (s == t ? 1.f : 0.f);
        }
        st_smem16(buf, SL::B_LM + sw128_offset(t, 8 * gg, kC * 128), pack8(x));
      }
      fence_proxy_async_smem();
      tc_fence_before();
      BackSync::sync();
      GDR_PREP_PHASE(11);

      // ---- MMA2: U = T^-1 V^ (N = DV), Y Diag(1/alpha_1) = T^-1 (K^ f) (N = DK); K = C.
      //      (Issued at M = 64: the transposed form, M = 128 and N = C, measured no faster for
      //      these shapes, and its channel-per-thread readout is slower.)
      if (warp == 0) {
        tc_fence_after();
        const uint32_t bb = sb + bi * SL::BUF;
        constexpr uint32_t id = idesc_bf16_f32(64, kDK, false, true);
        GDR_MMA_BEGIN()
#pragma unroll
        for (int s = 0; s < kC / 16; ++s) {
          const uint64_t ad = sdesc_sw128(bb + SL::B_LM + s * 32, 16, 1024);
          const uint64_t bu = sdesc_sw128(bb + SL::VH + s * 2048, kC * 128, 1024);
          const uint64_t by = sdesc_sw128(bb + SL::A_LM + s * 2048, 2 * kC * 128, 1024);
          mma_bf16_warp(tmem, ad, bu, id, s > 0);
          mma_bf16_warp(tmem + kDK, ad, by, id, s > 0);
        }
        mma_commit_warp(bar2);
        GDR_MMA_END(1, tbar + 1);
        if (lane == 0) cnt[kM2Iss] = j + 1;
      }
      if (!group_wait<BackSync>(bar2, j & 1, sabort, poller)) break;
      tc_fence_after();
      GDR_PREP_PHASE(12);

      // ---- the buffer is free: load chunk j + 2's tiles into it
      if (gt == 32 && j + 2 < nloc) {
        fence_proxy_async_smem();
        const int it = item_of(j + 2), cn = c_of(it), bhn = bh_of(it);
        load_tiles(buf, maps, bfull + bi, bhn / H, bhn % H, cn * kC, has_b);
        cnt[kBIss0 + bi] += 1;
      }
      if constexpr (kMuir)
        if (j + 2 < nloc) prefetch_q(j + 2);

      // ---- U and Y (x alpha_1) -> bf16 record tiles.  M = 64 accumulators: row
      //      16 qd + r in TMEM lane 32 qd + r.  Warp (qd, cpart) reads U (cpart 0) or
      //      Y (cpart 1) of its 16 rows, 64 columns per load: lanes 0..15 the first
      //      32, lanes 16..31 the next 32.
      {
        const bool is_y = cpart == 1;
        const uint32_t lane_q = (uint32_t)(32 * qd) << 16;
        const int t = 16 * qd + (lane & 15);
#pragma unroll
        for (int part = 0; part < 2; ++part) {
          const int col = 64 * part + 32 * (lane >> 4);
          float x[32];
          tmem_ld_16x32bx2_x32_split32(tmem + lane_q + (is_y ? kDK : 0) + 64 * part, x);
          tmem_ld_wait();
          if (is_y) {
#pragma unroll
            for (int i = 0; i < 32; i += 4) {
              const float4 a = *reinterpret_cast<const float4 *>(a1s + col + i);
              x[i] *= a.x; x[i + 1] *= a.y; x[i + 2] *= a.z; x[i + 3] *= a.w;
            }
          }
#pragma unroll
          for (int i = 0; i < 32; i += 8)
            *reinterpret_cast<uint4 *>(
                rec + (is_y ? Rec::QY + sw128_offset(kC + t, col + i, Rec::QY_STRIDE)
                            : Rec::U + sw128_offset(t, col + i, kC * 128))) = pack8(x + i);
        }
      }
      if (flags) __threadfence();
      tc_fence_before();
      BackSync::sync();          // U / Y read before the next MMA2 overwrites them
      if (flags && gt == 0) publish(flags + (size_t)bh * nch + c);
      GDR_PREP_PHASE(13);
      if constexpr (kMuir)
        if (j + 2 < nloc && !activate_q(j + 2)) break;
    }
  }

  GDR_PHASE_FINI(1)
  GDR_MMA_FINI(1)
  __syncthreads();
  if (tid == 0 && *sabort) {
    if (p.status) atomicExch(p.status, (uint32_t)GDR_ERR_TIMEOUT);
    // let every TMA load and MMA group still in flight land (each wait bounded)
    for (int bq = 0; bq < 2; ++bq) {
      for (uint32_t d = cnt[kBDone0 + bq]; d < cnt[kBIss0 + bq]; ++d)
        if (!mbar_wait_bounded(bfull + bq, d & 1, kWaitLimitNs)) break;
      for (uint32_t d = cnt[kWDone0 + bq]; d < cnt[kWIss0 + bq]; ++d)
        if (!mbar_wait_bounded(wfull + bq, d & 1, kWaitLimitNs)) break;
      for (uint32_t d = cnt[kM1Done0 + bq]; d < cnt[kM1Iss0 + bq]; ++d)
        if (!mbar_wait_bounded(bar1 + bq, d & 1, kWaitLimitNs)) break;
    }
    for (uint32_t d = cnt[kLDone]; d < cnt[kLIss]; ++d)
      if (!mbar_wait_bounded(lfull, d & 1, kWaitLimitNs)) break;
    if (cnt[kM2Iss] > 0) mbar_wait_bounded(bar2, (cnt[kM2Iss] - 1) & 1, kWaitLimitNs);
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, 2 * kTmemCols);
  }
}

template <bool kMuir>
__global__ void __launch_bounds__(kPrepThreads, 1)
    tc_prep_kernel(FwdParams p, uint8_t *records, const __grid_constant__ PrepMaps maps) {
  prep_body<kMuir>(p, records, maps, PrepWork{(int)blockIdx.x, (int)gridDim.x, p.B * p.H, false},
                   nullptr);
}

// ============================================================== chain kernel
// Per chunk, for one (b, h, value slice of NV = 64 or 128 columns), with S0 the bf16 copy of the
// fp32 state kept in registers:
//   MMA3   D[c&1] = [Q_pi; Y] S0          (M = 2C = 128, K = DK)   rows 0..C-1: Q_pi S0
//   V~ = U - (Y S0)                        (warps on TMEM lanes C..2C-1)
//   MMA4   DS = K~^T V~                    (M = DK, K = C)
//          D[c&1] += [M; *] V~             (M = 128, K = C; rows C..2C-1 are discarded)
//   S <- Diag(pi_n) S + DS                 (fp32, all warps)
//   O = rows 0..C-1 of D[c&1]              (read while MMA3 of chunk c + 1 runs)
// Warp 0 issues the MMAs (lane 0, from converged code); warp 1 refills the record
// ring (three records for NV = 32 and 64, two for NV = 128, the size shared memory
// allows) as soon as MMA4 has released a buffer.  Threads: 32 value columns each (NV = 32
// runs 128 threads, 128 runs 512).  NV = 32 (few long sequences: twice the chains, each
// CTA with half the threads and N = 32 products) keeps S0's bf16 copy and V~ in the
// 64-byte swizzle, whose atom is the slice's 32 columns, and fetches the whole 64-column
// block of U that holds them.
template <int NV>
struct ChainSmem {
  // per buffer: QY | KT | MM | U block(s) (C x UB) | pi.  The U block sits directly after
  // M, so [M; U] is a valid 128-row K-major operand whose lower half only feeds
  // accumulator rows that are discarded.
  static constexpr int UB = NV == 32 ? 64 : NV;                // U columns fetched
  static constexpr int NBUF = NV == 128 ? 2 : 3;               // records in the ring
  static constexpr int NT = 4 * NV;                            // threads: 32 columns each
  static constexpr uint32_t TMEM_COLS = NV == 32 ? 128 : 4 * NV;   // D x 2 and DS, NV columns each
  static constexpr uint32_t B_U = Rec::FRONT;
  static constexpr uint32_t B_PI = B_U + kC * UB * 2;
  static constexpr uint32_t BUF = ((B_PI + kDK * 4 + 1023) / 1024) * 1024;
  static constexpr uint32_t S0B = NBUF * BUF;                 // bf16 S0   DK x NV
  static constexpr uint32_t VT = S0B + kDK * NV * 2;          // bf16 V~   C x NV
  static constexpr uint32_t MISC = VT + kC * NV * 2;          // barriers, TMEM slot, flags
  static constexpr uint32_t ALLOC = MISC + 128 + 1024;
  static constexpr uint32_t TX = Rec::FRONT + kC * UB * 2 + kDK * 4;  // bytes per record fetch
  static_assert(NV == 32 || NV == 64 || NV == 128, "a half, one or both 64-column blocks of U");
  static_assert(VT % 1024 == 0 && S0B % 1024 == 0, "swizzled operand tiles aligned");
  static_assert(B_U == Rec::MM + kC * kC * 2,
                "[M; first 64 columns of U] must form one 128-row operand");
  static_assert(ALLOC <= 227 * 1024, "shared memory");
};

struct ChainMisc {          // byte offsets inside ChainSmem::MISC
  static constexpr uint32_t FULL = 0;      // uint64_t [NBUF] record-arrival barriers
  static constexpr uint32_t BAR3 = 24;     // uint64_t MMA3 completion
  static constexpr uint32_t BAR4 = 32;     // uint64_t MMA4 completion
  static constexpr uint32_t SLOT = 40;     // uint32_t TMEM base
  static constexpr uint32_t ABORT = 44;    // int      a bounded wait ran out
  static constexpr uint32_t FISS = 48;     // uint32_t [NBUF] fetches issued per buffer
  static constexpr uint32_t FDONE = 64;    // uint32_t [NBUF] fetches waited for per buffer
  static constexpr uint32_t TBAR = 80;     // uint64_t timing build: MMA group timing
};

// One lane: fetch record `c` of this CTA's sequence into buffer c % NBUF.
template <int NV>
__device__ __forceinline__ void fetch_record(uint8_t *smem, uint64_t *full, uint32_t *fiss,
                                             const uint8_t *recs, int c, int slice) {
  using SL = ChainSmem<NV>;
  const int buf = c % SL::NBUF;
  uint8_t *dst = smem + buf * SL::BUF;
  const uint8_t *src = recs + (size_t)c * Rec::BYTES;
  ++fiss[buf];
  mbar_arrive_expect_tx(full + buf, SL::TX);
  bulk_g2s(dst, src, Rec::FRONT, full + buf);
  const int ublk = NV == 32 ? slice >> 1 : slice;      // the 64-column block(s) of U
  bulk_g2s(dst + SL::B_U, src + Rec::U + ublk * (kC * 128), kC * SL::UB * 2, full + buf);
  bulk_g2s(dst + SL::B_PI, src + Rec::PI, kDK * 4, full + buf);
}

// Waits (one lane, bounded) until a prep CTA has published record `flag` of the same
// launch; then orders the later bulk copy of it after the publishing CTA's stores.
__device__ __forceinline__ bool wait_published(const uint32_t *flag, volatile int *abort) {
  uint32_t v;
  asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(flag) : "memory");
  if (v == 0) {
    const uint64_t t0 = globaltimer_ns();
    do {
      if (*abort != 0 || globaltimer_ns() - t0 > kWaitLimitNs) return false;
      asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(flag) : "memory");
    } while (v == 0);
  }
  asm volatile("fence.proxy.async.global;" ::: "memory");
  return true;
}

// Barrier of the chain's 256 threads (a named barrier, so that a CTA of more threads can
// run the chain with the rest idle).
template <int NT>
using ChainSync = GroupSync<3, NT>;

// Bounded wait for the MMA group committed to `bar`: thread 0 polls, the chain barrier
// passes the completion on.  Returns false, with the abort flag set, when it ran out.
template <int NT>
__device__ __forceinline__ bool chain_wait_mma(uint64_t *bar, uint32_t &phase, volatile int *abort) {
  if (threadIdx.x == 0 && *abort == 0 && !mbar_wait_bounded(bar, phase, kWaitLimitNs)) *abort = 1;
  phase ^= 1u;
  ChainSync<NT>::sync();
  tc_fence_after();
  return *abort == 0;
}

// The chain of one (b, h, value slice), run by threads 0 .. 255.  `flags` (or null):
// records are published by prep CTAs of the same launch and waited for before fetching.
template <int NV>
__device__ __forceinline__ void chain_body(const FwdParams &p, const uint8_t *records, int slice,
                                           int h, int b, const uint32_t *flags) {
  using SL = ChainSmem<NV>;
  constexpr int NBUF = SL::NBUF, NT = SL::NT;
  constexpr int HALF = 32;      // value columns per thread: NT / 128 column groups of 32
  // bf16 S0 copy and V~ (MN-major B operands of N = NV): byte offsets and descriptors
  auto s0_off = [](int row, int col) -> uint32_t {
    return NV == 32 ? sw64_offset(row, col) : sw128_offset(row, col, kDK * 128);
  };
  auto vt_off = [](int row, int col) -> uint32_t {
    return NV == 32 ? sw64_offset(row, col) : sw128_offset(row, col, kC * 128);
  };
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  uint8_t *smem = smem_raw + (((raw + 1023u) & ~1023u) - raw);
  const uint32_t sb = smem_u32(smem);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int qd = warp & 3, hf = warp >> 2;
  const int c0 = slice * NV;
  const int T = p.T, H = p.H, nch = num_chunks(T);
  const uint32_t *rflags = flags ? flags + ((size_t)b * H + h) * nch : nullptr;
  const uint8_t *recs = records + (size_t)((size_t)b * H + h) * nch * Rec::BYTES;
  GDR_PHASE_INIT

  uint8_t *misc = smem + SL::MISC;
  uint64_t *full = reinterpret_cast<uint64_t *>(misc + ChainMisc::FULL);
  uint64_t *bar3 = reinterpret_cast<uint64_t *>(misc + ChainMisc::BAR3);
  uint64_t *bar4 = reinterpret_cast<uint64_t *>(misc + ChainMisc::BAR4);
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(misc + ChainMisc::SLOT);
  volatile int *sabort = reinterpret_cast<volatile int *>(misc + ChainMisc::ABORT);
  uint32_t *fiss = reinterpret_cast<uint32_t *>(misc + ChainMisc::FISS);
  uint32_t *fdone = reinterpret_cast<uint32_t *>(misc + ChainMisc::FDONE);

  if (warp == 0) {
    tmem_alloc(tmem_slot, SL::TMEM_COLS);
    tmem_relinquish();
  }
  if (tid == 0) {
    for (int i = 0; i < NBUF; ++i) {
      mbar_init(full + i, 1);
      fiss[i] = fdone[i] = 0;
    }
    mbar_init(bar3, 1);
    mbar_init(bar4, 1);
#ifdef GDR_PHASE_TIMING
    mbar_init(reinterpret_cast<uint64_t *>(misc + ChainMisc::TBAR), 1);
#endif
    fence_mbar_init();
    *sabort = 0;
    for (int cc = 0; cc < NBUF && cc < nch; ++cc) {
      if (rflags && !wait_published(rflags + cc, sabort)) {
        *sabort = 1;
        break;
      }
      fetch_record<NV>(smem, full, fiss, recs, cc, slice);
    }
  }

  // fp32 state: key channel jrow, value columns [hf*HALF, hf*HALF + HALF) of this slice
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
    st_smem16(smem, SL::S0B + s0_off(jrow, hf * HALF + i), pack8(st + i));
  fence_proxy_async_smem();
  tc_fence_before();
  ChainSync<NT>::sync();
  tc_fence_after();
  const uint32_t tmem = __shfl_sync(0xffffffffu, *tmem_slot, 0);
  const uint32_t tDS = tmem + 2 * NV;
  const uint32_t lane_q = (uint32_t)(32 * qd) << 16;

  uint64_t *tbar = reinterpret_cast<uint64_t *>(misc + ChainMisc::TBAR);
  GDR_MMA_DECL(0)
  (void)tbar;
  // Warp 0 (all lanes): wait for record c, then MMA3 of chunk c into D[c & 1].  Returns
  // false (and issues nothing) if the record did not arrive in time.
  auto start_chunk = [&](int c) {
    const int buf = c % NBUF;
    bool got = true;
    if (lane == 0) {
      got = mbar_wait_bounded(full + buf, (c / NBUF) & 1, kWaitLimitNs);
      if (got) ++fdone[buf];
    }
    got = __shfl_sync(0xffffffffu, got ? 1 : 0, 0) != 0;
    if (!got) return false;
    GDR_CHAIN_PHASE(7);   // the record has arrived
    const uint32_t bb = sb + buf * SL::BUF;
    constexpr uint32_t id = idesc_bf16_f32(2 * kC, NV, false, true);
    tc_fence_after();
    GDR_MMA_BEGIN()
#pragma unroll
    for (int s = 0; s < kDK / 16; ++s) {
      const uint64_t a = sdesc_sw128(bb + Rec::QY + (s >> 2) * Rec::QY_STRIDE + (s & 3) * 32, 16, 1024);
      const uint64_t bs = NV == 32 ? sdesc_sw64(sb + SL::S0B + s * 1024, kDK * 64, 512)
                                   : sdesc_sw128(sb + SL::S0B + s * 2048, kDK * 128, 1024);
      mma_bf16_warp(tmem + NV * (c & 1), a, bs, id, s > 0);
    }
    mma_commit_warp(bar3);
    GDR_MMA_END(0, tbar);
    return true;
  };
  uint32_t iss3 = 0, iss4 = 0;   // MMA groups committed (counted by warp 0)
  uint32_t ph3 = 0, ph4 = 0;     // completions every thread has waited for
  if (warp == 0) {
    if (start_chunk(0)) ++iss3;
    else if (lane == 0) *sabort = 1;
  }

  bool ok = true;
  for (int c = 0; c < nch; ++c) {
    const int buf = c % NBUF, t0 = c * kC, n = min(kC, T - t0);
    const uint32_t bb = sb + buf * SL::BUF;
    const uint8_t *bsm = smem + buf * SL::BUF;
    const uint32_t tD = tmem + NV * (c & 1);
    GDR_CHAIN_PHASE(0);
    // ---- wait for MMA3 (c): [Q_pi S0; Y S0] in D[c & 1]
    if (!(ok = chain_wait_mma<NT>(bar3, ph3, sabort))) break;
    const float pn = reinterpret_cast<const float *>(bsm + SL::B_PI)[jrow];
    // one-launch path: warp 1 (idle while V~ is formed) sees whether record c + NBUF has
    // been published, so that the acquire's round trip overlaps V~; the same lane issues
    // the refill below
    bool published = true;
    if (rflags && warp == 1 && lane == 0 && c + NBUF < nch && !*sabort)
      published = wait_published(rflags + c + NBUF, sabort);

    GDR_CHAIN_PHASE(1);
    // ---- V~ = U - Y S0 -> bf16 (rows = tokens), on the warps that own lanes C..2C-1
    if (qd >= 2) {
      const int t = 32 * (qd - 2) + lane;
      float d[32];
      tmem_ld_32x32b_x32(tD + lane_q + hf * HALF, d);
      tmem_ld_wait();
#pragma unroll
      for (int i = 0; i < HALF; i += 8) {
        float u8[8];
        const int ucol = (NV == 32 ? (slice & 1) * 32 : hf * HALF) + i;   // column in the U block
        unpack8(*reinterpret_cast<const uint4 *>(bsm + SL::B_U + sw128_offset(t, ucol, kC * 128)), u8);
#pragma unroll
        for (int e = 0; e < 8; ++e) u8[e] = (t < n) ? u8[e] - d[i + e] : 0.f;
        st_smem16(smem, SL::VT + vt_off(t, hf * HALF + i), pack8(u8));
      }
    }
    fence_proxy_async_smem();
    tc_fence_before();
    ChainSync<NT>::sync();

    GDR_CHAIN_PHASE(2);
    // ---- MMA4: DS = K~^T V~ (M = DK) and D[c & 1] += [M; *] V~ (M = 128); K = C
    if (warp == 0) {
      tc_fence_after();
      constexpr uint32_t ids = idesc_bf16_f32(128, NV, true, true);
      constexpr uint32_t ido = idesc_bf16_f32(128, NV, false, true);
      GDR_MMA_BEGIN()
#pragma unroll
      for (int s = 0; s < kC / 16; ++s) {
        const uint64_t ak = sdesc_sw128(bb + Rec::KT + s * 2048, kC * 128, 1024);
        const uint64_t bv = NV == 32 ? sdesc_sw64(sb + SL::VT + s * 1024, kC * 64, 512)
                                     : sdesc_sw128(sb + SL::VT + s * 2048, kC * 128, 1024);
        const uint64_t am = sdesc_sw128(bb + Rec::MM + s * 32, 16, 1024);
        mma_bf16_warp(tDS, ak, bv, ids, s > 0);
        mma_bf16_warp(tD, am, bv, ido, 1);
      }
      mma_commit_warp(bar4);
      GDR_MMA_END(1, tbar);
      ++iss4;
    }
    if (!(ok = chain_wait_mma<NT>(bar4, ph4, sabort))) break;
    // every read of this chunk's buffer is done: refill it NBUF chunks ahead
    if (warp == 1 && lane == 0 && c + NBUF < nch && !*sabort) {
      if (!published) {
        *sabort = 1;
      } else {
        fence_proxy_async_smem();   // the CTA's reads of the buffer come before the refill
        fetch_record<NV>(smem, full, fiss, recs, c + NBUF, slice);
      }
    }

    GDR_CHAIN_PHASE(3);
    // ---- state update (fp32) and its bf16 copy for the next MMA3
    {
      float d[32];
      tmem_ld_32x32b_x32(tDS + lane_q + hf * HALF, d);
      tmem_ld_wait();
#pragma unroll
      for (int i = 0; i < HALF; ++i) st[i] = pn * st[i] + d[i];
#pragma unroll
      for (int i = 0; i < HALF; i += 8)
        st_smem16(smem, SL::S0B + s0_off(jrow, hf * HALF + i), pack8(st + i));
    }
    fence_proxy_async_smem();
    tc_fence_before();
    ChainSync<NT>::sync();

    GDR_CHAIN_PHASE(4);
    // ---- warp 0 starts chunk c + 1; warps owning lanes 0..C-1 store O (c) meanwhile
    if (warp == 0 && c + 1 < nch && !*sabort) {
      if (start_chunk(c + 1)) ++iss3;
      else if (lane == 0) *sabort = 1;
    }
    GDR_CHAIN_PHASE(5);
    if (qd < 2) {
      float o[32];
      tmem_ld_32x32b_x32(tD + lane_q + hf * HALF, o);
      tmem_ld_wait();
      const int t = 32 * qd + lane;
      if (t < n) {
        float4 *dst = reinterpret_cast<float4 *>(
            p.o + (((size_t)b * T + t0 + t) * H + h) * kDK + c0 + hf * HALF);
#pragma unroll
        for (int i = 0; i < HALF; i += 4) dst[i / 4] = make_float4(o[i], o[i + 1], o[i + 2], o[i + 3]);
      }
    }
    tc_fence_before();
    GDR_CHAIN_PHASE(6);
  }

  GDR_PHASE_FINI(0)
  GDR_MMA_FINI(0)
  if (ok && p.S_T) {
#pragma unroll
    for (int i = 0; i < HALF; i += 4)
      *reinterpret_cast<float4 *>(p.S_T + s_off + i) = make_float4(st[i], st[i + 1], st[i + 2], st[i + 3]);
  }
  // after a timeout: let the MMAs and record copies already in flight land before
  // the CTA exits (every wait bounded)
  ChainSync<NT>::sync();
  if (!ok && tid == 0) {   // thread 0 is warp 0's issuing lane: iss3 / iss4 are its counts
    if (p.status) atomicExch(p.status, (uint32_t)GDR_ERR_TIMEOUT);
    // groups complete in order: wait for the last one committed on each barrier
    if (iss3 > 0) mbar_wait_bounded(bar3, (iss3 - 1) & 1, kWaitLimitNs);
    if (iss4 > 0) mbar_wait_bounded(bar4, (iss4 - 1) & 1, kWaitLimitNs);
    for (int bq = 0; bq < NBUF; ++bq)
      while (fdone[bq] < fiss[bq]) {
        if (!mbar_wait_bounded(full + bq, fdone[bq] & 1, kWaitLimitNs)) break;
        ++fdone[bq];
      }
  }
  tc_fence_before();
  ChainSync<NT>::sync();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, SL::TMEM_COLS);
  }
}

template <int NV>
__global__ void __launch_bounds__(ChainSmem<NV>::NT, 1) tc_chain_kernel(FwdParams p, const uint8_t *records) {
  chain_body<NV>(p, records, blockIdx.x, blockIdx.y, blockIdx.z, nullptr);
}

// Few long sequences (the chain CTAs leave most SMs idle): one cooperative launch in which
// CTAs 0 .. nchain-1 run the chain of one (b, h, value slice) each while the others walk
// the chunks chunk-major as prep CTAs and publish each finished record; a chain CTA waits
// (bounded) for a record's flag before fetching it.  Only prep CTAs make records and they
// wait on no chain CTA, and the cooperative launch keeps every CTA resident, so each wait
// ends.
template <bool kMuir, int NV>
__global__ void __launch_bounds__(kPrepThreads, 1)
    tc_fused_kernel(FwdParams p, uint8_t *records, const __grid_constant__ PrepMaps maps,
                    uint32_t *flags, int nchain) {
  static_assert(kPrepThreads >= ChainSmem<NV>::NT, "the chain runs on the first NT threads");
  if ((int)blockIdx.x < nchain) {
    if ((int)threadIdx.x >= ChainSmem<NV>::NT) return;   // the chain's barriers count its own threads
    const int nsl = p.dv / NV, i = blockIdx.x;
    chain_body<NV>(p, records, i % nsl, (i / nsl) % p.H, i / nsl / p.H, flags);
  } else {
    prep_body<kMuir>(p, records, maps,
                     PrepWork{(int)blockIdx.x - nchain, (int)gridDim.x - nchain, p.B * p.H, true},
                     flags);
  }
}

}  // namespace

// GDN-2 and GLA (GDN-2 with b = 0), bf16, d_k = d_v = 128; chunk 64, or 128 served
// as two 64-token chunks.
bool forward_tc_split_supported(const FwdParams &p, gdr_dtype dtype) {
  return (p.form == GDR_FORM_GDN2 || p.form == GDR_FORM_GLA) && dtype == GDR_BF16 &&
         p.dk == kDK && p.dv == kDK && (p.chunk == kC || p.chunk == 2 * kC);
}

// Header, one record per (b, h, chunk), then one publication flag per record (used when
// the records are consumed as they are made).
size_t forward_tc_split_workspace_bytes(const FwdParams &p) {
  const size_t recs = (size_t)p.B * p.H * num_chunks(p.T);
  return kHeaderBytes + recs * Rec::BYTES + ((recs * 4 + 255) & ~(size_t)255);
}

namespace {

// [B][T][H][128] input as the prep kernel's 4-D map: boxes of `box0` channels x C tokens.
bool encode_input_map(CUtensorMap *m, const void *base, CUtensorMapDataType type, int elem,
                      int box0, CUtensorMapSwizzle swizzle, const FwdParams &p) {
  return tma::encode_input_map(m, base, type, elem, box0, kC, swizzle, p.H, p.T, p.B);
}

// The one-launch path with value slices of NV columns (tc_fused_kernel): one CTA per SM,
// the first B H (d_v / NV) running the chains.  *launched stays false when the kernel
// cannot keep one CTA resident per SM (the caller then takes the two launches).
template <int NV>
cudaError_t launch_fused(const FwdParams &p, uint8_t *records, const PrepMaps &maps, int sms,
                         int items, cudaStream_t stream, bool *launched) {
  *launched = false;
  auto fused = p.muir ? tc_fused_kernel<true, NV> : tc_fused_kernel<false, NV>;
  const int smem = (int)(PrepSmem::ALLOC > ChainSmem<NV>::ALLOC ? PrepSmem::ALLOC : ChainSmem<NV>::ALLOC);
  cudaError_t e = cudaFuncSetAttribute(fused, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  int per_sm = 0;
  if ((e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, fused, kPrepThreads, smem)) != cudaSuccess)
    return e;
  if (per_sm < 1) return cudaSuccess;
  uint32_t *flags = reinterpret_cast<uint32_t *>(records + (size_t)items * Rec::BYTES);
  if ((e = cudaMemsetAsync(flags, 0, (size_t)items * 4, stream)) != cudaSuccess) return e;
  FwdParams pp = p;
  PrepMaps mm = maps;
  int nchain = (p.dv / NV) * p.H * p.B;
  void *args[] = {&pp, &records, &mm, &flags, &nchain};
  *launched = true;
  return cudaLaunchCooperativeKernel(reinterpret_cast<const void *>(fused), dim3(sms), dim3(kPrepThreads),
                                     args, (size_t)smem, stream);
}

}  // namespace

cudaError_t launch_forward_tc_split(const FwdParams &p, void *workspace, cudaStream_t stream) {
  constexpr int NV = 64;
  PrepMaps maps;
  memset(&maps, 0, sizeof(maps));
  // bf16 tiles: 64-channel boxes with the 128-byte swizzle (the MMA operand layout);
  // log w: one 128-channel fp32 box, row-major
  const CUtensorMapDataType bf = CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
  const CUtensorMapSwizzle sw = CU_TENSOR_MAP_SWIZZLE_128B;
  const bool has_b = p.form == GDR_FORM_GDN2;
  const bool lw_ok = p.muir ? encode_input_map(&maps.lw, p.zf, bf, 2, kDK, CU_TENSOR_MAP_SWIZZLE_NONE, p)
                            : encode_input_map(&maps.lw, p.log_w, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4,
                                               kDK, CU_TENSOR_MAP_SWIZZLE_NONE, p);
  if (!encode_input_map(&maps.k, p.k, bf, 2, 64, sw, p) ||
      (has_b && !encode_input_map(&maps.b, p.e1, bf, 2, 64, sw, p)) ||
      !encode_input_map(&maps.q, p.q, bf, 2, 64, sw, p) ||
      !encode_input_map(&maps.v, p.v, bf, 2, 64, sw, p) ||
      (has_b && p.e2 && !encode_input_map(&maps.wg, p.e2, bf, 2, 64, sw, p)) || !lw_ok)
    return cudaErrorInvalidValue;
  if (p.muir && (!has_b || !p.e2 || !p.zq || !p.a_log)) return cudaErrorInvalidValue;
  uint8_t *records = static_cast<uint8_t *>(workspace) + kHeaderBytes;
  auto prep = p.muir ? tc_prep_kernel<true> : tc_prep_kernel<false>;
  cudaError_t e = cudaFuncSetAttribute(prep, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)PrepSmem::ALLOC);
  if (e != cudaSuccess) return e;
  e = cudaFuncSetAttribute(tc_chain_kernel<NV>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           (int)ChainSmem<NV>::ALLOC);
  if (e != cudaSuccess) return e;
  int dev = 0, sms = 0;
  if ((e = cudaGetDevice(&dev)) != cudaSuccess) return e;
  if ((e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess) return e;
  const int nch = num_chunks(p.T);
  const int items = p.B * p.H * nch;
  if (nch >= kFusedMinChunks) {
    // few long sequences: chains and prep in one cooperative launch (tc_fused_kernel), with
    // 32-column value slices while their chains take at most half the SMs, else 64-column
    // slices while theirs take at most a third
    const int bh = p.B * p.H;
    bool launched = false;
    if (bh * (p.dv / 32) * 2 <= sms)
      e = launch_fused<32>(p, records, maps, sms, items, stream, &launched);
    else if (bh * (p.dv / NV) * 3 <= sms)
      e = launch_fused<NV>(p, records, maps, sms, items, stream, &launched);
    if (e != cudaSuccess || launched) return e;
  }
  prep<<<min(items, sms), kPrepThreads, PrepSmem::ALLOC, stream>>>(p, records, maps);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  dim3 gc(p.dv / NV, p.H, p.B);
  tc_chain_kernel<NV><<<gc, ChainSmem<NV>::NT, ChainSmem<NV>::ALLOC, stream>>>(p, records);
  return cudaGetLastError();
}

}  // namespace gdr

#ifdef GDR_PHASE_TIMING
// Timing build only: copies the per-phase cycle sums ([2][16]: chain, prep) and the number
// of recording threads ([2]) to host memory, then clears them.  Returns 0 or a CUDA error.
extern "C" int gdr_phase_timing_read(unsigned long long *cycles, unsigned long long *threads,
                                     unsigned long long *mma_cycles, unsigned long long *mma_groups) {
  cudaError_t e = cudaDeviceSynchronize();
  if (e == cudaSuccess) e = cudaMemcpyFromSymbol(cycles, gdr::g_phase_cycles, sizeof(gdr::g_phase_cycles));
  if (e == cudaSuccess) e = cudaMemcpyFromSymbol(threads, gdr::g_phase_threads, sizeof(gdr::g_phase_threads));
  if (e == cudaSuccess) e = cudaMemcpyFromSymbol(mma_cycles, gdr::g_mma_cycles, sizeof(gdr::g_mma_cycles));
  if (e == cudaSuccess) e = cudaMemcpyFromSymbol(mma_groups, gdr::g_mma_groups, sizeof(gdr::g_mma_groups));
  static const unsigned long long zc[2][16] = {}, zt[2] = {}, zm[2][8] = {};
  if (e == cudaSuccess) e = cudaMemcpyToSymbol(gdr::g_phase_cycles, zc, sizeof(zc));
  if (e == cudaSuccess) e = cudaMemcpyToSymbol(gdr::g_phase_threads, zt, sizeof(zt));
  if (e == cudaSuccess) e = cudaMemcpyToSymbol(gdr::g_mma_cycles, zm, sizeof(zm));
  if (e == cudaSuccess) e = cudaMemcpyToSymbol(gdr::g_mma_groups, zm, sizeof(zm));
  return (int)e;
}

// Timing build only: copies the MMA-group interval log (g_mma_log [2][256][256][2],
// g_mma_log_group [2][256][256], g_mma_log_n [2][256]) to host memory and clears the counts.
// Returns 0 or a CUDA error.
extern "C" int gdr_phase_timing_read_log(unsigned long long *intervals, unsigned int *groups,
                                         unsigned int *counts) {
  cudaError_t e = cudaDeviceSynchronize();
  if (e == cudaSuccess) e = cudaMemcpyFromSymbol(intervals, gdr::g_mma_log, sizeof(gdr::g_mma_log));
  if (e == cudaSuccess) e = cudaMemcpyFromSymbol(groups, gdr::g_mma_log_group, sizeof(gdr::g_mma_log_group));
  if (e == cudaSuccess) e = cudaMemcpyFromSymbol(counts, gdr::g_mma_log_n, sizeof(gdr::g_mma_log_n));
  static const unsigned int zn[2][gdr::kMmaLogCtas] = {};
  if (e == cudaSuccess) e = cudaMemcpyToSymbol(gdr::g_mma_log_n, zn, sizeof(zn));
  return (int)e;
}
#endif
