// gdr_phase_timing.cuh -- per-phase cycle accounting of the two-kernel tensor-core forward,
// for a separate timing build (compiled with -DGDR_PHASE_TIMING into libgdr_timing.so by
// `python -m matrix_memory_rnn_b200.build --timing`; libgdr.so leaves the hooks empty).
//
// The kernels mark the phases of their per-chunk loops with GDR_PREP_PHASE(i) /
// GDR_CHAIN_PHASE(i).  Here a few recording threads (listed below) add the clock64 cycles
// between consecutive marks to register totals, and at the end of the kernel
// (GDR_PHASE_FINI(slot)) add them to device-wide sums: slot 0 the chain kernel, slot 1 the
// prep kernel, 16 phases each.
// gdr_phase_timing_read() returns and clears the sums.  The marks cost a few cycles and
// one register array; the totals include the time a thread waits at the next mark.
#pragma once

#ifdef GDR_PHASE_TIMING
namespace gdr {
__device__ unsigned long long g_phase_cycles[2][16];
__device__ unsigned long long g_phase_threads[2];
// Tensor-core groups: per kernel (slot) and group, the summed cycles from the issue of the
// group's first MMA to the arrival of its completion, and the number of groups timed.
__device__ unsigned long long g_mma_cycles[2][8];
__device__ unsigned long long g_mma_groups[2][8];
// The same groups as intervals, per kernel and CTA (linear block index): [start, end] in the
// SM's clock64 and the group, for the first kMmaLogEntries groups of the first kMmaLogCtas
// CTAs; so that the host can take the union of the intervals in which a CTA had a group in
// flight (the prep kernel's two warp groups overlap theirs).
constexpr int kMmaLogCtas = 256, kMmaLogEntries = 256;
__device__ unsigned long long g_mma_log[2][kMmaLogCtas][kMmaLogEntries][2];
__device__ unsigned int g_mma_log_group[2][kMmaLogCtas][kMmaLogEntries];
__device__ unsigned int g_mma_log_n[2][kMmaLogCtas];
}  // namespace gdr

// MMA-group timing, in the issuing warp (GDR_MMA_DECL(slot): 0 the chain, 1 prep):
// GDR_MMA_BEGIN before a group's first MMA;
// GDR_MMA_END(g, tbar) after its commit commits once more to the timing-only mbarrier
// `tbar`, waits for it (bounded), and adds the elapsed cycles to group g.  The issuing
// warp thus waits for each group before issuing the next, so the measured interval is
// the group's own issue, execution and completion, not time queued behind other groups
// of the same warp.
#define GDR_MMA_DECL(slot)                                 \
  long long gdr_mc_[8] = {0};                              \
  unsigned gdr_mn_[8] = {0};                               \
  uint32_t gdr_mp_ = 0;                                    \
  long long gdr_mb_ = 0;                                   \
  const int gdr_ms_ = (slot);
#define GDR_MMA_BEGIN() gdr_mb_ = clock64();
// (only when the call asked for it: the waits change the kernel's schedule, so the phase
// accounting above is taken in a separate pass without them)
#define GDR_MMA_END(g, tbar)                                                   \
  do {                                                                         \
    if (p.debug & kDebugTimeMma) {                                             \
      mma_commit_warp(tbar);                                                   \
      if ((threadIdx.x & 31) == 0) mbar_wait_bounded(tbar, gdr_mp_ & 1u, 1000000000ull); \
      __syncwarp();                                                            \
      ++gdr_mp_;                                                               \
      const long long gdr_me_ = clock64();                                     \
      gdr_mc_[g] += gdr_me_ - gdr_mb_;                                         \
      ++gdr_mn_[g];                                                            \
      const unsigned gdr_cta_ = blockIdx.x + gridDim.x * (blockIdx.y + gridDim.y * blockIdx.z); \
      if ((threadIdx.x & 31) == 0 && gdr_cta_ < (unsigned)gdr::kMmaLogCtas) {   \
        const unsigned k_ = atomicAdd(&gdr::g_mma_log_n[gdr_ms_][gdr_cta_], 1u); \
        if (k_ < (unsigned)gdr::kMmaLogEntries) {                              \
          gdr::g_mma_log[gdr_ms_][gdr_cta_][k_][0] = (unsigned long long)gdr_mb_; \
          gdr::g_mma_log[gdr_ms_][gdr_cta_][k_][1] = (unsigned long long)gdr_me_; \
          gdr::g_mma_log_group[gdr_ms_][gdr_cta_][k_] = (unsigned)(g);          \
        }                                                                      \
      }                                                                        \
    }                                                                          \
  } while (0)
#define GDR_MMA_FINI(slot)                                                      \
  if ((threadIdx.x & 31) == 0) {                                               \
    for (int i_ = 0; i_ < 8; ++i_)                                             \
      if (gdr_mn_[i_]) {                                                       \
        atomicAdd(&gdr::g_mma_cycles[slot][i_], (unsigned long long)gdr_mc_[i_]); \
        atomicAdd(&gdr::g_mma_groups[slot][i_], (unsigned long long)gdr_mn_[i_]); \
      }                                                                        \
  }

// Recording threads: the prep kernel's threads 0 (back group) and 256 (front group), the
// chain kernel's thread 0.
#define GDR_PHASE_INIT                                    \
  long long gdr_pa_[16] = {0};                            \
  long long gdr_pl_ = 0;
#define GDR_PHASE_MARK_(on, i)                            \
  do {                                                    \
    if (on) {                                             \
      const long long n_ = clock64();                     \
      if (gdr_pl_) gdr_pa_[i] += n_ - gdr_pl_;            \
      gdr_pl_ = n_;                                       \
    }                                                     \
  } while (0)
#define GDR_PREP_PHASE(i) GDR_PHASE_MARK_(threadIdx.x == 0 || threadIdx.x == 256, i)
#define GDR_CHAIN_PHASE(i) GDR_PHASE_MARK_(threadIdx.x == 0, i)
#define GDR_PHASE_FINI(slot)                                                               \
  if (gdr_pl_) {                                                                           \
    for (int i_ = 0; i_ < 16; ++i_)                                                        \
      if (gdr_pa_[i_]) atomicAdd(&gdr::g_phase_cycles[slot][i_], (unsigned long long)gdr_pa_[i_]); \
    atomicAdd(&gdr::g_phase_threads[slot], 1ull);                                          \
  }
#endif
