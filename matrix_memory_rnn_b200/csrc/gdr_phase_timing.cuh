// gdr_phase_timing.cuh -- per-phase cycle accounting of the two-kernel tensor-core forward,
// for a separate timing build (compiled with -DGDR_PHASE_TIMING into libgdr_timing.so by
// `python -m matrix_memory_rnn_b200.build --timing`; libgdr.so leaves the hooks empty).
//
// The kernels mark the start of each phase of their per-chunk loop with GDR_PREP_PHASE(i) /
// GDR_CHAIN_PHASE(i).  Here one thread per warp group (thread 0, and thread 256 in the
// prep kernel's front group) adds the clock64 cycles between consecutive marks to
// register totals, and at the end of the kernel (GDR_PHASE_FINI(slot)) adds them to
// device-wide sums: slot 0 the chain kernel, slot 1 the prep kernel, 16 phases each.
// gdr_phase_timing_read() returns and clears the sums.  The marks cost a few cycles and
// one register array; the totals include the time a thread waits at the next mark.
#pragma once

#ifdef GDR_PHASE_TIMING
namespace gdr {
__device__ unsigned long long g_phase_cycles[2][16];
__device__ unsigned long long g_phase_threads[2];
}  // namespace gdr

#define GDR_PHASE_INIT                                    \
  long long gdr_pa_[16] = {0};                            \
  long long gdr_pl_ = 0;                                  \
  const bool gdr_pon_ = threadIdx.x == 0 || threadIdx.x == 256;
#define GDR_PHASE_MARK_(i)                                \
  do {                                                    \
    if (gdr_pon_) {                                       \
      const long long n_ = clock64();                     \
      if (gdr_pl_) gdr_pa_[i] += n_ - gdr_pl_;            \
      gdr_pl_ = n_;                                       \
    }                                                     \
  } while (0)
#define GDR_PREP_PHASE(i) GDR_PHASE_MARK_(i)
#define GDR_CHAIN_PHASE(i) GDR_PHASE_MARK_(i)
#define GDR_PHASE_FINI(slot)                                                               \
  if (gdr_pon_) {                                                                          \
    for (int i_ = 0; i_ < 16; ++i_)                                                        \
      if (gdr_pa_[i_]) atomicAdd(&gdr::g_phase_cycles[slot][i_], (unsigned long long)gdr_pa_[i_]); \
    atomicAdd(&gdr::g_phase_threads[slot], 1ull);                                          \
  }
#endif
