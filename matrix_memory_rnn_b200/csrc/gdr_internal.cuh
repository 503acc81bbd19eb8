// gdr_internal.cuh -- device helpers and launcher declarations shared by the
// libgdr kernels (not part of the public ABI; see include/gdr.h).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "gdr.h"

namespace gdr {

// Widening loads of the two input element types.
__device__ __forceinline__ float ld_in(const float *p, size_t i) { return __ldg(p + i); }
__device__ __forceinline__ float ld_in(const __nv_bfloat16 *p, size_t i) {
  return __bfloat162float(p[i]);
}

// The form's erase vector u_j and erase key z_j for one token, from the raw
// arguments (include/gdr.h): general u = e1, z = e2; GDN-2 u = alpha b k, z = k;
// RWKV-7 u = c a, z = a; GLA u = z = 0.  `wj` is the decay exp(log_w_j).
template <typename Tin>
__device__ __forceinline__ void erase_pair(gdr_form form, const Tin *k, const Tin *e1,
                                           const Tin *e2, size_t idx_k, size_t idx_s,
                                           float wj, float &u, float &z) {
  switch (form) {
    case GDR_FORM_GENERAL:
      u = ld_in(e1, idx_k);
      z = ld_in(e2, idx_k);
      break;
    case GDR_FORM_GDN2: {
      const float kj = ld_in(k, idx_k);
      u = wj * ld_in(e1, idx_k) * kj;
      z = kj;
      break;
    }
    case GDR_FORM_RWKV7: {
      const float a = ld_in(e1, idx_k);
      u = ld_in(e2, idx_s) * a;
      z = a;
      break;
    }
    default:
      u = 0.f;
      z = 0.f;
      break;
  }
}

struct FwdParams {
  gdr_form form;
  int B, H, T, dk, dv, chunk;
  const void *q, *k, *v, *e1, *e2;
  const float *log_w;
  const float *S0;
  float *o;
  float *S_T;
  uint32_t *status;  // device status word (workspace), may be null
  uint32_t debug;    // fault-injection bits (kDebug...), 0 in normal use
  // The Muir mixer's prologue inside the tensor-core forward (gdr_muir_forward):
  // q, k, v, e1, e2 then hold the raw q, k, v, z_b, z_w, and the decay comes from
  // z_f and a_log instead of log_w.
  bool muir;
  const void *zf, *zq;
  const float *a_log, *gamma_stat;
};

// Fault injection for the tests of the bounded waits (set through the environment
// variable GDR_DEBUG_FAULT, read per call on the host): the prep kernel's front warp
// group never hands its chunks to the back group, the single-kernel tensor-core forward
// never commits its first product, and the tcgen05 mLSTM kernel never commits its
// [P~ V | P~ 1] product; in each a bounded wait then runs out.
constexpr uint32_t kDebugSkipHandoff = 1u;
// Timing build only (environment variable GDR_TIMING_MMA): the MMA-issuing warps wait for
// each tensor-core group and time it.
constexpr uint32_t kDebugTimeMma = 2u;

// Reverse mode (gdr_backward_chunked).  Chunks of kBwdChunk tokens, nc of them per
// sequence; the workspace sections hold, per chunk, the records of the two chains
// (rec), the chunk-start states plus the final state (states, nc + 1 per sequence)
// and the adjoints of the chunk-end states (adj).
constexpr int kBwdChunk = 32;
struct BwdParams {
  gdr_form form;
  int B, H, T, dk, dv, nc;
  const void *q, *k, *v, *e1, *e2;
  const float *log_w, *S0, *dO, *dS_T;
  float *gq, *gk, *gv, *glw, *ge1, *ge2, *gS0;
  float *rec, *states, *adj;
};
size_t backward_workspace_bytes(int form, int B, int H, int T, int dk, int dv);
bool backward_supported(int dk, int dv);
cudaError_t launch_backward(const BwdParams &p, gdr_dtype dtype, void *workspace,
                            cudaStream_t stream);

// The Muir token mixer (gdr_muir_forward): raw activations and gate logits.
struct MuirParams {
  int B, H, T, dk, dv;
  const void *q, *k, *v, *zf, *zb, *zw, *zq, *zg;
  const float *a_log, *gamma_stat, *rms_weight;
  float rms_eps;
};
// Prologue into activated inputs of the GDN-2 forward (q^, k^, v^, b, w at the input
// type; log alpha fp32), and the RMSNorm (.) SiLU(zg) epilogue of o into y.
cudaError_t launch_muir_prologue(const MuirParams &m, gdr_dtype dtype, void *qh, void *kh,
                                 void *vh, void *b, void *w, float *log_w, cudaStream_t stream);
cudaError_t launch_muir_epilogue(const MuirParams &m, gdr_dtype dtype, const float *o, float *y,
                                 cudaStream_t stream);

// S_out = M S_in + Q per head (gdr_state_compose).
cudaError_t launch_state_compose(float *S_out, const float *M, const float *S_in, const float *Q,
                                 int BH, int dk, int dv, cudaStream_t stream);

// xLSTM's mLSTM cell (gdr_mlstm_forward); p[0 .. n) = x.  bf16 inputs with d_k = d_v = 128
// take the tensor-core kernel, the rest the warp-MMA kernel.
cudaError_t launch_mlstm(const gdr_mlstm_args &a, cudaStream_t stream);
bool mlstm_tc_supported(const gdr_mlstm_args &a);
cudaError_t launch_mlstm_tc(const gdr_mlstm_args &a, cudaStream_t stream);
cudaError_t fill_f32(float *p, size_t n, float x, cudaStream_t stream);

// Launchers (host).  Return cudaSuccess or the launch error.
cudaError_t launch_decode(const gdr_step_args &a, cudaStream_t stream);
cudaError_t launch_forward_fp32(const FwdParams &p, gdr_dtype dtype, cudaStream_t stream);
bool forward_fp32_supported(int dk, int dv);
cudaError_t launch_forward_recur(const FwdParams &p, gdr_dtype dtype, cudaStream_t stream);
bool forward_recur_supported(int dk, int dv);
cudaError_t launch_forward_tc(const FwdParams &p, cudaStream_t stream);
bool forward_tc_supported(const FwdParams &p, gdr_dtype dtype);
// Tensor-core path for the two-stream forms (general, RWKV-7), d_k = d_v = 64: one
// fused kernel per (b, h); needs only the status word as workspace.
bool forward_tc_general_supported(const FwdParams &p, gdr_dtype dtype);
cudaError_t launch_forward_tc_general(const FwdParams &p, cudaStream_t stream);
// Two-kernel tensor-core path: per-chunk records in the workspace.
bool forward_tc_split_supported(const FwdParams &p, gdr_dtype dtype);
size_t forward_tc_split_workspace_bytes(const FwdParams &p);
cudaError_t launch_forward_tc_split(const FwdParams &p, void *workspace, cudaStream_t stream);

// Smallest workspace any forward path accepts (the device status word, padded).
constexpr size_t kStatusBytes = 256;

// Which kernel gdr_forward_chunked runs for given arguments and workspace size.
enum class FwdPath { kNone, kCopyState, kTcGeneral, kTcSplit, kTcSingle, kFp32, kRecur };
// Host validation and selection (no CUDA call): every check gdr_forward_chunked makes on
// its arguments and on a workspace at `workspace` (alignment; may be null) of
// `workspace_bytes` bytes, except that a null workspace on a path that needs one is
// reported by the caller.
gdr_status forward_plan(const gdr_fwd_args *a, const void *workspace, size_t workspace_bytes,
                        FwdPath *path);
size_t forward_fp32_smem_bytes(int dk, int dv, int chunk);

}  // namespace gdr
