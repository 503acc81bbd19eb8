// gdr_api.cu -- the extern "C" entry points of libgdr: argument validation,
// kernel selection and launch.  Declarations and the contract: include/gdr.h.
#include <cmath>
#include <cstdint>
#include <cstdlib>
#include <cstring>

#include "gdr_internal.cuh"

namespace {

bool dim_ok(int d) { return d == 16 || d == 32 || d == 64 || d == 128; }
bool chunk_ok(int c) { return c == 16 || c == 32 || c == 64 || c == 128; }
bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
bool form_ok(gdr_form f) { return f >= GDR_FORM_GENERAL && f <= GDR_FORM_GLA; }
bool dtype_ok(gdr_dtype d) { return d == GDR_F32 || d == GDR_BF16; }

// Which of e1 / e2 a form needs (e2 is optional for GDN-2: the write gate).
bool needs_e1(gdr_form f) { return f != GDR_FORM_GLA; }
bool needs_e2(gdr_form f) { return f == GDR_FORM_GENERAL || f == GDR_FORM_RWKV7; }

gdr_status cuda_status(cudaError_t e) { return e == cudaSuccess ? GDR_OK : GDR_ERR_CUDA; }

// Common pointer checks of the token inputs.  `tokens` = B*T*H (or B*H).
gdr_status check_token_ptrs(gdr_form form, size_t tokens, const void *q, const void *k,
                            const void *v, const float *log_w, const void *e1, const void *e2,
                            const float *o) {
  if (tokens == 0) return GDR_OK;
  if (!q || !k || !v || !log_w || !o) return GDR_ERR_INVALID_ARG;
  if (needs_e1(form) && !e1) return GDR_ERR_INVALID_ARG;
  if (needs_e2(form) && !e2) return GDR_ERR_INVALID_ARG;
  const void *ptrs[] = {q, k, v, log_w, o, e1, e2};
  for (const void *p : ptrs)
    if (p && !aligned16(p)) return GDR_ERR_MISALIGNED;
  return GDR_OK;
}

using gdr::kStatusBytes;

// FwdParams of a forward call (pointers as given).
gdr::FwdParams fwd_params(const gdr_fwd_args *a) {
  gdr::FwdParams p{};
  p.form = a->form;
  p.B = a->B;
  p.H = a->H;
  p.T = a->T;
  p.dk = a->dk;
  p.dv = a->dv;
  p.chunk = a->chunk;
  p.q = a->q;
  p.k = a->k;
  p.v = a->v;
  p.e1 = a->e1;
  p.e2 = a->e2;
  p.log_w = a->log_w;
  p.S0 = a->S0;
  p.o = a->o;
  p.S_T = a->S_T;
  p.status = static_cast<uint32_t *>(a->workspace);
  const char *fault = getenv("GDR_DEBUG_FAULT");
  p.debug = (fault && strcmp(fault, "skip_handoff") == 0) ? gdr::kDebugSkipHandoff : 0u;
#ifdef GDR_PHASE_TIMING
  if (getenv("GDR_TIMING_MMA")) p.debug |= gdr::kDebugTimeMma;
#endif
  return p;
}

bool uses_tc(const gdr_fwd_args *a, const gdr::FwdParams &p) {
  return (a->algo == GDR_ALGO_TC || a->algo == GDR_ALGO_AUTO) &&
         gdr::forward_tc_split_supported(p, a->dtype);
}
bool uses_tc_general(const gdr_fwd_args *a, const gdr::FwdParams &p) {
  return (a->algo == GDR_ALGO_TC || a->algo == GDR_ALGO_AUTO) &&
         gdr::forward_tc_general_supported(p, a->dtype);
}

// Workspace of gdr_muir_forward: the forward's own workspace, then (generic path) the
// activated inputs and o, each section 256-byte aligned.
struct MuirLayout {
  size_t fwd, qh, kh, bh, vh, wh, lw, o, total;
};
size_t align256(size_t x) { return (x + 255) & ~(size_t)255; }

gdr_fwd_args muir_fwd_args(const gdr_muir_args *a) {
  gdr_fwd_args f;
  memset(&f, 0, sizeof(f));
  f.form = GDR_FORM_GDN2;
  f.dtype = a->dtype;
  f.B = a->B;
  f.H = a->H;
  f.T = a->T;
  f.dk = a->dk;
  f.dv = a->dv;
  f.chunk = a->chunk;
  f.algo = a->algo;
  f.S0 = a->S0;
  f.S_T = a->S_T;
  return f;
}

// The fused path: bf16, d_k = d_v = 128, the two-kernel tensor-core forward with the
// mixer's activations in its chunk-parallel kernel.
gdr::FwdParams muir_fused_params(const gdr_muir_args *a) {
  gdr::FwdParams p{};
  p.form = GDR_FORM_GDN2;
  p.B = a->B;
  p.H = a->H;
  p.T = a->T;
  p.dk = a->dk;
  p.dv = a->dv;
  p.chunk = a->chunk;
  p.q = a->q;
  p.k = a->k;
  p.v = a->v;
  p.e1 = a->zb;
  p.e2 = a->zw;
  p.S0 = a->S0;
  p.S_T = a->S_T;
  p.status = static_cast<uint32_t *>(a->workspace);
  p.muir = true;
  p.zf = a->zf;
  p.zq = a->zq;
  p.a_log = a->a_log;
  p.gamma_stat = a->gamma_stat;
  return p;
}
bool muir_fused(const gdr_muir_args *a) {
  return !a->unfused && a->algo != GDR_ALGO_FP32 &&
         gdr::forward_tc_split_supported(muir_fused_params(a), a->dtype);
}

MuirLayout muir_layout(const gdr_muir_args *a) {
  MuirLayout L;
  const size_t n = (size_t)a->B * a->T * a->H, eb = a->dtype == GDR_BF16 ? 2 : 4;
  size_t off = 0;
  if (muir_fused(a)) {
    L.fwd = off; off = align256(off + gdr::forward_tc_split_workspace_bytes(muir_fused_params(a)));
    L.qh = L.kh = L.bh = L.vh = L.wh = L.lw = off;
    L.o = off; off = align256(off + n * a->dv * 4);
    L.total = off;
    return L;
  }
  const gdr_fwd_args f = muir_fwd_args(a);
  size_t fwd = kStatusBytes;
  gdr_forward_workspace_size(&f, &fwd);
  L.fwd = off; off = align256(off + fwd);
  L.qh = off; off = align256(off + n * a->dk * eb);
  L.kh = off; off = align256(off + n * a->dk * eb);
  L.bh = off; off = align256(off + n * a->dk * eb);
  L.vh = off; off = align256(off + n * a->dv * eb);
  L.wh = off; off = align256(off + n * a->dv * eb);
  L.lw = off; off = align256(off + n * a->dk * 4);
  L.o = off; off = align256(off + n * a->dv * 4);
  L.total = off;
  return L;
}

}  // namespace

namespace gdr {

// Host validation and kernel selection of gdr_forward_chunked for a workspace of
// `workspace_bytes` bytes; no CUDA call.
gdr_status forward_plan(const gdr_fwd_args *a, const void *workspace, size_t workspace_bytes,
                        FwdPath *path) {
  if (!a || !path) return GDR_ERR_INVALID_ARG;
  if (!form_ok(a->form) || !dtype_ok(a->dtype)) return GDR_ERR_INVALID_ARG;
  if (a->B < 0 || a->H < 0 || a->T < 0) return GDR_ERR_INVALID_ARG;
  if (!dim_ok(a->dk) || !dim_ok(a->dv) || !chunk_ok(a->chunk)) return GDR_ERR_UNSUPPORTED;
  if (a->algo < GDR_ALGO_AUTO || a->algo > GDR_ALGO_RECURRENT) return GDR_ERR_INVALID_ARG;
  const size_t tokens = (size_t)a->B * a->T * a->H;
  gdr_status st = check_token_ptrs(a->form, tokens, a->q, a->k, a->v, a->log_w, a->e1, a->e2,
                                   a->o);
  if (st != GDR_OK) return st;
  if ((a->S0 && !aligned16(a->S0)) || (a->S_T && !aligned16(a->S_T))) return GDR_ERR_MISALIGNED;
  if (workspace && (reinterpret_cast<uintptr_t>(workspace) & 255u)) return GDR_ERR_MISALIGNED;
  if (a->B == 0 || a->H == 0) {
    *path = FwdPath::kNone;
    return GDR_OK;
  }
  if (a->T == 0) {
    *path = a->S_T ? FwdPath::kCopyState : FwdPath::kNone;
    return GDR_OK;
  }
  const FwdParams p = fwd_params(a);
  if (a->algo == GDR_ALGO_RECURRENT) {
    if (!forward_recur_supported(a->dk, a->dv)) return GDR_ERR_UNSUPPORTED;
    *path = FwdPath::kRecur;   // needs no workspace
    return GDR_OK;
  }
  if (uses_tc_general(a, p)) {   // two-stream forms, d = 64: one fused kernel, status word only
    if (workspace_bytes < kStatusBytes) return GDR_ERR_WORKSPACE;
    *path = FwdPath::kTcGeneral;
    return GDR_OK;
  }
  const bool tc_ok = forward_tc_split_supported(p, a->dtype);
  if (a->algo == GDR_ALGO_TC || (a->algo == GDR_ALGO_AUTO && tc_ok)) {
    if (!tc_ok) return GDR_ERR_UNSUPPORTED;
    if (workspace_bytes < kStatusBytes) return GDR_ERR_WORKSPACE;
    // the two-kernel path when the workspace holds its per-chunk records, else the
    // single-kernel path (status word only; GDN-2 alone)
    if (workspace_bytes >= forward_tc_split_workspace_bytes(p)) {
      *path = FwdPath::kTcSplit;
      return GDR_OK;
    }
    if (forward_tc_supported(p, a->dtype)) {
      *path = FwdPath::kTcSingle;
      return GDR_OK;
    }
    if (a->algo == GDR_ALGO_TC) return GDR_ERR_WORKSPACE;
  }
  // AUTO without a tensor-core path: the token recurrence, which ran faster than the fp32
  // chunkwise kernel on every shape measured (that kernel stays behind GDR_ALGO_FP32)
  if (a->algo == GDR_ALGO_AUTO && forward_recur_supported(a->dk, a->dv)) {
    *path = FwdPath::kRecur;
    return GDR_OK;
  }
  if (!forward_fp32_supported(a->dk, a->dv)) return GDR_ERR_UNSUPPORTED;
  *path = FwdPath::kFp32;     // needs no workspace (a status word is used when given)
  return GDR_OK;
}

}  // namespace gdr

extern "C" {

const char *gdr_status_string(gdr_status s) {
  switch (s) {
    case GDR_OK: return "ok";
    case GDR_ERR_INVALID_ARG: return "invalid argument";
    case GDR_ERR_UNSUPPORTED: return "unsupported size or form";
    case GDR_ERR_MISALIGNED: return "pointer not 16-byte aligned";
    case GDR_ERR_CUDA: return "CUDA runtime or launch error";
    case GDR_ERR_DEVICE_CHECK: return "device-side check failed";
    case GDR_ERR_TIMEOUT: return "bounded device wait ran out";
    case GDR_ERR_WORKSPACE: return "workspace missing or too small";
  }
  return "unknown status";
}

int gdr_version(void) { return 100; }

gdr_status gdr_forward_workspace_size(const gdr_fwd_args *a, size_t *bytes) {
  if (!a || !bytes) return GDR_ERR_INVALID_ARG;
  *bytes = kStatusBytes;
  if (a->B > 0 && a->H > 0 && a->T > 0 && dtype_ok(a->dtype) && form_ok(a->form)) {
    const gdr::FwdParams p = fwd_params(a);
    if (uses_tc(a, p)) *bytes = gdr::forward_tc_split_workspace_bytes(p);
  }
  return GDR_OK;
}

gdr_status gdr_state_init(float *S, int B, int H, int dk, int dv, const float *src,
                          void *stream) {
  if (B < 0 || H < 0 || !dim_ok(dk) || !dim_ok(dv)) return GDR_ERR_INVALID_ARG;
  const size_t n = (size_t)B * H * dk * dv;
  if (n == 0) return GDR_OK;
  if (!S) return GDR_ERR_INVALID_ARG;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (src) {
    if (src == S) return GDR_OK;
    return cuda_status(cudaMemcpyAsync(S, src, n * sizeof(float), cudaMemcpyDeviceToDevice, st));
  }
  return cuda_status(cudaMemsetAsync(S, 0, n * sizeof(float), st));
}

gdr_status gdr_forward_kernel_name(const gdr_fwd_args *a, const char **name) {
  if (!name) return GDR_ERR_INVALID_ARG;
  gdr::FwdPath path;
  const gdr_status st = gdr::forward_plan(a, a ? a->workspace : nullptr, a ? a->workspace_bytes : 0,
                                          &path);
  if (st != GDR_OK) return st;
  switch (path) {
    case gdr::FwdPath::kNone: *name = "none"; break;
    case gdr::FwdPath::kCopyState: *name = "copy_state"; break;
    case gdr::FwdPath::kTcGeneral: *name = "tc_two_stream"; break;
    case gdr::FwdPath::kTcSplit: *name = "tc_split"; break;
    case gdr::FwdPath::kTcSingle: *name = "tc_single"; break;
    case gdr::FwdPath::kRecur: *name = "recurrent"; break;
    default: *name = "fp32"; break;
  }
  return GDR_OK;
}

gdr_status gdr_forward_chunked(const gdr_fwd_args *a, void *stream) {
  gdr::FwdPath path;
  const gdr_status st = gdr::forward_plan(a, a ? a->workspace : nullptr, a ? a->workspace_bytes : 0,
                                          &path);
  if (st != GDR_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  switch (path) {
    case gdr::FwdPath::kNone:
      return GDR_OK;
    case gdr::FwdPath::kCopyState:   // no tokens: S_T = S0
      return gdr_state_init(a->S_T, a->B, a->H, a->dk, a->dv, a->S0, stream);
    default:
      break;
  }
  if (path != gdr::FwdPath::kFp32 && path != gdr::FwdPath::kRecur && !a->workspace)
    return GDR_ERR_WORKSPACE;
  const gdr::FwdParams p = fwd_params(a);
  switch (path) {
    case gdr::FwdPath::kTcGeneral: return cuda_status(gdr::launch_forward_tc_general(p, s));
    case gdr::FwdPath::kTcSplit: return cuda_status(gdr::launch_forward_tc_split(p, a->workspace, s));
    case gdr::FwdPath::kTcSingle: return cuda_status(gdr::launch_forward_tc(p, s));
    case gdr::FwdPath::kRecur: return cuda_status(gdr::launch_forward_recur(p, a->dtype, s));
    default: return cuda_status(gdr::launch_forward_fp32(p, a->dtype, s));
  }
}

gdr_status gdr_decode_step(const gdr_step_args *a, void *stream) {
  if (!a) return GDR_ERR_INVALID_ARG;
  if (!form_ok(a->form) || !dtype_ok(a->dtype)) return GDR_ERR_INVALID_ARG;
  if (a->B < 0 || a->H < 0) return GDR_ERR_INVALID_ARG;
  if (!dim_ok(a->dk) || !dim_ok(a->dv)) return GDR_ERR_UNSUPPORTED;
  const size_t tokens = (size_t)a->B * a->H;
  gdr_status st = check_token_ptrs(a->form, tokens, a->q, a->k, a->v, a->log_w, a->e1, a->e2,
                                   a->o);
  if (st != GDR_OK) return st;
  if (tokens == 0) return GDR_OK;
  if (!a->S) return GDR_ERR_INVALID_ARG;
  if (!aligned16(a->S)) return GDR_ERR_MISALIGNED;
  return cuda_status(gdr::launch_decode(*a, static_cast<cudaStream_t>(stream)));
}

gdr_status gdr_backward_workspace_size(const gdr_bwd_args *a, size_t *bytes) {
  if (!a || !bytes) return GDR_ERR_INVALID_ARG;
  *bytes = kStatusBytes;
  if (a->B > 0 && a->H > 0 && a->T > 0 && form_ok(a->form) && gdr::backward_supported(a->dk, a->dv))
    *bytes = gdr::backward_workspace_bytes(a->form, a->B, a->H, a->T, a->dk, a->dv);
  return GDR_OK;
}

gdr_status gdr_backward_chunked(const gdr_bwd_args *a, void *stream) {
  if (!a) return GDR_ERR_INVALID_ARG;
  if (!form_ok(a->form) || !dtype_ok(a->dtype)) return GDR_ERR_INVALID_ARG;
  if (a->B < 0 || a->H < 0 || a->T < 0) return GDR_ERR_INVALID_ARG;
  if (!chunk_ok(a->chunk)) return GDR_ERR_UNSUPPORTED;
  if (!dim_ok(a->dk) || !dim_ok(a->dv)) return GDR_ERR_UNSUPPORTED;
  if (!gdr::backward_supported(a->dk, a->dv)) return GDR_ERR_UNSUPPORTED;
  const size_t tokens = (size_t)a->B * a->T * a->H;
  gdr_status st = check_token_ptrs(a->form, tokens, a->q, a->k, a->v, a->log_w, a->e1, a->e2,
                                   a->dO);
  if (st != GDR_OK) return st;
  if (tokens > 0) {
    if (!a->g_q || !a->g_k || !a->g_v || !a->g_log_w) return GDR_ERR_INVALID_ARG;
    if (needs_e1(a->form) && !a->g_e1) return GDR_ERR_INVALID_ARG;
    if (a->e2 && a->form != GDR_FORM_GLA && !a->g_e2) return GDR_ERR_INVALID_ARG;
  }
  const void *outs[] = {a->S0, a->dS_T, a->g_q, a->g_k, a->g_v, a->g_log_w, a->g_e1, a->g_e2,
                        a->g_S0};
  for (const void *p : outs)
    if (p && !aligned16(p)) return GDR_ERR_MISALIGNED;
  if (a->B == 0 || a->H == 0) return GDR_OK;
  if (a->T == 0) {  // no tokens: dL/dS0 = dS_T
    if (!a->g_S0) return GDR_OK;
    return gdr_state_init(a->g_S0, a->B, a->H, a->dk, a->dv, a->dS_T, stream);
  }
  const size_t need = gdr::backward_workspace_bytes(a->form, a->B, a->H, a->T, a->dk, a->dv);
  if (!a->workspace || a->workspace_bytes < need) return GDR_ERR_WORKSPACE;
  if (reinterpret_cast<uintptr_t>(a->workspace) & 255u) return GDR_ERR_MISALIGNED;
  gdr::BwdParams p;
  memset(&p, 0, sizeof(p));
  p.form = a->form;
  p.B = a->B;
  p.H = a->H;
  p.T = a->T;
  p.dk = a->dk;
  p.dv = a->dv;
  p.q = a->q;
  p.k = a->k;
  p.v = a->v;
  p.e1 = a->e1;
  p.e2 = a->form == GDR_FORM_GLA ? nullptr : a->e2;
  p.log_w = a->log_w;
  p.S0 = a->S0;
  p.dO = a->dO;
  p.dS_T = a->dS_T;
  p.gq = a->g_q;
  p.gk = a->g_k;
  p.gv = a->g_v;
  p.glw = a->g_log_w;
  p.ge1 = a->g_e1;
  p.ge2 = a->g_e2;
  p.gS0 = a->g_S0;
  return cuda_status(gdr::launch_backward(p, a->dtype, a->workspace,
                                          static_cast<cudaStream_t>(stream)));
}

gdr_status gdr_muir_workspace_size(const gdr_muir_args *a, size_t *bytes) {
  if (!a || !bytes) return GDR_ERR_INVALID_ARG;
  *bytes = kStatusBytes;
  if (a->B > 0 && a->H > 0 && a->T > 0 && dtype_ok(a->dtype) && dim_ok(a->dk) && dim_ok(a->dv))
    *bytes = muir_layout(a).total;
  return GDR_OK;
}

gdr_status gdr_muir_forward(const gdr_muir_args *a, void *stream) {
  if (!a) return GDR_ERR_INVALID_ARG;
  if (!dtype_ok(a->dtype)) return GDR_ERR_INVALID_ARG;
  if (a->B < 0 || a->H < 0 || a->T < 0) return GDR_ERR_INVALID_ARG;
  if (!dim_ok(a->dk) || !dim_ok(a->dv) || !chunk_ok(a->chunk)) return GDR_ERR_UNSUPPORTED;
  if (a->algo < GDR_ALGO_AUTO || a->algo > GDR_ALGO_TC) return GDR_ERR_INVALID_ARG;
  if (!(a->rms_eps >= 0.f)) return GDR_ERR_INVALID_ARG;
  const size_t tokens = (size_t)a->B * a->T * a->H;
  if (tokens > 0) {
    const void *need[] = {a->q, a->k, a->v, a->zf, a->zb, a->zw, a->zq, a->zg, a->a_log, a->y};
    for (const void *p : need)
      if (!p) return GDR_ERR_INVALID_ARG;
    const void *al[] = {a->q, a->k, a->v, a->zf, a->zb, a->zw, a->zq, a->zg, a->y};
    for (const void *p : al)
      if (!aligned16(p)) return GDR_ERR_MISALIGNED;
  }
  if ((a->S0 && !aligned16(a->S0)) || (a->S_T && !aligned16(a->S_T))) return GDR_ERR_MISALIGNED;
  if ((a->gamma_stat && !aligned16(a->gamma_stat)) || (a->rms_weight && !aligned16(a->rms_weight)))
    return GDR_ERR_MISALIGNED;
  if (a->B == 0 || a->H == 0) return GDR_OK;
  if (a->T == 0) {
    if (!a->S_T) return GDR_OK;
    return gdr_state_init(a->S_T, a->B, a->H, a->dk, a->dv, a->S0, stream);
  }
  const MuirLayout L = muir_layout(a);
  if (!a->workspace || a->workspace_bytes < L.total) return GDR_ERR_WORKSPACE;
  if (reinterpret_cast<uintptr_t>(a->workspace) & 255u) return GDR_ERR_MISALIGNED;
  uint8_t *ws = static_cast<uint8_t *>(a->workspace);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  gdr::MuirParams m;
  m.B = a->B;
  m.H = a->H;
  m.T = a->T;
  m.dk = a->dk;
  m.dv = a->dv;
  m.q = a->q;
  m.k = a->k;
  m.v = a->v;
  m.zf = a->zf;
  m.zb = a->zb;
  m.zw = a->zw;
  m.zq = a->zq;
  m.zg = a->zg;
  m.a_log = a->a_log;
  m.gamma_stat = a->gamma_stat;
  m.rms_weight = a->rms_weight;
  m.rms_eps = a->rms_eps;
  float *o = reinterpret_cast<float *>(ws + L.o);
  if (muir_fused(a)) {   // activations inside the forward's chunk-parallel kernel, then the readout
    gdr::FwdParams p = muir_fused_params(a);
    p.o = o;
    gdr_status st = cuda_status(gdr::launch_forward_tc_split(p, ws + L.fwd, s));
    if (st != GDR_OK) return st;
    return cuda_status(gdr::launch_muir_epilogue(m, a->dtype, o, a->y, s));
  }
  // activated inputs, then the GDN-2 forward on them, then the readout
  gdr_status st = cuda_status(gdr::launch_muir_prologue(
      m, a->dtype, ws + L.qh, ws + L.kh, ws + L.vh, ws + L.bh, ws + L.wh,
      reinterpret_cast<float *>(ws + L.lw), s));
  if (st != GDR_OK) return st;
  gdr_fwd_args f = muir_fwd_args(a);
  f.q = ws + L.qh;
  f.k = ws + L.kh;
  f.v = ws + L.vh;
  f.log_w = reinterpret_cast<const float *>(ws + L.lw);
  f.e1 = ws + L.bh;
  f.e2 = ws + L.wh;
  f.o = o;
  f.workspace = ws + L.fwd;
  f.workspace_bytes = L.qh - L.fwd;
  st = gdr_forward_chunked(&f, stream);
  if (st != GDR_OK) return st;
  return cuda_status(gdr::launch_muir_epilogue(m, a->dtype, o, a->y, s));
}

gdr_status gdr_mlstm_forward(const gdr_mlstm_args *a, void *stream) {
  if (!a) return GDR_ERR_INVALID_ARG;
  if (!dtype_ok(a->dtype)) return GDR_ERR_INVALID_ARG;
  if (a->B < 0 || a->H < 0 || a->T < 0) return GDR_ERR_INVALID_ARG;
  if ((a->dk != 64 && a->dk != 128) || (a->dv != 64 && a->dv != 128)) return GDR_ERR_UNSUPPORTED;
  const size_t tokens = (size_t)a->B * a->T * a->H;
  if (tokens > 0 && (!a->q || !a->k || !a->v || !a->f_pre || !a->i_pre || !a->h))
    return GDR_ERR_INVALID_ARG;
  // the state comes whole or not at all
  if ((a->C0 != nullptr) != (a->n0 != nullptr) || (a->C0 != nullptr) != (a->m0 != nullptr))
    return GDR_ERR_INVALID_ARG;
  const void *al[] = {a->q, a->k, a->v, a->h, a->C0, a->C_T};
  for (const void *p : al)
    if (p && !aligned16(p)) return GDR_ERR_MISALIGNED;
  if (a->B == 0 || a->H == 0) return GDR_OK;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (a->T == 0) {   // no tokens: the final state is the initial one (empty: zeros, m = -inf)
    const size_t nbh = (size_t)a->B * a->H;
    if (a->C_T) {
      gdr_status st = gdr_state_init(a->C_T, a->B, a->H, a->dk, a->dv, a->C0, stream);
      if (st != GDR_OK) return st;
    }
    if (a->n_T) {
      cudaError_t e = a->n0 ? cudaMemcpyAsync(a->n_T, a->n0, nbh * a->dk * 4, cudaMemcpyDeviceToDevice, s)
                            : cudaMemsetAsync(a->n_T, 0, nbh * a->dk * 4, s);
      if (e != cudaSuccess) return GDR_ERR_CUDA;
    }
    if (a->m_T) {
      if (a->m0) return cuda_status(cudaMemcpyAsync(a->m_T, a->m0, nbh * 4, cudaMemcpyDeviceToDevice, s));
      return cuda_status(gdr::fill_f32(a->m_T, nbh, -INFINITY, s));
    }
    return GDR_OK;
  }
  return cuda_status(gdr::launch_mlstm(*a, s));
}

gdr_status gdr_state_compose(float *S_out, const float *M, const float *S_in, const float *Q,
                             int BH, int dk, int dv, void *stream) {
  if (BH < 0 || !dim_ok(dk) || !dim_ok(dv)) return GDR_ERR_INVALID_ARG;
  if (BH == 0) return GDR_OK;
  if (!S_out || !M) return GDR_ERR_INVALID_ARG;
  if (S_in && S_in == S_out) return GDR_ERR_INVALID_ARG;
  return cuda_status(gdr::launch_state_compose(S_out, M, S_in, Q, BH, dk, dv,
                                               static_cast<cudaStream_t>(stream)));
}

gdr_status gdr_read_status(void *workspace, void *stream, gdr_status *device_status) {
  if (!workspace || !device_status) return GDR_ERR_INVALID_ARG;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (cudaStreamSynchronize(s) != cudaSuccess) return GDR_ERR_CUDA;
  uint32_t word = 0;
  if (cudaMemcpy(&word, workspace, sizeof(word), cudaMemcpyDeviceToHost) != cudaSuccess)
    return GDR_ERR_CUDA;
  if (cudaMemset(workspace, 0, sizeof(word)) != cudaSuccess) return GDR_ERR_CUDA;
  *device_status = static_cast<gdr_status>(word);
  return GDR_OK;
}

}  // extern "C"
