/*
 * gdr.h -- C ABI of libgdr: the generalized delta-rule matrix memory on B200.
 *
 * The recurrence (column form; the state S is d_v x d_k):
 *
 *     e_t = S_{t-1} u_t
 *     S_t = S_{t-1} Diag(w_t) - e_t z_t^T + v_t k_t^T  = S_{t-1}(Diag(w_t) - u_t z_t^T) + v_t k_t^T
 *     o_t = S_t q_t                                      (readout after the update)
 *
 * Sources:
 *  - "Exponential gates and matrix memory: xLSTM and RWKV-7", section 13.3
 *    (the generalized delta rule S_t = S_{t-1}(Diag(w_t) - c_t a_t a_t^T) + u_t b_t^T,
 *    retrieval by S q with the transition acting on the right), section 13.1
 *    (the generalized transition Diag(w) - c a a^T with a unit a).
 *  - "Muir: Linear Attention with Sensitivity-Allocated Gating and Matched-Filter
 *    Readout", section 2.1 eq. (1) (GDN-2 update with channel-wise decay alpha,
 *    erase gate b, write gate w) and section 4.2 eq. (8) (Muir readout with the
 *    gain-modulated query); section 2.2 and section 4.2 eq. (10) give the chunkwise
 *    form that gdr_forward_chunked evaluates.
 *
 * Storage orientation.  Every state buffer is stored as [B][H][d_k][d_v] fp32,
 * row-major: element (j, c) is key channel j, value channel c.  That is the Muir
 * page's orientation (S in R^{d_k x d_v}, row vectors, o = q S), i.e. the transpose
 * of the column form above.  Both describe the same numbers.
 *
 * Forms (how u_t and z_t are built from the arguments e1, e2; w_t = exp(log_w_t)):
 *   GDR_FORM_GENERAL : e1 = u [.., d_k], e2 = z [.., d_k]; write (v, k).
 *   GDR_FORM_GDN2    : e1 = b erase gate [.., d_k]; e2 = write gate wg [.., d_v] or NULL (= 1).
 *                      u = alpha (.) b (.) k, z = k; written value wg (.) v with key k.
 *                      (Muir eq. (1)/(8) transposed: the erase acts on the decayed state
 *                      Diag(alpha) S_{t-1}, which is why alpha is folded into u.)
 *                      For Muir pass q_hat = gamma (.) q as q.
 *   GDR_FORM_RWKV7   : e1 = a unit removal direction [.., d_k]; e2 = c removal coefficient,
 *                      one scalar per (b, t, h), i.e. [B][T][H]; u = c a, z = a; write (v, k).
 *                      (the chapter's u_t b_t^T write is passed here as v = u_t, k = b_t.)
 *   GDR_FORM_GLA     : u = 0 (gated linear attention); e1 = e2 = NULL.
 *
 * Memory and ownership.  The caller owns every buffer; pointers are device
 * pointers unless stated otherwise.  libgdr allocates no device memory, keeps no
 * global state between calls (apart from the fixed scratch array behind
 * gdr_forward_chunked_noalloc), and never synchronizes the stream except where a
 * function says so.  Everything is enqueued asynchronously on the given stream
 * (a cudaStream_t passed as void*, NULL = legacy default stream).
 *
 * Errors.  Every function returns a gdr_status.  Invalid arguments are rejected on
 * the host before any launch.  Launch failures come back as GDR_ERR_CUDA.  Faults
 * that happen later on the device surface at the caller's next synchronization.
 * Kernels that wait on an mbarrier bound each wait; a wait that runs out writes
 * GDR_ERR_TIMEOUT into the caller's workspace status word, which
 * gdr_read_status() returns.  No function aborts, exits or traps.
 * For tests of that path, the environment variable GDR_DEBUG_FAULT=skip_handoff
 * makes the two-kernel tensor-core forward withhold a hand-off between its warp
 * groups (the single-kernel forward and the tcgen05 mLSTM kernel the completion
 * signal of one product), so a bounded wait runs out (about 2 s) and GDR_ERR_TIMEOUT
 * is reported; the context stays usable.
 */
#ifndef GDR_H_
#define GDR_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  GDR_OK = 0,
  GDR_ERR_INVALID_ARG = 1,   /* null pointer where one is required, negative size, bad enum */
  GDR_ERR_UNSUPPORTED = 2,   /* a size or form this build has no kernel for (see each call) */
  GDR_ERR_MISALIGNED = 3,    /* a pointer is not 16-byte aligned                            */
  GDR_ERR_CUDA = 4,          /* a CUDA runtime call or a launch failed                       */
  GDR_ERR_DEVICE_CHECK = 5,  /* a device-side argument check failed (read via gdr_read_status) */
  GDR_ERR_TIMEOUT = 6,       /* a bounded device wait ran out (read via gdr_read_status)       */
  GDR_ERR_WORKSPACE = 7      /* workspace missing or smaller than gdr_forward_workspace_size   */
} gdr_status;

typedef enum { GDR_F32 = 0, GDR_BF16 = 1 } gdr_dtype;

typedef enum {
  GDR_FORM_GENERAL = 0,
  GDR_FORM_GDN2 = 1,
  GDR_FORM_RWKV7 = 2,
  GDR_FORM_GLA = 3
} gdr_form;

/* Kernel selection for gdr_forward_chunked. */
typedef enum {
  GDR_ALGO_AUTO = 0,   /* tensor-core kernel where it applies, else the token-recurrent
                          kernel (measured faster than the fp32 chunkwise kernel on every
                          fp32 shape tried, from B=1, H=2, T=256 to B=8, H=32, T=2048)      */
  GDR_ALGO_FP32 = 1,   /* fp32 CUDA-core kernel: every product in fp32 (all forms, all dtypes) */
  GDR_ALGO_TC = 2,     /* tcgen05/TMEM kernels: bf16 operands, fp32 accumulate and state.
                          They apply to bf16 inputs with chunk >= 64 for
                            GDN2, dk = dv = 128: two kernels with a per-chunk record
                                 workspace, or one kernel with the status word only;
                            GLA, dk = dv = 128: the two kernels (GDR_ERR_WORKSPACE
                                 without the record workspace; AUTO then takes the
                                 token-recurrent kernel);
                            every form, dk = dv = 64: one kernel, status word only;
                          GDR_ERR_UNSUPPORTED elsewhere.                                  */
  GDR_ALGO_RECURRENT = 3  /* the recurrence token by token (fp32 state in registers, one warp
                          per value column; all forms, dtypes and sizes; no workspace).  No
                          chunk parallelism: its time grows with T at a fixed cost per token,
                          which for few heads and short sequences is far below the chunkwise
                          kernels' cost per chunk.  The chunk length is ignored.        */
} gdr_algo;

/*
 * Arguments of gdr_forward_chunked.  Shapes are token-major and contiguous:
 *   q, k, log_w, and e1 for GENERAL/GDN2/RWKV7 : [B][T][H][dk]
 *   v, o, and e2 for GDN2                      : [B][T][H][dv]
 *   e2 for GENERAL                             : [B][T][H][dk]
 *   e2 for RWKV7                               : [B][T][H]
 *   S0, S_T                                    : [B][H][dk][dv]
 * q, k, v, e1, e2 have element type `dtype`; log_w, S0, S_T, o are fp32.
 */
typedef struct {
  gdr_form form;
  gdr_dtype dtype;
  int B, H, T, dk, dv;  /* B, H, T >= 0 (zero sizes are a no-op apart from S_T = S0);
                           dk, dv in {16, 32, 64, 128}                                  */
  int chunk;            /* chunk length C of the chunkwise form: 16, 32, 64 or 128.
                           T need not be a multiple of C (the last chunk is partial).
                           The kernels may split a chunk further: the fp32 kernel uses
                           min(C, 64, 4096 / dk), the tensor-core kernels 64 for C >= 64.
                           The result depends on the chunk length only through rounding. */
  gdr_algo algo;
  const void *q, *k, *v;
  const float *log_w;   /* log of the decay, must be <= 0 (decay w = exp(log_w) in (0,1]) */
  const void *e1, *e2;  /* per form, above                                             */
  const float *S0;      /* initial state, or NULL for S0 = 0                           */
  float *o;             /* outputs o_t, required                                       */
  float *S_T;           /* final state, or NULL; may alias S0 (read before written)    */
  void *workspace;      /* device scratch of gdr_forward_workspace_size bytes, 256-B aligned */
  size_t workspace_bytes;
} gdr_fwd_args;

/* Workspace bytes gdr_forward_chunked needs for these arguments (host-only, no CUDA call). */
gdr_status gdr_forward_workspace_size(const gdr_fwd_args *args, size_t *bytes);

/*
 * Which kernel gdr_forward_chunked runs for these arguments, workspace included (host-only:
 * no CUDA call and no pointer dereferenced; the same checks, so a call it rejects returns the
 * same status).  *name is a
 * static string: "none" (no work), "copy_state" (T = 0: S_T = S0), "tc_two_stream" (every
 * form at d = 64 on tcgen05), "tc_split" (prep and chain kernels with per-chunk records),
 * "tc_single" (one tensor-core kernel), "fp32" (the fp32 chunkwise kernel) or "recurrent"
 * (the token-recurrent kernel).
 */
gdr_status gdr_forward_kernel_name(const gdr_fwd_args *args, const char **name);

/*
 * Chunkwise-parallel forward over whole sequences: for every (b, h) runs the
 * recurrence over t = 1..T from S0 and writes every o_t and, if S_T != NULL, the
 * final state.  Chunkwise algorithm: "Muir ...", section 2.2 (effective write,
 * the unit lower-triangular system T V~ = V^ - K^_pi S0, S_C and O as matrix
 * products) and section 4.2 eq. (10) (outputs and end state affine in S0),
 * generalized to a separate erase key z (e_t and v_t carried as two write streams).
 * Cumulative decays are formed in log space and exponentiated only as differences:
 * the fp32 kernel at non-positive arguments; the tensor-core kernel splits each
 * pairwise decay at the chunk's first token, with both exponents bounded by 80
 * (checked per chunk and channel; a chunk that decays more forms its products from
 * the exact pairwise decays) -- the role section 4.2's boundary pivots play on the
 * Muir page.  No factor is divided out and nothing overflows.
 */
gdr_status gdr_forward_chunked(const gdr_fwd_args *args, void *stream);

/*
 * gdr_forward_chunked for callers that cannot allocate device memory.  (No
 * counterpart in the papers: this is a deployment convenience.)
 *
 * Some callers are not allowed to allocate: a plugin whose host application owns
 * every device allocation, a serving loop that forbids allocation once its memory
 * plan is fixed, code where cudaMalloc is unavailable or would synchronize.  This
 * call ignores args->workspace / workspace_bytes and uses a fixed scratch array
 * compiled into libgdr instead (a static __device__ array of 4096 bytes that every
 * GPU loading the library holds until process exit).  It calls no cudaMalloc,
 * cudaFree or other allocating routine.
 *
 * Kernels.  The array holds only the status word, so the call takes the paths of
 * gdr_forward_chunked that need no per-chunk records:
 *   - GDN2, bf16, dk = dv = 128, algo AUTO or TC: the single-kernel tensor-core
 *     forward (not the faster two-kernel one, whose records do not fit);
 *   - GLA, bf16, dk = dv = 128: algo TC returns GDR_ERR_WORKSPACE; algo AUTO runs
 *     the token-recurrent kernel;
 *   - every form at bf16, dk = dv = 64, algo AUTO or TC: the two-stream
 *     tensor-core kernel, as gdr_forward_chunked;
 *   - everything else: algo FP32 the fp32 chunkwise kernel, algo AUTO or RECURRENT
 *     (fp32 inputs, other sizes) the token-recurrent kernel, as gdr_forward_chunked.
 * The results are those of the kernel named, within the same error bars.
 *
 *   - Arguments are checked on the host, as gdr_forward_chunked checks them, before
 *     anything is enqueued.
 *   - The array's device address is looked up (cudaGetSymbolAddress, with the
 *     device current) on a device's first call and cached with the id of the CUDA
 *     context it belongs to; a call in another context (after cudaDeviceReset, or
 *     once the primary context was released and created again) looks it up anew.
 *     Make the first call of each context before any stream capture.
 *   - All calls share the one array; calls that overlap on the GPU (different
 *     streams, or different host threads on the same device) race on it.
 *     Serialize them.
 *   - The array keeps the last call's contents; each call clears the status word
 *     it uses on `stream` before the launch.
 *   - The device status word lives in the library's array: read it with
 *     gdr_noalloc_read_status (below), not gdr_read_status.
 * Errors and all other arguments: as gdr_forward_chunked.
 */
gdr_status gdr_forward_chunked_noalloc(const gdr_fwd_args *args, void *stream);

/*
 * The device status word of gdr_forward_chunked_noalloc on the current device: waits for
 * `stream` (cudaStreamSynchronize), copies the word from the library's array to
 * *device_status (GDR_OK, or GDR_ERR_TIMEOUT after a bounded wait of a kernel ran out)
 * and clears it, as gdr_read_status does for a caller's workspace.  Allocates nothing.
 * Returns GDR_ERR_INVALID_ARG for a NULL device_status, GDR_ERR_CUDA if a CUDA call fails.
 */
gdr_status gdr_noalloc_read_status(void *stream, gdr_status *device_status);

/*
 * Arguments of gdr_backward_chunked: the forward's inputs plus the loss gradient.
 * With L the caller's loss, dO = dL/do [B][T][H][dv] fp32 (required) and
 * dS_T = dL/dS_T [B][H][dk][dv] fp32 (NULL = 0).  Outputs g_x = dL/dx, all fp32,
 * each the full gradient (overwritten, not accumulated):
 *   g_q, g_k, g_log_w : [B][T][H][dk]          g_v : [B][T][H][dv]
 *   g_e1              : shaped like e1 (GENERAL, GDN2, RWKV7; NULL for GLA)
 *   g_e2              : shaped like e2 (GENERAL; RWKV7 [B][T][H]; GDN2 when e2 != NULL)
 *   g_S0              : [B][H][dk][dv], or NULL when not wanted
 * GDN2's gradients are those of its raw arguments (k receives the write, erase-key
 * and erase-vector terms; log_w includes alpha's share in u); RWKV7's those of a
 * and c.  dtype, shapes and forms as in gdr_fwd_args; dk, dv in {64, 128}.
 */
typedef struct {
  gdr_form form;
  gdr_dtype dtype;
  int B, H, T, dk, dv;
  int chunk;            /* accepted values as gdr_fwd_args; the kernels use 32-token
                           chunks whatever is passed (the result depends on it only
                           through rounding)                                          */
  const void *q, *k, *v;
  const float *log_w;
  const void *e1, *e2;
  const float *S0;      /* initial state of the forward, or NULL (= 0)                */
  const float *dO;
  const float *dS_T;
  float *g_q, *g_k, *g_v, *g_log_w, *g_e1, *g_e2, *g_S0;
  void *workspace;      /* device scratch of gdr_backward_workspace_size bytes, 256-B aligned */
  size_t workspace_bytes;
} gdr_bwd_args;

/* Workspace bytes gdr_backward_chunked needs (host-only, no CUDA call).  About
 * (2 dk dv / 32 + 5 dk) * 4 bytes per token and head: the chunk-start states, their
 * adjoints and the per-chunk records of the two chains. */
gdr_status gdr_backward_workspace_size(const gdr_bwd_args *args, size_t *bytes);

/*
 * Reverse mode of gdr_forward_chunked: every gradient of L = <dO, o> + <dS_T, S_T>.
 * Chunkwise adjoint of the same algebra ("Muir ...", section 2.2 and section 4.2
 * eq. (10): outputs and end state are affine in the chunk's start state, so the
 * adjoint of the start state is the same affine map transposed, carried backwards
 * over the chunks).  Per 32-token chunk, with W = T^-1 U~ and the decayed keys
 * K~, Z~ of the forward:
 *     S_end   = Diag(pi) S - Z~^T (W S) + (K~ - (T^-1 B)^T Z~)^T V      (forward chain)
 *     dS      = Diag(pi) dS_end - W^T (Z~ dS_end) + (Q~ - M_z W)^T dO    (adjoint chain)
 * and the token gradients follow chunk-parallel from S and dS_end by the adjoints
 * of E = T^-1 (U~ S + B V), O = Q~ S + M_k V - M_z E, S_end = Diag(pi) S + K~^T V - Z~^T E.
 * The decay gradient is a reverse cumulative sum over the sequence:
 *     dlog_w_t = sum_{r >= t} (q dq - k dk - z dz + u du)_r - u_t du_t + diag(S_T^T dS_T)
 * (effective u, z, k of the form; for GDN2 the last two terms cancel the share of
 * alpha in u).  Products on the tensor cores (tf32 operands with fp32 accumulate;
 * bf16 inputs use one tf32 product, fp32 inputs three, which keeps fp32 accuracy).
 * Four kernels, no device waits.  Errors as gdr_forward_chunked; GDR_ERR_UNSUPPORTED
 * for dk or dv outside {64, 128}; GDR_ERR_WORKSPACE when the workspace is missing
 * or too small.
 */
gdr_status gdr_backward_chunked(const gdr_bwd_args *args, void *stream);

/*
 * Arguments of gdr_muir_forward: the Muir token mixer around the GDN-2 recurrence
 * ("Muir ...", section 2.1 and section 4.1, eqs. (8)-(9)), from the activations that
 * leave the projections and the depthwise causal convolution:
 *   q, k, zf, zb, zq : [B][T][H][dk]      v, zw, zg : [B][T][H][dv]     (element type dtype)
 *   a_log            : [H] fp32, the per-head log decay rate
 *   gamma_stat       : [H][dk] fp32 static readout gain, or NULL (= 1)
 *   rms_weight       : [dv] fp32 RMSNorm weight shared by the heads, or NULL (= 1)
 *   y                : [B][T][H][dv] fp32, required;  S0, S_T as gdr_fwd_args
 * It computes, per token and head,
 *   q^ = gamma_stat (.) 2 sigmoid(zq) (.) l2norm(silu(q)),  k^ = l2norm(silu(k)),  v^ = silu(v)
 *   log alpha = -exp(a_log) softplus(zf),  b = 2 sigmoid(zb),  w = sigmoid(zw)
 *   o = the GDN-2 recurrence on (q^, k^, v^, log alpha, b, w)   (as gdr_forward_chunked)
 *   y = rms_weight (.) o / sqrt(mean_c o_c^2 + rms_eps) (.) silu(zg)
 * with l2norm(x) = x / max(||x||_2, 1e-12).  Every array pointer, gamma_stat and
 * rms_weight included, must be 16-byte aligned (GDR_ERR_MISALIGNED otherwise).
 */
typedef struct {
  gdr_dtype dtype;
  int B, H, T, dk, dv, chunk;
  gdr_algo algo;
  const void *q, *k, *v;
  const void *zf, *zb, *zw, *zq, *zg;
  const float *a_log;
  const float *gamma_stat;
  const float *rms_weight;
  float rms_eps;
  int unfused;          /* 0: the activations run inside the tensor-core forward where it
                           applies (bf16, dk = dv = 128); 1: always the separate prologue */
  const float *S0;
  float *y;
  float *S_T;
  void *workspace;      /* device scratch of gdr_muir_workspace_size bytes, 256-B aligned */
  size_t workspace_bytes;
} gdr_muir_args;

/* Workspace bytes gdr_muir_forward needs (host-only, no CUDA call). */
gdr_status gdr_muir_workspace_size(const gdr_muir_args *args, size_t *bytes);

/*
 * The Muir mixer above.  Fused (unfused = 0; bf16 inputs, dk = dv = 128, algo AUTO or
 * TC): the activations run inside the tensor-core forward's chunk-parallel kernel, on
 * the tiles it loads (no activated copy of the inputs is written), and one light kernel
 * applies RMSNorm (.) SiLU(zg) to o.  Otherwise a prologue kernel writes the activated
 * inputs into the workspace, gdr_forward_chunked runs on them, and the same epilogue
 * follows.  Errors as gdr_forward_chunked.
 */
gdr_status gdr_muir_forward(const gdr_muir_args *args, void *stream);

/*
 * Arguments of gdr_mlstm_forward: xLSTM's mLSTM cell ("Exponential gates and matrix
 * memory: xLSTM and RWKV-7", section 13.4 and the solution to Exercise 13.6).
 *   q, k : [B][T][H][dk]    v : [B][T][H][dv]    (element type dtype)
 *   f_pre, i_pre : [B][T][H] fp32, forget and input gate pre-activations f~, i~
 *   C0 [B][H][dk][dv], n0 [B][H][dk], m0 [B][H] : the stabilized state (memory in the
 *       storage orientation, normalizer, running max), or all NULL for an empty memory
 *   h : [B][T][H][dv] fp32, required;  C_T, n_T, m_T : the final state, or NULL
 * Per (b, h), with f_t = sigmoid(f~_t) and i_t = exp(i~_t):
 *   m_t = max(log f_t + m_{t-1}, i~_t)      (m_0 = -inf for an empty memory)
 *   C_t = e^{log f_t + m_{t-1} - m_t} C_{t-1} + e^{i~_t - m_t} v_t k_t^T,  n_t likewise with k_t
 *   h_t = C_t q_t / max(|n_t . q_t|, e^{-m_t})
 * i.e. the naive recurrence (C_t = f_t C_{t-1} + i_t v_t k_t^T, floor 1) carried in the
 * coordinates C e^{-m_t}, which never overflow.
 */
typedef struct {
  gdr_dtype dtype;
  int B, H, T, dk, dv;  /* dk, dv in {64, 128} */
  const void *q, *k, *v;
  const float *f_pre, *i_pre;
  const float *C0, *n0, *m0;
  float *h;
  float *C_T, *n_T, *m_T;
  uint32_t *status;  /* device word or NULL: GDR_ERR_TIMEOUT after a bounded wait ran out */
} gdr_mlstm_args;

/*
 * The mLSTM cell over whole sequences, chunkwise: per 64-token chunk with A_t the
 * cumulative log f_t inside the chunk and (C, n, m) carried from the previous chunk,
 *   m_t = A_t + max(m, max_{s <= t} (i~_s - A_s)),
 *   h_t = (sum_{s<=t} w_ts (q_t.k_s) v_s + g_t C q_t) / max(|sum_{s<=t} w_ts (q_t.k_s) + g_t n.q_t|, e^{-m_t})
 * with w_ts = e^{A_t - A_s + i~_s - m_t} and g_t = e^{A_t + m - m_t}, all <= 1; the chunk's
 * products on the tensor cores: tcgen05 with TMEM accumulators for bf16 at dk = dv = 128,
 * warp-level MMAs otherwise (tf32, three products for fp32 inputs).  No workspace.
 * Errors as gdr_forward_chunked; GDR_ERR_UNSUPPORTED for dk or dv outside {64, 128}.  The
 * tcgen05 kernel bounds its waits on the tensor cores and copies (about 2 s); one that runs
 * out writes GDR_ERR_TIMEOUT to `status` when given (gdr_read_status reads and clears it)
 * and leaves h and the final state undefined.
 */
gdr_status gdr_mlstm_forward(const gdr_mlstm_args *args, void *stream);

/*
 * Arguments of gdr_decode_step: one token for each (b, h).
 *   q, k, log_w, e1 (GENERAL/GDN2/RWKV7) : [B][H][dk]
 *   v, o, e2 (GDN2)                      : [B][H][dv]
 *   e2 (GENERAL)                         : [B][H][dk]
 *   e2 (RWKV7)                           : [B][H]
 *   S                                    : [B][H][dk][dv] fp32, updated in place
 */
typedef struct {
  gdr_form form;
  gdr_dtype dtype;
  int B, H, dk, dv;     /* dk, dv in {16, 32, 64, 128}; B, H >= 0 */
  const void *q, *k, *v;
  const float *log_w;
  const void *e1, *e2;
  float *S;
  float *o;             /* [B][H][dv] fp32, required */
} gdr_step_args;

/*
 * One recurrent step (decode).  "Muir ...", section 2.1 eq. (1) and section 4.2
 * eq. (8); "Exponential gates and matrix memory ...", section 13.3.  Reads S once:
 * e = S u and S (w (.) q) come from the old state in the same pass, then
 * o = S(w (.) q) - e <z, q> + v <k, q> and S <- S Diag(w) - e z^T + v k^T in place.
 */
gdr_status gdr_decode_step(const gdr_step_args *args, void *stream);

/*
 * S_out[i] = M[i] S_in[i] + Q[i] for i < BH: M [BH][dk][dk], S_in, Q, S_out [BH][dk][dv],
 * fp32 (S_in or Q NULL = 0; S_out may alias Q, not S_in).  In the storage orientation a
 * sequence segment maps its entry state affinely to its exit state, S_out = M S_in + Q
 * ("Muir ...", section 4.2 eq. (10): the chunk's end state is affine in its start state,
 * and so is any run of chunks); M is the segment run from S_in = I with v = 0, Q the run
 * from S_in = 0.  Composing the maps of consecutive segments gives each segment its entry
 * state (sequence parallelism).  Products as tf32 with the three-product split (fp32
 * accuracy).  dk, dv in {16, 32, 64, 128}.
 */
gdr_status gdr_state_compose(float *S_out, const float *M, const float *S_in, const float *Q,
                             int BH, int dk, int dv, void *stream);

/* S[B][H][dk][dv] = src (device pointer, same layout) or 0 when src == NULL. */
gdr_status gdr_state_init(float *S, int B, int H, int dk, int dv, const float *src, void *stream);

/*
 * Synchronizes `stream`, then reads and clears the status word the kernels keep
 * at the start of `workspace` (GDR_OK if no device check or bounded wait failed).
 * The only call here that synchronizes.
 */
gdr_status gdr_read_status(void *workspace, void *stream, gdr_status *device_status);

/* Static text for a status code; never NULL. */
const char *gdr_status_string(gdr_status s);

/* ABI version: major * 10000 + minor * 100 + patch. */
int gdr_version(void);

#ifdef __cplusplus
}
#endif

#endif /* GDR_H_ */
