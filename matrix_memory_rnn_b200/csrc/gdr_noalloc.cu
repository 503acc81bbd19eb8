// gdr_noalloc.cu -- gdr_forward_chunked_noalloc: the chunked forward for callers
// that are not allowed to allocate device memory.
//
// gdr_forward_chunked needs a small device workspace (its status word).  Most
// callers get it from their allocator.  Some cannot: a plugin or extension whose
// host application owns every device allocation, a serving loop that forbids
// allocation after start-up so its memory plan cannot be broken mid-flight, or
// code that runs where cudaMalloc would synchronize the device or is simply not
// available.  For them this entry point takes its workspace from a fixed array
// compiled into the library instead.
//
// The array is a file-scope static __device__ symbol, so every GPU that loads
// libgdr holds it (kNoAllocScratchBytes bytes) until the process exits.  Host
// code cannot use the symbol's name as a device address (on the host it names a
// stand-in object), so the device address is looked up with cudaGetSymbolAddress,
// with the device current, and cached per device together with the id of the CUDA
// context it was looked up in.  A call made in another context than the cached
// one (after cudaDeviceReset, or once the primary context has been released and
// created again, the module is loaded anew and the array may have moved) looks
// the address up again.  Nothing here calls cudaMalloc, cudaFree or any
// allocating routine.
#include <cuda.h>

#include <mutex>

#include "gdr_internal.cuh"

namespace {

// Stated maximum workspace of the no-alloc path.  Every path it takes needs only
// the status word (gdr::kStatusBytes); a call that would need more is rejected.
constexpr size_t kNoAllocScratchBytes = 4096;
static_assert(gdr::kStatusBytes <= kNoAllocScratchBytes,
              "the no-alloc scratch must hold the forward's status word");
constexpr int kMaxDevices = 64;

static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

struct ScratchEntry {
  unsigned long long ctx_id;   // id of the context the address belongs to (0: none yet)
  void *ptr;
};
std::mutex g_scratch_mutex;
ScratchEntry g_scratch[kMaxDevices] = {};

using CtxGetCurrentFn = CUresult (*)(CUcontext *);
using CtxGetIdFn = CUresult (*)(CUcontext, unsigned long long *);

// Driver entry points of the two context queries (looked up once; null if missing).
struct CtxQueries {
  CtxGetCurrentFn get_current = nullptr;
  CtxGetIdFn get_id = nullptr;
};
const CtxQueries &ctx_queries() {
  static CtxQueries q;
  static std::once_flag once;
  std::call_once(once, [] {
    void *fn = nullptr;
    cudaDriverEntryPointQueryResult r;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &fn, cudaEnableDefault, &r) == cudaSuccess &&
        r == cudaDriverEntryPointSuccess)
      q.get_current = reinterpret_cast<CtxGetCurrentFn>(fn);
    fn = nullptr;
    if (cudaGetDriverEntryPoint("cuCtxGetId", &fn, cudaEnableDefault, &r) == cudaSuccess &&
        r == cudaDriverEntryPointSuccess)
      q.get_id = reinterpret_cast<CtxGetIdFn>(fn);
  });
  return q;
}

// Id of the context current on this thread, or 0 if there is none (or it cannot be read).
unsigned long long current_ctx_id() {
  const CtxQueries &q = ctx_queries();
  CUcontext ctx = nullptr;
  unsigned long long id = 0;
  if (!q.get_current || !q.get_id || q.get_current(&ctx) != CUDA_SUCCESS || !ctx) return 0;
  if (q.get_id(ctx, &id) != CUDA_SUCCESS) return 0;
  return id;
}

// Device address of g_noalloc_scratch in the current device's current context.
gdr_status scratch_for_current_device(void **out) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return GDR_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_scratch_mutex);
  unsigned long long id = current_ctx_id();
  if (id == 0 || g_scratch[dev].ctx_id != id) {
    void *p = nullptr;
    // also makes the device's primary context current if no context was
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p) return GDR_ERR_CUDA;
    if (id == 0) id = current_ctx_id();
    g_scratch[dev] = {id, p};   // id 0 (context not readable): looked up again next call
  }
  *out = g_scratch[dev].ptr;
  return GDR_OK;
}

}  // namespace

extern "C" gdr_status gdr_forward_chunked_noalloc(const gdr_fwd_args *args, void *stream) {
  if (!args) return GDR_ERR_INVALID_ARG;
  // Every host check of gdr_forward_chunked, for a workspace of the array's size, before
  // anything is enqueued: a rejected call leaves the array (and a call still running on
  // another stream) untouched.
  gdr::FwdPath path;
  gdr_status st = gdr::forward_plan(args, nullptr, kNoAllocScratchBytes, &path);
  if (st != GDR_OK) return st;
  gdr_fwd_args a = *args;
  if (path == gdr::FwdPath::kNone || path == gdr::FwdPath::kCopyState) {
    a.workspace = nullptr;      // nothing runs that uses scratch
    a.workspace_bytes = 0;
    return gdr_forward_chunked(&a, stream);
  }
  void *scratch = nullptr;
  st = scratch_for_current_device(&scratch);
  if (st != GDR_OK) return st;
  // The array keeps whatever the previous call left: clear the status word.
  if (cudaMemsetAsync(scratch, 0, gdr::kStatusBytes, static_cast<cudaStream_t>(stream)) != cudaSuccess)
    return GDR_ERR_CUDA;
  a.workspace = scratch;
  a.workspace_bytes = kNoAllocScratchBytes;
  return gdr_forward_chunked(&a, stream);
}

extern "C" gdr_status gdr_noalloc_read_status(void *stream, gdr_status *device_status) {
  if (!device_status) return GDR_ERR_INVALID_ARG;
  void *scratch = nullptr;
  const gdr_status st = scratch_for_current_device(&scratch);
  if (st != GDR_OK) return st;
  return gdr_read_status(scratch, stream, device_status);
}
