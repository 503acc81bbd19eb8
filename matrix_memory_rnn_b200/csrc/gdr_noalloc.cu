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
// stand-in object), so the device address is looked up with cudaGetSymbolAddress
// once per device, with that device current, on that device's first call, and
// cached.  Nothing here calls cudaMalloc, cudaFree or any allocating routine.
#include <mutex>

#include "gdr_internal.cuh"

namespace {

// Stated maximum workspace of the no-alloc path.  gdr_forward_workspace_size
// reports what a call needs; a call needing more is rejected.
constexpr size_t kNoAllocScratchBytes = 4096;
constexpr int kMaxDevices = 64;

static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

std::mutex g_scratch_mutex;
void *g_scratch_ptr[kMaxDevices] = {};

// Device address of g_noalloc_scratch on the current device (looked up once per device).
gdr_status scratch_for_current_device(void **out) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return GDR_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_scratch_mutex);
  if (!g_scratch_ptr[dev]) {
    void *p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p) return GDR_ERR_CUDA;
    g_scratch_ptr[dev] = p;
  }
  *out = g_scratch_ptr[dev];
  return GDR_OK;
}

}  // namespace

extern "C" gdr_status gdr_forward_chunked_noalloc(const gdr_fwd_args *args, void *stream) {
  if (!args) return GDR_ERR_INVALID_ARG;
  // The smallest workspace gdr_forward_chunked accepts: with it the tensor-core
  // path runs as a single kernel (the two-kernel path needs per-chunk records).
  const size_t need = gdr::kStatusBytes;
  if (need > kNoAllocScratchBytes) return GDR_ERR_WORKSPACE;
  gdr_status st = GDR_OK;
  void *scratch = nullptr;
  st = scratch_for_current_device(&scratch);
  if (st != GDR_OK) return st;
  // The array keeps whatever the previous call left: clear the status word.
  if (cudaMemsetAsync(scratch, 0, need, static_cast<cudaStream_t>(stream)) != cudaSuccess)
    return GDR_ERR_CUDA;
  gdr_fwd_args a = *args;
  a.workspace = scratch;
  a.workspace_bytes = kNoAllocScratchBytes;
  return gdr_forward_chunked(&a, stream);
}
