// gdr_tma_host.cuh -- host side of the TMA copies: the driver's tensor-map encoder (looked up
// once through the runtime) and the 4-D map of a token-major [B][T][H][channels] tensor.
#pragma once

#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>

#include <mutex>

namespace gdr {
namespace tma {

inline PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
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

// [B][T][H][channels] tensor (channels 128 unless given) of `elem`-byte elements as a 4-D map
// (channel, head, token, batch) with a (box0, 1, box_tokens, 1) box.  Tokens past T read as
// zeros (and are not written by stores).
inline bool encode_input_map(CUtensorMap *m, const void *base, CUtensorMapDataType type, int elem,
                             int box0, int box_tokens, CUtensorMapSwizzle swizzle, int H, int T, int B,
                             int channels = 128) {
  PFN_cuTensorMapEncodeTiled_v12000 enc = tensor_map_encoder();
  if (!enc) return false;
  const cuuint64_t ch = (cuuint64_t)channels;
  const cuuint64_t dims[4] = {ch, (cuuint64_t)H, (cuuint64_t)T, (cuuint64_t)B};
  const cuuint64_t strides[3] = {ch * elem, (cuuint64_t)H * ch * elem, (cuuint64_t)T * H * ch * elem};
  const cuuint32_t box[4] = {(cuuint32_t)box0, 1, (cuuint32_t)box_tokens, 1};
  const cuuint32_t estr[4] = {1, 1, 1, 1};
  return enc(m, type, 4, const_cast<void *>(base), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace tma
}  // namespace gdr
