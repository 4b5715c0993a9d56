// gdn_tmap.h -- host side of tensor-map (TMA) copies: cuTensorMapEncodeTiled
// reached through the runtime's driver entry point, so that the library does
// not link against the driver library.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace gdn {

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

// The encoder, or null when the driver does not provide it.
inline EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  if (!fn) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  }
  return fn;
}

// Maps over a [T][H][D] bf16 input (row-major, tokens outermost) whose boxes
// cover box_tokens consecutive tokens of one head.
//   plane map: a 4-D map over (8 channels, T tokens, D / 8 channel groups,
//     H heads); a box of 8 x box_tokens x box_groups x 1 lands in shared
//     memory as [group][token][8], the core-matrix layout of a plane with
//     box_tokens rows (coordinates: 0, first token, first group, head).
//   row map: a 3-D map over (D channels, H heads, T tokens); a box of
//     D x 1 x box_tokens lands as [token][channel] (coordinates: 0, head,
//     first token).
// Tokens past T read as zeros.  False if the encoder is missing or refuses.
inline bool encode_plane_map(CUtensorMap* map, const void* base, int64_t T, int H, int D,
                             int box_tokens, int box_groups) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  const cuuint64_t dims[4] = {8, (cuuint64_t)T, (cuuint64_t)D / 8, (cuuint64_t)H};
  const cuuint64_t strides[3] = {(cuuint64_t)H * D * 2, 16, (cuuint64_t)D * 2};  // bytes, dims 1..3
  const cuuint32_t box[4] = {8, (cuuint32_t)box_tokens, (cuuint32_t)box_groups, 1};
  const cuuint32_t estr[4] = {1, 1, 1, 1};
  return fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(base), dims, strides, box,
            estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}
inline bool encode_row_map(CUtensorMap* map, const void* base, int64_t T, int H, int D,
                           int box_tokens) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  const cuuint64_t dims[3] = {(cuuint64_t)D, (cuuint64_t)H, (cuuint64_t)T};
  const cuuint64_t strides[2] = {(cuuint64_t)D * 2, (cuuint64_t)H * D * 2};  // bytes, dims 1..2
  const cuuint32_t box[3] = {(cuuint32_t)D, 1, (cuuint32_t)box_tokens};
  const cuuint32_t estr[3] = {1, 1, 1};
  return fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box,
            estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace gdn
