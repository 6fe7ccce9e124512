// Host-side TMA tensor-map encoding for [batch, seqlen, heads, headdim]
// tensors.  cuTensorMapEncodeTiled is reached through the runtime's driver
// entry-point lookup, so the library does not link libcuda directly.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <cstdint>

namespace fa {

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

inline EncodeTiledFn encode_tiled_fn() {
  static EncodeTiledFn fn = nullptr;
  if (!fn) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  }
  return fn;
}

// Map over a [B, N, H, D] tensor (D innermost) whose box is `box_inner`
// elements of D by 1 head by `box_rows` sequence positions by 1 batch, with
// 128-byte swizzle.  Positions past N read as zero.  Returns 0 on success.
inline int encode_bnhd(CUtensorMap* map, const void* base, CUtensorMapDataType dt, int elem_bytes,
                       int B, int N, int H, int D, int box_inner, int box_rows) {
  EncodeTiledFn fn = encode_tiled_fn();
  if (!fn) return -1;
  cuuint64_t dims[4] = {(cuuint64_t)D, (cuuint64_t)H, (cuuint64_t)N, (cuuint64_t)B};
  cuuint64_t strides[3] = {(cuuint64_t)D * elem_bytes, (cuuint64_t)H * D * elem_bytes,
                           (cuuint64_t)N * H * D * elem_bytes};
  cuuint32_t box[4] = {(cuuint32_t)box_inner, 1u, (cuuint32_t)box_rows, 1u};
  cuuint32_t estr[4] = {1u, 1u, 1u, 1u};
  CUresult r = fn(map, dt, 4, const_cast<void*>(base), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? 0 : -2;
}

// Map over an attention mask [Bm, Hm, N_q, N_k] (keys innermost; row stride
// sq, head stride sh, batch stride sb in elements, a stride of 0 making that
// dimension one deep) whose box is `box_inner` keys by 128 rows, 128-byte
// swizzle.  Rows past N_q and keys past N_k read as zero.  Returns 0 on
// success.
inline int encode_mask(CUtensorMap* map, const void* base, CUtensorMapDataType dt, int elem_bytes, int B, int H,
                       int Nq, int Nk, long long sb, long long sh, long long sq, int box_inner) {
  EncodeTiledFn fn = encode_tiled_fn();
  if (!fn) return -1;
  const cuuint64_t row = (cuuint64_t)sq * elem_bytes;
  cuuint64_t dims[4] = {(cuuint64_t)Nk, (cuuint64_t)Nq, (cuuint64_t)(sh != 0 ? H : 1), (cuuint64_t)(sb != 0 ? B : 1)};
  // a one-deep dimension still needs a valid stride: the row stride
  cuuint64_t strides[3] = {row, sh != 0 ? (cuuint64_t)sh * elem_bytes : row,
                           sb != 0 ? (cuuint64_t)sb * elem_bytes : row};
  cuuint32_t box[4] = {(cuuint32_t)box_inner, 128u, 1u, 1u};
  cuuint32_t estr[4] = {1u, 1u, 1u, 1u};
  CUresult r = fn(map, dt, 4, const_cast<void*>(base), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? 0 : -2;
}

}  // namespace fa
