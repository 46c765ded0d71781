// Host-side TMA tensor-map construction for BF16 tensors: dense [B*H, N, d]
// and packed variable-length [total, H, d].
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>

#include <mutex>
#include <string>

namespace eab {

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

// cuTensorMapEncodeTiled through the runtime's driver entry-point lookup, so
// the library does not link libcuda directly.
inline EncodeTiledFn get_encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

// Encodes a 3-D BF16 tensor map: dims innermost first (dims[0] = d, 2-byte
// elements, contiguous), byte strides of dims 1 and 2, box = 64 columns of d
// (128 bytes, 128-byte swizzle) x box1 x box2.  Coordinates outside the dims
// read as zero and are clipped on store.  Returns false (and a message) on failure.
inline bool encode_bf16_3d(CUtensorMap* tm, const void* base, const cuuint64_t dims[3],
                           const cuuint64_t strides[2], cuuint32_t box1, cuuint32_t box2,
                           std::string* err) {
  EncodeTiledFn enc = get_encode_fn();
  if (!enc) {
    *err = "cuTensorMapEncodeTiled unavailable";
    return false;
  }
  const cuuint32_t box[3] = {64u, box1, box2};
  const cuuint32_t estr[3] = {1u, 1u, 1u};
  CUresult r = enc(tm, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides,
                   box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) {
    *err = "cuTensorMapEncodeTiled failed (CUresult " + std::to_string(static_cast<int>(r)) + ")";
    return false;
  }
  return true;
}

// 8-bit elements: a 3-D map [BH, N, d] of bytes, box = 128 columns (128 bytes,
// 128-byte swizzle) x box_rows rows x 1; coordinates (column, row, head).
inline bool make_tmap_u8_3d(CUtensorMap* tm, const void* base, int BH, int N, int d, int box_rows,
                            std::string* err) {
  EncodeTiledFn enc = get_encode_fn();
  if (!enc) {
    *err = "cuTensorMapEncodeTiled unavailable";
    return false;
  }
  const cuuint64_t dims[3] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(N),
                              static_cast<cuuint64_t>(BH)};
  const cuuint64_t strides[2] = {static_cast<cuuint64_t>(d),
                                 static_cast<cuuint64_t>(N) * static_cast<cuuint64_t>(d)};
  const cuuint32_t box[3] = {128u, static_cast<cuuint32_t>(box_rows), 1u};
  const cuuint32_t estr[3] = {1u, 1u, 1u};
  CUresult r = enc(tm, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<void*>(base), dims, strides, box,
                   estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) {
    *err = "cuTensorMapEncodeTiled failed (CUresult " + std::to_string(static_cast<int>(r)) + ")";
    return false;
  }
  return true;
}

// FP32 [BH, N, d] with 32-column (128-byte, 128-byte swizzle) x box_rows boxes;
// coordinates (column, row, head).  Used for reductions into an accumulator.
inline bool make_tmap_f32_3d(CUtensorMap* tm, const void* base, int BH, int N, int d, int box_rows,
                             std::string* err) {
  EncodeTiledFn enc = get_encode_fn();
  if (!enc) {
    *err = "cuTensorMapEncodeTiled unavailable";
    return false;
  }
  const cuuint64_t dims[3] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(N),
                              static_cast<cuuint64_t>(BH)};
  const cuuint64_t strides[2] = {static_cast<cuuint64_t>(d) * 4,
                                 static_cast<cuuint64_t>(N) * static_cast<cuuint64_t>(d) * 4};
  const cuuint32_t box[3] = {32u, static_cast<cuuint32_t>(box_rows), 1u};
  const cuuint32_t estr[3] = {1u, 1u, 1u};
  CUresult r = enc(tm, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, const_cast<void*>(base), dims, strides, box,
                   estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) {
    *err = "cuTensorMapEncodeTiled failed (CUresult " + std::to_string(static_cast<int>(r)) + ")";
    return false;
  }
  return true;
}

// FP32 packed [total, H, d] with 32-column x 1-head x box_rows boxes (the same
// shared-memory layout as make_tmap_f32_3d's); coordinates (column, head, row).
inline bool make_tmap_f32_packed(CUtensorMap* tm, const void* base, int total, int H, int d,
                                 int box_rows, std::string* err) {
  EncodeTiledFn enc = get_encode_fn();
  if (!enc) {
    *err = "cuTensorMapEncodeTiled unavailable";
    return false;
  }
  const cuuint64_t dims[3] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(H),
                              static_cast<cuuint64_t>(total)};
  const cuuint64_t strides[2] = {static_cast<cuuint64_t>(d) * 4,
                                 static_cast<cuuint64_t>(H) * static_cast<cuuint64_t>(d) * 4};
  const cuuint32_t box[3] = {32u, 1u, static_cast<cuuint32_t>(box_rows)};
  const cuuint32_t estr[3] = {1u, 1u, 1u};
  CUresult r = enc(tm, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, const_cast<void*>(base), dims, strides, box,
                   estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) {
    *err = "cuTensorMapEncodeTiled failed (CUresult " + std::to_string(static_cast<int>(r)) + ")";
    return false;
  }
  return true;
}

// Dense [BH, N, d]: coordinates (column, row, head); rows past N of one head
// read as zero (never as the next head's rows) and are clipped on store.
inline bool make_tmap_bf16_3d(CUtensorMap* tm, const void* base, int BH, int N, int d,
                              int box_rows, std::string* err) {
  const cuuint64_t dims[3] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(N),
                              static_cast<cuuint64_t>(BH)};
  const cuuint64_t strides[2] = {static_cast<cuuint64_t>(d) * 2,
                                 static_cast<cuuint64_t>(N) * static_cast<cuuint64_t>(d) * 2};
  return encode_bf16_3d(tm, base, dims, strides, static_cast<cuuint32_t>(box_rows), 1u, err);
}

// Packed [total, H, d] (sequences back to back): coordinates (column, head,
// row); a box is box_rows consecutive rows of one head.  Rows past `total`
// read as zero and are clipped on store; rows past the end of one sequence are
// the next sequence's, so the kernel masks them (keys) or stores around them (O).
inline bool make_tmap_bf16_packed(CUtensorMap* tm, const void* base, int total, int H, int d,
                                  int box_rows, std::string* err) {
  const cuuint64_t dims[3] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(H),
                              static_cast<cuuint64_t>(total)};
  const cuuint64_t strides[2] = {static_cast<cuuint64_t>(d) * 2,
                                 static_cast<cuuint64_t>(H) * static_cast<cuuint64_t>(d) * 2};
  return encode_bf16_3d(tm, base, dims, strides, 1u, static_cast<cuuint32_t>(box_rows), err);
}

}  // namespace eab
