// tma_host.h -- host-side construction of TMA tensor maps (cuTensorMapEncodeTiled),
// fetched through the runtime's driver entry point so the library does not link libcuda.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace fa {

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

inline EncodeTiledFn encode_tiled_fn() {
  static EncodeTiledFn fn = nullptr;
  if (fn == nullptr) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess) {
      fn = reinterpret_cast<EncodeTiledFn>(p);
    }
  }
  return fn;
}

// Element encodings of the tensor maps: bf16, fp16 (2 bytes) and e4m3 (1 byte, moved as
// raw bytes).
enum class MapElem { kBf16, kF16, kE4M3 };

inline CUtensorMapDataType map_type(MapElem e) {
  return e == MapElem::kF16 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16
                            : (e == MapElem::kE4M3 ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16);
}
inline int map_bytes(MapElem e) { return e == MapElem::kE4M3 ? 1 : 2; }

// A [B, N, H, d] tensor (d innermost) seen as a 4-D tiled map with boxes of `box_rows`
// sequence positions x 128 bytes of head dimension of one (batch, head), written into
// shared memory with the 128-byte swizzle.  Rows past N read as zero.
inline bool make_bshd_map(CUtensorMap* map, const void* base, int B, int N, int H, int d, int box_rows,
                          MapElem e = MapElem::kBf16) {
  EncodeTiledFn enc = encode_tiled_fn();
  if (enc == nullptr) return false;
  const cuuint64_t eb = map_bytes(e);
  cuuint64_t dims[4] = {(cuuint64_t)d, (cuuint64_t)H, (cuuint64_t)N, (cuuint64_t)B};
  cuuint64_t strides[3] = {(cuuint64_t)d * eb, (cuuint64_t)H * d * eb, (cuuint64_t)N * H * d * eb};
  cuuint32_t box[4] = {(cuuint32_t)(128 / eb), 1, (cuuint32_t)box_rows, 1};
  cuuint32_t estr[4] = {1, 1, 1, 1};
  CUresult r = enc(map, map_type(e), 4, const_cast<void*>(base), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// Decoding queries [B, N_q, H, d]: one box holds the G consecutive heads starting at a
// given head for all N_q positions of one sequence, 64 columns wide.  In shared memory it
// lands as rows r = i * G + g of 128 bytes (128-byte swizzle), the row order of a
// 128-row MMA tile.
inline bool make_decode_q_map(CUtensorMap* map, const void* base, int B, int N_q, int H, int d, int G,
                              MapElem e = MapElem::kBf16) {
  EncodeTiledFn enc = encode_tiled_fn();
  if (enc == nullptr) return false;
  cuuint64_t dims[4] = {(cuuint64_t)d, (cuuint64_t)H, (cuuint64_t)N_q, (cuuint64_t)B};
  cuuint64_t strides[3] = {(cuuint64_t)d * 2, (cuuint64_t)H * d * 2, (cuuint64_t)N_q * H * d * 2};
  cuuint32_t box[4] = {64, (cuuint32_t)G, (cuuint32_t)N_q, 1};
  cuuint32_t estr[4] = {1, 1, 1, 1};
  CUresult r = enc(map, map_type(e), 4, const_cast<void*>(base), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// The backward's fp32 dQ accumulator [B*H, N, d] as a 3-D map {d, N, B*H} for TMA
// reduce-adds from shared memory: boxes of 32 rows x 32 columns (128 bytes, 128-byte
// swizzle).  Rows at or past N lie outside the map and are not written.
inline bool make_dqacc_map(CUtensorMap* map, void* base, long long BH, int N, int d) {
  EncodeTiledFn enc = encode_tiled_fn();
  if (enc == nullptr) return false;
  cuuint64_t dims[3] = {(cuuint64_t)d, (cuuint64_t)N, (cuuint64_t)BH};
  cuuint64_t strides[2] = {(cuuint64_t)d * 4, (cuuint64_t)N * d * 4};
  cuuint32_t box[3] = {32, 32, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, base, dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_NONE,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

}  // namespace fa
