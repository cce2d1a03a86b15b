// fa4q_internal.h - host-side helpers shared by the fa4q translation units.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <algorithm>

#include "fa4q.h"

namespace fa4q {

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Map the launch result of the kernels just enqueued to a status code.
inline fa4q_status launch_status() {
  const cudaError_t e = cudaGetLastError();
  return e == cudaSuccess ? FA4Q_OK : FA4Q_ERR_CUDA;
}

// cuTensorMapEncodeTiled through the runtime's driver entry point (no link against libcuda)
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

inline EncodeTiledFn get_encode_fn() {
  static EncodeTiledFn fn = nullptr;
  if (!fn) {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(ptr);
  }
  return fn;
}

// 3-D byte tensor [d2][d1][d0 bytes] with box (box0 bytes, box1 rows, 1)
inline bool make_map_3d(CUtensorMap* m, const void* base, uint64_t d0, uint64_t d1, uint64_t d2,
                        uint32_t box0, uint32_t box1, CUtensorMapSwizzle swz) {
  EncodeTiledFn enc = get_encode_fn();
  if (!enc) return false;
  const cuuint64_t dims[3] = {d0, d1, d2};
  const cuuint64_t strides[2] = {d0, d0 * d1};
  const cuuint32_t box[3] = {box0, box1, 1};
  const cuuint32_t estr[3] = {1, 1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<void*>(base), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, swz, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Streaming multiprocessors of the current device (cached per device; 148 on B200).
inline int num_sms() {
  static int cached[64] = {0};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) dev = 0;
  if (cached[dev] == 0) {
    int n = 0;
    cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    cached[dev] = n > 0 ? n : 148;
  }
  return cached[dev];
}

// Dual-residual NVFP4 query tiles of the FP4 tensor-core decode (quantize.cu): q bf16
// [B][Hq][128] -> qt [B*Hkv][2][128][64] packed, qt_sf [B*Hkv][2][2][512] tiled atoms; rows
// 0..G-1 hold the group's q-heads and rows G..15 are zero (rows 16..127, which the decode does
// not read, are not written).
fa4q_status launch_dec_query(const uint16_t* q, int B, int Hq, int Hkv, uint8_t* qt, uint8_t* qt_sf,
                             cudaStream_t st);
// log-sum-exp merge of decode split partials [rows][splits][d + 2] (m in log2 units, l, o)
// into bf16 rows (decode.cu)
fa4q_status launch_decode_combine(const float* ws, int rows, int splits, uint16_t* out, cudaStream_t st);

// Each translation unit with bounded device waits owns one status word; these host
// functions read-and-clear them (stream-ordered, then synchronised by the caller).
cudaError_t attn_status_fetch(cudaStream_t st, uint32_t* host_word);
cudaError_t decode_status_fetch(cudaStream_t st, uint32_t* host_word);
cudaError_t dectc_status_fetch(cudaStream_t st, uint32_t* host_word);
cudaError_t hy_status_fetch(cudaStream_t st, uint32_t* host_word);
cudaError_t vl_status_fetch(cudaStream_t st, uint32_t* host_word);

}  // namespace fa4q
