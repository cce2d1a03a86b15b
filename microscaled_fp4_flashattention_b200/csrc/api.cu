// api.cu - status helpers of the fa4q C ABI.
#include "fa4q_common.cuh"
#include "fa4q_internal.h"

extern "C" const char* fa4q_status_string(fa4q_status s) {
  switch (s) {
    case FA4Q_OK: return "ok";
    case FA4Q_ERR_INVALID_ARG: return "invalid argument";
    case FA4Q_ERR_UNSUPPORTED: return "unsupported shape or format";
    case FA4Q_ERR_CUDA: return "CUDA launch or runtime error";
    case FA4Q_ERR_TIMEOUT: return "a bounded device wait expired";
  }
  return "unknown status";
}

extern "C" int fa4q_version(void) { return 100; }

extern "C" fa4q_status fa4q_device_status(void* stream, uint32_t* detail) {
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  uint32_t a = 0, d = 0, t = 0, h = 0, v = 0;
  if (fa4q::attn_status_fetch(st, &a) != cudaSuccess) return FA4Q_ERR_CUDA;
  if (fa4q::decode_status_fetch(st, &d) != cudaSuccess) return FA4Q_ERR_CUDA;
  if (fa4q::dectc_status_fetch(st, &t) != cudaSuccess) return FA4Q_ERR_CUDA;
  if (fa4q::hy_status_fetch(st, &h) != cudaSuccess) return FA4Q_ERR_CUDA;
  if (fa4q::vl_status_fetch(st, &v) != cudaSuccess) return FA4Q_ERR_CUDA;
  const uint32_t word = a | d | t | h | v;
  if (detail) *detail = word;
  return word ? FA4Q_ERR_TIMEOUT : FA4Q_OK;
}
