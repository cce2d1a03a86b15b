// hybrid.cu - BF16 tensor-core self-test for the hybrid-precision prefill (sm_100a).
//
// The hybrid prefill (HyQuant: vertical-line and sliding-window keys in FP16/BF16, the rest
// 4-bit, one online softmax) runs inside the prefill kernel (attn_fwd.cu): its full-precision
// tiles are BF16 tcgen05 products (kind::f16).  This file holds the diagnostic that pins that
// MMA path - instruction descriptor, 128-byte swizzle, K-major and MN-major operand
// descriptors - against an FP64 product, and the status word of its kernel.
#include <math.h>

#include "fa4q_common.cuh"
#include "fa4q_internal.h"

namespace fa4q {

static __device__ uint32_t g_hy_status;

cudaError_t hy_status_fetch(cudaStream_t st, uint32_t* host_word) {
  cudaError_t e = cudaMemcpyFromSymbolAsync(host_word, g_hy_status, sizeof(uint32_t), 0, cudaMemcpyDeviceToHost, st);
  if (e != cudaSuccess) return e;
  const uint32_t zero = 0;
  e = cudaMemcpyToSymbolAsync(g_hy_status, &zero, sizeof(uint32_t), 0, cudaMemcpyHostToDevice, st);
  if (e != cudaSuccess) return e;
  return cudaStreamSynchronize(st);
}

// ---------------------------------------------------------------------------------------
// self-test: one 128 x N x K BF16 tensor-core product through the operand layouts the
// hybrid prefill uses - A K-major, B K-major ([N][K]) or MN-major ([K][N]), 128-byte
// swizzled 64-element column chunks
// ---------------------------------------------------------------------------------------
__global__ void __launch_bounds__(128, 1)
    selftest_bf16_kernel(const uint16_t* __restrict__ a, const uint16_t* __restrict__ b, int N, int K,
                         int b_mn, float* __restrict__ d_out) {
  extern __shared__ __align__(1024) uint8_t st_smem[];
  uint8_t* sa = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(st_smem) + 1023) & ~uintptr_t(1023));
  uint8_t* sb = sa + 2 * 16384;
  __shared__ uint64_t bar;
  __shared__ uint32_t tbase;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // A [128][K]: chunk h (64 columns) of row r at sa + h * 16384 + swz128(r, column / 8)
  for (int i = threadIdx.x; i < 128 * K / 8; i += 128) {
    const int r = i / (K / 8), c8 = i % (K / 8);
    const uint4 v = *reinterpret_cast<const uint4*>(a + r * K + 8 * c8);
    *reinterpret_cast<uint4*>(sa + (c8 >> 3) * 16384 + swz128_offset(r, c8 & 7)) = v;
  }
  if (!b_mn) {
    // B [N][K] K-major: chunk h of row n at sb + h * (N * 128)
    for (int i = threadIdx.x; i < N * K / 8; i += 128) {
      const int r = i / (K / 8), c8 = i % (K / 8);
      const uint4 v = *reinterpret_cast<const uint4*>(b + r * K + 8 * c8);
      *reinterpret_cast<uint4*>(sb + (c8 >> 3) * (N * 128) + swz128_offset(r, c8 & 7)) = v;
    }
  } else {
    // B [K][N] MN-major: chunk h (64 columns of N) of row k at sb + h * (K * 128)
    for (int i = threadIdx.x; i < K * N / 8; i += 128) {
      const int r = i / (N / 8), c8 = i % (N / 8);
      const uint4 v = *reinterpret_cast<const uint4*>(b + r * N + 8 * c8);
      *reinterpret_cast<uint4*>(sb + (c8 >> 3) * (K * 128) + swz128_offset(r, c8 & 7)) = v;
    }
  }
  fence_proxy_async_smem();
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    fence_barrier_init();
  }
  if (warp == 0) {
    tmem_alloc(&tbase, 256);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tbase;
  if (warp == 0 && elect_one()) {
    const uint32_t idesc = make_idesc_bf16(N, b_mn != 0);
    for (int kk = 0; kk < K / 16; ++kk) {
      const uint64_t ad = make_smem_desc(smem_u32(sa) + (kk >> 2) * 16384 + 32 * (kk & 3), 16, 1024, kSwiz128);
      const uint64_t bd = b_mn ? make_smem_desc(smem_u32(sb) + kk * 2048, K * 128, 1024, kSwiz128)
                               : make_smem_desc(smem_u32(sb) + (kk >> 2) * (N * 128) + 32 * (kk & 3), 16, 1024, kSwiz128);
      mma_bf16(tmem, ad, bd, idesc, kk > 0);
    }
    tc_commit(&bar);
  }
  __syncwarp();
  mbar_wait(&bar, 0, &g_hy_status, kStatusTimeoutProbe);
  tc_fence_after();
  const int r = warp * 32 + lane;
  const uint32_t lb = tmem + (static_cast<uint32_t>(warp * 32) << 16);
  for (int c = 0; c < N; c += 16) {
    uint32_t raw[16];
    tmem_ld16(lb + c, raw);
    tmem_wait_ld();
    for (int i = 0; i < 16; ++i) d_out[r * N + c + i] = __uint_as_float(raw[i]);
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, 256);
  }
}

}  // namespace fa4q

using namespace fa4q;

extern "C" fa4q_status fa4q_selftest_bf16_mma(const void* a, const void* b, int N, int K, int b_mn_major,
                                              float* d_out, void* stream) {
  if (!a || !b || !d_out) return FA4Q_ERR_INVALID_ARG;
  if (K != 64 && K != 128) return FA4Q_ERR_UNSUPPORTED;
  if (b_mn_major != 0 && b_mn_major != 1) return FA4Q_ERR_INVALID_ARG;
  if (b_mn_major ? (N != 64 && N != 128) : (N != 16 && N != 64 && N != 128)) return FA4Q_ERR_UNSUPPORTED;
  if (!aligned16(a) || !aligned16(b)) return FA4Q_ERR_INVALID_ARG;
  const size_t smem = 2 * 16384 + 2 * 16384 + 1024;
  if (cudaFuncSetAttribute(selftest_bf16_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) != cudaSuccess)
    return FA4Q_ERR_CUDA;
  selftest_bf16_kernel<<<1, 128, smem, static_cast<cudaStream_t>(stream)>>>(
      static_cast<const uint16_t*>(a), static_cast<const uint16_t*>(b), N, K, b_mn_major, d_out);
  return launch_status();
}
