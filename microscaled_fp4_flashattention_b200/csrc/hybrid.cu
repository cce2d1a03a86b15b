// hybrid.cu - hybrid-precision prefill: the full-precision part of the online softmax (sm_100a).
//
// What it computes, per (batch b, q-head h) and query row i of a causal prefill:
//   full-precision keys  F_i = window {j : i - W < j <= i}  +  vertical lines {v : v <= i - W}
//   x_j = (q_i . k_j) * sm_scale * log2(e)             bf16 q, k; FP32 accumulation
//   m0 = max_j x_j,  l0 = sum_j 2^(x_j - m0),  o0 = sum_j 2^(x_j - m0) v_j    (P unquantised)
// written per row as [m0, l0, -, -, o0[0..d)] in FP32 (row stride d + 4: o0 16-byte aligned).  The FP4 prefill kernel continues the same
// online softmax from this state over the remaining keys (FP4 tiles, the vertical lines and
// the window masked out), so every key enters one softmax once.
// Source: HyQuant (Hybrid-Precision Quantization for LLM Attention) - vertical-line and
// sliding-window tokens stay in FP16/BF16, the rest is 4-bit; low-bit and full-precision
// GEMMs share one FlashAttention-style online softmax.
//
// Design: the full-precision keys are a small share of a long prefill (a 128-token window
// and a few percent of vertical lines per row), so this part runs FlashAttention-2 style
// on BF16 mma.sync tiles: CTA = 64 query rows (4 warps x 16 rows) of one (b, h); key chunks
// of 64 rows (the window span first, then the gathered vertical-line rows of the kv-head)
// stream through a two-stage cp.async ring; scores, running maximum and sum stay in
// registers, P goes to BF16 A fragments, V fragments come from ldmatrix.trans.
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

constexpr int kHyD = 128;
constexpr int kHyRows = 64;                      // query rows per CTA
constexpr int kHyKeys = 64;                      // keys per chunk
constexpr int kHyRow = kHyD + 8;                 // padded smem row (bf16 elements)
constexpr int kHyThreads = 128;
constexpr float kHyLog2e = 1.4426950408889634f;

FA4Q_DEVINL void hy_ldsm_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}

FA4Q_DEVINL void hy_ldsm_x4_trans(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}

// D (16x8, FP32) += A (16x16, row) * B (16x8, col), BF16 inputs
FA4Q_DEVINL void hy_mma(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3, uint32_t b0,
                        uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
      "{%8,%9}, {%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// 16-byte async copy global -> shared; src_bytes = 0 fills zeros without reading
FA4Q_DEVINL void hy_cp16(uint32_t dst, const void* src, uint32_t src_bytes) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(src_bytes)
               : "memory");
}
FA4Q_DEVINL void hy_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
FA4Q_DEVINL void hy_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }

FA4Q_DEVINL float hy_ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

FA4Q_DEVINL uint32_t hy_pack_bf16(float lo, float hi) {
  uint32_t d;
  asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(d) : "f"(hi), "f"(lo));
  return d;
}

__global__ void __launch_bounds__(kHyThreads, 2) hybrid_full_kernel(const HyParams p) {
  extern __shared__ __align__(16) uint8_t hy_smem[];
  uint16_t* sq = reinterpret_cast<uint16_t*>(hy_smem);               // [64][kHyRow]
  uint16_t* sk = sq + kHyRows * kHyRow;                               // [2][64][kHyRow]
  uint16_t* sv = sk + 2 * kHyKeys * kHyRow;                           // [2][64][kHyRow]
  int* spos = reinterpret_cast<int*>(sv + 2 * kHyKeys * kHyRow);      // [2][64] key positions

  const int r0 = blockIdx.x * kHyRows, h = blockIdx.y, b = blockIdx.z;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int hk = h / (p.Hq / p.Hkv);
  const int64_t bh_q = static_cast<int64_t>(b) * p.Hq + h;
  const int64_t bh_k = static_cast<int64_t>(b) * p.Hkv + hk;
  const int S = p.S, W = p.W;

  // window span of the CTA's rows, then the vertical lines any of its rows keeps
  const int w_lo = max(0, r0 - W + 1), w_hi = min(S, r0 + kHyRows);
  const int n_wc = (w_hi - w_lo + kHyKeys - 1) / kHyKeys;
  const int n_vl_all = p.vl_count ? min(p.vl_count[bh_k], p.max_vl) : 0;
  const int vl_bound = min(r0 + kHyRows - 1, S - 1) - W;      // largest position any row keeps
  int n_vl = 0;
  for (int base = 0; base < n_vl_all; base += kHyThreads) {
    const int idx = base + threadIdx.x;
    n_vl += __syncthreads_count(idx < n_vl_all && p.vl_pos[bh_k * p.max_vl + idx] <= vl_bound);
  }
  const int n_chunks = n_wc + (n_vl + kHyKeys - 1) / kHyKeys;

  // query rows -> shared memory (rows past S are zero)
  for (int idx = threadIdx.x; idx < kHyRows * (kHyD / 8); idx += kHyThreads) {
    const int r = idx / (kHyD / 8), c = idx % (kHyD / 8);
    const int row = r0 + r;
    const bool in = row < S;
    hy_cp16(smem_u32(sq + r * kHyRow + 8 * c), p.q + (bh_q * S + (in ? row : 0)) * kHyD + 8 * c, in ? 16u : 0u);
  }
  auto load_chunk = [&](int c, int buf) {
    const bool win = c < n_wc;
    const int base = win ? w_lo + c * kHyKeys : (c - n_wc) * kHyKeys;
    const int lim = win ? w_hi : n_vl;
    for (int idx = threadIdx.x; idx < kHyKeys * (kHyD / 8); idx += kHyThreads) {
      const int r = idx / (kHyD / 8), cc = idx % (kHyD / 8);
      const int e = base + r;
      const bool in = e < lim;
      const int64_t off = win ? (bh_k * S + (in ? e : 0)) * kHyD : (bh_k * p.max_vl + (in ? e : 0)) * kHyD;
      const uint16_t* ks = (win ? p.k : p.vl_k) + off + 8 * cc;
      const uint16_t* vs = (win ? p.v : p.vl_v) + off + 8 * cc;
      hy_cp16(smem_u32(sk + (buf * kHyKeys + r) * kHyRow + 8 * cc), ks, in ? 16u : 0u);
      hy_cp16(smem_u32(sv + (buf * kHyKeys + r) * kHyRow + 8 * cc), vs, in ? 16u : 0u);
    }
    if (threadIdx.x < kHyKeys) {
      const int e = base + threadIdx.x;
      // a position no row accepts marks an empty slot
      spos[buf * kHyKeys + threadIdx.x] =
          e < lim ? (win ? e : p.vl_pos[bh_k * p.max_vl + e]) : 0x7fffffff;
    }
    hy_commit();
  };
  if (n_chunks > 0) load_chunk(0, 0);
  else hy_commit();

  const int g4 = lane >> 2, t4 = lane & 3;
  const int row_a = r0 + warp * 16 + g4, row_b = row_a + 8;    // this thread's two rows
  float o[kHyD / 8][4];
#pragma unroll
  for (int i = 0; i < kHyD / 8; ++i) o[i][0] = o[i][1] = o[i][2] = o[i][3] = 0.0f;
  float m_a = -INFINITY, m_b = -INFINITY, l_a = 0.0f, l_b = 0.0f;
  const uint32_t a_base = smem_u32(sq + (warp * 16 + ((lane >> 3) & 1) * 8 + (lane & 7)) * kHyRow + (lane >> 4) * 8);

  for (int c = 0; c < n_chunks; ++c) {
    const int buf = c & 1;
    if (c + 1 < n_chunks) {
      load_chunk(c + 1, buf ^ 1);
      hy_wait<1>();
    } else {
      hy_wait<0>();
    }
    __syncthreads();
    const bool win = c < n_wc;
    // S = Q K^T for this warp's 16 rows and the chunk's 64 keys
    float s[8][4];
#pragma unroll
    for (int nt = 0; nt < 8; ++nt) s[nt][0] = s[nt][1] = s[nt][2] = s[nt][3] = 0.0f;
#pragma unroll
    for (int ks = 0; ks < kHyD / 16; ++ks) {
      uint32_t a0, a1, a2, a3;
      hy_ldsm_x4(a_base + ks * 32, a0, a1, a2, a3);
#pragma unroll
      for (int np2 = 0; np2 < 4; ++np2) {
        const int key = np2 * 16 + (lane >> 4) * 8 + (lane & 7);
        const int col = ks * 16 + ((lane >> 3) & 1) * 8;
        uint32_t b0, b1, b2, b3;
        hy_ldsm_x4(smem_u32(sk + (buf * kHyKeys + key) * kHyRow + col), b0, b1, b2, b3);
        hy_mma(s[2 * np2], a0, a1, a2, a3, b0, b1);
        hy_mma(s[2 * np2 + 1], a0, a1, a2, a3, b2, b3);
      }
    }
    // masks: window keys i - W < pos <= i; vertical lines pos <= i - W
    float tmax_a = -INFINITY, tmax_b = -INFINITY;
#pragma unroll
    for (int nt = 0; nt < 8; ++nt)
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const int pos = spos[buf * kHyKeys + nt * 8 + 2 * t4 + e];
        const bool va = win ? (pos <= row_a && pos > row_a - W) : (pos <= row_a - W);
        const bool vb = win ? (pos <= row_b && pos > row_b - W) : (pos <= row_b - W);
        s[nt][e] = va ? s[nt][e] * p.c2 : -INFINITY;
        s[nt][2 + e] = vb ? s[nt][2 + e] * p.c2 : -INFINITY;
        tmax_a = fmaxf(tmax_a, s[nt][e]);
        tmax_b = fmaxf(tmax_b, s[nt][2 + e]);
      }
#pragma unroll
    for (int off = 1; off <= 2; off <<= 1) {
      tmax_a = fmaxf(tmax_a, __shfl_xor_sync(0xffffffffu, tmax_a, off));
      tmax_b = fmaxf(tmax_b, __shfl_xor_sync(0xffffffffu, tmax_b, off));
    }
    const float mn_a = fmaxf(m_a, tmax_a), mn_b = fmaxf(m_b, tmax_b);
    // rows with no key yet keep (m, l, o) = (-inf, 0, 0): no NaN from -inf - -inf
    const float al_a = mn_a == -INFINITY ? 1.0f : hy_ex2(m_a - mn_a);
    const float al_b = mn_b == -INFINITY ? 1.0f : hy_ex2(m_b - mn_b);
    const float ref_a = mn_a == -INFINITY ? 0.0f : mn_a, ref_b = mn_b == -INFINITY ? 0.0f : mn_b;
    float ps_a = 0.0f, ps_b = 0.0f;
    uint32_t pa[8][2];
#pragma unroll
    for (int nt = 0; nt < 8; ++nt) {
      const float p0 = hy_ex2(s[nt][0] - ref_a), p1 = hy_ex2(s[nt][1] - ref_a);
      const float p2 = hy_ex2(s[nt][2] - ref_b), p3 = hy_ex2(s[nt][3] - ref_b);
      ps_a += p0 + p1;
      ps_b += p2 + p3;
      pa[nt][0] = hy_pack_bf16(p0, p1);
      pa[nt][1] = hy_pack_bf16(p2, p3);
    }
    l_a = l_a * al_a + ps_a;
    l_b = l_b * al_b + ps_b;
    m_a = mn_a;
    m_b = mn_b;
#pragma unroll
    for (int dt = 0; dt < kHyD / 8; ++dt) {
      o[dt][0] *= al_a;
      o[dt][1] *= al_a;
      o[dt][2] *= al_b;
      o[dt][3] *= al_b;
    }
    // O += P V: k-steps of 16 keys; A = P (score accumulators repacked), B = V via ldmatrix.trans
#pragma unroll
    for (int kk = 0; kk < kHyKeys / 16; ++kk) {
      const uint32_t a0 = pa[2 * kk][0], a1 = pa[2 * kk][1], a2 = pa[2 * kk + 1][0], a3 = pa[2 * kk + 1][1];
      const int key = kk * 16 + (lane & 7) + ((lane >> 3) & 1) * 8;
#pragma unroll
      for (int dp = 0; dp < kHyD / 16; ++dp) {
        const int col = dp * 16 + (lane >> 4) * 8;
        uint32_t b0, b1, b2, b3;
        hy_ldsm_x4_trans(smem_u32(sv + (buf * kHyKeys + key) * kHyRow + col), b0, b1, b2, b3);
        hy_mma(o[2 * dp], a0, a1, a2, a3, b0, b1);
        hy_mma(o[2 * dp + 1], a0, a1, a2, a3, b2, b3);
      }
    }
    __syncthreads();      // buffer buf is refilled by the next iteration's load
  }
  // the four threads of a row hold partial sums of l
#pragma unroll
  for (int off = 1; off <= 2; off <<= 1) {
    l_a += __shfl_xor_sync(0xffffffffu, l_a, off);
    l_b += __shfl_xor_sync(0xffffffffu, l_b, off);
  }
  const int rows[2] = {row_a, row_b};
  const float ms[2] = {m_a, m_b}, ls[2] = {l_a, l_b};
#pragma unroll
  for (int hf = 0; hf < 2; ++hf) {
    if (rows[hf] >= S) continue;
    float* dst = p.part + (bh_q * S + rows[hf]) * (kHyD + 4);
    if (t4 == 0) {
      dst[0] = ms[hf];
      dst[1] = ls[hf];
    }
#pragma unroll
    for (int dt = 0; dt < kHyD / 8; ++dt)
      *reinterpret_cast<float2*>(dst + 4 + dt * 8 + 2 * t4) = make_float2(o[dt][2 * hf], o[dt][2 * hf + 1]);
  }
}

constexpr size_t kHySmem = (size_t)(kHyRows + 4 * kHyKeys) * kHyRow * 2 + 2 * kHyKeys * sizeof(int);

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

fa4q_status launch_hybrid_full(const HyParams& p, cudaStream_t st) {
  if (cudaFuncSetAttribute(hybrid_full_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kHySmem) !=
      cudaSuccess)
    return FA4Q_ERR_CUDA;
  const dim3 grid((p.S + kHyRows - 1) / kHyRows, p.Hq, p.B);
  hybrid_full_kernel<<<grid, kHyThreads, kHySmem, st>>>(p);
  return launch_status();
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
