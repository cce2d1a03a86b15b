// decode.cu - one-token decode attention over the hybrid FP4 / BF16 KV cache (sm_100a).
//
// What it computes, per (sequence b, q-head h):
//   out = softmax(q K^T * sm_scale) V  over the union of
//         FP4 paged remainder (dequantised inside the scan; excluded slots masked),
//         BF16 vertical-line set, BF16 window;  every key counted once, one softmax.
// Sources: HyQuant (Hybrid-Precision Quantization for LLM Attention) - vertical-line and
// window tokens in full precision, 4-bit remainder, dequantisation fused into the decode
// scan so no full-precision cache is materialised; BitDecoding-FP4, "System-Level
// Optimization" - paged cache behind a block table, query MMAs stacked over the pages.
//
// Design: the scan is HBM-bound (1 byte of cache feeds ~4 multiply-adds per GQA head), so
// the kernel streams each 64-token page once with coalesced 16-byte loads, dequantises in
// registers (E2M1 x E4M3 products are exact in FP16) straight into mma.sync m16n8k16
// fragments (FP32 accumulate), and never stages dequantised data in shared memory.
//   scores  D[16 x 8] = Q[16 heads x 16 dims] * K^T[16 dims x 8 tokens]
//   output  O[16 x 8] += P[16 heads x 16 tokens] * V[16 tokens x 8 channels]
// The token order inside a page is permuted so that the score accumulators of a thread are
// exactly its P fragment for the output MMA (no shuffles), and every V^T fragment is one
// 8-byte load covering a whole 16-token scale block.
// Grid: (split, kv-head, sequence); each warp runs its own online softmax over a strided
// subset of the split's 64-token chunks; warps merge in shared memory, splits merge in the
// combine kernel (log-sum-exp weighted).
#include <math.h>

#include "fa4q_common.cuh"
#include "fa4q_internal.h"

namespace fa4q {

static __device__ uint32_t g_decode_status;

constexpr int kDecWarps = 4;
constexpr int kDecD = 128;
constexpr float kDecLog2e = 1.4426950408889634f;

struct DecParams {
  const uint16_t* q;
  const uint8_t* kp;
  const uint8_t* ksf;
  const uint8_t* vp;
  const uint8_t* vsf;
  const int32_t* table;
  const int32_t* fp4_len;
  const uint64_t* excl;
  const uint16_t* hp_k;
  const uint16_t* hp_v;
  const int32_t* hp_count;
  const uint16_t* win_k;
  const uint16_t* win_v;
  const int32_t* win_len;
  int B, Hq, Hkv, G, max_pages, max_hp, W;
  float sc_fp4, sc_bf16, g_v;
  int n_ch_fp4, n_ch_hp, n_ch_win, chunks_per_split, splits;
  float* ws;
  uint16_t* out;
};

FA4Q_DEVINL void mma_f16(float (&d)[4], uint32_t a0, uint32_t a2, uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(0u), "r"(a2), "r"(0u), "r"(b0), "r"(b1));
}

// two E2M1 codes (one byte, low nibble first) -> f16x2 (low half = low nibble)
FA4Q_DEVINL uint32_t e2m1x2_to_f16x2(uint32_t byte) {
  uint32_t out;
  asm("{\n\t.reg .b8 b;\n\tcvt.u8.u32 b, %1;\n\tcvt.rn.f16x2.e2m1x2 %0, b;\n\t}" : "=r"(out) : "r"(byte));
  return out;
}

// two E4M3 bytes (low byte first) -> f16x2
FA4Q_DEVINL uint32_t e4m3x2_to_f16x2(uint32_t two) {
  uint32_t out;
  const uint16_t h = static_cast<uint16_t>(two);
  asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(out) : "h"(h));
  return out;
}

FA4Q_DEVINL uint32_t hmul2(uint32_t a, uint32_t b) {
  uint32_t d;
  asm("mul.rn.f16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
  return d;
}

FA4Q_DEVINL uint32_t f32x2_to_f16x2(float lo, float hi) {
  uint32_t d;
  asm("cvt.rn.f16x2.f32 %0, %1, %2;" : "=r"(d) : "f"(hi), "f"(lo));
  return d;
}

FA4Q_DEVINL uint32_t bf16x2_to_f16x2(uint32_t w) {
  return f32x2_to_f16x2(__uint_as_float(w << 16), __uint_as_float(w & 0xFFFF0000u));
}

FA4Q_DEVINL float ex2f(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__global__ void __launch_bounds__(kDecWarps * 32, 3) decode_split_kernel(const DecParams p) {
  __shared__ float s_o[kDecWarps][8][kDecD];
  __shared__ float s_m[kDecWarps][8];
  __shared__ float s_l[kDecWarps][8];
  const int split = blockIdx.x, hk = blockIdx.y, b = blockIdx.z;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = lane >> 2, t = lane & 3;
  const int G = p.G;
  const int bh = b * p.Hkv + hk;

  // ---- query fragments: row g = GQA head g of this kv-head (rows >= G are zero)
  uint32_t qa[8][2];
  {
    const bool real = g < G;
    const uint16_t* qrow = p.q + ((int64_t)b * p.Hq + hk * G + (real ? g : 0)) * kDecD;
#pragma unroll
    for (int kc = 0; kc < 8; ++kc) {
      const int d0 = 32 * t + 4 * kc;
      const uint32_t w01 = real ? *reinterpret_cast<const uint32_t*>(qrow + d0) : 0u;
      const uint32_t w23 = real ? *reinterpret_cast<const uint32_t*>(qrow + d0 + 2) : 0u;
      qa[kc][0] = bf16x2_to_f16x2(w01);
      qa[kc][1] = bf16x2_to_f16x2(w23);
    }
  }
  float o[16][4];
#pragma unroll
  for (int i = 0; i < 16; ++i) o[i][0] = o[i][1] = o[i][2] = o[i][3] = 0.0f;
  float m = -INFINITY, l = 0.0f;

  const int n_fp4 = min(p.fp4_len[b], p.max_pages * 64);
  const int n_hp = p.hp_count ? min(p.hp_count[bh], p.max_hp) : 0;
  const int n_win = p.win_len ? min(p.win_len[b], p.W) : 0;
  const int total_chunks = p.n_ch_fp4 + p.n_ch_hp + p.n_ch_win;
  const int c_begin = split * p.chunks_per_split;
  const int c_end = min(total_chunks, c_begin + p.chunks_per_split);

  for (int ch = c_begin + warp; ch < c_end; ch += kDecWarps) {
    // ---- classify the chunk; skip chunks with no valid key
    int kind, base, nvalid;
    if (ch < p.n_ch_fp4) {
      kind = 0; base = ch * 64; nvalid = n_fp4 - base;
    } else if (ch < p.n_ch_fp4 + p.n_ch_hp) {
      kind = 1; base = (ch - p.n_ch_fp4) * 64; nvalid = n_hp - base;
    } else {
      kind = 2; base = (ch - p.n_ch_fp4 - p.n_ch_hp) * 64; nvalid = n_win - base;
    }
    if (nvalid <= 0) continue;
    uint64_t vmask = nvalid >= 64 ? ~0ull : ((1ull << nvalid) - 1ull);
    const uint8_t* kpage = nullptr;
    const uint8_t* ksfp = nullptr;
    const uint8_t* vpage = nullptr;
    const uint8_t* vsfp = nullptr;
    const uint16_t* kb16 = nullptr;
    const uint16_t* vb16 = nullptr;
    if (kind == 0) {
      const int64_t phys = p.table[(int64_t)b * p.max_pages + ch];
      if (p.excl) vmask &= ~p.excl[(int64_t)bh * p.max_pages + ch];
      kpage = p.kp + (phys * p.Hkv + hk) * 64 * (kDecD / 2);
      ksfp = p.ksf + (phys * p.Hkv + hk) * 64 * (kDecD / 16);
      vpage = p.vp + (phys * p.Hkv + hk) * kDecD * 32;
      vsfp = p.vsf + (phys * p.Hkv + hk) * kDecD * 4;
    } else if (kind == 1) {
      kb16 = p.hp_k + ((int64_t)bh * p.max_hp + base) * kDecD;
      vb16 = p.hp_v + ((int64_t)bh * p.max_hp + base) * kDecD;
    } else {
      kb16 = p.win_k + ((int64_t)bh * p.W + base) * kDecD;
      vb16 = p.win_v + ((int64_t)bh * p.W + base) * kDecD;
    }
    if (vmask == 0ull) continue;
    const float sc = kind == 0 ? p.sc_fp4 : p.sc_bf16;

    // ---- scores for 8 groups (c, sigma): thread's own token in group = 16(g>>1)+4c+2sigma+(g&1)
    float s[8][2];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int c = i >> 1, sg = i & 1;
      const int tok = 16 * (g >> 1) + 4 * c + 2 * sg + (g & 1);
      uint32_t bfr[8][2];
      if (kind == 0) {
        const uint4 kw = *reinterpret_cast<const uint4*>(kpage + tok * 64 + 16 * t);
        const uint32_t sfw = *reinterpret_cast<const uint16_t*>(ksfp + tok * 8 + 2 * t);
        const uint32_t sf2 = e4m3x2_to_f16x2(sfw);
        const uint32_t sfa = __byte_perm(sf2, 0, 0x1010), sfb = __byte_perm(sf2, 0, 0x3232);
        const uint32_t words[4] = {kw.x, kw.y, kw.z, kw.w};
#pragma unroll
        for (int kc = 0; kc < 8; ++kc) {
          const uint32_t wd = words[kc >> 1];
          const int sh = (kc & 1) * 16;
          const uint32_t scl = kc < 4 ? sfa : sfb;
          bfr[kc][0] = hmul2(e2m1x2_to_f16x2((wd >> sh) & 0xFF), scl);
          bfr[kc][1] = hmul2(e2m1x2_to_f16x2((wd >> (sh + 8)) & 0xFF), scl);
        }
      } else {
        const uint16_t* kr = kb16 + (int64_t)tok * kDecD + 32 * t;
        if (tok < nvalid) {
#pragma unroll
          for (int kc = 0; kc < 8; ++kc) {
            const uint2 w = *reinterpret_cast<const uint2*>(kr + 4 * kc);
            bfr[kc][0] = bf16x2_to_f16x2(w.x);
            bfr[kc][1] = bf16x2_to_f16x2(w.y);
          }
        } else {
#pragma unroll
          for (int kc = 0; kc < 8; ++kc) bfr[kc][0] = bfr[kc][1] = 0u;
        }
      }
      float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int kc = 0; kc < 8; ++kc) mma_f16(acc, qa[kc][0], qa[kc][1], bfr[kc][0], bfr[kc][1]);
      // accumulator (row g, columns 2t, 2t+1) = tokens 16t + 4c + 2sigma + {0, 1}
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const int tk = 16 * t + 4 * c + 2 * sg + e;
        s[i][e] = ((vmask >> tk) & 1ull) ? acc[e] * sc : -INFINITY;
      }
    }
    // ---- online softmax update (row g; the 4 threads of a group share the row)
    float cmax = s[0][0];
#pragma unroll
    for (int i = 0; i < 8; ++i) cmax = fmaxf(cmax, fmaxf(s[i][0], s[i][1]));
    cmax = fmaxf(cmax, __shfl_xor_sync(0xffffffffu, cmax, 1));
    cmax = fmaxf(cmax, __shfl_xor_sync(0xffffffffu, cmax, 2));
    const float m_new = fmaxf(m, cmax);
    const float alpha = ex2f(m - m_new);
    const float gv = kind == 0 ? p.g_v : 1.0f;
    uint32_t pa[8];
    float psum = 0.0f;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const float p0 = ex2f(s[i][0] - m_new), p1 = ex2f(s[i][1] - m_new);
      psum += p0 + p1;
      pa[i] = f32x2_to_f16x2(p0 * gv, p1 * gv);
    }
    l = l * alpha + psum;
    m = m_new;
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      o[i][0] *= alpha;
      o[i][1] *= alpha;
    }
    // ---- O += P V: channel 8*nt + g, tokens 16t + 4c + {0..3}
#pragma unroll
    for (int nt = 0; nt < 16; ++nt) {
      const int chn = 8 * nt + g;
      uint32_t vb[4][2];
      if (kind == 0) {
        const uint2 vw = *reinterpret_cast<const uint2*>(vpage + chn * 32 + 8 * t);
        const uint32_t sfv = vsfp[chn * 4 + t];
        const uint32_t s2 = e4m3x2_to_f16x2(sfv | (sfv << 8));
        const uint32_t words[2] = {vw.x, vw.y};
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          const uint32_t wd = words[c >> 1];
          const int sh = (c & 1) * 16;
          vb[c][0] = hmul2(e2m1x2_to_f16x2((wd >> sh) & 0xFF), s2);
          vb[c][1] = hmul2(e2m1x2_to_f16x2((wd >> (sh + 8)) & 0xFF), s2);
        }
      } else {
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          uint32_t hv[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const int tk = 16 * t + 4 * c + e;
            hv[e] = tk < nvalid ? static_cast<uint32_t>(vb16[(int64_t)tk * kDecD + chn]) : 0u;
          }
          vb[c][0] = bf16x2_to_f16x2(hv[0] | (hv[1] << 16));
          vb[c][1] = bf16x2_to_f16x2(hv[2] | (hv[3] << 16));
        }
      }
#pragma unroll
      for (int c = 0; c < 4; ++c) mma_f16(o[nt], pa[2 * c], pa[2 * c + 1], vb[c][0], vb[c][1]);
    }
  }
  // ---- merge the 4 warps of the CTA
  l += __shfl_xor_sync(0xffffffffu, l, 1);
  l += __shfl_xor_sync(0xffffffffu, l, 2);
  if (g < G) {
#pragma unroll
    for (int nt = 0; nt < 16; ++nt) {
      s_o[warp][g][8 * nt + 2 * t] = o[nt][0];
      s_o[warp][g][8 * nt + 2 * t + 1] = o[nt][1];
    }
    if (t == 0) {
      s_m[warp][g] = m;
      s_l[warp][g] = l;
    }
  }
  __syncthreads();
  const int stride = kDecD + 2;
  for (int idx = threadIdx.x; idx < G * kDecD; idx += blockDim.x) {
    const int hh = idx / kDecD, c = idx % kDecD;
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < kDecWarps; ++w) M = fmaxf(M, s_m[w][hh]);
    float acc = 0.0f, lsum = 0.0f;
    if (M != -INFINITY) {
#pragma unroll
      for (int w = 0; w < kDecWarps; ++w) {
        const float wt = ex2f(s_m[w][hh] - M);
        acc += wt * s_o[w][hh][c];
        lsum += wt * s_l[w][hh];
      }
    }
    float* dst = p.ws + (((int64_t)b * p.Hq + hk * G + hh) * p.splits + split) * stride;
    dst[2 + c] = acc;
    if (c == 0) {
      dst[0] = M;
      dst[1] = lsum;
    }
  }
}

// one warp per (sequence, q-head): log-sum-exp merge of the split partials
__global__ void decode_combine_kernel(const float* __restrict__ ws, int n_rows, int splits,
                                      uint16_t* __restrict__ out) {
  const int row = blockIdx.x * (blockDim.x / 32) + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (row >= n_rows) return;
  const int stride = kDecD + 2;
  const float* base = ws + (int64_t)row * splits * stride;
  float M = -INFINITY;
  for (int s = lane; s < splits; s += 32) M = fmaxf(M, base[s * stride]);
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, off));
  float acc[4] = {0.f, 0.f, 0.f, 0.f};
  float lsum = 0.0f;
  if (M != -INFINITY) {
    for (int s = 0; s < splits; ++s) {
      const float wt = ex2f(base[s * stride] - M);
      lsum += wt * base[s * stride + 1];
#pragma unroll
      for (int i = 0; i < 4; ++i) acc[i] += wt * base[s * stride + 2 + lane * 4 + i];
    }
  }
  const float inv = lsum > 0.0f ? 1.0f / lsum : 0.0f;
  __nv_bfloat162 lo = __floats2bfloat162_rn(acc[0] * inv, acc[1] * inv);
  __nv_bfloat162 hi = __floats2bfloat162_rn(acc[2] * inv, acc[3] * inv);
  uint2 w;
  w.x = *reinterpret_cast<uint32_t*>(&lo);
  w.y = *reinterpret_cast<uint32_t*>(&hi);
  *reinterpret_cast<uint2*>(out + (int64_t)row * kDecD + lane * 4) = w;
}

cudaError_t decode_status_fetch(cudaStream_t st, uint32_t* host_word) {
  cudaError_t e = cudaMemcpyFromSymbolAsync(host_word, g_decode_status, sizeof(uint32_t), 0,
                                            cudaMemcpyDeviceToHost, st);
  if (e != cudaSuccess) return e;
  const uint32_t zero = 0;
  e = cudaMemcpyToSymbolAsync(g_decode_status, &zero, sizeof(uint32_t), 0, cudaMemcpyHostToDevice, st);
  if (e != cudaSuccess) return e;
  return cudaStreamSynchronize(st);
}

static int decode_chunks(int max_pages, int max_hp, int W) {
  return max_pages + (max_hp + 63) / 64 + (W + 63) / 64;
}

static int decode_auto_splits(int B, int Hkv, int chunks) {
  const int target_ctas = 148 * 3 * 4;                    // ~4 waves of 3 CTAs per SM
  int s = (target_ctas + B * Hkv - 1) / (B * Hkv);
  s = s < 1 ? 1 : s;
  const int max_s = (chunks + kDecWarps - 1) / kDecWarps;  // at least a chunk per warp
  return s > max_s ? max_s : s;
}

}  // namespace fa4q

using namespace fa4q;

extern "C" size_t fa4q_decode_workspace_size(int B, int Hq, int Hkv, int d, int max_pages, int num_splits) {
  if (B <= 0 || Hq <= 0 || Hkv <= 0 || d != kDecD || max_pages < 0) return 0;
  // the hp set and window sizes only enter through the split count; size for the worst case
  const int splits = num_splits > 0 ? num_splits : decode_auto_splits(B, Hkv, max_pages + 64);
  return (size_t)B * Hq * splits * (kDecD + 2) * sizeof(float);
}

extern "C" fa4q_status fa4q_decode(const void* q, const uint8_t* k_pages, const uint8_t* k_sf,
                                   const uint8_t* vt_pages, const uint8_t* vt_sf,
                                   const int32_t* block_table, const int32_t* fp4_len,
                                   const uint64_t* excl_mask, const void* hp_k, const void* hp_v,
                                   const int32_t* hp_count, const void* win_k, const void* win_v,
                                   const int32_t* win_len, int B, int Hq, int Hkv, int d,
                                   int max_pages, int max_hp, int W, fa4q_format fmt, float g_k,
                                   float g_v, float sm_scale, void* out, void* workspace,
                                   size_t workspace_bytes, int num_splits, void* stream) {
  if (fmt != FA4Q_NVFP4 && fmt != FA4Q_MXFP4) return FA4Q_ERR_INVALID_ARG;
  if (fmt == FA4Q_MXFP4) return FA4Q_ERR_UNSUPPORTED;
  if (!q || !out || !fp4_len || !workspace) return FA4Q_ERR_INVALID_ARG;
  if (B <= 0 || Hq <= 0 || Hkv <= 0 || Hq % Hkv != 0) return FA4Q_ERR_INVALID_ARG;
  if (Hq / Hkv > 8) return FA4Q_ERR_UNSUPPORTED;
  if (d != kDecD) return FA4Q_ERR_UNSUPPORTED;
  if (max_pages < 0 || max_hp < 0 || W < 0 || num_splits < 0) return FA4Q_ERR_INVALID_ARG;
  if (max_pages > 0 && (!k_pages || !k_sf || !vt_pages || !vt_sf || !block_table))
    return FA4Q_ERR_INVALID_ARG;
  if (max_hp > 0 && (!hp_k || !hp_v || !hp_count)) return FA4Q_ERR_INVALID_ARG;
  if (W > 0 && (!win_k || !win_v || !win_len)) return FA4Q_ERR_INVALID_ARG;
  if (!(g_k > 0.0f) || !(g_v > 0.0f)) return FA4Q_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(out) || (k_pages && !aligned16(k_pages)) ||
      (vt_pages && !aligned16(vt_pages)) || (hp_k && !aligned16(hp_k)) ||
      (hp_v && !aligned16(hp_v)) || (win_k && !aligned16(win_k)) || (win_v && !aligned16(win_v)) ||
      !aligned16(workspace))
    return FA4Q_ERR_INVALID_ARG;
  if (B > 65535 || Hkv > 65535) return FA4Q_ERR_UNSUPPORTED;
  const int chunks = decode_chunks(max_pages, max_hp, W);
  const int splits = num_splits > 0 ? num_splits : decode_auto_splits(B, Hkv, chunks);
  const size_t need = (size_t)B * Hq * splits * (kDecD + 2) * sizeof(float);
  if (workspace_bytes < need) return FA4Q_ERR_INVALID_ARG;
  DecParams p;
  p.q = (const uint16_t*)q;
  p.kp = k_pages;
  p.ksf = k_sf;
  p.vp = vt_pages;
  p.vsf = vt_sf;
  p.table = block_table;
  p.fp4_len = fp4_len;
  p.excl = excl_mask;
  p.hp_k = (const uint16_t*)hp_k;
  p.hp_v = (const uint16_t*)hp_v;
  p.hp_count = max_hp > 0 ? hp_count : nullptr;
  p.win_k = (const uint16_t*)win_k;
  p.win_v = (const uint16_t*)win_v;
  p.win_len = W > 0 ? win_len : nullptr;
  p.B = B;
  p.Hq = Hq;
  p.Hkv = Hkv;
  p.G = Hq / Hkv;
  p.max_pages = max_pages;
  p.max_hp = max_hp;
  p.W = W;
  const float sms = sm_scale > 0.0f ? sm_scale : 1.0f / sqrtf((float)d);
  p.sc_fp4 = sms * g_k * kDecLog2e;
  p.sc_bf16 = sms * kDecLog2e;
  p.g_v = g_v;
  p.n_ch_fp4 = max_pages;
  p.n_ch_hp = (max_hp + 63) / 64;
  p.n_ch_win = (W + 63) / 64;
  p.splits = splits;
  p.chunks_per_split = (chunks + splits - 1) / splits;
  p.ws = static_cast<float*>(workspace);
  p.out = static_cast<uint16_t*>(out);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  dim3 grid(splits, Hkv, B);
  decode_split_kernel<<<grid, kDecWarps * 32, 0, st>>>(p);
  const int rows = B * Hq;
  decode_combine_kernel<<<(rows + 3) / 4, 128, 0, st>>>(p.ws, rows, splits, p.out);
  return launch_status();
}

// =======================================================================================
// fa4q_decode_noalloc: the same decode with its split partials in a static device array
// =======================================================================================
#include <mutex>

namespace fa4q {

// Upper bound of the static scratch: every GPU that loads the library holds these 8 MiB
// until the process exits.  Enough for the split partials of B * Hq <= 1024 query heads at
// the automatic split count of a 32768-key cache (about 3.7 MiB at d = 128).
constexpr size_t kNoAllocScratchBytes = size_t(8) << 20;
static __device__ __align__(256) float g_decode_scratch[kNoAllocScratchBytes / sizeof(float)];

// Device address of g_decode_scratch, looked up once per device with that device current.
// (In host code the symbol is only a host-side handle; passing it to a kernel directly
// would address the wrong memory.)
constexpr int kMaxDevices = 64;
static std::mutex g_scratch_mu;
static void* g_scratch_addr[kMaxDevices] = {};

static fa4q_status scratch_address(void** out) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) return FA4Q_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return FA4Q_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  if (g_scratch_addr[dev] == nullptr) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_decode_scratch) != cudaSuccess || p == nullptr) return FA4Q_ERR_CUDA;
    g_scratch_addr[dev] = p;
  }
  *out = g_scratch_addr[dev];
  return FA4Q_OK;
}

}  // namespace fa4q

extern "C" fa4q_status fa4q_decode_noalloc(const void* q, const uint8_t* k_pages, const uint8_t* k_sf,
                                           const uint8_t* vt_pages, const uint8_t* vt_sf,
                                           const int32_t* block_table, const int32_t* fp4_len,
                                           const uint64_t* excl_mask, const void* hp_k,
                                           const void* hp_v, const int32_t* hp_count,
                                           const void* win_k, const void* win_v,
                                           const int32_t* win_len, int B, int Hq, int Hkv, int d,
                                           int max_pages, int max_hp, int W, fa4q_format fmt,
                                           float g_k, float g_v, float sm_scale, void* out,
                                           int num_splits, void* stream) {
  if (d != kDecD) return FA4Q_ERR_UNSUPPORTED;
  if (B <= 0 || Hq <= 0 || Hkv <= 0 || max_pages < 0 || max_hp < 0 || W < 0 || num_splits < 0)
    return FA4Q_ERR_INVALID_ARG;
  const size_t per_split = (size_t)B * Hq * (kDecD + 2) * sizeof(float);
  int splits = num_splits;
  if (splits == 0) {
    splits = decode_auto_splits(B, Hkv, decode_chunks(max_pages, max_hp, W));
    const size_t cap = kNoAllocScratchBytes / per_split;
    if (cap < 1) return FA4Q_ERR_UNSUPPORTED;  // even one split's partials exceed the array
    if ((size_t)splits > cap) splits = (int)cap;
  } else if (per_split * (size_t)splits > kNoAllocScratchBytes) {
    return FA4Q_ERR_UNSUPPORTED;               // the requested splits need more than 8 MiB
  }
  void* scratch = nullptr;
  const fa4q_status st = scratch_address(&scratch);
  if (st != FA4Q_OK) return st;
  return fa4q_decode(q, k_pages, k_sf, vt_pages, vt_sf, block_table, fp4_len, excl_mask, hp_k, hp_v,
                     hp_count, win_k, win_v, win_len, B, Hq, Hkv, d, max_pages, max_hp, W, fmt, g_k,
                     g_v, sm_scale, out, scratch, kNoAllocScratchBytes, splits, stream);
}
