// quantize.cu - blockwise E2M1 quantisation kernels and their C-ABI entry points.
//
// Block microscaling: BitDecoding-FP4 (Algorithm-System Co-Design for Native FP4 KV Cache
// Decoding), "The KV Cache Bottleneck in Long-Context LLM Serving" - blocks share one scale,
// elements are E2M1, MX blocks have 32 elements with E8M0 scales, NVFP4 blocks 16 elements
// with E4M3 scales.  Scale bound: MXAttention, Abstract (OCP MXFP4 and the universal optimal
// scaling bound Qmax = 7.25).  Smoothing: HiFA4, Abstract (Smooth-QK multiplier before
// quantisation).  Hybrid cache: HyQuant (vertical-line tokens kept in full precision; their
// 4-bit slots are zero here).
//
// All three kernels are HBM-bound streaming passes: 16-byte coalesced loads of bf16,
// FP32 scale arithmetic in the fixed IEEE order, packed E2M1 stores.
#include <math.h>
#include <stdio.h>

#include "fa4q_common.cuh"
#include "fa4q_internal.h"

namespace fa4q {

// ---------------------------------------------------------------------------------------
// per-block quantisation (FP32 values in registers)
// ---------------------------------------------------------------------------------------
// x / d rounded to nearest (IEEE), given r = 1/d rounded to nearest and d > 0: the product
// q = RN(x r) is within an ulp of x/d, the remainder x - d q is exact in one FMA, and
// RN(q + (x - d q) r) is the correctly rounded quotient (Markstein's theorem on FMA
// division).  Quotients in the subnormal range may differ from IEEE division; they lie far
// below the smallest E2M1 rounding threshold (0.25), so the codes do not.  The sign is
// taken from x so that -0 stays -0; a product that overflows is returned as the infinity
// IEEE division gives (the correction step would turn it into NaN).
FA4Q_DEVINL float div_rn_recip(float x, float d, float r) {
  const float q = __fmul_rn(x, r);
  if (isinf(q)) return q;
  const float e = __fmaf_rn(-q, d, x);
  return copysignf(__fmaf_rn(e, r, q), x);
}

// NVFP4: s = UE4M3(amax / (qmax*g)); y = x / (float(s)*g); 16 elements -> 8 bytes.
FA4Q_DEVINL uint32_t quant_block16_nvfp4(const float* v, float denom, float g, uint2& packed) {
  float amax = 0.0f;
#pragma unroll
  for (int i = 0; i < 16; ++i) amax = fmaxf(amax, fabsf(v[i]));
  const float t = __fdiv_rn(amax, denom);
  const uint32_t s = ue4m3_encode(t);
  const float div = __fmul_rn(ue4m3_decode(s), g);
  float y[16];
  if (div > 0.0f) {
    const float r = __frcp_rn(div);
#pragma unroll
    for (int i = 0; i < 16; ++i) y[i] = div_rn_recip(v[i], div, r);
  } else {
#pragma unroll
    for (int i = 0; i < 16; ++i) y[i] = v[i] * 0.0f;
  }
  packed.x = e2m1x8(y[0], y[1], y[2], y[3], y[4], y[5], y[6], y[7]);
  packed.y = e2m1x8(y[8], y[9], y[10], y[11], y[12], y[13], y[14], y[15]);
  return s;
}

// MXFP4: e from the OCP or UOS rule, y = x * 2^-e (exact); 32 elements -> 16 bytes.
FA4Q_DEVINL uint32_t quant_block32_mxfp4(const float* v, float qmax, uint4& packed) {
  float amax = 0.0f;
#pragma unroll
  for (int i = 0; i < 32; ++i) amax = fmaxf(amax, fabsf(v[i]));
  const int e = mx_exponent(amax, qmax);
  const float inv = exp2i(-e);
  float y[32];
#pragma unroll
  for (int i = 0; i < 32; ++i) y[i] = v[i] * inv;
  packed.x = e2m1x8(y[0], y[1], y[2], y[3], y[4], y[5], y[6], y[7]);
  packed.y = e2m1x8(y[8], y[9], y[10], y[11], y[12], y[13], y[14], y[15]);
  packed.z = e2m1x8(y[16], y[17], y[18], y[19], y[20], y[21], y[22], y[23]);
  packed.w = e2m1x8(y[24], y[25], y[26], y[27], y[28], y[29], y[30], y[31]);
  return static_cast<uint32_t>(e + 127);
}

FA4Q_DEVINL void load_bf16x8(const uint16_t* p, float* out) {
  const uint4 u = *reinterpret_cast<const uint4*>(p);
  const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    out[2 * i] = __uint_as_float(w[i] << 16);
    out[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
  }
}

// Byte offset of (row r, scale column k) in one matrix's tiled scale array with nG groups.
FA4Q_DEVINL int64_t sf_tiled_offset(int64_t r, int64_t k, int64_t nG) {
  return ((r >> 7) * nG + (k >> 2)) * 512 + (r & 31) * 16 + ((r & 127) >> 5) * 4 + (k & 3);
}

// ---------------------------------------------------------------------------------------
// AXIS_INNER: one thread per block (enough independent loads in flight to stream at HBM
// rate); in the tiled layout the index space also covers the padding rows and scale columns,
// whose bytes are written as the scale of an all-zero block (0)
// ---------------------------------------------------------------------------------------
struct InnerArgs {
  const uint16_t* x;
  int64_t rows, cols, row_stride;
  float qmax, g;
  const float* mul;
  int64_t mheads, mratio;
  int tiled;
  uint8_t* packed;
  uint8_t* sf;
};

// Geometry of one group's scale space: `nblk` real blocks per row, `ncol_sp` scale slots per
// row (the tiled layout pads the columns to whole 128-element tiles), `rows_sp` rows (padded
// to 128 when tiled).
struct InnerGeom {
  int nblk, rows_i, rows_sp, nG, ncol_sp;
  int64_t sf_group_bytes;
};

template <int BLK>
FA4Q_DEVINL InnerGeom inner_geom(const InnerArgs& a) {
  InnerGeom q;
  q.nblk = static_cast<int>(a.cols / BLK);
  q.rows_i = static_cast<int>(a.rows);
  q.rows_sp = a.tiled ? ((q.rows_i + 127) / 128) * 128 : q.rows_i;
  q.nG = a.tiled ? static_cast<int>((a.cols + 127) / 128) * (32 / BLK) : 0;
  q.ncol_sp = a.tiled ? q.nG * 4 : q.nblk;
  q.sf_group_bytes = a.tiled ? (int64_t)((q.rows_i + 127) / 128) * q.nG * 512 : (int64_t)q.rows_i * q.nblk;
  return q;
}

// bf16 block (r, kb) of group gi -> FP32, times the Smooth-QK multiplier when given
template <int BLK>
FA4Q_DEVINL void inner_load(const InnerArgs& a, int64_t gi, int r, int kb, float* v) {
  const uint16_t* src = a.x + (gi * a.rows + r) * a.row_stride + kb * BLK;
#pragma unroll
  for (int c = 0; c < BLK; c += 8) load_bf16x8(src + c, v + c);
  if (a.mul != nullptr) {
    const int mrow = (static_cast<int>(gi) % static_cast<int>(a.mheads)) / static_cast<int>(a.mratio);
    const float* m = a.mul + (int64_t)mrow * a.cols + kb * BLK;
#pragma unroll
    for (int c = 0; c < BLK; c += 4) {
      const float4 mm = *reinterpret_cast<const float4*>(m + c);
      v[c] = __fmul_rn(v[c], mm.x);
      v[c + 1] = __fmul_rn(v[c + 1], mm.y);
      v[c + 2] = __fmul_rn(v[c + 2], mm.z);
      v[c + 3] = __fmul_rn(v[c + 3], mm.w);
    }
  }
}

// quantise block (r, kb) (when `real`) and write its scale slot (always)
template <int BLK>
FA4Q_DEVINL void inner_store(const InnerArgs& a, const InnerGeom& q, int64_t gi, int r, int kb, const float* v,
                             bool real) {
  uint32_t s = 0;
  if (real) {
    uint8_t* dst = a.packed + (gi * a.rows + r) * (a.cols / 2) + kb * (BLK / 2);
    if constexpr (BLK == 16) {
      uint2 p;
      s = quant_block16_nvfp4(v, __fmul_rn(a.qmax, a.g), a.g, p);
      *reinterpret_cast<uint2*>(dst) = p;
    } else {
      uint4 p;
      s = quant_block32_mxfp4(v, a.qmax, p);
      *reinterpret_cast<uint4*>(dst) = p;
    }
  }
  if (a.tiled)
    a.sf[gi * q.sf_group_bytes + sf_tiled_offset(r, kb, q.nG)] = (uint8_t)s;
  else
    a.sf[gi * q.sf_group_bytes + (int64_t)r * q.nblk + kb] = (uint8_t)s;
}

// flat slots 2*pair and 2*pair + 1 of a group, each decoded to its own row and block (a row
// with an odd number of slots ends inside a pair), both loads issued before either block is
// quantised (NVFP4: twice the bytes in flight per thread at little register cost; MXFP4
// blocks are already 64 bytes and run one per thread)
template <int BLK>
FA4Q_DEVINL void quant_inner_pair(const InnerArgs& a, int64_t gi, int pair) {
  const InnerGeom q = inner_geom<BLK>(a);
  const int total = q.rows_sp * q.ncol_sp;
  const int idx = 2 * pair;
  if (idx >= total) return;
  const int r0 = idx / q.ncol_sp, kb0 = idx - r0 * q.ncol_sp;
  const bool has1 = idx + 1 < total;
  const int r1 = kb0 + 1 < q.ncol_sp ? r0 : r0 + 1, kb1 = kb0 + 1 < q.ncol_sp ? kb0 + 1 : 0;
  const bool real0 = r0 < q.rows_i && kb0 < q.nblk, real1 = has1 && r1 < q.rows_i && kb1 < q.nblk;
  float v0[BLK], v1[BLK];
  if (real0) inner_load<BLK>(a, gi, r0, kb0, v0);
  if (real1) inner_load<BLK>(a, gi, r1, kb1, v1);
  inner_store<BLK>(a, q, gi, r0, kb0, v0, real0);
  if (has1) inner_store<BLK>(a, q, gi, r1, kb1, v1, real1);
}

// slots handled by one thread of the inner quantiser
template <int BLK>
__host__ __device__ constexpr int inner_slots_per_thread() { return BLK == 16 ? 2 : 1; }

template <int BLK>
FA4Q_DEVINL void quant_inner_work(const InnerArgs& a, int64_t gi, int unit);

// slot idx of group gi's scale space (32-bit in-group indices: no 64-bit divisions per block)
template <int BLK>
FA4Q_DEVINL void quant_inner_slot(const InnerArgs& a, int64_t gi, int idx) {
  const InnerGeom q = inner_geom<BLK>(a);
  if (idx >= q.rows_sp * q.ncol_sp) return;
  const int r = idx / q.ncol_sp;
  const int kb = idx - r * q.ncol_sp;
  const bool real = r < q.rows_i && kb < q.nblk;
  float v[BLK];
  if (real) inner_load<BLK>(a, gi, r, kb, v);
  inner_store<BLK>(a, q, gi, r, kb, v, real);
}

template <int BLK>
FA4Q_DEVINL void quant_inner_work(const InnerArgs& a, int64_t gi, int unit) {
  if constexpr (inner_slots_per_thread<BLK>() == 2) quant_inner_pair<BLK>(a, gi, unit);
  else quant_inner_slot<BLK>(a, gi, unit);
}

template <int BLK>
__global__ void __launch_bounds__(256) quant_inner_kernel(const InnerArgs a) {
  // grid: x over the work units (one or two slots) of one group's scale space, y = group
  quant_inner_work<BLK>(a, blockIdx.y, blockIdx.x * blockDim.x + threadIdx.x);
}

// ---------------------------------------------------------------------------------------
// AXIS_INNER with a Hadamard rotation of every row before quantisation (BitDecoding-FP4,
// "Outlier-Aware Key Quantization": an orthogonal Hadamard transform of the keys spreads
// channel outliers; the same transform of the queries keeps Q K^T up to the factor cols).
// Unnormalised Sylvester order, FP32 butterflies in stages h = 1, 2, ..., cols/2: the stages
// inside a block run in registers, the rest as warp shuffles between the lanes of one row
// (slots idx = r * ncol_sp + kb, so a row's ncol_sp lanes are consecutive and aligned).
// cols is 64 or 128.
// ---------------------------------------------------------------------------------------
template <int BLK>
__global__ void __launch_bounds__(256) quant_rotated_kernel(const InnerArgs a) {
  const InnerGeom q = inner_geom<BLK>(a);
  const int64_t gi = blockIdx.y;
  const int idx = blockIdx.x * blockDim.x + threadIdx.x;
  const bool in_space = idx < q.rows_sp * q.ncol_sp;
  // warps wholly past the slot space leave; a partial warp holds whole rows (the space is a
  // multiple of ncol_sp), so every lane left takes part in every shuffle below
  if (__all_sync(0xffffffffu, !in_space)) return;
  const int r = idx / q.ncol_sp;
  const int kb = idx - r * q.ncol_sp;
  const bool real = in_space && r < q.rows_i && kb < q.nblk;
  float v[BLK];
#pragma unroll
  for (int i = 0; i < BLK; ++i) v[i] = 0.0f;
  if (real) inner_load<BLK>(a, gi, r, kb, v);
#pragma unroll
  for (int h = 1; h < BLK; h *= 2)
#pragma unroll
    for (int i = 0; i < BLK; ++i)
      if ((i & h) == 0) {
        const float x0 = v[i], x1 = v[i + h];
        v[i] = __fadd_rn(x0, x1);
        v[i + h] = __fsub_rn(x0, x1);
      }
  for (int hb = 1; hb * BLK < static_cast<int>(a.cols); hb *= 2) {   // lane distance h / BLK
    const bool upper = (kb & hb) != 0;
#pragma unroll
    for (int i = 0; i < BLK; ++i) {
      const float o = __shfl_xor_sync(0xffffffffu, v[i], hb);
      v[i] = upper ? __fsub_rn(o, v[i]) : __fadd_rn(v[i], o);
    }
  }
  if (!in_space) return;
  inner_store<BLK>(a, q, gi, r, kb, v, real);
}

// ---------------------------------------------------------------------------------------
// AXIS_OUTER: blocks along tokens, transposed output.  One tile = (group, 128 tokens,
// 64 channels) handled by 128 threads t (t = 0..127) through a shared-memory transpose.
// ---------------------------------------------------------------------------------------
struct OuterArgs {
  const uint16_t* x;
  int64_t rows, cols, row_stride;
  float qmax, g;
  int tiled;
  uint8_t* packed;
  uint8_t* sf;
};

// every thread of the CTA calls this (it synchronises the CTA once); `valid` false makes the
// thread's half a no-op that still takes part in the synchronisation
// The tile holds the bf16 bit patterns (exact, half the shared memory of FP32): 64 channels
// x 130 halves, an odd number of 32-bit words per row.
constexpr int kOuterTileRow = 130;

template <int BLK>
FA4Q_DEVINL void quant_outer_tile(const OuterArgs& a, int64_t gi, int64_t tok_tile, int64_t ch_tile, int t,
                                  uint16_t (*tile)[kOuterTileRow], bool valid) {
  const int64_t tok0 = tok_tile * 128;
  const int64_t ch0 = ch_tile * 64;
  const int64_t rows_pad = (a.rows + 31) / 32 * 32;
  // load [128 tokens][64 channels] -> tile[ch][tok]
  if (valid) {
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int u = t + 128 * i;
      const int tr = u >> 3, c8 = (u & 7) * 8;
      uint4 w = make_uint4(0u, 0u, 0u, 0u);
      if (tok0 + tr < a.rows && ch0 + c8 < a.cols)
        w = *reinterpret_cast<const uint4*>(a.x + (gi * a.rows + tok0 + tr) * a.row_stride + ch0 + c8);
      const uint32_t ww[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        tile[c8 + 2 * k][tr] = static_cast<uint16_t>(ww[k] & 0xFFFFu);
        tile[c8 + 2 * k + 1][tr] = static_cast<uint16_t>(ww[k] >> 16);
      }
    }
  }
  __syncthreads();
  if (!valid) return;
  const float denom = __fmul_rn(a.qmax, a.g);
  // thread -> (channel, 4 consecutive blocks of tokens)
  constexpr int kGroupTok = 4 * BLK;                  // 64 (NVFP4) or 128 (MXFP4)
  constexpr int kGroupsPerTile = 128 / kGroupTok;     // 2 or 1
  if (t >= 64 * kGroupsPerTile) return;
  const int c = t / kGroupsPerTile;
  const int tg = t % kGroupsPerTile;
  const int64_t ch = ch0 + c;
  // channels in [cols, 128*ceil(cols/128)) are padding rows of the tiled scale layout: their
  // (all-zero) blocks give scale 0, which is written; packed data exists only for ch < cols
  const bool real_ch = ch < a.cols;
  if (!real_ch && !a.tiled) return;
  const int64_t nblk_t = rows_pad / BLK;               // blocks per channel row
  const int64_t nG = ((rows_pad + 127) / 128) * (32 / BLK);
  const int64_t sf_group_bytes = a.tiled ? ((a.cols + 127) / 128) * nG * 512 : a.cols * nblk_t;
  uint32_t sword = 0;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int lt = tg * kGroupTok + i * BLK;           // local token of the block
    const int64_t kb = (tok0 + lt) / BLK;              // block index along the channel row
    float v[BLK];
#pragma unroll
    for (int k = 0; k < BLK; ++k) v[k] = bf16_to_f32(tile[c][lt + k]);
    uint32_t s;
    uint8_t* dst = a.packed + (gi * a.cols + ch) * (rows_pad / 2) + (tok0 + lt) / 2;
    const bool inside = real_ch && tok0 + lt < rows_pad;
    if constexpr (BLK == 16) {
      uint2 p;
      s = quant_block16_nvfp4(v, denom, a.g, p);
      if (inside) *reinterpret_cast<uint2*>(dst) = p;
    } else {
      uint4 p;
      s = quant_block32_mxfp4(v, a.qmax, p);
      if (inside) *reinterpret_cast<uint4*>(dst) = p;
    }
    sword |= s << (8 * i);
    if (!a.tiled && inside) a.sf[gi * sf_group_bytes + ch * nblk_t + kb] = (uint8_t)s;
  }
  if (a.tiled) {
    const int64_t k0 = (tok0 + tg * kGroupTok) / BLK;
    *reinterpret_cast<uint32_t*>(a.sf + gi * sf_group_bytes + sf_tiled_offset(ch, k0, nG)) = sword;
  }
}

template <int BLK>
__global__ void __launch_bounds__(128) quant_outer_kernel(const OuterArgs a) {
  __shared__ uint16_t tile[64][kOuterTileRow];
  quant_outer_tile<BLK>(a, blockIdx.z, blockIdx.x, blockIdx.y, threadIdx.x, tile, true);
}

// ---------------------------------------------------------------------------------------
// Q, K (blocks along d) and V (blocks along tokens, transposed) in one launch: CTAs
// [0, n_q) take Q slots, [n_q, n_q + n_k) K slots, the rest two V tiles each (one per 128
// threads), so the small K and V work runs in the same wave as Q instead of two more launches.
// ---------------------------------------------------------------------------------------
struct QkvGrid {
  int64_t per_group_q, per_group_k;       // inner slots per group
  int64_t groups_q, groups_k, groups_v;
  int64_t n_q, n_k;                       // CTAs of the Q and K parts
  int64_t tok_tiles, ch_tiles, n_vtiles;  // V tiles: groups_v * tok_tiles * ch_tiles
};

template <int BLK>
__global__ void __launch_bounds__(256) quant_qkv_kernel(const InnerArgs aq, const InnerArgs ak,
                                                        const OuterArgs av, const QkvGrid gr) {
  extern __shared__ __align__(16) uint16_t qkv_tile[];   // [2][64][kOuterTileRow]
  const int64_t cta = blockIdx.x;
  if (cta < gr.n_q + gr.n_k) {
    const bool is_q = cta < gr.n_q;
    const int64_t flat = (is_q ? cta : cta - gr.n_q) * 256 + threadIdx.x;
    constexpr int64_t spt = inner_slots_per_thread<BLK>();
    const int64_t per = ((is_q ? gr.per_group_q : gr.per_group_k) + spt - 1) / spt;
    const int64_t gi = flat / per;
    if (gi < (is_q ? gr.groups_q : gr.groups_k)) quant_inner_work<BLK>(is_q ? aq : ak, gi, (int)(flat - gi * per));
    return;
  }
  const int half = threadIdx.x >> 7;
  const int64_t ti = 2 * (cta - gr.n_q - gr.n_k) + half;
  const bool valid = ti < gr.n_vtiles;
  const int64_t per_g = gr.tok_tiles * gr.ch_tiles;
  const int64_t gi = valid ? ti / per_g : 0, rem = valid ? ti - gi * per_g : 0;
  uint16_t(*tile)[kOuterTileRow] =
      reinterpret_cast<uint16_t(*)[kOuterTileRow]>(qkv_tile + half * 64 * kOuterTileRow);
  quant_outer_tile<BLK>(av, gi, rem / gr.ch_tiles, rem % gr.ch_tiles, threadIdx.x & 127, tile, valid);
}

// ---------------------------------------------------------------------------------------
// Paged KV quantisation: CTA = (page j, kv-head h, sequence b)
// ---------------------------------------------------------------------------------------
template <int BLK>
__global__ void __launch_bounds__(128) quant_kv_pages_kernel(
    const uint16_t* __restrict__ k, const uint16_t* __restrict__ v, int Hkv, int L, int d,
    const int32_t* __restrict__ fp4_len, const uint64_t* __restrict__ excl, const int32_t* __restrict__ table,
    int max_pages, float g_k, float g_v, uint8_t* __restrict__ k_pages, uint8_t* __restrict__ k_sf,
    uint8_t* __restrict__ vt_pages, uint8_t* __restrict__ vt_sf) {
  __shared__ float tile[128][65];                      // V^T: [channel][token]
  const int j = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int n = min(fp4_len[b], L);
  if (j * 64 >= n) return;
  const int64_t phys = table[(int64_t)b * max_pages + j];
  const uint64_t ex = excl ? excl[((int64_t)b * Hkv + h) * max_pages + j] : 0ull;
  const int t = threadIdx.x;
  const int64_t base = (((int64_t)b * Hkv + h) * L + (int64_t)j * 64) * d;
  // ---- K rows: thread -> (token, group of 4 blocks along d)
  const int ngrp = d / (4 * BLK);                      // 2 (NVFP4, d=128) / 1
  const float denom_k = __fmul_rn(6.0f, g_k);
  for (int u = t; u < 64 * ngrp; u += 128) {
    const int tok = u / ngrp, gq = u % ngrp;
    const bool valid = (j * 64 + tok < n) && !((ex >> tok) & 1ull);
    uint32_t sword = 0;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int c0 = (gq * 4 + i) * BLK;
      float vals[BLK];
      if (valid) {
#pragma unroll
        for (int c = 0; c < BLK; c += 8) load_bf16x8(k + base + (int64_t)tok * d + c0 + c, vals + c);
      } else {
#pragma unroll
        for (int c = 0; c < BLK; ++c) vals[c] = 0.0f;
      }
      uint8_t* dst = k_pages + ((phys * Hkv + h) * 64 + tok) * (d / 2) + c0 / 2;
      uint32_t s;
      if constexpr (BLK == 16) {
        uint2 p;
        s = quant_block16_nvfp4(vals, denom_k, g_k, p);
        *reinterpret_cast<uint2*>(dst) = p;
      } else {
        uint4 p;
        s = quant_block32_mxfp4(vals, 0.0f, p);
        *reinterpret_cast<uint4*>(dst) = p;
      }
      sword |= s << (8 * i);
    }
    uint8_t* sdst = k_sf + ((phys * Hkv + h) * 64 + tok) * (d / BLK) + gq * 4;
    *reinterpret_cast<uint32_t*>(sdst) = sword;
  }
  // ---- V: stage [64 tokens][d] as tile[ch][tok], invalid tokens zero
  for (int u = t; u < 64 * (d / 8); u += 128) {
    const int tok = u / (d / 8), c8 = (u % (d / 8)) * 8;
    float vals[8] = {0, 0, 0, 0, 0, 0, 0, 0};
    const bool valid = (j * 64 + tok < n) && !((ex >> tok) & 1ull);
    if (valid) load_bf16x8(v + base + (int64_t)tok * d + c8, vals);
#pragma unroll
    for (int q = 0; q < 8; ++q) tile[c8 + q][tok] = vals[q];
  }
  __syncthreads();
  const float denom_v = __fmul_rn(6.0f, g_v);
  for (int c = t; c < d; c += 128) {
    uint8_t* dst = vt_pages + ((phys * Hkv + h) * d + c) * 32;
    uint8_t* sdst = vt_sf + ((phys * Hkv + h) * d + c) * (64 / BLK);
#pragma unroll
    for (int i = 0; i < 64 / BLK; ++i) {
      float vals[BLK];
#pragma unroll
      for (int q = 0; q < BLK; ++q) vals[q] = tile[c][i * BLK + q];
      uint32_t s;
      if constexpr (BLK == 16) {
        uint2 p;
        s = quant_block16_nvfp4(vals, denom_v, g_v, p);
        *reinterpret_cast<uint2*>(dst + i * 8) = p;
      } else {
        uint4 p;
        s = quant_block32_mxfp4(vals, 0.0f, p);
        *reinterpret_cast<uint4*>(dst + i * 16) = p;
      }
      sdst[i] = (uint8_t)s;
    }
  }
}

// ---------------------------------------------------------------------------------------
// Smooth-QK calibration: CTA = kv-head, thread = channel
// ---------------------------------------------------------------------------------------
__global__ void smooth_calibrate_kernel(const uint16_t* __restrict__ q, const uint16_t* __restrict__ k,
                                        int Hq, int Hkv, int T, int d, float* __restrict__ mul_q,
                                        float* __restrict__ mul_k) {
  const int h = blockIdx.x;
  const int grp = Hq / Hkv;
  for (int c = threadIdx.x; c < d; c += blockDim.x) {
    float qm = 0.0f, km = 0.0f;
    for (int hq = h * grp; hq < (h + 1) * grp; ++hq)
      for (int t = 0; t < T; ++t) qm = fmaxf(qm, fabsf(bf16_to_f32(q[((int64_t)hq * T + t) * d + c])));
    for (int t = 0; t < T; ++t) km = fmaxf(km, fabsf(bf16_to_f32(k[((int64_t)h * T + t) * d + c])));
    const float r = __fdiv_rn(km, qm);
    int e;
    if (r != r) {
      e = 0;
    } else if (r == 0.0f) {
      e = -8;
    } else if (isinf(r)) {
      e = 8;
    } else {
      const int E1 = floor_log2(r) + 1;               // e = floor((floor(log2 r) + 1) / 2)
      e = E1 >= 0 ? E1 / 2 : -((1 - E1) / 2);
      e = e < -8 ? -8 : (e > 8 ? 8 : e);
    }
    mul_q[h * d + c] = exp2i(e);
    mul_k[h * d + c] = exp2i(-e);
  }
}

}  // namespace fa4q

using namespace fa4q;

// =======================================================================================
// C ABI
// =======================================================================================
extern "C" size_t fa4q_sf_tiled_bytes(int64_t rows, int64_t cols, fa4q_format fmt) {
  if (rows <= 0 || cols <= 0) return 0;
  const int64_t blk = fmt == FA4Q_MXFP4 ? 32 : 16;
  return (size_t)(((rows + 127) / 128) * ((cols + 127) / 128) * (32 / blk) * 512);
}

extern "C" fa4q_status fa4q_quantize(const void* x, int64_t groups, int64_t rows, int64_t cols,
                                     int64_t row_stride, fa4q_format fmt, fa4q_axis axis,
                                     float qmax, float tensor_scale, const float* smooth_mul,
                                     int64_t smooth_heads, int64_t smooth_ratio,
                                     fa4q_sf_layout sf_layout, uint8_t* packed_out,
                                     uint8_t* scales_out, void* stream) {
  if (fmt != FA4Q_NVFP4 && fmt != FA4Q_MXFP4) return FA4Q_ERR_INVALID_ARG;
  if (axis != FA4Q_AXIS_INNER && axis != FA4Q_AXIS_OUTER) return FA4Q_ERR_INVALID_ARG;
  if (sf_layout != FA4Q_SF_ROWMAJOR && sf_layout != FA4Q_SF_TILED) return FA4Q_ERR_INVALID_ARG;
  if (groups < 0 || rows < 0 || cols < 0) return FA4Q_ERR_INVALID_ARG;
  if (groups == 0 || rows == 0 || cols == 0) return FA4Q_OK;
  if (!x || !packed_out || !scales_out) return FA4Q_ERR_INVALID_ARG;
  if (row_stride < cols || row_stride % 8 != 0 || cols % 8 != 0) return FA4Q_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(packed_out)) return FA4Q_ERR_INVALID_ARG;
  if (sf_layout == FA4Q_SF_TILED && !aligned16(scales_out)) return FA4Q_ERR_INVALID_ARG;
  if (!(qmax >= 0.0f) || !isfinite(qmax)) return FA4Q_ERR_INVALID_ARG;
  const float g = fmt == FA4Q_NVFP4 ? tensor_scale : 1.0f;
  if (!(g > 0.0f) || !isfinite(g)) return FA4Q_ERR_INVALID_ARG;
  const int blk = fmt == FA4Q_MXFP4 ? 32 : 16;
  const float qm = (fmt == FA4Q_NVFP4 && qmax == 0.0f) ? 6.0f : qmax;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const int tiled = sf_layout == FA4Q_SF_TILED;
  if (axis == FA4Q_AXIS_INNER) {
    if (cols % blk != 0) return FA4Q_ERR_UNSUPPORTED;
    if (smooth_mul && (smooth_heads <= 0 || smooth_ratio <= 0 || !aligned16(smooth_mul)))
      return FA4Q_ERR_INVALID_ARG;
    const int64_t nblk = cols / blk;
    const int64_t rows_sp = tiled ? (rows + 127) / 128 * 128 : rows;
    const int64_t ncol_sp = tiled ? (cols + 127) / 128 * (32 / blk) * 4 : nblk;
    const int64_t per_group = rows_sp * ncol_sp;
    if (groups > 65535 || per_group > (int64_t)1 << 30 || rows > ((int64_t)1 << 30)) return FA4Q_ERR_UNSUPPORTED;
    const int64_t spt = blk == 16 ? inner_slots_per_thread<16>() : inner_slots_per_thread<32>();
    dim3 grid((unsigned)(((per_group + spt - 1) / spt + 255) / 256), (unsigned)groups);
    const int64_t mh = smooth_heads > 0 ? smooth_heads : 1, mr = smooth_ratio > 0 ? smooth_ratio : 1;
    const InnerArgs ia{(const uint16_t*)x, rows, cols, row_stride, qm, g, smooth_mul, mh, mr, tiled,
                       packed_out, scales_out};
    if (blk == 16)
      quant_inner_kernel<16><<<grid, 256, 0, st>>>(ia);
    else
      quant_inner_kernel<32><<<grid, 256, 0, st>>>(ia);
  } else {
    if (smooth_mul) return FA4Q_ERR_UNSUPPORTED;
    if (groups > 65535) return FA4Q_ERR_UNSUPPORTED;
    const int64_t rows_pad = (rows + 31) / 32 * 32;
    const int64_t ch_tiles = tiled ? (cols + 127) / 128 * 2 : (cols + 63) / 64;
    dim3 grid((unsigned)((rows_pad + 127) / 128), (unsigned)ch_tiles, (unsigned)groups);
    if (grid.y > 65535) return FA4Q_ERR_UNSUPPORTED;
    const OuterArgs oa{(const uint16_t*)x, rows, cols, row_stride, qm, g, tiled, packed_out, scales_out};
    if (blk == 16)
      quant_outer_kernel<16><<<grid, 128, 0, st>>>(oa);
    else
      quant_outer_kernel<32><<<grid, 128, 0, st>>>(oa);
  }
  return launch_status();
}

namespace fa4q {

// ---------------------------------------------------------------------------------------
// Dual-residual NVFP4 query tiles for the FP4 tensor-core decode (BitDecoding-FP4, "Error
// Sources": the query as the sum of two FP4 tensors, the second quantising the residual of
// the first).  Per (sequence, kv-head) group: two 128-row tiles (residual 0 and 1) whose
// rows 0..G-1 are the group's q-heads, packed [128][d/2] with tiled scale atoms, the layout
// the decode kernel reads for its query operand.
//   q1 = NVFP4(q);  r = q - deq(q1) (FP32, deq exact);  q2 = NVFP4(r)
// ---------------------------------------------------------------------------------------
// Signed E2M1 value of a 4-bit code, from its bit fields (exponent e, mantissa m):
// e = 0 -> m * 0.5, e > 0 -> 2^(e-1) * (1 + m/2).
FA4Q_DEVINL float e2m1_value(uint32_t code) {
  const uint32_t c = code & 7u, e = c >> 1, m = c & 1u;
  const uint32_t mag = e ? (((e + 126u) << 23) | (m << 22)) : (m ? 0x3F000000u : 0u);
  return __uint_as_float(mag | ((code & 8u) << 28));
}

// Query tiles of the FP4 tensor-core decode: one CTA of 128 threads per (sequence, kv-head)
// group, thread t quantising NVFP4 block t % 8 (elements 16 (t % 8) .. +15) of query head
// t / 8 of the group, first q (16-element blocks, UE4M3, tensor scale 1), then the FP32
// residual r = q - deq(q1) (exact: deq(q1) is an FP32 product).  Heads G..15 are zero rows.
// The decode reads rows 0..15 of each 128-row tile (and of its two scale atoms), so only
// those are written: 8 bytes of codes per thread and pass (a warp covers four whole rows),
// and per four blocks one 4-byte scale word gathered by shuffles.
__global__ void __launch_bounds__(128) dec_query_kernel(const uint16_t* __restrict__ q, int Hq, int Hkv,
                                                        uint8_t* __restrict__ qt, uint8_t* __restrict__ qt_sf) {
  constexpr int D = 128;
  const int grp = blockIdx.x, t = threadIdx.x, h = t >> 3, kb = t & 7, lane = t & 31;
  const int G = Hq / Hkv;
  const int b = grp / Hkv, hk = grp - b * Hkv;
  float x[16];
  if (h < G) {
    const uint16_t* src = q + ((int64_t)b * Hq + hk * G + h) * D + 16 * kb;
    load_bf16x8(src, x);
    load_bf16x8(src + 8, x + 8);
  } else {
#pragma unroll
    for (int c = 0; c < 16; ++c) x[c] = 0.0f;
  }
#pragma unroll
  for (int res = 0; res < 2; ++res) {
    uint2 pk;
    const uint32_t sc = quant_block16_nvfp4(x, 6.0f, 1.0f, pk);
    *reinterpret_cast<uint2*>(qt + ((int64_t)grp * 2 + res) * 128 * (D / 2) + h * (D / 2) + 8 * kb) = pk;
    // tiled scale layout: row h (< 32), scale column kb -> atom kb / 4, byte h * 16 + kb % 4;
    // lanes 4i..4i+3 hold one row's four bytes of an atom
    const uint32_t w = sc | (__shfl_down_sync(0xffffffffu, sc, 1) << 8) | (__shfl_down_sync(0xffffffffu, sc, 2) << 16) |
                       (__shfl_down_sync(0xffffffffu, sc, 3) << 24);
    if ((lane & 3) == 0)
      *reinterpret_cast<uint32_t*>(qt_sf + ((int64_t)grp * 2 + res) * 2 * 512 + (kb >> 2) * 512 + h * 16) = w;
    if (res == 0) {
      // residual of this block: x - code * scale (the product is exact in FP32)
      const float sv = ue4m3_decode(sc);
#pragma unroll
      for (int i = 0; i < 16; ++i)
        x[i] = __fsub_rn(x[i], e2m1_value((i < 8 ? pk.x : pk.y) >> (4 * (i & 7))) * sv);
    }
  }
}

fa4q_status launch_dec_query(const uint16_t* q, int B, int Hq, int Hkv, uint8_t* qt, uint8_t* qt_sf,
                             cudaStream_t st) {
  dec_query_kernel<<<B * Hkv, 128, 0, st>>>(q, Hq, Hkv, qt, qt_sf);
  return launch_status();
}

}  // namespace fa4q

extern "C" fa4q_status fa4q_quantize_rotated(const void* x, int64_t groups, int64_t rows, int64_t cols,
                                             int64_t row_stride, fa4q_format fmt, float qmax,
                                             float tensor_scale, const float* smooth_mul,
                                             int64_t smooth_heads, int64_t smooth_ratio,
                                             fa4q_sf_layout sf_layout, uint8_t* packed_out,
                                             uint8_t* scales_out, void* stream) {
  if (fmt != FA4Q_NVFP4 && fmt != FA4Q_MXFP4) return FA4Q_ERR_INVALID_ARG;
  if (sf_layout != FA4Q_SF_ROWMAJOR && sf_layout != FA4Q_SF_TILED) return FA4Q_ERR_INVALID_ARG;
  if (groups < 0 || rows < 0 || cols < 0) return FA4Q_ERR_INVALID_ARG;
  if (groups == 0 || rows == 0 || cols == 0) return FA4Q_OK;
  if (cols != 64 && cols != 128) return FA4Q_ERR_UNSUPPORTED;
  if (!x || !packed_out || !scales_out) return FA4Q_ERR_INVALID_ARG;
  if (row_stride < cols || row_stride % 8 != 0) return FA4Q_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(packed_out)) return FA4Q_ERR_INVALID_ARG;
  if (sf_layout == FA4Q_SF_TILED && !aligned16(scales_out)) return FA4Q_ERR_INVALID_ARG;
  if (!(qmax >= 0.0f) || !isfinite(qmax)) return FA4Q_ERR_INVALID_ARG;
  const float g = fmt == FA4Q_NVFP4 ? tensor_scale : 1.0f;
  if (!(g > 0.0f) || !isfinite(g)) return FA4Q_ERR_INVALID_ARG;
  if (smooth_mul && (smooth_heads <= 0 || smooth_ratio <= 0 || !aligned16(smooth_mul)))
    return FA4Q_ERR_INVALID_ARG;
  const int blk = fmt == FA4Q_MXFP4 ? 32 : 16;
  const float qm = (fmt == FA4Q_NVFP4 && qmax == 0.0f) ? 6.0f : qmax;
  const int tiled = sf_layout == FA4Q_SF_TILED;
  const int64_t nblk = cols / blk;
  const int64_t rows_sp = tiled ? (rows + 127) / 128 * 128 : rows;
  const int64_t ncol_sp = tiled ? (cols + 127) / 128 * (32 / blk) * 4 : nblk;
  const int64_t per_group = rows_sp * ncol_sp;
  if (groups > 65535 || per_group > (int64_t)1 << 30 || rows > ((int64_t)1 << 30)) return FA4Q_ERR_UNSUPPORTED;
  dim3 grid((unsigned)((per_group + 255) / 256), (unsigned)groups);
  const int64_t mh = smooth_heads > 0 ? smooth_heads : 1, mr = smooth_ratio > 0 ? smooth_ratio : 1;
  const InnerArgs ia{(const uint16_t*)x, rows, cols, row_stride, qm, g, smooth_mul, mh, mr, tiled,
                     packed_out, scales_out};
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (blk == 16)
    quant_rotated_kernel<16><<<grid, 256, 0, st>>>(ia);
  else
    quant_rotated_kernel<32><<<grid, 256, 0, st>>>(ia);
  return launch_status();
}

extern "C" fa4q_status fa4q_quantize_qkv(const void* q, const void* k, const void* v, int B, int Hq,
                                         int Hkv, int S_q, int S_k, int d, fa4q_format fmt, float qmax,
                                         float g_q, float g_k, float g_v, const float* mul_q,
                                         const float* mul_k, uint8_t* q_packed, uint8_t* q_sf,
                                         uint8_t* k_packed, uint8_t* k_sf, uint8_t* vt_packed,
                                         uint8_t* vt_sf, void* stream) {
  if (fmt != FA4Q_NVFP4 && fmt != FA4Q_MXFP4) return FA4Q_ERR_INVALID_ARG;
  if (!q || !k || !v || !q_packed || !q_sf || !k_packed || !k_sf || !vt_packed || !vt_sf)
    return FA4Q_ERR_INVALID_ARG;
  if (B < 0 || Hq <= 0 || Hkv <= 0 || Hq % Hkv != 0 || S_q < 0 || S_k < 0) return FA4Q_ERR_INVALID_ARG;
  if (d != 64 && d != 128) return FA4Q_ERR_UNSUPPORTED;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(q_packed) || !aligned16(k_packed) ||
      !aligned16(vt_packed) || !aligned16(q_sf) || !aligned16(k_sf) || !aligned16(vt_sf) ||
      (mul_q && !aligned16(mul_q)) || (mul_k && !aligned16(mul_k)))
    return FA4Q_ERR_INVALID_ARG;
  if (!(qmax >= 0.0f) || !isfinite(qmax)) return FA4Q_ERR_INVALID_ARG;
  const bool nv = fmt == FA4Q_NVFP4;
  if (!nv) g_q = g_k = g_v = 1.0f;
  if (!(g_q > 0.0f) || !(g_k > 0.0f) || !(g_v > 0.0f) || !isfinite(g_q) || !isfinite(g_k) || !isfinite(g_v))
    return FA4Q_ERR_INVALID_ARG;
  if (B == 0 || (S_q == 0 && S_k == 0)) return FA4Q_OK;
  const int blk = nv ? 16 : 32;
  const float qm = (nv && qmax == 0.0f) ? 6.0f : qmax;
  // inner (Q, K) slot spaces of the tiled layout, V tiles of 128 tokens x 64 channels
  const int64_t ncol_sp = (d + 127) / 128 * (32 / blk) * 4;
  QkvGrid gr;
  gr.per_group_q = (static_cast<int64_t>(S_q) + 127) / 128 * 128 * ncol_sp;
  gr.per_group_k = (static_cast<int64_t>(S_k) + 127) / 128 * 128 * ncol_sp;
  gr.groups_q = static_cast<int64_t>(B) * Hq;
  gr.groups_k = gr.groups_v = static_cast<int64_t>(B) * Hkv;
  const int64_t spt = blk == 16 ? inner_slots_per_thread<16>() : inner_slots_per_thread<32>();
  gr.n_q = S_q > 0 ? (gr.groups_q * ((gr.per_group_q + spt - 1) / spt) + 255) / 256 : 0;
  gr.n_k = S_k > 0 ? (gr.groups_k * ((gr.per_group_k + spt - 1) / spt) + 255) / 256 : 0;
  const int64_t rows_pad_v = (static_cast<int64_t>(S_k) + 31) / 32 * 32;
  gr.tok_tiles = S_k > 0 ? (rows_pad_v + 127) / 128 : 0;
  gr.ch_tiles = (d + 127) / 128 * 2;                  // tiled layout: channels padded to 128
  gr.n_vtiles = gr.groups_v * gr.tok_tiles * gr.ch_tiles;
  const int64_t n_ctas = gr.n_q + gr.n_k + (gr.n_vtiles + 1) / 2;
  if (gr.per_group_q > ((int64_t)1 << 30) || gr.per_group_k > ((int64_t)1 << 30) || n_ctas > 0x7fffffff)
    return FA4Q_ERR_UNSUPPORTED;
  if (n_ctas == 0) return FA4Q_OK;
  const InnerArgs aq{(const uint16_t*)q, S_q, d, d, qm, g_q, mul_q, Hq, Hq / Hkv, 1, q_packed, q_sf};
  const InnerArgs ak{(const uint16_t*)k, S_k, d, d, qm, g_k, mul_k, Hkv, 1, 1, k_packed, k_sf};
  const OuterArgs av{(const uint16_t*)v, S_k, d, d, qm, g_v, 1, vt_packed, vt_sf};
  const int smem = 2 * 64 * kOuterTileRow * static_cast<int>(sizeof(uint16_t));
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (blk == 16) {
    if (cudaFuncSetAttribute(quant_qkv_kernel<16>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess)
      return FA4Q_ERR_CUDA;
    quant_qkv_kernel<16><<<static_cast<unsigned>(n_ctas), 256, smem, st>>>(aq, ak, av, gr);
  } else {
    if (cudaFuncSetAttribute(quant_qkv_kernel<32>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess)
      return FA4Q_ERR_CUDA;
    quant_qkv_kernel<32><<<static_cast<unsigned>(n_ctas), 256, smem, st>>>(aq, ak, av, gr);
  }
  return launch_status();
}

extern "C" fa4q_status fa4q_smooth_calibrate(const void* q_cal, const void* k_cal, int Hq, int Hkv,
                                             int T, int d, float* mul_q, float* mul_k,
                                             void* stream) {
  if (!q_cal || !k_cal || !mul_q || !mul_k) return FA4Q_ERR_INVALID_ARG;
  if (Hq <= 0 || Hkv <= 0 || T <= 0 || d <= 0 || Hq % Hkv != 0) return FA4Q_ERR_INVALID_ARG;
  smooth_calibrate_kernel<<<Hkv, 128, 0, static_cast<cudaStream_t>(stream)>>>(
      (const uint16_t*)q_cal, (const uint16_t*)k_cal, Hq, Hkv, T, d, mul_q, mul_k);
  return launch_status();
}

extern "C" fa4q_status fa4q_quantize_kv_pages(const void* k, const void* v, int B, int Hkv, int L,
                                              int d, const int32_t* fp4_len,
                                              const uint64_t* excl_mask,
                                              const int32_t* block_table, int max_pages,
                                              fa4q_format fmt, float g_k, float g_v,
                                              uint8_t* k_pages, uint8_t* k_sf, uint8_t* vt_pages,
                                              uint8_t* vt_sf, void* stream) {
  if (fmt != FA4Q_NVFP4 && fmt != FA4Q_MXFP4) return FA4Q_ERR_INVALID_ARG;
  if (!k || !v || !fp4_len || !block_table || !k_pages || !k_sf || !vt_pages || !vt_sf)
    return FA4Q_ERR_INVALID_ARG;
  if (B <= 0 || Hkv <= 0 || L <= 0 || max_pages <= 0) return FA4Q_ERR_INVALID_ARG;
  if (d != 128) return FA4Q_ERR_UNSUPPORTED;
  if ((int64_t)max_pages * 64 < 1 || B > 65535 || Hkv > 65535) return FA4Q_ERR_UNSUPPORTED;
  if (!aligned16(k) || !aligned16(v) || !aligned16(k_pages) || !aligned16(vt_pages))
    return FA4Q_ERR_INVALID_ARG;
  const float gk = fmt == FA4Q_NVFP4 ? g_k : 1.0f, gv = fmt == FA4Q_NVFP4 ? g_v : 1.0f;
  if (!(gk > 0.0f) || !(gv > 0.0f)) return FA4Q_ERR_INVALID_ARG;
  dim3 grid(max_pages, Hkv, B);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (fmt == FA4Q_NVFP4)
    quant_kv_pages_kernel<16><<<grid, 128, 0, st>>>((const uint16_t*)k, (const uint16_t*)v, Hkv, L,
                                                    d, fp4_len, excl_mask, block_table, max_pages,
                                                    gk, gv, k_pages, k_sf, vt_pages, vt_sf);
  else
    quant_kv_pages_kernel<32><<<grid, 128, 0, st>>>((const uint16_t*)k, (const uint16_t*)v, Hkv, L,
                                                    d, fp4_len, excl_mask, block_table, max_pages,
                                                    gk, gv, k_pages, k_sf, vt_pages, vt_sf);
  return launch_status();
}
