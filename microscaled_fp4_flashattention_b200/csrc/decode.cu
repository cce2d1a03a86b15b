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
// each warp streams its work units (64-token FP4 pages, 16-token BF16 slices) once through a
// private ring of cp.async.bulk copies, dequantises in registers (E2M1 x E4M3 products are
// exact in FP16) straight into mma.sync m16n8k16 fragments (FP32 accumulate), and never
// stages dequantised data.  Swap-AB form, tokens / channels in M and the GQA heads in N:
//   scores  S^T[16 tokens x 8 heads]   = K[16 tokens x 16 dims] * q^T[16 dims x 8 heads]
//   output  O^T[16 chans x 8 heads]   += V^T[16 chans x 16 tokens] * P^T[16 tokens x 8 heads]
// The score accumulators, packed to f16 and transposed by movmatrix, are the P^T operand.
// The token order inside a page is permuted so that every V^T fragment of a thread is one
// 8-byte load covering a whole 16-token scale block.
// Grid: (split, kv-head, sequence); each warp runs its own online softmax over a strided
// subset of the split's units; warps merge in shared memory, splits merge in the combine
// kernel (log-sum-exp weighted).
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

// D[16x8] += A[16x16] * B[16x8] with all four A registers (rows g, g+8; k halves)
FA4Q_DEVINL void mma_f16x4(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                           uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// transpose of an 8x8 b16 matrix held one row pair per thread (the mma accumulator layout)
FA4Q_DEVINL uint32_t movmatrix_t(uint32_t x) {
  uint32_t y;
  asm volatile("movmatrix.sync.aligned.m8n8.trans.b16 %0, %1;" : "=r"(y) : "r"(x));
  return y;
}

// two E2M1 codes (one byte, low nibble first) -> f16x2 (low half = low nibble)
FA4Q_DEVINL uint32_t e2m1x2_to_f16x2(uint32_t byte) {
  uint32_t out;
  asm("{\n\t.reg .b8 b;\n\tcvt.u8.u32 b, %1;\n\tcvt.rn.f16x2.e2m1x2 %0, b;\n\t}" : "=r"(out) : "r"(byte));
  return out;
}

// four E2M1 codes (the low 16 bits of w, low nibble first) -> two f16x2 (codes 0,1 and 2,3)
FA4Q_DEVINL void e2m1x4_to_f16x2x2(uint32_t w, uint32_t& lo, uint32_t& hi) {
  asm("{\n\t.reg .b8 b0, b1, b2, b3;\n\tmov.b32 {b0, b1, b2, b3}, %2;\n\t"
      "cvt.rn.f16x2.e2m1x2 %0, b0;\n\tcvt.rn.f16x2.e2m1x2 %1, b1;\n\t}"
      : "=r"(lo), "=r"(hi)
      : "r"(w));
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

// Work units of one (sequence, kv-head): FP4 pages (64 tokens) first, then 16-token slices
// of the BF16 vertical-line set, then 16-token slices of the BF16 window.
constexpr int kStageBytes = 9216;          // K page 4096 + K scales 512 + V^T page 4096 + scales 512
// scale bytes of one page piece: 64 tokens x 8 (NVFP4) / 4 (MXFP4) blocks of K; 128 channels x
// 4 / 2 blocks of V^T
template <bool MX>
__host__ __device__ constexpr uint32_t page_sf_bytes() { return MX ? 256u : 512u; }
constexpr int kDecStages = 2;              // per-warp ring depth (2 x 9 KB: 3 CTAs per SM fit)

struct UnitInfo {
  int kind;        // 0 FP4 page, 1 vertical-line slice, 2 window slice
  int base;        // first token of the unit within its class
  int nvalid;      // tokens of the unit that exist (<= 64 or 16)
};

FA4Q_DEVINL UnitInfo unit_info(const DecParams& p, int u, int n_fp4, int n_hp, int n_win) {
  UnitInfo x;
  if (u < p.n_ch_fp4) {
    x.kind = 0; x.base = u * 64; x.nvalid = min(64, n_fp4 - x.base);
  } else if (u < p.n_ch_fp4 + p.n_ch_hp) {
    x.kind = 1; x.base = (u - p.n_ch_fp4) * 16; x.nvalid = min(16, n_hp - x.base);
  } else {
    x.kind = 2; x.base = (u - p.n_ch_fp4 - p.n_ch_hp) * 16; x.nvalid = min(16, n_win - x.base);
  }
  return x;
}

FA4Q_DEVINL void ldsm_x4_trans(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}

// Block-table entry of unit u (FP4 pages only; 0 otherwise).  Read one unit before the
// unit is issued, so the lookup's latency is not on the path of the copy.
FA4Q_DEVINL int64_t unit_page(const DecParams& p, int b, int u) {
  return u < p.n_ch_fp4 ? static_cast<int64_t>(p.table[(int64_t)b * p.max_pages + u]) : 0;
}

// Issue the copies of unit `u` (physical page `phys` for an FP4 page) into one ring stage
// (lane 0 only).
template <bool MX>
FA4Q_DEVINL void issue_unit(const DecParams& p, const UnitInfo& x, int hk, int bh, int64_t phys,
                            uint8_t* stage, uint64_t* bar) {
  if (x.kind == 0) {
    constexpr uint32_t sf = page_sf_bytes<MX>();
    const int64_t ph = phys * p.Hkv + hk;
    mbar_arrive_expect_tx(bar, 2 * (4096 + sf));
    bulk_load(stage, p.kp + ph * 64 * (kDecD / 2), 4096, bar);
    bulk_load(stage + 4096, p.ksf + ph * sf, sf, bar);
    bulk_load(stage + 4608, p.vp + ph * kDecD * 32, 4096, bar);
    bulk_load(stage + 8704, p.vsf + ph * sf, sf, bar);
  } else {
    const uint16_t* kb = x.kind == 1 ? p.hp_k + ((int64_t)bh * p.max_hp + x.base) * kDecD
                                     : p.win_k + ((int64_t)bh * p.W + x.base) * kDecD;
    const uint16_t* vb = x.kind == 1 ? p.hp_v + ((int64_t)bh * p.max_hp + x.base) * kDecD
                                     : p.win_v + ((int64_t)bh * p.W + x.base) * kDecD;
    const uint32_t bytes = static_cast<uint32_t>(x.nvalid) * kDecD * 2;
    mbar_arrive_expect_tx(bar, 2 * bytes);
    bulk_load(stage, kb, bytes, bar);
    bulk_load(stage + 4608, vb, bytes, bar);
  }
}

// f16x2 holding 2^rel twice (rel <= 0): exact down to the smallest subnormal 2^-24, zero below
FA4Q_DEVINL uint32_t f16x2_pow2(int rel) {
  const uint32_t h = rel >= -14 ? static_cast<uint32_t>(rel + 15) << 10 : (rel >= -24 ? 1u << (rel + 24) : 0u);
  return h | (h << 16);
}

// largest of the four bytes of w
FA4Q_DEVINL int max_byte4(uint32_t w) {
  uint32_t m = __vmaxu4(w, w >> 16);
  m = __vmaxu4(m, m >> 8);
  return static_cast<int>(m & 0xFFu);
}

template <bool MX>
__global__ void __launch_bounds__(kDecWarps * 32, 3) decode_split_kernel(const DecParams p) {
  extern __shared__ __align__(128) uint8_t dsm[];
  // [rings of all warps][mbarriers]; after the scan the rings are reused for the warp merge
  uint64_t* bars = reinterpret_cast<uint64_t*>(dsm + kDecWarps * kDecStages * kStageBytes);
  float* s_o = reinterpret_cast<float*>(dsm);                  // [warps][8][128]  (aliases rings)
  float* s_m = s_o + kDecWarps * 8 * kDecD;                    // [warps][8]
  float* s_l = s_m + kDecWarps * 8;                            // [warps][8]
  const int split = blockIdx.x, hk = blockIdx.y, b = blockIdx.z;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = lane >> 2, t = lane & 3;
  const int G = p.G;
  const int bh = b * p.Hkv + hk;
  uint8_t* ring = dsm + warp * kDecStages * kStageBytes;
  uint64_t* full = bars + warp * kDecStages;
  if (lane == 0) {
    for (int st = 0; st < kDecStages; ++st) mbar_init(&full[st], 1);
    fence_barrier_init();
  }
  __syncwarp();

  // ---- query fragments: row g = GQA head g of this kv-head (rows >= G are zero).  The
  // reduction order of the score MMA is permuted: logical k = 2t+e / 2t+8+e of chunk kc is
  // head dim 32t + 4kc + e / 32t + 4kc + 2 + e, so a thread's B operand is 32 consecutive dims.
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
  // swap-AB accumulators: O^T tile ct holds channels 16ct+g / 16ct+g+8 for heads 2t / 2t+1
  float o[8][4];
#pragma unroll
  for (int i = 0; i < 8; ++i) o[i][0] = o[i][1] = o[i][2] = o[i][3] = 0.0f;
  float m0 = -INFINITY, m1 = -INFINITY, l0 = 0.0f, l1 = 0.0f;   // heads 2t, 2t+1

  const int n_fp4 = min(p.fp4_len[b], p.max_pages * 64);
  const int n_hp = p.hp_count ? min(p.hp_count[bh], p.max_hp) : 0;
  const int n_win = p.win_len ? min(p.win_len[b], p.W) : 0;
  const int total = p.n_ch_fp4 + p.n_ch_hp + p.n_ch_win;
  const int c_begin = split * p.chunks_per_split;
  const int c_end = min(total, c_begin + p.chunks_per_split);
  // this warp's units: c_begin + warp, + kDecWarps, ... skipping units without a valid token
  auto next_valid = [&](int u) {
    while (u < c_end && unit_info(p, u, n_fp4, n_hp, n_win).nvalid <= 0) u += kDecWarps;
    return u;
  };
  int u_issue = next_valid(c_begin + warp);
  int n_issued = 0;
  int64_t page_next = 0;                          // lane 0: block-table entry of u_issue
  if (lane == 0) {
    page_next = u_issue < c_end ? unit_page(p, b, u_issue) : 0;
    for (int k = 0; k < kDecStages - 1 && u_issue < c_end; ++k) {
      issue_unit<MX>(p, unit_info(p, u_issue, n_fp4, n_hp, n_win), hk, bh, page_next,
                     ring + (n_issued % kDecStages) * kStageBytes, &full[n_issued % kDecStages]);
      ++n_issued;
      u_issue = next_valid(u_issue + kDecWarps);
      page_next = u_issue < c_end ? unit_page(p, b, u_issue) : 0;
    }
  } else {
    for (int k = 0; k < kDecStages - 1 && u_issue < c_end; ++k) {
      ++n_issued;
      u_issue = next_valid(u_issue + kDecWarps);
    }
  }
  int n_done = 0;
  bool ok = true;
  for (int u = next_valid(c_begin + warp); u < c_end; u = next_valid(u + kDecWarps)) {
    // keep the ring full: the stage refilled now was consumed in the previous iteration
    // (after a failed wait nothing new is issued; copies already in flight are still awaited)
    __syncwarp();
    if (ok && u_issue < c_end) {
      if (lane == 0) {
        issue_unit<MX>(p, unit_info(p, u_issue, n_fp4, n_hp, n_win), hk, bh, page_next,
                       ring + (n_issued % kDecStages) * kStageBytes, &full[n_issued % kDecStages]);
      }
      ++n_issued;
      u_issue = next_valid(u_issue + kDecWarps);
      if (lane == 0) page_next = u_issue < c_end ? unit_page(p, b, u_issue) : 0;
    }
    const UnitInfo x = unit_info(p, u, n_fp4, n_hp, n_win);
    const int stg = n_done % kDecStages;
    if (n_done >= n_issued) break;                  // stopped issuing after a failed wait
    // the exclusion word is read before the wait, so its latency overlaps the copy's
    const uint64_t excl_word = (x.kind == 0 && p.excl) ? p.excl[(int64_t)bh * p.max_pages + u] : 0ull;
    ok = __all_sync(0xffffffffu, mbar_wait(&full[stg], (n_done / kDecStages) & 1, &g_decode_status,
                                           kStatusTimeoutDecode)) && ok;
    const uint8_t* st8 = ring + stg * kStageBytes;
    ++n_done;
    if (!ok) continue;
    uint64_t vmask = x.nvalid >= 64 ? ~0ull : ((1ull << x.nvalid) - 1ull);
    vmask &= ~excl_word;
    if (vmask == 0ull) continue;

    // Both unit kinds use the swap-AB form: score rows = tokens (M = 16), columns = the GQA
    // heads (N = 8; rows of q past G are zero), so half as many MMAs as with heads in M.  The
    // score accumulators, packed to f16 and transposed with movmatrix, are the B operand of
    // O^T[channels x heads] += V^T[channels x tokens] * P^T.
    float s4[4][4];     // [chunk][(T_lo,h0) (T_lo,h1) (T_hi,h0) (T_hi,h1)]
    int nchunk;
    if (x.kind == 0) {
      // FP4 page, chunk c of 16 tokens: score row r (0..7) = token 16(r>>1) + 4c + (r&1), row
      // r+8 = that + 2; the PV reduction index k = 2t+e is token 16t + 4c + e and k = 2t+8+e
      // is 16t + 4c + 2 + e, so one 8-byte V^T load per channel covers all four chunks.
      nchunk = 4;
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        const int tlo = 16 * (g >> 1) + 4 * c + (g & 1), thi = tlo + 2;
        const uint4 klo = *reinterpret_cast<const uint4*>(st8 + tlo * 64 + 16 * t);
        const uint4 khi = *reinterpret_cast<const uint4*>(st8 + thi * 64 + 16 * t);
        // Scales of this thread's dims 32t..32t+31.  NVFP4: two UE4M3 blocks, exact in FP16.
        // MXFP4: one E8M0 block 2^(e-127); FP16 cannot hold every power of two, so the codes
        // are scaled by 2^(e - E) with E the token's largest block exponent (exact down to
        // 2^-24 below it) and the score by 2^(E-127) in FP32.
        uint32_t sla, slb, sha, shb;
        float sc_lo = p.sc_fp4, sc_hi = p.sc_fp4;
        if constexpr (MX) {
          const uint32_t wlo = *reinterpret_cast<const uint32_t*>(st8 + 4096 + tlo * 4);
          const uint32_t whi = *reinterpret_cast<const uint32_t*>(st8 + 4096 + thi * 4);
          const int elo = max_byte4(wlo), ehi = max_byte4(whi);
          sla = slb = f16x2_pow2(static_cast<int>((wlo >> (8 * t)) & 0xFFu) - elo);
          sha = shb = f16x2_pow2(static_cast<int>((whi >> (8 * t)) & 0xFFu) - ehi);
          sc_lo *= exp2i(elo - 127);
          sc_hi *= exp2i(ehi - 127);
        } else {
          const uint32_t flo = e4m3x2_to_f16x2(*reinterpret_cast<const uint16_t*>(st8 + 4096 + tlo * 8 + 2 * t));
          const uint32_t fhi = e4m3x2_to_f16x2(*reinterpret_cast<const uint16_t*>(st8 + 4096 + thi * 8 + 2 * t));
          sla = __byte_perm(flo, 0, 0x1010);
          slb = __byte_perm(flo, 0, 0x3232);
          sha = __byte_perm(fhi, 0, 0x1010);
          shb = __byte_perm(fhi, 0, 0x3232);
        }
        const uint32_t wl[4] = {klo.x, klo.y, klo.z, klo.w}, wh[4] = {khi.x, khi.y, khi.z, khi.w};
        float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int kc = 0; kc < 8; ++kc) {
          uint32_t la, lb, ha, hb;
          e2m1x4_to_f16x2x2(wl[kc >> 1] >> ((kc & 1) * 16), la, lb);
          e2m1x4_to_f16x2x2(wh[kc >> 1] >> ((kc & 1) * 16), ha, hb);
          const uint32_t sl = kc < 4 ? sla : slb, sh = kc < 4 ? sha : shb;
          mma_f16x4(acc, hmul2(la, sl), hmul2(ha, sh), hmul2(lb, sl), hmul2(hb, sh), qa[kc][0], qa[kc][1]);
        }
        const bool vl = (vmask >> tlo) & 1ull, vh = (vmask >> thi) & 1ull;
        s4[c][0] = vl ? acc[0] * sc_lo : -INFINITY;
        s4[c][1] = vl ? acc[1] * sc_lo : -INFINITY;
        s4[c][2] = vh ? acc[2] * sc_hi : -INFINITY;
        s4[c][3] = vh ? acc[3] * sc_hi : -INFINITY;
      }
    } else {
      // BF16 slice of 16 tokens in natural order: score rows g and g+8 are tokens g and g+8;
      // rows past nvalid are not loaded (zeros) and the MMAs stay outside the per-lane test,
      // because mma.sync.aligned must be executed by all lanes of the warp together
      nchunk = 1;
      const float sc = p.sc_bf16;
      const bool hl = g < x.nvalid, hh = g + 8 < x.nvalid;
      float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int q4 = 0; q4 < 4; ++q4) {
        const uint4 zl = make_uint4(0u, 0u, 0u, 0u);
        const uint4 wl = hl ? *reinterpret_cast<const uint4*>(st8 + g * 256 + 64 * t + 16 * q4) : zl;
        const uint4 wh = hh ? *reinterpret_cast<const uint4*>(st8 + (g + 8) * 256 + 64 * t + 16 * q4) : zl;
        mma_f16x4(acc, bf16x2_to_f16x2(wl.x), bf16x2_to_f16x2(wh.x), bf16x2_to_f16x2(wl.y),
                  bf16x2_to_f16x2(wh.y), qa[2 * q4][0], qa[2 * q4][1]);
        mma_f16x4(acc, bf16x2_to_f16x2(wl.z), bf16x2_to_f16x2(wh.z), bf16x2_to_f16x2(wl.w),
                  bf16x2_to_f16x2(wh.w), qa[2 * q4 + 1][0], qa[2 * q4 + 1][1]);
      }
      const bool vl = (vmask >> g) & 1ull, vh = (vmask >> (g + 8)) & 1ull;
      s4[0][0] = vl ? acc[0] * sc : -INFINITY;
      s4[0][1] = vl ? acc[1] * sc : -INFINITY;
      s4[0][2] = vh ? acc[2] * sc : -INFINITY;
      s4[0][3] = vh ? acc[3] * sc : -INFINITY;
#pragma unroll
      for (int c = 1; c < 4; ++c) s4[c][0] = s4[c][1] = s4[c][2] = s4[c][3] = -INFINITY;
    }
    // ---- online softmax per head (the 8 lanes sharing t hold one head pair)
    float mx0 = -INFINITY, mx1 = -INFINITY;
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      mx0 = fmaxf(mx0, fmaxf(s4[c][0], s4[c][2]));
      mx1 = fmaxf(mx1, fmaxf(s4[c][1], s4[c][3]));
    }
#pragma unroll
    for (int off = 4; off < 32; off <<= 1) {
      mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, off));
      mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, off));
    }
    const float mn0 = fmaxf(m0, mx0), mn1 = fmaxf(m1, mx1);
    const float al0 = ex2f(m0 - mn0), al1 = ex2f(m1 - mn1);
    const float gv = x.kind == 0 ? p.g_v : 1.0f;
    uint32_t pb0[4], pb1[4];
    float ps0 = 0.0f, ps1 = 0.0f;
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      if (c < nchunk) {
        const float q0 = ex2f(s4[c][0] - mn0), q1 = ex2f(s4[c][1] - mn1);
        const float q2 = ex2f(s4[c][2] - mn0), q3 = ex2f(s4[c][3] - mn1);
        ps0 += q0 + q2;
        ps1 += q1 + q3;
        pb0[c] = movmatrix_t(f32x2_to_f16x2(q0 * gv, q1 * gv));
        pb1[c] = movmatrix_t(f32x2_to_f16x2(q2 * gv, q3 * gv));
      }
    }
    l0 = l0 * al0 + ps0;
    l1 = l1 * al1 + ps1;
    m0 = mn0;
    m1 = mn1;
#pragma unroll
    for (int ct = 0; ct < 8; ++ct) {
      o[ct][0] *= al0;
      o[ct][1] *= al1;
      o[ct][2] *= al0;
      o[ct][3] *= al1;
    }
    // ---- O^T += V^T P^T, channel tiles of 16
    if (x.kind == 0) {
#pragma unroll
      for (int ct = 0; ct < 8; ++ct) {
        const int cha = 16 * ct + g, chb = cha + 8;
        const uint2 va = *reinterpret_cast<const uint2*>(st8 + 4608 + cha * 32 + 8 * t);
        const uint2 vb = *reinterpret_cast<const uint2*>(st8 + 4608 + chb * 32 + 8 * t);
        if constexpr (MX) {
          // this thread's tokens 16t..16t+15 lie in the channel's 32-token block t/2; the
          // codes take 2^(e - F), F the larger of the page's two block exponents, and the
          // page's products are added to O scaled by 2^(F-127) in FP32
          const uint32_t ea = *reinterpret_cast<const uint16_t*>(st8 + 8704 + cha * 2);
          const uint32_t eb = *reinterpret_cast<const uint16_t*>(st8 + 8704 + chb * 2);
          const int Fa = max(static_cast<int>(ea & 0xFFu), static_cast<int>(ea >> 8));
          const int Fb = max(static_cast<int>(eb & 0xFFu), static_cast<int>(eb >> 8));
          const uint32_t sa = f16x2_pow2(static_cast<int>((ea >> (8 * (t >> 1))) & 0xFFu) - Fa);
          const uint32_t sb = f16x2_pow2(static_cast<int>((eb >> (8 * (t >> 1))) & 0xFFu) - Fb);
          float pg[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
          for (int c = 0; c < 4; ++c) {
            uint32_t la, ha, lb, hb;
            e2m1x4_to_f16x2x2((c >> 1 ? va.y : va.x) >> ((c & 1) * 16), la, ha);
            e2m1x4_to_f16x2x2((c >> 1 ? vb.y : vb.x) >> ((c & 1) * 16), lb, hb);
            mma_f16x4(pg, hmul2(la, sa), hmul2(lb, sb), hmul2(ha, sa), hmul2(hb, sb), pb0[c], pb1[c]);
          }
          const float xa = exp2i(Fa - 127), xb = exp2i(Fb - 127);
          o[ct][0] = fmaf(pg[0], xa, o[ct][0]);
          o[ct][1] = fmaf(pg[1], xa, o[ct][1]);
          o[ct][2] = fmaf(pg[2], xb, o[ct][2]);
          o[ct][3] = fmaf(pg[3], xb, o[ct][3]);
        } else {
          const uint32_t fa = st8[8704 + cha * 4 + t], fb = st8[8704 + chb * 4 + t];
          const uint32_t sa = e4m3x2_to_f16x2(fa | (fa << 8)), sb = e4m3x2_to_f16x2(fb | (fb << 8));
#pragma unroll
          for (int c = 0; c < 4; ++c) {
            uint32_t la, ha, lb, hb;
            e2m1x4_to_f16x2x2((c >> 1 ? va.y : va.x) >> ((c & 1) * 16), la, ha);
            e2m1x4_to_f16x2x2((c >> 1 ? vb.y : vb.x) >> ((c & 1) * 16), lb, hb);
            mma_f16x4(o[ct], hmul2(la, sa), hmul2(lb, sb), hmul2(ha, sa), hmul2(hb, sb), pb0[c], pb1[c]);
          }
        }
      }
    } else {
      // V rows [token][channel] -> A fragments by ldmatrix.trans; halves of rows past nvalid
      // are zeroed (P is zero there, but 0 * NaN is not)
      const uint32_t vbase = smem_u32(st8 + 4608);
      const int tok_ld = (lane & 7) + ((lane >> 4) & 1) * 8, ch_ld = ((lane >> 3) & 1) * 8;
      const uint32_t k0 = x.nvalid >= 16 ? 0xFFFFFFFFu
                          : ((2 * t < x.nvalid ? 0xFFFFu : 0u) | (2 * t + 1 < x.nvalid ? 0xFFFF0000u : 0u));
      const uint32_t k1 = x.nvalid >= 16 ? 0xFFFFFFFFu
                          : ((2 * t + 8 < x.nvalid ? 0xFFFFu : 0u) | (2 * t + 9 < x.nvalid ? 0xFFFF0000u : 0u));
#pragma unroll
      for (int ct = 0; ct < 8; ++ct) {
        uint32_t r0, r1, r2, r3;
        ldsm_x4_trans(vbase + tok_ld * 256 + (16 * ct + ch_ld) * 2, r0, r1, r2, r3);
        mma_f16x4(o[ct], bf16x2_to_f16x2(r0) & k0, bf16x2_to_f16x2(r1) & k0, bf16x2_to_f16x2(r2) & k1,
                  bf16x2_to_f16x2(r3) & k1, pb0[0], pb1[0]);
      }
    }
  }
  // ---- merge the warps of the CTA (the rings are free once every warp has left the scan)
  __syncthreads();
#pragma unroll
  for (int off = 4; off < 32; off <<= 1) {
    l0 += __shfl_xor_sync(0xffffffffu, l0, off);
    l1 += __shfl_xor_sync(0xffffffffu, l1, off);
  }
  const int h0 = 2 * t, h1 = 2 * t + 1;
#pragma unroll
  for (int ct = 0; ct < 8; ++ct) {
    const int cha = 16 * ct + g, chb = cha + 8;
    if (h0 < G) {
      s_o[(warp * 8 + h0) * kDecD + cha] = o[ct][0];
      s_o[(warp * 8 + h0) * kDecD + chb] = o[ct][2];
    }
    if (h1 < G) {
      s_o[(warp * 8 + h1) * kDecD + cha] = o[ct][1];
      s_o[(warp * 8 + h1) * kDecD + chb] = o[ct][3];
    }
  }
  if (g == 0) {
    if (h0 < G) { s_m[warp * 8 + h0] = m0; s_l[warp * 8 + h0] = l0; }
    if (h1 < G) { s_m[warp * 8 + h1] = m1; s_l[warp * 8 + h1] = l1; }
  }
  __syncthreads();
  const int stride = kDecD + 2;
  for (int idx = threadIdx.x; idx < G * kDecD; idx += blockDim.x) {
    const int hh = idx / kDecD, c = idx % kDecD;
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < kDecWarps; ++w) M = fmaxf(M, s_m[w * 8 + hh]);
    float acc = 0.0f, lsum = 0.0f;
    if (M != -INFINITY) {
#pragma unroll
      for (int w = 0; w < kDecWarps; ++w) {
        const float wt = ex2f(s_m[w * 8 + hh] - M);
        acc += wt * s_o[(w * 8 + hh) * kDecD + c];
        lsum += wt * s_l[w * 8 + hh];
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

constexpr size_t kDecSmem = (size_t)kDecWarps * kDecStages * kStageBytes + kDecWarps * kDecStages * 8;
static_assert(kDecWarps * 8 * kDecD * 4 + 2 * kDecWarps * 8 * 4 <= kDecWarps * kDecStages * kStageBytes,
              "merge buffers must fit in the rings they alias");

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

fa4q_status launch_decode_combine(const float* ws, int rows, int splits, uint16_t* out, cudaStream_t st) {
  decode_combine_kernel<<<(rows + 3) / 4, 128, 0, st>>>(ws, rows, splits, out);
  return launch_status();
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
  return max_pages + (max_hp + 15) / 16 + (W + 15) / 16;
}

static int decode_auto_splits(int B, int Hkv, int chunks) {
  const int target_ctas = 148 * 8;                        // 1184: ~2.9 waves of 3 CTAs per SM at B*Hkv = 256
  int s = (target_ctas + B * Hkv - 1) / (B * Hkv);
  const int max_s = (chunks + kDecWarps - 1) / kDecWarps;  // at least a chunk per warp
  s = s > max_s ? max_s : s;
  return s < 1 ? 1 : s;
}

}  // namespace fa4q

using namespace fa4q;

extern "C" size_t fa4q_decode_workspace_size(int B, int Hq, int Hkv, int d, int max_pages, int num_splits) {
  if (B <= 0 || Hq <= 0 || Hkv <= 0 || d != kDecD || max_pages < 0) return 0;
  // the automatic split count is capped by the number of work units; size for the uncapped
  // value, an upper bound for any cache shape
  const int splits = num_splits > 0 ? num_splits : decode_auto_splits(B, Hkv, 1 << 30);
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
      (vt_pages && !aligned16(vt_pages)) || (k_sf && !aligned16(k_sf)) ||
      (vt_sf && !aligned16(vt_sf)) || (hp_k && !aligned16(hp_k)) ||
      (hp_v && !aligned16(hp_v)) || (win_k && !aligned16(win_k)) || (win_v && !aligned16(win_v)) ||
      !aligned16(workspace))
    return FA4Q_ERR_INVALID_ARG;
  if (B > 65535 || Hkv > 65535) return FA4Q_ERR_UNSUPPORTED;
  const int chunks = decode_chunks(max_pages, max_hp, W);
  if (chunks == 0) return FA4Q_ERR_INVALID_ARG;   // no key slot at all: nothing to attend to
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
  const bool mx = fmt == FA4Q_MXFP4;
  if (mx) g_k = g_v = 1.0f;                       // MXFP4 pages carry no tensor scale
  p.sc_fp4 = sms * g_k * kDecLog2e;
  p.sc_bf16 = sms * kDecLog2e;
  p.g_v = g_v;
  p.n_ch_fp4 = max_pages;
  p.n_ch_hp = (max_hp + 15) / 16;
  p.n_ch_win = (W + 15) / 16;
  p.splits = splits;
  p.chunks_per_split = (chunks + splits - 1) / splits;
  p.ws = static_cast<float*>(workspace);
  p.out = static_cast<uint16_t*>(out);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  dim3 grid(splits, Hkv, B);
  auto kern = mx ? decode_split_kernel<true> : decode_split_kernel<false>;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kDecSmem) != cudaSuccess)
    return FA4Q_ERR_CUDA;
  kern<<<grid, kDecWarps * 32, kDecSmem, st>>>(p);
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
  const int chunks = decode_chunks(max_pages, max_hp, W);
  if (chunks == 0) return FA4Q_ERR_INVALID_ARG;   // no key slot at all: nothing to attend to
  const size_t per_split = (size_t)B * Hq * (kDecD + 2) * sizeof(float);
  int splits = num_splits;
  if (splits == 0) {
    splits = decode_auto_splits(B, Hkv, chunks);
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
