// attn_fwd.cu - fused 4-bit microscaled FlashAttention prefill for B200 (sm_100a).
//
// What it computes (per (batch, q-head), 128-row query tile, key tiles of 128):
//   S_j = Q_hat K_hat_j^T                 block-scaled FP4 tensor-core MMA, FP32 in TMEM
//   m   = max(m, rowmax S_j)              exact running maximum every tile
//   P~  = exp(S_j - m)                    unnormalised exponentials (FP32)
//   P^  = E2M1 blocks of P~ along keys    pre-normalisation quantisation (PNQ)
//   [O | l] = alpha [O | l] + P^ [V_hat | 1]   both FP4 MMAs; l accumulates the same P^
//   out = O / l * g_v
// Sources: HiFA4 (Training-Free 4-bit FlashAttention on Ascend HIF4 NPUs), Abstract -
// QK^T and PV as 4-bit GEMMs under an online softmax, P-Reordering (normaliser from the
// quantised P^, fused into the PV GEMM); MXAttention, Abstract - Pre-Normalization
// Quantization of the unnormalised exponentials before the row sum; BitDecoding-FP4,
// "Underflow-Aware Probability Scaling" - NVFP4 P with the static tensor scale 1/(6*448);
// "System-Level Optimization" - transposed softmax: P blocks run along the MMA reduction
// (key) axis so P is quantised in registers and never leaves the SM.
//
// Kernel structure (384 threads, one CTA per SM).  A work item is one 128-row query tile of
// one (batch, q-head).  Launches whose items are short (causal attention over a few thousand
// keys) run persistently, one CTA per SM walking a longest-first item list; the others run
// one CTA per item.  Roles:
//   warp 0      TMA producer: each item's Q tile (two slots, so the next item's Q loads
//               during this one), then K, V^T tiles and their scale atoms through an
//               NST-deep shared-memory ring (cp.async.bulk.tensor / cp.async.bulk).
//   warp 1      TMEM owner and MMA issuer (one elected thread): tcgen05.cp of the scale
//               atoms into TMEM, tcgen05.mma kind::mxf4nvf4 (NVFP4) or kind::mxf4 (MXFP4).
//   warps 2-3   idle (they complete warpgroup 0 for the register split)
//   warps 4-11  softmax: two groups of four warps take alternate key tiles, one query row
//               per thread; tcgen05.ld of S, mask, running max (passed between the groups),
//               exp2 (two of every eight on the FMA pipe by a polynomial, the rest on MUFU),
//               block scales, cvt to E2M1, P^ to shared memory (the A operand of the PV MMA),
//               rescale of the group's O and l in TMEM, epilogue.
// TMEM (512 columns): S [0,128), O even/odd tiles [128,256) and [256,384), l even/odd
// [384,400) and [400,416), scale factors [416,488).  Every mbarrier wait is bounded; on expiry the CTA records a status bit,
// skips the remaining waits, drains its own copies and MMAs and exits.
#include <math.h>

#include <cstring>

#include "fa4q_common.cuh"
#include "fa4q_internal.h"

namespace fa4q {

static __device__ uint32_t g_attn_status;

constexpr int kBM = 128;
constexpr int kBN = 128;
constexpr int kThreads = 384;
// Register split (setmaxnreg): launched at 168 per thread (3 warps per scheduler x 168 x 32 =
// 16128 of the scheduler's 16384); warpgroup 0 (TMA, MMA, 2 idle warps) drops to 56 and the
// two softmax warpgroups rise to 224: 56*32 + 2*224*32 = 16128, the launch total exactly.
constexpr int kRegsIssue = 56, kRegsSoftmax = 224;
// The hybrid instantiation's TMA and MMA warps carry the full-precision rings' counters,
// barriers and descriptors on top: 56 registers made them spill 156 bytes; 104 / 200 keeps
// the block's total (4 x 32 x 104 + 8 x 32 x 200 = 384 x 168) and spills 4 bytes.
constexpr int kRegsIssueHyb = 104, kRegsSoftmaxHyb = 200;
constexpr int kStages = 4;      // K/V tile stages (tiles mostly served from L2)
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kGpNvfp4 = 1.0f / 2688.0f;  // g_P = 1/(6*448), rounded to FP32
// 1 / (6 g_P) in FP32: the P scale t = amax / (6 g_P) is taken as one multiply (t may differ
// from the IEEE quotient by one ulp; amax itself comes from an approximate exponential)
constexpr float kInvSixGp = 1.0f / (6.0f * kGpNvfp4);
// polynomial 2^f ~ c0 + c1 f + c2 f^2 + c3 f^3 on [0, 1) (see ex2_poly2)
constexpr float kExp2C0 = 0.9999252557754517f, kExp2C1 = 0.6958334445953369f;
constexpr float kExp2C2 = 0.22606724500656128f, kExp2C3 = 0.07802451401948929f;
constexpr int kEmulPer8 = 2;  // exponentials of every 8 computed by ex2_poly2 (the rest on MUFU)


// TMEM column map: one S buffer, two O and l accumulators (even / odd key tiles), scales
constexpr uint32_t kColS = 0, kColO0 = 128, kColO1 = 256, kColL0 = 384, kColL1 = 400;
// (Q scales double-buffered by work item, K scales by key tile, P and V scales by group)
constexpr uint32_t kColSfQ = 416, kColSfK = 432, kColSfP = 448, kColSfV = 464, kColSfOne = 480;

template <int D, bool MX>
struct Cfg {
  static constexpr int kBlk = MX ? 32 : 16;
  static constexpr int kQBytes = kBM * D / 2;
  static constexpr int kKBytes = kBN * D / 2;
  static constexpr int kVBytes = D * kBN / 2;
  static constexpr int kPBytes = kBM * kBN / 2;
  static constexpr int kSfQAtoms = (D / kBlk + 3) / 4;  // atoms per row tile actually read
  static constexpr int kSfGroups = 32 / kBlk;           // padded groups per 128 columns
  static constexpr int kSfTileAtoms = 32 / kBlk;        // atoms per 128-key tile (P, V)
  static constexpr int kKStepsQK = D / 64;
  static constexpr int kQKSwizzle = D == 128 ? kSwiz64 : kSwiz32;
  static constexpr int kQKSbo = D == 128 ? 512 : 256;
};

// Full-precision tiles of the hybrid prefill (HYB): bf16 Q, K, V as 64-column (128-byte)
// chunks with the 128-byte swizzle, 64 keys per tile.
constexpr int kHyKeys = 64;       // keys per full-precision tile
constexpr int kHyStages = 2;      // K/V stages of the full-precision tiles
template <bool HYB>
struct HybSmem {
  uint8_t unused;
};
template <>
struct __align__(1024) HybSmem<true> {
  uint8_t q[2][128 * 128];          // bf16 Q of the work item: two chunks of 128 rows x 128 B
  uint8_t kv[kHyStages][4][kHyKeys * 128];   // K chunk 0, K chunk 1, V chunk 0, V chunk 1
  uint8_t ones[16 * kHyKeys * 2];   // B operand of the normaliser: 16 rows of g_v (bf16)
  uint64_t bar_q, q_free;
  // K and V of a stage have their own barriers: the K slot frees as soon as its S product
  // completes, so S can run two tiles ahead of PV with two stages
  uint64_t kfull[kHyStages], kempty[kHyStages], vfull[kHyStages], vempty[kHyStages];
};

template <int D, bool MX, bool HYB = false>
struct __align__(1024) Smem {
  using C = Cfg<D, MX>;
  static constexpr int kNst = HYB ? 3 : kStages;   // FP4 K/V stages (the hybrid's BF16 tiles take room)
  uint8_t q[2][C::kQBytes];                 // double-buffered by work item
  uint8_t k[kNst][C::kKBytes];
  uint8_t v[kNst][C::kVBytes];
  uint8_t p[2][HYB ? 128 * kHyKeys * 2 : C::kPBytes];   // P^ per group (hybrid: bf16 P as well)
  uint8_t ones[1024];
  uint8_t sfq[2][2 * 512];
  uint8_t sfk[kNst][2 * 512];
  uint8_t sfv[kNst][2 * 512];
  uint8_t sfp[2][2 * 512];
  uint8_t sfone[2 * 512];
  HybSmem<HYB> hy;
  uint64_t bar_q[2];         // Q tile (and its scales) of work item k landed, slot k % 2
  uint64_t q_free[2];        // all S products of work item k issued and complete
  uint64_t o_free;           // all eight softmax warps have read O and l in the epilogue
  uint64_t kv_full[kNst];
  uint64_t kv_empty[kNst];
  uint64_t s_full[2];        // S of an even / odd key tile ready (one per softmax group)
  uint64_t s_free;
  uint64_t p_full[2];
  uint64_t o_done[2];
  uint64_t drain;
  float m_xchg[2][kBM];       // running maximum after tile j, slot j%2, per row
  float m_last[2][kBM];       // per group: the maximum its accumulator is relative to
  float l_last[2][kBM];       // per group: the normaliser summed from P~ (ablation only)
  uint32_t tmem_base;
  uint32_t abort_flag;
};

struct AttnParams {
  const uint8_t* q_sf;
  const uint8_t* k_sf;
  const uint8_t* vt_sf;
  void* out;
  float* lse;
  int B, Hq, Hkv, S_q, S_k, S_kpad;
  int n_qtiles;
  int n_items;             // B * Hq * n_qtiles work items
  float score_scale_log2;  // sm_scale * g_q * g_k * log2(e)
  float g_v;
  float qmax_p;
  // MXFP4 P scale without an exponential: with x = (bmax - m) * sc the block maximum is 2^x,
  // so the OCP exponent floor(log2 amax) - 2 is floor(x) - 2 and the bound-Q rule (smallest
  // e with amax <= Q 2^e) is ceil(x - log2 Q).
  float log2_qmax_p;
  // Conditional rescaling (FlashAttention-4, as named in the FLAMIA page's abstract): the
  // reference maximum moves only when a tile's maximum exceeds it by more than tau binades
  // (tau = 0: the exact running maximum).  NVFP4 P then takes the tensor scale
  // gp = g_P * 2^tau, and the P scale t = amax / (6 gp) is one multiply by inv6gp (t may
  // differ from the IEEE quotient by one ulp; amax itself comes from an approximate
  // exponential).
  float tau;
  float gp;
  float inv6gp;
  // Ablation of P-Reordering (HiFA4, Abstract): 1 takes the normaliser from the unquantised
  // exponentials P~ (summed in FP32 by the softmax threads) instead of from the P_hat that
  // feeds the PV product; the numerator is unchanged, so each output row is scaled by
  // sum P_hat / sum P~.
  int l_from_ptilde;
  // Hybrid-precision prefill (HyQuant): each work item first takes its full-precision keys
  // in BF16 tiles of 64 - the window band {j : i - W < j <= i}, then the vertical lines
  // {v : v <= i - W} from their gathered rows - and then its FP4 tiles with those keys
  // masked out (window: key > row - W; vertical lines: bit set in hy_excl), all under one
  // online softmax.
  const uint64_t* hy_excl;   // [B][Hkv][hy_excl_words]
  const int32_t* hy_vl_pos;  // [B][Hkv][hy_max_vl] ascending positions of the vertical lines
  const int32_t* hy_vl_count;  // [B][Hkv]
  int hy_window;
  int hy_excl_words;
  int hy_max_vl;
  float hy_inv_gqgk;         // BF16 scores -> the FP4 products' units (1 / (g_q g_k))
  float hy_lp16;             // log2 of the units of P in the FP4 PV products, times g_v (NVFP4:
                             // g_P g_v; MXFP4: 1) - a BF16 tile's P is 2^(s sc - m sc - hy_lp16)
  uint32_t hy_ones_bits;     // bf16 bits of g_v (exact): the full-precision normaliser's operand
  int causal;
  int out_fp32;
};

// Bounded wait that gives up at once when another role of the CTA already gave up.
FA4Q_DEVINL bool cta_wait(uint64_t* bar, uint32_t parity, volatile uint32_t* abort_flag,
                          uint32_t code) {
  if (*abort_flag) return false;
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = globaltimer_ns();
  while (true) {
    if (mbar_try_wait(bar, parity)) return true;
    if (*abort_flag) return false;
    if (globaltimer_ns() - t0 > kWaitNs) break;
  }
  atomicOr(&g_attn_status, code);
  *abort_flag = 1;
  return false;
}

FA4Q_DEVINL bool mbar_test_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}\n"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

// Warp-uniform bounded wait for the softmax warps: a non-blocking test first (the phase has
// usually completed long before), the suspending bounded wait only when it has not.
FA4Q_DEVINL bool warp_wait(uint64_t* bar, uint32_t parity, volatile uint32_t* abort_flag, uint32_t code) {
  if (__all_sync(0xffffffffu, mbar_test_wait(bar, parity))) return true;
  return __all_sync(0xffffffffu, cta_wait(bar, parity, abort_flag, code));
}

// Wait of the MMA-issuing thread: a non-blocking test first (its inputs are usually ready),
// then the bounded suspending wait.
FA4Q_DEVINL bool mma_wait(uint64_t* bar, uint32_t parity, volatile uint32_t* abort_flag) {
  if (mbar_test_wait(bar, parity)) return true;
  return cta_wait(bar, parity, abort_flag, kStatusTimeoutMma);
}

FA4Q_DEVINL float ex2_approx(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

FA4Q_DEVINL float lg2_approx(float x) {
  float y;
  asm("lg2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// (lo, hi) -> bf16x2 (round to nearest even), lo in the low half
FA4Q_DEVINL uint32_t pack_bf16x2(float lo, float hi) {
  uint32_t d;
  asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(d) : "f"(hi), "f"(lo));
  return d;
}

FA4Q_DEVINL float fmax3(float a, float b, float c) {
  float d;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}

// (x0, x1) *= (a, a) in one packed FP32 instruction
FA4Q_DEVINL void fmul2_inplace(uint32_t& x0, uint32_t& x1, float a) {
  asm("{\n\t.reg .b64 rx, ra;\n\t"
      "mov.b64 rx, {%0, %1};\n\tmov.b64 ra, {%2, %2};\n\t"
      "mul.rn.f32x2 rx, rx, ra;\n\tmov.b64 {%0, %1}, rx;\n\t}\n"
      : "+r"(x0), "+r"(x1)
      : "f"(a));
}

// (d0, d1) = (a0 * b0 + c0, a1 * b1 + c1) in one packed FP32 instruction
FA4Q_DEVINL void ffma2(float& d0, float& d1, float a0, float a1, float b0, float b1, float c0, float c1) {
  asm("{\n\t.reg .b64 ra, rb, rc, rd;\n\t"
      "mov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\tmov.b64 rc, {%6, %7};\n\t"
      "fma.rn.f32x2 rd, ra, rb, rc;\n\tmov.b64 {%0, %1}, rd;\n\t}\n"
      : "=f"(d0), "=f"(d1)
      : "f"(a0), "f"(a1), "f"(b0), "f"(b1), "f"(c0), "f"(c1));
}

// 2^x for two values on the FMA pipe (Cody-Waite style range reduction and a polynomial),
// used for part of the exponentials so that the MUFU and FMA pipes share the work (FLAMIA,
// Abstract: FlashAttention-4's software-emulated exponential on Blackwell):
//   x := max(x, -126)                        (2^-126 and below quantise to 0 anyway; p(0)
//                                            is just below 1, so -126 is the lowest floor
//                                            whose exponent sum stays non-negative)
//   t  = x + 1.5*2^23 rounded toward -inf    -> the low mantissa bits of t hold floor(x)
//   f  = x - (t - 1.5*2^23)                  in [0, 1), exact
//   p  = c0 + f (c1 + f (c2 + f c3))         2^f, minimax (relative) fit on [0, 1),
//                                            max relative error 7.5e-5
//   2^x = p * 2^floor(x): floor(x) added to the exponent field of p (bits of t << 23)
// The coefficients come from an iteratively reweighted least-squares fit of 2^f on [0, 1)
// (fit_exp2_poly.py beside this file).  The result feeds E2M1 rounding (3 significant bits).
FA4Q_DEVINL void ex2_poly2(float& y0, float& y1, float x0, float x1) {
  x0 = fmaxf(x0, -126.0f);
  x1 = fmaxf(x1, -126.0f);
  uint32_t t0, t1, p0, p1;
  asm("{\n\t.reg .b64 rx, rt, rj, rf, rp, rm, c0, c1, c2, c3;\n\t"
      "mov.b64 rx, {%4, %5};\n\tmov.b64 rm, {%6, %6};\n\t"
      "add.rm.f32x2 rt, rx, rm;\n\tsub.rn.f32x2 rj, rt, rm;\n\tsub.rn.f32x2 rf, rx, rj;\n\t"
      "mov.b64 c3, {%10, %10};\n\tmov.b64 c2, {%9, %9};\n\tmov.b64 c1, {%8, %8};\n\tmov.b64 c0, {%7, %7};\n\t"
      "fma.rn.f32x2 rp, c3, rf, c2;\n\tfma.rn.f32x2 rp, rp, rf, c1;\n\tfma.rn.f32x2 rp, rp, rf, c0;\n\t"
      "mov.b64 {%0, %1}, rt;\n\tmov.b64 {%2, %3}, rp;\n\t}"
      : "=r"(t0), "=r"(t1), "=r"(p0), "=r"(p1)
      : "f"(x0), "f"(x1), "f"(12582912.0f), "f"(kExp2C0), "f"(kExp2C1), "f"(kExp2C2), "f"(kExp2C3));
  y0 = __uint_as_float(p0 + (t0 << 23));
  y1 = __uint_as_float(p1 + (t1 << 23));
}

// maximum of N consecutive values, as a tree of 3-input maxima
template <int N>
FA4Q_DEVINL float block_max(const float* v) {
  float a[(N + 2) / 3];
#pragma unroll
  for (int i = 0; i < N / 3; ++i) a[i] = fmax3(v[3 * i], v[3 * i + 1], v[3 * i + 2]);
  if constexpr (N % 3 == 1) a[N / 3] = v[N - 1];
  if constexpr (N % 3 == 2) a[N / 3] = fmaxf(v[N - 2], v[N - 1]);
  if constexpr ((N + 2) / 3 == 1) {
    return a[0];
  } else {
    return block_max<(N + 2) / 3>(a);
  }
}

template <int N>
FA4Q_DEVINL void setmaxnreg_inc() {
  asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(N));
}
template <int N>
FA4Q_DEVINL void setmaxnreg_dec() {
  asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(N));
}

FA4Q_DEVINL void named_bar_arrive(int id, int count) {
  asm volatile("bar.arrive %0, %1;" ::"r"(id), "r"(count) : "memory");
}

FA4Q_DEVINL void named_bar_sync(int id, int count) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(count) : "memory");
}

FA4Q_DEVINL void tmem_ld1(uint32_t taddr, uint32_t& r) {
  asm volatile("tcgen05.ld.sync.aligned.32x32b.x1.b32 {%0}, [%1];" : "=r"(r) : "r"(taddr));
}
FA4Q_DEVINL void tmem_st1(uint32_t taddr, uint32_t r) {
  asm volatile("tcgen05.st.sync.aligned.32x32b.x1.b32 [%0], {%1};" ::"r"(taddr), "r"(r) : "memory");
}

// byte offset of (row r, 16-byte chunk c) in a K-major tile with 64-byte rows, 64B swizzle
FA4Q_DEVINL uint32_t swz64_offset(uint32_t r, uint32_t c) {
  return (r >> 3) * 512 + (r & 7) * 64 + ((c ^ ((r >> 1) & 3)) << 4);
}
// ... 32-byte rows, 32B swizzle
FA4Q_DEVINL uint32_t swz32_offset(uint32_t r, uint32_t c) {
  return (r >> 3) * 256 + (r & 7) * 32 + ((c ^ ((r >> 2) & 1)) << 4);
}

// Issue one block-scaled FP4 MMA step.  For MXFP4 the two scales of a 64-element step sit
// at byte 2*(step%2) of the 4-byte TMEM scale word (selected by the descriptor's sf id).
template <bool MX>
FA4Q_DEVINL void mma_step(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, int N, int step,
                          uint32_t sfa_col, uint32_t sfb_col, uint32_t acc) {
  if constexpr (MX) {
    const uint32_t id = 2u * (step & 1);
    const uint32_t idesc = make_idesc_fp4(N, true, id, id);
    mma_mxf4(d_tmem, adesc, bdesc, idesc, sfa_col + 4u * (step >> 1), sfb_col + 4u * (step >> 1),
             acc);
  } else {
    const uint32_t idesc = make_idesc_fp4(N, false, 0, 0);
    mma_nvf4(d_tmem, adesc, bdesc, idesc, sfa_col + 4u * step, sfb_col + 4u * step, acc);
  }
}

// ABL: the ablations of fa4q_attn_fwd_ex (conditional rescaling, normaliser from P~) are
// compiled into separate instantiations so the default kernel carries none of their work.
// HYB: the hybrid-precision prefill (causal only, D = 128): full-precision tiles first, then
// the FP4 tiles; tm_q16 .. tm_vlv are its bf16 operands (unused by the other instantiations).
template <int D, bool MX, bool CAUSAL, bool PERSIST, bool ABL, bool HYB = false>
__global__ void __launch_bounds__(kThreads, 1)
    attn_fwd_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                    const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_q16,
                    const __grid_constant__ CUtensorMap tm_k16, const __grid_constant__ CUtensorMap tm_v16,
                    const __grid_constant__ CUtensorMap tm_vlk, const __grid_constant__ CUtensorMap tm_vlv,
                    const AttnParams p) {
  using C = Cfg<D, MX>;
  using SM = Smem<D, MX, HYB>;
  constexpr int NST = SM::kNst;
  extern __shared__ uint8_t smem_raw[];
  SM& sm = *reinterpret_cast<SM*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  volatile uint32_t* abort_flag = &sm.abort_flag;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // Persistent CTAs (one per SM) walk one list of work items (batch, q-head, query tile).
  // Causal lists are query-tile-major with the heaviest (last) query tiles of every head
  // first; non-causal lists are head-major, so the items in flight share few heads whose
  // K/V tiles stay in L2.  CTA c takes items c, 2G-1-c, 2G+c, 4G-1-c, ... (G CTAs): a snake
  // over the longest-first list that evens out the work.  Every role walks the same items,
  // so the barrier phases below follow from counters each role keeps itself.
  // n_tiles counts every key tile of the item; the hybrid's are nw window tiles (64 keys,
  // starting at key 64 w0), then nv vertical-line tiles (64 gathered rows each), then FP4.
  struct Item {
    int b, h, qt, n_tiles;
    int nw, w0, nv;
  };
  const int n_ktiles_all = (p.S_k + kBN - 1) / kBN;
  auto item_index = [&](int k) -> int {
    if constexpr (!PERSIST) return k == 0 ? static_cast<int>(blockIdx.x) : -1;   // one item per CTA
    const int G = gridDim.x, c = blockIdx.x;
    const int64_t u = static_cast<int64_t>(k) * G + ((k & 1) ? (G - 1 - c) : c);
    return u < p.n_items ? static_cast<int>(u) : -1;
  };
  auto decode_item = [&](int u) -> Item {
    Item it;
    if (CAUSAL) {
      const int per = p.B * p.Hq, rem = u % per;
      it.qt = p.n_qtiles - 1 - u / per;
      it.b = rem / p.Hq;
      it.h = rem % p.Hq;
      it.n_tiles = min(it.qt + 1, n_ktiles_all);
      it.nw = it.w0 = it.nv = 0;
      if constexpr (HYB) {
        // rows [r0, r1] of the item: window keys (r0 - W, r1], vertical lines up to r1 - W,
        // FP4 keys up to r1 - W (the window tiles always hold each row's own key)
        const int r0 = it.qt * kBM, r1 = min(r0 + kBM - 1, p.S_q - 1), last = r1 - p.hy_window;
        it.w0 = max(0, r0 - p.hy_window + 1) / kHyKeys;
        it.nw = r1 / kHyKeys - it.w0 + 1;
        int nvis = 0;
        if (p.hy_max_vl > 0 && last >= 0) {
          const int bh_k = it.b * p.Hkv + it.h / (p.Hq / p.Hkv);
          const int32_t* pos = p.hy_vl_pos + (int64_t)bh_k * p.hy_max_vl;
          int lo = 0, hi = min(p.hy_vl_count[bh_k], p.hy_max_vl);     // first position > last
          while (lo < hi) {
            const int mid = (lo + hi) >> 1;
            if (pos[mid] <= last) lo = mid + 1;
            else hi = mid;
          }
          nvis = lo;
        }
        it.nv = (nvis + kHyKeys - 1) / kHyKeys;
        it.n_tiles = it.nw + it.nv + min(it.n_tiles, last >= 0 ? last / kBN + 1 : 0);
      }
    } else {
      const int per = p.Hq * p.n_qtiles, rem = u % per;
      it.b = u / per;
      it.h = rem / p.n_qtiles;
      it.qt = rem % p.n_qtiles;
      it.n_tiles = n_ktiles_all;
      it.nw = it.w0 = it.nv = 0;
    }
    return it;
  };

  // ---------------------------------------------------------------- setup
  if (threadIdx.x == 0) {
    for (int s = 0; s < 2; ++s) {
      mbar_init(&sm.bar_q[s], 1);
      mbar_init(&sm.q_free[s], 1);
    }
    for (int s = 0; s < NST; ++s) {
      mbar_init(&sm.kv_full[s], 1);
      mbar_init(&sm.kv_empty[s], 1);
    }
    if constexpr (HYB) {
      mbar_init(&sm.hy.bar_q, 1);
      mbar_init(&sm.hy.q_free, 1);
      for (int s = 0; s < kHyStages; ++s) {
        mbar_init(&sm.hy.kfull[s], 1);
        mbar_init(&sm.hy.kempty[s], 1);
        mbar_init(&sm.hy.vfull[s], 1);
        mbar_init(&sm.hy.vempty[s], 1);
      }
    }
    mbar_init(&sm.s_free, 4);
    for (int s = 0; s < 2; ++s) {
      mbar_init(&sm.s_full[s], 1);
      mbar_init(&sm.p_full[s], 4);
      mbar_init(&sm.o_done[s], 1);
    }
    mbar_init(&sm.o_free, 8);
    mbar_init(&sm.drain, 1);
    sm.abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 2) {
    // constant B operand of the normaliser MMA: 16 rows of E2M1 ones (code 2) and unit scales
    uint32_t* o32 = reinterpret_cast<uint32_t*>(sm.ones);
    for (int i = lane; i < 256; i += 32) o32[i] = 0x22222222u;
    uint32_t* s32 = reinterpret_cast<uint32_t*>(sm.sfone);
    const uint32_t one = MX ? 0x7F7F7F7Fu : 0x38383838u;
    for (int i = lane; i < 256; i += 32) s32[i] = one;
    if constexpr (HYB) {
      // B operand of the full-precision tiles' normaliser: 16 rows of g_v in bf16 (every
      // element equal, so the swizzle is immaterial)
      uint32_t* h32 = reinterpret_cast<uint32_t*>(sm.hy.ones);
      for (int i = lane; i < 16 * kHyKeys / 2; i += 32) h32[i] = p.hy_ones_bits * 0x10001u;
    }
    fence_proxy_async_smem();
  }
  if (warp == 1) {
    tmem_alloc(&sm.tmem_base, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sm.tmem_base;

  if (warp < 4) {
  setmaxnreg_dec<HYB ? kRegsIssueHyb : kRegsIssue>();
  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (elect_one()) {
      prefetch_tmap(&tm_q);
      prefetch_tmap(&tm_k);
      prefetch_tmap(&tm_v);
      if constexpr (HYB) {
        prefetch_tmap(&tm_q16);
        prefetch_tmap(&tm_k16);
        prefetch_tmap(&tm_v16);
        prefetch_tmap(&tm_vlk);
        prefetch_tmap(&tm_vlv);
      }
      const int nrt_q = (p.S_q + 127) / 128, nrt_k = (p.S_k + 127) / 128;
      const int ng_v = ((p.S_kpad + 127) / 128) * C::kSfGroups;
      int T = 0, q_issued = 0;                     // FP4 key tiles / Q tiles issued so far
      int Tb = 0, Tbv = 0;                         // full-precision K / V tiles issued so far
      int q16_issued = 0;                          // bf16 Q tiles issued so far
      bool go = true;
      for (int k = 0; go && (PERSIST || k < 1); ++k) {
        const int u = item_index(k);
        if (u < 0) break;
        const Item it = decode_item(u);
        const int bh_q = it.b * p.Hq + it.h, bh_k = it.b * p.Hkv + it.h / (p.Hq / p.Hkv);
        const int qs = k & 1;
        if constexpr (HYB) {
          // bf16 Q: the slot was last read by the full-precision S products of item k-1
          if (k >= 1 && !cta_wait(&sm.hy.q_free, (k - 1) & 1, abort_flag, kStatusTimeoutTmaFull)) break;
          mbar_arrive_expect_tx(&sm.hy.bar_q, 2 * 128 * 128);
          tma_load_3d(sm.hy.q[0], &tm_q16, 0, it.qt * kBM, bh_q, &sm.hy.bar_q);
          tma_load_3d(sm.hy.q[1], &tm_q16, 128, it.qt * kBM, bh_q, &sm.hy.bar_q);
          q16_issued = k + 1;
        }
        // Q slot qs was last read by the S products of item k-2
        if (k >= 2 && !cta_wait(&sm.q_free[qs], ((k - 2) >> 1) & 1, abort_flag, kStatusTimeoutTmaFull)) break;
        mbar_arrive_expect_tx(&sm.bar_q[qs], C::kQBytes + C::kSfQAtoms * 512);
        tma_load_3d(sm.q[qs], &tm_q, 0, it.qt * kBM, bh_q, &sm.bar_q[qs]);
        bulk_load(sm.sfq[qs], p.q_sf + ((int64_t)bh_q * nrt_q + it.qt) * C::kSfGroups * 512,
                  C::kSfQAtoms * 512, &sm.bar_q[qs]);
        q_issued = k + 1;
        if constexpr (HYB) {
          // full-precision tiles: K and V rows of the window band, then the gathered
          // vertical-line rows (past the sequence / the row count TMA fills zeros)
          for (int i = 0; i < it.nw + it.nv; ++i, ++Tb) {
            const int hs = Tb % kHyStages;
            const uint32_t ph = ((Tb / kHyStages) - 1) & 1;
            const bool win = i < it.nw;
            const CUtensorMap* mk = win ? &tm_k16 : &tm_vlk;
            const CUtensorMap* mv = win ? &tm_v16 : &tm_vlv;
            const int y = win ? (it.w0 + i) * kHyKeys : (i - it.nw) * kHyKeys;
            if (Tb >= kHyStages && !cta_wait(&sm.hy.kempty[hs], ph, abort_flag, kStatusTimeoutTmaFull)) {
              go = false;
              break;
            }
            mbar_arrive_expect_tx(&sm.hy.kfull[hs], 2 * kHyKeys * 128);
            tma_load_3d(sm.hy.kv[hs][0], mk, 0, y, bh_k, &sm.hy.kfull[hs]);
            tma_load_3d(sm.hy.kv[hs][1], mk, 128, y, bh_k, &sm.hy.kfull[hs]);
            if (Tb >= kHyStages && !cta_wait(&sm.hy.vempty[hs], ph, abort_flag, kStatusTimeoutTmaFull)) {
              go = false;
              ++Tb;                                // its K copy is in flight (drained below)
              break;
            }
            mbar_arrive_expect_tx(&sm.hy.vfull[hs], 2 * kHyKeys * 128);
            tma_load_3d(sm.hy.kv[hs][2], mv, 0, y, bh_k, &sm.hy.vfull[hs]);
            tma_load_3d(sm.hy.kv[hs][3], mv, 128, y, bh_k, &sm.hy.vfull[hs]);
            ++Tbv;
          }
          if (!go) break;
        }
        const int nf = it.n_tiles - it.nw - it.nv;
        for (int j = 0; j < nf; ++j, ++T) {
          const int s = T % NST;
          if (T >= NST && !cta_wait(&sm.kv_empty[s], ((T / NST) - 1) & 1, abort_flag,
                                    kStatusTimeoutTmaFull)) {
            go = false;
            break;
          }
          mbar_arrive_expect_tx(&sm.kv_full[s], C::kKBytes + C::kVBytes + C::kSfQAtoms * 512 +
                                                    C::kSfTileAtoms * 512);
          tma_load_3d(sm.k[s], &tm_k, 0, j * kBN, bh_k, &sm.kv_full[s]);
          bulk_load(sm.sfk[s], p.k_sf + ((int64_t)bh_k * nrt_k + j) * C::kSfGroups * 512,
                    C::kSfQAtoms * 512, &sm.kv_full[s]);
          tma_load_3d(sm.v[s], &tm_v, j * (kBN / 2), 0, bh_k, &sm.kv_full[s]);
          bulk_load(sm.sfv[s], p.vt_sf + (int64_t)bh_k * ng_v * 512 + (int64_t)j * C::kSfTileAtoms * 512,
                    C::kSfTileAtoms * 512, &sm.kv_full[s]);
        }
      }
      // drain: every issued copy must have landed before the CTA may exit
      for (int t = max(0, T - NST); t < T; ++t)
        mbar_wait(&sm.kv_full[t % NST], (t / NST) & 1, &g_attn_status, kStatusTimeoutDrain);
      for (int k = max(0, q_issued - 2); k < q_issued; ++k)
        mbar_wait(&sm.bar_q[k & 1], (k >> 1) & 1, &g_attn_status, kStatusTimeoutDrain);
      if constexpr (HYB) {
        for (int t = max(0, Tb - kHyStages); t < Tb; ++t)
          mbar_wait(&sm.hy.kfull[t % kHyStages], (t / kHyStages) & 1, &g_attn_status, kStatusTimeoutDrain);
        for (int t = max(0, Tbv - kHyStages); t < Tbv; ++t)
          mbar_wait(&sm.hy.vfull[t % kHyStages], (t / kHyStages) & 1, &g_attn_status, kStatusTimeoutDrain);
        if (q16_issued > 0) mbar_wait(&sm.hy.bar_q, (q16_issued - 1) & 1, &g_attn_status, kStatusTimeoutDrain);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (elect_one()) {
      // Every shared-memory descriptor is formed once: a tile at byte offset o from the
      // shared-memory base has the base's descriptor plus o/16 (the start-address field;
      // shared memory is below 256 KB, so the field never carries), so issuing an MMA is a
      // few integer adds (this single thread's latency sits on the softmax groups' path).
      const uint32_t base = smem_u32(&sm);
      const uint64_t d_qk = make_smem_desc(base, 16, C::kQKSbo, C::kQKSwizzle);   // Q and K tiles
      const uint64_t d_pv = make_smem_desc(base, 16, 512, kSwiz64);               // P, V^T, ones
      const uint64_t d_sf = make_smem_desc(base, 0, 128, kSwizNone);              // scale atoms
      constexpr uint64_t oq = offsetof(SM, q) >> 4, ok_ = offsetof(SM, k) >> 4, ov = offsetof(SM, v) >> 4;
      constexpr uint64_t op = offsetof(SM, p) >> 4, oones = offsetof(SM, ones) >> 4;
      constexpr uint64_t osfq = offsetof(SM, sfq) >> 4, osfk = offsetof(SM, sfk) >> 4;
      constexpr uint64_t osfv = offsetof(SM, sfv) >> 4, osfp = offsetof(SM, sfp) >> 4;
      constexpr uint64_t osfone = offsetof(SM, sfone) >> 4;
      constexpr uint64_t kQStride = C::kQBytes >> 4, kKStride = C::kKBytes >> 4, kVStride = C::kVBytes >> 4;
      constexpr uint64_t kPStride = sizeof(sm.p[0]) >> 4, kSfStride = 1024 >> 4;
      // full-precision tiles (hybrid): bf16 chunks of 128-byte rows, 128-byte swizzle
      const uint64_t d_h = make_smem_desc(base, 16, 1024, kSwiz128);               // K-major (Q, K, P, ones)
      const uint64_t d_hv = make_smem_desc(base, kHyKeys * 128, 1024, kSwiz128);   // V, MN-major
      constexpr uint64_t ohq = HYB ? offsetof(SM, hy) >> 4 : 0;
      constexpr uint64_t kHq = 128 * 128 >> 4, kHc = kHyKeys * 128 >> 4, kHst = 4 * kHc;
      constexpr uint64_t ohkv = ohq + 2 * kHq, ohones = ohkv + kHyStages * kHst;
      const uint32_t id_hs = make_idesc_bf16(kHyKeys, false), id_ho = make_idesc_bf16(D, true);
      const uint32_t id_hl = make_idesc_bf16(16, false);
      // instruction descriptors (MXFP4: the 64-element step selects its scale byte pair)
      const uint32_t id_s[2] = {make_idesc_fp4(kBN, MX, 0, 0), make_idesc_fp4(kBN, MX, MX ? 2 : 0, MX ? 2 : 0)};
      const uint32_t id_o[2] = {make_idesc_fp4(D, MX, 0, 0), make_idesc_fp4(D, MX, MX ? 2 : 0, MX ? 2 : 0)};
      const uint32_t id_l[2] = {make_idesc_fp4(16, MX, 0, 0), make_idesc_fp4(16, MX, MX ? 2 : 0, MX ? 2 : 0)};
      // TMEM scale column of the 64-element step kk (MXFP4: two steps share a 4-column atom)
      auto sf_step = [](int kk) -> uint32_t { return MX ? 4u * (kk >> 1) : 4u * kk; };
      auto mma = [&](uint32_t d, uint64_t ad, uint64_t bd, uint32_t idesc, uint32_t sfa, uint32_t sfb, uint32_t acc) {
        if constexpr (MX) mma_mxf4(d, ad, bd, idesc, sfa, sfb, acc);
        else mma_nvf4(d, ad, bd, idesc, sfa, sfb, acc);
      };
      for (int a = 0; a < C::kSfTileAtoms; ++a) tmem_cp_sf_desc(tmem + kColSfOne + 4 * a, d_sf + osfone + 32 * a);
      bool ok = true;
      int T = 0;                                   // key tiles of all earlier items
      int T4 = 0, T4p = 0;                         // FP4 tiles whose S / PV products were issued
      int Tb = 0, Tbp = 0;                         // full-precision tiles (hybrid), S / PV
      int n_pv0 = 0, n_pv1 = 0;                    // PV products issued per softmax group
      for (int k = 0; ok && (PERSIST || k < 1); ++k) {
        const int u = item_index(k);
        if (u < 0) break;
        const Item it = decode_item(u);
        const int qs = k & 1, T0 = T, n_tiles = it.n_tiles, nb = it.nw + it.nv;
        if (!mma_wait(&sm.bar_q[qs], (k >> 1) & 1, abort_flag)) break;
        tc_fence_after();
        // item k-2 used this scale slot; all of its products completed before item k-1 ended
        for (int a = 0; a < C::kSfQAtoms; ++a) tmem_cp_sf_desc(tmem + kColSfQ + 8 * qs + 4 * a, d_sf + osfq + qs * kSfStride + 32 * a);
        const uint64_t qd = d_qk + oq + qs * kQStride;
        if constexpr (HYB) {
          if (!mma_wait(&sm.hy.bar_q, k & 1, abort_flag)) break;
        }
        // S_j = Q K_j^T into the single S buffer once the softmax group of the previous key
        // tile (of this item or the last) holds its scores in registers
        auto issue_s = [&](int j) -> bool {
          const int t = T0 + j;
          if (t >= 1 && !mma_wait(&sm.s_free, (t - 1) & 1, abort_flag)) return false;
          if constexpr (HYB) {
            if (j < nb) {
              // full-precision tile: S = Q K^T on bf16 (M = 128, N = 64, K = 16 per MMA)
              const int hs = Tb % kHyStages;
              if (!mma_wait(&sm.hy.kfull[hs], (Tb / kHyStages) & 1, abort_flag)) return false;
              tc_fence_after();
#pragma unroll
              for (int kk = 0; kk < D / 16; ++kk)
                mma_bf16(tmem + kColS, d_h + ohq + (kk >> 2) * kHq + 2 * (kk & 3),
                         d_h + ohkv + hs * kHst + (kk >> 2) * kHc + 2 * (kk & 3), id_hs, kk > 0);
              tc_commit(&sm.s_full[j & 1]);
              tc_commit(&sm.hy.kempty[hs]);
              ++Tb;
              if (j == nb - 1) tc_commit(&sm.hy.q_free);   // every product that read the bf16 Q
              return true;
            }
          }
          const int s = T4 % NST, kb = T4 & 1;
          if (!mma_wait(&sm.kv_full[s], (T4 / NST) & 1, abort_flag)) return false;
          tc_fence_after();
          for (int a = 0; a < C::kSfQAtoms; ++a)
            tmem_cp_sf_desc(tmem + kColSfK + 8 * kb + 4 * a, d_sf + osfk + s * kSfStride + 32 * a);
          const uint64_t kd = d_qk + ok_ + s * kKStride;
#pragma unroll
          for (int kk = 0; kk < C::kKStepsQK; ++kk)
            mma(tmem + kColS, qd + 2 * kk, kd + 2 * kk, id_s[kk & 1], tmem + kColSfQ + 8 * qs + sf_step(kk),
                tmem + kColSfK + 8 * kb + sf_step(kk), kk > 0);
          tc_commit(&sm.s_full[j & 1]);
          ++T4;
          return true;
        };
        // [O | l]_{j%2} (+)= P^_j [V_j | 1] once the softmax group has written P^_j; the first
        // product of an item waits until the previous item's epilogue has read O and l
        auto issue_pv = [&](int jp) -> bool {
          const int pb = jp & 1;
          if (jp == 0 && k >= 1 && !mma_wait(&sm.o_free, (k - 1) & 1, abort_flag)) return false;
          int& n_pv = pb ? n_pv1 : n_pv0;
          if (!mma_wait(&sm.p_full[pb], n_pv & 1, abort_flag)) return false;
          ++n_pv;
          tc_fence_after();
          const uint32_t o_col = pb ? kColO1 : kColO0, l_col = pb ? kColL1 : kColL0;
          if constexpr (HYB) {
            if (jp < nb) {
              // full-precision tile: [O | l] (+)= P [V | g_v] on bf16 (K = 16 keys per MMA; V is
              // [keys][d], the MN-major B operand, in two 64-channel chunks)
              const int hs = Tbp % kHyStages;
              if (!mma_wait(&sm.hy.vfull[hs], (Tbp / kHyStages) & 1, abort_flag)) return false;
              tc_fence_after();
#pragma unroll
              for (int kk = 0; kk < kHyKeys / 16; ++kk) {
                const uint32_t acc = (jp >= 2 || kk > 0) ? 1u : 0u;
                const uint64_t pd = d_h + op + pb * kPStride + 2 * kk;
                mma_bf16(tmem + o_col, pd, d_hv + ohkv + hs * kHst + 2 * kHc + kk * 128, id_ho, acc);
                mma_bf16(tmem + l_col, pd, d_h + ohones + 2 * kk, id_hl, acc);
              }
              tc_commit(&sm.o_done[pb]);
              tc_commit(&sm.hy.vempty[hs]);
              ++Tbp;
              return true;
            }
          }
          const int s = T4p % NST;
          for (int a = 0; a < C::kSfTileAtoms; ++a) {
            tmem_cp_sf_desc(tmem + kColSfP + 8 * pb + 4 * a, d_sf + osfp + pb * kSfStride + 32 * a);
            tmem_cp_sf_desc(tmem + kColSfV + 8 * pb + 4 * a, d_sf + osfv + s * kSfStride + 32 * a);
          }
          const uint64_t pd = d_pv + op + pb * kPStride, vd = d_pv + ov + s * kVStride, od = d_pv + oones;
#pragma unroll
          for (int kk = 0; kk < 2; ++kk) {
            const uint32_t acc = (jp >= 2 || kk > 0) ? 1u : 0u;
            mma(tmem + o_col, pd + 2 * kk, vd + 2 * kk, id_o[kk], tmem + kColSfP + 8 * pb + sf_step(kk),
                tmem + kColSfV + 8 * pb + sf_step(kk), acc);
            mma(tmem + l_col, pd + 2 * kk, od + 2 * kk, id_l[kk], tmem + kColSfP + 8 * pb + sf_step(kk),
                tmem + kColSfOne + sf_step(kk), acc);
          }
          tc_commit(&sm.o_done[pb]);
          tc_commit(&sm.kv_empty[s]);
          ++T4p;
          return true;
        };
        // Issue order S_0, S_1, PV_0, S_2, PV_1, ...: S runs two products ahead of PV, so the
        // next S is computed as soon as the S buffer is free (the other group has loaded its
        // scores, early in its tile) instead of waiting behind the previous tile's P^.  The
        // first scores of the next item are computed while this item's epilogue runs.
        ok = issue_s(0);
        for (int j = 0; ok && j <= n_tiles; ++j) {
          if (j + 1 < n_tiles && !issue_s(j + 1)) ok = false;
          else if (j >= 1 && !issue_pv(j - 1)) ok = false;
        }
        tc_commit(&sm.q_free[qs]);                 // every product that read Q slot qs
        T += n_tiles;
      }
      // drain: all MMAs this thread issued complete before TMEM is released
      tc_commit(&sm.drain);
      mbar_wait(&sm.drain, 0, &g_attn_status, kStatusTimeoutDrain);
    }
  }
  } else {
    setmaxnreg_inc<HYB ? kRegsSoftmaxHyb : kRegsSoftmax>();
    // ------------------------------------------------------------ softmax / PNQ / epilogue
    // Two softmax groups of four warps: group A (warps 4-7) takes the even key tiles, group B
    // (warps 8-11) the odd ones; each thread owns one full query row of its tiles, and the TMEM
    // lane quadrant of a warp is warp % 4.  Only the running maximum passes from one tile to
    // the next: the group finishing tile j publishes m_j in shared memory and arrives on a
    // named barrier the other group synchronises on.  Each group accumulates its own O and l,
    // so the rescale before a tile's PV product waits on the group's previous PV product,
    // issued two tiles earlier.  The loops never leave early (after an abort every wait
    // returns at once), so arrivals and synchronisations on the named barriers always pair.
    const int g = (warp - 4) >> 2;                 // softmax group: 0 = even tiles, 1 = odd
    const int wq = warp & 3;                       // TMEM lane quadrant
    const int r = wq * 32 + lane;                  // row within the query tile
    const uint32_t lane_base = tmem + (static_cast<uint32_t>(wq * 32) << 16);
    const int bar_send = 1 + 4 * g + wq, bar_recv = 1 + 4 * (g ^ 1) + wq, bar_epi = 9 + wq;
    const float sc = p.score_scale_log2;
    constexpr int kNB = kBN / C::kBlk;             // P blocks per row: 8 (NVFP4) / 4 (MXFP4)
    // Running maximum kept in the raw MMA-score domain.  Block maxima are taken from the
    // exact difference (bmax - m) * sc, so the block holding the row maximum gets amax = 1
    // exactly: the MX OCP exponent floor(log2 amax) - 2 jumps at every power of two, and a
    // fused s*sc - round(m*sc) that lands 1 ulp below 0 would move that block's scale.
    bool ok = true;
    int done_a = 0, done_b = 0;                    // key tiles each group processed in earlier items
    for (int k = 0; PERSIST || k < 1; ++k) {
    const int u = item_index(k);
    if (u < 0) break;
    const Item it = decode_item(u);
    const int qt = it.qt, n_tiles = it.n_tiles;
    const int bh_q = it.b * p.Hq + it.h;
    const int row = qt * kBM + r;                  // query index
    const int done_g = g ? done_b : done_a;
    float m_acc = -INFINITY;                       // maximum of this group's last tile
    float lpt = 0.0f;                              // sum of P~ of this group (ABL), MMA units
    const float gp_item = ABL ? p.gp : kGpNvfp4;
    const int nb = it.nw + it.nv;                  // full-precision tiles (hybrid) come first
    // vertical-line entries visible to this row (positions ascending: those <= row - W), so a
    // vertical-line tile masks by entry index alone
    int nvis_row = 0;
    if constexpr (HYB) {
      if (it.nv > 0) {
        const int bh_k = it.b * p.Hkv + it.h / (p.Hq / p.Hkv), lim = row - p.hy_window;
        const int32_t* pos = p.hy_vl_pos + (int64_t)bh_k * p.hy_max_vl;
        int lo = 0, hi = min(p.hy_vl_count[bh_k], p.hy_max_vl);
        while (lo < hi) {
          const int mid = (lo + hi) >> 1;
          if (pos[mid] <= lim) lo = mid + 1;
          else hi = mid;
        }
        nvis_row = lo;
      }
    }
    // bring accumulator g from the maximum it holds (tile j-2) to m_new (rows whose maximum
    // did not move keep alpha = 1; -inf to -inf, a row without a visible key yet, too)
    auto rescale_to = [&](int j, float m_new) {
      if (j >= 2) {
        tc_fence_after();
        const float alpha = m_acc == m_new ? 1.0f : ex2_approx((m_acc - m_new) * sc);
        if (__any_sync(0xffffffffu, alpha != 1.0f)) {
          const uint32_t o_col = g ? kColO1 : kColO0, l_col = g ? kColL1 : kColL0;
          uint32_t raw[D / 32][32];
          uint32_t lr;
#pragma unroll
          for (int c = 0; c < D / 32; ++c) tmem_ld32(lane_base + o_col + 32 * c, raw[c]);
          tmem_ld1(lane_base + l_col, lr);
          tmem_wait_ld();
#pragma unroll
          for (int c = 0; c < D / 32; ++c) {
#pragma unroll
            for (int i = 0; i < 32; i += 2) fmul2_inplace(raw[c][i], raw[c][i + 1], alpha);
            tmem_st32(lane_base + o_col + 32 * c, raw[c]);
          }
          tmem_st1(lane_base + l_col, __float_as_uint(__uint_as_float(lr) * alpha));
          tmem_wait_st();
        }
      }
      m_acc = m_new;
    };
    for (int j = g; j < n_tiles; j += 2) {
      ok = warp_wait(&sm.s_full[g], (done_g + (j >> 1)) & 1, abort_flag, kStatusTimeoutSoftmax) && ok;
      tc_fence_after();
      if constexpr (HYB) {
        if (j < nb) {
          // ---- full-precision tile (64 keys): scores, masks, maximum, unquantised P in bf16
          float sh[kHyKeys];
          {
            uint32_t raw[2][32];
            tmem_ld32(lane_base + kColS, raw[0]);
            tmem_ld32(lane_base + kColS + 32, raw[1]);
            tmem_wait_ld();
#pragma unroll
            for (int c = 0; c < 2; ++c)
#pragma unroll
              for (int i = 0; i < 32; ++i) sh[32 * c + i] = __uint_as_float(raw[c][i]);
          }
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&sm.s_free);
          if (j < it.nw) {
            // window band: row - W < key <= row, key < S_k
            const int k0 = (it.w0 + j) * kHyKeys;
#pragma unroll
            for (int i = 0; i < kHyKeys; ++i) {
              const int key = k0 + i;
              if (!(key <= row && key > row - p.hy_window && key < p.S_k)) sh[i] = -INFINITY;
            }
          } else {
            // gathered vertical lines: entry e visible to this row when e < nvis_row
            const int e0 = (j - it.nw) * kHyKeys;
#pragma unroll
            for (int i = 0; i < kHyKeys; ++i)
              if (e0 + i >= nvis_row) sh[i] = -INFINITY;
          }
          // the bf16 products times hy_inv_gqgk are in the FP4 tiles' score units (a positive
          // factor: the maximum converts after the fact, the exponent takes it in its scale)
          const float tmax = block_max<kHyKeys>(sh) * p.hy_inv_gqgk;
          float m_prev = -INFINITY;
          if (j > 0) {
            named_bar_sync(bar_recv, 64);
            m_prev = sm.m_xchg[(j - 1) & 1][r];
          }
          const float m_new = fmaxf(m_prev, tmax);
          sm.m_xchg[j & 1][r] = m_new;
          named_bar_arrive(bar_send, 64);
          // P = 2^(s sc - m sc - lp16): the FP4 PV products' units, divided by g_v (the
          // normaliser's B operand holds g_v); a row with no visible key yet gets P = 0
          const float off = m_new > -INFINITY ? m_new * sc + p.hy_lp16 : 0.0f;
          const float sch = sc * p.hy_inv_gqgk;
          uint32_t pk[kHyKeys / 2];
#pragma unroll
          for (int i = 0; i < kHyKeys / 2; ++i) {
            float y0, y1;
            ffma2(y0, y1, sh[2 * i], sh[2 * i + 1], sch, sch, -off, -off);
            pk[i] = pack_bf16x2(ex2_approx(y0), ex2_approx(y1));
          }
          // P buffer g was last read by this group's previous PV product
          if (j >= 2)
            ok = warp_wait(&sm.o_done[g], (done_g + (j >> 1) - 1) & 1, abort_flag, kStatusTimeoutSoftmax) && ok;
#pragma unroll
          for (int c = 0; c < kHyKeys / 8; ++c)
            *reinterpret_cast<uint4*>(sm.p[g] + swz128_offset(r, c)) =
                make_uint4(pk[4 * c], pk[4 * c + 1], pk[4 * c + 2], pk[4 * c + 3]);
          fence_proxy_async_smem();
          rescale_to(j, m_new);
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&sm.p_full[g]);
          continue;
        }
      }
      float s[kBN];
      {
        uint32_t raw[kBN / 32][32];
#pragma unroll
        for (int c = 0; c < kBN / 32; ++c) tmem_ld32(lane_base + kColS + 32 * c, raw[c]);
        tmem_wait_ld();
#pragma unroll
        for (int c = 0; c < kBN / 32; ++c)
#pragma unroll
          for (int i = 0; i < 32; ++i) s[32 * c + i] = __uint_as_float(raw[c][i]);
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&sm.s_free);
      // masking: keys beyond S_k, and (causal) keys after this query
      const int key0 = (HYB ? j - nb : j) * kBN;
      if constexpr (HYB) {
        // FP4 keys of row i: key <= i - window and not a vertical line
        const int lim = min(p.S_k - key0, row - p.hy_window - key0 + 1);
        const uint64_t* ex = p.hy_excl + (int64_t)(it.b * p.Hkv + it.h / (p.Hq / p.Hkv)) * p.hy_excl_words;
        const int w0 = key0 >> 6;
        const uint64_t e0 = w0 < p.hy_excl_words ? ex[w0] : 0ull;
        const uint64_t e1 = w0 + 1 < p.hy_excl_words ? ex[w0 + 1] : 0ull;
        const uint32_t ew[4] = {static_cast<uint32_t>(e0), static_cast<uint32_t>(e0 >> 32),
                                static_cast<uint32_t>(e1), static_cast<uint32_t>(e1 >> 32)};
#pragma unroll
        for (int q4 = 0; q4 < 4; ++q4) {
          if (ew[q4] == 0u) continue;              // no vertical line among these 32 keys
#pragma unroll
          for (int i = 0; i < 32; ++i)
            if (ew[q4] & (1u << i)) s[32 * q4 + i] = -INFINITY;
        }
        if (lim < kBN) {                           // the window band (the last FP4 tiles)
#pragma unroll
          for (int i = 0; i < kBN; ++i)
            if (i >= lim) s[i] = -INFINITY;
        }
      } else {
        const bool edge = (key0 + kBN > p.S_k) || (CAUSAL && key0 + kBN - 1 > qt * kBM);
        if (edge) {
          const int lim = CAUSAL ? min(p.S_k - key0, row - key0 + 1) : (p.S_k - key0);
#pragma unroll
          for (int i = 0; i < kBN; ++i)
            if (i >= lim) s[i] = -INFINITY;
        }
      }
      // block maxima of the raw scores (the scale is positive), tree-shaped for ILP
      float bmax[kNB];
#pragma unroll
      for (int bi = 0; bi < kNB; ++bi) bmax[bi] = block_max<C::kBlk>(s + bi * C::kBlk);
      float tmax = bmax[0];
#pragma unroll
      for (int bi = 1; bi < kNB; ++bi) tmax = fmaxf(tmax, bmax[bi]);
      // running maximum: take m_{j-1} from the other group, publish m_j
      float m_prev = -INFINITY;
      if (j > 0) {
        named_bar_sync(bar_recv, 64);
        m_prev = sm.m_xchg[(j - 1) & 1][r];
      }
      float m_new = fmaxf(m_prev, tmax);
      if constexpr (ABL) {
        const bool grow = !(m_prev > -INFINITY) || (tmax - m_prev) * sc > p.tau;
        if (!grow) m_new = m_prev;
      }
      sm.m_xchg[j & 1][r] = m_new;
      named_bar_arrive(bar_send, 64);
      const float mref = m_new * sc;
      // per block: scale from the block maximum 2^((bmax - m)*sc); y_i = exp2(s_i*sc - m*sc -
      // log2(scale)).  MXFP4 takes the exponent from (bmax - m)*sc directly, so its scales
      // need no MUFU work (the MUFU unit is the softmax's scarcest resource); NVFP4 rounds
      // amax / (6 g_P) to UE4M3 and takes the logarithm of the decoded scale.
      const float gp = ABL ? p.gp : kGpNvfp4;
      float lsc[kNB];                              // log2 of each block's scale (+inf: zero block)
      const float inv6gp = ABL ? p.inv6gp : kInvSixGp;
      uint32_t sfw[kNB / 4];
#pragma unroll
      for (int w = 0; w < kNB / 4; ++w) sfw[w] = 0;
#pragma unroll
      for (int bi = 0; bi < kNB; ++bi) {
        const float x = (bmax[bi] - m_new) * sc;   // log2 of the block maximum, <= 0
        uint32_t code;
        if constexpr (MX) {
          int e = -127;
          if (x > -160.0f) {
            e = p.qmax_p == 0.0f ? static_cast<int>(floorf(x)) - 2 : static_cast<int>(ceilf(x - p.log2_qmax_p));
            e = max(e, -127);
          }
          code = static_cast<uint32_t>(e + 127);
          lsc[bi] = x > -INFINITY ? static_cast<float>(e) : INFINITY;
        } else {
          const float t = ex2_approx(x) * inv6gp;                  // amax / (6 * gp)
          code = ue4m3_encode(t);
          const float sf = ue4m3_decode(code);
          lsc[bi] = sf > 0.0f ? lg2_approx(sf * gp) : INFINITY;
        }
        sfw[bi >> 2] |= code << (8 * (bi & 3));
      }
      uint32_t packed[kBN / 8];
      auto quantise_row = [&](auto exponent_argument, auto observe) {
#pragma unroll
        for (int g8 = 0; g8 < kBN / 8; ++g8) {
          const float l8 = lsc[(g8 * 8) / C::kBlk];
          float y[8];
#pragma unroll
          for (int i = 0; i < 8; i += 2) exponent_argument(y[i], y[i + 1], s[8 * g8 + i], s[8 * g8 + i + 1], l8);
#pragma unroll
          for (int i = 0; i < kEmulPer8; i += 2) ex2_poly2(y[i], y[i + 1], y[i], y[i + 1]);
#pragma unroll
          for (int i = kEmulPer8; i < 8; ++i) y[i] = ex2_approx(y[i]);
          observe(g8, y);
          packed[g8] = e2m1x8(y[0], y[1], y[2], y[3], y[4], y[5], y[6], y[7]);
        }
      };
      auto no_observer = [](int, const float*) {};
      auto standard_argument = [&](float& y0, float& y1, float s0, float s1, float l8) {
        const float o8 = mref + l8;
        ffma2(y0, y1, s0, s1, sc, sc, -o8, -o8);
      };
      float ysum[ABL ? kNB : 1];
      if constexpr (!ABL) {
        quantise_row(standard_argument, no_observer);
      } else {
        // scaled exponentials of the whole row for the P~ normaliser: per block, (sum of y)
        // times the block's scale in MMA units (2^e for MXFP4, the UE4M3 value for NVFP4)
#pragma unroll
        for (int bi = 0; bi < kNB; ++bi) ysum[bi] = 0.0f;
        auto sum_observer = [&](int g8, const float* y) {
          ysum[(g8 * 8) / C::kBlk] += ((y[0] + y[1]) + (y[2] + y[3])) + ((y[4] + y[5]) + (y[6] + y[7]));
        };
        if (p.tau > 0.0f) {
          // Reference kept from an earlier tile: a key whose score equals it has P~ = 1 in a
          // block whose scale is 2^e, e possibly 2, so y = 2^-e may sit exactly on the E2M1
          // tie 0.25.  The argument is formed from the exact difference s - m, so such a key
          // gets exactly -e (2^-2 from MUFU, or just below from the polynomial: both round to
          // 0 like the tie itself).
          const float mn = m_new;
          auto exact_argument = [&](float& y0, float& y1, float s0, float s1, float l8) {
            ffma2(y0, y1, s0, s1, 1.0f, 1.0f, -mn, -mn);
            ffma2(y0, y1, y0, y1, sc, sc, -l8, -l8);
          };
          if (p.l_from_ptilde) quantise_row(exact_argument, sum_observer);
          else quantise_row(exact_argument, no_observer);
        } else {
          quantise_row(standard_argument, sum_observer);
        }
      }
      // accumulator g and P buffer g were last used by this group's previous PV product
      if (j >= 2)
        ok = warp_wait(&sm.o_done[g], (done_g + (j >> 1) - 1) & 1, abort_flag, kStatusTimeoutSoftmax) && ok;
      uint8_t* pbuf = sm.p[g];
#pragma unroll
      for (int c = 0; c < 4; ++c)
        *reinterpret_cast<uint4*>(pbuf + swz64_offset(r, c)) =
            make_uint4(packed[4 * c], packed[4 * c + 1], packed[4 * c + 2], packed[4 * c + 3]);
#pragma unroll
      for (int a = 0; a < C::kSfTileAtoms; ++a)
        *reinterpret_cast<uint32_t*>(sm.sfp[g] + 512 * a + (r & 31) * 16 + (r >> 5) * 4) = sfw[a];
      fence_proxy_async_smem();
      // bring accumulator g from the maximum it holds (tile j-2) to m_j
      if (ABL && p.l_from_ptilde) {
        float add = 0.0f;
#pragma unroll
        for (int bi = 0; bi < kNB; ++bi) {
          const uint32_t code = (sfw[bi >> 2] >> (8 * (bi & 3))) & 0xFFu;
          const float scale = MX ? exp2i(static_cast<int>(code) - 127) : ue4m3_decode(code);
          add += ysum[bi] * scale;
        }
        lpt = (j >= 2 ? lpt * ex2_approx((m_acc - m_new) * sc) : 0.0f) + add;
      }
      rescale_to(j, m_new);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&sm.p_full[g]);
    }
    // the group that did not process the last tile consumes its maximum (keeps the named
    // barrier arrivals and synchronisations paired)
    if (((n_tiles - 1) & 1) != g) named_bar_sync(bar_recv, 64);
    // ---------------------------------------------------------------- epilogue
    // out = (O_A 2^((mA - m) sc) + O_B 2^((mB - m) sc)) / (l_A ... + l_B ...) * g_v with m the
    // final maximum; group A writes output columns [0, D/2), group B [D/2, D)
    sm.m_last[g][r] = m_acc;
    if constexpr (ABL) sm.l_last[g][r] = lpt;
    named_bar_sync(bar_epi, 64);
    const float mA = sm.m_last[0][r], mB = sm.m_last[1][r];
    const float m = fmaxf(mA, mB);
    // the last PV product of each group in this item is the most recent phase of its o_done
    // barrier (the next item's products wait on o_free, which needs this epilogue)
    const int cnt_a = (n_tiles + 1) / 2, cnt_b = n_tiles / 2;   // key tiles of each group
    ok = warp_wait(&sm.o_done[0], (done_a + cnt_a - 1) & 1, abort_flag, kStatusTimeoutSoftmax) && ok;
    if (cnt_b > 0)
      ok = warp_wait(&sm.o_done[1], (done_b + cnt_b - 1) & 1, abort_flag, kStatusTimeoutSoftmax) && ok;
    if (ok) {
      tc_fence_after();
      const bool has_b = cnt_b > 0;
      const float wa = ex2_approx((mA - m) * sc), wb = has_b ? ex2_approx((mB - m) * sc) : 0.0f;
      uint32_t lra, lrb = 0;
      tmem_ld1(lane_base + kColL0, lra);
      if (has_b) tmem_ld1(lane_base + kColL1, lrb);
      uint32_t rawa[D / 64][32], rawb[D / 64][32];
#pragma unroll
      for (int c = 0; c < D / 64; ++c) {
        tmem_ld32(lane_base + kColO0 + g * (D / 2) + 32 * c, rawa[c]);
        tmem_ld32(lane_base + kColO1 + g * (D / 2) + 32 * c, rawb[c]);
      }
      tmem_wait_ld();
      const float la = (ABL && p.l_from_ptilde) ? sm.l_last[0][r] : __uint_as_float(lra);
      const float lb = (ABL && p.l_from_ptilde) ? sm.l_last[1][r] : __uint_as_float(lrb);
      const float l = la * wa + (has_b ? lb * wb : 0.0f);
      const float inva = p.g_v / l * wa, invb = p.g_v / l * wb;
      const bool store = row < p.S_q;
      const int64_t orow = (int64_t)bh_q * p.S_q + row;
      if (store) {
#pragma unroll
        for (int c = 0; c < D / 64; ++c) {
          const int ocol = g * (D / 2) + 32 * c;
          float o[32];
#pragma unroll
          for (int i = 0; i < 32; ++i)
            o[i] = __uint_as_float(rawa[c][i]) * inva + (has_b ? __uint_as_float(rawb[c][i]) * invb : 0.0f);
          if (p.out_fp32) {
            float4* dst = reinterpret_cast<float4*>(static_cast<float*>(p.out) + orow * D + ocol);
#pragma unroll
            for (int i = 0; i < 8; ++i) dst[i] = make_float4(o[4 * i], o[4 * i + 1], o[4 * i + 2], o[4 * i + 3]);
          } else {
            uint4* dst = reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(p.out) + orow * D + ocol);
#pragma unroll
            for (int i = 0; i < 4; ++i) {
              uint32_t w[4];
#pragma unroll
              for (int q = 0; q < 4; ++q) {
                __nv_bfloat162 pr = __floats2bfloat162_rn(o[8 * i + 2 * q], o[8 * i + 2 * q + 1]);
                w[q] = *reinterpret_cast<uint32_t*>(&pr);
              }
              dst[i] = make_uint4(w[0], w[1], w[2], w[3]);
            }
          }
        }
        if (g == 0 && p.lse != nullptr) {
          const float lscale = MX ? 1.0f : gp_item;
          p.lse[orow] = m * sc * 0.69314718055994531f + logf(l * lscale);
        }
      }
    }
    done_a += cnt_a;
    done_b += cnt_b;
    // O and l have been read: the next item's first PV product may overwrite them
    tc_fence_before();
    __syncwarp();
    if (lane == 0) mbar_arrive(&sm.o_free);
    }
  }
  // ---------------------------------------------------------------- teardown
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// =======================================================================================
// self-test: one block-scaled MMA through the same descriptors and scale path
// =======================================================================================
template <bool MX>
__global__ void __launch_bounds__(128, 1)
    selftest_mma_kernel(const uint8_t* __restrict__ a, const uint8_t* __restrict__ a_sf,
                        const uint8_t* __restrict__ bmat, const uint8_t* __restrict__ b_sf, int N,
                        int K, float* __restrict__ d_out) {
  constexpr int kBlk = MX ? 32 : 16;
  __shared__ __align__(1024) uint8_t sa[128 * 64];
  __shared__ __align__(1024) uint8_t sb[256 * 64];
  __shared__ __align__(1024) uint8_t ssfa[2 * 512];
  __shared__ __align__(1024) uint8_t ssfb[4 * 512];
  __shared__ uint64_t bar;
  __shared__ uint32_t tbase;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int rb = K / 2;                                        // bytes per row (32 or 64)
  // operands -> swizzled K-major shared-memory tiles (same pattern TMA produces)
  for (int i = threadIdx.x; i < 128 * rb / 16; i += 128) {
    const int r = i / (rb / 16), c = i % (rb / 16);
    const uint4 v = *reinterpret_cast<const uint4*>(a + r * rb + c * 16);
    *reinterpret_cast<uint4*>(sa + (rb == 64 ? swz64_offset(r, c) : swz32_offset(r, c))) = v;
  }
  for (int i = threadIdx.x; i < N * rb / 16; i += 128) {
    const int r = i / (rb / 16), c = i % (rb / 16);
    const uint4 v = *reinterpret_cast<const uint4*>(bmat + r * rb + c * 16);
    *reinterpret_cast<uint4*>(sb + (rb == 64 ? swz64_offset(r, c) : swz32_offset(r, c))) = v;
  }
  // scale atoms: A has one row tile; B has ceil(N/128); groups per row tile = 32/kBlk
  const int ng = 32 / kBlk, nrt_b = (N + 127) / 128;
  for (int i = threadIdx.x; i < ng * 512 / 16; i += 128)
    reinterpret_cast<uint4*>(ssfa)[i] = reinterpret_cast<const uint4*>(a_sf)[i];
  for (int i = threadIdx.x; i < nrt_b * ng * 512 / 16; i += 128)
    reinterpret_cast<uint4*>(ssfb)[i] = reinterpret_cast<const uint4*>(b_sf)[i];
  fence_proxy_async_smem();
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    fence_barrier_init();
  }
  if (warp == 0) {
    tmem_alloc(&tbase, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tbase;
  // TMEM: D [0, N), SFA at 256 (4 columns per group), SFB at 272 (8 columns per group:
  // row tile rt of group g at 272 + 8g + 4rt)
  if (warp == 0 && elect_one()) {
    for (int g = 0; g < ng; ++g) {
      tmem_cp_sf_atom(tmem + 256 + 4 * g, smem_u32(ssfa + 512 * g));
      for (int rt = 0; rt < nrt_b; ++rt)
        tmem_cp_sf_atom(tmem + 272 + 8 * g + 4 * rt, smem_u32(ssfb + 512 * (rt * ng + g)));
    }
    const int steps = K / 64;
    const uint32_t swz = rb == 64 ? kSwiz64 : kSwiz32;
    const uint32_t sbo = rb == 64 ? 512 : 256;
    for (int ks = 0; ks < steps; ++ks) {
      const uint64_t ad = make_smem_desc(smem_u32(sa) + 32 * ks, 16, sbo, swz);
      const uint64_t bd = make_smem_desc(smem_u32(sb) + 32 * ks, 16, sbo, swz);
      if constexpr (MX) {
        const uint32_t id = 2u * (ks & 1);
        mma_mxf4(tmem, ad, bd, make_idesc_fp4(N, true, id, id), tmem + 256 + 4 * (ks >> 1),
                 tmem + 272 + 8 * (ks >> 1), ks > 0);
      } else {
        mma_nvf4(tmem, ad, bd, make_idesc_fp4(N, false, 0, 0), tmem + 256 + 4 * ks,
                 tmem + 272 + 8 * ks, ks > 0);
      }
    }
    tc_commit(&bar);
  }
  __syncwarp();
  mbar_wait(&bar, 0, &g_attn_status, kStatusTimeoutProbe);
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
    tmem_dealloc(tmem, 512);
  }
}

// elementwise 2^x through ex2_poly2 (two values per thread)
__global__ void selftest_exp2_kernel(const float* __restrict__ x, float* __restrict__ y, int64_t npairs) {
  const int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (i >= npairs) return;
  const float2 v = reinterpret_cast<const float2*>(x)[i];
  float a, b;
  ex2_poly2(a, b, v.x, v.y);
  reinterpret_cast<float2*>(y)[i] = make_float2(a, b);
}

// bounded-wait probe: waits on a barrier nothing will complete, for `wait_us` microseconds
__global__ void wait_probe_kernel(uint32_t wait_us) {
  __shared__ uint64_t bar;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    fence_barrier_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) mbar_wait(&bar, 0, &g_attn_status, kStatusTimeoutProbe, uint64_t(wait_us) * 1000);
}

cudaError_t attn_status_fetch(cudaStream_t st, uint32_t* host_word) {
  cudaError_t e = cudaMemcpyFromSymbolAsync(host_word, g_attn_status, sizeof(uint32_t), 0,
                                            cudaMemcpyDeviceToHost, st);
  if (e != cudaSuccess) return e;
  const uint32_t zero = 0;
  e = cudaMemcpyToSymbolAsync(g_attn_status, &zero, sizeof(uint32_t), 0, cudaMemcpyHostToDevice, st);
  if (e != cudaSuccess) return e;
  return cudaStreamSynchronize(st);
}

// Host side of the MXFP4 P scale rule: log2 of the bound (rounded once to FP32).
static void fill_p_scale_rule(AttnParams& prm) {
  prm.log2_qmax_p = prm.qmax_p > 0.0f ? static_cast<float>(std::log2(static_cast<double>(prm.qmax_p))) : 0.0f;
}

// bf16 operands of the hybrid prefill's full-precision tiles (rows of d = 128 bf16 = 256 bytes,
// loaded as two 128-byte chunks with the 128-byte swizzle)
struct HyOperands {
  const void *q, *k, *v, *vl_k, *vl_v;
  int max_vl;
};

template <int D, bool MX, bool CAUSAL, bool ABL = false, bool HYB = false>
static fa4q_status launch_attn(const uint8_t* q, const uint8_t* k, const uint8_t* vt,
                               const AttnParams& prm, cudaStream_t st, const HyOperands* hy = nullptr) {
  CUtensorMap tq, tk, tv;
  const CUtensorMapSwizzle qk_swz = D == 128 ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_32B;
  if (!make_map_3d(&tq, q, D / 2, prm.S_q, (uint64_t)prm.B * prm.Hq, D / 2, kBM, qk_swz) ||
      !make_map_3d(&tk, k, D / 2, prm.S_k, (uint64_t)prm.B * prm.Hkv, D / 2, kBN, qk_swz) ||
      !make_map_3d(&tv, vt, prm.S_kpad / 2, D, (uint64_t)prm.B * prm.Hkv, kBN / 2, D,
                   CU_TENSOR_MAP_SWIZZLE_64B))
    return FA4Q_ERR_CUDA;
  CUtensorMap tq16 = tq, tk16 = tq, tv16 = tq, tvlk = tq, tvlv = tq;   // unused unless hybrid
  if (HYB) {
    const CUtensorMapSwizzle sw = CU_TENSOR_MAP_SWIZZLE_128B;
    const uint64_t nq = (uint64_t)prm.B * prm.Hq, nk = (uint64_t)prm.B * prm.Hkv;
    if (!hy || !make_map_3d(&tq16, hy->q, 2 * D, prm.S_q, nq, 128, kBM, sw) ||
        !make_map_3d(&tk16, hy->k, 2 * D, prm.S_k, nk, 128, kHyKeys, sw) ||
        !make_map_3d(&tv16, hy->v, 2 * D, prm.S_k, nk, 128, kHyKeys, sw))
      return FA4Q_ERR_CUDA;
    if (hy->max_vl > 0 && (!make_map_3d(&tvlk, hy->vl_k, 2 * D, hy->max_vl, nk, 128, kHyKeys, sw) ||
                           !make_map_3d(&tvlv, hy->vl_v, 2 * D, hy->max_vl, nk, 128, kHyKeys, sw)))
      return FA4Q_ERR_CUDA;
  }
  const size_t smem = sizeof(Smem<D, MX, HYB>) + 1024;
  // Short items (few key tiles on average, as in causal attention over a few thousand keys)
  // run persistently, one CTA per SM walking the item list, so the per-CTA setup and the
  // pipeline fill and drain of an item overlap the neighbouring items.  Long items run one
  // CTA per item: the block scheduler then balances them dynamically across the SMs, and the
  // kernel is compiled without the item loop.
  const int n_ktiles = (prm.S_k + kBN - 1) / kBN;
  const double avg_tiles = CAUSAL ? 0.5 * (std::min(prm.n_qtiles, n_ktiles) + 1) : n_ktiles;
  const bool persist = avg_tiles <= 48.0 && prm.n_items > num_sms();
  auto kern = persist ? attn_fwd_kernel<D, MX, CAUSAL, true, ABL, HYB> : attn_fwd_kernel<D, MX, CAUSAL, false, ABL, HYB>;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) != cudaSuccess)
    return FA4Q_ERR_CUDA;
  const dim3 grid(static_cast<unsigned>(persist ? num_sms() : prm.n_items));
  kern<<<grid, kThreads, smem, st>>>(tq, tk, tv, tq16, tk16, tv16, tvlk, tvlv, prm);
  return launch_status();
}

}  // namespace fa4q

using namespace fa4q;

extern "C" fa4q_status fa4q_attn_fwd_ex(const uint8_t* q, const uint8_t* q_sf, const uint8_t* k,
                                        const uint8_t* k_sf, const uint8_t* vt, const uint8_t* vt_sf,
                                        float g_q, float g_k, float g_v, int B, int Hq, int Hkv,
                                        int S_q, int S_k, int d, fa4q_format fmt, float qmax_p,
                                        int causal, float sm_scale, int rescale_tau,
                                        int l_from_ptilde, void* out, int out_is_fp32, float* lse,
                                        void* stream) {
  if (fmt != FA4Q_NVFP4 && fmt != FA4Q_MXFP4) return FA4Q_ERR_INVALID_ARG;
  if (rescale_tau < 0 || rescale_tau > 30) return FA4Q_ERR_INVALID_ARG;
  if (l_from_ptilde != 0 && l_from_ptilde != 1) return FA4Q_ERR_INVALID_ARG;
  // NVFP4 P under a kept reference: a key equal to the reference lands on 1/(s g_P 2^tau),
  // an E2M1 tie for some UE4M3 s, which the exponential form cannot reproduce exactly
  if (rescale_tau > 0 && fmt == FA4Q_NVFP4) return FA4Q_ERR_UNSUPPORTED;
  if (!q || !q_sf || !k || !k_sf || !vt || !vt_sf || !out) return FA4Q_ERR_INVALID_ARG;
  if (B < 0 || Hq <= 0 || Hkv <= 0 || S_q < 0 || S_k < 0) return FA4Q_ERR_INVALID_ARG;
  if (Hq % Hkv != 0) return FA4Q_ERR_INVALID_ARG;
  if (causal && S_q != S_k) return FA4Q_ERR_INVALID_ARG;
  if (d != 64 && d != 128) return FA4Q_ERR_UNSUPPORTED;
  if (!(qmax_p >= 0.0f) || !isfinite(qmax_p)) return FA4Q_ERR_INVALID_ARG;
  if (fmt == FA4Q_MXFP4) { g_q = g_k = g_v = 1.0f; }
  if (!(g_q > 0.0f) || !(g_k > 0.0f) || !(g_v > 0.0f)) return FA4Q_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(vt) || !aligned16(q_sf) || !aligned16(k_sf) ||
      !aligned16(vt_sf) || !aligned16(out))
    return FA4Q_ERR_INVALID_ARG;
  if (B == 0 || S_q == 0) return FA4Q_OK;
  if (S_k == 0) return FA4Q_ERR_INVALID_ARG;
  const int n_qtiles = (S_q + kBM - 1) / kBM;
  if (static_cast<int64_t>(B) * Hq * n_qtiles > 0x7fffffff) return FA4Q_ERR_UNSUPPORTED;
  AttnParams prm{};
  prm.q_sf = q_sf;
  prm.k_sf = k_sf;
  prm.vt_sf = vt_sf;
  prm.out = out;
  prm.lse = lse;
  prm.B = B;
  prm.Hq = Hq;
  prm.Hkv = Hkv;
  prm.S_q = S_q;
  prm.S_k = S_k;
  prm.S_kpad = (S_k + 31) / 32 * 32;
  prm.n_qtiles = n_qtiles;
  prm.n_items = B * Hq * n_qtiles;
  const float sms = sm_scale > 0.0f ? sm_scale : 1.0f / sqrtf((float)d);
  prm.score_scale_log2 = sms * g_q * g_k * kLog2e;
  prm.g_v = g_v;
  prm.qmax_p = qmax_p;
  prm.tau = static_cast<float>(rescale_tau);
  prm.gp = kGpNvfp4 * static_cast<float>(1u << rescale_tau);     // exact power-of-two multiple
  prm.inv6gp = 1.0f / (6.0f * prm.gp);
  fill_p_scale_rule(prm);
  prm.l_from_ptilde = l_from_ptilde;
  prm.causal = causal;
  prm.out_fp32 = out_is_fp32;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const bool mx = fmt == FA4Q_MXFP4;
  if (rescale_tau > 0 || l_from_ptilde) {
    if (d != 128) return FA4Q_ERR_UNSUPPORTED;   // the ablation kernels are built for d = 128
    if (mx) return causal ? launch_attn<128, true, true, true>(q, k, vt, prm, st) : launch_attn<128, true, false, true>(q, k, vt, prm, st);
    return causal ? launch_attn<128, false, true, true>(q, k, vt, prm, st) : launch_attn<128, false, false, true>(q, k, vt, prm, st);
  }
  if (d == 128) {
    if (mx) return causal ? launch_attn<128, true, true>(q, k, vt, prm, st) : launch_attn<128, true, false>(q, k, vt, prm, st);
    return causal ? launch_attn<128, false, true>(q, k, vt, prm, st) : launch_attn<128, false, false>(q, k, vt, prm, st);
  }
  if (mx) return causal ? launch_attn<64, true, true>(q, k, vt, prm, st) : launch_attn<64, true, false>(q, k, vt, prm, st);
  return causal ? launch_attn<64, false, true>(q, k, vt, prm, st) : launch_attn<64, false, false>(q, k, vt, prm, st);
}

extern "C" fa4q_status fa4q_attn_fwd(const uint8_t* q, const uint8_t* q_sf, const uint8_t* k,
                                     const uint8_t* k_sf, const uint8_t* vt, const uint8_t* vt_sf,
                                     float g_q, float g_k, float g_v, int B, int Hq, int Hkv,
                                     int S_q, int S_k, int d, fa4q_format fmt, float qmax_p,
                                     int causal, float sm_scale, void* out, int out_is_fp32,
                                     float* lse, void* stream) {
  return fa4q_attn_fwd_ex(q, q_sf, k, k_sf, vt, vt_sf, g_q, g_k, g_v, B, Hq, Hkv, S_q, S_k, d, fmt,
                          qmax_p, causal, sm_scale, 0, 0, out, out_is_fp32, lse, stream);
}

extern "C" fa4q_status fa4q_selftest_block_mma(const uint8_t* a, const uint8_t* a_sf, const uint8_t* b,
                                               const uint8_t* b_sf, int N, int K, fa4q_format fmt,
                                               float* d_out, void* stream) {
  if (!a || !a_sf || !b || !b_sf || !d_out) return FA4Q_ERR_INVALID_ARG;
  if (K != 64 && K != 128) return FA4Q_ERR_UNSUPPORTED;
  if (N < 16 || N > 256 || N % 16 != 0) return FA4Q_ERR_UNSUPPORTED;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (fmt == FA4Q_MXFP4)
    selftest_mma_kernel<true><<<1, 128, 0, st>>>(a, a_sf, b, b_sf, N, K, d_out);
  else if (fmt == FA4Q_NVFP4)
    selftest_mma_kernel<false><<<1, 128, 0, st>>>(a, a_sf, b, b_sf, N, K, d_out);
  else
    return FA4Q_ERR_INVALID_ARG;
  return launch_status();
}

extern "C" fa4q_status fa4q_selftest_exp2(const float* x, float* y, int64_t n, void* stream) {
  if (!x || !y || n < 0 || (n & 1)) return FA4Q_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(x) | reinterpret_cast<uintptr_t>(y)) & 7) return FA4Q_ERR_INVALID_ARG;
  if (n == 0) return FA4Q_OK;
  const int64_t npairs = n / 2;
  const int64_t blocks = (npairs + 255) / 256;
  if (blocks > 0x7fffffff) return FA4Q_ERR_UNSUPPORTED;
  selftest_exp2_kernel<<<static_cast<unsigned>(blocks), 256, 0, static_cast<cudaStream_t>(stream)>>>(x, y, npairs);
  return launch_status();
}

extern "C" fa4q_status fa4q_selftest_wait_timeout(uint32_t wait_us, void* stream) {
  wait_probe_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(wait_us);
  return launch_status();
}

// =======================================================================================
// hybrid-precision prefill: one kernel, the full-precision tiles first, then the FP4 tiles
// =======================================================================================
extern "C" fa4q_status fa4q_attn_fwd_hybrid(
    const uint8_t* q, const uint8_t* q_sf, const uint8_t* k, const uint8_t* k_sf, const uint8_t* vt,
    const uint8_t* vt_sf, const void* q_bf16, const void* k_bf16, const void* v_bf16,
    const int32_t* vl_pos, const int32_t* vl_count, const void* vl_k, const void* vl_v, int max_vl,
    const uint64_t* vl_excl, float g_q, float g_k, float g_v, int B, int Hq, int Hkv, int S, int d,
    int window, fa4q_format fmt, float qmax_p, float sm_scale, void* out, int out_is_fp32, float* lse,
    void* stream) {
  if (fmt != FA4Q_NVFP4 && fmt != FA4Q_MXFP4) return FA4Q_ERR_INVALID_ARG;
  if (!q || !q_sf || !k || !k_sf || !vt || !vt_sf || !q_bf16 || !k_bf16 || !v_bf16 || !out)
    return FA4Q_ERR_INVALID_ARG;
  if (B < 0 || Hq <= 0 || Hkv <= 0 || S < 0 || Hq % Hkv != 0 || window < 1 || max_vl < 0)
    return FA4Q_ERR_INVALID_ARG;
  if (max_vl > 0 && (!vl_pos || !vl_count || !vl_k || !vl_v || !vl_excl)) return FA4Q_ERR_INVALID_ARG;
  if (d != 128) return FA4Q_ERR_UNSUPPORTED;
  if (!(qmax_p >= 0.0f) || !isfinite(qmax_p)) return FA4Q_ERR_INVALID_ARG;
  if (fmt == FA4Q_MXFP4) { g_q = g_k = g_v = 1.0f; }
  if (!(g_q > 0.0f) || !(g_k > 0.0f) || !(g_v > 0.0f)) return FA4Q_ERR_INVALID_ARG;
  // the full-precision normaliser multiplies by g_v in bf16: g_v must be a bf16 value
  uint32_t gv_bits;
  std::memcpy(&gv_bits, &g_v, sizeof(gv_bits));
  if ((gv_bits & 0xFFFFu) != 0u) return FA4Q_ERR_UNSUPPORTED;
  if (!aligned16(q) || !aligned16(k) || !aligned16(vt) || !aligned16(q_sf) || !aligned16(k_sf) ||
      !aligned16(vt_sf) || !aligned16(out) || !aligned16(q_bf16) || !aligned16(k_bf16) ||
      !aligned16(v_bf16) || (vl_k && !aligned16(vl_k)) || (vl_v && !aligned16(vl_v)))
    return FA4Q_ERR_INVALID_ARG;
  if (B == 0 || S == 0) return FA4Q_OK;
  const int n_qtiles = (S + kBM - 1) / kBM;
  if (static_cast<int64_t>(B) * Hq * n_qtiles > 0x7fffffff || B > 65535 || Hq > 65535) return FA4Q_ERR_UNSUPPORTED;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const float sms = sm_scale > 0.0f ? sm_scale : 1.0f / sqrtf((float)d);
  AttnParams prm{};
  prm.q_sf = q_sf;
  prm.k_sf = k_sf;
  prm.vt_sf = vt_sf;
  prm.out = out;
  prm.lse = lse;
  prm.B = B;
  prm.Hq = Hq;
  prm.Hkv = Hkv;
  prm.S_q = S;
  prm.S_k = S;
  prm.S_kpad = (S + 31) / 32 * 32;
  prm.n_qtiles = n_qtiles;
  prm.n_items = B * Hq * n_qtiles;
  prm.score_scale_log2 = sms * g_q * g_k * kLog2e;
  prm.g_v = g_v;
  prm.qmax_p = qmax_p;
  prm.causal = 1;
  prm.out_fp32 = out_is_fp32;
  prm.gp = kGpNvfp4;
  prm.inv6gp = kInvSixGp;
  fill_p_scale_rule(prm);
  prm.hy_window = window;
  prm.hy_excl_words = max_vl > 0 ? (S + 63) / 64 : 0;
  prm.hy_excl = max_vl > 0 ? vl_excl : nullptr;     // read only while a word index is < hy_excl_words
  prm.hy_vl_pos = max_vl > 0 ? vl_pos : nullptr;
  prm.hy_vl_count = max_vl > 0 ? vl_count : nullptr;
  prm.hy_max_vl = max_vl;
  prm.hy_inv_gqgk = 1.0f / (g_q * g_k);
  const double units = fmt == FA4Q_MXFP4 ? 1.0 : static_cast<double>(kGpNvfp4) * g_v;
  prm.hy_lp16 = static_cast<float>(std::log2(units));
  prm.hy_ones_bits = gv_bits >> 16;
  const HyOperands hy{q_bf16, k_bf16, v_bf16, vl_k, vl_v, max_vl};
  if (fmt == FA4Q_MXFP4) return launch_attn<128, true, true, false, true>(q, k, vt, prm, st, &hy);
  return launch_attn<128, false, true, false, true>(q, k, vt, prm, st, &hy);
}
