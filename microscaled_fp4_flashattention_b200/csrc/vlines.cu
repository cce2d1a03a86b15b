// vlines.cu - vertical-line identification for the hybrid KV cache (sm_100a).
//
// What it computes, per (sequence b, kv-head h), over the candidate prefix [0, n_prefix[b]):
//   s_ij   = (q_i . k_j) * sm_scale     q_i: the R = (Hq/Hkv) * n_obs observation query rows
//                                       of the group's q-heads (BF16), k_j BF16
//   p_ij   = softmax_j(s_ij)            exact, over the whole candidate prefix
//   mass_j = sum_i p_ij                 accumulated column mass of key j
//   keep   = the ceil(rho * n_prefix) largest masses, equal masses lowest position first
// and writes the kept positions (ascending), the exclusion mask of the paged FP4 cache and
// the BF16 K / V rows of the kept tokens (the full-precision set the decode reads).
// Source: HyQuant (Hybrid-Precision Quantization for LLM Attention) - the tokens that
// receive a large accumulated attention mass from later queries ("vertical lines") stay in
// full precision, the rest of the non-window prefix is stored in 4 bits; the mass is
// gathered from a set of observation queries.
//
// Kernels:
//   colmass_kernel<D, 0>  persistent CTAs over (sequence, kv-head, 1024-key chunk) items:
//                         S = Q K^T on the tensor cores (tcgen05 kind::f16, M = 128 rows,
//                         N = 128 keys, FP32 in TMEM), one observation row per TMEM lane, so
//                         each thread keeps its rows' running maximum and sum of exp2 alone;
//                         two softmax groups take alternate key tiles -> partials (m, l) per
//                         (row, chunk, group)
//   vl_lse_kernel         partials -> -lse2[row] = -(m + log2(l))   (log2 domain)
//   colmass_kernel<D, 1>  the same products transposed, S^T = K Q^T (M = 128 keys, N = 128
//                         rows, twice), one key per TMEM lane: each thread sums exp2(s2_ij - lse2_i)
//                         over the 256 rows of its key alone and writes the key's mass
//   vl_select_kernel      grid (kv-head, sequence): the masses in shared memory, an 8-bit
//                         radix select of the threshold (4 passes), an ordered compaction
//                         (positions ascending) and the exclusion-mask words
//   vl_gather_kernel      the kept rows of K and V, position order
// In both column-mass passes ten of every sixteen exponentials run on MUFU, six on the FMA
// pipe.
// The scores are computed twice rather than stored (R x n_prefix FP32 per group would be
// 33 MB per (sequence, kv-head) at 32K keys).
#include <math.h>
#include <stddef.h>

#include "fa4q_common.cuh"
#include "fa4q_internal.h"

namespace fa4q {

static __device__ uint32_t g_vl_status;

cudaError_t vl_status_fetch(cudaStream_t st, uint32_t* host_word) {
  cudaError_t e = cudaMemcpyFromSymbolAsync(host_word, g_vl_status, sizeof(uint32_t), 0, cudaMemcpyDeviceToHost, st);
  if (e != cudaSuccess) return e;
  const uint32_t zero = 0;
  e = cudaMemcpyToSymbolAsync(g_vl_status, &zero, sizeof(uint32_t), 0, cudaMemcpyHostToDevice, st);
  if (e != cudaSuccess) return e;
  return cudaStreamSynchronize(st);
}

constexpr int kVlChunk = 1024;           // keys per work item (one partial per row)
constexpr int kCmKeys = 128;             // keys per tile
constexpr int kCmRows = 256;             // observation rows held per group (R <= 256)
constexpr int kCmStages = 4;             // K tiles in flight
constexpr int kCmThreads = 320;          // warp 0 TMA, warp 1 MMA, warps 2..9 two warpgroups
constexpr int kSelThreads = 1024;
constexpr float kVlLog2e = 1.4426950408889634f;

struct VlParams {
  const int32_t* n_prefix;   // [B]
  float* part;               // [B][Hkv][R][chunks][2 softmax groups][2]: (m, l)
  float* nlse2;              // [B][Hkv][R]: -log2 sum_j 2^(s2_ij) per row
  float* mass;               // [B][Hkv][L]
  int B, Hq, Hkv, n_obs, L, d, R, chunks, n_items;
  float c2;                  // sm_scale * log2(e)
};

FA4Q_DEVINL float vl_ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// Packed FP32 pairs (f32x2 instructions: one issue slot for two lanes of work)
FA4Q_DEVINL float2 fma2(float2 a, float2 b, float2 c) {
  float2 d;
  asm("{\n\t.reg .b64 ra, rb, rc, rd;\n\t"
      "mov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\tmov.b64 rc, {%6, %7};\n\t"
      "fma.rn.f32x2 rd, ra, rb, rc;\n\tmov.b64 {%0, %1}, rd;\n\t}"
      : "=f"(d.x), "=f"(d.y)
      : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y), "f"(c.x), "f"(c.y));
  return d;
}
FA4Q_DEVINL float2 add2(float2 a, float2 b) {
  float2 d;
  asm("{\n\t.reg .b64 ra, rb, rd;\n\t"
      "mov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\t"
      "add.rn.f32x2 rd, ra, rb;\n\tmov.b64 {%0, %1}, rd;\n\t}"
      : "=f"(d.x), "=f"(d.y)
      : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y));
  return d;
}
FA4Q_DEVINL float vl_max3(float a, float b, float c) {
  float d;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}

// 2^x for a pair of values on the FMA pipe (the MUFU pipe is the column-mass passes' limit,
// so six of every sixteen exponentials take this path):
//   x clamped at -126 (2^-126 stands for anything smaller: far below any mass that counts)
//   t = x + 1.5*2^23 rounded toward -inf -> floor(x) in the low mantissa bits of t
//   f = x - (t - 1.5*2^23) in [0, 1), exact
//   p = c0 + f (c1 + f (c2 + f (c3 + f c4)))   2^f, minimax (relative) on [0, 1),
//                                              max relative error 2.7e-6
//   2^x = p * 2^floor(x): floor(x) added to the exponent field of p (bits of t << 23)
// Coefficients: degree-4 Lawson fit of 2^f on [0, 1) (fit_exp2_poly.py beside this file).
constexpr float kVlE0 = 1.0000026226043701f, kVlE1 = 0.6930038332939148f, kVlE2 = 0.2414427399635315f;
constexpr float kVlE3 = 0.05201146751642227f, kVlE4 = 0.01353417057543993f;
FA4Q_DEVINL float2 vl_ex2_fma2(float2 x) {
  x.x = fmaxf(x.x, -126.0f);
  x.y = fmaxf(x.y, -126.0f);
  uint32_t t0, t1, p0, p1;
  asm("{\n\t.reg .b64 rx, rt, rj, rf, rp, rm, c0, c1, c2, c3, c4;\n\t"
      "mov.b64 rx, {%4, %5};\n\tmov.b64 rm, {%6, %6};\n\t"
      "add.rm.f32x2 rt, rx, rm;\n\tsub.rn.f32x2 rj, rt, rm;\n\tsub.rn.f32x2 rf, rx, rj;\n\t"
      "mov.b64 c4, {%11, %11};\n\tmov.b64 c3, {%10, %10};\n\tmov.b64 c2, {%9, %9};\n\t"
      "mov.b64 c1, {%8, %8};\n\tmov.b64 c0, {%7, %7};\n\t"
      "fma.rn.f32x2 rp, c4, rf, c3;\n\tfma.rn.f32x2 rp, rp, rf, c2;\n\t"
      "fma.rn.f32x2 rp, rp, rf, c1;\n\tfma.rn.f32x2 rp, rp, rf, c0;\n\t"
      "mov.b64 {%0, %1}, rt;\n\tmov.b64 {%2, %3}, rp;\n\t}"
      : "=r"(t0), "=r"(t1), "=r"(p0), "=r"(p1)
      : "f"(x.x), "f"(x.y), "f"(12582912.0f), "f"(kVlE0), "f"(kVlE1), "f"(kVlE2), "f"(kVlE3), "f"(kVlE4));
  return make_float2(__uint_as_float(p0 + (t0 << 23)), __uint_as_float(p1 + (t1 << 23)));
}

// sum of 2^x over sixteen values (x = s * c2 + o, pairs): ten on MUFU, six on the FMA pipe,
// as two packed partial sums
FA4Q_DEVINL void vl_sum16(const uint32_t* s, float2 c2, const float2* o, float2& acc0, float2& acc1) {
  float2 x[8];
#pragma unroll
  for (int k = 0; k < 8; ++k) x[k] = fma2(make_float2(__uint_as_float(s[2 * k]), __uint_as_float(s[2 * k + 1])), c2, o[k]);
#pragma unroll
  for (int k = 0; k < 5; ++k) {
    const float2 y = make_float2(vl_ex2(x[k].x), vl_ex2(x[k].y));
    if (k & 1) acc1 = add2(acc1, y);
    else acc0 = add2(acc0, y);
  }
  acc1 = add2(acc1, vl_ex2_fma2(x[5]));
  acc0 = add2(acc0, vl_ex2_fma2(x[6]));
  acc1 = add2(acc1, vl_ex2_fma2(x[7]));
}

// (m, l) of two partial softmax sums merged (m = -inf means empty)
FA4Q_DEVINL void merge_ml(float& m, float& l, float m2, float l2) {
  const float mn = fmaxf(m, m2);
  if (mn == -INFINITY) return;
  l = (m == -INFINITY ? 0.0f : l * vl_ex2(m - mn)) + (m2 == -INFINITY ? 0.0f : l2 * vl_ex2(m2 - mn));
  m = mn;
}

// Shared memory of the column-mass kernel: the group's observation rows and a ring of key
// tiles, both as 64-element column chunks of 128-byte rows with the 128-byte swizzle (the
// layout TMA writes and the K-major MMA operand reads), 1024-byte aligned.
template <int D>
struct CmSmem {
  static constexpr int kChunks = D / 64;
  uint8_t q[kChunks][kCmRows * 128];
  uint8_t k[kCmStages][kChunks][kCmKeys * 128];
  float nlse[kCmRows];                   // pass 1: -lse2 of the group's rows, -inf past R
  uint64_t q_full, q_free;
  uint64_t k_full[kCmStages], k_empty[kCmStages];
  uint64_t s_full[2][2], s_free[2][2];   // [buffer][128-column half]
  uint64_t drain;
  uint32_t tmem_base;
  uint32_t abort_flag;
};

// Bounded wait shared by the roles of one CTA: a wait that expires records `code` and sets
// the CTA's abort flag, after which every later wait returns false at once.
FA4Q_DEVINL bool cm_wait(uint64_t* bar, uint32_t parity, volatile uint32_t* abort_flag, uint32_t code) {
  if (*abort_flag) return false;
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = globaltimer_ns();
  while (true) {
    if (mbar_try_wait(bar, parity)) return true;
    if (*abort_flag) return false;
    if (globaltimer_ns() - t0 > kWaitNs) break;
  }
  atomicOr(&g_vl_status, code);
  *abort_flag = 1;
  return false;
}

FA4Q_DEVINL bool cm_warp_wait(uint64_t* bar, uint32_t parity, volatile uint32_t* abort_flag, uint32_t code) {
  return __all_sync(0xffffffffu, cm_wait(bar, parity, abort_flag, code));
}

struct CmItem {
  int bh, b, h, chunk, key_begin, key_end, n_tiles;
};

FA4Q_DEVINL CmItem cm_item(const VlParams& p, int u) {
  CmItem it;
  it.bh = u / p.chunks;
  it.chunk = u - it.bh * p.chunks;
  it.b = it.bh / p.Hkv;
  it.h = it.bh - it.b * p.Hkv;
  const int n_pre = min(max(p.n_prefix[it.b], 0), p.L);
  it.key_begin = it.chunk * kVlChunk;
  it.key_end = min(it.key_begin + kVlChunk, n_pre);
  it.n_tiles = it.key_end > it.key_begin ? (it.key_end - it.key_begin + kCmKeys - 1) / kCmKeys : 0;
  return it;
}

// Persistent column-mass pass (PASS 0: per-row partials of the log-sum-exp; PASS 1: column
// masses).  CTA c takes the contiguous item range [c n / G, (c+1) n / G) of the
// (sequence, kv-head, chunk) list, so it changes group (and reloads the observation rows)
// once or twice; every role walks the same items and derives its barrier phases from its own
// counters.
template <int D, int PASS>
__global__ void __launch_bounds__(kCmThreads, 1)
    colmass_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                   const VlParams p) {
  using SM = CmSmem<D>;
  constexpr int kCh = SM::kChunks;
  extern __shared__ uint8_t smem_raw[];
  SM& sm = *reinterpret_cast<SM*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  volatile uint32_t* abort_flag = &sm.abort_flag;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int G = p.Hq / p.Hkv;
  const int u0 = static_cast<int>(static_cast<int64_t>(blockIdx.x) * p.n_items / gridDim.x);
  const int u1 = static_cast<int>(static_cast<int64_t>(blockIdx.x + 1) * p.n_items / gridDim.x);

  if (threadIdx.x == 0) {
    mbar_init(&sm.q_full, 1);
    mbar_init(&sm.q_free, PASS == 1 ? 9 : 1);      // the MMA commit (+ the 8 softmax warps)
    for (int s = 0; s < kCmStages; ++s) {
      mbar_init(&sm.k_full[s], 1);
      mbar_init(&sm.k_empty[s], 1);
    }
    for (int s = 0; s < 2; ++s)
      for (int hh = 0; hh < 2; ++hh) {
        mbar_init(&sm.s_full[s][hh], 1);
        mbar_init(&sm.s_free[s][hh], 4);          // the four warps of softmax group s
      }
    mbar_init(&sm.drain, 1);
    sm.abort_flag = 0;
    fence_barrier_init();
  }
  if constexpr (PASS == 1) {
    // rows past R take no part: 2^(s - inf) = 0 on MUFU, 2^-126 on the FMA path (the copies
    // below write only [0, R))
    for (int i = p.R + static_cast<int>(threadIdx.x); i < kCmRows; i += kCmThreads) sm.nlse[i] = -INFINITY;
  }
  if (warp == 1) {
    tmem_alloc(&sm.tmem_base, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sm.tmem_base;

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (elect_one()) {
      prefetch_tmap(&tm_q);
      prefetch_tmap(&tm_k);
      int T = 0, nq = 0, cur = -1;
      bool go = true;
      for (int u = u0; go && u < u1; ++u) {
        const CmItem it = cm_item(p, u);
        if (it.n_tiles == 0) continue;
        if (it.bh != cur) {
          // the observation rows of the new group (+ its -lse2 in pass 1) once every product
          // (and, in pass 1, every softmax warp) is done with the previous group's
          if (nq > 0 && !cm_wait(&sm.q_free, (nq - 1) & 1, abort_flag, kStatusTimeoutTmaFull)) break;
          const int row0 = (it.b * p.Hq + it.h * G) * p.n_obs;
          mbar_arrive_expect_tx(&sm.q_full, kCh * kCmRows * 128 + (PASS == 1 ? p.R * 4 : 0));
          for (int c = 0; c < kCh; ++c) {
            tma_load_3d(sm.q[c], &tm_q, 128 * c, row0, 0, &sm.q_full);
            tma_load_3d(sm.q[c] + 128 * 128, &tm_q, 128 * c, row0 + 128, 0, &sm.q_full);
          }
          if constexpr (PASS == 1) bulk_load(sm.nlse, p.nlse2 + static_cast<int64_t>(it.bh) * p.R, p.R * 4, &sm.q_full);
          ++nq;
          cur = it.bh;
        }
        for (int j = 0; j < it.n_tiles; ++j, ++T) {
          const int s = T % kCmStages;
          if (T >= kCmStages &&
              !cm_wait(&sm.k_empty[s], ((T / kCmStages) - 1) & 1, abort_flag, kStatusTimeoutTmaFull)) {
            go = false;
            break;
          }
          mbar_arrive_expect_tx(&sm.k_full[s], kCh * kCmKeys * 128);
          for (int c = 0; c < kCh; ++c)
            tma_load_3d(sm.k[s][c], &tm_k, 128 * c, it.key_begin + j * kCmKeys, it.bh, &sm.k_full[s]);
        }
      }
      // drain: every issued copy lands before the CTA may exit
      for (int t = max(0, T - kCmStages); t < T; ++t)
        mbar_wait(&sm.k_full[t % kCmStages], (t / kCmStages) & 1, &g_vl_status, kStatusTimeoutDrain);
      if (nq > 0) mbar_wait(&sm.q_full, (nq - 1) & 1, &g_vl_status, kStatusTimeoutDrain);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (elect_one()) {
      // descriptors: base descriptor + byte offset / 16 (shared memory < 256 KB: no carry)
      const uint64_t dsc = make_smem_desc(smem_u32(&sm), 16, 1024, kSwiz128);
      constexpr uint64_t oq = offsetof(SM, q) >> 4, ok = offsetof(SM, k) >> 4;
      constexpr uint64_t kQc = kCmRows * 128 >> 4, kKc = kCmKeys * 128 >> 4, kKs = kCh * kKc;
      constexpr uint64_t kQh = 128 * 128 >> 4;
      const uint32_t idesc = make_idesc_bf16(128, false);
      int T = 0, nq = 0, cur = -1;
      bool ok_run = true;
      for (int u = u0; ok_run && u < u1; ++u) {
        const CmItem it = cm_item(p, u);
        if (it.n_tiles == 0) continue;
        if (it.bh != cur) {
          if (nq > 0) tc_commit(&sm.q_free);
          if (!cm_wait(&sm.q_full, nq & 1, abort_flag, kStatusTimeoutMma)) break;
          tc_fence_after();
          ++nq;
          cur = it.bh;
        }
        for (int j = 0; j < it.n_tiles && ok_run; ++j, ++T) {
          const int s = T % kCmStages, buf = T & 1;
          if (!cm_wait(&sm.k_full[s], (T / kCmStages) & 1, abort_flag, kStatusTimeoutMma)) {
            ok_run = false;
            break;
          }
          // the two 128-column halves of the buffer (rows 0..127 and 128..255), each issued
          // as soon as the softmax group has read that half of the tile two steps back
#pragma unroll
          for (int hh = 0; hh < 2; ++hh) {
            if (T >= 2 && !cm_wait(&sm.s_free[buf][hh], ((T >> 1) - 1) & 1, abort_flag, kStatusTimeoutMma)) {
              ok_run = false;
              break;
            }
            tc_fence_after();
            const uint32_t dcol = tmem + 256u * buf + 128u * hh;
#pragma unroll
            for (int kk = 0; kk < D / 16; ++kk) {
              const uint64_t qd = dsc + oq + (kk >> 2) * kQc + hh * kQh + 2 * (kk & 3);
              const uint64_t kd = dsc + ok + s * kKs + (kk >> 2) * kKc + 2 * (kk & 3);
              if constexpr (PASS == 0) mma_bf16(dcol, qd, kd, idesc, kk > 0);   // S[row][key]
              else mma_bf16(dcol, kd, qd, idesc, kk > 0);                       // S^T[key][row]
            }
            tc_commit(&sm.s_full[buf][hh]);
          }
          if (!ok_run) break;
          tc_commit(&sm.k_empty[s]);
        }
      }
      // drain: every product this thread issued completes before TMEM is released
      tc_commit(&sm.drain);
      mbar_wait(&sm.drain, 0, &g_vl_status, kStatusTimeoutDrain);
    }
  } else {
    // ------------------------------------------------------------ softmax groups
    // Two groups of four warps take alternate key tiles (group g the tiles T with T % 2 = g,
    // whose products sit in S buffer g), so one group's wait for its products and its TMEM
    // loads overlap the other group's exponentials.  Warp w reads TMEM lanes 32 (w % 4) ..;
    // a thread takes the buffer's two 128-column halves one after the other (pass 0: rows
    // lq and 128 + lq, a running maximum and sum each; pass 1: rows 0..255 of key lq).
    const int g = (warp - 2) >> 2, lq = 32 * (warp & 3) + lane;
    const uint32_t tl = tmem + (static_cast<uint32_t>(32 * (warp & 3)) << 16) + 256u * g;
    const float2 c2 = make_float2(p.c2, p.c2);
    int T = 0, nq = 0, cur = -1;
    bool ok_run = true;
    for (int u = u0; ok_run && u < u1; ++u) {
      const CmItem it = cm_item(p, u);
      const int64_t bh = it.bh;
      const int T0 = T;
      T += it.n_tiles;
      if constexpr (PASS == 0) {
        float m_run[2] = {-INFINITY, -INFINITY}, l_run[2] = {0.0f, 0.0f};
        for (int j = ((T0 & 1) == g) ? 0 : 1; j < it.n_tiles; j += 2) {
          const int t = T0 + j;
          const int valid = min(kCmKeys, it.key_end - (it.key_begin + j * kCmKeys));
#pragma unroll
          for (int hh = 0; hh < 2; ++hh) {
            if (!cm_warp_wait(&sm.s_full[g][hh], (t >> 1) & 1, abort_flag, kStatusTimeoutSoftmax)) {
              ok_run = false;
              break;
            }
            tc_fence_after();
            uint32_t r[4][32];
#pragma unroll
            for (int q4 = 0; q4 < 4; ++q4) tmem_ld32(tl + 128u * hh + 32u * q4, r[q4]);
            tmem_wait_ld();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&sm.s_free[g][hh]);
            if (valid < kCmKeys) {
#pragma unroll
              for (int q4 = 0; q4 < 4; ++q4)
#pragma unroll
                for (int i = 0; i < 32; ++i)
                  if (32 * q4 + i >= valid) r[q4][i] = __float_as_uint(-INFINITY);
            }
            float mx[4];
#pragma unroll
            for (int q4 = 0; q4 < 4; ++q4) {
              float tt[11];
#pragma unroll
              for (int i = 0; i < 10; ++i)
                tt[i] = vl_max3(__uint_as_float(r[q4][3 * i]), __uint_as_float(r[q4][3 * i + 1]),
                                __uint_as_float(r[q4][3 * i + 2]));
              tt[10] = fmaxf(__uint_as_float(r[q4][30]), __uint_as_float(r[q4][31]));
              const float u0 = vl_max3(tt[0], tt[1], tt[2]), u1 = vl_max3(tt[3], tt[4], tt[5]);
              const float u2 = vl_max3(tt[6], tt[7], tt[8]), u3 = fmaxf(tt[9], tt[10]);
              mx[q4] = fmaxf(vl_max3(u0, u1, u2), u3);
            }
            const float m_old = m_run[hh];
            const float m_new = fmaxf(m_old, fmaxf(fmaxf(mx[0], mx[1]), fmaxf(mx[2], mx[3])) * p.c2);
            const float2 nm2 = make_float2(-m_new, -m_new);
            const float2 o[8] = {nm2, nm2, nm2, nm2, nm2, nm2, nm2, nm2};
            float2 acc0 = make_float2(0.0f, 0.0f), acc1 = make_float2(0.0f, 0.0f);
#pragma unroll
            for (int q4 = 0; q4 < 4; ++q4)
#pragma unroll
              for (int i = 0; i < 32; i += 16) vl_sum16(&r[q4][i], c2, o, acc0, acc1);
            l_run[hh] = (m_old == -INFINITY ? 0.0f : l_run[hh] * vl_ex2(m_old - m_new)) +
                        ((acc0.x + acc0.y) + (acc1.x + acc1.y));
            m_run[hh] = m_new;
          }
          if (!ok_run) break;
        }
        if (!ok_run) break;
        // this group's partial of rows lq and 128 + lq over its tiles of the chunk
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
          const int row = 128 * hh + lq;
          if (row < p.R) {
            float* dst = p.part + (((bh * p.R + row) * p.chunks + it.chunk) * 2 + g) * 2;
            dst[0] = m_run[hh];
            dst[1] = l_run[hh];
          }
        }
      } else {
        const int zero_end = min(it.key_begin + kVlChunk, p.L);
        if (it.n_tiles > 0) {
          if (it.bh != cur) {
            if (nq > 0) {
              __syncwarp();
              if (lane == 0) mbar_arrive(&sm.q_free);   // done with the previous group's -lse2
            }
            if (!cm_warp_wait(&sm.q_full, nq & 1, abort_flag, kStatusTimeoutSoftmax)) break;
            ++nq;
            cur = it.bh;
          }
          const float2* nlse2 = reinterpret_cast<const float2*>(sm.nlse);
          for (int j = ((T0 & 1) == g) ? 0 : 1; j < it.n_tiles; j += 2) {
            const int t = T0 + j;
            float2 acc0 = make_float2(0.0f, 0.0f), acc1 = make_float2(0.0f, 0.0f);
#pragma unroll
            for (int hh = 0; hh < 2; ++hh) {
              if (!cm_warp_wait(&sm.s_full[g][hh], (t >> 1) & 1, abort_flag, kStatusTimeoutSoftmax)) {
                ok_run = false;
                break;
              }
              tc_fence_after();
              uint32_t r[4][32];
#pragma unroll
              for (int q4 = 0; q4 < 4; ++q4) tmem_ld32(tl + 128u * hh + 32u * q4, r[q4]);
              tmem_wait_ld();
              tc_fence_before();
              __syncwarp();
              if (lane == 0) mbar_arrive(&sm.s_free[g][hh]);
#pragma unroll
              for (int q4 = 0; q4 < 4; ++q4)
#pragma unroll
                for (int i = 0; i < 32; i += 16)
                  vl_sum16(&r[q4][i], c2, &nlse2[(128 * hh + 32 * q4 + i) / 2], acc0, acc1);
            }
            if (!ok_run) break;
            const int key = it.key_begin + j * kCmKeys + lq;
            if (key < it.key_end) p.mass[bh * p.L + key] = (acc0.x + acc0.y) + (acc1.x + acc1.y);
          }
        }
        // positions of the chunk past the candidate prefix carry no mass
        if (g == 0)
          for (int key = max(it.key_end, it.key_begin) + lq; key < zero_end; key += 128) p.mass[bh * p.L + key] = 0.0f;
      }
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

// partials (m, l) of every chunk and softmax group -> -lse2 = -(m + log2(l)) per row
__global__ void vl_lse_kernel(const float* __restrict__ part, float* __restrict__ nlse2, int R, int chunks) {
  const int64_t bh = blockIdx.x;
  const int row = threadIdx.x;
  if (row >= R) return;
  const float* src = part + (bh * R + row) * chunks * 4;
  float m = -INFINITY, l = 0.0f;
  for (int c = 0; c < 2 * chunks; ++c) merge_ml(m, l, src[2 * c], src[2 * c + 1]);
  nlse2[bh * R + row] = l > 0.0f ? -(m + log2f(l)) : -INFINITY;
}

struct SelParams {
  const float* mass;
  const uint16_t* k;
  const uint16_t* v;
  const int32_t* n_prefix;
  int32_t* positions;
  int32_t* counts;
  unsigned long long* excl;
  uint16_t* hp_k;
  uint16_t* hp_v;
  int L, d, Hkv, max_select, max_pages;
  double rho;
};

// exclusive prefix sum of `v` over the block in thread order; *total = the block's sum
// (every thread of the block calls it; wsum holds 33 words)
FA4Q_DEVINL uint32_t block_excl_sum(uint32_t v, uint32_t* wsum, uint32_t* total) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  uint32_t incl = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t y = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += y;
  }
  if (lane == 31) wsum[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    const uint32_t w = lane < (kSelThreads / 32) ? wsum[lane] : 0u;
    uint32_t wi = w;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t y = __shfl_up_sync(0xffffffffu, wi, o);
      if (lane >= o) wi += y;
    }
    if (lane < (kSelThreads / 32)) wsum[lane] = wi - w;
    if (lane == 31) wsum[32] = wi;
  }
  __syncthreads();
  const uint32_t r = wsum[warp] + incl - v;
  *total = wsum[32];
  __syncthreads();
  return r;
}

// one CTA per (kv-head, sequence); the candidates' masses live in shared memory
__global__ void __launch_bounds__(kSelThreads, 1) vl_select_kernel(const SelParams p) {
  extern __shared__ __align__(16) uint8_t smem_raw[];
  unsigned long long* mask = reinterpret_cast<unsigned long long*>(smem_raw);   // [max_pages]
  uint32_t* bits = reinterpret_cast<uint32_t*>(mask + p.max_pages);             // [L]
  int32_t* pos = reinterpret_cast<int32_t*>(bits + p.L);                        // [max_select]
  uint32_t* hist = reinterpret_cast<uint32_t*>(pos + p.max_select);             // [256]
  uint32_t* wsum = hist + 256;                                                  // [33]
  __shared__ uint32_t s_prefix, s_remaining;
  const int h = blockIdx.x, b = blockIdx.y;
  const int64_t bh = static_cast<int64_t>(b) * p.Hkv + h;
  const int tid = threadIdx.x, lane = tid & 31;
  const int n = min(max(p.n_prefix[b], 0), p.L);
  int cnt = static_cast<int>(ceil(p.rho * static_cast<double>(n) - 1e-9));
  cnt = min(max(cnt, 0), n);

  // masses are >= 0, so their bit patterns order like the values
  for (int j = tid; j < n; j += kSelThreads) bits[j] = __float_as_uint(p.mass[bh * p.L + j]);
  for (int i = tid; i < p.max_pages; i += kSelThreads) mask[i] = 0ull;
  __syncthreads();

  // radix select of the cnt-th largest pattern T, 8 bits at a time from the top; at the end
  // `remaining` is how many of the elements equal to T belong to the top cnt.  Masses of one
  // group share few exponents, so the lanes of a warp that fall in the same bin add their
  // count with one atomic (lanes grouped by __match_any_sync).
  uint32_t prefix = 0, pmask = 0, remaining = static_cast<uint32_t>(cnt);
  if (cnt > 0) {
    for (int shift = 24; shift >= 0; shift -= 8) {
      for (int i = tid; i < 256; i += kSelThreads) hist[i] = 0;
      __syncthreads();
      for (int j0 = 0; j0 < n; j0 += kSelThreads) {       // uniform per warp
        const int j = j0 + tid;
        const uint32_t x = j < n ? bits[j] : 0u;
        const bool in = j < n && (x & pmask) == prefix;
        const uint32_t bin = in ? (x >> shift) & 255u : 256u;
        const uint32_t peers = __match_any_sync(0xffffffffu, bin);
        if (in && lane == __ffs(peers) - 1) atomicAdd(&hist[bin], static_cast<uint32_t>(__popc(peers)));
      }
      __syncthreads();
      if (tid == 0) {
        uint32_t above = 0;
        int bin = 255;
        for (; bin > 0; --bin) {
          if (above + hist[bin] >= remaining) break;
          above += hist[bin];
        }
        s_prefix = prefix | (static_cast<uint32_t>(bin) << shift);
        s_remaining = remaining - above;
      }
      __syncthreads();
      prefix = s_prefix;
      remaining = s_remaining;
      pmask |= 255u << shift;
    }
    // ordered compaction: every element above T, and the first `remaining` equal to T in
    // position order (the lowest positions win ties); positions come out ascending.  Thread
    // t takes the 32 consecutive positions base + 32 t .. (read in a lane-rotated order, so
    // the shared-memory loads of a warp hit 32 banks), as bit masks.
    uint32_t eq_before = 0, sel_before = 0;
    for (int base = 0; base < n; base += 32 * kSelThreads) {
      const int j0 = base + 32 * tid;
      uint32_t gtm = 0, eqm = 0;
#pragma unroll 8
      for (int i = 0; i < 32; ++i) {
        const int bi = (i + lane) & 31;
        const int j = j0 + bi;
        if (j < n) {
          const uint32_t x = bits[j];
          gtm |= static_cast<uint32_t>(x > prefix) << bi;
          eqm |= static_cast<uint32_t>(x == prefix) << bi;
        }
      }
      uint32_t eq_tot, sel_tot;
      const uint32_t eq_rank = eq_before + block_excl_sum(__popc(eqm), wsum, &eq_tot);
      // the lowest `take` equal elements of this thread are kept
      const uint32_t take = remaining > eq_rank ? min(remaining - eq_rank, static_cast<uint32_t>(__popc(eqm))) : 0u;
      uint32_t selm = gtm, e = eqm;
      for (uint32_t t = 0; t < take; ++t) {
        selm |= e & (0u - e);                             // lowest set bit
        e &= e - 1u;
      }
      const uint32_t sel_rank = sel_before + block_excl_sum(__popc(selm), wsum, &sel_tot);
      uint32_t k = sel_rank;
      for (uint32_t s = selm; s != 0u && k < static_cast<uint32_t>(cnt); s &= s - 1u, ++k)
        pos[k] = j0 + __ffs(s) - 1;
      if (selm != 0u && p.max_pages > 0)
        atomicOr(&mask[j0 >> 6], static_cast<unsigned long long>(selm) << (j0 & 63));
      eq_before += eq_tot;
      sel_before += sel_tot;
    }
  }
  __syncthreads();
  if (tid == 0) p.counts[bh] = cnt;
  for (int i = tid; i < cnt; i += kSelThreads) p.positions[bh * p.max_select + i] = pos[i];
  if (p.excl != nullptr)
    for (int i = tid; i < p.max_pages; i += kSelThreads) p.excl[bh * p.max_pages + i] = mask[i];
}

// The kept rows of K and V in 16-byte pieces (d / 8 per row), four pieces of each per thread
// in flight at a time; grid (piece blocks, kv-head, sequence), after vl_select_kernel.
constexpr int kGatherThreads = 256, kGatherUnroll = 4;
__global__ void __launch_bounds__(kGatherThreads) vl_gather_kernel(const SelParams p) {
  const int h = blockIdx.y, b = blockIdx.z;
  const int64_t bh = static_cast<int64_t>(b) * p.Hkv + h;
  const int shift_c = p.d == 128 ? 4 : 3;
  const int total = p.counts[bh] << shift_c;
  const int32_t* pos = p.positions + bh * p.max_select;
  for (int i0 = blockIdx.x * kGatherThreads * kGatherUnroll; i0 < total;
       i0 += gridDim.x * kGatherThreads * kGatherUnroll) {
    uint4 kk[kGatherUnroll], vv[kGatherUnroll];
#pragma unroll
    for (int u = 0; u < kGatherUnroll; ++u) {
      const int idx = i0 + u * kGatherThreads + static_cast<int>(threadIdx.x);
      if (idx < total) {
        const int r = idx >> shift_c, c = idx & ((1 << shift_c) - 1);
        const int64_t src = (bh * p.L + pos[r]) * p.d + 8 * c;
        if (p.hp_k != nullptr) kk[u] = *reinterpret_cast<const uint4*>(p.k + src);
        if (p.hp_v != nullptr) vv[u] = *reinterpret_cast<const uint4*>(p.v + src);
      }
    }
#pragma unroll
    for (int u = 0; u < kGatherUnroll; ++u) {
      const int idx = i0 + u * kGatherThreads + static_cast<int>(threadIdx.x);
      if (idx < total) {
        const int r = idx >> shift_c, c = idx & ((1 << shift_c) - 1);
        const int64_t dst = (bh * p.max_select + r) * p.d + 8 * c;
        if (p.hp_k != nullptr) *reinterpret_cast<uint4*>(p.hp_k + dst) = kk[u];
        if (p.hp_v != nullptr) *reinterpret_cast<uint4*>(p.hp_v + dst) = vv[u];
      }
    }
  }
}

namespace {

int vl_rows(int Hq, int Hkv, int n_obs) { return (Hq / Hkv) * n_obs; }
int vl_chunks(int L) { return (L + kVlChunk - 1) / kVlChunk; }
size_t vl_select_smem(int L, int max_select, int max_pages) {
  return static_cast<size_t>(max_pages) * 8 + static_cast<size_t>(L) * 4 + static_cast<size_t>(max_select) * 4 +
         (256 + 33) * 4;
}
template <int D>
size_t vl_colmass_smem() { return sizeof(CmSmem<D>) + 1024; }

template <int D>
fa4q_status vl_launch(const VlParams& vp, const SelParams& sp, const void* q_obs, const void* k, cudaStream_t st,
                      size_t sel_smem) {
  const size_t cm = vl_colmass_smem<D>();
  if (cudaFuncSetAttribute(colmass_kernel<D, 0>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)cm) != cudaSuccess ||
      cudaFuncSetAttribute(colmass_kernel<D, 1>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)cm) != cudaSuccess ||
      cudaFuncSetAttribute(vl_select_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sel_smem) != cudaSuccess)
    return FA4Q_ERR_CUDA;
  // observation rows as one [B*Hq*n_obs][2D bytes] matrix, keys as [B*Hkv][L][2D bytes]; 128-byte
  // boxes (one 64-element column chunk) of 128 rows, 128-byte swizzle; rows past either
  // tensor's end read as zeros
  CUtensorMap tq, tk;
  const uint64_t q_rows = static_cast<uint64_t>(vp.B) * vp.Hq * vp.n_obs;
  if (!make_map_3d(&tq, q_obs, 2 * D, q_rows, 1, 128, 128, CU_TENSOR_MAP_SWIZZLE_128B) ||
      !make_map_3d(&tk, k, 2 * D, vp.L, static_cast<uint64_t>(vp.B) * vp.Hkv, 128, kCmKeys, CU_TENSOR_MAP_SWIZZLE_128B))
    return FA4Q_ERR_CUDA;
  const int grid = std::min(vp.n_items, num_sms());
  colmass_kernel<D, 0><<<grid, kCmThreads, cm, st>>>(tq, tk, vp);
  vl_lse_kernel<<<vp.B * vp.Hkv, vp.R, 0, st>>>(vp.part, vp.nlse2, vp.R, vp.chunks);
  colmass_kernel<D, 1><<<grid, kCmThreads, cm, st>>>(tq, tk, vp);
  vl_select_kernel<<<dim3(vp.Hkv, vp.B), kSelThreads, sel_smem, st>>>(sp);
  if (sp.hp_k != nullptr || sp.hp_v != nullptr) {
    const int pieces = sp.max_select * (D / 8);
    const int gx = (pieces + kGatherThreads * kGatherUnroll - 1) / (kGatherThreads * kGatherUnroll);
    vl_gather_kernel<<<dim3(gx, vp.Hkv, vp.B), kGatherThreads, 0, st>>>(sp);
  }
  return launch_status();
}

}  // namespace
}  // namespace fa4q

using namespace fa4q;

extern "C" size_t fa4q_vlines_workspace_size(int B, int Hq, int Hkv, int n_obs, int L) {
  if (B <= 0 || Hq <= 0 || Hkv <= 0 || Hq % Hkv != 0 || n_obs <= 0 || L <= 0) return 0;
  const size_t rows = static_cast<size_t>(B) * Hkv * vl_rows(Hq, Hkv, n_obs);
  return rows * (4 * static_cast<size_t>(vl_chunks(L)) + 1) * sizeof(float);
}

extern "C" fa4q_status fa4q_select_vertical_lines(
    const void* q_obs, const void* k, const void* v, const int32_t* n_prefix, int B, int Hq, int Hkv,
    int n_obs, int L, int d, double rho, float sm_scale, float* mass, int32_t* positions, int32_t* counts,
    int max_select, uint64_t* excl_mask, int max_pages, void* hp_k, void* hp_v, void* workspace,
    size_t workspace_bytes, void* stream) {
  if (!q_obs || !k || !n_prefix || !mass || !positions || !counts || !workspace) return FA4Q_ERR_INVALID_ARG;
  if ((hp_v != nullptr) && v == nullptr) return FA4Q_ERR_INVALID_ARG;
  if (B <= 0 || Hq <= 0 || Hkv <= 0 || Hq % Hkv != 0 || n_obs <= 0 || L <= 0) return FA4Q_ERR_INVALID_ARG;
  if (!(rho > 0.0) || rho > 1.0 || !(sm_scale >= 0.0f) || !isfinite(sm_scale)) return FA4Q_ERR_INVALID_ARG;
  if (d != 64 && d != 128) return FA4Q_ERR_UNSUPPORTED;
  const int R = vl_rows(Hq, Hkv, n_obs);
  if (R % 32 != 0 || R > kCmRows) return FA4Q_ERR_UNSUPPORTED;
  const double need = ceil(rho * static_cast<double>(L) - 1e-9);
  if (static_cast<double>(max_select) < need || max_select <= 0) return FA4Q_ERR_INVALID_ARG;
  if (excl_mask != nullptr && static_cast<int64_t>(max_pages) * 64 < L) return FA4Q_ERR_INVALID_ARG;
  if (excl_mask == nullptr) max_pages = 0;
  if (!aligned16(q_obs) || !aligned16(k) || (v && !aligned16(v)) || (hp_k && !aligned16(hp_k)) ||
      (hp_v && !aligned16(hp_v)) || !aligned16(workspace) ||
      (reinterpret_cast<uintptr_t>(mass) & 3))
    return FA4Q_ERR_INVALID_ARG;
  if (workspace_bytes < fa4q_vlines_workspace_size(B, Hq, Hkv, n_obs, L)) return FA4Q_ERR_INVALID_ARG;
  if (B > 65535 || Hkv > 65535 || static_cast<int64_t>(B) * Hkv > 0x7fffffff) return FA4Q_ERR_UNSUPPORTED;
  const size_t sel_smem = vl_select_smem(L, max_select, max_pages);
  if (sel_smem > 227 * 1024) return FA4Q_ERR_UNSUPPORTED;   // candidates held in shared memory
  VlParams vp;
  vp.n_prefix = n_prefix;
  vp.chunks = vl_chunks(L);
  if (static_cast<int64_t>(B) * Hkv * vp.chunks > 0x7fffffff) return FA4Q_ERR_UNSUPPORTED;
  vp.n_items = B * Hkv * vp.chunks;
  vp.part = static_cast<float*>(workspace);
  vp.nlse2 = vp.part + static_cast<size_t>(B) * Hkv * R * vp.chunks * 4;
  vp.mass = mass;
  vp.B = B; vp.Hq = Hq; vp.Hkv = Hkv; vp.n_obs = n_obs; vp.L = L; vp.d = d; vp.R = R;
  const float sm = sm_scale > 0.0f ? sm_scale : 1.0f / sqrtf(static_cast<float>(d));
  vp.c2 = sm * kVlLog2e;
  SelParams sp;
  sp.mass = mass;
  sp.k = static_cast<const uint16_t*>(k);
  sp.v = static_cast<const uint16_t*>(v);
  sp.n_prefix = n_prefix;
  sp.positions = positions;
  sp.counts = counts;
  sp.excl = reinterpret_cast<unsigned long long*>(excl_mask);
  sp.hp_k = static_cast<uint16_t*>(hp_k);
  sp.hp_v = static_cast<uint16_t*>(hp_v);
  sp.L = L; sp.d = d; sp.Hkv = Hkv; sp.max_select = max_select; sp.max_pages = max_pages;
  sp.rho = rho;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  return d == 128 ? vl_launch<128>(vp, sp, q_obs, k, st, sel_smem) : vl_launch<64>(vp, sp, q_obs, k, st, sel_smem);
}
