// decode_tc.cu - decode on the FP4 tensor cores with a dual-residual query (sm_100a).
//
// What it computes, per (sequence b, q-head h) over an all-FP4 paged cache:
//   out = softmax(s) v_hat with s = (deq(q1) + deq(q2)) . k_hat * sm_scale, where
//   q1 = NVFP4(q) and q2 = NVFP4(q - deq(q1)); the probabilities are quantised to NVFP4
//   before the PV product, against the running maximum of 128-key tiles (pre-normalisation
//   quantisation, g_P = 1/(6*448)), and the normaliser is the sum of that same P_hat.
// Sources: BitDecoding-FP4 (Algorithm-System Co-Design for Native FP4 KV Cache Decoding),
// "Error Sources" (the query as the sum of two FP4 tensors, the second quantising the
// residual of the first) and "System-Level Optimization" (the softmax transposed so that P
// is quantised inside its reduction; query MMAs stacked over the paged cache).
//
// Design (swap-AB on tcgen05).  One decode step has G = Hq/Hkv query rows per kv-head, far
// below the 128-row MMA tile, so the keys and channels take the M side and the query heads
// the N side (N = 16):
//   S^T[128 keys x (16 + 16)]     = K_hat[128 x d] [Q_hat1 ; Q_hat2]^T      2 MMAs
//   O^T[128 channels x 16 heads] += V_hat^T[128 x 128 keys] P_hat^T           2 MMAs
// (the four S^T partials, residual x half of d, are added by the softmax, the two O^T
// accumulators in the epilogue).
// A softmax thread owns one key of the tile (its TMEM lane): the 16-key P blocks are 16
// lanes (block maxima by shuffles), the tile maximum goes through shared memory, and P_hat^T
// is packed by shuffles into the K-major [heads][keys] operand.  The normaliser is summed
// from the dequantised P_hat in registers.  Warp 0 streams page pairs through the block
// table by TMA (5 stages of 18 KB), warp 1 issues the MMAs, warps 2 and 3 permute the raw
// page scales into the MMA's scale atoms.  Two softmax groups (warps 4-7, 8-11) take the even
// and the odd tiles, so one tile's softmax overlaps the next; only the running maximum
// passes from group to group, each keeps its own O^T accumulators and normaliser, and the
// epilogue merges the two.  Two CTAs share an SM.
#include <math.h>

#include "fa4q_common.cuh"
#include "fa4q_internal.h"

namespace fa4q {

static __device__ uint32_t g_dectc_status;

constexpr int kTcD = 128;                 // head dimension
constexpr int kTcN = 16;                  // query heads per MMA (the N side)
constexpr int kTcStages = 5;
constexpr int kTcThreads = 384;
constexpr int kTcDefaultTilesPerSplit = 32;   // 4096 keys per range when the caller passes 0
constexpr float kTcLog2e = 1.4426950408889634f;
constexpr float kTcGp = 1.0f / 2688.0f;   // g_P = 1/(6*448), rounded to FP32
constexpr float kTcInvSixGp = 1.0f / (6.0f * kTcGp);

// TMEM columns (256 allocated).  S^T per tile parity: two products (one per half of d) of
// 32 columns, the first 16 against Q1 and the next 16 against Q2 (the two residual tiles are
// one N = 32 operand); O^T per softmax group two accumulators (one per page of the pair).
constexpr uint32_t kTcColS = 0, kTcColO = 128, kTcColSfQ = 192, kTcColSfK = 200, kTcColSfV = 216, kTcColSfP = 232;
constexpr uint32_t kTcTmemCols = 256;

struct TcParams {
  const uint8_t* q_sf;      // [B*Hkv][2][2][512] query scale atoms
  const uint8_t* k_sf;      // [P*Hkv][64 tokens][8] raw page scales
  const uint8_t* v_sf;      // [P*Hkv][128 channels][4]
  const int32_t* table;     // [B][max_pages]
  const int32_t* len;       // [B]
  float* ws;                // [B*Hq][splits][d + 2] split partials
  int B, Hq, Hkv, G, max_pages, n_phys, splits, tiles_per_split;
  float sc;                 // sm_scale * g_k * log2(e)
  float g_v;
};

struct __align__(1024) TcSmem {
  uint8_t k[kTcStages][8192];   // two 64-token K pages: [128 keys][64 B], 64B swizzle
  uint8_t v[kTcStages][8192];   // two V^T pages, each [128 channels][32 B], 32B swizzle
  uint8_t sf[kTcStages][2048];  // page scales: raw as loaded, then in place as scale atoms
                                // (K atoms per half of d at 0 / 512, V^T atoms per page at 1024 / 1536)
  uint8_t q[2][1024];           // residual query tiles [16 rows][64 B], 64B swizzle
  uint8_t sfq[2][1024];         // their scale atoms (one per half of d)
  uint8_t sfqc[2][512];         // per half of d: Q1's scales in rows 0-15, Q2's in rows 16-31
  uint8_t p[2][1024];           // P_hat^T [16 heads][64 B], 64B swizzle, by tile parity
  uint8_t sfp[2][1024];         // its scale atoms (one per page of keys)
  uint64_t bar_q;
  uint64_t kv_full[kTcStages];
  uint64_t kv_empty[kTcStages];
  uint64_t sf_ready[kTcStages];
  uint64_t s_full[2];
  uint64_t s_free[2];
  uint64_t p_full[2];
  uint64_t o_done[2];
  uint64_t drain;
  float qx[2][2][4][kTcN];      // per group, slot (tile / 2) % 2: each lane quadrant's maximum per head
  float mx[2][kTcN];            // running maximum after tile j, slot j % 2
  float mlast[2][kTcN];         // per group: the maximum its accumulators are relative to
  float red[2][4][kTcN];        // per group: normaliser partial sums per lane quadrant
  uint32_t tmem_base;
  uint32_t abort_flag;
};

// Bounded waits (the same scheme as the prefill kernel): a role that gives up raises the
// CTA's abort flag, after which every other wait returns at once.
FA4Q_DEVINL bool tc_cta_wait(uint64_t* bar, uint32_t parity, volatile uint32_t* abort_flag, uint32_t code) {
  if (*abort_flag) return false;
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = globaltimer_ns();
  while (true) {
    if (mbar_try_wait(bar, parity)) return true;
    if (*abort_flag) return false;
    if (globaltimer_ns() - t0 > kWaitNs) break;
  }
  atomicOr(&g_dectc_status, code);
  *abort_flag = 1;
  return false;
}

FA4Q_DEVINL bool tc_warp_wait(uint64_t* bar, uint32_t parity, volatile uint32_t* abort_flag, uint32_t code) {
  return __all_sync(0xffffffffu, tc_cta_wait(bar, parity, abort_flag, code));
}

FA4Q_DEVINL float tc_ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

FA4Q_DEVINL float tc_lg2(float x) {
  float y;
  asm("lg2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

FA4Q_DEVINL void tc_bar_sync(int id, int count) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(count) : "memory");
}

// value of a non-negative E2M1 code (0, 0.5, 1, 1.5, 2, 3, 4, 6)
FA4Q_DEVINL float e2m1_magnitude(uint32_t c) {
  c &= 7u;
  return c < 2u ? 0.5f * static_cast<float>(c) : __uint_as_float((((c >> 1) + 126u) << 23) | ((c & 1u) << 22));
}

// N consecutive 32-bit TMEM columns of this warp's lane quadrant (N = 2, 4, 8, 16)
template <int N>
FA4Q_DEVINL void tmem_ldn(uint32_t taddr, uint32_t (&r)[N]) {
  if constexpr (N == 2) {
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x2.b32 {%0,%1}, [%2];" : "=r"(r[0]), "=r"(r[1]) : "r"(taddr));
  } else if constexpr (N == 4) {
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x4.b32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                 : "r"(taddr));
  } else if constexpr (N == 16) {
    tmem_ld16(taddr, r);
  } else {
    static_assert(N == 8, "2, 4, 8 or 16 columns");
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
                   "=r"(r[7])
                 : "r"(taddr));
  }
}

template <int N>
FA4Q_DEVINL void tmem_stn(uint32_t taddr, const uint32_t (&r)[N]) {
  if constexpr (N == 2) {
    asm volatile("tcgen05.st.sync.aligned.32x32b.x2.b32 [%0], {%1,%2};" ::"r"(taddr), "r"(r[0]), "r"(r[1])
                 : "memory");
  } else if constexpr (N == 4) {
    asm volatile("tcgen05.st.sync.aligned.32x32b.x4.b32 [%0], {%1,%2,%3,%4};" ::"r"(taddr), "r"(r[0]),
                 "r"(r[1]), "r"(r[2]), "r"(r[3])
                 : "memory");
  } else if constexpr (N == 16) {
    tmem_st16(taddr, r);
  } else {
    static_assert(N == 8, "2, 4, 8 or 16 columns");
    asm volatile("tcgen05.st.sync.aligned.32x32b.x8.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8};" ::"r"(taddr),
                 "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7])
                 : "memory");
  }
}

// byte offset of (row r, 16-byte chunk c) in a K-major tile with 64-byte rows, 64B swizzle
FA4Q_DEVINL uint32_t tc_swz64(uint32_t r, uint32_t c) {
  return (r >> 3) * 512 + (r & 7) * 64 + ((c ^ ((r >> 1) & 3)) << 4);
}

// NH: query heads handled per kv-head (G <= NH <= 16, NH = 4, 8 or 16; rows G..15 of the
// query tile are zero)
template <int NH>
__global__ void __launch_bounds__(kTcThreads, 2)
    decode_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                     const __grid_constant__ CUtensorMap tm_v, const TcParams p) {
  extern __shared__ uint8_t smem_raw[];
  TcSmem& sm = *reinterpret_cast<TcSmem*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                           ~static_cast<uintptr_t>(1023));
  volatile uint32_t* abort_flag = &sm.abort_flag;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  // work item: (sequence, kv-head, split)
  const int grp = blockIdx.x / p.splits, split = blockIdx.x - grp * p.splits;
  const int b = grp / p.Hkv, hk = grp - b * p.Hkv;
  const int L = max(0, min(p.len[b], p.max_pages * 64));
  const int n_all = (L + 127) / 128;
  const int n_tiles = max(0, min(p.tiles_per_split, n_all - split * p.tiles_per_split));
  const int key0 = split * p.tiles_per_split * 128;

  // ---------------------------------------------------------------- setup
  if (threadIdx.x == 0) {
    mbar_init(&sm.bar_q, 1);
    for (int s = 0; s < kTcStages; ++s) {
      mbar_init(&sm.kv_full[s], 1);
      mbar_init(&sm.kv_empty[s], 1);
      mbar_init(&sm.sf_ready[s], 2);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(&sm.s_full[s], 1);
      mbar_init(&sm.s_free[s], 4);
      mbar_init(&sm.p_full[s], 4);
      mbar_init(&sm.o_done[s], 1);
    }
    mbar_init(&sm.drain, 1);
    sm.abort_flag = 0;
    fence_barrier_init();
  }
  if (warp >= 4) {
    // P_hat^T rows of heads >= NH and their scales are never written: clear both buffers
    uint4* z = reinterpret_cast<uint4*>(sm.p[0]);
    for (int i = threadIdx.x - 128; i < 4 * 1024 / 16; i += 256) z[i] = make_uint4(0u, 0u, 0u, 0u);
    fence_proxy_async_smem();
  }
  if (warp == 1) {
    tmem_alloc(&sm.tmem_base, kTcTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sm.tmem_base;

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    // The whole warp reads the block table in windows of 32 logical pages (16 tiles), one
    // window ahead of the copies, so no lookup latency sits on the path of a copy; lane 0
    // issues the copies.
    if (n_tiles > 0) {
      if (lane == 0) {
        prefetch_tmap(&tm_q);
        prefetch_tmap(&tm_k);
        prefetch_tmap(&tm_v);
        mbar_arrive_expect_tx(&sm.bar_q, 2 * (1024 + 1024));
        for (int r = 0; r < 2; ++r) {
          tma_load_3d(sm.q[r], &tm_q, 0, 0, grp * 2 + r, &sm.bar_q);
          bulk_load(sm.sfq[r], p.q_sf + ((int64_t)grp * 2 + r) * 1024, 1024, &sm.bar_q);
        }
      }
      const int n_pages = (L + 63) / 64, lp_base = 2 * split * p.tiles_per_split;
      const int64_t n_rows = (int64_t)p.n_phys * p.Hkv;
      const int32_t* trow = p.table + (int64_t)b * p.max_pages;
      // physical (page, kv-head) row of logical page lp (the last page repeats past the end;
      // ids are clamped to the cache so no copy leaves it)
      auto page_row = [&](int lp) -> int {
        const int64_t r = (int64_t)trow[min(lp, n_pages - 1)] * p.Hkv + hk;
        return static_cast<int>(min(max(r, (int64_t)0), n_rows - 1));
      };
      int win = page_row(lp_base + lane);
      int win_next = page_row(lp_base + 32 + lane);
      int T = 0;
      for (int j = 0; j < n_tiles; ++j) {
        if (j > 0 && (j & 15) == 0) {
          win = win_next;
          win_next = page_row(lp_base + 32 * ((j >> 4) + 1) + lane);
        }
        const int ph0 = __shfl_sync(0xffffffffu, win, 2 * (j & 15));
        const int ph1 = __shfl_sync(0xffffffffu, win, 2 * (j & 15) + 1);
        const int s = j % kTcStages;
        if (j >= kTcStages &&
            !tc_warp_wait(&sm.kv_empty[s], ((j / kTcStages) - 1) & 1, abort_flag, kStatusTimeoutTmaFull))
          break;
        if (lane == 0) {
          mbar_arrive_expect_tx(&sm.kv_full[s], 8192 + 8192 + 2048);
          tma_load_3d(sm.k[s], &tm_k, 0, 0, ph0, &sm.kv_full[s]);
          tma_load_3d(sm.k[s] + 4096, &tm_k, 0, 0, ph1, &sm.kv_full[s]);
          tma_load_3d(sm.v[s], &tm_v, 0, 0, ph0, &sm.kv_full[s]);
          tma_load_3d(sm.v[s] + 4096, &tm_v, 0, 0, ph1, &sm.kv_full[s]);
          bulk_load(sm.sf[s], p.k_sf + (int64_t)ph0 * 512, 512, &sm.kv_full[s]);
          bulk_load(sm.sf[s] + 512, p.k_sf + (int64_t)ph1 * 512, 512, &sm.kv_full[s]);
          bulk_load(sm.sf[s] + 1024, p.v_sf + (int64_t)ph0 * 512, 512, &sm.kv_full[s]);
          bulk_load(sm.sf[s] + 1536, p.v_sf + (int64_t)ph1 * 512, 512, &sm.kv_full[s]);
        }
        __syncwarp();
        ++T;
      }
      // drain: every issued copy must have landed before the CTA may exit
      if (lane == 0) {
        for (int t = max(0, T - kTcStages); t < T; ++t)
          mbar_wait(&sm.kv_full[t % kTcStages], (t / kTcStages) & 1, &g_dectc_status, kStatusTimeoutDrain);
        mbar_wait(&sm.bar_q, 0, &g_dectc_status, kStatusTimeoutDrain);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    bool ok = n_tiles > 0 && tc_warp_wait(&sm.bar_q, 0, abort_flag, kStatusTimeoutMma);
    if (ok) {
      // scale atoms of the N = 32 query operand: row r < 16 from Q1's atom, r >= 16 from Q2's
      // (byte (r % 32) * 16 + k of an atom; rows >= 32 are not read)
      for (int st = 0; st < 2; ++st) {
        uint32_t* dst = reinterpret_cast<uint32_t*>(sm.sfqc[st]);
        const uint32_t* src = reinterpret_cast<const uint32_t*>(sm.sfq[lane >> 4] + 512 * st);
        dst[lane * 4] = src[(lane & 15) * 4];
        dst[lane * 4 + 1] = 0u;
        dst[lane * 4 + 2] = 0u;
        dst[lane * 4 + 3] = 0u;
      }
      fence_proxy_async_smem();
      __syncwarp();
    }
    if (ok && elect_one()) {
      const uint32_t idesc = make_idesc_fp4(kTcN, false, 0, 0);
      const uint32_t idesc_s = make_idesc_fp4(2 * kTcN, false, 0, 0);
      tc_fence_after();
      for (int st = 0; st < 2; ++st) tmem_cp_sf_atom(tmem + kTcColSfQ + 4 * st, smem_u32(sm.sfqc[st]));
      // S^T_j = K_j [Q1 ; Q2]^T as two products (halves of d) into S buffer j % 2
      auto issue_s = [&](int j) -> bool {
        const int s = j % kTcStages, sb = j & 1;
        const uint32_t ph = (j / kTcStages) & 1;
        if (!tc_cta_wait(&sm.kv_full[s], ph, abort_flag, kStatusTimeoutMma)) return false;
        if (!tc_cta_wait(&sm.sf_ready[s], ph, abort_flag, kStatusTimeoutMma)) return false;
        if (j >= 2 && !tc_cta_wait(&sm.s_free[sb], ((j >> 1) - 1) & 1, abort_flag, kStatusTimeoutMma))
          return false;
        tc_fence_after();
        for (int st = 0; st < 2; ++st)
          tmem_cp_sf_atom(tmem + kTcColSfK + 8 * sb + 4 * st, smem_u32(sm.sf[s] + 512 * st));
        const uint32_t k_addr = smem_u32(sm.k[s]), q_addr = smem_u32(sm.q[0]);
        for (int st = 0; st < 2; ++st) {
          const uint64_t ad = make_smem_desc(k_addr + 32 * st, 16, 512, kSwiz64);
          const uint64_t bd = make_smem_desc(q_addr + 32 * st, 16, 512, kSwiz64);
          mma_nvf4(tmem + kTcColS + 64 * sb + 32 * st, ad, bd, idesc_s, tmem + kTcColSfK + 8 * sb + 4 * st,
                   tmem + kTcColSfQ + 4 * st, 0u);
        }
        tc_commit(&sm.s_full[sb]);
        return true;
      };
      // O^T_{j%2} += V_j^T P_j^T once the softmax group of tile j has written P_j (one K-step
      // per page, page ks into accumulator ks of the group)
      auto issue_pv = [&](int j) -> bool {
        const int s = j % kTcStages, pb = j & 1;
        if (!tc_cta_wait(&sm.p_full[pb], (j >> 1) & 1, abort_flag, kStatusTimeoutMma)) return false;
        tc_fence_after();
        for (int ks = 0; ks < 2; ++ks) {
          tmem_cp_sf_atom(tmem + kTcColSfV + 8 * pb + 4 * ks, smem_u32(sm.sf[s] + 1024 + 512 * ks));
          tmem_cp_sf_atom(tmem + kTcColSfP + 8 * pb + 4 * ks, smem_u32(sm.sfp[pb] + 512 * ks));
        }
        const uint32_t v_addr = smem_u32(sm.v[s]), p_addr = smem_u32(sm.p[pb]);
        for (int ks = 0; ks < 2; ++ks) {
          const uint64_t ad = make_smem_desc(v_addr + 4096 * ks, 16, 256, kSwiz32);
          const uint64_t bd = make_smem_desc(p_addr + 32 * ks, 16, 512, kSwiz64);
          mma_nvf4(tmem + kTcColO + 32 * pb + 16 * ks, ad, bd, idesc, tmem + kTcColSfV + 8 * pb + 4 * ks,
                   tmem + kTcColSfP + 8 * pb + 4 * ks, j >= 2 ? 1u : 0u);
        }
        tc_commit(&sm.o_done[pb]);
        tc_commit(&sm.kv_empty[s]);
        return true;
      };
      // S runs two tiles ahead of PV: S_{j+2} goes out as soon as the group of tile j has
      // loaded S_j (its buffer is then free), ahead of PV_j, which waits for that group's P_j;
      // the group's next tile then never waits for its own previous PV to be issued
      ok = ok && issue_s(0);
      if (ok && n_tiles > 1) ok = issue_s(1);
      for (int j = 0; ok && j < n_tiles; ++j) {
        if (j + 2 < n_tiles) ok = issue_s(j + 2);
        if (ok) ok = issue_pv(j);
      }
      tc_commit(&sm.drain);
      mbar_wait(&sm.drain, 0, &g_dectc_status, kStatusTimeoutDrain);
    }
  } else if (warp < 4) {
    // ------------------------------------------------------------ scale atoms
    // In place, per stage: warp 2 turns the raw K scales (page, token, 8 blocks along d) into
    // two atoms (one per half of d; row = key of the pair), warp 3 the raw V^T scales (page,
    // channel, 4 blocks of 16 keys) into one atom per page (row = channel).  Atom layout:
    // byte (row % 32) * 16 + (row / 32) * 4 + block.
    const bool kside = warp == 2;
    for (int j = 0; j < n_tiles; ++j) {
      const int s = j % kTcStages;
      if (!tc_warp_wait(&sm.kv_full[s], (j / kTcStages) & 1, abort_flag, kStatusTimeoutMma)) break;
      uint32_t* w32 = reinterpret_cast<uint32_t*>(sm.sf[s] + (kside ? 0 : 1024));
      uint32_t w[8];
#pragma unroll
      for (int n = 0; n < 8; ++n) w[n] = w32[lane + 32 * n];
      __syncwarp();
#pragma unroll
      for (int n = 0; n < 8; ++n) {
        const int i = lane + 32 * n;
        int off;
        if (kside) {        // word i = page * 128 + token * 2 + half
          const int row = ((i >> 7) << 6) + ((i >> 1) & 63);
          off = 512 * (i & 1) + (row & 31) * 16 + (row >> 5) * 4;
        } else {            // word i = page * 128 + channel
          const int ch = i & 127;
          off = 512 * (i >> 7) + (ch & 31) * 16 + (ch >> 5) * 4;
        }
        *reinterpret_cast<uint32_t*>(reinterpret_cast<uint8_t*>(w32) + off) = w[n];
      }
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(&sm.sf_ready[s]);
    }
  } else {
    // ------------------------------------------------------------ softmax / PNQ / epilogue
    // Thread = key kr of the tile (TMEM lane kr of S^T) and, in the epilogue, channel kr of
    // O^T.  Group g = 0 (warps 4-7) takes the even tiles, g = 1 (warps 8-11) the odd ones;
    // the group finishing tile j publishes the running maximum m_j in shared memory and
    // arrives on a named barrier the other group synchronises on before tile j + 1.  The
    // loops never leave early (after an abort every wait returns at once), so the barrier
    // arrivals and synchronisations always pair.
    const int g = (warp - 4) >> 2, wq = warp & 3;
    const int kr = wq * 32 + lane;
    const uint32_t lane_base = tmem + (static_cast<uint32_t>(wq * 32) << 16);
    const int bar_grp = 1 + g, bar_send = 3 + g, bar_recv = 3 + (g ^ 1), bar_epi = 5;
    const float sc = p.sc;
    const int G = p.G;
    float macc[NH], l[NH];                         // this group's maximum (raw score units), normaliser part
#pragma unroll
    for (int h = 0; h < NH; ++h) {
      macc[h] = -INFINITY;
      l[h] = 0.0f;
    }
    bool ok = true;
    for (int j = g; j < n_tiles; j += 2) {
      const int sb = j & 1;                        // = g: S buffer, P buffer, O accumulators
      ok = tc_warp_wait(&sm.s_full[sb], (j >> 1) & 1, abort_flag, kStatusTimeoutSoftmax) && ok;
      tc_fence_after();
      uint32_t raw[4][NH];
#pragma unroll
      for (int part = 0; part < 4; ++part) tmem_ldn<NH>(lane_base + kTcColS + 64 * sb + 16 * part, raw[part]);
      tmem_wait_ld();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&sm.s_free[sb]);
      const bool valid = key0 + j * 128 + kr < L;
      float* qx = sm.qx[g][(j >> 1) & 1][0];
      float s[NH], bm[NH];
#pragma unroll
      for (int h = 0; h < NH; ++h) {
        const float sum = (__uint_as_float(raw[0][h]) + __uint_as_float(raw[1][h])) +
                          (__uint_as_float(raw[2][h]) + __uint_as_float(raw[3][h]));
        s[h] = valid ? sum : -INFINITY;
        float x = s[h];                            // maximum of the 16-key block (16 lanes)
        x = fmaxf(x, __shfl_xor_sync(0xffffffffu, x, 1));
        x = fmaxf(x, __shfl_xor_sync(0xffffffffu, x, 2));
        x = fmaxf(x, __shfl_xor_sync(0xffffffffu, x, 4));
        x = fmaxf(x, __shfl_xor_sync(0xffffffffu, x, 8));
        bm[h] = x;
        const float wm = fmaxf(x, __shfl_xor_sync(0xffffffffu, x, 16));
        if (lane == h) qx[wq * kTcN + h] = wm;
      }
      // tile maximum over the four lane quadrants (slot (j / 2) % 2 of this group: a warp
      // rewrites it two tiles of the group later, after all four passed the barrier between)
      tc_bar_sync(bar_grp, 128);
      // running maximum: take m_{j-1} from the other group, publish m_j
      float mprev[NH];
#pragma unroll
      for (int h = 0; h < NH; ++h) mprev[h] = -INFINITY;
      if (j > 0) {
        tc_bar_sync(bar_recv, 256);
#pragma unroll
        for (int h = 0; h < NH; ++h) mprev[h] = sm.mx[(j - 1) & 1][h];
      }
      float mn[NH], al[NH];
      bool grow = false;
#pragma unroll
      for (int h = 0; h < NH; ++h) {
        const float t = fmaxf(fmaxf(qx[h], qx[kTcN + h]), fmaxf(qx[2 * kTcN + h], qx[3 * kTcN + h]));
        mn[h] = fmaxf(mprev[h], t);
        al[h] = tc_ex2((macc[h] - mn[h]) * sc);    // 0 before the group's first tile
        grow = grow || al[h] != 1.0f;
      }
      if (wq == 0 && lane < NH) {
#pragma unroll
        for (int h = 0; h < NH; ++h)
          if (lane == h) sm.mx[j & 1][h] = mn[h];
      }
      asm volatile("bar.arrive %0, %1;" ::"r"(bar_send), "r"(256) : "memory");
      // P_hat: per block of 16 keys, scale = UE4M3(amax / (6 g_P)) with amax = exp2((bmax - m) c);
      // y = exp2(s c - m c - log2(scale g_P)) rounded to E2M1
      uint32_t scode[NH];
      float sfv[NH];
      uint32_t codes[(NH + 7) / 8];
#pragma unroll
      for (int w8 = 0; w8 < (NH + 7) / 8; ++w8) {
        float y[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int i = 0; i < 8 && 8 * w8 + i < NH; ++i) {
          const int h = 8 * w8 + i;
          const float amax = tc_ex2((bm[h] - mn[h]) * sc);
          scode[h] = ue4m3_encode(amax * kTcInvSixGp);
          sfv[h] = ue4m3_decode(scode[h]);
          const float lsc = sfv[h] > 0.0f ? tc_lg2(sfv[h] * kTcGp) : INFINITY;
          y[i] = tc_ex2(fmaf(s[h], sc, -(mn[h] * sc + lsc)));
        }
        codes[w8] = e2m1x8(y[0], y[1], y[2], y[3], y[4], y[5], y[6], y[7]);
      }
      // P buffer and accumulators of this group were last used by its PV product of tile j - 2
      if (j >= 2) ok = tc_warp_wait(&sm.o_done[sb], ((j >> 1) - 1) & 1, abort_flag, kStatusTimeoutSoftmax) && ok;
#pragma unroll
      for (int h = 0; h < NH; ++h) {
        const uint32_t c = (codes[h >> 3] >> (4 * (h & 7))) & 0xFu;
        l[h] = fmaf(l[h], al[h], e2m1_magnitude(c) * sfv[h]);
        // eight keys' codes of head h into one word (key kr at nibble kr % 8)
        uint32_t wd = c << (4 * (lane & 7));
        wd |= __shfl_xor_sync(0xffffffffu, wd, 1);
        wd |= __shfl_xor_sync(0xffffffffu, wd, 2);
        wd |= __shfl_xor_sync(0xffffffffu, wd, 4);
        if ((lane & 7) == 0) *reinterpret_cast<uint32_t*>(sm.p[sb] + tc_swz64(h, wq) + 4 * (lane >> 3)) = wd;
        // scale of the 16-key block: atom of page wq/2, block 2 (wq % 2) + lane / 16
        if ((lane & 15) == 0) sm.sfp[sb][512 * (wq >> 1) + h * 16 + 2 * (wq & 1) + (lane >> 4)] = static_cast<uint8_t>(scode[h]);
      }
      fence_proxy_async_smem();
      if (grow && j >= 2) {
        // bring the group's O^T accumulators (its tiles < j) from its previous maximum to m_j
        tc_fence_after();
        uint32_t o[2][NH];
        tmem_ldn<NH>(lane_base + kTcColO + 32 * sb, o[0]);
        tmem_ldn<NH>(lane_base + kTcColO + 32 * sb + 16, o[1]);
        tmem_wait_ld();
#pragma unroll
        for (int h = 0; h < NH; ++h) {
          o[0][h] = __float_as_uint(__uint_as_float(o[0][h]) * al[h]);
          o[1][h] = __float_as_uint(__uint_as_float(o[1][h]) * al[h]);
        }
        tmem_stn<NH>(lane_base + kTcColO + 32 * sb, o[0]);
        tmem_stn<NH>(lane_base + kTcColO + 32 * sb + 16, o[1]);
        tmem_wait_st();
      }
#pragma unroll
      for (int h = 0; h < NH; ++h) macc[h] = mn[h];
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&sm.p_full[sb]);
    }
    // the group that did not process the last tile consumes its maximum
    if (n_tiles > 0 && ((n_tiles - 1) & 1) != g) tc_bar_sync(bar_recv, 256);
    // ---------------------------------------------------------------- epilogue
    // out partial of q-head h for this split: m in log2 units, l and o in true units (the MMA
    // operands carry neither g_P nor g_v); O = O_A 2^((mA - m) c) + O_B 2^((mB - m) c)
    const int stride = kTcD + 2;
    if (n_tiles == 0) {
      for (int h = g; h < G && h < NH; h += 2) {
        float* dst = p.ws + (((int64_t)b * p.Hq + hk * G + h) * p.splits + split) * stride;
        dst[2 + kr] = 0.0f;
        if (kr == 0) {
          dst[0] = -INFINITY;
          dst[1] = 0.0f;
        }
      }
    } else {
#pragma unroll
      for (int h = 0; h < NH; ++h) {
        float x = l[h];
        x += __shfl_xor_sync(0xffffffffu, x, 16);
        x += __shfl_xor_sync(0xffffffffu, x, 8);
        x += __shfl_xor_sync(0xffffffffu, x, 4);
        x += __shfl_xor_sync(0xffffffffu, x, 2);
        x += __shfl_xor_sync(0xffffffffu, x, 1);
        if (lane == h) {
          sm.red[g][wq][h] = x;
          if (wq == 0) sm.mlast[g][h] = macc[h];
        }
      }
      tc_bar_sync(bar_epi, 256);
      // the last PV product of each group
      const int cnt_a = (n_tiles + 1) / 2, cnt_b = n_tiles / 2;
      ok = tc_warp_wait(&sm.o_done[0], (cnt_a - 1) & 1, abort_flag, kStatusTimeoutSoftmax) && ok;
      if (cnt_b > 0) ok = tc_warp_wait(&sm.o_done[1], (cnt_b - 1) & 1, abort_flag, kStatusTimeoutSoftmax) && ok;
      if (ok) {
        tc_fence_after();
        uint32_t oa[2][NH], ob[2][NH];
        tmem_ldn<NH>(lane_base + kTcColO, oa[0]);
        tmem_ldn<NH>(lane_base + kTcColO + 16, oa[1]);
        tmem_ldn<NH>(lane_base + kTcColO + 32, ob[0]);
        tmem_ldn<NH>(lane_base + kTcColO + 48, ob[1]);
        tmem_wait_ld();
        const float so = kTcGp * p.g_v;
#pragma unroll
        for (int h = 0; h < NH; ++h) {
          if ((h & 1) == g && h < G) {
            const float mA = sm.mlast[0][h], mB = sm.mlast[1][h];
            const float m = fmaxf(mA, mB);
            const float wa = tc_ex2((mA - m) * sc), wb = cnt_b > 0 ? tc_ex2((mB - m) * sc) : 0.0f;
            const float la = (sm.red[0][0][h] + sm.red[0][1][h]) + (sm.red[0][2][h] + sm.red[0][3][h]);
            const float lb = (sm.red[1][0][h] + sm.red[1][1][h]) + (sm.red[1][2][h] + sm.red[1][3][h]);
            const float o = (__uint_as_float(oa[0][h]) + __uint_as_float(oa[1][h])) * wa +
                            (cnt_b > 0 ? (__uint_as_float(ob[0][h]) + __uint_as_float(ob[1][h])) * wb : 0.0f);
            float* dst = p.ws + (((int64_t)b * p.Hq + hk * G + h) * p.splits + split) * stride;
            dst[2 + kr] = o * so;
            if (kr == 0) {
              dst[0] = m * sc;
              dst[1] = (la * wa + (cnt_b > 0 ? lb * wb : 0.0f)) * kTcGp;
            }
          }
        }
      }
    }
  }
  // ---------------------------------------------------------------- teardown
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, kTcTmemCols);
  }
}

struct TcPlan {
  int splits, tiles_per_split;
  size_t off_qt, off_qsf, total;
};

// The scan of each sequence restarts its running state every T tiles (T = tiles_per_split,
// 0 -> kTcDefaultTilesPerSplit): T is part of the result, so it never depends on the batch,
// the head count or the GPU.  The split count follows from the longest sequence the block
// table can map: ceil(ceil(max_pages / 2) / T).
static TcPlan tc_plan(int B, int Hq, int Hkv, int max_pages, int tiles_per_split) {
  TcPlan pl;
  const int tiles = std::max(1, (max_pages + 1) / 2);
  pl.tiles_per_split = tiles_per_split > 0 ? tiles_per_split : kTcDefaultTilesPerSplit;
  pl.splits = (tiles + pl.tiles_per_split - 1) / pl.tiles_per_split;
  const size_t part = (size_t)B * Hq * pl.splits * (kTcD + 2) * sizeof(float);
  pl.off_qt = (part + 1023) / 1024 * 1024;
  pl.off_qsf = pl.off_qt + (size_t)B * Hkv * 2 * 128 * (kTcD / 2);
  pl.total = pl.off_qsf + (size_t)B * Hkv * 2 * 2 * 512;
  return pl;
}

cudaError_t dectc_status_fetch(cudaStream_t st, uint32_t* host_word) {
  cudaError_t e = cudaMemcpyFromSymbolAsync(host_word, g_dectc_status, sizeof(uint32_t), 0,
                                            cudaMemcpyDeviceToHost, st);
  if (e != cudaSuccess) return e;
  const uint32_t zero = 0;
  e = cudaMemcpyToSymbolAsync(g_dectc_status, &zero, sizeof(uint32_t), 0, cudaMemcpyHostToDevice, st);
  if (e != cudaSuccess) return e;
  return cudaStreamSynchronize(st);
}

template <int NH>
static fa4q_status launch_tc(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                             const TcParams& prm, int grid, cudaStream_t st) {
  auto kern = decode_tc_kernel<NH>;
  const size_t smem = sizeof(TcSmem) + 1024;
  static_assert(2 * (sizeof(TcSmem) + 1024 + 1024) <= 228 * 1024, "two CTAs per SM");
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) != cudaSuccess)
    return FA4Q_ERR_CUDA;
  kern<<<grid, kTcThreads, smem, st>>>(tq, tk, tv, prm);
  return launch_status();
}

}  // namespace fa4q

using namespace fa4q;

extern "C" size_t fa4q_decode_fp4q_workspace_size(int B, int Hq, int Hkv, int d, int max_pages,
                                                  int tiles_per_split) {
  if (B <= 0 || Hq <= 0 || Hkv <= 0 || d != kTcD || max_pages <= 0 || tiles_per_split < 0) return 0;
  return tc_plan(B, Hq, Hkv, max_pages, tiles_per_split).total;
}

extern "C" fa4q_status fa4q_decode_fp4q(const void* q, const uint8_t* k_pages, const uint8_t* k_sf,
                                        const uint8_t* vt_pages, const uint8_t* vt_sf,
                                        const int32_t* block_table, const int32_t* fp4_len,
                                        int n_phys_pages, int B, int Hq, int Hkv, int d, int max_pages,
                                        fa4q_format fmt, float g_k, float g_v, float sm_scale, void* out,
                                        void* workspace, size_t workspace_bytes, int tiles_per_split,
                                        void* stream) {
  if (fmt != FA4Q_NVFP4 && fmt != FA4Q_MXFP4) return FA4Q_ERR_INVALID_ARG;
  if (fmt == FA4Q_MXFP4) return FA4Q_ERR_UNSUPPORTED;          // the query residuals are NVFP4
  if (!q || !k_pages || !k_sf || !vt_pages || !vt_sf || !block_table || !fp4_len || !out || !workspace)
    return FA4Q_ERR_INVALID_ARG;
  if (B <= 0 || Hq <= 0 || Hkv <= 0 || Hq % Hkv != 0 || max_pages <= 0 || n_phys_pages <= 0 || tiles_per_split < 0)
    return FA4Q_ERR_INVALID_ARG;
  if (d != kTcD || Hq / Hkv > kTcN) return FA4Q_ERR_UNSUPPORTED;
  if (!(g_k > 0.0f) || !(g_v > 0.0f)) return FA4Q_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k_pages) || !aligned16(k_sf) || !aligned16(vt_pages) || !aligned16(vt_sf) ||
      !aligned16(out) || !aligned16(workspace))
    return FA4Q_ERR_INVALID_ARG;
  if ((int64_t)n_phys_pages * Hkv > 0x7fffffff || (int64_t)B * Hkv * 2 > 0x7fffffff) return FA4Q_ERR_UNSUPPORTED;
  const TcPlan pl = tc_plan(B, Hq, Hkv, max_pages, tiles_per_split);
  if (workspace_bytes < pl.total) return FA4Q_ERR_INVALID_ARG;
  if ((int64_t)B * Hkv * pl.splits > 0x7fffffff) return FA4Q_ERR_UNSUPPORTED;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  uint8_t* qt = ws + pl.off_qt;
  uint8_t* qt_sf = ws + pl.off_qsf;
  fa4q_status stt = launch_dec_query(static_cast<const uint16_t*>(q), B, Hq, Hkv, qt, qt_sf, st);
  if (stt != FA4Q_OK) return stt;
  CUtensorMap tq, tk, tv;
  if (!make_map_3d(&tq, qt, kTcD / 2, 128, (uint64_t)B * Hkv * 2, kTcD / 2, kTcN, CU_TENSOR_MAP_SWIZZLE_64B) ||
      !make_map_3d(&tk, k_pages, kTcD / 2, 64, (uint64_t)n_phys_pages * Hkv, kTcD / 2, 64,
                   CU_TENSOR_MAP_SWIZZLE_64B) ||
      !make_map_3d(&tv, vt_pages, 32, kTcD, (uint64_t)n_phys_pages * Hkv, 32, kTcD, CU_TENSOR_MAP_SWIZZLE_32B))
    return FA4Q_ERR_CUDA;
  const float sms = sm_scale > 0.0f ? sm_scale : 1.0f / sqrtf((float)d);
  TcParams prm{};
  prm.q_sf = qt_sf;
  prm.k_sf = k_sf;
  prm.v_sf = vt_sf;
  prm.table = block_table;
  prm.len = fp4_len;
  prm.ws = reinterpret_cast<float*>(ws);
  prm.B = B;
  prm.Hq = Hq;
  prm.Hkv = Hkv;
  prm.G = Hq / Hkv;
  prm.max_pages = max_pages;
  prm.n_phys = n_phys_pages;
  prm.splits = pl.splits;
  prm.tiles_per_split = pl.tiles_per_split;
  prm.sc = sms * g_k * kTcLog2e;
  prm.g_v = g_v;
  const int grid = B * Hkv * pl.splits;
  const int G = Hq / Hkv;
  stt = G <= 4 ? launch_tc<4>(tq, tk, tv, prm, grid, st)
               : (G <= 8 ? launch_tc<8>(tq, tk, tv, prm, grid, st) : launch_tc<16>(tq, tk, tv, prm, grid, st));
  if (stt != FA4Q_OK) return stt;
  return launch_decode_combine(reinterpret_cast<const float*>(ws), B * Hq, pl.splits, static_cast<uint16_t*>(out), st);
}
