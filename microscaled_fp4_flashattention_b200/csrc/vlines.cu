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
//   colmass_kernel<0>  grid (key chunk, kv-head, sequence), 8 warps, 32 query rows each:
//                      BF16 mma.sync m16n8k16 scores of the R rows against the chunk's keys
//                      (K streamed through a two-stage cp.async ring), per row a running
//                      maximum and sum of exp2 -> partials (m, l) per (row, chunk)
//   lse_kernel         partials -> lse2[row] = m + log2(l)   (log2 domain)
//   colmass_kernel<1>  the same scores again; mass_j = sum_i exp2(s2_ij - lse2_i), reduced
//                      over the rows of a warp by shuffles and over the warps in shared memory
//   select_kernel      grid (kv-head, sequence): the masses in shared memory, an 8-bit radix
//                      select of the threshold (4 passes), an ordered compaction (positions
//                      ascending), the exclusion-mask words and the gather of the kept rows
// The scores are computed twice rather than stored (R x n_prefix FP32 per group would be
// 33 MB per (sequence, kv-head) at 32K keys).
#include <math.h>

#include "fa4q_common.cuh"
#include "fa4q_internal.h"

namespace fa4q {

constexpr int kVlThreads = 256;          // 8 warps x 32 query rows = up to 256 rows
constexpr int kVlTile = 64;              // keys per sub-tile
constexpr int kVlChunk = 1024;           // keys per CTA
constexpr int kVlPad = 8;                // bf16 elements of row padding (16 bytes)
constexpr int kSelThreads = 1024;
constexpr float kVlLog2e = 1.4426950408889634f;

struct VlParams {
  const uint16_t* q_obs;     // [B][Hq][n_obs][d]
  const uint16_t* k;         // [B][Hkv][L][d]
  const int32_t* n_prefix;   // [B]
  float* part;               // [B][Hkv][R][chunks][2]
  float* lse2;               // [B][Hkv][R]
  float* mass;               // [B][Hkv][L]
  int B, Hq, Hkv, n_obs, L, d, R, chunks;
  float c2;                  // sm_scale * log2(e)
};

FA4Q_DEVINL void ldsm_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}

// D (16x8, FP32) += A (16x16, row) * B (16x8, col), BF16 inputs
FA4Q_DEVINL void mma_bf16(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
      "{%8,%9}, {%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// 16-byte async copy global -> shared; src_bytes = 0 fills zeros without reading
FA4Q_DEVINL void cp_async16(uint32_t dst, const void* src, uint32_t src_bytes) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(src_bytes)
               : "memory");
}
FA4Q_DEVINL void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
FA4Q_DEVINL void cp_async_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }

FA4Q_DEVINL float vl_ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// (m, l) of two partial softmax sums merged (m = -inf means empty)
FA4Q_DEVINL void merge_ml(float& m, float& l, float m2, float l2) {
  const float mn = fmaxf(m, m2);
  if (mn == -INFINITY) return;
  l = (m == -INFINITY ? 0.0f : l * vl_ex2(m - mn)) + (m2 == -INFINITY ? 0.0f : l2 * vl_ex2(m2 - mn));
  m = mn;
}

template <int D, int PASS>
__global__ void __launch_bounds__(kVlThreads, 2) colmass_kernel(const VlParams p) {
  constexpr int kRow = D + kVlPad;                 // padded row, bf16 elements
  constexpr int kKs = D / 16;                      // k-steps
  extern __shared__ __align__(16) uint8_t smem_raw[];
  uint16_t* sq = reinterpret_cast<uint16_t*>(smem_raw);                 // [R][kRow]
  uint16_t* sk = sq + kVlThreads * kRow;                                // [2][kVlTile][kRow]
  float* red = reinterpret_cast<float*>(sk + 2 * kVlTile * kRow);       // [8][kVlTile]

  const int chunk = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int G = p.Hq / p.Hkv;
  const int n_pre = min(max(p.n_prefix[b], 0), p.L);
  const int key_begin = chunk * kVlChunk;
  const int key_end = min(key_begin + kVlChunk, n_pre);
  const int n_tiles = key_end > key_begin ? (key_end - key_begin + kVlTile - 1) / kVlTile : 0;
  const bool active = warp * 32 < p.R;             // rows [32 warp, 32 warp + 32)
  const int64_t bh = static_cast<int64_t>(b) * p.Hkv + h;

  // observation rows -> shared memory (row i = g * n_obs + t of q-head h*G + g)
  for (int idx = threadIdx.x; idx < p.R * (D / 8); idx += kVlThreads) {
    const int i = idx / (D / 8), c = idx % (D / 8);
    const int g = i / p.n_obs, t = i % p.n_obs;
    const uint16_t* src = p.q_obs + ((static_cast<int64_t>(b) * p.Hq + h * G + g) * p.n_obs + t) * D + 8 * c;
    *reinterpret_cast<uint4*>(sq + i * kRow + 8 * c) = *reinterpret_cast<const uint4*>(src);
  }
  const uint16_t* kbase = p.k + bh * p.L * D;
  auto load_tile = [&](int tile, int buf) {
    const int key0 = key_begin + tile * kVlTile;
    for (int idx = threadIdx.x; idx < kVlTile * (D / 8); idx += kVlThreads) {
      const int r = idx / (D / 8), c = idx % (D / 8);
      const int key = key0 + r;
      const bool in = key < p.L;
      const uint16_t* src = kbase + static_cast<int64_t>(in ? key : 0) * D + 8 * c;
      cp_async16(smem_u32(sk + (buf * kVlTile + r) * kRow + 8 * c), src, in ? 16u : 0u);
    }
    cp_async_commit();
  };
  if (n_tiles > 0) load_tile(0, 0);
  __syncthreads();

  // ldmatrix addresses of this warp's A fragments (rows 32 warp + 16 mt + ...), k-step 0
  const uint32_t a_addr0 = smem_u32(sq + (warp * 32 + ((lane >> 3) & 1) * 8 + (lane & 7)) * kRow + (lane >> 4) * 8);
  // per thread: rows r(mt, hf) = 32 warp + 16 mt + g + 8 hf, g = lane / 4
  const int g4 = lane >> 2, t4 = lane & 3;
  float m_run[2][2], l_run[2][2], lse[2][2];
#pragma unroll
  for (int mt = 0; mt < 2; ++mt)
#pragma unroll
    for (int hf = 0; hf < 2; ++hf) {
      m_run[mt][hf] = -INFINITY;
      l_run[mt][hf] = 0.0f;
      const int row = warp * 32 + mt * 16 + g4 + 8 * hf;
      lse[mt][hf] = (PASS == 1 && active) ? p.lse2[bh * p.R + row] : 0.0f;
    }

  for (int tile = 0; tile < n_tiles; ++tile) {
    const int buf = tile & 1;
    if (tile + 1 < n_tiles) {
      load_tile(tile + 1, buf ^ 1);
      cp_async_wait<1>();
    } else {
      cp_async_wait<0>();
    }
    __syncthreads();
    const int key0 = key_begin + tile * kVlTile;
    float acc[2][8][4];
#pragma unroll
    for (int mt = 0; mt < 2; ++mt)
#pragma unroll
      for (int nt = 0; nt < 8; ++nt)
#pragma unroll
        for (int e = 0; e < 4; ++e) acc[mt][nt][e] = 0.0f;
    if (active) {
#pragma unroll
      for (int ks = 0; ks < kKs; ++ks) {
        uint32_t a[2][4];
#pragma unroll
        for (int mt = 0; mt < 2; ++mt)
          ldsm_x4(a_addr0 + (mt * 16 * kRow + ks * 16) * 2, a[mt][0], a[mt][1], a[mt][2], a[mt][3]);
#pragma unroll
        for (int np2 = 0; np2 < 4; ++np2) {
          const int key = np2 * 16 + (lane >> 4) * 8 + (lane & 7);
          const int col = ks * 16 + ((lane >> 3) & 1) * 8;
          uint32_t b0, b1, b2, b3;
          ldsm_x4(smem_u32(sk + (buf * kVlTile + key) * kRow + col), b0, b1, b2, b3);
#pragma unroll
          for (int mt = 0; mt < 2; ++mt) {
            mma_bf16(acc[mt][2 * np2], a[mt], b0, b1);
            mma_bf16(acc[mt][2 * np2 + 1], a[mt], b2, b3);
          }
        }
      }
    }
    // scores in the log2 domain; keys outside the candidate prefix do not take part
    float colsum[8][2];
#pragma unroll
    for (int nt = 0; nt < 8; ++nt) colsum[nt][0] = colsum[nt][1] = 0.0f;
#pragma unroll
    for (int mt = 0; mt < 2; ++mt)
#pragma unroll
      for (int hf = 0; hf < 2; ++hf) {
        float v[16];
#pragma unroll
        for (int nt = 0; nt < 8; ++nt)
#pragma unroll
          for (int c = 0; c < 2; ++c) {
            const int key = key0 + nt * 8 + 2 * t4 + c;
            v[2 * nt + c] = key < key_end ? acc[mt][nt][2 * hf + c] * p.c2 : -INFINITY;
          }
        if constexpr (PASS == 0) {
          float tmax = v[0];
#pragma unroll
          for (int i = 1; i < 16; ++i) tmax = fmaxf(tmax, v[i]);
          const float mn = fmaxf(m_run[mt][hf], tmax);
          if (mn != -INFINITY) {
            float s = 0.0f;
#pragma unroll
            for (int i = 0; i < 16; ++i) s += vl_ex2(v[i] - mn);
            l_run[mt][hf] = (m_run[mt][hf] == -INFINITY ? 0.0f : l_run[mt][hf] * vl_ex2(m_run[mt][hf] - mn)) + s;
            m_run[mt][hf] = mn;
          }
        } else {
#pragma unroll
          for (int nt = 0; nt < 8; ++nt)
#pragma unroll
            for (int c = 0; c < 2; ++c) colsum[nt][c] += vl_ex2(v[2 * nt + c] - lse[mt][hf]);
        }
      }
    if constexpr (PASS == 1) {
      // sum over the 8 row groups of the warp (lanes with the same t4), then over the warps
#pragma unroll
      for (int nt = 0; nt < 8; ++nt)
#pragma unroll
        for (int c = 0; c < 2; ++c) {
          float x = colsum[nt][c];
          x += __shfl_xor_sync(0xffffffffu, x, 4);
          x += __shfl_xor_sync(0xffffffffu, x, 8);
          x += __shfl_xor_sync(0xffffffffu, x, 16);
          colsum[nt][c] = x;
        }
      if (g4 == 0) {
#pragma unroll
        for (int nt = 0; nt < 8; ++nt)
#pragma unroll
          for (int c = 0; c < 2; ++c) red[warp * kVlTile + nt * 8 + 2 * t4 + c] = active ? colsum[nt][c] : 0.0f;
      }
      __syncthreads();
      if (threadIdx.x < kVlTile) {
        const int key = key0 + threadIdx.x;
        float sum = 0.0f;
#pragma unroll
        for (int w = 0; w < kVlThreads / 32; ++w) sum += red[w * kVlTile + threadIdx.x];
        if (key < key_end) p.mass[bh * p.L + key] = sum;
      }
    }
    __syncthreads();   // the buffer is refilled two tiles later; red is reused next tile
  }
  if constexpr (PASS == 1) {
    // positions of this chunk outside the candidate prefix carry no mass
    const int z0 = max(key_begin, n_pre), z1 = min(key_begin + kVlChunk, p.L);
    for (int key = z0 + threadIdx.x; key < z1; key += kVlThreads) p.mass[bh * p.L + key] = 0.0f;
  }
  if constexpr (PASS == 0) {
    // merge the four threads of each row (t4), then one lane writes the row's partial
#pragma unroll
    for (int mt = 0; mt < 2; ++mt)
#pragma unroll
      for (int hf = 0; hf < 2; ++hf) {
        float m = m_run[mt][hf], l = l_run[mt][hf];
#pragma unroll
        for (int o = 1; o <= 2; o <<= 1) {
          const float m2 = __shfl_xor_sync(0xffffffffu, m, o);
          const float l2 = __shfl_xor_sync(0xffffffffu, l, o);
          merge_ml(m, l, m2, l2);
        }
        const int row = warp * 32 + mt * 16 + g4 + 8 * hf;
        if (active && t4 == 0) {
          float* dst = p.part + ((bh * p.R + row) * p.chunks + chunk) * 2;
          dst[0] = m;
          dst[1] = l;
        }
      }
  }
}

// partials (m, l) of every chunk -> lse2 = m + log2(l) per observation row
__global__ void vl_lse_kernel(const float* __restrict__ part, float* __restrict__ lse2, int R, int chunks) {
  const int64_t bh = blockIdx.x;
  const int row = threadIdx.x;
  if (row >= R) return;
  const float* src = part + (bh * R + row) * chunks * 2;
  float m = -INFINITY, l = 0.0f;
  for (int c = 0; c < chunks; ++c) merge_ml(m, l, src[2 * c], src[2 * c + 1]);
  lse2[bh * R + row] = l > 0.0f ? m + log2f(l) : INFINITY;
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

// exclusive prefix count of `flag` over the block in thread order; *total = the block's count
FA4Q_DEVINL uint32_t block_excl_count(bool flag, uint32_t* wsum, uint32_t* total) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t ballot = __ballot_sync(0xffffffffu, flag);
  const uint32_t lane_rank = __popc(ballot & ((1u << lane) - 1u));
  if (lane == 0) wsum[warp] = __popc(ballot);
  __syncthreads();
  if (warp == 0) {
    const uint32_t v = lane < (kSelThreads / 32) ? wsum[lane] : 0u;
    uint32_t incl = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t y = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += y;
    }
    if (lane < (kSelThreads / 32)) wsum[lane] = incl - v;
    if (lane == 31) wsum[32] = incl;
  }
  __syncthreads();
  const uint32_t rank = wsum[warp] + lane_rank;
  *total = wsum[32];
  __syncthreads();
  return rank;
}

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
  const int tid = threadIdx.x;
  const int n = min(max(p.n_prefix[b], 0), p.L);
  int cnt = static_cast<int>(ceil(p.rho * static_cast<double>(n) - 1e-9));
  cnt = min(max(cnt, 0), n);

  // masses are >= 0, so their bit patterns order like the values
  for (int j = tid; j < n; j += kSelThreads) bits[j] = __float_as_uint(p.mass[bh * p.L + j]);
  for (int i = tid; i < p.max_pages; i += kSelThreads) mask[i] = 0ull;
  __syncthreads();

  // radix select of the cnt-th largest pattern T, 8 bits at a time from the top; at the end
  // `remaining` is how many of the elements equal to T belong to the top cnt
  uint32_t prefix = 0, pmask = 0, remaining = static_cast<uint32_t>(cnt);
  if (cnt > 0) {
    for (int shift = 24; shift >= 0; shift -= 8) {
      for (int i = tid; i < 256; i += kSelThreads) hist[i] = 0;
      __syncthreads();
      for (int j = tid; j < n; j += kSelThreads) {
        const uint32_t x = bits[j];
        if ((x & pmask) == prefix) atomicAdd(&hist[(x >> shift) & 255u], 1u);
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
    // position order (the lowest positions win ties); positions come out ascending
    uint32_t base_eq = 0, base_sel = 0;
    for (int t0 = 0; t0 < n; t0 += kSelThreads) {
      const int j = t0 + tid;
      const uint32_t x = j < n ? bits[j] : 0u;
      const bool eq = j < n && x == prefix;
      const bool gt = j < n && x > prefix;
      uint32_t tot_eq, tot_sel;
      const uint32_t eq_rank = block_excl_count(eq, wsum, &tot_eq);
      const bool sel = gt || (eq && base_eq + eq_rank < remaining);
      const uint32_t sel_rank = block_excl_count(sel, wsum, &tot_sel);
      if (sel && base_sel + sel_rank < static_cast<uint32_t>(cnt)) {
        pos[base_sel + sel_rank] = j;
        atomicOr(&mask[j >> 6], 1ull << (j & 63));
      }
      base_eq += tot_eq;
      base_sel += tot_sel;
    }
  }
  __syncthreads();
  if (tid == 0) p.counts[bh] = cnt;
  for (int i = tid; i < cnt; i += kSelThreads) p.positions[bh * p.max_select + i] = pos[i];
  if (p.excl != nullptr)
    for (int i = tid; i < p.max_pages; i += kSelThreads) p.excl[bh * p.max_pages + i] = mask[i];
  // the kept rows, 16 bytes per lane
  const int warp = tid >> 5, lane = tid & 31, chunks = p.d / 8;
  for (int i = warp; i < cnt; i += kSelThreads / 32) {
    if (lane >= chunks) continue;
    const int64_t src = (bh * p.L + pos[i]) * p.d + 8 * lane;
    const int64_t dst = (bh * p.max_select + i) * p.d + 8 * lane;
    if (p.hp_k != nullptr)
      *reinterpret_cast<uint4*>(p.hp_k + dst) = *reinterpret_cast<const uint4*>(p.k + src);
    if (p.hp_v != nullptr)
      *reinterpret_cast<uint4*>(p.hp_v + dst) = *reinterpret_cast<const uint4*>(p.v + src);
  }
}

namespace {

int vl_rows(int Hq, int Hkv, int n_obs) { return (Hq / Hkv) * n_obs; }
int vl_chunks(int L) { return (L + kVlChunk - 1) / kVlChunk; }
size_t vl_select_smem(int L, int max_select, int max_pages) {
  return static_cast<size_t>(max_pages) * 8 + static_cast<size_t>(L) * 4 + static_cast<size_t>(max_select) * 4 +
         (256 + 33) * 4;
}
size_t vl_colmass_smem(int d) {
  return static_cast<size_t>(kVlThreads + 2 * kVlTile) * (d + kVlPad) * 2 + (kVlThreads / 32) * kVlTile * 4;
}

template <int D>
fa4q_status vl_launch(const VlParams& vp, const SelParams& sp, cudaStream_t st, size_t sel_smem) {
  const size_t cm = vl_colmass_smem(D);
  if (cudaFuncSetAttribute(colmass_kernel<D, 0>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)cm) != cudaSuccess ||
      cudaFuncSetAttribute(colmass_kernel<D, 1>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)cm) != cudaSuccess ||
      cudaFuncSetAttribute(vl_select_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sel_smem) != cudaSuccess)
    return FA4Q_ERR_CUDA;
  const dim3 grid(vp.chunks, vp.Hkv, vp.B);
  colmass_kernel<D, 0><<<grid, kVlThreads, cm, st>>>(vp);
  vl_lse_kernel<<<vp.B * vp.Hkv, vp.R, 0, st>>>(vp.part, vp.lse2, vp.R, vp.chunks);
  colmass_kernel<D, 1><<<grid, kVlThreads, cm, st>>>(vp);
  vl_select_kernel<<<dim3(vp.Hkv, vp.B), kSelThreads, sel_smem, st>>>(sp);
  return launch_status();
}

}  // namespace
}  // namespace fa4q

using namespace fa4q;

extern "C" size_t fa4q_vlines_workspace_size(int B, int Hq, int Hkv, int n_obs, int L) {
  if (B <= 0 || Hq <= 0 || Hkv <= 0 || Hq % Hkv != 0 || n_obs <= 0 || L <= 0) return 0;
  const size_t rows = static_cast<size_t>(B) * Hkv * vl_rows(Hq, Hkv, n_obs);
  return rows * (2 * static_cast<size_t>(vl_chunks(L)) + 1) * sizeof(float);
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
  if (R % 32 != 0 || R > kVlThreads) return FA4Q_ERR_UNSUPPORTED;
  const double need = ceil(rho * static_cast<double>(L) - 1e-9);
  if (static_cast<double>(max_select) < need || max_select <= 0) return FA4Q_ERR_INVALID_ARG;
  if (excl_mask != nullptr && static_cast<int64_t>(max_pages) * 64 < L) return FA4Q_ERR_INVALID_ARG;
  if (excl_mask == nullptr) max_pages = 0;
  if (!aligned16(q_obs) || !aligned16(k) || (v && !aligned16(v)) || (hp_k && !aligned16(hp_k)) ||
      (hp_v && !aligned16(hp_v)) || (reinterpret_cast<uintptr_t>(workspace) & 7) ||
      (reinterpret_cast<uintptr_t>(mass) & 3))
    return FA4Q_ERR_INVALID_ARG;
  if (workspace_bytes < fa4q_vlines_workspace_size(B, Hq, Hkv, n_obs, L)) return FA4Q_ERR_INVALID_ARG;
  if (B > 65535 || Hkv > 65535 || static_cast<int64_t>(B) * Hkv > 0x7fffffff) return FA4Q_ERR_UNSUPPORTED;
  const size_t sel_smem = vl_select_smem(L, max_select, max_pages);
  if (sel_smem > 227 * 1024) return FA4Q_ERR_UNSUPPORTED;   // candidates held in shared memory
  VlParams vp;
  vp.q_obs = static_cast<const uint16_t*>(q_obs);
  vp.k = static_cast<const uint16_t*>(k);
  vp.n_prefix = n_prefix;
  vp.chunks = vl_chunks(L);
  vp.part = static_cast<float*>(workspace);
  vp.lse2 = vp.part + static_cast<size_t>(B) * Hkv * R * vp.chunks * 2;
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
  return d == 128 ? vl_launch<128>(vp, sp, st, sel_smem) : vl_launch<64>(vp, sp, st, sel_smem);
}
