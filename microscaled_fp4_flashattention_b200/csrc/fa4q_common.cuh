// fa4q_common.cuh - device helpers shared by the fa4q kernels (sm_100a only).
//
// Inline-PTX wrappers for mbarriers, TMA bulk copies and the tcgen05 tensor-core
// family (TMEM allocation, block-scaled MMA, scale-factor copies, TMEM loads and
// stores), plus the FP4 / E4M3 / E8M0 conversions of the microscaling formats.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <stdint.h>

#include "fa4q.h"

#if defined(__CUDA_ARCH__) && (__CUDA_ARCH__ < 1000)
#error "fa4q kernels target sm_100a only"
#endif

#define FA4Q_DEVINL __device__ __forceinline__

namespace fa4q {

// ---------------------------------------------------------------------------------------
// status word: set by kernels whose bounded waits expire (one per translation unit;
// fa4q_device_status ORs them together).
// ---------------------------------------------------------------------------------------
enum : uint32_t {
  kStatusTimeoutTmaFull = 1u << 0,
  kStatusTimeoutMma = 1u << 1,
  kStatusTimeoutSoftmax = 1u << 2,
  kStatusTimeoutDrain = 1u << 3,
  kStatusTimeoutProbe = 1u << 4,
  kStatusTimeoutDecode = 1u << 5,
};

// Time limit of a bounded wait (global timer nanoseconds): far above any legitimate wait,
// short enough that a wait nothing will satisfy ends in seconds.
constexpr uint64_t kWaitNs = 2000000000ull;

FA4Q_DEVINL uint64_t globaltimer_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

// ---------------------------------------------------------------------------------------
// basic address helpers
// ---------------------------------------------------------------------------------------
FA4Q_DEVINL uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

FA4Q_DEVINL uint32_t elect_one() {
  uint32_t pred = 0;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "elect.sync _|p, 0xffffffff;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}\n"
      : "=r"(pred));
  return pred;
}

// ---------------------------------------------------------------------------------------
// mbarrier
// ---------------------------------------------------------------------------------------
FA4Q_DEVINL void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count));
}

FA4Q_DEVINL void fence_barrier_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

FA4Q_DEVINL void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

FA4Q_DEVINL void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

FA4Q_DEVINL void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)),
               "r"(bytes)
               : "memory");
}

FA4Q_DEVINL bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, 0xF4240;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}\n"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

// Bounded wait on phase `parity` (each try_wait suspends at most 1 ms); returns false, and
// records `code` in *status, once `limit_ns` have passed without the phase completing.
FA4Q_DEVINL bool mbar_wait(uint64_t* bar, uint32_t parity, uint32_t* status, uint32_t code,
                           uint64_t limit_ns = kWaitNs) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = globaltimer_ns();
  while (true) {
    if (mbar_try_wait(bar, parity)) return true;
    if (globaltimer_ns() - t0 > limit_ns) break;
  }
  atomicOr(status, code);
  return false;
}

// ---------------------------------------------------------------------------------------
// TMA: tiled tensor loads and untiled bulk loads into shared memory
// ---------------------------------------------------------------------------------------
FA4Q_DEVINL void tma_load_3d(void* dst, const CUtensorMap* map, int x, int y, int z,
                             uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3, %4}], [%5];" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(z), "r"(smem_u32(bar))
      : "memory");
}

FA4Q_DEVINL void bulk_load(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::
          "r"(smem_u32(dst)),
      "l"(src), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}

FA4Q_DEVINL void prefetch_tmap(const CUtensorMap* map) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}

// ---------------------------------------------------------------------------------------
// tcgen05: tensor memory, MMA, copies
// ---------------------------------------------------------------------------------------
FA4Q_DEVINL void tmem_alloc(uint32_t* smem_dst, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                   smem_u32(smem_dst)),
               "r"(ncols)
               : "memory");
}

FA4Q_DEVINL void tmem_relinquish() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}

FA4Q_DEVINL void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols)
               : "memory");
}

FA4Q_DEVINL void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
FA4Q_DEVINL void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// Arrive on `bar` once all prior tcgen05 async operations of this thread complete.
FA4Q_DEVINL void tc_commit(uint64_t* bar) {
  asm volatile(
      "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
          smem_u32(bar))
      : "memory");
}

// Shared-memory matrix descriptor (K-major operand tile), sm_100 encoding:
// start address >> 4 in [0,14), leading-dim byte offset >> 4 in [16,30), stride-dim byte
// offset >> 4 in [32,46), version 1 in [46,48), swizzle mode in [61,64).
enum SwizzleMode : uint32_t { kSwizNone = 0, kSwiz128 = 2, kSwiz64 = 4, kSwiz32 = 6 };

FA4Q_DEVINL uint64_t make_smem_desc(uint32_t saddr, uint32_t lbo_bytes, uint32_t sbo_bytes,
                                    uint32_t swizzle) {
  uint64_t d = 0;
  d |= static_cast<uint64_t>((saddr >> 4) & 0x3FFF);
  d |= static_cast<uint64_t>((lbo_bytes >> 4) & 0x3FFF) << 16;
  d |= static_cast<uint64_t>((sbo_bytes >> 4) & 0x3FFF) << 32;
  d |= static_cast<uint64_t>(1) << 46;
  d |= static_cast<uint64_t>(swizzle & 7) << 61;
  return d;
}

// Instruction descriptor of the block-scaled FP4 MMA (kind::mxf4 / kind::mxf4nvf4), both
// operands K-major E2M1, M = 128, FP32 accumulate.  Fields: b_sf_id [4,6), a/b format
// (E2M1 = 1) [7,10)/[10,13), N>>3 [17,23), scale format (0 UE4M3, 1 UE8M0) [23],
// M>>4 [24,29), a_sf_id [29,31).
FA4Q_DEVINL uint32_t make_idesc_fp4(int N, bool ue8m0, uint32_t a_sf_id, uint32_t b_sf_id) {
  uint32_t d = 0;
  d |= (b_sf_id & 3u) << 4;
  d |= 1u << 7;
  d |= 1u << 10;
  d |= (static_cast<uint32_t>(N) >> 3) << 17;
  d |= (ue8m0 ? 1u : 0u) << 23;
  d |= (128u >> 4) << 24;
  d |= (a_sf_id & 3u) << 29;
  return d;
}

// Instruction descriptor of the BF16 MMA (kind::f16, FP32 accumulate), M = 128.  Fields:
// D format (F32 = 1) [4,6), A / B format (BF16 = 1) [7,10) / [10,13), A major [15] (0: K-major),
// B major [16] (0: K-major, 1: MN-major), N>>3 [17,23), M>>4 [24,29).
FA4Q_DEVINL uint32_t make_idesc_bf16(int N, bool b_mn_major) {
  uint32_t d = 0;
  d |= 1u << 4;
  d |= 1u << 7;
  d |= 1u << 10;
  d |= (b_mn_major ? 1u : 0u) << 16;
  d |= (static_cast<uint32_t>(N) >> 3) << 17;
  d |= (128u >> 4) << 24;
  return d;
}

// D[tmem] (+)= A[smem] * B[smem] (BF16 operands, FP32 accumulate), K = 16 per instruction.
FA4Q_DEVINL void mma_bf16(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t"
      "}\n" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// byte offset of (row r, 16-byte chunk c) in a tile of 128-byte rows with the 128-byte swizzle
// (1024-byte atoms of 8 rows; chunk c of row r stored at chunk c ^ (r % 8)) - the layout TMA
// writes with CU_TENSOR_MAP_SWIZZLE_128B and the MMA reads with the 128B swizzle mode
FA4Q_DEVINL uint32_t swz128_offset(uint32_t r, uint32_t c) {
  return (r >> 3) * 1024 + (r & 7) * 128 + ((c ^ (r & 7)) << 4);
}

// D[tmem] (+)= A[smem] * B[smem]^T with per-16-element UE4M3 scales (NVFP4).
FA4Q_DEVINL void mma_nvf4(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                          uint32_t sfa_tmem, uint32_t sfb_tmem, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::mxf4nvf4.block_scale.block16 [%0], %1, %2, %3, [%5], [%6], p;\n\t"
      "}\n" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate), "r"(sfa_tmem), "r"(sfb_tmem)
      : "memory");
}

// Same with per-32-element UE8M0 scales (MXFP4).
FA4Q_DEVINL void mma_mxf4(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                          uint32_t sfa_tmem, uint32_t sfb_tmem, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::mxf4.block_scale.block32 [%0], %1, %2, %3, [%5], [%6], p;\n\t"
      "}\n" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate), "r"(sfa_tmem), "r"(sfb_tmem)
      : "memory");
}

// Copy one 512-byte scale atom (32 rows x 16 bytes, rows 16 bytes apart) from shared memory
// into 4 TMEM columns of every lane quadrant (the scale-factor layout the MMA reads).
FA4Q_DEVINL void tmem_cp_sf_atom(uint32_t taddr, uint32_t atom_saddr) {
  const uint64_t desc = make_smem_desc(atom_saddr, 0, 128, kSwizNone);
  asm volatile("tcgen05.cp.cta_group::1.32x128b.warpx4 [%0], %1;" ::"r"(taddr), "l"(desc)
               : "memory");
}

// The same with the atom's shared-memory descriptor already formed.
FA4Q_DEVINL void tmem_cp_sf_desc(uint32_t taddr, uint64_t desc) {
  asm volatile("tcgen05.cp.cta_group::1.32x128b.warpx4 [%0], %1;" ::"r"(taddr), "l"(desc)
               : "memory");
}

// 32 consecutive 32-bit TMEM columns of this warp's lane quadrant -> 32 registers / thread.
FA4Q_DEVINL void tmem_ld32(uint32_t taddr, uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]),
        "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]),
        "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
}

FA4Q_DEVINL void tmem_ld16(uint32_t taddr, uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15])
      : "r"(taddr));
}

FA4Q_DEVINL void tmem_st32(uint32_t taddr, const uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], "
      "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,"
      "%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),
      "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]),
      "r"(r[15]), "r"(r[16]), "r"(r[17]), "r"(r[18]), "r"(r[19]), "r"(r[20]), "r"(r[21]),
      "r"(r[22]), "r"(r[23]), "r"(r[24]), "r"(r[25]), "r"(r[26]), "r"(r[27]), "r"(r[28]),
      "r"(r[29]), "r"(r[30]), "r"(r[31])
      : "memory");
}

FA4Q_DEVINL void tmem_st16(uint32_t taddr, const uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], "
      "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),
      "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]),
      "r"(r[15])
      : "memory");
}

FA4Q_DEVINL void tmem_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }
FA4Q_DEVINL void tmem_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

// ---------------------------------------------------------------------------------------
// microscaling format conversions
// ---------------------------------------------------------------------------------------
// Eight FP32 values (already divided by their block scale) -> eight E2M1 nibbles,
// element 0 in the lowest nibble; round to nearest even, saturating at +-6.
FA4Q_DEVINL uint32_t e2m1x8(float x0, float x1, float x2, float x3, float x4, float x5,
                            float x6, float x7) {
  uint32_t out;
  asm("{\n\t.reg .b8 b0, b1, b2, b3;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b0, %2, %1;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b1, %4, %3;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b2, %6, %5;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b3, %8, %7;\n\t"
      "mov.b32 %0, {b0, b1, b2, b3};\n\t}\n"
      : "=r"(out)
      : "f"(x0), "f"(x1), "f"(x2), "f"(x3), "f"(x4), "f"(x5), "f"(x6), "f"(x7));
  return out;
}

// Unsigned E4M3 code of t >= 0 (round to nearest even, saturating at 448).
FA4Q_DEVINL uint32_t ue4m3_encode(float t) {
  uint16_t two;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(two) : "f"(0.0f), "f"(t));
  return static_cast<uint32_t>(two) & 0x7Fu;
}

// Exact FP32 value of an unsigned E4M3 code.
FA4Q_DEVINL float ue4m3_decode(uint32_t code) {
  const uint32_t e = (code >> 3) & 0xF, m = code & 7;
  if (e == 0) return static_cast<float>(m) * 0.001953125f;  // m * 2^-9
  return __uint_as_float(((e + 120u) << 23) | (m << 20));
}

// floor(log2(a)) for finite a > 0 (normal or subnormal), exact.
FA4Q_DEVINL int floor_log2(float a) {
  const uint32_t u = __float_as_uint(a);
  const int ef = static_cast<int>((u >> 23) & 0xFF);
  if (ef != 0) return ef - 127;
  return -127 - (__clz(u & 0x7FFFFF) - 9);  // subnormal
}

// Shared MX exponent of a block with maximum amax: OCP rule when qmax == 0, otherwise the
// smallest e with amax <= qmax * 2^e (exact mantissa comparison).  Clamped to [-127, 127].
FA4Q_DEVINL int mx_exponent(float amax, float qmax) {
  if (!(amax > 0.0f)) return -127;
  const int E = floor_log2(amax);
  int e;
  if (qmax == 0.0f) {
    e = E - 2;
  } else {
    const int Eq = floor_log2(qmax);
    // mantissas as integers in [2^23, 2^24): amax = ma*2^(E-23), qmax = mq*2^(Eq-23)
    const uint32_t ua = __float_as_uint(amax), uq = __float_as_uint(qmax);
    const uint32_t ma = ((ua >> 23) & 0xFF) ? ((ua & 0x7FFFFF) | 0x800000)
                                            : ((ua & 0x7FFFFF) << (__clz(ua & 0x7FFFFF) - 8));
    const uint32_t mq = (uq & 0x7FFFFF) | 0x800000;
    e = E - Eq + (ma > mq ? 1 : 0);
  }
  return e < -127 ? -127 : (e > 127 ? 127 : e);
}

// 2^e as FP32 for e in [-127, 127] (2^-127 is subnormal, still exact).
FA4Q_DEVINL float exp2i(int e) {
  if (e >= -126) return __uint_as_float(static_cast<uint32_t>(e + 127) << 23);
  return __uint_as_float(0x400000u);  // 2^-127
}

FA4Q_DEVINL float bf16_to_f32(uint16_t b) { return __uint_as_float(static_cast<uint32_t>(b) << 16); }

}  // namespace fa4q
