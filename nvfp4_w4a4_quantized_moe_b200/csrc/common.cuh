// Device helpers shared by the NVFP4 MoE kernels (sm_100a only).
//
// NVFP4 element formats follow the "K-EXAONE-152B-A23B-REAP-80E-NVFP4" model
// card, section "Quantization Setup": FP4 E2M1 values in groups of 16 with an
// FP8 E4M3 block scale, under an fp32 per-tensor global scale (the
// double-scale structure of the NetsPresso AQ article, section "The Standard
// NVFP4 Serving Spec").
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <stdint.h>

#define NVDEV __device__ __forceinline__

namespace nvfp4moe {

constexpr int kQBlock = 16;          // elements per E4M3 block scale
constexpr int kRowTile = 128;        // rows per MMA tile and per scale atom
constexpr int kAtomBytes = 512;      // 128 rows x 4 scales
constexpr uint64_t kWaitLimitNs = 2000000000ull;   // 2 s per wait, then give up

// Device status word values (first word of every workspace).
enum : uint32_t { kDevOk = 0, kDevTimeout = 1 };

NVDEV uint64_t globaltimer_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

// ---------------------------------------------------------------------------
// bf16 <-> fp32
// ---------------------------------------------------------------------------
NVDEV float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
NVDEV float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }
NVDEV void unpack_bf16x8(const uint4& u, float* v) {
  v[0] = bf16_lo(u.x); v[1] = bf16_hi(u.x); v[2] = bf16_lo(u.y); v[3] = bf16_hi(u.y);
  v[4] = bf16_lo(u.z); v[5] = bf16_hi(u.z); v[6] = bf16_lo(u.w); v[7] = bf16_hi(u.w);
}
// Round two fp32 values to bf16 (nearest, ties to even); `lo` in the low half.
NVDEV uint32_t pack_bf16x2(float lo, float hi) {
  uint32_t r;
  asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
  return r;
}

// ---------------------------------------------------------------------------
// FP4 E2M1 and FP8 E4M3 conversions
// ---------------------------------------------------------------------------
// Eight fp32 values -> four bytes of packed E2M1 codes, element 2i in the low
// nibble of byte i.  Hardware conversion: round to nearest even, saturating
// to +-6, sign kept.
NVDEV uint32_t e2m1x8_hw(const float* v) {
  uint32_t r;
  asm("{\n\t.reg .b8 b0, b1, b2, b3;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b0, %2, %1;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b1, %4, %3;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b2, %6, %5;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b3, %8, %7;\n\t"
      "mov.b32 %0, {b0, b1, b2, b3};\n\t}"
      : "=r"(r)
      : "f"(v[0]), "f"(v[1]), "f"(v[2]), "f"(v[3]), "f"(v[4]), "f"(v[5]), "f"(v[6]), "f"(v[7]));
  return r;
}

// The same rounding written as the seven midpoint decisions of the E2M1 grid
// {0, .5, 1, 1.5, 2, 3, 4, 6}; a midpoint goes to the even code.  Used only to
// cross-check the hardware conversion.
NVDEV uint32_t e2m1_sw(float y) {
  const float a = fabsf(y);
  uint32_t m = (a > 0.25f) + (a >= 0.75f) + (a > 1.25f) + (a >= 1.75f) +
               (a > 2.5f) + (a >= 3.5f) + (a > 5.0f);
  return m | ((__float_as_uint(y) >> 31) << 3);
}

// Non-negative fp32 -> E4M3 code (nearest, ties to even, saturating at 448).
NVDEV uint32_t e4m3_code(float s) {
  uint16_t r;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(0.0f), "f"(s));
  return r & 0xFFu;
}
// E4M3 code -> its value (exact).
NVDEV float e4m3_value(uint32_t code) {
  uint32_t h2;
  const uint16_t in = (uint16_t)(code & 0xFFu);
  asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h2) : "h"(in));
  return __half2float(__ushort_as_half((unsigned short)(h2 & 0xFFFFu)));
}

// Two independent IEEE fp32 multiplies (round to nearest) in one instruction.
NVDEV uint64_t mul_f32x2(uint64_t a, uint64_t b) {
  uint64_t r;
  asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
  return r;
}
NVDEV uint64_t pack_f32x2(float lo, float hi) {
  return (uint64_t)__float_as_uint(lo) | ((uint64_t)__float_as_uint(hi) << 32);
}
NVDEV float lo_f32(uint64_t p) { return __uint_as_float((uint32_t)p); }
NVDEV float hi_f32(uint64_t p) { return __uint_as_float((uint32_t)(p >> 32)); }

// The per-tensor constants of the block scale: g, d = 6 g, and RN(1/d) for
// the division below when d is in the range where it is exact.
struct BlockScaler {
  float g, d, rcp_d;
  bool fast;
};
NVDEV BlockScaler make_scaler(float g) {
  BlockScaler b;
  b.g = g;
  b.d = __fmul_rn(6.0f, g);
  // 2^-60 <= d <= 2^100: the residual below stays a normal number for every
  // quotient that can give a non-zero scale, and 1/d is normal
  b.fast = b.d >= 8.673617e-19f && b.d <= 1.2676506e30f;
  b.rcp_d = b.fast ? __frcp_rn(b.d) : 0.0f;
  return b;
}
// a / d rounded to nearest (IEEE), for 0 <= a and the scaler's fast range,
// by Markstein's correction of the product with the correctly rounded
// reciprocal y = RN(1/d): q = RN(a y), r = a - d q (exact, one fused
// multiply-add), q' = RN(q + r y) is RN(a / d) (P. Markstein, "Computation of
// elementary functions on the IBM RISC System/6000 processor", IBM J. Res.
// Dev. 34(1), 1990; the theorem also in Muller et al., "Handbook of
// Floating-Point Arithmetic", on division by fused multiply-add).  Three
// instructions instead of a full division.  Only the quotient's E4M3 code is
// used, and that is always IEEE division's: a quotient of 464 or more (every
// such value gives the saturated scale 448) may come out as 464 instead, an
// overflowing product's NaN is mapped there too, and a quotient far below the
// smallest scale (where subnormal operands void the method's exactness) may
// differ in its last bit while its code stays 0.  Checked against CUDA's IEEE
// division by the test hooks.
NVDEV float div_markstein(float a, const BlockScaler& b) {
  const float q = __fmul_rn(a, b.rcp_d);
  const float r = __fmaf_rn(-q, b.d, a);
  return fminf(__fmaf_rn(r, b.rcp_d, q), 464.0f);
}
// s_raw = amax / d (0 if d = 0), rounded to nearest.
NVDEV float block_scale_raw(float amax, const BlockScaler& b) {
  if (b.fast) return div_markstein(amax, b);
  return (b.d == 0.0f) ? 0.0f : __fdiv_rn(amax, b.d);
}

// The block scale of R2: s = E4M3(amax / d), S = s * g, inv = 1 / S (zero d
// or S gives s = 0 and inv = 0).
NVDEV uint32_t block_scale(float amax, const BlockScaler& b, float& inv) {
  const uint32_t s = e4m3_code(block_scale_raw(amax, b));
  const float S = __fmul_rn(e4m3_value(s), b.g);
  inv = (S == 0.0f) ? 0.0f : __frcp_rn(S);
  return s;
}

// Quantise one 16-element block of fp32 values under global scale g
// (d = 6 g), one IEEE rounding per step:  s = E4M3(amax / d);  S = s * g;
// inv = 1 / S;  q_i = E2M1(x_i * inv).  Returns the scale code; writes 8
// bytes of packed codes.
NVDEV uint32_t quant_block16(const float* v, const BlockScaler& b, uint2& codes) {
  float amax = 0.0f;
#pragma unroll
  for (int i = 0; i < 16; ++i) amax = fmaxf(amax, fabsf(v[i]));
  float inv;
  const uint32_t s = block_scale(amax, b, inv);
  const uint64_t inv2 = pack_f32x2(inv, inv);
  float y[16];
#pragma unroll
  for (int i = 0; i < 16; i += 2) {
    const uint64_t r = mul_f32x2(pack_f32x2(v[i], v[i + 1]), inv2);
    y[i] = lo_f32(r);
    y[i + 1] = hi_f32(r);
  }
  codes.x = e2m1x8_hw(y);
  codes.y = e2m1x8_hw(y + 8);
  return s;
}

// Lane-wise max(|a|, |b|) of two packed bf16 pairs in one instruction; the
// sign bits of the result are not meaningful (clear them at the end).
NVDEV uint32_t max_abs_bf16x2(uint32_t a, uint32_t b) {
  uint32_t r;
  asm("max.xorsign.abs.bf16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
  return r;
}

// max |x| of eight packed bf16 pairs (exact: a bf16 maximum), as fp32.
NVDEV float amax16_bf16(const uint32_t* w) {
  const uint32_t m = max_abs_bf16x2(max_abs_bf16x2(max_abs_bf16x2(w[0], w[1]), max_abs_bf16x2(w[2], w[3])),
                                    max_abs_bf16x2(max_abs_bf16x2(w[4], w[5]), max_abs_bf16x2(w[6], w[7]))) &
                     0x7FFF7FFFu;
  return fmaxf(__uint_as_float(m << 16), __uint_as_float(m & 0xFFFF0000u));
}

// The same quantisation of a block given as 16 packed bf16 values (32 bytes).
NVDEV uint32_t quant_block16_bf16(const uint4& u0, const uint4& u1, const BlockScaler& b, uint2& codes) {
  const uint32_t w[8] = {u0.x, u0.y, u0.z, u0.w, u1.x, u1.y, u1.z, u1.w};
  float inv;
  const uint32_t s = block_scale(amax16_bf16(w), b, inv);
  const uint64_t inv2 = pack_f32x2(inv, inv);
  float y[16];
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const uint64_t r = mul_f32x2(((uint64_t)(w[i] & 0xFFFF0000u) << 32) | (uint64_t)(w[i] << 16), inv2);
    y[2 * i] = lo_f32(r);
    y[2 * i + 1] = hi_f32(r);
  }
  codes.x = e2m1x8_hw(y);
  codes.y = e2m1x8_hw(y + 8);
  return s;
}

// Byte offset of (row, 16-element block kb) in the tiled scale layout that the
// tensor-core MMA reads: 128-row x 4-block atoms of 512 bytes, atoms ordered
// (row tile, block group) with nblk4 = K / 64 groups per row tile; inside an
// atom row r sits at (r % 32) * 16 + (r / 32 % 4) * 4.
NVDEV size_t tiled_scale_offset(int row, int kb, int nblk4) {
  const size_t atom = (size_t)(row >> 7) * nblk4 + (kb >> 2);
  return atom * kAtomBytes + (row & 31) * 16 + ((row >> 5) & 3) * 4 + (kb & 3);
}

// Staged code layout (NVFP4_LAYOUT_STAGED): the 8-byte unit that holds the
// codes of 16-element block kb of `row` (nblk blocks per row, a multiple of
// 16).  128 rows by one 256-element K stage form a 16 KiB tile; tiles are
// stage-major within a row tile.  Inside a tile, row r fills bytes
// [128 r, 128 r + 128) and its 16-byte chunk c (blocks 2c and 2c + 1) sits at
// chunk c ^ (r % 8): the image a 128-byte-swizzled TMA box leaves in shared
// memory, so that one plain bulk copy of a tile is an MMA operand.
constexpr int kStagedTileBytes = 16384;
NVDEV size_t staged_code_unit(size_t row, int kb, int nblk) {
  const size_t tile = (row >> 7) * (size_t)(nblk >> 4) + (size_t)(kb >> 4);
  const int r = (int)(row & 127), c = (kb & 15) >> 1;
  return tile * (kStagedTileBytes / 8) + (size_t)r * 16 + (size_t)(((c ^ (r & 7)) << 1) | (kb & 1));
}

// ---------------------------------------------------------------------------
// Shared memory, mbarriers, TMA
// ---------------------------------------------------------------------------
NVDEV uint32_t smem_u32(const void* p) { return (uint32_t)__cvta_generic_to_shared(p); }

NVDEV void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count));
}
NVDEV void fence_barrier_init() { asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory"); }
// SiLU of the gated MLPs: z / (1 + e^-z) with CUDA's fast exponential and division
NVDEV float silu(float z) { return __fdividef(z, 1.0f + __expf(-z)); }
NVDEV void fence_proxy_async() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }
// TMA store of one box from shared memory (bulk async-group completion);
// x is the innermost coordinate in elements.
NVDEV void tma_store_2d(const CUtensorMap* map, const void* src, int x, int y) {
  asm volatile("cp.async.bulk.tensor.2d.global.shared::cta.bulk_group [%0, {%1, %2}], [%3];" ::"l"(map), "r"(x),
               "r"(y), "r"(smem_u32(src))
               : "memory");
}
NVDEV void bulk_commit_group() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
// this thread's bulk stores no longer read their shared-memory source
NVDEV void bulk_wait_read_all() { asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory"); }
// this thread's bulk stores are complete
NVDEV void bulk_wait_all() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }
NVDEV void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
               : "memory");
}
NVDEV void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}
NVDEV bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}
// Non-blocking probe of a phase (never suspends the thread).
NVDEV bool mbar_test_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}
// Like mbar_wait, but spinning on test_wait: the latency-critical single
// threads (TMA producer, MMA issuer) see a completed phase at once.
NVDEV bool mbar_wait_spin(uint64_t* bar, uint32_t parity, volatile int* abort) {
  if (mbar_test_wait(bar, parity)) return true;
  uint64_t t0 = 0;
  for (uint32_t i = 1;; ++i) {
    if (mbar_test_wait(bar, parity)) return true;
    if ((i & 1023u) == 0) {
      if (*abort) return false;
      const uint64_t now = globaltimer_ns();
      if (t0 == 0) {
        t0 = now;
      } else if (now - t0 > kWaitLimitNs) {
        return false;
      }
    }
  }
}

// Wait for the phase with the given parity to complete.  Gives up (returns
// false) after limit_ns (kWaitLimitNs unless a test asks for less) or when
// *abort is set by another warp.  The abort flag and the clock are looked at
// only every 256 polls, so a phase that completes is seen without the cost
// of a timer read.
NVDEV bool mbar_wait(uint64_t* bar, uint32_t parity, volatile int* abort, uint64_t limit_ns = kWaitLimitNs) {
  if (mbar_try_wait(bar, parity)) return true;
  uint64_t t0 = 0;
  for (uint32_t i = 1;; ++i) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((i & 255u) == 0) {
      if (*abort) return false;
      const uint64_t now = globaltimer_ns();
      if (t0 == 0) {
        t0 = now;
      } else if (now - t0 > limit_ns) {
        return false;
      }
    }
  }
}

NVDEV void tma_load_2d(void* dst, const CUtensorMap* map, int x, int y, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];" ::
          "r"(smem_u32(dst)),
      "l"(map), "r"(x), "r"(y), "r"(smem_u32(bar))
      : "memory");
}
NVDEV void bulk_load(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
  asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
                   smem_u32(dst)),
               "l"(src), "r"(bytes), "r"(smem_u32(bar))
               : "memory");
}
// Bring a byte range into L2 ahead of its loads (no shared memory involved).
NVDEV void bulk_prefetch_l2(const void* src, uint32_t bytes) {
  asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(src), "r"(bytes) : "memory");
}
NVDEV void prefetch_tmap(const CUtensorMap* map) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(map) : "memory");
}

// ---------------------------------------------------------------------------
// tcgen05: tensor memory, MMA, copies
// ---------------------------------------------------------------------------
NVDEV void tmem_alloc(uint32_t* dst_smem, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(dst_smem)),
               "r"(ncols));
}
NVDEV void tmem_relinquish() { asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;"); }
NVDEV void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols));
}
NVDEV void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
NVDEV void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }
// Arrive once on `bar` when every earlier tcgen05 async op of this thread is done.
NVDEV void tc_commit(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                   smem_u32(bar))
               : "memory");
}

// D[tmem] (+)= (A * sfA) x (B * sfB)^T, FP4 E2M1 operands from shared memory,
// UE4M3 scales (one per 16 elements) from tensor memory, fp32 accumulate.
NVDEV void mma_fp4(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc, uint32_t sfa_tmem,
                   uint32_t sfb_tmem, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::mxf4nvf4.block_scale.scale_vec::4X [%0], %1, %2, %3, [%5], [%6], p;\n\t}" ::
          "r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate), "r"(sfa_tmem), "r"(sfb_tmem));
}
// D[tmem] (+)= A x B^T, bf16 operands, fp32 accumulate.
NVDEV void mma_bf16(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate));
}
// Copy one 512-byte scale atom (32 rows of 16 bytes) from shared memory into
// 4 tensor-memory columns, replicated into all four 32-lane sub-partitions.
NVDEV void tc_cp_scale_atom(uint32_t taddr, uint64_t sdesc) {
  asm volatile("tcgen05.cp.cta_group::1.32x128b.warpx4 [%0], %1;" ::"r"(taddr), "l"(sdesc));
}

// Copy 128 rows x 32 bytes from shared memory into 8 tensor-memory columns of
// all 128 lanes (no replication).
NVDEV void tc_cp_128x256b(uint32_t taddr, uint64_t sdesc) {
  asm volatile("tcgen05.cp.cta_group::1.128x256b [%0], %1;" ::"r"(taddr), "l"(sdesc));
}
// Descriptor of a no-swizzle K-major source with 8-row x 16-byte core
// matrices: `lbo` bytes between the two 16-byte halves of a 32-byte row
// group, `sbo` bytes between groups of 8 rows.
NVDEV uint64_t sdesc_interleave(uint32_t saddr, uint32_t lbo, uint32_t sbo) {
  uint64_t d = (uint64_t)((saddr >> 4) & 0x3FFFu);
  d |= (uint64_t)((lbo >> 4) & 0x3FFFu) << 16;
  d |= (uint64_t)((sbo >> 4) & 0x3FFFu) << 32;
  d |= (uint64_t)1 << 46;
  return d;
}

// Shared-memory matrix descriptor, K-major operand with 128-byte swizzle:
// rows of 128 bytes, groups of 8 rows 1024 bytes apart.
NVDEV uint64_t sdesc_sw128(uint32_t saddr) {
  uint64_t d = (uint64_t)((saddr >> 4) & 0x3FFFu);
  d |= (uint64_t)1 << 16;                    // leading offset (unused when swizzled)
  d |= (uint64_t)(1024 >> 4) << 32;          // stride offset: 8 rows x 128 B
  d |= (uint64_t)1 << 46;                    // descriptor version for sm_100
  d |= (uint64_t)2 << 61;                    // 128-byte swizzle
  return d;
}
// Descriptor of a scale atom: 32 rows of 16 bytes, contiguous, no swizzle.
NVDEV uint64_t sdesc_scale_atom(uint32_t saddr) {
  uint64_t d = (uint64_t)((saddr >> 4) & 0x3FFFu);
  d |= (uint64_t)(128 >> 4) << 16;
  d |= (uint64_t)(128 >> 4) << 32;           // 8 rows x 16 B
  d |= (uint64_t)1 << 46;
  return d;
}
// Instruction descriptor: kind::mxf4nvf4, E2M1 x E2M1, UE4M3 scales, K-major
// operands, M x N tile.
__host__ __device__ constexpr uint32_t idesc_fp4(int M, int N) {
  return (1u << 7) | (1u << 10) | ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}
// Instruction descriptor: kind::f16 with bf16 operands and fp32 accumulator.
__host__ __device__ constexpr uint32_t idesc_bf16(int M, int N) {
  return (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}

// 32 consecutive fp32 columns of this warp's 32 TMEM lanes (one lane per thread).
NVDEV void tmem_ld32(uint32_t taddr, uint32_t* r) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, "
      "%16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
        "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
        "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
}
NVDEV void tmem_ld_wait() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }

// ---------------------------------------------------------------------------
// CTA pairs (a cluster of two CTAs sharing one tcgen05 MMA, .cta_group::2).
// The even CTA of the pair (rank 0) is the leader: it issues the pair's
// tensor-core copies and MMAs, which read both CTAs' shared memory and write
// both CTAs' tensor memory at the same addresses.  No load here uses cluster
// multicast: each CTA loads its own operands.
// ---------------------------------------------------------------------------
NVDEV uint32_t cluster_ctarank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
// Shared::cluster address of the variable at shared::cta address `addr` in
// the CTA of cluster rank `rank`.
NVDEV uint32_t mapa_shared(uint32_t addr, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(addr), "r"(rank));
  return r;
}
// Every thread of both CTAs: release this CTA's earlier memory operations to
// the cluster, then wait for the other CTA.
NVDEV void cluster_sync_all() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}
// Arrive on an mbarrier of either CTA of the pair (shared::cluster address),
// with the default CTA-scope release: the arrivals that cross to the other
// CTA only say that tensor-memory reads have finished (tcgen05.wait::ld came
// first), so no memory write needs to be made visible to it, and a
// cluster-scope release would stall the thread until its earlier global
// stores had landed.
NVDEV void mbar_arrive_remote(uint32_t bar) {
  asm volatile("mbarrier.arrive.shared::cluster.b64 _, [%0];" ::"r"(bar) : "memory");
}
// TMA tile load into this CTA's shared memory whose completion counts on an
// mbarrier of either CTA of the pair (`bar`, a shared::cluster address): the
// leader's stage barrier then covers the bytes of both CTAs.  No multicast.
NVDEV void tma_load_2d_pair(void* dst, const CUtensorMap* map, int x, int y, uint32_t bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3}], [%4];" ::"r"(smem_u32(dst)),
      "l"(map), "r"(x), "r"(y), "r"(bar)
      : "memory");
}
NVDEV void tmem_alloc_pair(uint32_t* dst_smem, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(dst_smem)),
               "r"(ncols));
}
NVDEV void tmem_relinquish_pair() { asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;"); }
NVDEV void tmem_dealloc_pair(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols));
}
// Arrive once on `bar` (shared::cluster address, either CTA) when every
// earlier pair-wide tcgen05 operation of this thread is done.
NVDEV void tc_commit_pair(uint32_t bar) {
  asm volatile("tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar) : "memory");
}
// The pair's block-scaled FP4 MMA: D (128 rows in each CTA's tensor memory)
// += A (each CTA's 128 rows) x B (N rows, the first N/2 from the leader's
// shared memory, the rest from the other CTA's), scales from each CTA's
// tensor memory.
NVDEV void mma_fp4_pair(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc, uint32_t sfa_tmem,
                        uint32_t sfb_tmem, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::mxf4nvf4.block_scale.scale_vec::4X [%0], %1, %2, %3, [%5], [%6], p;\n\t}" ::
          "r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate), "r"(sfa_tmem), "r"(sfb_tmem));
}
// One scale atom from each CTA's shared memory into its own tensor memory.
NVDEV void tc_cp_scale_atom_pair(uint32_t taddr, uint64_t sdesc) {
  asm volatile("tcgen05.cp.cta_group::2.32x128b.warpx4 [%0], %1;" ::"r"(taddr), "l"(sdesc));
}

// Programmatic dependent launch.  griddep_wait() blocks until the previous
// kernel in the stream has finished and its memory is visible (a no-op for a
// kernel launched without the attribute); griddep_launch() lets the next
// kernel's blocks be scheduled before this one finishes.
NVDEV void griddep_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
NVDEV void griddep_launch() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

NVDEV uint32_t elect_one() {
  uint32_t pred = 0;
  asm volatile(
      "{\n\t.reg .b32 r;\n\t.reg .pred p;\n\t"
      "elect.sync r|p, 0xffffffff;\n\t"
      "selp.b32 %0, 1, 0, p;\n\t}"
      : "=r"(pred));
  return pred;
}

}  // namespace nvfp4moe
