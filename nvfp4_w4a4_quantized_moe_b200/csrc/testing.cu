// Test hooks: element-wise access to the device conversions and the router's
// sigmoid, for comparison with an independent CPU implementation.
#include "../../include/nvfp4_moe_testing.h"
#include "common.cuh"
#include "host.cuh"
#include "route.cuh"
#include "route_math.cuh"

namespace nvfp4moe {

__global__ void test_e2m1_kernel(const float* y, int n, uint8_t* hw, uint8_t* sw) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= n) return;
  float v[8] = {y[i], 0, 0, 0, 0, 0, 0, 0};
  hw[i] = (uint8_t)(e2m1x8_hw(v) & 0xFu);
  sw[i] = (uint8_t)e2m1_sw(y[i]);
}

__global__ void test_e2m1_sweep_kernel(uint32_t first, uint64_t count, unsigned long long* mismatches,
                                       uint32_t* example) {
  unsigned long long local = 0;
  uint32_t bad = 0;
  bool have_bad = false;
  const uint64_t stride = (uint64_t)gridDim.x * blockDim.x * 8;
  for (uint64_t base = ((uint64_t)blockIdx.x * blockDim.x + threadIdx.x) * 8; base < count; base += stride) {
    float v[8];
    uint32_t sw = 0;
#pragma unroll
    for (int q = 0; q < 8; ++q) {
      const uint64_t idx = base + q;
      const uint32_t bits = (uint32_t)(first + idx);
      float f = __uint_as_float(bits);
      if (idx >= count || (bits & 0x7F800000u) == 0x7F800000u && (bits & 0x7FFFFFu)) f = 0.0f;   // skip NaN
      v[q] = f;
      sw |= e2m1_sw(f) << (4 * q);
    }
    const uint32_t hw = e2m1x8_hw(v);
    if (hw != sw) {
#pragma unroll
      for (int q = 0; q < 8; ++q) {
        if (((hw >> (4 * q)) & 0xF) != ((sw >> (4 * q)) & 0xF)) {
          ++local;
          if (!have_bad) {
            bad = (uint32_t)(first + base + q);
            have_bad = true;
          }
        }
      }
    }
  }
  if (local) {
    atomicAdd(mismatches, local);
    atomicExch(example, bad);
  }
}

__global__ void test_e4m3_kernel(const float* s, int n, uint8_t* codes, float* value) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= n) return;
  const uint32_t c = e4m3_code(s[i]);
  codes[i] = (uint8_t)c;
  value[i] = e4m3_value(c);
}

__global__ void test_sigmoid_kernel(const float* l, int n, float* out) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i < n) out[i] = sigmoid_fixed(l[i]);
}

// Issue helpers for a whole warp: every lane executes the instruction, only
// the lane whose `leader` is non-zero issues it.
NVDEV void mma_fp4_pred(uint32_t leader, uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                        uint32_t sfa_tmem, uint32_t sfb_tmem, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "setp.ne.b32 q, %7, 0;\n\t"
      "@q tcgen05.mma.cta_group::1.kind::mxf4nvf4.block_scale.scale_vec::4X [%0], %1, %2, %3, [%5], [%6], p;\n\t}" ::
          "r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate), "r"(sfa_tmem), "r"(sfb_tmem), "r"(leader));
}
NVDEV void tc_cp_scale_atom_pred(uint32_t leader, uint32_t taddr, uint64_t sdesc) {
  asm volatile(
      "{\n\t.reg .pred q;\n\t"
      "setp.ne.b32 q, %2, 0;\n\t"
      "@q tcgen05.cp.cta_group::1.32x128b.warpx4 [%0], %1;\n\t}" ::"r"(taddr),
      "l"(sdesc), "r"(leader));
}

// FP4 tensor-core rate without memory traffic: one thread per CTA issues
// `iters` groups of four 128 x N x 64 block-scaled MMAs on fixed shared-memory
// operands (zeros), optionally preceded by the 12 scale-factor copies a
// 256-wide K stage needs, then waits for completion.  Cycles are the CTA's
// clock64 span.
__global__ void __launch_bounds__(128, 1) mma_peak_kernel(int iters, int n, int with_cp,
                                                          unsigned long long* cycles, uint32_t* status) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  __shared__ __align__(8) uint64_t bar;
  __shared__ __align__(8) uint64_t full_bar[8];
  __shared__ __align__(8) uint64_t empty_bar[8];
  __shared__ __align__(8) uint64_t sf_bar[2];
  __shared__ __align__(8) uint64_t cp_drain;
  __shared__ uint32_t tmem_s;
  __shared__ int abort_s;
  const int warp = threadIdx.x >> 5;
  for (int i = threadIdx.x; i < (16384 + 32768 + 6144) / 16; i += blockDim.x)
    reinterpret_cast<uint4*>(smem)[i] = make_uint4(0, 0, 0, 0);
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    for (int i = 0; i < 8; ++i) {
      mbar_init(&full_bar[i], 1);
      mbar_init(&empty_bar[i], 1);
    }
    mbar_init(&sf_bar[0], 1);
    mbar_init(&sf_bar[1], 1);
    mbar_init(&cp_drain, 1);
    abort_s = 0;
    fence_barrier_init();
  }
  fence_proxy_async();
  if (warp == 0) {
    tmem_alloc(&tmem_s, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_s;
  if (warp == 1 && with_cp >= 19) {
    // the whole warp runs the loop; one elected lane issues (19: copies and
    // MMAs predicated; 20: MMAs only, predicated; 21: copies and MMAs inside
    // a branch taken by the elected lane)
    const uint32_t leader = elect_one();
    const uint32_t sA = smem_u32(smem), sB = sA + 16384, sSF = sB + 32768;
    const uint64_t adesc = sdesc_sw128(sA), bdesc = sdesc_sw128(sB);
    const uint64_t sf0 = sdesc_scale_atom(sSF);
    constexpr uint64_t kAtom = 512 >> 4;
    const uint32_t idesc = idesc_fp4(128, n);
    const uint32_t sfa = tmem + 256, sfb = tmem + 256 + 16;
    const unsigned long long t0 = clock64();
    if (with_cp == 19) {
      for (int it = 0; it < iters; ++it) {
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          tc_cp_scale_atom_pred(leader, sfa + 4 * j, sf0 + j * kAtom);
          tc_cp_scale_atom_pred(leader, sfb + 8 * j, sf0 + (4 + j) * kAtom);
          tc_cp_scale_atom_pred(leader, sfb + 8 * j + 4, sf0 + (8 + j) * kAtom);
        }
#pragma unroll
        for (int j = 0; j < 4; ++j)
          mma_fp4_pred(leader, tmem, adesc + 2 * j, bdesc + 2 * j, idesc, sfa + 4 * j, sfb + 8 * j, (it | j) != 0);
      }
    } else if (with_cp == 20) {
      for (int it = 0; it < iters; ++it) {
#pragma unroll
        for (int j = 0; j < 4; ++j)
          mma_fp4_pred(leader, tmem, adesc + 2 * j, bdesc + 2 * j, idesc, sfa + 4 * j, sfb + 8 * j, (it | j) != 0);
      }
    } else {
      for (int it = 0; it < iters; ++it) {
        if (leader) {
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            tc_cp_scale_atom(sfa + 4 * j, sf0 + j * kAtom);
            tc_cp_scale_atom(sfb + 8 * j, sf0 + (4 + j) * kAtom);
            tc_cp_scale_atom(sfb + 8 * j + 4, sf0 + (8 + j) * kAtom);
          }
#pragma unroll
          for (int j = 0; j < 4; ++j)
            mma_fp4(tmem, adesc + 2 * j, bdesc + 2 * j, idesc, sfa + 4 * j, sfb + 8 * j, (it | j) != 0);
        }
        __syncwarp();
      }
    }
    if (leader) {
      tc_commit(&bar);
      if (!mbar_wait(&bar, 0, &abort_s)) atomicExch(status, kDevTimeout);
      cycles[blockIdx.x] = clock64() - t0;
    }
    __syncwarp();
  } else if (threadIdx.x == 32) {
    const uint32_t sA = smem_u32(smem), sB = sA + 16384, sSF = sB + 32768;
    const uint64_t adesc = sdesc_sw128(sA), bdesc = sdesc_sw128(sB);
    const uint32_t idesc = idesc_fp4(128, n);
    const unsigned long long t0 = clock64();
    auto copies = [&](uint32_t sf) {
      for (int j = 0; j < 4; ++j) {
        tc_cp_scale_atom(sf + 4 * j, sdesc_scale_atom(sSF + 512 * j));
        tc_cp_scale_atom(sf + 16 + 8 * j, sdesc_scale_atom(sSF + 2048 + 512 * j));
        tc_cp_scale_atom(sf + 20 + 8 * j, sdesc_scale_atom(sSF + 4096 + 512 * j));
      }
    };
    auto wide_copies = [&](uint32_t sf) {      // 6 copies of 128 lanes x 8 columns
      for (int j = 0; j < 2; ++j) tc_cp_128x256b(sf + 8 * j, sdesc_interleave(sSF + 2048 * j, 128, 256));
      for (int j = 0; j < 4; ++j) tc_cp_128x256b(sf + 16 + 8 * j, sdesc_interleave(sSF + 512 * j, 128, 256));
    };
    if (with_cp == 3) copies(tmem + 256);
    if (with_cp == 17 || with_cp == 18) {
      // split issue: this thread issues only MMAs; a second thread issues the
      // scale-factor copies into two alternating column sets and signals
      // each set with a commit.  Mode 18 also waits for a producer's "full".
      for (int it = 0; it < iters; ++it) {
        const int st = it & 3, b = it & 1;
        if (with_cp == 18 && !mbar_wait(&full_bar[st], (uint32_t)(it >> 2) & 1u, &abort_s)) {
          atomicExch(status, kDevTimeout);
          break;
        }
        if (!mbar_wait(&sf_bar[b], (uint32_t)(it >> 1) & 1u, &abort_s)) {
          atomicExch(status, kDevTimeout);
          break;
        }
        tc_fence_after();
        const uint32_t sf = tmem + 256 + (uint32_t)b * 48;
#pragma unroll
        for (int j = 0; j < 4; ++j)
          mma_fp4(tmem, adesc + 2 * j, bdesc + 2 * j, idesc, sf + 4 * j, sf + 16 + 8 * j, (it | j) != 0);
        tc_commit(&empty_bar[st]);
      }
    }
    if (with_cp >= 5 && with_cp <= 12) {
      // the GEMM's stage handshake: wait "full" (arrived by a second warp once
      // it has seen the "empty" commit of `stages` stages back), MMAs, commit
      // "empty".  Modes 9-12: 8 stages; 11-12: stages of 2 MMAs (K = 128).
      const int stages = with_cp >= 9 ? 8 : 4;
      const int per = with_cp >= 11 ? 2 : 4;
      const bool cps = with_cp == 6 || with_cp == 8 || with_cp == 10 || with_cp == 12;
      uint32_t phase = 0;
      for (int it = 0; it < iters * (4 / per); ++it) {
        const int st = it & (stages - 1);
        if (!(with_cp == 7 || with_cp == 8 ? mbar_wait_spin(&full_bar[st], phase, &abort_s) : mbar_wait(&full_bar[st], phase, &abort_s))) { atomicExch(status, kDevTimeout); break; }
        tc_fence_after();
        const uint32_t sf = tmem + 256 + (uint32_t)(st & 3) * 48;
        if (cps) {
          for (int j = 0; j < per; ++j) {
            tc_cp_scale_atom(sf + 4 * j, sdesc_scale_atom(sSF + 512 * j));
            tc_cp_scale_atom(sf + 16 + 8 * j, sdesc_scale_atom(sSF + 2048 + 512 * j));
            tc_cp_scale_atom(sf + 20 + 8 * j, sdesc_scale_atom(sSF + 4096 + 512 * j));
          }
        }
        for (int j = 0; j < per; ++j)
          mma_fp4(tmem, adesc + 2 * j, bdesc + 2 * j, idesc, sf + 4 * j, sf + 16 + 8 * j, (it | j) != 0);
        tc_commit(&empty_bar[st]);
        if (st == stages - 1) phase ^= 1u;
      }
    }
    for (int it = 0; (with_cp < 5 || (with_cp >= 13 && with_cp <= 16)) && it < iters; ++it) {
      // with_cp: 1 one buffer; 2 four rotating buffers; 3 rotating buffers,
      // copies issued one iteration ahead; 4 six 128x256b copies.
      // 13-16 add one stage's bookkeeping without any wait: 13 copies and a
      // commit per iteration; 14 a commit only; 15 copies and a
      // fence::after_thread_sync; 16 copies and a commit every 2nd iteration.
      const uint32_t sf = tmem + 256 + (with_cp >= 2 && with_cp <= 4 ? (uint32_t)(it & 3) * 48 : 0u);
      if (with_cp == 1 || with_cp == 2 || with_cp == 13 || with_cp == 15 || with_cp == 16) copies(sf);
      if (with_cp == 3) copies(tmem + 256 + (uint32_t)((it + 1) & 3) * 48);
      if (with_cp == 4) wide_copies(sf);
      if (with_cp == 15) tc_fence_after();
      for (int j = 0; j < 4; ++j)
        mma_fp4(tmem, adesc + 2 * j, bdesc + 2 * j, idesc, sf + 4 * j, sf + 16 + 8 * j, (it | j) != 0);
      if (with_cp == 13 || with_cp == 14 || (with_cp == 16 && (it & 1))) tc_commit(&empty_bar[it & 3]);
    }
    tc_commit(&bar);
    if (!mbar_wait(&bar, 0, &abort_s)) atomicExch(status, kDevTimeout);
    const unsigned long long t1 = clock64();
    cycles[blockIdx.x] = t1 - t0;
  } else if (threadIdx.x == 96 && (with_cp == 17 || with_cp == 18)) {
    // the scale-factor copier of the split-issue modes
    const uint32_t sSF = smem_u32(smem) + 16384 + 32768;
    for (int it = 0; it < iters; ++it) {
      const int b = it & 1;
      if (it >= 2) {
        const int prev = it - 2;
        if (!mbar_wait(&empty_bar[prev & 3], (uint32_t)(prev >> 2) & 1u, &abort_s)) {
          atomicExch(status, kDevTimeout);
          break;
        }
      }
      tc_fence_after();
      const uint32_t sf = tmem + 256 + (uint32_t)b * 48;
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        tc_cp_scale_atom(sf + 4 * j, sdesc_scale_atom(sSF + 512 * j));
        tc_cp_scale_atom(sf + 16 + 8 * j, sdesc_scale_atom(sSF + 2048 + 512 * j));
        tc_cp_scale_atom(sf + 20 + 8 * j, sdesc_scale_atom(sSF + 4096 + 512 * j));
      }
      tc_commit(&sf_bar[b]);
    }
    // the copies complete before tensor memory is freed
    tc_commit(&cp_drain);
    volatile int never = 0;
    if (!mbar_wait(&cp_drain, 0, &never)) atomicExch(status, kDevTimeout);
  } else if (threadIdx.x == 64 && ((with_cp >= 5 && with_cp <= 12) || with_cp == 18)) {
    // the producer side of the handshake, with no loads
    const int stages = with_cp >= 9 && with_cp <= 12 ? 8 : 4;
    const int per = with_cp >= 11 && with_cp <= 12 ? 2 : 4;
    uint32_t phase = 0;
    for (int it = 0; it < iters * (4 / per); ++it) {
      const int st = it & (stages - 1);
      if (!(with_cp == 7 || with_cp == 8 ? mbar_wait_spin(&empty_bar[st], phase ^ 1u, &abort_s) : mbar_wait(&empty_bar[st], phase ^ 1u, &abort_s))) { atomicExch(status, kDevTimeout); break; }
      mbar_arrive(&full_bar[st]);
      if (st == stages - 1) phase ^= 1u;
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// The give-up path that every bounded wait of the library shares, made to
// run: one CTA sets up as the GEMMs do (a bulk copy in flight, tensor memory
// allocated), then its producer warp waits on a barrier that nothing ever
// completes, with the library's own bounded wait and a caller-chosen limit.
// When the wait gives up the warp sets the abort flag and the status word and
// lets its copy land; the MMA-side warp, waiting on the same barrier, leaves
// on the abort flag, drains its tcgen05 work through a commit and frees the
// tensor memory.  Nothing traps and the context stays usable.
__global__ void __launch_bounds__(64, 1)
    test_wait_timeout_kernel(const uint4* __restrict__ src, uint64_t limit_ns, uint32_t* status,
                             unsigned long long* elapsed_ns, uint32_t* copied) {
  constexpr int kWords = 256;                       // 4 KiB copied
  __shared__ __align__(128) uint4 buf[kWords];
  __shared__ __align__(8) uint64_t full_bar, never_bar, drain_bar;
  __shared__ uint32_t tmem_s;
  __shared__ int abort_s;
  volatile int* abort_flag = &abort_s;
  const int warp = threadIdx.x >> 5;
  if (threadIdx.x == 0) {
    mbar_init(&full_bar, 1);
    mbar_init(&never_bar, 1);
    mbar_init(&drain_bar, 1);
    abort_s = 0;
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(&tmem_s, 32);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_s;
  const uint32_t leader = elect_one();
  if (warp == 0) {
    if (leader) {
      mbar_arrive_expect_tx(&full_bar, sizeof(buf));
      bulk_load(buf, src, sizeof(buf), &full_bar);
    }
    __syncwarp();
    const uint64_t t0 = globaltimer_ns();
    const bool ok = __all_sync(0xffffffffu, mbar_wait(&never_bar, 0, abort_flag, limit_ns));
    const uint64_t t1 = globaltimer_ns();
    if (!ok && leader) {
      *abort_flag = 1;
      atomicExch(status, kDevTimeout);
      elapsed_ns[0] = t1 - t0;
      // the issued copy lands before the CTA's shared memory goes away
      volatile int never = 0;
      mbar_wait(&full_bar, 0, &never);
    }
    __syncwarp();
  } else {
    const uint64_t t0 = globaltimer_ns();
    const bool ok = __all_sync(0xffffffffu, mbar_wait(&never_bar, 0, abort_flag));
    const uint64_t t1 = globaltimer_ns();
    if (leader) {
      if (!ok) elapsed_ns[1] = t1 - t0;
      // every tcgen05 operation this lane issued completes before the
      // tensor memory is freed
      tc_commit(&drain_bar);
      volatile int never = 0;
      mbar_wait(&drain_bar, 0, &never);
    }
    __syncwarp();
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 32);
  }
  if (threadIdx.x == 0) {
    uint32_t x = 0;
    for (int i = 0; i < kWords; ++i) x ^= buf[i].x ^ buf[i].y ^ buf[i].z ^ buf[i].w;
    *copied = x;
  }
}

// The block scale's quotient s_raw = amax / (6 g), computed the library's way
// (block_scale_raw) and with CUDA's IEEE division, with both E4M3 codes.
__global__ void test_block_scale_div_kernel(const float* amax, const float* g, int n, float* q_lib, float* q_ieee,
                                            uint8_t* code_lib, uint8_t* code_ieee) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= n) return;
  const BlockScaler b = make_scaler(g[i]);
  const float ql = block_scale_raw(amax[i], b);
  const float qi = (b.d == 0.0f) ? 0.0f : __fdiv_rn(amax[i], b.d);
  q_lib[i] = ql;
  q_ieee[i] = qi;
  code_lib[i] = (uint8_t)e4m3_code(ql);
  code_ieee[i] = (uint8_t)e4m3_code(qi);
}

}  // namespace nvfp4moe

using namespace nvfp4moe;

extern "C" nvfp4_status nvfp4_test_mma_peak(int iters, int n, int with_cp, int ctas, unsigned long long* cycles,
                                            uint32_t* status, void* stream) {
  NV_REQUIRE(cycles && status && iters > 0 && ctas > 0 && (n == 128 || n == 256) && with_cp >= 0 && with_cp <= 21,
             NVFP4_ERR_INVALID_ARG,
             "nvfp4_test_mma_peak: bad arguments");
  int sms = 0;
  NV_CHECK(device_sm_count(&sms));
  const int smem = 16384 + 32768 + 6144 + 1024;
  NV_CHECK(check_cuda(cudaFuncSetAttribute(mma_peak_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem),
                      "cudaFuncSetAttribute"));
  mma_peak_kernel<<<ctas, 128, smem, as_stream(stream)>>>(iters, n, with_cp, cycles, status);
  return check_launch("mma_peak_kernel");
}

extern "C" nvfp4_status nvfp4_test_e2m1(const float* y, int n, uint8_t* hw, uint8_t* sw, void* stream) {
  NV_REQUIRE(y && hw && sw && n >= 0, NVFP4_ERR_INVALID_ARG, "nvfp4_test_e2m1: bad arguments");
  int sms = 0;
  NV_CHECK(device_sm_count(&sms));
  if (n == 0) return NVFP4_OK;
  test_e2m1_kernel<<<(n + 255) / 256, 256, 0, as_stream(stream)>>>(y, n, hw, sw);
  return check_launch("test_e2m1_kernel");
}

extern "C" nvfp4_status nvfp4_test_e2m1_sweep(uint32_t first, uint64_t count, unsigned long long* mismatches,
                                              uint32_t* example, void* stream) {
  NV_REQUIRE(mismatches && example, NVFP4_ERR_INVALID_ARG, "nvfp4_test_e2m1_sweep: bad arguments");
  NV_REQUIRE(count <= (1ull << 32) && (uint64_t)first + count <= (1ull << 32), NVFP4_ERR_INVALID_ARG,
             "nvfp4_test_e2m1_sweep: range beyond 2^32");
  int sms = 0;
  NV_CHECK(device_sm_count(&sms));
  if (count == 0) return NVFP4_OK;
  test_e2m1_sweep_kernel<<<sms * 8, 256, 0, as_stream(stream)>>>(first, count, mismatches, example);
  return check_launch("test_e2m1_sweep_kernel");
}

extern "C" nvfp4_status nvfp4_test_e4m3(const float* s, int n, uint8_t* codes, float* value, void* stream) {
  NV_REQUIRE(s && codes && value && n >= 0, NVFP4_ERR_INVALID_ARG, "nvfp4_test_e4m3: bad arguments");
  int sms = 0;
  NV_CHECK(device_sm_count(&sms));
  if (n == 0) return NVFP4_OK;
  test_e4m3_kernel<<<(n + 255) / 256, 256, 0, as_stream(stream)>>>(s, n, codes, value);
  return check_launch("test_e4m3_kernel");
}

extern "C" nvfp4_status nvfp4_test_sigmoid(const float* l, int n, float* out, void* stream) {
  NV_REQUIRE(l && out && n >= 0, NVFP4_ERR_INVALID_ARG, "nvfp4_test_sigmoid: bad arguments");
  int sms = 0;
  NV_CHECK(device_sm_count(&sms));
  if (n == 0) return NVFP4_OK;
  test_sigmoid_kernel<<<(n + 255) / 256, 256, 0, as_stream(stream)>>>(l, n, out);
  return check_launch("test_sigmoid_kernel");
}

extern "C" nvfp4_status nvfp4_test_wait_timeout(const void* src, uint64_t limit_ns, void* ws, size_t ws_bytes,
                                                unsigned long long* elapsed_ns, uint32_t* copied, void* stream) {
  NV_REQUIRE(src && ws && elapsed_ns && copied, NVFP4_ERR_INVALID_ARG, "nvfp4_test_wait_timeout: a pointer is NULL");
  NV_REQUIRE(limit_ns > 0 && limit_ns <= 1000000000ull, NVFP4_ERR_INVALID_ARG,
             "nvfp4_test_wait_timeout: limit_ns=%llu must be in (0, 1e9]", (unsigned long long)limit_ns);
  NV_REQUIRE(ws_bytes >= 256 && aligned(ws, 256) && aligned(src, 16), NVFP4_ERR_WORKSPACE,
             "nvfp4_test_wait_timeout: needs a 256-byte aligned workspace of at least 256 bytes and a 16-byte "
             "aligned source");
  int sms = 0;
  NV_CHECK(device_sm_count(&sms));
  cudaStream_t s = as_stream(stream);
  test_wait_timeout_kernel<<<1, 64, 0, s>>>(static_cast<const uint4*>(src), limit_ns, static_cast<uint32_t*>(ws),
                                            elapsed_ns, copied);
  return check_launch("test_wait_timeout_kernel");
}

extern "C" nvfp4_status nvfp4_test_block_scale_div(const float* amax, const float* g, int n, float* q_lib,
                                                   float* q_ieee, uint8_t* code_lib, uint8_t* code_ieee,
                                                   void* stream) {
  NV_REQUIRE(amax && g && q_lib && q_ieee && code_lib && code_ieee && n >= 0, NVFP4_ERR_INVALID_ARG,
             "nvfp4_test_block_scale_div: bad argument");
  if (n == 0) return NVFP4_OK;
  test_block_scale_div_kernel<<<(n + 255) / 256, 256, 0, as_stream(stream)>>>(amax, g, n, q_lib, q_ieee, code_lib,
                                                                              code_ieee);
  return check_launch("test_block_scale_div_kernel");
}

extern "C" int nvfp4_test_router_splits(int T, int H, int* stages_per_split) {
  if (T < 1 || H <= 0 || H % 64 != 0) return -1;
  const int splits = nvfp4moe::router_splits(T, H);
  if (stages_per_split) *stages_per_split = (H / 64 + splits - 1) / splits;
  return splits;
}
