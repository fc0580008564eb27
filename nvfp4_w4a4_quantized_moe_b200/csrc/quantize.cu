// NVFP4 quantisers: the dynamic activation quantiser and the offline RTN
// weight quantiser ("K-EXAONE-152B-A23B-REAP-80E-NVFP4" model card, section
// "Quantization Setup").  Both are HBM-bound streams: 128-bit loads of bf16,
// 64-bit stores of packed codes, one scale byte per 16 elements.
#include <mutex>

#include "common.cuh"
#include "host.cuh"

namespace nvfp4moe {

// Writes the scale codes of 16-element blocks kb .. kb+nb-1 of `row`.  In the
// tiled layout four consecutive blocks of a row form one 32-bit word, so the
// lanes holding a group of four combine their bytes with shuffles first.
// Requires every lane of the warp to call it (inactive lanes pass valid=false).
template <int NB>
NVDEV void store_scales(uint8_t* scales, int layout, int row, int kb, int nblk, const uint32_t* s, bool valid) {
  if (layout == NVFP4_LAYOUT_CANONICAL) {
    if (!valid) return;
    uint8_t* p = scales + (size_t)row * nblk + kb;
    if (NB == 1) {
      p[0] = (uint8_t)s[0];
    } else {
      *reinterpret_cast<uint16_t*>(p) = (uint16_t)(s[0] | (s[1] << 8));
    }
    return;
  }
  // tiled: NB == 1 -> groups of 4 lanes; NB == 2 -> groups of 2 lanes
  const int lane = threadIdx.x & 31;
  uint32_t word = (NB == 1) ? s[0] : (s[0] | (s[1] << 8));
  if (NB == 1) {
    uint32_t w1 = __shfl_down_sync(0xffffffffu, word, 1);
    uint32_t w2 = __shfl_down_sync(0xffffffffu, word, 2);
    uint32_t w3 = __shfl_down_sync(0xffffffffu, word, 3);
    word = word | (w1 << 8) | (w2 << 16) | (w3 << 24);
    if (!valid || (lane & 3)) return;
  } else {
    uint32_t w1 = __shfl_down_sync(0xffffffffu, word, 1);
    word = word | (w1 << 16);
    if (!valid || (lane & 1)) return;
  }
  *reinterpret_cast<uint32_t*>(scales + tiled_scale_offset(row, kb, nblk >> 2)) = word;
}

// ---------------------------------------------------------------------------
// Activations: one thread per 16-element block, a warp covers 1 KiB of bf16.
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(256) quantize_act_kernel(const uint4* __restrict__ x, int rows, int cols,
                                                          const float* __restrict__ gscale, int layout,
                                                          uint2* __restrict__ codes, uint8_t* __restrict__ scales) {
  const float g = *gscale;
  const float d = __fmul_rn(6.0f, g);
  const int nblk = cols / kQBlock;
  const long long total = (long long)rows * nblk;
  const long long stride = (long long)gridDim.x * blockDim.x;
  // every lane iterates the same number of times so shuffles stay converged
  const long long iters = (total + stride - 1) / stride;
  long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  for (long long it = 0; it < iters; ++it, i += stride) {
    const bool valid = i < total;
    uint32_t s = 0;
    int row = 0, kb = 0;
    if (valid) {
      row = (int)(i / nblk);
      kb = (int)(i % nblk);
      const uint4 u0 = __ldg(x + i * 2), u1 = __ldg(x + i * 2 + 1);
      uint2 c;
      s = quant_block16_bf16(u0, u1, g, d, c);
      codes[i] = c;
    }
    store_scales<1>(scales, layout, row, kb, nblk, &s, valid);
  }
}

// Zero scale rows [rows, padded_rows) of a tiled scale buffer.
__global__ void zero_tiled_scale_rows(uint8_t* scales, int rows, int padded_rows, int nblk) {
  const long long total = (long long)(padded_rows - rows) * nblk;
  for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < total;
       i += (long long)gridDim.x * blockDim.x) {
    const int row = rows + (int)(i / nblk), kb = (int)(i % nblk);
    scales[tiled_scale_offset(row, kb, nblk >> 2)] = 0;
  }
}

// ---------------------------------------------------------------------------
// Weights: one cooperative launch (every CTA resident).  Each CTA owns an
// even share of every matrix and splits its warps in two groups that run side
// by side:
//   * amax warps stream matrix after matrix, publish one atomic max and one
//     completion count per matrix, and stay at most two matrices ahead of
//     their own CTA's quantise warps (so the matrices in flight fit in L2);
//   * quantise warps take matrix m once every CTA has published its amax
//     (a bounded wait), re-read their share (from L2: the amax pass asked L2
//     to keep the lines, this pass lets them go) and write codes and scales.
// Waits only ever point at earlier matrices, so with all CTAs resident they
// always end.
// ---------------------------------------------------------------------------
constexpr int kWAmax = 256;                     // amax threads per CTA (the DRAM stream)
constexpr int kWQuant = 256;                    // quantise threads per CTA (re-read from L2)
constexpr int kWThreads = kWAmax + kWQuant;
constexpr int kWAhead = 1;                      // amax may lead quantise by this many matrices

struct WeightQuantState {
  uint32_t status;          // device status word (first word of the workspace)
  uint32_t pad[63];
  // followed by amax_bits[n_mats], done[n_mats]
};

NVDEV uint32_t ld_acquire_u32(const uint32_t* p) {
  uint32_t v;
  asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}
NVDEV uint64_t l2_policy_evict_last() {
  uint64_t pol;
  asm volatile("createpolicy.fractional.L2::evict_last.b64 %0, 1.0;" : "=l"(pol));
  return pol;
}
NVDEV uint64_t l2_policy_evict_first() {
  uint64_t pol;
  asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(pol));
  return pol;
}
NVDEV uint4 ld_hint(const uint4* p, uint64_t pol) {
  uint4 v;
  asm volatile("ld.global.nc.L2::cache_hint.v4.u32 {%0, %1, %2, %3}, [%4], %5;"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p), "l"(pol));
  return v;
}
template <int N>
NVDEV void group_sync(int id) { asm volatile("bar.sync %0, %1;" ::"r"(id), "n"(N) : "memory"); }

__global__ void __launch_bounds__(kWThreads) quantize_weights_kernel(
    const uint4* __restrict__ w, int n_mats, int rows, int cols, int layout, uint2* __restrict__ codes,
    uint8_t* __restrict__ scales, float* __restrict__ gscale, WeightQuantState* st, uint32_t* amax_bits,
    uint32_t* done) {
  __shared__ uint32_t s_red[kWAmax / 32];
  __shared__ int s_ok_amax, s_ok_quant;
  __shared__ volatile int quantised;            // matrices this CTA's quantise warps have finished
  __shared__ volatile int failed;
  const long long per_mat = (long long)rows * cols;
  const long long blocks = per_mat / kQBlock;                  // 16-element blocks per matrix
  const int nblk = cols / kQBlock;
  const int lane = threadIdx.x & 31;
  const int gt = threadIdx.x < kWAmax ? threadIdx.x : threadIdx.x - kWAmax;   // index within its group
  // this CTA's share of every matrix, in whole groups of 4 blocks
  const long long share = ((blocks + gridDim.x - 1) / gridDim.x + 3) / 4 * 4;
  const long long b_begin = min(blocks, share * blockIdx.x), b_end = min(blocks, b_begin + share);
  if (threadIdx.x == 0) {
    quantised = 0;
    failed = 0;
  }
  __syncthreads();

  if (threadIdx.x < kWAmax) {
    // ------------------------------------------------------------ amax warps
    const uint64_t keep = l2_policy_evict_last();
    for (int mat = 0; mat < n_mats; ++mat) {
      if (gt == 0) {
        const uint64_t t0 = globaltimer_ns();
        while (quantised < mat - kWAhead && !failed) {
          if (globaltimer_ns() - t0 > kWaitLimitNs) {
            failed = 1;
            atomicExch(&st->status, kDevTimeout);
          }
        }
        s_ok_amax = !failed;
      }
      group_sync<kWAmax>(1);
      if (!s_ok_amax) break;
      const uint4* src = w + (long long)mat * per_mat / 8;
      const long long v1 = b_end * 2;                          // uint4 range (8 bf16 each)
      // running max of |x| on packed bf16 pairs (exact)
      __nv_bfloat162 m2 = __floats2bfloat162_rn(0.0f, 0.0f);
      auto absmax4 = [&](const uint4& u) {
        const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
        for (int j = 0; j < 4; ++j) m2 = __hmax2(m2, __habs2(*reinterpret_cast<const __nv_bfloat162*>(&w[j])));
      };
      long long i = b_begin * 2 + gt;
      for (; i + 7 * kWAmax < v1; i += 8 * kWAmax) {
        uint4 u[8];
#pragma unroll
        for (int q = 0; q < 8; ++q) u[q] = ld_hint(src + i + q * kWAmax, keep);
#pragma unroll
        for (int q = 0; q < 8; ++q) absmax4(u[q]);
      }
      for (; i < v1; i += kWAmax) absmax4(ld_hint(src + i, keep));
      const float m = fmaxf(__low2float(m2), __high2float(m2));
      uint32_t mb = __float_as_uint(m);
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) mb = max(mb, __shfl_xor_sync(0xffffffffu, mb, o));
      if (lane == 0) s_red[gt >> 5] = mb;
      group_sync<kWAmax>(1);
      if (gt == 0) {
        uint32_t bm = 0;
        for (int q = 0; q < kWAmax / 32; ++q) bm = max(bm, s_red[q]);
        atomicMax(amax_bits + mat, bm);         // non-negative floats order like their bits
        __threadfence();
        atomicAdd(done + mat, 1u);
      }
    }
  } else {
    // ------------------------------------------------------------ quantise warps
    const uint64_t drop = l2_policy_evict_first();
    for (int mat = 0; mat < n_mats; ++mat) {
      if (gt == 0) {
        int ok = 1;
        if (ld_acquire_u32(done + mat) < gridDim.x) {
          const uint64_t t0 = globaltimer_ns();
          while (ld_acquire_u32(done + mat) < gridDim.x) {
            if (failed || globaltimer_ns() - t0 > kWaitLimitNs) {
              ok = 0;
              failed = 1;
              atomicExch(&st->status, kDevTimeout);
              break;
            }
          }
        }
        s_ok_quant = ok;
      }
      group_sync<kWQuant>(2);
      if (!s_ok_quant) break;
      const float amax = __uint_as_float(ld_acquire_u32(amax_bits + mat));
      const float g = __fdiv_rn(amax, 2688.0f);
      const float d = __fmul_rn(6.0f, g);
      if (blockIdx.x == 0 && gt == 0) gscale[mat] = g;
      const uint4* src = w + (long long)mat * per_mat / 8;
      const float inv_nblk = 1.0f / (float)nblk;
      // every lane of a warp runs the same number of iterations (shuffles
      // below); each iteration has two blocks per thread in flight
      const long long n_iter = (b_end - b_begin + 2 * kWQuant - 1) / (2 * kWQuant);
      for (long long it = 0; it < n_iter; ++it) {
        uint4 u[2][2];
        bool valid[2];
        long long b[2];
#pragma unroll
        for (int q = 0; q < 2; ++q) {
          b[q] = b_begin + (2 * it + q) * kWQuant + gt;
          valid[q] = b[q] < b_end;
          if (valid[q]) {
            u[q][0] = ld_hint(src + 2 * b[q], drop);
            u[q][1] = ld_hint(src + 2 * b[q] + 1, drop);
          }
        }
#pragma unroll
        for (int q = 0; q < 2; ++q) {
          uint32_t sc = 0;
          int row = 0, kb = 0;
          if (valid[q]) {
            uint2 c;
            sc = quant_block16_bf16(u[q][0], u[q][1], g, d, c);
            codes[(long long)mat * blocks + b[q]] = c;
            // b < 2^24 (checked on the host): a float quotient off by at most
            // one, then an exact integer correction
            const uint32_t bb = (uint32_t)b[q];
            uint32_t qt = (uint32_t)__fmul_rz((float)bb, inv_nblk);
            int32_t rem = (int32_t)(bb - qt * (uint32_t)nblk);
            if (rem < 0) { --qt; rem += nblk; }
            if (rem >= nblk) { ++qt; rem -= nblk; }
            row = (int)qt;
            kb = rem;
          }
          store_scales<1>(scales, layout, mat * rows + row, kb, nblk, &sc, valid[q]);
        }
      }
      group_sync<kWQuant>(2);
      if (gt == 0) quantised = mat + 1;
    }
  }
  __syncthreads();
}

// Cooperative launch: the phases need every CTA resident at once.
static nvfp4_status launch_weight_quantiser(const void* w_bf16, int n_mats, int rows, int cols, int layout,
                                           uint8_t* codes, uint8_t* scales, float* global_scale,
                                           WeightQuantState* st, uint32_t* amax, uint32_t* done, int sms,
                                           cudaStream_t s) {
  int per_sm = 0;
  NV_CHECK(check_cuda(cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, quantize_weights_kernel, kWThreads, 0),
                      "occupancy"));
  per_sm = std::max(1, std::min(per_sm, 2));
  const uint4* w = static_cast<const uint4*>(w_bf16);
  uint2* c = reinterpret_cast<uint2*>(codes);
  void* args[] = {(void*)&w, (void*)&n_mats, (void*)&rows, (void*)&cols, (void*)&layout, (void*)&c,
                  (void*)&scales, (void*)&global_scale, (void*)&st, (void*)&amax, (void*)&done};
  return check_cuda(cudaLaunchCooperativeKernel((const void*)quantize_weights_kernel, dim3(sms * per_sm),
                                                dim3(kWThreads), args, 0, s),
                    "cudaLaunchCooperativeKernel(quantize_weights_kernel)");
}

}  // namespace nvfp4moe

using namespace nvfp4moe;

extern "C" nvfp4_status nvfp4_quantize_act(const void* x_bf16, int rows, int cols, const float* global_scale,
                                           int layout, uint8_t* codes, uint8_t* scales, void* stream) {
  NV_REQUIRE(x_bf16 && global_scale && codes && scales, NVFP4_ERR_INVALID_ARG,
             "nvfp4_quantize_act: a pointer argument is NULL");
  NV_REQUIRE(rows >= 0 && cols > 0, NVFP4_ERR_INVALID_ARG, "nvfp4_quantize_act: rows=%d cols=%d", rows, cols);
  NV_REQUIRE(layout == NVFP4_LAYOUT_CANONICAL || layout == NVFP4_LAYOUT_TILED, NVFP4_ERR_INVALID_ARG,
             "nvfp4_quantize_act: unknown layout %d", layout);
  NV_REQUIRE(cols % 32 == 0 && (layout == NVFP4_LAYOUT_CANONICAL || cols % 64 == 0), NVFP4_ERR_UNSUPPORTED_SHAPE,
             "nvfp4_quantize_act: cols=%d must be a multiple of 32 (64 for the tiled layout)", cols);
  NV_REQUIRE(aligned(x_bf16, 16) && aligned(codes, 16) && aligned(scales, 4), NVFP4_ERR_INVALID_ARG,
             "nvfp4_quantize_act: x and codes need 16-byte alignment, scales 4-byte");
  int sms = 0;
  NV_CHECK(device_sm_count(&sms));
  cudaStream_t s = as_stream(stream);
  const long long blocks_needed = ((long long)rows * (cols / 16) + 255) / 256;
  if (blocks_needed > 0) {
    const int grid = (int)std::min<long long>(blocks_needed, (long long)sms * 16);
    quantize_act_kernel<<<grid, 256, 0, s>>>(static_cast<const uint4*>(x_bf16), rows, cols, global_scale, layout,
                                             reinterpret_cast<uint2*>(codes), scales);
    NV_CHECK(check_launch("quantize_act_kernel"));
  }
  if (layout == NVFP4_LAYOUT_TILED) {
    const int padded = (rows + 127) / 128 * 128;
    if (padded > rows) {
      zero_tiled_scale_rows<<<16, 256, 0, s>>>(scales, rows, padded, cols / 16);
      NV_CHECK(check_launch("zero_tiled_scale_rows"));
    }
  }
  return NVFP4_OK;
}

extern "C" size_t nvfp4_quantize_weights_workspace_size(int n_mats) {
  if (n_mats < 0) return 0;
  Carver c(nullptr);
  c.take<WeightQuantState>(1);
  c.take<uint32_t>((size_t)n_mats);
  c.take<uint32_t>((size_t)n_mats);
  return c.size();
}

extern "C" nvfp4_status nvfp4_quantize_weights(const void* w_bf16, int n_mats, int rows, int cols, int layout,
                                               uint8_t* codes, uint8_t* scales, float* global_scale, void* ws,
                                               size_t ws_bytes, void* stream) {
  NV_REQUIRE(w_bf16 && codes && scales && global_scale, NVFP4_ERR_INVALID_ARG,
             "nvfp4_quantize_weights: a pointer argument is NULL");
  NV_REQUIRE(n_mats >= 0 && rows >= 0 && cols > 0, NVFP4_ERR_INVALID_ARG,
             "nvfp4_quantize_weights: n_mats=%d rows=%d cols=%d", n_mats, rows, cols);
  NV_REQUIRE(layout == NVFP4_LAYOUT_CANONICAL || layout == NVFP4_LAYOUT_TILED, NVFP4_ERR_INVALID_ARG,
             "nvfp4_quantize_weights: unknown layout %d", layout);
  NV_REQUIRE(cols % 32 == 0, NVFP4_ERR_UNSUPPORTED_SHAPE, "nvfp4_quantize_weights: cols=%d must be a multiple of 32",
             cols);
  NV_REQUIRE(layout == NVFP4_LAYOUT_CANONICAL || (cols % 64 == 0 && rows % 128 == 0), NVFP4_ERR_UNSUPPORTED_SHAPE,
             "nvfp4_quantize_weights: the tiled layout needs rows %% 128 == 0 and cols %% 64 == 0 (got %d x %d)", rows,
             cols);
  NV_REQUIRE((long long)rows * cols / 16 < (1ll << 24) && n_mats < (1 << 24),
             NVFP4_ERR_UNSUPPORTED_SHAPE, "nvfp4_quantize_weights: too many elements");
  const size_t need = nvfp4_quantize_weights_workspace_size(n_mats);
  NV_REQUIRE(ws != nullptr && ws_bytes >= need && aligned(ws, 256), NVFP4_ERR_WORKSPACE,
             "nvfp4_quantize_weights: needs a 256-byte aligned workspace of %zu bytes", need);
  NV_REQUIRE(aligned(w_bf16, 16) && aligned(codes, 16) && aligned(scales, 4), NVFP4_ERR_INVALID_ARG,
             "nvfp4_quantize_weights: w and codes need 16-byte alignment, scales 4-byte");
  if (n_mats == 0 || rows == 0) return NVFP4_OK;
  int sms = 0;
  NV_CHECK(device_sm_count(&sms));
  cudaStream_t s = as_stream(stream);
  Carver c(ws);
  WeightQuantState* st = c.take<WeightQuantState>(1);
  uint32_t* amax = c.take<uint32_t>((size_t)n_mats);
  uint32_t* done = c.take<uint32_t>((size_t)n_mats);
  NV_CHECK(check_cuda(cudaMemsetAsync(ws, 0, need, s), "cudaMemsetAsync(workspace)"));
  return launch_weight_quantiser(w_bf16, n_mats, rows, cols, layout, codes, scales, global_scale, st, amax, done,
                                 sms, s);
}

namespace nvfp4moe {

// ---------------------------------------------------------------------------
// Weight quantiser for callers that cannot allocate device memory.
//
// Some hosts of this library cannot hand it a workspace: the process's device
// memory belongs to another allocator (a serving engine's arena, a plugin
// host's fixed pool) that the caller has no way to draw an extra buffer from,
// or the caller runs where device allocation calls are not permitted.  This
// entry point needs no workspace: the quantiser's scratch (work-queue head,
// status word, per-matrix amax and completion counters) lives in the array
// below, which every GPU that loads the library holds until the process
// exits.
// ---------------------------------------------------------------------------
constexpr int kStaticMaxMats = 1024;
constexpr size_t kStaticScratchBytes = 256 + 2 * 4 * kStaticMaxMats;   // state, amax[], done[]

static __device__ __align__(256) uint8_t g_weight_quant_scratch[kStaticScratchBytes];

// Device address of the scratch array, looked up once per device (the host
// symbol is only a stand-in and must never be passed to a kernel).
static nvfp4_status static_scratch_address(uint8_t** out) {
  static std::mutex mu;
  static uint8_t* addr[64] = {};
  int dev = 0;
  NV_CHECK(check_cuda(cudaGetDevice(&dev), "cudaGetDevice"));
  NV_REQUIRE(dev >= 0 && dev < 64, NVFP4_ERR_DEVICE, "device index %d out of range", dev);
  std::lock_guard<std::mutex> lock(mu);
  if (!addr[dev]) {
    void* p = nullptr;
    NV_CHECK(check_cuda(cudaGetSymbolAddress(&p, g_weight_quant_scratch), "cudaGetSymbolAddress"));
    addr[dev] = static_cast<uint8_t*>(p);
  }
  *out = addr[dev];
  return NVFP4_OK;
}

}  // namespace nvfp4moe

extern "C" nvfp4_status nvfp4_quantize_weights_noalloc(const void* w_bf16, int n_mats, int rows, int cols,
                                                       int layout, uint8_t* codes, uint8_t* scales,
                                                       float* global_scale, void* stream) {
  using namespace nvfp4moe;
  NV_REQUIRE(w_bf16 && codes && scales && global_scale, NVFP4_ERR_INVALID_ARG,
             "nvfp4_quantize_weights_noalloc: a pointer argument is NULL");
  NV_REQUIRE(n_mats >= 0 && rows >= 0 && cols > 0, NVFP4_ERR_INVALID_ARG,
             "nvfp4_quantize_weights_noalloc: n_mats=%d rows=%d cols=%d", n_mats, rows, cols);
  NV_REQUIRE(n_mats <= kStaticMaxMats, NVFP4_ERR_UNSUPPORTED_SHAPE,
             "nvfp4_quantize_weights_noalloc: n_mats=%d exceeds the built-in scratch limit of %d matrices per call "
             "(use nvfp4_quantize_weights with a workspace, or split the call)",
             n_mats, kStaticMaxMats);
  NV_REQUIRE(layout == NVFP4_LAYOUT_CANONICAL || layout == NVFP4_LAYOUT_TILED, NVFP4_ERR_INVALID_ARG,
             "nvfp4_quantize_weights_noalloc: unknown layout %d", layout);
  NV_REQUIRE(cols % 32 == 0, NVFP4_ERR_UNSUPPORTED_SHAPE,
             "nvfp4_quantize_weights_noalloc: cols=%d must be a multiple of 32", cols);
  NV_REQUIRE(layout == NVFP4_LAYOUT_CANONICAL || (cols % 64 == 0 && rows % 128 == 0), NVFP4_ERR_UNSUPPORTED_SHAPE,
             "nvfp4_quantize_weights_noalloc: the tiled layout needs rows %% 128 == 0 and cols %% 64 == 0");
  NV_REQUIRE((long long)rows * cols / 16 < (1ll << 24) && n_mats < (1 << 24),
             NVFP4_ERR_UNSUPPORTED_SHAPE, "nvfp4_quantize_weights_noalloc: too many elements");
  NV_REQUIRE(aligned(w_bf16, 16) && aligned(codes, 16) && aligned(scales, 4), NVFP4_ERR_INVALID_ARG,
             "nvfp4_quantize_weights_noalloc: w and codes need 16-byte alignment, scales 4-byte");
  if (n_mats == 0 || rows == 0) return NVFP4_OK;
  int sms = 0;
  NV_CHECK(device_sm_count(&sms));
  uint8_t* scratch = nullptr;
  NV_CHECK(static_scratch_address(&scratch));
  cudaStream_t s = as_stream(stream);
  // the array keeps the previous call's contents: clear the queue head, the
  // status word and the per-matrix amax and counters this call uses
  Carver c(scratch);
  WeightQuantState* st = c.take<WeightQuantState>(1);
  uint32_t* amax = c.take<uint32_t>((size_t)n_mats);
  uint32_t* done = c.take<uint32_t>((size_t)n_mats);
  NV_CHECK(check_cuda(cudaMemsetAsync(scratch, 0, c.size(), s), "cudaMemsetAsync(static scratch)"));
  return launch_weight_quantiser(w_bf16, n_mats, rows, cols, layout, codes, scales, global_scale, st, amax, done,
                                 sms, s);
}
