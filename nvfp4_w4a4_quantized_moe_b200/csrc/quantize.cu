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
      float v[16];
      const uint4 u0 = __ldg(x + i * 2), u1 = __ldg(x + i * 2 + 1);
      unpack_bf16x8(u0, v);
      unpack_bf16x8(u1, v + 8);
      uint2 c;
      s = quant_block16(v, g, d, c);
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
// Weights: a persistent kernel walking a queue of 32768-element items.  The
// queue interleaves the amax pass of matrix m+1 with the quantise pass of
// matrix m, so the second read of a matrix finds it in L2 (the first read
// asks L2 to keep the lines, the second lets them go).  A quantise item waits
// (bounded) until every amax item of its matrix has finished; those items
// were taken from the queue earlier by running blocks, so the wait always
// ends.  Each thread owns 4 x 32 consecutive elements of an item and issues
// all of its loads before it waits or computes.
// ---------------------------------------------------------------------------
constexpr int kWThreads = 256;
constexpr int kWPerThread = 32;                       // two 16-element blocks
constexpr int kWSub = 4;                              // sub-chunks per item
constexpr int kWSubElems = kWThreads * kWPerThread;   // 8192
constexpr int kWItem = kWSub * kWSubElems;            // 32768 elements

struct WeightQuantState {
  uint32_t status;          // device status word (first word of the workspace)
  uint32_t next_item;       // queue head
  uint32_t pad[62];
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

__global__ void __launch_bounds__(kWThreads) quantize_weights_kernel(
    const uint4* __restrict__ w, int n_mats, int rows, int cols, int layout, uint2* __restrict__ codes,
    uint8_t* __restrict__ scales, float* __restrict__ gscale, WeightQuantState* st, uint32_t* amax_bits,
    uint32_t* done) {
  __shared__ uint32_t s_item;
  __shared__ uint32_t s_red[kWThreads / 32];
  __shared__ int s_fail;
  const long long per_mat = (long long)rows * cols;
  const uint32_t chunks = (uint32_t)((per_mat + kWItem - 1) / kWItem);
  const uint32_t total_items = 2u * chunks * (uint32_t)n_mats;
  const int nblk = cols / kQBlock;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const uint64_t keep = l2_policy_evict_last(), drop = l2_policy_evict_first();

  for (;;) {
    if (threadIdx.x == 0) {
      s_item = atomicAdd(&st->next_item, 1u);
      s_fail = 0;
    }
    __syncthreads();
    const uint32_t item = s_item;
    if (item >= total_items) break;
    // decode the queue position: step 0 = amax(0); step s = amax(s), quant(s-1)
    bool is_amax;
    uint32_t mat, chunk;
    if (item < chunks) {
      is_amax = true; mat = 0; chunk = item;
    } else {
      const uint32_t j = item - chunks, step = 1 + j / (2 * chunks), r = j % (2 * chunks);
      if (step < (uint32_t)n_mats) {
        is_amax = r < chunks; mat = is_amax ? step : step - 1; chunk = is_amax ? r : r - chunks;
      } else {
        is_amax = false; mat = n_mats - 1; chunk = r;
      }
    }
    // element offsets of this thread's four 32-element runs
    long long e0[kWSub];
    bool valid[kWSub];
    uint4 raw[kWSub][4];
#pragma unroll
    for (int q = 0; q < kWSub; ++q) {
      e0[q] = (long long)chunk * kWItem + (long long)q * kWSubElems + (long long)threadIdx.x * kWPerThread;
      valid[q] = e0[q] < per_mat;
      const uint4* src = w + ((long long)mat * per_mat + e0[q]) / 8;
#pragma unroll
      for (int i = 0; i < 4; ++i)
        raw[q][i] = valid[q] ? ld_hint(src + i, is_amax ? keep : drop) : make_uint4(0, 0, 0, 0);
    }
    if (is_amax) {
      float m = 0.0f;
#pragma unroll
      for (int q = 0; q < kWSub; ++q)
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          float v[8];
          unpack_bf16x8(raw[q][i], v);
#pragma unroll
          for (int j = 0; j < 8; ++j) m = fmaxf(m, fabsf(v[j]));
        }
      uint32_t mb = __float_as_uint(m);
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) mb = max(mb, __shfl_xor_sync(0xffffffffu, mb, o));
      if (lane == 0) s_red[warp] = mb;
      __syncthreads();
      if (threadIdx.x == 0) {
        uint32_t bm = 0;
        for (int q = 0; q < kWThreads / 32; ++q) bm = max(bm, s_red[q]);
        atomicMax(amax_bits + mat, bm);     // non-negative floats order like their bits
        __threadfence();
        atomicAdd(done + mat, 1u);
      }
    } else {
      if (threadIdx.x == 0) {
        if (ld_acquire_u32(done + mat) < chunks) {
          const uint64_t t0 = globaltimer_ns();
          while (ld_acquire_u32(done + mat) < chunks) {
            if (globaltimer_ns() - t0 > kWaitLimitNs) {
              atomicExch(&st->status, kDevTimeout);
              s_fail = 1;
              break;
            }
          }
        }
      }
      __syncthreads();
      if (s_fail) break;
      const float amax = __uint_as_float(ld_acquire_u32(amax_bits + mat));
      const float g = __fdiv_rn(amax, 2688.0f);
      const float d = __fmul_rn(6.0f, g);
      if (chunk == 0 && threadIdx.x == 0) gscale[mat] = g;
#pragma unroll
      for (int q = 0; q < kWSub; ++q) {
        uint32_t s[2] = {0, 0};
        int row = 0, kb = 0;
        if (valid[q]) {
          float v[32];
#pragma unroll
          for (int i = 0; i < 4; ++i) unpack_bf16x8(raw[q][i], v + 8 * i);
          row = (int)(e0[q] / cols);
          kb = (int)((e0[q] % cols) / kQBlock);
          uint2 c0, c1;
          s[0] = quant_block16(v, g, d, c0);
          s[1] = quant_block16(v + 16, g, d, c1);
          *reinterpret_cast<uint4*>(codes + ((long long)mat * per_mat + e0[q]) / 16) =
              make_uint4(c0.x, c0.y, c1.x, c1.y);
        }
        store_scales<2>(scales, layout, mat * rows + row, kb, nblk, s, valid[q]);
      }
    }
    __syncthreads();
  }
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
  NV_REQUIRE((long long)n_mats * 2 * ((long long)rows * cols / 32768 + 1) < (1ll << 32),
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
  int per_sm = 0;
  NV_CHECK(check_cuda(cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, quantize_weights_kernel, kWThreads, 0),
                      "occupancy"));
  per_sm = per_sm < 1 ? 1 : per_sm;
  quantize_weights_kernel<<<sms * per_sm, kWThreads, 0, s>>>(static_cast<const uint4*>(w_bf16), n_mats, rows, cols,
                                                             layout, reinterpret_cast<uint2*>(codes), scales,
                                                             global_scale, st, amax, done);
  return check_launch("quantize_weights_kernel");
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
  NV_REQUIRE((long long)n_mats * 2 * ((long long)rows * cols / 32768 + 1) < (1ll << 32),
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
  int per_sm = 0;
  NV_CHECK(check_cuda(cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, quantize_weights_kernel, kWThreads, 0),
                      "occupancy"));
  per_sm = per_sm < 1 ? 1 : per_sm;
  quantize_weights_kernel<<<sms * per_sm, kWThreads, 0, s>>>(static_cast<const uint4*>(w_bf16), n_mats, rows, cols,
                                                             layout, reinterpret_cast<uint2*>(codes), scales,
                                                             global_scale, st, amax, done);
  return check_launch("quantize_weights_kernel");
}
