// Block-scale distortion statistics of NVFP4 tensors (the NetsPresso AQ
// article, section "Why 4-Bit Quantization of MoE Models Is Hard: Outliers in
// the Final Two Layers": the share of weights above 0.1 in magnitude, and how
// concentrated outliers distort the block scale and the other weights of
// their block).
//
// One thread per 16-element block: it reads the block's 32 bytes of bf16, its
// 8 bytes of codes and its scale byte, dequantises with the hardware E2M1 and
// E4M3 conversions, and classifies every element.  A block's squared errors
// and magnitudes are summed in fp32 (16 terms), the blocks in fp64.  Each
// CTA reduces its counts and sums in shared memory and adds them to the
// matrix's entry with one atomic per field: the counts are exact, the sums
// within about 1e-6 relative.  2.5625 bytes read per element.
#include "common.cuh"
#include "host.cuh"

namespace nvfp4moe {

constexpr int kDThreads = 256;
constexpr int kDInts = 9, kDDoubles = 6;

// E2M1 codes of one byte -> the two values (hardware conversion).
NVDEV void e2m1x2_values(uint32_t byte, float& lo, float& hi) {
  uint32_t h2;
  const uint16_t in = (uint16_t)(byte & 0xFFu);
  asm("{\n\t.reg .b8 t;\n\tcvt.u8.u16 t, %1;\n\tcvt.rn.f16x2.e2m1x2 %0, t;\n\t}" : "=r"(h2) : "h"(in));
  lo = __half2float(__ushort_as_half((unsigned short)(h2 & 0xFFFFu)));
  hi = __half2float(__ushort_as_half((unsigned short)(h2 >> 16)));
}

__global__ void __launch_bounds__(kDThreads) block_stats_kernel(const uint4* __restrict__ w,
                                                                const uint2* __restrict__ codes,
                                                                const uint8_t* __restrict__ scales,
                                                                const float* __restrict__ gscale, int rows, int cols,
                                                                int layout, float tau,
                                                                nvfp4_block_stats* __restrict__ stats) {
  const int mat = blockIdx.y;
  const long long blocks = (long long)rows * cols / kQBlock;
  const int nblk = cols / kQBlock;
  const float g = gscale[mat];
  uint32_t cnt[kDInts] = {0, 0, 0, 0, 0, 0, 0, 0, 0};
  double sum[kDDoubles] = {0, 0, 0, 0, 0, 0};
  auto account = [&](const uint4& u0, const uint4& u1, const uint2& c, uint32_t s) {
    const float sv = e4m3_value(s);
    const float S = __fmul_rn(sv, g);
    const float inv = (S == 0.0f) ? 0.0f : __frcp_rn(S);
    const uint32_t wv[8] = {u0.x, u0.y, u0.z, u0.w, u1.x, u1.y, u1.z, u1.w};
    const uint32_t cv[2] = {c.x, c.y};
    float x[16], dq[16];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      x[2 * i] = __uint_as_float(wv[i] << 16);
      x[2 * i + 1] = __uint_as_float(wv[i] & 0xFFFF0000u);
      float lo, hi;
      e2m1x2_values(cv[i >> 2] >> (8 * (i & 3)), lo, hi);
      dq[2 * i] = __fmul_rn(__fmul_rn(lo, sv), g);
      dq[2 * i + 1] = __fmul_rn(__fmul_rn(hi, sv), g);
    }
    uint32_t out_mask = 0;
#pragma unroll
    for (int i = 0; i < 16; ++i) out_mask |= (fabsf(x[i]) > tau ? 1u : 0u) << i;
    const bool has = out_mask != 0;
    const uint32_t nb_mask = has ? (~out_mask & 0xFFFFu) : 0u;      // neighbours
    float sq = 0.0f, e2 = 0.0f, sq_n = 0.0f, e2_n = 0.0f;
    uint32_t sat = 0;
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      const float e = x[i] - dq[i];
      const float a = x[i] * x[i], ee = e * e;
      sq += a;
      e2 += ee;
      const bool nb = (nb_mask >> i) & 1u;
      sq_n += nb ? a : 0.0f;
      e2_n += nb ? ee : 0.0f;
      sat += fabsf(__fmul_rn(x[i], inv)) > 6.0f ? 1u : 0u;
    }
    const uint32_t n_out = __popc(out_mask);
    cnt[0] += 16;
    cnt[1] += n_out;
    cnt[2] += 1;
    cnt[3] += has ? 1u : 0u;
    cnt[4] += s == 0 ? 1u : 0u;
    cnt[5] += (s >= 1 && s <= 7) ? 1u : 0u;
    cnt[6] += sat;
    cnt[7] += has ? 16u - n_out : 0u;
    cnt[8] += has ? 0u : 16u;
    sum[0] += sq;
    sum[1] += e2;
    sum[2] += sq_n;
    sum[3] += e2_n;
    if (!has) {
      sum[4] += sq;
      sum[5] += e2;
    }
  };
  auto code_unit = [&](long long b) -> size_t {
    if (layout != NVFP4_LAYOUT_STAGED) return (size_t)mat * blocks + b;
    return (size_t)mat * blocks + staged_code_unit((size_t)(b / nblk), (int)(b % nblk), nblk);
  };
  auto scale_of = [&](long long b) -> uint32_t {
    const int row = (int)(b / nblk), kb = (int)(b % nblk);
    const int srow = mat * rows + row;
    return scales[layout == NVFP4_LAYOUT_CANONICAL ? (size_t)srow * nblk + kb
                                                   : tiled_scale_offset(srow, kb, nblk >> 2)];
  };
  // two blocks per thread per iteration, both blocks' loads issued first
  const long long stride = (long long)gridDim.x * blockDim.x;
  for (long long b = (long long)blockIdx.x * blockDim.x + threadIdx.x; b < blocks; b += 2 * stride) {
    const long long b2 = b + stride;
    const bool two = b2 < blocks;
    const long long gb = (long long)mat * blocks + b, gb2 = (long long)mat * blocks + (two ? b2 : b);
    const uint4 u0 = __ldg(w + 2 * gb), u1 = __ldg(w + 2 * gb + 1);
    const uint4 v0 = __ldg(w + 2 * gb2), v1 = __ldg(w + 2 * gb2 + 1);
    const uint2 c = __ldg(codes + code_unit(b)), c2 = __ldg(codes + code_unit(two ? b2 : b));
    const uint32_t s = scale_of(b), s2 = scale_of(two ? b2 : b);
    account(u0, u1, c, s);
    if (two) account(v0, v1, c2, s2);
  }
  // warp, then CTA reduction; one atomic per field per CTA
  __shared__ unsigned long long s_cnt[kDThreads / 32][kDInts];
  __shared__ double s_sum[kDThreads / 32][kDDoubles];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
  for (int f = 0; f < kDInts; ++f) {
    unsigned long long v = cnt[f];
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    if (lane == 0) s_cnt[warp][f] = v;
  }
#pragma unroll
  for (int f = 0; f < kDDoubles; ++f) {
    double v = sum[f];
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    if (lane == 0) s_sum[warp][f] = v;
  }
  __syncthreads();
  if (threadIdx.x < kDInts) {
    unsigned long long v = 0;
    for (int q = 0; q < kDThreads / 32; ++q) v += s_cnt[q][threadIdx.x];
    unsigned long long* dst = reinterpret_cast<unsigned long long*>(&stats[mat].elements) + threadIdx.x;
    if (v) atomicAdd(dst, v);
  } else if (threadIdx.x >= 32 && threadIdx.x < 32 + kDDoubles) {
    const int f = threadIdx.x - 32;
    double v = 0;
    for (int q = 0; q < kDThreads / 32; ++q) v += s_sum[q][f];
    double* dst = &stats[mat].sum_sq + f;
    if (v != 0.0) atomicAdd(dst, v);
  }
}

}  // namespace nvfp4moe

using namespace nvfp4moe;

static_assert(sizeof(nvfp4_block_stats) == 9 * 8 + 6 * 8, "nvfp4_block_stats is 15 packed 8-byte fields");

extern "C" nvfp4_status nvfp4_block_stats_compute(const void* w_bf16, const uint8_t* codes, const uint8_t* scales,
                                                  const float* global_scale, int n_mats, int rows, int cols,
                                                  int layout, float outlier_threshold, nvfp4_block_stats* stats,
                                                  void* stream) {
  NV_REQUIRE(w_bf16 && codes && scales && global_scale && stats, NVFP4_ERR_INVALID_ARG,
             "nvfp4_block_stats_compute: a pointer argument is NULL");
  NV_REQUIRE(n_mats >= 1 && rows >= 1 && cols >= 1, NVFP4_ERR_INVALID_ARG,
             "nvfp4_block_stats_compute: n_mats=%d rows=%d cols=%d", n_mats, rows, cols);
  NV_REQUIRE(layout == NVFP4_LAYOUT_CANONICAL || layout == NVFP4_LAYOUT_TILED || layout == NVFP4_LAYOUT_STAGED,
             NVFP4_ERR_INVALID_ARG, "nvfp4_block_stats_compute: unknown layout %d", layout);
  NV_REQUIRE(cols % 16 == 0 && (layout == NVFP4_LAYOUT_CANONICAL || (cols % 64 == 0 && rows % 128 == 0)) &&
                 (layout != NVFP4_LAYOUT_STAGED || cols % 256 == 0),
             NVFP4_ERR_UNSUPPORTED_SHAPE, "nvfp4_block_stats_compute: cols=%d rows=%d do not fit the layout", cols,
             rows);
  NV_REQUIRE(n_mats <= 65535, NVFP4_ERR_UNSUPPORTED_SHAPE, "nvfp4_block_stats_compute: n_mats=%d > 65535",
             n_mats);
  NV_REQUIRE((long long)n_mats * rows < (1ll << 31), NVFP4_ERR_UNSUPPORTED_SHAPE,
             "nvfp4_block_stats_compute: n_mats * rows too large");
  NV_REQUIRE(aligned(w_bf16, 16) && aligned(codes, 8) && aligned(stats, 8), NVFP4_ERR_INVALID_ARG,
             "nvfp4_block_stats_compute: w needs 16-byte, codes and stats 8-byte alignment");
  int sms = 0;
  NV_CHECK(device_sm_count(&sms));
  cudaStream_t s = as_stream(stream);
  NV_CHECK(check_cuda(cudaMemsetAsync(stats, 0, sizeof(nvfp4_block_stats) * (size_t)n_mats, s), "clear stats"));
  const long long blocks = (long long)rows * cols / kQBlock;
  // enough CTAs in total for several waves of 148 SMs, at most one thread per block
  const long long want = std::max(1ll, (long long)sms * 8 / n_mats);
  const int gx = (int)std::min(want, (blocks + kDThreads - 1) / kDThreads);
  block_stats_kernel<<<dim3(gx, n_mats), kDThreads, 0, s>>>(static_cast<const uint4*>(w_bf16),
                                                             reinterpret_cast<const uint2*>(codes), scales,
                                                             global_scale, rows, cols, layout, outlier_threshold,
                                                             stats);
  return check_launch("block_stats_kernel");
}
