// The NVFP4 W4A4 routed-expert MoE layer, end to end on one stream:
//   router logits -> top-k -> permutation -> quantise x into permuted rows ->
//   grouped FP4 GEMM gate/up (+ SiLU*up, requantise) -> grouped FP4 GEMM down
//   (+ g2 g_down w) -> combine.
// Sources: "K-EXAONE-152B-A23B-REAP-80E-NVFP4" model card ("Quantization
// Setup"), "K-EXAONE-152B-A23B-REAP-80E-BF16" model card ("Pruning Setup",
// "Routing behavior").
#include <algorithm>
#include <mutex>
#include <unordered_map>

#include "common.cuh"
#include "gemm.cuh"
#include "host.cuh"
#include "route.cuh"

namespace nvfp4moe {

// Quantises token t's row once under g1 and writes it to each of its k
// permuted rows: packed codes and tiled scales.  One thread per 16-element
// block; groups of four lanes assemble a 32-bit scale word.
// Activation global-scale modes (NVFP4_ACT_SCALE_*): bit 0 = one scale per
// expert, bit 1 = g1 derived on the device from the batch amax.
constexpr int kActPerExpert = 1, kActDynamic = 2;

// g1 of the batch (dynamic modes): the weight rule, fl32(amax / 2688).
NVDEV float dynamic_gscale(uint32_t amax_bits) { return __fdiv_rn(__uint_as_float(amax_bits), 2688.0f); }

// Quantise x into its k permuted rows.  With one g1 for the tensor a block is
// quantised once and written k times; with one per expert each copy is
// quantised under its own expert's g1.  In the dynamic modes g1 comes from
// amax_bits ([0]: batch, [1 + e]: expert e) and block (0, 0) publishes it in
// act_gscale.
template <int MODE>
__global__ void __launch_bounds__(128) quantize_scatter_kernel(const uint4* __restrict__ x, int T, int H,
                                                               float* __restrict__ act_gscale,
                                                               const uint32_t* __restrict__ amax_bits,
                                                               const int32_t* __restrict__ inv_perm,
                                                               const int32_t* __restrict__ topk_idx, int k, int E,
                                                               uint2* __restrict__ a_codes,
                                                               uint8_t* __restrict__ a_scales) {
  // block (t, by): token t, 16-element blocks [128 by, 128 by + 128) of its row
  __shared__ int32_t rows[16];
  __shared__ float gs[16];
  const int t = blockIdx.x;
  const int nblk = H / kQBlock;
  const int lane = threadIdx.x & 31;
  const int kb = blockIdx.y * blockDim.x + threadIdx.x;
  const bool valid = kb < nblk;
  // x is the caller's input, so it is read before waiting for the routing;
  // with the tensor's own g1 (also an input) it is quantised there as well
  uint4 u0 = make_uint4(0, 0, 0, 0), u1 = u0;
  if (valid) {
    const uint4* src = x + ((size_t)t * H + (size_t)kb * kQBlock) / 8;
    u0 = __ldg(src);
    u1 = __ldg(src + 1);
  }
  uint2 c0 = make_uint2(0, 0);
  uint32_t s0 = 0;
  if (MODE == 0 && valid) {
    s0 = quant_block16_bf16(u0, u1, make_scaler(act_gscale[0]), c0);
  }
  griddep_wait();
  griddep_launch();
  if (threadIdx.x < k) {
    rows[threadIdx.x] = inv_perm[(size_t)t * k + threadIdx.x];
    if (MODE & kActPerExpert) {
      const int e = topk_idx[(size_t)t * k + threadIdx.x];
      gs[threadIdx.x] = (MODE & kActDynamic) ? dynamic_gscale(amax_bits[1 + e]) : act_gscale[e];
    }
  }
  if ((MODE & kActDynamic) && blockIdx.x == 0 && blockIdx.y == 0) {
    if (MODE & kActPerExpert) {
      for (int e = threadIdx.x; e < E; e += blockDim.x) act_gscale[e] = dynamic_gscale(amax_bits[1 + e]);
    } else if (threadIdx.x == 0) {
      act_gscale[0] = dynamic_gscale(amax_bits[0]);
    }
  }
  __syncthreads();
  auto write = [&](int row, const uint2& c, uint32_t s) {
    const uint32_t w1 = __shfl_down_sync(0xffffffffu, s, 1);
    const uint32_t w2 = __shfl_down_sync(0xffffffffu, s, 2);
    const uint32_t w3 = __shfl_down_sync(0xffffffffu, s, 3);
    const uint32_t word = s | (w1 << 8) | (w2 << 16) | (w3 << 24);
    if (valid) {
      a_codes[(size_t)row * nblk + kb] = c;
      if ((lane & 3) == 0) *reinterpret_cast<uint32_t*>(a_scales + tiled_scale_offset(row, kb, nblk >> 2)) = word;
    }
  };
  if (MODE & kActPerExpert) {
    for (int j = 0; j < k; ++j) {
      uint2 c = make_uint2(0, 0);
      uint32_t s = 0;
      if (valid) s = quant_block16_bf16(u0, u1, make_scaler(gs[j]), c);
      write(rows[j], c, s);
    }
  } else {
    if (MODE & kActDynamic) {
      if (valid) s0 = quant_block16_bf16(u0, u1, make_scaler(dynamic_gscale(amax_bits[0])), c0);
    }
    for (int j = 0; j < k; ++j) write(rows[j], c0, s0);
  }
}

// amax |x| of every token (exact, on packed bf16 pairs) into tok_amax[t] and
// the batch amax into amax_bits[0].  Non-negative floats order like their
// bits, so the maxima are integer atomics.
__global__ void __launch_bounds__(256) token_amax_kernel(const uint4* __restrict__ x, int H,
                                                         uint32_t* __restrict__ tok_amax,
                                                         uint32_t* __restrict__ amax_bits) {
  const int t = blockIdx.x;
  const int vpr = H / 8;
  __nv_bfloat162 m2 = __floats2bfloat162_rn(0.0f, 0.0f);
  for (int c = threadIdx.x; c < vpr; c += blockDim.x) {
    const uint4 u = __ldg(x + (size_t)t * vpr + c);
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int j = 0; j < 4; ++j) m2 = __hmax2(m2, __habs2(*reinterpret_cast<const __nv_bfloat162*>(&w[j])));
  }
  uint32_t mb = __float_as_uint(fmaxf(__low2float(m2), __high2float(m2)));
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) mb = max(mb, __shfl_xor_sync(0xffffffffu, mb, o));
  __shared__ uint32_t red[8];
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = mb;
  __syncthreads();
  if (threadIdx.x == 0) {
    for (int i = 1; i < (int)(blockDim.x >> 5); ++i) mb = max(mb, red[i]);
    tok_amax[t] = mb;
    atomicMax(amax_bits, mb);
  }
}

// REAP saliency of one batch ("Pruning Setup" of the BF16 model card): for
// expert e, the sum over its real rows of ||w y||_2 = w ||y||_2, from the
// down epilogue's per-thread sums of squares, in a fixed order (one block
// per expert, rows strided over threads, then a fixed tree), added to the
// caller's accumulators together with the row count.
constexpr int kSalThreads = 256;
__global__ void __launch_bounds__(kSalThreads) reap_saliency_kernel(const float* __restrict__ y_sq_part, int parts,
                                                                    const int32_t* __restrict__ offsets,
                                                                    const int32_t* __restrict__ counts,
                                                                    double* __restrict__ saliency_sum,
                                                                    unsigned long long* __restrict__ saliency_count) {
  const int e = blockIdx.x;
  const int r0 = offsets[e], n = counts[e];
  double acc = 0.0;
  for (int i = threadIdx.x; i < n; i += blockDim.x) {
    const float* p = y_sq_part + (size_t)(r0 + i) * parts;
    double ss = 0.0;
    for (int c = 0; c < parts; ++c) ss += (double)p[c];
    acc += sqrt(ss);
  }
  __shared__ double red[kSalThreads];
  red[threadIdx.x] = acc;
  __syncthreads();
  for (int o = kSalThreads / 2; o > 0; o >>= 1) {
    if (threadIdx.x < o) red[threadIdx.x] += red[threadIdx.x + o];
    __syncthreads();
  }
  if (threadIdx.x == 0) {
    saliency_sum[e] += red[0];
    saliency_count[e] += (unsigned long long)n;
  }
}

// REAP retention ("Pruning Setup" of the BF16 model card: the routed experts
// with the lowest saliency are removed): the mean saliency of expert e is
// saliency_sum[e] / saliency_count[e] (IEEE fp64 division; 0 for an expert
// never routed), and the `keep` highest means are retained, ties to the lower
// index, written in expert order.  One block, one thread per expert: a
// thread's rank is the number of experts ahead of it.
__global__ void __launch_bounds__(256) reap_keep_kernel(const double* __restrict__ saliency_sum,
                                                        const unsigned long long* __restrict__ saliency_count, int E,
                                                        int keep, int32_t* __restrict__ keep_idx) {
  __shared__ double mean[256];
  __shared__ int kept[256];
  const int e = threadIdx.x;
  if (e < E) {
    const unsigned long long n = saliency_count[e];
    mean[e] = n ? __ddiv_rn(saliency_sum[e], (double)n) : 0.0;
  }
  __syncthreads();
  int rank = 0;
  if (e < E)
    for (int j = 0; j < E; ++j) rank += (mean[j] > mean[e]) || (mean[j] == mean[e] && j < e);
  kept[e] = (e < E && rank < keep) ? 1 : 0;
  __syncthreads();
  if (kept[e]) {
    int pos = 0;
    for (int j = 0; j < e; ++j) pos += kept[j];
    keep_idx[pos] = e;
  }
}

// The shared expert's dense "grouping": one expert holding rows [0, T).
__global__ void dense_tiles_kernel(int T, int32_t* __restrict__ tile_expert, int32_t* __restrict__ num_mtiles,
                                   int32_t* __restrict__ offsets, int32_t* __restrict__ counts) {
  const int mt = (T + kRowTile - 1) / kRowTile;
  for (int i = threadIdx.x; i < mt; i += blockDim.x) tile_expert[i] = 0;
  if (threadIdx.x == 0) {
    *num_mtiles = mt;
    offsets[0] = 0;
    offsets[1] = mt * kRowTile;
    counts[0] = T;
  }
}

// Split K of the shared expert's bf16 GEMMs.  With few tokens their (m-tile,
// n-tile) tiles occupy a handful of the 148 SMs (at 16 tokens: 16 gate/up and
// 24 down tiles), so the weight stream would run on a tenth of the machine.
// Below half a wave of tiles each tile's K range is split over the largest
// divisor of its K stages (64 elements each, at most 16 parts) that keeps the
// CTAs within one wave.  Host arithmetic only, so the workspace size and the
// launch count follow the shape alone.
constexpr int kSplitWaveCtas = 148;
constexpr int kMaxSplit = 16;
static int shared_ksplit(int T, int n_tiles, int k_stages) {
  const int tiles = (T + kRowTile - 1) / kRowTile * n_tiles;
  if (2 * tiles > kSplitWaveCtas) return 1;
  int best = 1;
  for (int d = 2; d <= kMaxSplit && d <= k_stages; ++d)
    if (k_stages % d == 0 && tiles * d <= kSplitWaveCtas) best = d;
  return best;
}
static int shared_ksplit_gate_up(int T, int H, int I_s) { return shared_ksplit(T, I_s / 128, H / 64); }
static int shared_ksplit_down(int T, int H, int I_s) { return shared_ksplit(T, H / 256, I_s / 64); }

// The split parts of a shared-expert GEMM added in part order, then its
// epilogue: gate/up h = bf16(silu(gate) * up) ([T][cols], cols = I_shared;
// each partial row holds the gate sums then the up sums), down y = bf16(sum)
// ([T][cols], cols = H).  Four columns per thread.
template <bool kGateUp>
__global__ void __launch_bounds__(256) shared_split_reduce_kernel(const float* __restrict__ part, int S, int T,
                                                                  int cols, uint16_t* __restrict__ out) {
  griddep_wait();
  griddep_launch();
  const int ld = kGateUp ? 2 * cols : cols;
  const size_t slab = (size_t)T * ld;
  const int q = cols / 4;
  const size_t n = (size_t)T * q;
  for (size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (size_t)gridDim.x * blockDim.x) {
    const int t = (int)(i / q), c = (int)(i % q) * 4;
    const float* src = part + (size_t)t * ld + c;
    // every part's values are loaded before the first add (S <= kMaxSplit)
    float4 g[kMaxSplit], u[kMaxSplit];
#pragma unroll
    for (int sp = 0; sp < kMaxSplit; ++sp) {
      if (sp < S) {
        g[sp] = __ldcs(reinterpret_cast<const float4*>(src + sp * slab));
        if (kGateUp) u[sp] = __ldcs(reinterpret_cast<const float4*>(src + sp * slab + cols));
      }
    }
    float4 a = g[0], b = kGateUp ? u[0] : make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
    for (int sp = 1; sp < kMaxSplit; ++sp) {
      if (sp < S) {
        a = make_float4(__fadd_rn(a.x, g[sp].x), __fadd_rn(a.y, g[sp].y), __fadd_rn(a.z, g[sp].z),
                        __fadd_rn(a.w, g[sp].w));
        if (kGateUp)
          b = make_float4(__fadd_rn(b.x, u[sp].x), __fadd_rn(b.y, u[sp].y), __fadd_rn(b.z, u[sp].z),
                          __fadd_rn(b.w, u[sp].w));
      }
    }
    uint2 w;
    if (kGateUp) {
      w.x = pack_bf16x2(__fmul_rn(silu(a.x), b.x), __fmul_rn(silu(a.y), b.y));
      w.y = pack_bf16x2(__fmul_rn(silu(a.z), b.z), __fmul_rn(silu(a.w), b.w));
    } else {
      w.x = pack_bf16x2(a.x, a.y);
      w.y = pack_bf16x2(a.z, a.w);
    }
    *reinterpret_cast<uint2*>(out + (size_t)t * cols + c) = w;
  }
}

// amax of the tokens routed to each expert: amax_bits[1 + e].
__global__ void __launch_bounds__(256) expert_amax_kernel(const int32_t* __restrict__ topk_idx, int T, int k,
                                                          const uint32_t* __restrict__ tok_amax,
                                                          uint32_t* __restrict__ amax_bits) {
  griddep_wait();
  griddep_launch();
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i < T * k) atomicMax(amax_bits + 1 + topk_idx[i], tok_amax[i / k]);
}

// out[t] = bf16( [y_shared[t] +] sum_j y[inv_perm[t, j]] ), fp32 sum, shared
// row first, then slot order.  The routing weight is already folded into y by
// the down-projection epilogue.
// Block (t, by) covers token t's 8-column groups by*blockDim.x + i*gridDim.y*
// blockDim.x (+ threadIdx.x): a small batch spreads a row over several
// blocks, a large one keeps whole rows in one block for long contiguous
// reads.  A thread issues all k row loads of a column group before adding.
// KMAX bounds k at compile time: the common k <= 8 keeps half the registers
// of k <= 16, so twice the blocks (and loads in flight) fit on an SM.
constexpr int kCombineThreads = 256;

template <int KMAX>
__global__ void __launch_bounds__(kCombineThreads) combine_kernel(const uint4* __restrict__ y,
                                                                  const uint4* __restrict__ y_shared,
                                                                  const int32_t* __restrict__ inv_perm, int T, int H,
                                                                  int k, uint4* __restrict__ out) {
  __shared__ int32_t rows[KMAX];
  griddep_wait();
  griddep_launch();
  const int t = blockIdx.x;
  if (threadIdx.x < k) rows[threadIdx.x] = inv_perm[(size_t)t * k + threadIdx.x];
  __syncthreads();
  const int vpr = H / 8;
  for (int c = blockIdx.y * blockDim.x + threadIdx.x; c < vpr; c += gridDim.y * blockDim.x) {
    uint4 v[KMAX];
#pragma unroll
    for (int j = 0; j < KMAX; ++j)
      if (j < k) v[j] = __ldg(y + (size_t)rows[j] * vpr + c);
    float acc[8] = {0, 0, 0, 0, 0, 0, 0, 0};
    if (y_shared) unpack_bf16x8(__ldg(y_shared + (size_t)t * vpr + c), acc);   // the shared expert's row first
#pragma unroll
    for (int j = 0; j < KMAX; ++j) {
      if (j < k) {
        float f[8];
        unpack_bf16x8(v[j], f);
#pragma unroll
        for (int q = 0; q < 8; ++q) acc[q] = __fadd_rn(acc[q], f[q]);
      }
    }
    out[(size_t)t * vpr + c] = make_uint4(pack_bf16x2(acc[0], acc[1]), pack_bf16x2(acc[2], acc[3]),
                                          pack_bf16x2(acc[4], acc[5]), pack_bf16x2(acc[6], acc[7]));
  }
}

struct ForwardScratch {
  RouteScratch route;
  float* logits;
  int32_t* topk_idx;
  float* topk_w;
  int32_t* offsets;
  int32_t* perm;
  int32_t* inv_perm;
  uint8_t* a_codes;
  uint8_t* a_scales;
  uint8_t* h_codes;
  uint8_t* h_scales;
  uint16_t* y;
  uint32_t* amax_bits;      // [E + 1] batch amax, then per expert (dynamic modes)
  uint32_t* tok_amax;       // [T]
  float* y_sq_part;         // [rows][H/128] (saliency requested)
  // shared expert (I_shared > 0)
  uint16_t* sh_h;           // bf16 [T_pad][I_shared]
  uint16_t* sh_y;           // bf16 [T_pad][H]
  int32_t* sh_tiles;        // [T_pad / 128]
  int32_t* sh_ntiles;       // [1]
  int32_t* sh_offsets;      // [2]
  int32_t* sh_counts;       // [1]
  float* sh_partial;        // split K: fp32 [S][T][2 I_shared] (gate/up), then [S][T][H] (down)
};

static ForwardScratch carve_forward(Carver& c, int T, int E, int H, int I, int k, int I_shared) {
  ForwardScratch f;
  const int cap = route_rows_capacity(T, E, k);
  f.route = carve_route_scratch(c, T, E, k);
  f.logits = c.take<float>((size_t)T * E);
  f.topk_idx = c.take<int32_t>((size_t)T * k);
  f.topk_w = c.take<float>((size_t)T * k);
  f.offsets = c.take<int32_t>((size_t)E + 1);
  f.perm = c.take<int32_t>((size_t)cap);
  f.inv_perm = c.take<int32_t>((size_t)T * k);
  f.a_codes = c.take<uint8_t>((size_t)cap * H / 2);
  f.a_scales = c.take<uint8_t>((size_t)cap * H / 16);
  f.h_codes = c.take<uint8_t>((size_t)cap * I / 2);
  f.h_scales = c.take<uint8_t>((size_t)cap * I / 16);
  f.y = c.take<uint16_t>((size_t)cap * H);
  f.amax_bits = c.take<uint32_t>((size_t)E + 1);
  f.tok_amax = c.take<uint32_t>((size_t)T);
  f.y_sq_part = c.take<float>((size_t)cap * (H / 128));
  f.sh_h = f.sh_y = nullptr;
  f.sh_tiles = f.sh_ntiles = f.sh_offsets = f.sh_counts = nullptr;
  f.sh_partial = nullptr;
  if (I_shared > 0) {
    const size_t tp = (size_t)(T + kRowTile - 1) / kRowTile * kRowTile;
    f.sh_h = c.take<uint16_t>(tp * I_shared);
    f.sh_y = c.take<uint16_t>(tp * H);
    f.sh_tiles = c.take<int32_t>(tp / kRowTile);
    f.sh_ntiles = c.take<int32_t>(1);
    f.sh_offsets = c.take<int32_t>(2);
    f.sh_counts = c.take<int32_t>(1);
    const int s1 = shared_ksplit_gate_up(T, H, I_shared), s2 = shared_ksplit_down(T, H, I_shared);
    const size_t part = std::max(s1 > 1 ? (size_t)s1 * T * 2 * I_shared : 0, s2 > 1 ? (size_t)s2 * T * H : 0);
    if (part) f.sh_partial = c.take<float>(part);
  }
  return f;
}

static nvfp4_status mark(const moe_nvfp4_debug* dbg, int i, cudaStream_t s) {
  if (!dbg || !dbg->stage_events[i]) return NVFP4_OK;
  return check_cuda(cudaEventRecord(static_cast<cudaEvent_t>(dbg->stage_events[i]), s), "cudaEventRecord");
}

static nvfp4_status copy_out(void* dst, const void* src, size_t bytes, cudaStream_t s) {
  if (!dst || bytes == 0) return NVFP4_OK;
  return check_cuda(cudaMemcpyAsync(dst, src, bytes, cudaMemcpyDeviceToDevice, s), "copy debug output");
}

}  // namespace nvfp4moe

using namespace nvfp4moe;

extern "C" size_t moe_nvfp4_workspace_size_shared(int T, int E, int H, int I, int k, int I_shared) {
  if (T < 0 || E < 0 || H < 0 || I < 0 || k < 0 || I_shared < 0) return 0;
  Carver c(nullptr);
  carve_forward(c, T, E, H, I, k, I_shared);
  return c.size();
}

extern "C" size_t moe_nvfp4_workspace_size(int T, int E, int H, int I, int k) {
  return moe_nvfp4_workspace_size_shared(T, E, H, I, k, 0);
}

// Mirrors the launch sequence of forward_impl below.
extern "C" int moe_nvfp4_forward_launches(int T, int E, int H, int I, int k, int I_shared, int mode) {
  if (T < 1 || H <= 0 || H % 256 != 0 || I <= 0 || I % 128 != 0 || k < 1 || k > 16 || k > E || E > 256 ||
      I_shared < 0 || I_shared % 128 != 0 || mode < NVFP4_ACT_SCALE_TENSOR || mode > NVFP4_ACT_SCALE_DYNAMIC_EXPERT)
    return -1;
  int n = 0;
  if (I_shared > 0) {
    n += 1 + 2;                                                     // dense tile map, shared gate/up and down
    n += (shared_ksplit_gate_up(T, H, I_shared) > 1) + (shared_ksplit_down(T, H, I_shared) > 1);   // reductions
  }
  if (mode & kActDynamic) n += 1;                                   // token amax
  n += 1 + (T <= 256 ? 1 : 2);                                      // router GEMM, routing
  if (mode == NVFP4_ACT_SCALE_DYNAMIC_EXPERT) n += 1;               // expert amax
  if (!(mode == NVFP4_ACT_SCALE_TENSOR && route_fuses_x_quantise(T, H, k))) n += 1;   // quantise-scatter
  n += 2 + 1;                                                       // gate/up, down, combine
  return n;
}

template <int MODE>
static nvfp4_status launch_quantize_scatter(const ForwardScratch& f, const void* x_bf16, int T, int H, int E, int k,
                                            float* act_gscale, cudaStream_t s) {
  return launch_dependent("quantize_scatter_kernel", quantize_scatter_kernel<MODE>,
                          dim3(T, (H / kQBlock + 127) / 128), dim3(128), 0, s, static_cast<const uint4*>(x_bf16), T,
                          H, act_gscale, (const uint32_t*)f.amax_bits, (const int32_t*)f.inv_perm,
                          (const int32_t*)f.topk_idx, k, E, reinterpret_cast<uint2*>(f.a_codes), f.a_scales);
}

static nvfp4_status forward_impl(const moe_nvfp4_weights* W, const void* x_bf16, int T, int mode, float* act_gscale,
                                 const float* h_gscale, const float* logit_offset, void* out_bf16,
                                 const moe_nvfp4_debug* dbg, void* ws, size_t ws_bytes, void* stream) {
  NV_CHECK(nvfp4moe_check_weights(W));
  NV_REQUIRE(mode >= NVFP4_ACT_SCALE_TENSOR && mode <= NVFP4_ACT_SCALE_DYNAMIC_EXPERT, NVFP4_ERR_INVALID_ARG,
             "moe_nvfp4_forward: unknown activation scale mode %d", mode);
  NV_REQUIRE(x_bf16 && act_gscale && h_gscale && out_bf16, NVFP4_ERR_INVALID_ARG,
             "moe_nvfp4_forward: x, act_gscale, h_gscale and out are required");
  NV_REQUIRE(W->router_weight && W->bias && W->gate_codes && W->gate_scales && W->gate_gscale && W->up_codes &&
                 W->up_scales && W->up_gscale && W->down_codes && W->down_scales && W->down_gscale,
             NVFP4_ERR_INVALID_ARG, "moe_nvfp4_forward: a weight pointer is NULL");
  NV_REQUIRE(T >= 1, NVFP4_ERR_INVALID_ARG, "moe_nvfp4_forward: T=%d", T);
  NV_CHECK(check_route_shape(T, W->H, W->E, W->k));
  NV_REQUIRE(aligned(x_bf16, 16) && aligned(out_bf16, 16) && aligned(W->router_weight, 16) &&
                 aligned(W->gate_codes, 16) && aligned(W->up_codes, 16) && aligned(W->down_codes, 16) &&
                 aligned(W->gate_scales, 16) && aligned(W->up_scales, 16) && aligned(W->down_scales, 16),
             NVFP4_ERR_INVALID_ARG, "moe_nvfp4_forward: tensors need 16-byte alignment");
  const int E = W->E, H = W->H, I = W->I, k = W->k;
  const int I_s = W->I_shared;
  const bool shared = I_s > 0;
  const size_t need = moe_nvfp4_workspace_size_shared(T, E, H, I, k, I_s);
  NV_REQUIRE(ws && ws_bytes >= need && aligned(ws, 256), NVFP4_ERR_WORKSPACE,
             "moe_nvfp4_forward: needs a 256-byte aligned workspace of %zu bytes", need);
  int sms = 0;
  NV_CHECK(device_sm_count(&sms));
  cudaStream_t s = as_stream(stream);
  Carver c(ws);
  ForwardScratch f = carve_forward(c, T, E, H, I, k, I_s);
  const int cap = route_rows_capacity(T, E, k);

  // The status word is cleared by the first kernel when that is the router
  // GEMM (a memset would stop it from starting early behind the previous
  // kernel on the stream), else by a memset.
  const bool router_first = !shared && !(mode & kActDynamic);
  if (!router_first)
    NV_CHECK(check_cuda(cudaMemsetAsync(f.route.status, 0, sizeof(uint32_t), s), "clear status word"));
  NV_CHECK(mark(dbg, 0, s));
  if (shared) {
    dense_tiles_kernel<<<1, 128, 0, s>>>(T, f.sh_tiles, f.sh_ntiles, f.sh_offsets, f.sh_counts);
    NV_CHECK(check_launch("dense_tiles_kernel"));
  }
  if (mode & kActDynamic) {
    // 0: amax of every token and of the batch
    NV_CHECK(check_cuda(cudaMemsetAsync(f.amax_bits, 0, sizeof(uint32_t) * (size_t)(E + 1), s), "clear amax"));
    token_amax_kernel<<<T, 256, 0, s>>>(static_cast<const uint4*>(x_bf16), H, f.tok_amax, f.amax_bits);
    NV_CHECK(check_launch("token_amax_kernel"));
  }
  // 1-3: router, top-k, permutation
  RouteArgs ra;
  ra.x = x_bf16;
  ra.router_weight = W->router_weight;
  ra.logit_offset = logit_offset;
  ra.bias = W->bias;
  ra.T = T; ra.H = H; ra.E = E; ra.k = k; ra.rsf = W->routed_scaling_factor;
  ra.logits = f.logits;
  ra.topk_idx = f.topk_idx; ra.topk_w = f.topk_w; ra.expert_offsets = f.offsets;
  ra.perm = f.perm; ra.inv_perm = f.inv_perm;
  ra.clear_status = router_first;
  // small batches with the tensor's own g1: the routing kernel quantises x
  // and fills the permuted rows itself, one kernel fewer in the chain
  const bool fused_x = mode == NVFP4_ACT_SCALE_TENSOR && route_fuses_x_quantise(T, H, k);
  ra.quant_x = fused_x;
  ra.act_gscale = act_gscale;
  ra.a_codes = f.a_codes;
  ra.a_scales = f.a_scales;
  NV_CHECK(launch_route(ra, f.route, s));
  NV_CHECK(mark(dbg, 1, s));

  // 4: quantise x into its k permuted rows (under the batch's or each
  // expert's g1); the routing kernel has done it already when fused_x.
  // Padding rows are left as they are: an MMA row only feeds the same output
  // row, and the epilogues skip padding rows.
  if (mode == NVFP4_ACT_SCALE_DYNAMIC_EXPERT) {
    NV_CHECK(launch_dependent("expert_amax_kernel", expert_amax_kernel, dim3((T * k + 255) / 256), dim3(256), 0, s,
                              (const int32_t*)f.topk_idx, T, k, (const uint32_t*)f.tok_amax, f.amax_bits));
  }
  switch (fused_x ? -1 : mode) {
    case -1: break;
    case NVFP4_ACT_SCALE_TENSOR: NV_CHECK(launch_quantize_scatter<0>(f, x_bf16, T, H, E, k, act_gscale, s)); break;
    case NVFP4_ACT_SCALE_EXPERT: NV_CHECK(launch_quantize_scatter<1>(f, x_bf16, T, H, E, k, act_gscale, s)); break;
    case NVFP4_ACT_SCALE_DYNAMIC: NV_CHECK(launch_quantize_scatter<2>(f, x_bf16, T, H, E, k, act_gscale, s)); break;
    default: NV_CHECK(launch_quantize_scatter<3>(f, x_bf16, T, H, E, k, act_gscale, s)); break;
  }
  NV_CHECK(mark(dbg, 2, s));

  // 5-6: gate/up GEMM with SiLU*up and requantisation
  GroupedGemmArgs g1;
  g1.epi = kEpiGateUp;
  g1.E = E; g1.H = H; g1.I = I;
  g1.rows_capacity = cap;
  g1.a_codes = f.a_codes; g1.a_scales = f.a_scales;
  g1.b0_codes = W->gate_codes; g1.b0_scales = W->gate_scales; g1.b0_gscale = W->gate_gscale;
  g1.b1_codes = W->up_codes; g1.b1_scales = W->up_scales; g1.b1_gscale = W->up_gscale;
  g1.b_staged = W->codes_layout == NVFP4_LAYOUT_STAGED;
  g1.act_gscale = act_gscale;
  g1.tile_expert = f.route.tile_expert; g1.num_mtiles = f.route.num_mtiles;
  g1.expert_offsets = f.offsets; g1.expert_counts = f.route.counts;
  g1.h_gscale = h_gscale; g1.h_codes = f.h_codes; g1.h_scales = f.h_scales;
  g1.h_f32 = dbg ? dbg->h : nullptr;
  g1.h_amax = dbg ? dbg->h_amax : nullptr;
  g1.per_expert_scales = (mode & kActPerExpert) != 0;
  g1.status = f.route.status;
  g1.pair = T * k >= kPairMinRows;
  NV_CHECK(launch_grouped_gemm(g1, s));
  NV_CHECK(mark(dbg, 3, s));

  // 7: down GEMM with g2 * g_down * routing weight
  GroupedGemmArgs g2;
  g2.epi = kEpiDown;
  g2.E = E; g2.H = H; g2.I = I;
  g2.rows_capacity = cap;
  g2.a_codes = f.h_codes; g2.a_scales = f.h_scales;
  g2.b0_codes = W->down_codes; g2.b0_scales = W->down_scales; g2.b0_gscale = W->down_gscale;
  g2.b_staged = W->codes_layout == NVFP4_LAYOUT_STAGED;
  g2.act_gscale = h_gscale;
  g2.tile_expert = f.route.tile_expert; g2.num_mtiles = f.route.num_mtiles;
  g2.expert_offsets = f.offsets; g2.expert_counts = f.route.counts;
  g2.row_w = f.route.row_w; g2.y_bf16 = f.y; g2.y_f32 = dbg ? dbg->y : nullptr;
  g2.per_expert_scales = (mode & kActPerExpert) != 0;
  const bool saliency = dbg && dbg->saliency_sum && dbg->saliency_count;
  g2.y_sq_part = saliency ? f.y_sq_part : nullptr;
  g2.status = f.route.status;
  g2.pair = T * k >= kPairMinRows;
  NV_CHECK(launch_grouped_gemm(g2, s));
  NV_CHECK(mark(dbg, 4, s));

  // the shared expert (bf16): gate/up with SiLU*up, then down; its y goes
  // into the combine
  if (shared) {
    const int tp = (T + kRowTile - 1) / kRowTile * kRowTile;
    GroupedGemmArgs s1;
    s1.epi = kEpiSharedGateUp;
    s1.E = 1; s1.H = H; s1.I = I_s;
    s1.rows_capacity = tp;
    s1.a_rows = T;
    s1.a_codes = static_cast<const uint8_t*>(x_bf16);
    s1.b0_codes = static_cast<const uint8_t*>(W->shared_gate);
    s1.b1_codes = static_cast<const uint8_t*>(W->shared_up);
    s1.tile_expert = f.sh_tiles; s1.num_mtiles = f.sh_ntiles;
    s1.expert_offsets = f.sh_offsets; s1.expert_counts = f.sh_counts;
    s1.h_bf16 = f.sh_h;
    s1.status = f.route.status;
    s1.ksplit = shared_ksplit_gate_up(T, H, I_s);
    if (s1.ksplit > 1) {
      s1.h_bf16 = nullptr;
      s1.partial = f.sh_partial;
      s1.partial_rows = T;
    }
    NV_CHECK(launch_grouped_gemm(s1, s));
    if (s1.ksplit > 1) {
      NV_CHECK(launch_dependent("shared_split_reduce_kernel<gate_up>", shared_split_reduce_kernel<true>,
                                dim3((T * I_s / 4 + 255) / 256), dim3(256), 0, s, (const float*)f.sh_partial,
                                s1.ksplit, T, I_s, f.sh_h));
    }
    GroupedGemmArgs s2;
    s2.epi = kEpiSharedDown;
    s2.E = 1; s2.H = H; s2.I = I_s;
    s2.rows_capacity = tp;
    s2.a_codes = reinterpret_cast<const uint8_t*>(f.sh_h);
    s2.b0_codes = static_cast<const uint8_t*>(W->shared_down);
    s2.tile_expert = f.sh_tiles; s2.num_mtiles = f.sh_ntiles;
    s2.expert_offsets = f.sh_offsets; s2.expert_counts = f.sh_counts;
    s2.y_bf16 = f.sh_y;
    s2.status = f.route.status;
    s2.ksplit = shared_ksplit_down(T, H, I_s);
    if (s2.ksplit > 1) {
      s2.y_bf16 = nullptr;
      s2.partial = f.sh_partial;
      s2.partial_rows = T;
    }
    NV_CHECK(launch_grouped_gemm(s2, s));
    if (s2.ksplit > 1) {
      NV_CHECK(launch_dependent("shared_split_reduce_kernel<down>", shared_split_reduce_kernel<false>,
                                dim3((T * H / 4 + 255) / 256), dim3(256), 0, s, (const float*)f.sh_partial,
                                s2.ksplit, T, H, f.sh_y));
    }
    if (dbg && dbg->shared_event)
      NV_CHECK(check_cuda(cudaEventRecord(static_cast<cudaEvent_t>(dbg->shared_event), s), "cudaEventRecord"));
  }

  // 8: combine
  // below about two waves of whole-row blocks, split rows across blocks
  const int row_blocks = T >= 2 * sms ? 1 : (H / 8 + kCombineThreads - 1) / kCombineThreads;
  NV_CHECK(launch_dependent("combine_kernel", k <= 8 ? combine_kernel<8> : combine_kernel<16>, dim3(T, row_blocks),
                            dim3(kCombineThreads), 0, s, reinterpret_cast<const uint4*>(f.y),
                            shared ? reinterpret_cast<const uint4*>(f.sh_y) : (const uint4*)nullptr,
                            (const int32_t*)f.inv_perm, T, H, k, static_cast<uint4*>(out_bf16)));
  NV_CHECK(mark(dbg, 5, s));
  if (saliency) {
    reap_saliency_kernel<<<E, kSalThreads, 0, s>>>(f.y_sq_part, H / 128, f.offsets, f.route.counts,
                                                  dbg->saliency_sum, dbg->saliency_count);
    NV_CHECK(check_launch("reap_saliency_kernel"));
  }

  if (dbg) {
    NV_CHECK(copy_out(dbg->logits, f.logits, sizeof(float) * (size_t)T * E, s));
    NV_CHECK(copy_out(dbg->topk_idx, f.topk_idx, sizeof(int32_t) * (size_t)T * k, s));
    NV_CHECK(copy_out(dbg->topk_w, f.topk_w, sizeof(float) * (size_t)T * k, s));
    NV_CHECK(copy_out(dbg->expert_offsets, f.offsets, sizeof(int32_t) * (size_t)(E + 1), s));
    NV_CHECK(copy_out(dbg->perm, f.perm, sizeof(int32_t) * (size_t)cap, s));
    NV_CHECK(copy_out(dbg->inv_perm, f.inv_perm, sizeof(int32_t) * (size_t)T * k, s));
    NV_CHECK(copy_out(dbg->a_codes, f.a_codes, (size_t)cap * H / 2, s));
    NV_CHECK(copy_out(dbg->a_scales, f.a_scales, (size_t)cap * H / 16, s));
    NV_CHECK(copy_out(dbg->h_codes, f.h_codes, (size_t)cap * I / 2, s));
    NV_CHECK(copy_out(dbg->h_scales, f.h_scales, (size_t)cap * I / 16, s));
  }
  return NVFP4_OK;
}

extern "C" nvfp4_status moe_nvfp4_forward(const moe_nvfp4_weights* W, const void* x_bf16, int T,
                                          const float* act_gscale, const float* h_gscale, const float* logit_offset,
                                          void* out_bf16, const moe_nvfp4_debug* dbg, void* ws, size_t ws_bytes,
                                          void* stream) {
  // the tensor mode only reads act_gscale
  return forward_impl(W, x_bf16, T, NVFP4_ACT_SCALE_TENSOR, const_cast<float*>(act_gscale), h_gscale, logit_offset,
                      out_bf16, dbg, ws, ws_bytes, stream);
}

extern "C" nvfp4_status moe_nvfp4_forward_scaled(const moe_nvfp4_weights* W, const void* x_bf16, int T,
                                                 int act_scale_mode, float* act_gscale, const float* h_gscale,
                                                 const float* logit_offset, void* out_bf16,
                                                 const moe_nvfp4_debug* dbg, void* ws, size_t ws_bytes,
                                                 void* stream) {
  return forward_impl(W, x_bf16, T, act_scale_mode, act_gscale, h_gscale, logit_offset, out_bf16, dbg, ws, ws_bytes,
                      stream);
}

// ---------------------------------------------------------------------------
// The forward on host buffers.  x is copied into a staging buffer at the end
// of the workspace and out back from another, each on a copy stream of the
// library's own, so that consecutive calls on different workspaces overlap
// one call's copies with another's compute.  Per workspace the library keeps
// three events (x landed, forward done, out copied back); a call waits for
// the previous call on the same workspace before it overwrites that call's
// staging buffers.
// ---------------------------------------------------------------------------
namespace {
struct HostSlot {
  cudaEvent_t in = nullptr, done = nullptr, out = nullptr;
  bool used = false;
};
std::mutex g_host_mu;
std::unordered_map<const void*, HostSlot> g_host_slots;      // keyed by workspace
cudaStream_t g_copy_in[64], g_copy_out[64];                  // per device

size_t round256(size_t n) { return (n + 255) / 256 * 256; }

nvfp4_status host_slot_and_streams(const void* ws, HostSlot** slot, cudaStream_t* cin, cudaStream_t* cout) {
  int dev = 0;
  NV_CHECK(check_cuda(cudaGetDevice(&dev), "cudaGetDevice"));
  NV_REQUIRE(dev >= 0 && dev < 64, NVFP4_ERR_CUDA, "device ordinal %d out of range", dev);
  std::lock_guard<std::mutex> lock(g_host_mu);
  if (!g_copy_in[dev]) {
    NV_CHECK(check_cuda(cudaStreamCreateWithFlags(&g_copy_in[dev], cudaStreamNonBlocking), "cudaStreamCreate"));
    NV_CHECK(check_cuda(cudaStreamCreateWithFlags(&g_copy_out[dev], cudaStreamNonBlocking), "cudaStreamCreate"));
  }
  HostSlot& h = g_host_slots[ws];
  if (!h.in) {
    NV_CHECK(check_cuda(cudaEventCreateWithFlags(&h.in, cudaEventDisableTiming), "cudaEventCreate"));
    NV_CHECK(check_cuda(cudaEventCreateWithFlags(&h.done, cudaEventDisableTiming), "cudaEventCreate"));
    NV_CHECK(check_cuda(cudaEventCreateWithFlags(&h.out, cudaEventDisableTiming), "cudaEventCreate"));
  }
  *slot = &h;
  *cin = g_copy_in[dev];
  *cout = g_copy_out[dev];
  return NVFP4_OK;
}
}  // namespace

extern "C" size_t moe_nvfp4_workspace_size_host(int T, int E, int H, int I, int k, int I_shared) {
  if (T < 1 || H < 1) return 0;
  const size_t base = moe_nvfp4_workspace_size_shared(T, E, H, I, k, I_shared);
  if (base == 0) return 0;
  return round256(base) + 2 * round256((size_t)T * H * 2);
}

extern "C" nvfp4_status moe_nvfp4_forward_host(const moe_nvfp4_weights* W, const void* x_host_bf16, int T,
                                               const float* act_gscale, const float* h_gscale,
                                               const float* logit_offset, void* out_host_bf16, void* ws,
                                               size_t ws_bytes, void* stream) {
  NV_CHECK(nvfp4moe_check_weights(W));
  NV_REQUIRE(x_host_bf16 && out_host_bf16 && act_gscale && h_gscale, NVFP4_ERR_INVALID_ARG,
             "moe_nvfp4_forward_host: a required pointer is NULL");
  NV_REQUIRE(T >= 1, NVFP4_ERR_INVALID_ARG, "moe_nvfp4_forward_host: T=%d", T);
  const size_t need = moe_nvfp4_workspace_size_host(T, W->E, W->H, W->I, W->k, W->I_shared);
  NV_REQUIRE(ws && ws_bytes >= need && aligned(ws, 256), NVFP4_ERR_WORKSPACE,
             "moe_nvfp4_forward_host: needs a 256-byte aligned workspace of %zu bytes", need);
  const size_t base = round256(moe_nvfp4_workspace_size_shared(T, W->E, W->H, W->I, W->k, W->I_shared));
  const size_t io = (size_t)T * W->H * 2;
  uint8_t* x_dev = static_cast<uint8_t*>(ws) + base;
  uint8_t* out_dev = x_dev + round256(io);
  HostSlot* h = nullptr;
  cudaStream_t cin = nullptr, cout = nullptr;
  NV_CHECK(host_slot_and_streams(ws, &h, &cin, &cout));
  cudaStream_t s = as_stream(stream);
  // x in, once the previous call on this workspace has read its x
  if (h->used) NV_CHECK(check_cuda(cudaStreamWaitEvent(cin, h->done, 0), "cudaStreamWaitEvent"));
  NV_CHECK(check_cuda(cudaMemcpyAsync(x_dev, x_host_bf16, io, cudaMemcpyHostToDevice, cin), "copy x in"));
  NV_CHECK(check_cuda(cudaEventRecord(h->in, cin), "cudaEventRecord"));
  // the forward on the caller's stream, once x has landed and the previous
  // call's out has left the staging buffer
  NV_CHECK(check_cuda(cudaStreamWaitEvent(s, h->in, 0), "cudaStreamWaitEvent"));
  if (h->used) NV_CHECK(check_cuda(cudaStreamWaitEvent(s, h->out, 0), "cudaStreamWaitEvent"));
  NV_CHECK(forward_impl(W, x_dev, T, NVFP4_ACT_SCALE_TENSOR, const_cast<float*>(act_gscale), h_gscale,
                        logit_offset, out_dev, nullptr, ws, base, stream));
  NV_CHECK(check_cuda(cudaEventRecord(h->done, s), "cudaEventRecord"));
  // out back
  NV_CHECK(check_cuda(cudaStreamWaitEvent(cout, h->done, 0), "cudaStreamWaitEvent"));
  NV_CHECK(check_cuda(cudaMemcpyAsync(out_host_bf16, out_dev, io, cudaMemcpyDeviceToHost, cout), "copy out back"));
  NV_CHECK(check_cuda(cudaEventRecord(h->out, cout), "cudaEventRecord"));
  h->used = true;
  return NVFP4_OK;
}

extern "C" nvfp4_status moe_nvfp4_host_join(const void* ws, void* stream) {
  NV_REQUIRE(ws, NVFP4_ERR_INVALID_ARG, "moe_nvfp4_host_join: ws is NULL");
  cudaEvent_t ev = nullptr;
  {
    std::lock_guard<std::mutex> lock(g_host_mu);
    auto it = g_host_slots.find(ws);
    if (it == g_host_slots.end() || !it->second.used) return NVFP4_OK;
    ev = it->second.out;
  }
  return check_cuda(cudaStreamWaitEvent(as_stream(stream), ev, 0), "cudaStreamWaitEvent");
}

extern "C" nvfp4_status moe_nvfp4_host_release(const void* ws) {
  NV_REQUIRE(ws, NVFP4_ERR_INVALID_ARG, "moe_nvfp4_host_release: ws is NULL");
  HostSlot h;
  {
    std::lock_guard<std::mutex> lock(g_host_mu);
    auto it = g_host_slots.find(ws);
    if (it == g_host_slots.end()) return NVFP4_OK;
    h = it->second;
    g_host_slots.erase(it);
  }
  if (h.used) NV_CHECK(check_cuda(cudaEventSynchronize(h.out), "cudaEventSynchronize"));
  cudaEventDestroy(h.in);
  cudaEventDestroy(h.done);
  cudaEventDestroy(h.out);
  return NVFP4_OK;
}

extern "C" nvfp4_status moe_reap_keep(const double* saliency_sum, const unsigned long long* saliency_count, int E,
                                      int keep, int32_t* keep_idx, void* stream) {
  NV_REQUIRE(saliency_sum && saliency_count && keep_idx, NVFP4_ERR_INVALID_ARG, "moe_reap_keep: a pointer is NULL");
  NV_REQUIRE(E >= 1 && E <= 256 && keep >= 0 && keep <= E, NVFP4_ERR_INVALID_ARG,
             "moe_reap_keep: needs 1 <= E <= 256 and 0 <= keep <= E (E=%d keep=%d)", E, keep);
  NV_REQUIRE(aligned(saliency_sum, 8) && aligned(saliency_count, 8) && aligned(keep_idx, 4), NVFP4_ERR_INVALID_ARG,
             "moe_reap_keep: misaligned pointer");
  int sms = 0;
  NV_CHECK(device_sm_count(&sms));
  reap_keep_kernel<<<1, 256, 0, as_stream(stream)>>>(saliency_sum, saliency_count, E, keep, keep_idx);
  return check_launch("reap_keep_kernel");
}
