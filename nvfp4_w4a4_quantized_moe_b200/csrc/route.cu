// Router and permutation ("K-EXAONE-152B-A23B-REAP-80E-BF16" model card,
// section "Pruning Setup", "Routing behavior": renormalised sigmoid routing,
// sigmoid-and-bias selection, routed_scaling_factor; the router stays BF16 per
// the NVFP4 model card's "Quantization Setup").
#include <mutex>

#include "common.cuh"
#include "host.cuh"
#include "route.cuh"
#include "route_math.cuh"

namespace nvfp4moe {

// ---------------------------------------------------------------------------
// Router logits on the tensor cores: a bf16 x bf16 -> fp32 tcgen05 GEMM.
// One CTA computes a 128-token tile against all E experts (N = E rounded up
// to 16) over one slice of H; the slices' partial sums land in
// partial[split][T][E] and the top-k kernel adds them in split order, so the
// result does not depend on scheduling.  Warp 0 issues TMA loads (64 bf16 =
// 128 bytes of K per stage, 128-byte swizzle), warp 1 issues the MMAs from
// one thread, warps 2..5 read the accumulator out of tensor memory.
// ---------------------------------------------------------------------------
constexpr int kRBM = 128;
constexpr int kRBK = 64;                      // bf16 elements of K per stage
// Up to eight stages, as many as fit (router_stages): at 8192 tokens each CTA
// streams 1.3 MB of x and W_g, and four stages kept too few bytes in flight
// to cover the load latency.
constexpr int kRStages = 8;
constexpr int kRThreads = 192;
constexpr int kRAbytes = kRBM * kRBK * 2;     // 16 KiB

struct RouterGemmParams {
  int T, E, H, n_mma, kt_per_split, splits, clear_status;
  int stages;            // pipeline depth used (<= kRStages)
  float* partial;
  uint32_t* status;
};

static inline int router_n_mma(int E) { return (E + 15) / 16 * 16; }
static inline int router_stage_bytes(int E) { return kRAbytes + (router_n_mma(E) * 128 + 1023) / 1024 * 1024; }
static inline int router_stages(int E) {
  return std::max(2, std::min(kRStages, (227 * 1024 - 1024) / router_stage_bytes(E)));
}
static inline int router_smem_bytes(int E) { return router_stages(E) * router_stage_bytes(E) + 1024; }

// Split count: as many CTAs as fit on the SMs of a B200 (148) at one per SM,
// with at least four K stages each; rounding up instead (a second CTA on
// some SMs) measured slower.  A function of the shape only, so results are
// the same on every device.
int router_splits(int T, int H) {
  const int mt = std::max(1, (T + kRBM - 1) / kRBM);
  const int kt = H / kRBK;
  int sp = 148 / mt;
  sp = std::max(1, std::min(sp, std::max(1, kt / 4)));
  // each split takes ceil(kt / sp) stages; recount so that none is left
  // without any (25 stages over 6 splits of 5 would leave the sixth empty)
  const int per = (kt + sp - 1) / sp;
  return (kt + per - 1) / per;
}

__global__ void __launch_bounds__(kRThreads, 1)
    router_gemm_kernel(const __grid_constant__ CUtensorMap tmX, const __grid_constant__ CUtensorMap tmW,
                       const RouterGemmParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  __shared__ __align__(8) uint64_t full_bar[kRStages];
  __shared__ __align__(8) uint64_t empty_bar[kRStages];
  __shared__ __align__(8) uint64_t acc_bar;
  __shared__ uint32_t tmem_base_s;
  __shared__ int abort_s;
  volatile int* abort_flag = &abort_s;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int stage_bytes = kRAbytes + (p.n_mma * 128 + 1023) / 1024 * 1024;
  const uint32_t tcols = p.n_mma <= 32 ? 32 : p.n_mma <= 64 ? 64 : p.n_mma <= 128 ? 128 : 256;
  const int mt = blockIdx.x;
  const int KT = p.H / kRBK;
  const int kt0 = blockIdx.y * p.kt_per_split;
  const int nkt = min(kt0 + p.kt_per_split, KT) - kt0;

  if (threadIdx.x == 0) {
    for (int s = 0; s < p.stages; ++s) {
      mbar_init(&full_bar[s], 1);
      mbar_init(&empty_bar[s], 1);
    }
    mbar_init(&acc_bar, 1);
    abort_s = 0;
    fence_barrier_init();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tmap(&tmX);
    prefetch_tmap(&tmW);
  }
  if (warp == 1) {
    tmem_alloc(&tmem_base_s, tcols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_base_s;
  griddep_wait();
  griddep_launch();
  // first kernel of a call: the status word is cleared here, after the
  // stream's previous work, and before any wait of this call can give up
  if (p.clear_status && blockIdx.x == 0 && blockIdx.y == 0 && threadIdx.x == 0) *p.status = 0u;

  if (warp == 0) {
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0, filled = 0, fill_parity = 0;
      bool ok = true;
      for (int i = 0; i < nkt; ++i) {
        const int kt = kt0 + i;
        if (!mbar_wait(&empty_bar[stage], phase ^ 1u, abort_flag)) {
          *abort_flag = 1;
          atomicExch(p.status, kDevTimeout);
          ok = false;
          break;
        }
        uint8_t* sA = smem + stage * stage_bytes;
        mbar_arrive_expect_tx(&full_bar[stage], kRAbytes + p.n_mma * 128);
        tma_load_2d(sA, &tmX, kt * kRBK, mt * kRBM, &full_bar[stage]);
        tma_load_2d(sA + kRAbytes, &tmW, kt * kRBK, 0, &full_bar[stage]);
        filled |= 1u << stage;
        fill_parity = (fill_parity & ~(1u << stage)) | (phase << stage);
        if (++stage == p.stages) {
          stage = 0;
          phase ^= 1u;
        }
      }
      if (!ok) {
        volatile int never = 0;
        for (int s = 0; s < p.stages; ++s)
          if ((filled >> s) & 1u) mbar_wait(&full_bar[s], (fill_parity >> s) & 1u, &never);
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      const uint32_t idesc = idesc_bf16(kRBM, p.n_mma);
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      for (int i = 0; i < nkt; ++i) {
        if (!mbar_wait(&full_bar[stage], phase, abort_flag)) {
          *abort_flag = 1;
          atomicExch(p.status, kDevTimeout);
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t sA = smem_u32(smem + stage * stage_bytes);
        const uint64_t adesc = sdesc_sw128(sA), bdesc = sdesc_sw128(sA + kRAbytes);
#pragma unroll
        for (int j = 0; j < 4; ++j)      // 16 bf16 = 32 bytes of K per MMA
          mma_bf16(tmem, adesc + 2 * j, bdesc + 2 * j, idesc, (i > 0 || j > 0) ? 1u : 0u);
        tc_commit(&empty_bar[stage]);
        if (++stage == p.stages) {
          stage = 0;
          phase ^= 1u;
        }
      }
      tc_commit(&acc_bar);
      if (!ok) {
        volatile int never = 0;
        mbar_wait(&acc_bar, 0, &never);
      }
    }
  } else {
    const int quad = warp & 3;
    if (mbar_wait(&acc_bar, 0, abort_flag)) {
      tc_fence_after();
      const uint32_t tbase = tmem + ((uint32_t)(quad * 32) << 16);
      // The warp's 32 rows go through shared memory (the pipeline's stages,
      // idle once every MMA has completed) and leave as one contiguous block
      // of partial[split] with coalesced stores.
      float* stg = reinterpret_cast<float*>(smem) + (size_t)quad * 32 * p.E;
      const bool vec = (p.E & 3) == 0;   // rows of 16-byte multiples
      for (int c = 0; c < p.n_mma; c += 32) {
        uint32_t r[32];
        tmem_ld32(tbase + c, r);
        tmem_ld_wait();
        float* srow = stg + (size_t)lane * p.E + c;
        if (vec) {
#pragma unroll
          for (int i = 0; i < 32; i += 4)
            if (c + i < p.E)
              *reinterpret_cast<float4*>(srow + i) = make_float4(__uint_as_float(r[i]), __uint_as_float(r[i + 1]),
                                                                  __uint_as_float(r[i + 2]), __uint_as_float(r[i + 3]));
        } else {
#pragma unroll
          for (int i = 0; i < 32; ++i)
            if (c + i < p.E) srow[i] = __uint_as_float(r[i]);
        }
      }
      __syncwarp();
      const int row0 = mt * kRBM + quad * 32;
      const size_t n = (size_t)max(0, min(32, p.T - row0)) * p.E;
      float* dst = p.partial + ((size_t)blockIdx.y * p.T + row0) * p.E;
      if (vec) {
        const float4* s4 = reinterpret_cast<const float4*>(stg);
        float4* d4 = reinterpret_cast<float4*>(dst);
        for (size_t i = lane; i < n / 4; i += 32) d4[i] = s4[i];
      } else {
        for (size_t i = lane; i < n; i += 32) dst[i] = stg[i];
      }
    } else {
      *abort_flag = 1;
      atomicExch(p.status, kDevTimeout);
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, tcols);
  }
}

// ---------------------------------------------------------------------------
// Top-k: the logits (split-ordered sums of the router GEMM's partials), then
// sigma and the selection key of sigma + bias for every (token, expert), then
// k selection rounds per token by one warp, each a warp-wide argmax of
// sigma + bias (ties to the lower expert).
// ---------------------------------------------------------------------------
constexpr int kMaxE = 256, kMaxK = 16;

// Logit of (token t, expert e).  With splits > 0 it is the split-ordered sum
// of the router GEMM's partial sums (plus the optional offset), loaded kBatch
// at a time so that they are in flight together, and is written to
// `logits`; with splits == 0 `src` already holds the logits, and with
// splits < 0 it holds logits that this kernel wrote itself.
template <int kBatch = 8>
NVDEV float token_logit(const float* __restrict__ src, int splits, const float* __restrict__ offset,
                        float* __restrict__ logits, int T, int E, int t, int e) {
  const float* p = src + (size_t)t * E + e;
  if (splits == 0) return *p;
  if (splits < 0) return __ldcg(p);      // written earlier by this kernel: read through L2
  const size_t stride = (size_t)T * E;
  float l = 0.0f;
  for (int q0 = 0; q0 < splits; q0 += kBatch) {
    float v[kBatch];
#pragma unroll
    for (int u = 0; u < kBatch; ++u) v[u] = (q0 + u < splits) ? p[(size_t)(q0 + u) * stride] : 0.0f;
#pragma unroll
    for (int u = 0; u < kBatch; ++u)
      if (q0 + u < splits) l = (q0 + u == 0) ? v[u] : __fadd_rn(l, v[u]);
  }
  if (offset) l = __fadd_rn(l, offset[e]);
  logits[(size_t)t * E + e] = l;
  return l;
}

// Score of one (token, expert) logit: sigma, and the selection key of
// sigma + bias mapped to an unsigned integer in the same order (sign bit
// flipped for non-negative values, all bits for negative ones; sigma > 0, so
// the sum is never -0).
NVDEV void expert_score(float l, float b, float& sig, uint32_t& key) {
  sig = sigmoid_fixed(l);
  const uint32_t u = __float_as_uint(__fadd_rn(sig, b));
  key = (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// The k selection rounds of one token by one warp, from each lane's scores
// of experts lane, lane+32, ... (PER slots per lane, PER * 32 >= E; key 0
// for an absent expert).  Each round is a warp max of the keys, then a warp
// min of the expert ids that reach it: the largest score, ties to the lower
// expert.  Lane j < k returns slot j's expert and weight (sigma / sum of the
// selected sigmas, times rsf; the sum in slot order).  An absent expert's
// key 0 never wins a round, so every PER that covers E gives the same result.
template <int PER>
NVDEV void select_topk(const float* sig, uint32_t* key, int k, float rsf, int lane, int& out_idx, float& out_w) {
  float sum = 0.0f, my_sig = 0.0f;
  int my_idx = 0;
  for (int j = 0; j < k; ++j) {
    uint32_t bk = 0u, be = 0xffffffffu;
#pragma unroll
    for (int i = 0; i < PER; ++i)              // ascending i: a tie keeps the lower expert
      if (key[i] > bk) {
        bk = key[i];
        be = (uint32_t)(lane + 32 * i);
      }
    const uint32_t m = __reduce_max_sync(0xffffffffu, bk);
    const int win = (int)__reduce_min_sync(0xffffffffu, bk == m ? be : 0xffffffffu);
    // the owner lane marks the winner and broadcasts its sigma
    float s_own = 0.0f;
#pragma unroll
    for (int i = 0; i < PER; ++i)
      if (lane + 32 * i == win) {
        s_own = sig[i];
        key[i] = 0u;
      }
    const float s_sel = __shfl_sync(0xffffffffu, s_own, win & 31);
    sum = __fadd_rn(sum, s_sel);
    if (lane == j) {
      my_sig = s_sel;
      my_idx = win;
    }
  }
  out_idx = my_idx;
  out_w = __fmul_rn(__fdiv_rn(my_sig, sum), rsf);
}

// Top-k of one token whose scores sit in shared memory: sigma bits at
// s_sig[e], selection keys at s_key[e], e < E.
template <int PER>
NVDEV void select_topk_smem(const uint32_t* s_sig, const uint32_t* s_key, int E, int k, float rsf, int lane,
                            int& idx, float& w) {
  float sig[PER];
  uint32_t key[PER];
#pragma unroll
  for (int i = 0; i < PER; ++i) {
    const int e = lane + 32 * i;
    sig[i] = e < E ? __uint_as_float(s_sig[e]) : 0.0f;
    key[i] = e < E ? s_key[e] : 0u;
  }
  select_topk<PER>(sig, key, k, rsf, lane, idx, w);
}

// The same for any E <= 256, with the fewest slots per lane that cover E.
NVDEV void select_topk_smem_any(const uint32_t* s_sig, const uint32_t* s_key, int E, int k, float rsf, int lane,
                                int& idx, float& w) {
  switch ((E + 31) >> 5) {
    case 1: select_topk_smem<1>(s_sig, s_key, E, k, rsf, lane, idx, w); break;
    case 2: select_topk_smem<2>(s_sig, s_key, E, k, rsf, lane, idx, w); break;
    case 3: select_topk_smem<3>(s_sig, s_key, E, k, rsf, lane, idx, w); break;
    case 4: select_topk_smem<4>(s_sig, s_key, E, k, rsf, lane, idx, w); break;
    default: select_topk_smem<kMaxE / 32>(s_sig, s_key, E, k, rsf, lane, idx, w); break;
  }
}

// ---------------------------------------------------------------------------
// Larger batches (more than 256 tokens): two kernels.
//
// topk_bitmap_kernel: one block per 32 tokens.  Its threads compute every
// (token, expert) logit, sigma and selection key of the block's tokens into
// shared memory, one pair per thread and step; then one warp per token runs
// the selection rounds from there.  The block's tokens that chose expert e
// form one 32-bit word (bit = token's place in the block), written to
// bm[block][e], and its popcount to blk_counts[e][block].  The kernel also
// fills perm with -1 and row_w with 0 over the padded capacity.
//
// perm_scan_scatter_kernel: one block per 256 tokens.  Each block sums
// blk_counts per expert (one warp per expert) into the totals and the
// exclusive prefix of its own 32-token blocks, pads the totals to 128 rows
// and scans them into the experts' first rows, then places each of its
// (token, slot) pairs: row = expert's first row + rows of the expert's
// earlier blocks + popcount of the lower bits of the block's word.  That is
// the token's rank among the expert's tokens, so rows keep token order.
// Block 0 also writes expert_offsets, the counts and the m-tile map.
// Everything after the scores is integer and order-independent.
// ---------------------------------------------------------------------------
constexpr int kTkTokens = 32;                      // tokens per top-k block: one bitmap word
constexpr int kTkThreads = 1024;                   // one warp per token for the selection
constexpr int kTkPairs = kTkTokens * kMaxE / kTkThreads;   // (token, expert) pairs per thread, at most 8
constexpr int kScWords = 8;                        // bitmap words per scatter block
constexpr int kScTokens = kScWords * kTkTokens;    // 256 tokens
constexpr int kScThreads = 1024;

// In-place exclusive scan of sp[0..256) by warp 0 of the block (eight entries
// per lane, then a shuffle scan of the lane sums); the caller synchronises
// the block before and after.
NVDEV void warp0_exclusive_scan256(int32_t* sp) {
  if ((threadIdx.x >> 5) != 0) return;
  const int lane = threadIdx.x & 31;
  int ex[8], run = 0;
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    ex[j] = run;
    run += sp[lane * 8 + j];
  }
  int inc = run;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, inc, o);
    if (lane >= o) inc += y;
  }
#pragma unroll
  for (int j = 0; j < 8; ++j) sp[lane * 8 + j] = inc - run + ex[j];
}

// Dynamic shared memory of topk_bitmap_kernel: sigma bits and keys of the
// block's 32 tokens (64 KiB at E = 256).
inline int topk_bitmap_smem_bytes(int E) { return 2 * kTkTokens * E * (int)sizeof(uint32_t); }

__global__ void __launch_bounds__(kTkThreads, 1) topk_bitmap_kernel(
    const float* __restrict__ src, int splits, const float* __restrict__ offset, float* __restrict__ logits,
    const float* __restrict__ bias, int T, int E, int k, float rsf, int cap, int32_t* __restrict__ topk_idx,
    float* __restrict__ topk_w, uint32_t* __restrict__ bm, int32_t* __restrict__ blk_counts, int nblk,
    int32_t* __restrict__ perm, float* __restrict__ row_w) {
  extern __shared__ uint32_t s_score[];           // [32 * E] sigma bits, then [32 * E] keys
  __shared__ uint32_t s_bm[kMaxE];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  for (int e = tid; e < E; e += blockDim.x) s_bm[e] = 0u;
  griddep_wait();
  griddep_launch();
  for (int i = blockIdx.x * blockDim.x + tid; i < cap; i += gridDim.x * blockDim.x) {
    perm[i] = -1;
    row_w[i] = 0.0f;
  }
  const int t0 = blockIdx.x * kTkTokens;
  const int nt = min(kTkTokens, T - t0);
  const int np = nt * E;                          // the block's pairs are src[t0 * E + i], i < np
  // the logits of this thread's pairs i = tid + j * 1024: the split-ordered
  // sum of the partials, two splits' loads of every pair in flight at once
  float acc[kTkPairs];
  if (splits > 0) {
    const size_t stride = (size_t)T * E;
    const float* base = src + (size_t)t0 * E;
    for (int u0 = 0; u0 < splits; u0 += 2) {
      float v[2][kTkPairs];
#pragma unroll
      for (int uu = 0; uu < 2; ++uu)
#pragma unroll
        for (int j = 0; j < kTkPairs; ++j) {
          const int i = tid + j * kTkThreads;
          v[uu][j] = (u0 + uu < splits && i < np) ? base[(size_t)(u0 + uu) * stride + i] : 0.0f;
        }
#pragma unroll
      for (int uu = 0; uu < 2; ++uu)
#pragma unroll
        for (int j = 0; j < kTkPairs; ++j)
          if (u0 + uu < splits) acc[j] = (u0 + uu == 0) ? v[uu][j] : __fadd_rn(acc[j], v[uu][j]);
    }
  } else {
#pragma unroll
    for (int j = 0; j < kTkPairs; ++j) {
      const int i = tid + j * kTkThreads;
      acc[j] = i < np ? src[(size_t)t0 * E + i] : 0.0f;
    }
  }
#pragma unroll
  for (int j = 0; j < kTkPairs; ++j) {
    const int i = tid + j * kTkThreads;
    if (i < np) {
      const int e = i % E;
      float l = acc[j];
      if (splits > 0) {
        if (offset) l = __fadd_rn(l, offset[e]);
        logits[(size_t)t0 * E + i] = l;
      }
      float sig;
      uint32_t key;
      expert_score(l, bias[e], sig, key);
      s_score[i] = __float_as_uint(sig);
      s_score[kTkTokens * E + i] = key;
    }
  }
  __syncthreads();
  if (warp < nt) {
    int idx;
    float w;
    select_topk_smem_any(s_score + warp * E, s_score + kTkTokens * E + warp * E, E, k, rsf, lane, idx, w);
    if (lane < k) {
      topk_idx[(size_t)(t0 + warp) * k + lane] = idx;
      topk_w[(size_t)(t0 + warp) * k + lane] = w;
      atomicOr(&s_bm[idx], 1u << warp);
    }
  }
  __syncthreads();
  for (int e = tid; e < E; e += blockDim.x) {
    const uint32_t word = s_bm[e];
    bm[(size_t)blockIdx.x * E + e] = word;
    blk_counts[(size_t)e * nblk + blockIdx.x] = __popc(word);
  }
}

__global__ void __launch_bounds__(kScThreads, 1) perm_scan_scatter_kernel(
    const int32_t* __restrict__ topk_idx, const float* __restrict__ topk_w, int T, int E, int k,
    const uint32_t* __restrict__ bm, const int32_t* __restrict__ blk_counts, int nblk,
    int32_t* __restrict__ counts, int32_t* __restrict__ offsets, int32_t* __restrict__ tile_expert,
    int32_t* __restrict__ num_mtiles, int32_t* __restrict__ perm, int32_t* __restrict__ inv_perm,
    float* __restrict__ row_w) {
  __shared__ int32_t sp[256];
  __shared__ int32_t s_total[kMaxE];
  __shared__ int32_t s_pre[kMaxE][kScWords];       // rows of expert e in the 32-token blocks before b0 + s
  griddep_wait();
  griddep_launch();
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int b0 = blockIdx.x * kScWords;
  // one warp per expert; lane l sums the block counts [l * per, (l + 1) * per)
  const int per = (nblk + 31) >> 5;
  const int lo = min(lane * per, nblk), hi = min(lo + per, nblk);
  for (int e = warp; e < E; e += blockDim.x >> 5) {
    const int32_t* row = blk_counts + (size_t)e * nblk;
    int sum = 0;
#pragma unroll 8
    for (int b = lo; b < hi; ++b) sum += row[b];
    int inc = sum;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, inc, o);
      if (lane >= o) inc += y;
    }
    if (lane == 31) s_total[e] = inc;
    if (hi > b0 && lo < b0 + kScWords) {           // this lane's range holds some of the block's words
      int run = inc - sum;
      for (int b = lo; b < hi && b < b0 + kScWords; ++b) {
        if (b >= b0) s_pre[e][b - b0] = run;
        run += row[b];
      }
    }
  }
  __syncthreads();
  const int total = tid < E ? s_total[tid] : 0;
  const int padded = (total + kRowTile - 1) / kRowTile * kRowTile;
  if (tid < 256) sp[tid] = tid < E ? padded : 0;
  __syncthreads();
  warp0_exclusive_scan256(sp);
  __syncthreads();
  if (blockIdx.x == 0 && tid < E) {
    const int start = sp[tid];
    offsets[tid] = start;
    counts[tid] = total;
    for (int m = start / kRowTile; m < (start + padded) / kRowTile; ++m) tile_expert[m] = tid;
    if (tid == E - 1) {
      offsets[E] = start + padded;
      *num_mtiles = (start + padded) / kRowTile;
    }
  }
  // the block's (token, slot) pairs, consecutive pairs to consecutive threads
  const int p0 = blockIdx.x * kScTokens * k;
  const int np = min(kScTokens, T - blockIdx.x * kScTokens) * k;
  for (int q = tid; q < np; q += blockDim.x) {
    const int t = (p0 + q) / k;
    const int e = topk_idx[p0 + q];
    const int b = t >> 5;
    const int row = sp[e] + s_pre[e][b - b0] + __popc(bm[(size_t)b * E + e] & ((1u << (t & 31)) - 1u));
    perm[row] = t;
    inv_perm[p0 + q] = row;
    row_w[row] = topk_w[p0 + q];
  }
}

// ---------------------------------------------------------------------------
// Routing of a small batch (T <= 256) in one block: top-k, per-expert counts,
// the padded scan, and the scatter, with the padding fill of perm and row_w
// that the large-batch path does in its top-k kernel.  The scores (sigma and
// the selection key) are computed one (token, expert) per thread and kept in
// shared memory, so a token's warp only runs the selection rounds.  The
// arithmetic is the large-batch path's (expert_score, select_topk) and so
// is every integer result.  For small layers (route_fuses_x_quantise) the
// kernel also quantises x and writes it to the permuted rows, the work of the
// layer's quantise-scatter kernel, with the same bits.
// ---------------------------------------------------------------------------
constexpr int kSmallT = 256;
constexpr int kSmallThreads = 1024;

// Dynamic shared memory of the small-batch kernel: the scores of a chunk of
// tokens between the two phases, sigma (fp32) and the selection key (u32) of
// each (token, expert); every pair's top-k id, weight and permuted row; and,
// when the kernel also quantises x, each token's codes and scale bytes.
constexpr int kScoreSmemBytes = 64 * 1024;
constexpr int kRouteSmallMaxDyn = 200 * 1024;
__host__ __device__ inline int route_small_chunk_tokens(int T, int E) { return min(T, kScoreSmemBytes / (8 * E)); }
__host__ __device__ inline int route_small_xq_offset(int T, int E, int k) {   // bytes before x's codes, 16-byte aligned
  return (route_small_chunk_tokens(T, E) * E * 8 + T * k * 12 + 15) / 16 * 16;
}
int route_small_smem_bytes(int T, int E, int k, int H, bool quant_x) {
  return quant_x ? route_small_xq_offset(T, E, k) + T * (H / 2 + H / kQBlock) : route_small_chunk_tokens(T, E) * E * 8 + T * k * 12;
}
// Every permuted row of x then leaves through this one block.  Measured on
// B200: at 16 tokens x 8 slots of H = 6144 (442 KB of rows) the fused kernel
// took 39.6 us against 18.5 + 8.1 us for routing plus the separate quantise
// kernel, while at 32 x 2 slots of H = 256 (9 KB) the layer's step went down
// by 7 %.  So the fusion is kept to 64 KiB of rows.
constexpr long long kFusedXRowBytes = 64 * 1024;
bool route_fuses_x_quantise(int T, int H, int k) {
  return T <= kSmallT && (long long)T * k * (H / 2 + H / kQBlock) <= kFusedXRowBytes &&
         route_small_xq_offset(T, kMaxE, k) + T * (H / 2 + H / kQBlock) <= kRouteSmallMaxDyn;
}

__global__ void __launch_bounds__(kSmallThreads, 1)
    route_small_kernel(const float* __restrict__ src, int splits, const float* __restrict__ offset,
                       float* __restrict__ logits, const float* __restrict__ bias, int T, int E, int k, float rsf,
                       int cap, int chunk_t, int32_t* __restrict__ topk_idx, float* __restrict__ topk_w,
                       int32_t* __restrict__ counts, int32_t* __restrict__ offsets,
                       int32_t* __restrict__ tile_expert, int32_t* __restrict__ num_mtiles,
                       int32_t* __restrict__ perm, int32_t* __restrict__ inv_perm, float* __restrict__ row_w,
                       int quant_x, const uint4* __restrict__ x, int H, const float* __restrict__ act_gscale,
                       uint8_t* __restrict__ a_codes, uint8_t* __restrict__ a_scales) {
  __shared__ uint32_t bm[kMaxE][kSmallT / 32];
  __shared__ int32_t sp[256];
  __shared__ int32_t base[kMaxE];
  extern __shared__ uint32_t s_score[];          // [chunk_t * E] sigma bits, then [chunk_t * E] keys
  int32_t* s_idx = reinterpret_cast<int32_t*>(s_score + 2 * chunk_t * E);   // [T * k]
  float* s_w = reinterpret_cast<float*>(s_idx + T * k);                     // [T * k]
  int32_t* s_row = reinterpret_cast<int32_t*>(s_w + T * k);                 // [T * k]
  // quantised x: [T][H/2] codes, then [T][H/16] scale bytes
  uint8_t* xq_c = reinterpret_cast<uint8_t*>(s_score) + (quant_x ? route_small_xq_offset(T, E, k) : 0);
  uint8_t* xq_s = xq_c + (size_t)T * (H / 2);
  const int nblk = H / kQBlock;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  // the router GEMM before this kernel writes none of these, so the fill
  // overlaps it
  for (int i = tid; i < E * (kSmallT / 32); i += blockDim.x) bm[i / (kSmallT / 32)][i % (kSmallT / 32)] = 0;
  for (int i = tid; i < cap; i += blockDim.x) {
    perm[i] = -1;
    row_w[i] = 0.0f;
  }
  if (quant_x) {
    // x and g1 are the layer's inputs, complete once the router GEMM ahead of
    // this kernel has started (it waited for their producer), so they are
    // quantised here, before the wait, exactly as the quantise-scatter kernel
    // does: one 16-element block per thread and step, read through L2
    const BlockScaler bs = make_scaler(act_gscale[0]);
    for (int b = tid; b < T * nblk; b += blockDim.x) {
      uint2 c;
      const uint32_t sc = quant_block16_bf16(__ldcg(x + (size_t)b * 2), __ldcg(x + (size_t)b * 2 + 1), bs, c);
      reinterpret_cast<uint2*>(xq_c)[b] = c;
      xq_s[b] = (uint8_t)sc;
    }
  }
  griddep_wait();
  griddep_launch();
  for (int t0 = 0; t0 < T; t0 += chunk_t) {
    const int nt = min(chunk_t, T - t0);
    // every (token, expert) of the chunk, one per thread: the logit (the
    // split-ordered sum of the partials; the decode shape has 24 splits, all
    // loaded in one batch), then sigma and the selection key
    for (int i = tid; i < nt * E; i += blockDim.x) {
      const int t = t0 + i / E, e = i % E;
      const float l = splits > 0 ? token_logit<24>(src, splits, offset, logits, T, E, t, e) : src[(size_t)t * E + e];
      float sig;
      uint32_t key;
      expert_score(l, bias[e], sig, key);
      s_score[i] = __float_as_uint(sig);
      s_score[chunk_t * E + i] = key;
    }
    __syncthreads();
    // top-k, one warp per token
    for (int tt = warp; tt < nt; tt += blockDim.x >> 5) {
      const int t = t0 + tt;
      int idx;
      float w;
      select_topk_smem_any(s_score + tt * E, s_score + chunk_t * E + tt * E, E, k, rsf, lane, idx, w);
      if (lane < k) {
        topk_idx[(size_t)t * k + lane] = idx;
        topk_w[(size_t)t * k + lane] = w;
        s_idx[t * k + lane] = idx;
        s_w[t * k + lane] = w;
        atomicOr(&bm[idx][t >> 5], 1u << (t & 31));
      }
    }
    __syncthreads();
  }
  // per-expert totals, 128-row padding, exclusive scan (threads 0..255)
  int total = 0, padded = 0;
  if (tid < E)
    for (int w = 0; w < kSmallT / 32; ++w) total += __popc(bm[tid][w]);
  padded = (total + kRowTile - 1) / kRowTile * kRowTile;
  if (tid < 256) sp[tid] = tid < E ? padded : 0;
  __syncthreads();
  warp0_exclusive_scan256(sp);
  __syncthreads();
  if (tid < E) {
    const int start = sp[tid];
    base[tid] = start;
    offsets[tid] = start;
    counts[tid] = total;
    for (int m = start / kRowTile; m < (start + padded) / kRowTile; ++m) tile_expert[m] = tid;
    if (tid == E - 1) {
      offsets[E] = start + padded;
      *num_mtiles = (start + padded) / kRowTile;
    }
  }
  __syncthreads();
  // stable scatter: rank of token t among the tokens of expert e
  for (int i = tid; i < T * k; i += blockDim.x) {
    const int t = i / k;
    const int e = s_idx[i];
    int rank = __popc(bm[e][t >> 5] & ((1u << (t & 31)) - 1u));
    for (int w = 0; w < (t >> 5); ++w) rank += __popc(bm[e][w]);
    const int row = base[e] + rank;
    perm[row] = t;
    inv_perm[i] = row;
    row_w[row] = s_w[i];
    s_row[i] = row;
  }
  if (quant_x) {
    // each token's codes and scales to its k rows: 16-byte code chunks, and
    // the tiled scale layout's 4-block words
    __syncthreads();
    const int cpr = H / 32;
    for (int i = tid; i < T * k * cpr; i += blockDim.x) {
      const int pair = i / cpr, ch = i % cpr;
      reinterpret_cast<uint4*>(a_codes + (size_t)s_row[pair] * (H / 2))[ch] =
          reinterpret_cast<const uint4*>(xq_c + (size_t)(pair / k) * (H / 2))[ch];
    }
    const int wpr = nblk / 4;
    for (int i = tid; i < T * k * wpr; i += blockDim.x) {
      const int pair = i / wpr, w = i % wpr;
      *reinterpret_cast<uint32_t*>(a_scales + tiled_scale_offset(s_row[pair], 4 * w, nblk >> 2)) =
          *reinterpret_cast<const uint32_t*>(xq_s + (size_t)(pair / k) * nblk + 4 * w);
    }
  }
}

// Opts a routing kernel into `bytes` of dynamic shared memory, once per
// device (`done` is that kernel's own table).
template <typename Kernel>
static nvfp4_status allow_dyn_smem(Kernel kernel, int bytes, bool* done) {
  static std::mutex mu;
  int dev = 0;
  NV_CHECK(check_cuda(cudaGetDevice(&dev), "cudaGetDevice"));
  if (dev < 0 || dev >= 64) dev = 63;
  std::lock_guard<std::mutex> lock(mu);
  if (!done[dev]) {
    NV_CHECK(check_cuda(cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes),
                        "cudaFuncSetAttribute"));
    done[dev] = true;
  }
  return NVFP4_OK;
}

static nvfp4_status allow_route_small_smem() {
  static bool done[64] = {};
  return allow_dyn_smem(route_small_kernel, kRouteSmallMaxDyn, done);
}

static nvfp4_status allow_topk_bitmap_smem() {
  static bool done[64] = {};
  return allow_dyn_smem(topk_bitmap_kernel, topk_bitmap_smem_bytes(kMaxE), done);
}

RouteScratch carve_route_scratch(Carver& c, int T, int E, int k) {
  RouteScratch r;
  const int nblk = (T + kTkTokens - 1) / kTkTokens;
  const int cap = route_rows_capacity(T, E, k);
  r.status = c.take<uint32_t>(64);
  r.bm = c.take<uint32_t>((size_t)nblk * E);
  r.blk_counts = c.take<int32_t>((size_t)nblk * E);
  r.counts = c.take<int32_t>((size_t)E);
  r.tile_expert = c.take<int32_t>((size_t)cap / kRowTile + 1);
  r.num_mtiles = c.take<int32_t>(1);
  r.row_w = c.take<float>((size_t)cap);
  // router_splits() never exceeds ceil(148 / m-tiles), whatever H is
  const int mt = std::max(1, (T + kRBM - 1) / kRBM);
  r.partial = c.take<float>((size_t)((148 + mt - 1) / mt) * T * E);
  return r;
}

int route_rows_capacity(int T, int E, int k) {
  const long long rows = (long long)T * k + (long long)E * (kRowTile - 1);
  return (int)((rows + kRowTile - 1) / kRowTile * kRowTile);
}

nvfp4_status launch_route(const RouteArgs& a, const RouteScratch& r, cudaStream_t s) {
  const int cap = route_rows_capacity(a.T, a.E, a.k);
  int splits = 0;
  if (a.x) {
    splits = router_splits(a.T, a.H);
    const int n_mma = router_n_mma(a.E);
    CUtensorMap tmX, tmW;
    NV_CHECK(make_tmap_2d(&tmX, a.x, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, (uint64_t)a.H, (uint64_t)a.T,
                          (uint64_t)a.H * 2, kRBK, kRBM));
    NV_CHECK(make_tmap_2d(&tmW, a.router_weight, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, (uint64_t)a.H, (uint64_t)a.E,
                          (uint64_t)a.H * 2, kRBK, (uint32_t)n_mma));
    RouterGemmParams p;
    p.T = a.T; p.E = a.E; p.H = a.H; p.n_mma = n_mma;
    p.kt_per_split = (a.H / kRBK + splits - 1) / splits;
    p.splits = splits;
    p.clear_status = a.clear_status ? 1 : 0;
    p.stages = router_stages(a.E);
    p.partial = r.partial;
    p.status = r.status;
    const int smem = router_smem_bytes(a.E);
    // the epilogue stages the 128 x E fp32 tile in the pipeline's buffers
    NV_REQUIRE(smem - 1024 >= kRBM * a.E * (int)sizeof(float), NVFP4_ERR_UNSUPPORTED_SHAPE,
               "router: E=%d does not fit the epilogue's staging", a.E);
    NV_CHECK(check_cuda(cudaFuncSetAttribute(router_gemm_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem),
                        "cudaFuncSetAttribute"));
    dim3 grid((a.T + kRBM - 1) / kRBM, splits);
    // a programmatic dependent too: its setup overlaps the previous kernel on
    // the stream, and it waits for that kernel before reading x
    NV_CHECK(launch_dependent("router_gemm_kernel", router_gemm_kernel, grid, dim3(kRThreads), smem, s, tmX, tmW, p));
  }
  if (a.T <= kSmallT) {
    const int chunk_t = route_small_chunk_tokens(a.T, a.E);
    const bool qx = a.quant_x && route_fuses_x_quantise(a.T, a.H, a.k);
    const int smem = route_small_smem_bytes(a.T, a.E, a.k, a.H, qx);
    NV_CHECK(allow_route_small_smem());
    return launch_dependent("route_small_kernel", route_small_kernel, dim3(1), dim3(kSmallThreads), smem, s,
                            (const float*)(splits ? r.partial : a.logits), splits, a.logit_offset, a.logits, a.bias,
                            a.T, a.E, a.k, a.rsf, cap, chunk_t, a.topk_idx, a.topk_w, r.counts, a.expert_offsets,
                            r.tile_expert, r.num_mtiles, a.perm, a.inv_perm, r.row_w, qx ? 1 : 0,
                            static_cast<const uint4*>(a.x), a.H, a.act_gscale, a.a_codes, a.a_scales);
  }
  // both kernels wait for their predecessor's results (griddepcontrol.wait)
  // before reading them, so programmatic launch only hides the launch latency
  const int nblk = (a.T + kTkTokens - 1) / kTkTokens;
  NV_CHECK(allow_topk_bitmap_smem());
  NV_CHECK(launch_dependent("topk_bitmap_kernel", topk_bitmap_kernel, dim3(nblk), dim3(kTkThreads),
                            topk_bitmap_smem_bytes(a.E), s, (const float*)(splits ? r.partial : a.logits), splits,
                            a.logit_offset, a.logits, a.bias, a.T, a.E, a.k, a.rsf, cap, a.topk_idx, a.topk_w, r.bm,
                            r.blk_counts, nblk, a.perm, r.row_w));
  return launch_dependent("perm_scan_scatter_kernel", perm_scan_scatter_kernel,
                          dim3((a.T + kScTokens - 1) / kScTokens), dim3(kScThreads), 0, s,
                          (const int32_t*)a.topk_idx, (const float*)a.topk_w, a.T, a.E, a.k, (const uint32_t*)r.bm,
                          (const int32_t*)r.blk_counts, nblk, r.counts, a.expert_offsets, r.tile_expert,
                          r.num_mtiles, a.perm, a.inv_perm, r.row_w);
}

nvfp4_status check_route_shape(int T, int H, int E, int k) {
  NV_REQUIRE(T >= 1 && E >= 1 && k >= 1, NVFP4_ERR_INVALID_ARG, "route: T=%d E=%d k=%d", T, E, k);
  NV_REQUIRE(k <= kMaxK && k <= E && E <= kMaxE, NVFP4_ERR_UNSUPPORTED_SHAPE,
             "route: needs 1 <= k <= 16 and k <= E <= 256 (k=%d E=%d)", k, E);
  NV_REQUIRE(H % 64 == 0 && H > 0, NVFP4_ERR_UNSUPPORTED_SHAPE, "route: H=%d must be a positive multiple of 64", H);
  NV_REQUIRE((long long)T * k + (long long)E * 128 < (1ll << 30), NVFP4_ERR_UNSUPPORTED_SHAPE,
             "route: T*k=%lld too large", (long long)T * k);
  return NVFP4_OK;
}

}  // namespace nvfp4moe

using namespace nvfp4moe;

extern "C" int moe_route_rows_capacity(int T, int E, int k) {
  if (T < 0 || E < 0 || k < 0) return 0;
  return route_rows_capacity(T, E, k);
}

extern "C" size_t moe_route_workspace_size(int T, int E, int k) {
  if (T < 0 || E < 0 || k < 0) return 0;
  Carver c(nullptr);
  carve_route_scratch(c, T, E, k);
  c.take<float>((size_t)T * E);     // logits when the caller does not keep them
  return c.size();
}

extern "C" nvfp4_status moe_route(const void* x_bf16, const void* router_weight_bf16, const float* logits_in,
                                  const float* bias, const float* logit_offset, int T, int H, int E, int k,
                                  float routed_scaling_factor, float* logits_out, int32_t* topk_idx, float* topk_w,
                                  int32_t* expert_offsets, int32_t* perm, int32_t* inv_perm, void* ws,
                                  size_t ws_bytes, void* stream) {
  NV_REQUIRE(bias && topk_idx && topk_w && expert_offsets && perm && inv_perm, NVFP4_ERR_INVALID_ARG,
             "moe_route: a required pointer is NULL");
  if (logits_in) {
    NV_REQUIRE(!x_bf16 && !router_weight_bf16 && !logit_offset, NVFP4_ERR_INVALID_ARG,
               "moe_route: with logits_in, x, router weight and logit_offset must be NULL");
    NV_CHECK(check_route_shape(T, 64, E, k));
  } else {
    NV_REQUIRE(x_bf16 && router_weight_bf16, NVFP4_ERR_INVALID_ARG, "moe_route: x and router weight are required");
    NV_REQUIRE(aligned(x_bf16, 16) && aligned(router_weight_bf16, 16), NVFP4_ERR_INVALID_ARG,
               "moe_route: x and router weight need 16-byte alignment");
    NV_CHECK(check_route_shape(T, H, E, k));
  }
  const size_t need = moe_route_workspace_size(T, E, k);
  NV_REQUIRE(ws && ws_bytes >= need && aligned(ws, 256), NVFP4_ERR_WORKSPACE,
             "moe_route: needs a 256-byte aligned workspace of %zu bytes", need);
  int sms = 0;
  NV_CHECK(device_sm_count(&sms));
  cudaStream_t s = as_stream(stream);
  Carver c(ws);
  RouteScratch r = carve_route_scratch(c, T, E, k);
  float* own_logits = c.take<float>((size_t)T * E);
  NV_CHECK(check_cuda(cudaMemsetAsync(r.status, 0, sizeof(uint32_t), s), "clear status word"));
  RouteArgs a;
  a.x = logits_in ? nullptr : x_bf16;
  a.router_weight = router_weight_bf16;
  a.logit_offset = logit_offset;
  a.bias = bias;
  a.T = T; a.H = H; a.E = E; a.k = k; a.rsf = routed_scaling_factor;
  a.topk_idx = topk_idx; a.topk_w = topk_w; a.expert_offsets = expert_offsets; a.perm = perm; a.inv_perm = inv_perm;
  if (logits_in) {
    a.logits = const_cast<float*>(logits_in);
  } else {
    a.logits = logits_out ? logits_out : own_logits;
  }
  NV_CHECK(launch_route(a, r, s));
  if (logits_in && logits_out)
    NV_CHECK(check_cuda(cudaMemcpyAsync(logits_out, logits_in, sizeof(float) * (size_t)T * E,
                                        cudaMemcpyDeviceToDevice, s), "copy logits"));
  return NVFP4_OK;
}
