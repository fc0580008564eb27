// NVFP4 quantisers: the dynamic activation quantiser and the offline RTN
// weight quantiser ("K-EXAONE-152B-A23B-REAP-80E-NVFP4" model card, section
// "Quantization Setup").  Both are HBM-bound streams: 128-bit loads of bf16,
// 64-bit stores of packed codes, one scale byte per 16 elements.
#include <algorithm>
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
  const BlockScaler bs = make_scaler(*gscale);
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
      s = quant_block16_bf16(u0, u1, bs, c);
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
// Weights: one cooperative launch (every CTA resident, one per SM).  Each CTA
// owns an even share of every matrix and runs two streams over it side by
// side.  Each stream is a ring of 16 KiB shared-memory chunks that its own
// producer warp fills with bulk asynchronous copies (the copy engine holds the
// bytes in flight, not registers), and eight consumer warps drain:
//   * the amax stream reads matrix after matrix from HBM (L2 evict_last); its
//     consumers keep a running max and, at the end of each matrix, publish
//     one atomic max and one completion count.  Its producer stays at most
//     one matrix ahead of this CTA's quantise consumers, so the matrices in
//     flight stay in L2;
//   * the quantise stream's producer waits (bounded) until every CTA has
//     published matrix m's amax, then re-reads this CTA's share from L2
//     (evict_first); its consumers write codes and tiled scales.
// Waits only ever point at earlier work, so with all CTAs resident they
// always end.
// ---------------------------------------------------------------------------
// Quantising a block costs far more instructions than taking its max, so the
// quantise stream gets four times the amax stream's consumer warps.  One
// 1024-thread CTA per SM: with two CTAs per SM the later one fell behind by
// a fifth, and every matrix waits for the slowest CTA.
constexpr int kWChunkBlocks = 768;                       // 16-element blocks per chunk
constexpr int kWChunkBytes = kWChunkBlocks * 32;         // 24 KiB of bf16
constexpr int kWSlotsA = 4;                              // ring depth of the amax stream (HBM)
constexpr int kWSlotsQ = 3;                              // ring depth of the quantise stream (L2)
constexpr int kWAmaxConsumers = 192;                     // 8 x 16 bytes of each chunk per thread
constexpr int kWQuantConsumers = 768;                    // one block of each chunk per thread
constexpr int kWThreads = 64 + kWAmaxConsumers + kWQuantConsumers;   // + one producer warp per stream
// The amax stream may start matrix m once this CTA's quantise consumers are
// no more than `lead` eighths of a matrix behind it: (8 m - lead) / 8
// matrices' worth of chunks done.  The matrices in flight (the lead plus the
// one being quantised) must stay in L2 for the quantise stream's re-read,
// and the amax stream should not stall at the end of every quantise pass.
// The lead is sized from an L2 budget of kWL2BudgetBytes: for 25 MB matrices
// 20 eighths (2.5 matrices) measured 3 % faster than 14, and 24 or more made
// the re-read miss L2 and took 20 % longer.
constexpr long long kWL2BudgetBytes = 84ll << 20;
constexpr int kWLeadMin = 8, kWLeadMax = 64;
static int weight_lead_eighths(long long mat_bytes) {
  const long long lead = 8 * kWL2BudgetBytes / (mat_bytes > 0 ? mat_bytes : 1) - 8;
  return (int)std::min<long long>(kWLeadMax, std::max<long long>(kWLeadMin, lead));
}
constexpr int kWDynSmem = (kWSlotsA + kWSlotsQ) * kWChunkBytes + 128;
// warp roles
constexpr int kWAmaxProducer = 0;                        // warp 0
constexpr int kWQuantProducer = 1;                       // warp 1
constexpr int kWAmaxWarp0 = 2;                           // warps 2..7
constexpr int kWQuantWarp0 = 2 + kWAmaxConsumers / 32;   // warps 8..31
static_assert(kWChunkBlocks % kWQuantConsumers == 0 && (2 * kWChunkBlocks) % kWAmaxConsumers == 0,
              "chunks split evenly over the consumers");
static_assert(kWChunkBlocks % 4 == 0, "a chunk holds whole 4-block scale words");

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
// cp.async.bulk global -> shared with an L2 cache policy.
NVDEV void bulk_load_hint(void* dst, const void* src, uint32_t bytes, uint64_t* bar, uint64_t pol) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint [%0], [%1], %2, [%3], %4;" ::
          "r"(smem_u32(dst)),
      "l"(src), "r"(bytes), "r"(smem_u32(bar)), "l"(pol)
      : "memory");
}
template <int N>
NVDEV void group_sync(int id) { asm volatile("bar.sync %0, %1;" ::"r"(id), "n"(N) : "memory"); }
// Named-barrier AND over the N threads of a group: every thread gets the same
// answer, so a group leaves its loops together.
template <int N>
NVDEV bool group_all(int id, bool v) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.u32 p, %1, 0;\n\t"
      "bar.red.and.pred q, %2, %3, p;\n\t"
      "selp.u32 %0, 1, 0, q;\n\t}"
      : "=r"(r)
      : "r"((uint32_t)v), "r"(id), "n"(N)
      : "memory");
  return r != 0;
}

// The producer side of one stream: fills ring slots in order with this CTA's
// share of matrices [0, n_mats).  `ready(mat)` is a bounded wait for the
// stream's precondition on matrix mat (it returns false on give-up).  Before
// returning it waits for every copy it issued, so none lands after the CTA
// exits.
template <int SLOTS, class Ready>
NVDEV void weight_stream_producer(const uint8_t* w, long long mat_bytes, long long byte_begin, long long byte_end,
                                  int n_mats, uint8_t* ring, uint64_t* full, uint64_t* empty, uint64_t pol,
                                  volatile int* abort_flag, uint32_t* status, Ready ready) {
  int slot = 0;
  uint32_t phase = 0;
  uint32_t filled = 0, fill_parity = 0;
  bool ok = true;
  for (int mat = 0; ok && mat < n_mats; ++mat) {
    if (!ready(mat)) {
      ok = false;
      break;
    }
    for (long long off = byte_begin; off < byte_end; off += kWChunkBytes) {
      if (!mbar_wait(&empty[slot], phase ^ 1u, abort_flag)) {
        ok = false;
        break;
      }
      const uint32_t bytes = (uint32_t)min((long long)kWChunkBytes, byte_end - off);
      mbar_arrive_expect_tx(&full[slot], bytes);
      bulk_load_hint(ring + slot * kWChunkBytes, w + mat * mat_bytes + off, bytes, &full[slot], pol);
      filled |= 1u << slot;
      fill_parity = (fill_parity & ~(1u << slot)) | (phase << slot);
      if (++slot == SLOTS) {
        slot = 0;
        phase ^= 1u;
      }
    }
  }
  if (!ok) {
    *abort_flag = 1;
    atomicExch(status, kDevTimeout);
  }
  volatile int never = 0;
  for (int s = 0; s < SLOTS; ++s)
    if ((filled >> s) & 1u) mbar_wait(&full[s], (fill_parity >> s) & 1u, &never);
}

__global__ void __launch_bounds__(kWThreads, 1) quantize_weights_kernel(
    const uint4* __restrict__ w, int n_mats, int rows, int cols, int layout, uint2* __restrict__ codes,
    uint8_t* __restrict__ scales, float* __restrict__ gscale, WeightQuantState* st, uint32_t* amax_bits,
    uint32_t* done, int lead) {
  extern __shared__ uint8_t wq_smem_raw[];
  uint8_t* ring_a = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(wq_smem_raw) + 127) & ~uintptr_t(127));
  uint8_t* ring_q = ring_a + kWSlotsA * kWChunkBytes;
  __shared__ __align__(8) uint64_t full_a[kWSlotsA], empty_a[kWSlotsA], full_q[kWSlotsQ], empty_q[kWSlotsQ];
  __shared__ uint32_t s_red[kWAmaxConsumers / 32];
  __shared__ float s_amax[4];                   // amax of matrix m at [m % 4], set by the quantise producer
  __shared__ float s_inv[2][256];               // matrix m's 1 / (E4M3(s) g) for every scale code s, at [m % 2]
  __shared__ volatile int quantised;            // matrices this CTA's quantise consumers have finished
  __shared__ unsigned int q_chunk_warps;        // (chunk, warp) pairs the quantise consumers have finished
  __shared__ int abort_s;
  volatile int* abort_flag = &abort_s;
  const long long per_mat = (long long)rows * cols;
  const long long blocks = per_mat / kQBlock;                  // 16-element blocks per matrix
  const int nblk = cols / kQBlock;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // this CTA's share of every matrix, in whole groups of 4 blocks
  const long long share = ((blocks + gridDim.x - 1) / gridDim.x + 3) / 4 * 4;
  const long long b_begin = min(blocks, share * blockIdx.x), b_end = min(blocks, b_begin + share);
  const int n_chunks = (int)((b_end - b_begin + kWChunkBlocks - 1) / kWChunkBlocks);
  if (threadIdx.x == 0) {
    for (int i = 0; i < kWSlotsA; ++i) {
      mbar_init(&full_a[i], 1);
      mbar_init(&empty_a[i], kWAmaxConsumers / 32);
    }
    for (int i = 0; i < kWSlotsQ; ++i) {
      mbar_init(&full_q[i], 1);
      mbar_init(&empty_q[i], kWQuantConsumers / 32);
    }
    quantised = 0;
    q_chunk_warps = 0;
    abort_s = 0;
    fence_barrier_init();
  }
  __syncthreads();
  const uint8_t* wb = reinterpret_cast<const uint8_t*>(w);

  if (warp == kWAmaxProducer) {
    // ------------------------------------------------------------ amax producer
    if (lane == 0) {
      auto gate = [&](int mat) {
        const long long need_eighths = 8ll * mat - lead;
        if (need_eighths <= 0) return true;
        const long long need = (need_eighths * n_chunks + 7) / 8 * (kWQuantConsumers / 32);
        const uint64_t t0 = globaltimer_ns();
        while ((long long)*reinterpret_cast<volatile unsigned int*>(&q_chunk_warps) < need) {
          if (*abort_flag || globaltimer_ns() - t0 > kWaitLimitNs) return false;
        }
        return true;
      };
      weight_stream_producer<kWSlotsA>(wb, per_mat * 2, b_begin * 32, b_end * 32, n_mats, ring_a, full_a, empty_a,
                             l2_policy_evict_last(), abort_flag, &st->status, gate);
    }
  } else if (warp == kWQuantProducer) {
    // ------------------------------------------------------------ quantise producer
    if (lane == 0) {
      auto amax_ready = [&](int mat) {
        const uint64_t t0 = globaltimer_ns();
        while (ld_acquire_u32(done + mat) < gridDim.x) {
          if (*abort_flag || globaltimer_ns() - t0 > kWaitLimitNs) return false;
        }
        // published before the matrix's first chunk is announced, so the
        // consumers see it once that chunk's barrier completes
        s_amax[mat & 3] = __uint_as_float(ld_acquire_u32(amax_bits + mat));
        return true;
      };
      weight_stream_producer<kWSlotsQ>(wb, per_mat * 2, b_begin * 32, b_end * 32, n_mats, ring_q, full_q, empty_q,
                             l2_policy_evict_first(), abort_flag, &st->status, amax_ready);
    }
  } else if (warp < kWQuantWarp0) {
    // ------------------------------------------------------------ amax consumers
    const int gt = threadIdx.x - kWAmaxWarp0 * 32;
    int slot = 0;
    uint32_t phase = 0;
    bool ok = true;
    for (int mat = 0; mat < n_mats; ++mat) {
      // running max of |x| on packed bf16 pairs (exact; sign bits cleared at the end)
      uint32_t m2 = 0u;
      for (int c = 0; ok && c < n_chunks; ++c) {
        if (!mbar_wait(&full_a[slot], phase, abort_flag)) {
          ok = false;
          break;
        }
        const long long c0 = b_begin + (long long)c * kWChunkBlocks;
        const int nvec = (int)min((long long)kWChunkBlocks, b_end - c0) * 2;     // uint4 in this chunk
        const uint4* src = reinterpret_cast<const uint4*>(ring_a + slot * kWChunkBytes);
#pragma unroll
        for (int i = 0; i < 2 * kWChunkBlocks / kWAmaxConsumers; ++i) {
          const int v = gt + i * kWAmaxConsumers;
          if (v < nvec) {
            const uint4 u = src[v];
            const uint32_t ws[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
            for (int j = 0; j < 4; ++j) m2 = max_abs_bf16x2(m2, ws[j]);
          }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty_a[slot]);
        if (++slot == kWSlotsA) {
          slot = 0;
          phase ^= 1u;
        }
      }
      m2 &= 0x7FFF7FFFu;
      const float m = fmaxf(__uint_as_float(m2 << 16), __uint_as_float(m2 & 0xFFFF0000u));
      uint32_t mb = __float_as_uint(m);
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) mb = max(mb, __shfl_xor_sync(0xffffffffu, mb, o));
      if (lane == 0) s_red[gt >> 5] = mb;
      ok = group_all<kWAmaxConsumers>(1, ok && !*abort_flag);
      if (gt == 0) {
        uint32_t bm = 0;
        for (int q = 0; q < kWAmaxConsumers / 32; ++q) bm = max(bm, s_red[q]);
        atomicMax(amax_bits + mat, bm);         // non-negative floats order like their bits
        __threadfence();
        atomicAdd(done + mat, 1u);
      }
      group_sync<kWAmaxConsumers>(1);
      if (!ok) {
        // publish the remaining matrices so that no other CTA waits on them
        if (gt == 0)
          for (int mm = mat + 1; mm < n_mats; ++mm) atomicAdd(done + mm, 1u);
        *abort_flag = 1;
        atomicExch(&st->status, kDevTimeout);
        break;
      }
    }
  } else {
    // ------------------------------------------------------------ quantise consumers
    const int gt = threadIdx.x - kWQuantWarp0 * 32;
    int slot = 0;
    uint32_t phase = 0;
    bool ok = true;
    // (row, block column) of this thread's block in chunk 0; each further
    // chunk moves it kWChunkBlocks blocks on
    const long long bt0 = b_begin + gt;
    const int row_t0 = (int)(bt0 / nblk), kb_t0 = (int)(bt0 % nblk);
    const int step_rows = kWChunkBlocks / nblk, step_kb = kWChunkBlocks % nblk;
    for (int mat = 0; ok && mat < n_mats; ++mat) {
      float g = 0.0f;
      BlockScaler bs = make_scaler(0.0f);
      int row = row_t0, kb = kb_t0;
      float* inv_tab = s_inv[mat & 1];
      for (int c = 0; c < n_chunks; ++c) {
        const bool landed = mbar_wait(&full_q[slot], phase, abort_flag);
        if (c == 0) {
          // the matrix's global scale and, for each of the 256 scale codes,
          // the reciprocal its blocks multiply by: 1 / (E4M3(s) g), 0 for 0.
          // Every warp takes part in the barrier, landed or not.
          if (landed) {
            g = __fdiv_rn(s_amax[mat & 3], 2688.0f);
            bs = make_scaler(g);
            if (gt < 256) {
              const float S = __fmul_rn(e4m3_value((uint32_t)gt), g);
              inv_tab[gt] = (S == 0.0f) ? 0.0f : __frcp_rn(S);
            }
          }
          if (!group_all<kWQuantConsumers>(2, landed)) {
            ok = false;
            break;
          }
        } else if (!landed) {
          ok = false;
          break;
        }
        const long long c0 = b_begin + (long long)c * kWChunkBlocks;
        const int nb = (int)min((long long)kWChunkBlocks, b_end - c0);
        const uint4* src = reinterpret_cast<const uint4*>(ring_q + slot * kWChunkBytes);
        const int j = gt;                             // this thread's block within the chunk
        if (j < nb) {
          const uint4 u0 = src[2 * j], u1 = src[2 * j + 1];
          const uint32_t w8[8] = {u0.x, u0.y, u0.z, u0.w, u1.x, u1.y, u1.z, u1.w};
          const uint32_t sc = e4m3_code(block_scale_raw(amax16_bf16(w8), bs));
          const float inv = inv_tab[sc];
          const uint64_t inv2 = pack_f32x2(inv, inv);
          float y[16];
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            const uint64_t r = mul_f32x2(((uint64_t)(w8[i] & 0xFFFF0000u) << 32) | (uint64_t)(w8[i] << 16), inv2);
            y[2 * i] = lo_f32(r);
            y[2 * i + 1] = hi_f32(r);
          }
          codes[(long long)mat * blocks +
                (layout == NVFP4_LAYOUT_STAGED ? (long long)staged_code_unit(row, kb, nblk) : c0 + j)] =
              make_uint2(e2m1x8_hw(y), e2m1x8_hw(y + 8));
          const int srow = mat * rows + row;
          scales[layout == NVFP4_LAYOUT_CANONICAL ? (size_t)srow * nblk + kb
                                                  : tiled_scale_offset(srow, kb, nblk >> 2)] = (uint8_t)sc;
        }
        row += step_rows;
        kb += step_kb;
        if (kb >= nblk) {
          kb -= nblk;
          ++row;
        }
        __syncwarp();
        if (lane == 0) {
          mbar_arrive(&empty_q[slot]);
          atomicAdd(&q_chunk_warps, 1u);
        }
        if (++slot == kWSlotsQ) {
          slot = 0;
          phase ^= 1u;
        }
      }
      if (ok && n_chunks == 0) {
        // an empty share still waits for the matrix so that its gscale is written
        const uint64_t t0 = globaltimer_ns();
        while (ld_acquire_u32(done + mat) < gridDim.x)
          if (*abort_flag || globaltimer_ns() - t0 > kWaitLimitNs) {
            ok = false;
            break;
          }
        if (ok) g = __fdiv_rn(__uint_as_float(ld_acquire_u32(amax_bits + mat)), 2688.0f);
      }
      if (blockIdx.x == 0 && gt == 0 && ok) gscale[mat] = g;
      ok = group_all<kWQuantConsumers>(2, ok);
      if (gt == 0 && ok) quantised = mat + 1;
    }
    if (!ok) {
      *abort_flag = 1;
      atomicExch(&st->status, kDevTimeout);
    }
  }
  __syncthreads();
}

// Cooperative launch: the phases need every CTA resident at once.
static nvfp4_status launch_weight_quantiser(const void* w_bf16, int n_mats, int rows, int cols, int layout,
                                           uint8_t* codes, uint8_t* scales, float* global_scale,
                                           WeightQuantState* st, uint32_t* amax, uint32_t* done, int sms,
                                           cudaStream_t s) {
  {
    static std::mutex mu;
    static bool attr_set[64] = {};
    int dev = 0;
    NV_CHECK(check_cuda(cudaGetDevice(&dev), "cudaGetDevice"));
    std::lock_guard<std::mutex> lock(mu);
    if (dev < 0 || dev >= 64 || !attr_set[dev]) {
      NV_CHECK(check_cuda(cudaFuncSetAttribute(quantize_weights_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                               kWDynSmem),
                          "cudaFuncSetAttribute"));
      if (dev >= 0 && dev < 64) attr_set[dev] = true;
    }
  }
  int per_sm = 0;
  NV_CHECK(check_cuda(
      cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, quantize_weights_kernel, kWThreads, kWDynSmem),
      "occupancy"));
  NV_REQUIRE(per_sm >= 1, NVFP4_ERR_CUDA, "quantize_weights_kernel cannot be resident");
  per_sm = 1;
  const uint4* w = static_cast<const uint4*>(w_bf16);
  uint2* c = reinterpret_cast<uint2*>(codes);
  int lead = weight_lead_eighths((long long)rows * cols * 2);
  void* args[] = {(void*)&w, (void*)&n_mats, (void*)&rows, (void*)&cols, (void*)&layout, (void*)&c,
                  (void*)&scales, (void*)&global_scale, (void*)&st, (void*)&amax, (void*)&done, (void*)&lead};
  return check_cuda(cudaLaunchCooperativeKernel((const void*)quantize_weights_kernel, dim3(sms * per_sm),
                                                dim3(kWThreads), args, kWDynSmem, s),
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

// Layout and shape checks shared by both weight-quantiser entry points.
static nvfp4_status check_weight_layout(const char* fn, int layout, int rows, int cols) {
  NV_REQUIRE(layout == NVFP4_LAYOUT_CANONICAL || layout == NVFP4_LAYOUT_TILED || layout == NVFP4_LAYOUT_STAGED,
             NVFP4_ERR_INVALID_ARG, "%s: unknown layout %d", fn, layout);
  NV_REQUIRE(cols % 32 == 0, NVFP4_ERR_UNSUPPORTED_SHAPE, "%s: cols=%d must be a multiple of 32", fn, cols);
  NV_REQUIRE(layout == NVFP4_LAYOUT_CANONICAL || (cols % 64 == 0 && rows % 128 == 0), NVFP4_ERR_UNSUPPORTED_SHAPE,
             "%s: the tiled and staged layouts need rows %% 128 == 0 and cols %% 64 == 0 (got %d x %d)", fn, rows,
             cols);
  NV_REQUIRE(layout != NVFP4_LAYOUT_STAGED || cols % 256 == 0, NVFP4_ERR_UNSUPPORTED_SHAPE,
             "%s: the staged layout needs cols %% 256 == 0 (got %d)", fn, cols);
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
  NV_CHECK(check_weight_layout("nvfp4_quantize_weights", layout, rows, cols));
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

// Device address of the scratch array in the current context.  The host
// symbol is only a stand-in and must never be passed to a kernel.  A
// __device__ array's address belongs to a CUDA context, not to a device (a
// host may switch between its own contexts on one device, or reset the
// device), so it is looked up on every call: a cheap host-side query.
static nvfp4_status static_scratch_address(uint8_t** out) {
  void* p = nullptr;
  NV_CHECK(check_cuda(cudaGetSymbolAddress(&p, g_weight_quant_scratch), "cudaGetSymbolAddress"));
  *out = static_cast<uint8_t*>(p);
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
  NV_CHECK(check_weight_layout("nvfp4_quantize_weights_noalloc", layout, rows, cols));
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

extern "C" nvfp4_status nvfp4_quantize_weights_noalloc_status(void* stream) {
  using namespace nvfp4moe;
  uint8_t* scratch = nullptr;
  NV_CHECK(static_scratch_address(&scratch));
  // the status word is the first word of the scratch array (WeightQuantState)
  uint32_t word = 0;
  cudaStream_t s = as_stream(stream);
  NV_CHECK(check_cuda(cudaMemcpyAsync(&word, scratch, sizeof(word), cudaMemcpyDeviceToHost, s), "read status"));
  NV_CHECK(check_cuda(cudaStreamSynchronize(s), "cudaStreamSynchronize"));
  if (word != 0) {
    NV_CHECK(check_cuda(cudaMemsetAsync(scratch, 0, sizeof(word), s), "reset status"));
    NV_CHECK(check_cuda(cudaStreamSynchronize(s), "cudaStreamSynchronize"));
    return set_error(NVFP4_ERR_TIMEOUT, "nvfp4_quantize_weights_noalloc: a device-side wait gave up (status word %u)",
                     word);
  }
  return NVFP4_OK;
}
