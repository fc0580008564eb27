// Grouped block-scaled FP4 GEMMs of the routed experts on the 5th-generation
// tensor cores (tcgen05, sm_100a).
//
// The expert GEMMs of an NVFP4 W4A4 MoE layer ("K-EXAONE-152B-A23B-REAP-80E-
// NVFP4" model card, "Quantization Setup": E2M1 weights and activations with
// one E4M3 scale per 16 elements, per-expert Linear granularity; the global
// times block scale structure of the NetsPresso AQ article, "The Standard
// NVFP4 Serving Spec").  The block scales are applied inside the MMA
// (kind::mxf4nvf4, scale_vec::4X); the per-tensor global scales in the
// epilogue.
//
// Tile: 128 permuted rows x 256 weight rows x 256 K elements per stage.
//   gate/up: the 256 weight rows are 128 gate rows and the same 128 up rows,
//            so one tile yields 128 columns of h = silu(gate) * up, which the
//            epilogue re-quantises to NVFP4 (16-column blocks stay in-thread).
//   down:    256 output columns, scaled by g2 * g_down[e] * w(row).
// Warp roles (320 threads): warp 0 issues the loads (TMA for A and row-major
// weight codes, plain bulk copies for staged weight codes and the scale
// atoms), warp 1 owns tensor memory and issues MMAs, warps 2..9 drain the
// accumulator (warp w reads TMEM lanes 32*(w%4).., columns split in two
// halves).  The grid is persistent: one CTA
// per SM walks the (m-tile, n-tile) list, whose length is read on the device.
// Batches of at least 2048 rows run the FP4 kinds on CTA pairs (clusters of
// two sharing one 256-row MMA, each CTA loading half of B), whose down
// epilogue writes y by TMA tensor stores; at small batches the bf16 kinds of
// the shared expert split K over several CTAs and store fp32 partial sums.
// Every wait is bounded in time; a wait that gives up sets the workspace
// status word and the CTA winds down after its outstanding copies land.
#include <cstring>
#include <mutex>

#include "common.cuh"
#include "gemm.cuh"
#include "host.cuh"

namespace nvfp4moe {

constexpr int kBM = 128, kBN = 256;
constexpr int kBK = 256;                         // K elements per stage
constexpr int kBKBytes = kBK / 2;                // 128 bytes of packed FP4 per row
constexpr int kABytes = kBM * kBKBytes;          // 16 KiB
constexpr int kBBytes = kBN * kBKBytes;          // 32 KiB
constexpr int kSfaBytes = kBM * kBK / kQBlock;   // 2 KiB (4 scale atoms)
constexpr int kSfbBytes = kBN * kBK / kQBlock;   // 4 KiB (8 scale atoms)
constexpr int kStageBytes = kABytes + kBBytes + kSfaBytes + kSfbBytes;
constexpr int kThreads = 320;
constexpr int kEpiWarps = 8;
// Operand kinds: FP4 stages hold 256 K elements (128-byte rows) plus their
// scale atoms; bf16 stages hold 64 K elements in the same 128-byte rows and
// no scales, so the MMA descriptors advance identically (32 bytes per MMA).
// A CTA pair (PAIR) shares one 256 x 256 MMA: each CTA holds its own 128 A
// rows, half of the 256 B rows and all of B's scales, 38 KiB a stage.
template <int EPI> __host__ __device__ constexpr bool is_bf16() { return EPI >= kEpiSharedGateUp; }
template <int EPI> __host__ __device__ constexpr bool is_gate_up() {
  return EPI == kEpiGateUp || EPI == kEpiSharedGateUp;
}
// B rows one CTA loads per stage: all 256, or its half of the pair's tile
template <bool PAIR> __host__ __device__ constexpr int b_rows_of() { return PAIR ? kBN / 2 : kBN; }
template <int EPI, bool PAIR> __host__ __device__ constexpr int stage_bytes_of() {
  return PAIR ? kABytes + b_rows_of<PAIR>() * kBKBytes + kSfaBytes + kSfbBytes
              : (is_bf16<EPI>() ? kABytes + kBBytes : kStageBytes);
}
template <int EPI> __host__ __device__ constexpr int bk_of() { return is_bf16<EPI>() ? 64 : kBK; }
// Pipeline stages: four in every one-CTA kind, five for a CTA pair (38 KiB
// a stage per CTA).  The down
// GEMMs stage y in shared memory, 32 rows x y_pass_cols_of() bf16 columns per
// warp at a time: 64 columns (4 KiB) for the bf16 kind and the CTA pair, 16
// (1 KiB) for the one-CTA FP4 kind, whose four stages leave no room for more.
template <int EPI, bool PAIR> __host__ __device__ constexpr int stages_of() { return PAIR ? 5 : 4; }
template <int EPI, bool PAIR> __host__ __device__ constexpr int y_pass_cols_of() {
  return EPI == kEpiDown && !PAIR ? 16 : 64;
}
template <int EPI, bool PAIR> __host__ __device__ constexpr int y_stage_bytes_of() {
  return 32 * y_pass_cols_of<EPI, PAIR>() * 2;
}
template <int EPI, bool PAIR> __host__ __device__ constexpr int smem_bytes_of() {
  return stages_of<EPI, PAIR>() * stage_bytes_of<EPI, PAIR>() + 1024 +
         (is_gate_up<EPI>() ? 0 : kEpiWarps * y_stage_bytes_of<EPI, PAIR>());
}
static_assert(smem_bytes_of<kEpiDown, false>() <= 232448 - 256, "FP4 down GEMM shared memory");
static_assert(smem_bytes_of<kEpiGateUp, false>() <= 232448 - 256, "FP4 gate/up GEMM shared memory");
static_assert(smem_bytes_of<kEpiSharedDown, false>() <= 232448 - 256, "bf16 down GEMM shared memory");
static_assert(smem_bytes_of<kEpiDown, true>() <= 232448 - 2048, "FP4 down GEMM (CTA pair) shared memory");
static_assert(smem_bytes_of<kEpiGateUp, true>() <= 232448 - 2048, "FP4 gate/up GEMM (CTA pair) shared memory");
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kAccCol = 0;                  // 256 fp32 accumulator columns
// Scale factors of one stage: 4 MMA k-steps x (4 SFA + 8 SFB) columns.  The
// copies and MMAs of one thread run in issue order, so every stage reuses the
// same 48 columns.
constexpr uint32_t kSfCol = 256;
constexpr uint32_t kSfaOff = 0, kSfbOff = 16;
constexpr int kMaxExperts = 256;

struct GemmParams {
  const uint8_t* a_sf;
  const uint8_t* b0_sf;
  const uint8_t* b1_sf;
  int K;                // reduction length (elements)
  int E;                // experts (tile_expert entries are clamped to [0, E))
  int Nw;               // weight rows per expert in B0 / B1
  int n_tiles;          // n-tiles per m-tile
  int cap_tiles;        // 128-row tiles in the row capacity (CTA pairs: tiles past it are skipped)
  const int32_t* tile_expert;
  const int32_t* num_mtiles;
  const int32_t* expert_offsets;
  const int32_t* expert_counts;
  const float* g_act;
  const float* g_b0;
  const float* g_b1;
  const float* g_h;
  uint8_t* h_codes;
  uint8_t* h_sf;
  float* h_f32;
  float* h_amax;
  int I;
  const float* row_w;
  uint16_t* y_bf16;
  float* y_f32;
  float* y_sq_part;
  uint16_t* h_bf16;
  int H;
  int per_expert;       // g_act, g_h and h_amax are [E] arrays
  // B codes in the staged layout: each 128-row group of a stage is one
  // contiguous 16 KiB tile, fetched with a plain bulk copy instead of TMA
  int b_staged;
  const uint8_t* b0_codes;
  const uint8_t* b1_codes;
  uint32_t* status;
  // split K (bf16 kinds): each (m-tile, n-tile) is ksplit tiles over K / ksplit
  // elements, whose epilogues store fp32 partial sums of their data rows to
  // partial [ksplit][partial_rows][2I (gate/up: gate then up) or H (down)]
  int ksplit;
  int partial_rows;
  float* partial;
};

// Tensor maps only the CTA-pair kernel reads: the scale atoms as rows of 512
// bytes (A's and B's; b1 is up's for gate/up), loaded by TMA so that their
// bytes count on the leader CTA's stage barrier.
struct PairMaps {
  CUtensorMap sfa, sfb0, sfb1;
  // down: y as bf16 [rows][H], boxes of 32 rows x 64 columns, 128-byte
  // swizzle; written by TMA stores (all zero when y_bf16 is NULL)
  CUtensorMap y;
};

NVDEV void give_up(uint32_t* status, volatile int* abort_flag) {
  *abort_flag = 1;
  if (status) atomicExch(status, kDevTimeout);
}

// A CTA of a pair that gives up also raises the other CTA's abort flag, so
// that its waits end at once instead of running into their own limits.
NVDEV void give_up_pair(uint32_t* status, volatile int* abort_flag, uint32_t peer_abort_addr) {
  give_up(status, abort_flag);
  asm volatile("st.relaxed.cluster.shared::cluster.u32 [%0], 1;" ::"r"(peer_abort_addr) : "memory");
}


// A tile of the work list: its expert, its 128-row m-tile in this CTA, its
// n-tile, and whether this CTA stores anything (the second CTA of a pair
// whose expert has an odd number of m-tiles has no rows of its own).
struct TileCoord {
  int e, mt, nt;
  int ks;               // split-K part (bf16 kinds at small batches; 0 otherwise)
  bool valid;
};

template <int EPI>
__global__ void __launch_bounds__(kThreads, 1)
    grouped_fp4_gemm_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmA32,
                            const __grid_constant__ CUtensorMap tmB0, const __grid_constant__ CUtensorMap tmB1,
                            const GemmParams p);

// PAIR = false: one CTA per SM, each walking (m-tile, n-tile) tiles of 128 x 256.
// PAIR = true: clusters of two CTAs; a pair walks (pair of m-tiles of one
// expert, n-tile) tiles of 256 x 256 with one .cta_group::2 MMA per k-step.
template <int EPI, bool PAIR>
NVDEV void gemm_body(const CUtensorMap& tmA, const CUtensorMap& tmA32, const CUtensorMap& tmB0,
                     const CUtensorMap& tmB1, const PairMaps* pm, const GemmParams& p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  constexpr int kStages = stages_of<EPI, PAIR>();
  constexpr bool kBf16 = is_bf16<EPI>();
  constexpr bool kGateUp = is_gate_up<EPI>();
  constexpr int kSB = stage_bytes_of<EPI, PAIR>();
  constexpr int kBRows = b_rows_of<PAIR>();
  constexpr int kBLoad = kBRows * kBKBytes;                   // B bytes this CTA loads per stage
  static_assert(!PAIR || !kBf16, "CTA pairs run the FP4 GEMMs only");
  __shared__ __align__(8) uint64_t full_bar[kStages];
  __shared__ __align__(8) uint64_t empty_bar[kStages];
  __shared__ __align__(8) uint64_t acc_full_bar;
  __shared__ __align__(8) uint64_t acc_empty_bar;
  __shared__ __align__(8) uint64_t drain_bar;
  __shared__ uint32_t tmem_base_s;
  __shared__ int abort_s;
  __shared__ int pair_start[PAIR ? kMaxExperts + 1 : 1];   // first pair m-tile of each expert
  volatile int* abort_flag = &abort_s;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = PAIR ? cluster_ctarank() : 0u;
  const bool leader = rank == 0;
  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      // pair: only the leader's producer arrives on the leader's stage
      // barrier, expecting the bytes of both CTAs
      mbar_init(&full_bar[s], 1);
      mbar_init(&empty_bar[s], 1);
    }
    mbar_init(&acc_full_bar, 1);
    // pair: the leader's accumulator is drained by both CTAs' epilogues
    mbar_init(&acc_empty_bar, PAIR ? 2 * kEpiWarps : kEpiWarps);
    mbar_init(&drain_bar, 1);
    abort_s = 0;
    fence_barrier_init();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tmap(&tmA);
    prefetch_tmap(&tmA32);
    prefetch_tmap(&tmB0);
    if (kGateUp) prefetch_tmap(&tmB1);
    if constexpr (PAIR) {
      prefetch_tmap(&pm->sfa);
      prefetch_tmap(&pm->sfb0);
      prefetch_tmap(&pm->sfb1);
      if (EPI == kEpiDown && p.y_bf16) prefetch_tmap(&pm->y);
    }
  }
  if (warp == 1) {
    if constexpr (PAIR) {
      tmem_alloc_pair(&tmem_base_s, kTmemCols);
      tmem_relinquish_pair();
    } else {
      tmem_alloc(&tmem_base_s, kTmemCols);
      tmem_relinquish();
    }
  }
  tc_fence_before();
  if constexpr (PAIR) {
    cluster_sync_all();          // both CTAs' barriers exist before either touches the other's
  } else {
    __syncthreads();
  }
  tc_fence_after();
  const uint32_t tmem = tmem_base_s;
  // shared::cluster addresses of the leader's barriers and of the other CTA's abort flag
  const uint32_t peer_abort = PAIR ? mapa_shared(smem_u32(&abort_s), rank ^ 1u) : 0u;
  // everything above overlaps the previous kernel; its outputs are read below
  griddep_wait();
  griddep_launch();

  int num_tiles;
  if constexpr (PAIR) {
    // pair m-tiles per expert: ceil(m-tiles / 2); exclusive prefix in shared memory
    if (warp == 0) {
      int carry = 0;
      for (int e0 = 0; e0 < p.E; e0 += 32) {
        const int e = e0 + lane;
        int v = 0;
        if (e < p.E) {
          const int mt = max(0, (p.expert_offsets[e + 1] - p.expert_offsets[e]) / kBM);
          v = (mt + 1) >> 1;
        }
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const int u = __shfl_up_sync(0xffffffffu, v, o);
          if (lane >= o) v += u;
        }
        if (e < p.E) pair_start[e + 1] = carry + v;
        carry += __shfl_sync(0xffffffffu, v, 31);
      }
      if (lane == 0) pair_start[0] = 0;
    }
    __syncthreads();
    num_tiles = pair_start[p.E] * p.n_tiles;
  } else {
    num_tiles = (*p.num_mtiles) * p.n_tiles * p.ksplit;
  }
  // tile t of the work list: one-CTA tiles are (m-tile, n-tile); pair tiles
  // are (pair m-tile, n-tile), this CTA taking the pair's m-tile `rank`
  auto tile_of = [&](int t) -> TileCoord {
    TileCoord c;
    c.ks = 0;
    if constexpr (PAIR) {
      c.nt = t % p.n_tiles;
      const int pmt = t / p.n_tiles;
      int lo = 0, hi = p.E - 1;                  // the last expert whose pairs start at or before pmt
      while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (pair_start[mid] <= pmt) lo = mid; else hi = mid - 1;
      }
      c.e = lo;
      const int j = pmt - pair_start[lo];
      const int e_mt = (p.expert_offsets[lo + 1] - p.expert_offsets[lo]) / kBM;
      const int first = p.expert_offsets[lo] / kBM + 2 * j;
      c.valid = (2 * j + (int)rank < e_mt) && first + (int)rank < p.cap_tiles;
      // a CTA without rows of its own loads the pair's first m-tile again
      c.mt = c.valid ? first + (int)rank : min(first, p.cap_tiles - 1);
    } else {
      // split K: the ksplit parts of one (m-tile, n-tile) are consecutive tiles
      const int tt = t / p.ksplit;
      c.ks = t - tt * p.ksplit;
      c.nt = tt % p.n_tiles;
      c.mt = tt / p.n_tiles;
      c.e = min(max(p.tile_expert[c.mt], 0), p.E - 1);
      c.valid = true;
    }
    return c;
  };
  // each CTA of a pair strides over pair tiles by cluster
  const int t_first = PAIR ? (int)(blockIdx.x >> 1) : (int)blockIdx.x;
  const int t_step = PAIR ? (int)(gridDim.x >> 1) : (int)gridDim.x;
  // K stages per tile (a split-K tile covers K / ksplit)
  const int KT = (p.K + bk_of<EPI>() - 1) / bk_of<EPI>() / p.ksplit;
  const int nblk4 = p.K / 64;                    // FP4: scale atoms per 128-row tile

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    // The whole warp runs the loop (waits and bookkeeping stay warp-uniform);
    // one elected lane issues the copies.
    const uint32_t elected = elect_one();
    int stage = 0;
    uint32_t phase = 0;
    uint32_t filled = 0, fill_parity = 0;       // per stage: ever filled / parity of last fill
    bool ok = true;
    uint8_t* const st0 = smem;
    const size_t tile_sf_bytes = (size_t)nblk4 * kAtomBytes;       // one 128-row tile's scales
    for (int t = t_first; ok && t < num_tiles; t += t_step) {
      const TileCoord tc = tile_of(t);
      const int e = tc.e, mt = tc.mt, nt = tc.nt;
      const int arow = mt * kBM;
      const int brow = e * p.Nw + nt * (kGateUp ? 128 : kBN);
      const uint8_t* asf = kBf16 ? nullptr : p.a_sf + (size_t)mt * tile_sf_bytes;
      const uint8_t* bsf0 = kBf16 ? nullptr : p.b0_sf + (size_t)(brow / kRowTile) * tile_sf_bytes;
      const uint8_t* bsf1 = kBf16 ? nullptr
                                  : (kGateUp ? p.b1_sf + (size_t)(brow / kRowTile) * tile_sf_bytes
                                             : bsf0 + tile_sf_bytes);
      // A rows to load: the tile's data rows rounded up to 32-row boxes (a
      // decode tile holds a handful of tokens).  Rows past them keep stale
      // shared memory; they only feed accumulator rows the epilogue never
      // stores.  Pairs load whole tiles.
      int a_boxes = 4;
      if (!PAIR && p.expert_counts) {
        const int real = p.expert_counts[e] - (arow - p.expert_offsets[e]);
        a_boxes = min(4, max(1, (real + 31) / 32));
      }
      const uint32_t a_bytes = (uint32_t)a_boxes * (kABytes / 4);
      for (int kt = 0; kt < KT; ++kt) {
        ok = __all_sync(0xffffffffu, mbar_wait(&empty_bar[stage], phase ^ 1u, abort_flag));
        if (!ok) {
          if (elected) {
            if constexpr (PAIR) give_up_pair(p.status, abort_flag, peer_abort);
            else give_up(p.status, abort_flag);
          }
          break;
        }
        if (elected) {
          uint8_t* sA = st0 + stage * kSB;
          uint8_t* sB = sA + kABytes;
          // x in tensor-map elements: 128 bytes of K per stage either way
          const int x = (tc.ks * KT + kt) * (kBf16 ? 64 : kBKBytes);
          if constexpr (PAIR) {
            // every load of both CTAs counts on the leader's stage barrier,
            // which the leader alone arms with the bytes of both; the other
            // CTA's bytes may land first (the barrier's phase cannot complete
            // before the leader's arrival)
            const uint32_t fb = mapa_shared(smem_u32(&full_bar[stage]), 0);
            if (leader) mbar_arrive_expect_tx(&full_bar[stage], 2u * (uint32_t)kSB);
            uint8_t* sSFA = sB + kBLoad;
            uint8_t* sSFB = sSFA + kSfaBytes;
            // scale atoms: rows of 512 bytes (128 32-bit words), 4 per stage
            const int ka = kt * 4;
            tma_load_2d_pair(sSFA, &pm->sfa, 0, mt * nblk4 + ka, fb);
            tma_load_2d_pair(sSFB, &pm->sfb0, 0, (brow / kRowTile) * nblk4 + ka, fb);
            if (kGateUp) {
              tma_load_2d_pair(sSFB + kSfbBytes / 2, &pm->sfb1, 0, (brow / kRowTile) * nblk4 + ka, fb);
            } else {
              tma_load_2d_pair(sSFB + kSfbBytes / 2, &pm->sfb0, 0, (brow / kRowTile + 1) * nblk4 + ka, fb);
            }
            tma_load_2d_pair(sA, &tmA, x, arow, fb);
            // B: gate/up - the leader loads the 128 gate rows, the other CTA
            // the same 128 up rows; down - each CTA 128 of the 256 rows
            const CUtensorMap* bm = (kGateUp && rank == 1) ? &tmB1 : &tmB0;
            const int bro = kGateUp ? brow : brow + (int)rank * kRowTile;
            if (p.b_staged) {
              // staged tiles viewed as rows of 128 bytes: tile (row group, stage)
              const int ks = p.K / kBK;
              tma_load_2d_pair(sB, bm, 0, ((bro / kRowTile) * ks + kt) * kRowTile, fb);
            } else {
              tma_load_2d_pair(sB, bm, x, bro, fb);
            }
          } else {
            if (kBf16) {
              mbar_arrive_expect_tx(&full_bar[stage], a_bytes + kBBytes);
            } else {
              const int katoms = min(4, (p.K - kt * kBK) / 64);
              const uint32_t sf_bytes = (uint32_t)katoms * kAtomBytes;
              mbar_arrive_expect_tx(&full_bar[stage], a_bytes + kBBytes + 3 * sf_bytes);
              uint8_t* sSFA = sB + kBBytes;
              uint8_t* sSFB = sSFA + kSfaBytes;
              const size_t sf_off = (size_t)kt * 4 * kAtomBytes;
              bulk_load(sSFA, asf + sf_off, sf_bytes, &full_bar[stage]);
              bulk_load(sSFB, bsf0 + sf_off, sf_bytes, &full_bar[stage]);
              bulk_load(sSFB + kSfbBytes / 2, bsf1 + sf_off, sf_bytes, &full_bar[stage]);
            }
            if (a_boxes == 4) {
              tma_load_2d(sA, &tmA, x, arow, &full_bar[stage]);
            } else {
              for (int i = 0; i < a_boxes; ++i)
                tma_load_2d(sA + i * (kABytes / 4), &tmA32, x, arow + 32 * i, &full_bar[stage]);
            }
            if (!kBf16 && p.b_staged) {
              // gate/up: the gate and up tiles of rows [brow, brow + 128);
              // down: the tiles of rows [brow, brow + 128) and the next 128
              const size_t ks = (size_t)(p.K / kBK);
              const size_t t0 = ((size_t)(brow / kRowTile) * ks + kt) * kStagedTileBytes;
              bulk_load(sB, p.b0_codes + t0, kStagedTileBytes, &full_bar[stage]);
              bulk_load(sB + kBBytes / 2, kGateUp ? p.b1_codes + t0 : p.b0_codes + t0 + ks * kStagedTileBytes,
                        kStagedTileBytes, &full_bar[stage]);
            } else {
              tma_load_2d(sB, &tmB0, x, brow, &full_bar[stage]);
              if (kGateUp) tma_load_2d(sB + kBBytes / 2, &tmB1, x, brow, &full_bar[stage]);
            }
          }
        }
        __syncwarp();
        filled |= 1u << stage;
        fill_parity = (fill_parity & ~(1u << stage)) | (phase << stage);
        if (++stage == kStages) {
          stage = 0;
          phase ^= 1u;
        }
      }
    }
    if (!PAIR && !ok && elected) {
      // let every copy already issued land before the CTA's shared memory goes away
      volatile int never = 0;
      for (int s = 0; s < kStages; ++s)
        if ((filled >> s) & 1u) mbar_wait(&full_bar[s], (fill_parity >> s) & 1u, &never);
    }
    __syncwarp();
  } else if (warp == 1 && leader) {
    // ------------------------------------------------------------ MMA issuer
    // The whole warp runs the loop and one elected lane issues the tcgen05
    // instructions: a loop run by a single divergent lane issues them too
    // slowly to keep the tensor pipe busy.  Shared-memory descriptors are
    // built once; a stage only adds constant offsets to their address fields.
    // In a pair only the leader's warp issues; the other CTA's warp 1 only
    // owns its half of the tensor-memory allocation.
    const uint32_t elected = elect_one();
    const uint32_t idesc = kBf16 ? idesc_bf16(kBM, kBN) : idesc_fp4(PAIR ? 2 * kBM : kBM, kBN);
    const uint32_t s0 = smem_u32(smem);
    const uint64_t a0 = sdesc_sw128(s0), b0 = sdesc_sw128(s0 + kABytes);
    const uint64_t sfa0 = sdesc_scale_atom(s0 + kABytes + kBLoad);
    const uint64_t sfb0 = sdesc_scale_atom(s0 + kABytes + kBLoad + kSfaBytes);
    constexpr uint64_t kStageStep = kSB >> 4;                  // start address is in 16-byte units
    constexpr uint64_t kAtomStep = kAtomBytes >> 4;
    constexpr uint64_t kSfbHalfStep = (kSfbBytes / 2) >> 4;
    const uint32_t sfa_t = tmem + kSfCol + kSfaOff, sfb_t = tmem + kSfCol + kSfbOff;
    const uint32_t acc_t = tmem + kAccCol;
    // pair: stage and accumulator releases go to both CTAs' barriers
    const uint32_t empty_own = PAIR ? mapa_shared(smem_u32(&empty_bar[0]), 0) : 0u;
    const uint32_t empty_peer = PAIR ? mapa_shared(smem_u32(&empty_bar[0]), 1) : 0u;
    const uint32_t accf_own = PAIR ? mapa_shared(smem_u32(&acc_full_bar), 0) : 0u;
    const uint32_t accf_peer = PAIR ? mapa_shared(smem_u32(&acc_full_bar), 1) : 0u;
    int stage = 0;
    uint32_t phase = 0, acc_phase = 0;
    bool ok = true;
    for (int t = t_first; ok && t < num_tiles; t += t_step) {
      ok = __all_sync(0xffffffffu, mbar_wait(&acc_empty_bar, acc_phase ^ 1u, abort_flag));
      if (!ok) {
        if (elected) {
          if constexpr (PAIR) give_up_pair(p.status, abort_flag, peer_abort);
          else give_up(p.status, abort_flag);
        }
        break;
      }
      tc_fence_after();
      uint32_t accumulate = 0;
      for (int kt = 0; kt < KT; ++kt) {
        // the copies wrote this stage through the async proxy that the MMAs read
        // through; the completed barrier phase is all the ordering needed
        ok = __all_sync(0xffffffffu, mbar_wait(&full_bar[stage], phase, abort_flag));
        if (!ok) {
          if (elected) {
            if constexpr (PAIR) give_up_pair(p.status, abort_flag, peer_abort);
            else give_up(p.status, abort_flag);
          }
          break;
        }
        const uint64_t d = (uint64_t)stage * kStageStep;
        const int katoms = kBf16 ? 4 : min(4, (p.K - kt * kBK) / 64);
        if constexpr (PAIR) {
          if (elected) {
#pragma unroll
            for (int j = 0; j < 4; ++j) {
              tc_cp_scale_atom_pair(sfa_t + 4 * j, sfa0 + d + j * kAtomStep);
              tc_cp_scale_atom_pair(sfb_t + 8 * j, sfb0 + d + j * kAtomStep);
              tc_cp_scale_atom_pair(sfb_t + 8 * j + 4, sfb0 + d + kSfbHalfStep + j * kAtomStep);
            }
#pragma unroll
            for (int j = 0; j < 4; ++j)
              mma_fp4_pair(acc_t, a0 + d + 2 * j, b0 + d + 2 * j, idesc, sfa_t + 4 * j, sfb_t + 8 * j,
                           accumulate | j);
            tc_commit_pair(empty_own + 8u * stage);
            tc_commit_pair(empty_peer + 8u * stage);
          }
        } else if (elected && kBf16) {
          // 4 x (K = 16 bf16 = 32 bytes) per 128-byte stage row
#pragma unroll
          for (int j = 0; j < 4; ++j) mma_bf16(acc_t, a0 + d + 2 * j, b0 + d + 2 * j, idesc, accumulate | j);
          tc_commit(&empty_bar[stage]);
        } else if (elected) {
          if (katoms == 4) {
#pragma unroll
            for (int j = 0; j < 4; ++j) {
              tc_cp_scale_atom(sfa_t + 4 * j, sfa0 + d + j * kAtomStep);
              tc_cp_scale_atom(sfb_t + 8 * j, sfb0 + d + j * kAtomStep);
              tc_cp_scale_atom(sfb_t + 8 * j + 4, sfb0 + d + kSfbHalfStep + j * kAtomStep);
            }
#pragma unroll
            for (int j = 0; j < 4; ++j) {
              // +32 bytes (64 FP4 values) along K inside the 128-byte swizzle atom
              mma_fp4(acc_t, a0 + d + 2 * j, b0 + d + 2 * j, idesc, sfa_t + 4 * j, sfb_t + 8 * j, accumulate | j);
            }
          } else {
            for (int j = 0; j < katoms; ++j) {
              tc_cp_scale_atom(sfa_t + 4 * j, sfa0 + d + j * kAtomStep);
              tc_cp_scale_atom(sfb_t + 8 * j, sfb0 + d + j * kAtomStep);
              tc_cp_scale_atom(sfb_t + 8 * j + 4, sfb0 + d + kSfbHalfStep + j * kAtomStep);
            }
            for (int j = 0; j < katoms; ++j)
              mma_fp4(acc_t, a0 + d + 2 * j, b0 + d + 2 * j, idesc, sfa_t + 4 * j, sfb_t + 8 * j, accumulate | j);
          }
          tc_commit(&empty_bar[stage]);
        }
        __syncwarp();
        accumulate = 1;
        if (++stage == kStages) {
          stage = 0;
          phase ^= 1u;
        }
      }
      if (!ok) break;
      if (elected) {
        if constexpr (PAIR) {
          tc_commit_pair(accf_own);
          tc_commit_pair(accf_peer);
        } else {
          tc_commit(&acc_full_bar);
        }
      }
      __syncwarp();
      acc_phase ^= 1u;
    }
    // every MMA issued by the elected lane completes before tensor memory is freed
    if (elected) {
      if constexpr (PAIR) {
        tc_commit_pair(mapa_shared(smem_u32(&drain_bar), 0));
      } else {
        tc_commit(&drain_bar);
      }
      volatile int never = 0;
      mbar_wait(&drain_bar, 0, &never);
    }
    __syncwarp();
  } else if (warp >= 2) {
    // ------------------------------------------------------------ epilogue
    const int quad = warp & 3;
    const int half = (warp - 2) >> 2;
    const int row_in_tile = quad * 32 + lane;
    const uint32_t tbase = tmem + ((uint32_t)(quad * 32) << 16);
    // pair: the accumulator is handed back to the leader's MMA warp
    const uint32_t acce_leader = PAIR ? mapa_shared(smem_u32(&acc_empty_bar), 0) : 0u;
    const uint32_t tacc = tbase + kAccCol;
    uint32_t acc_phase = 0;
    for (int t = t_first; t < num_tiles; t += t_step) {
      const TileCoord tc = tile_of(t);
      const int e = tc.e, mt = tc.mt, nt = tc.nt;
      const int grow = mt * kBM + row_in_tile;
      const bool real =
          tc.valid && (p.expert_counts ? (grow - p.expert_offsets[e] < p.expert_counts[e]) : true);
      // the tile's scalars are loaded before the accumulator is ready, so that
      // no global load sits between the accumulator-full wait and the hand-back
      const int se = p.per_expert ? e : 0;                  // index of this tile's scales
      const float g_act = kBf16 ? 1.0f : p.g_act[se];
      const float g_b0 = kBf16 ? 1.0f : p.g_b0[e];
      const float g_b1 = kBf16 || !kGateUp ? 1.0f : p.g_b1[e];
      const float g_h = EPI == kEpiGateUp ? p.g_h[se] : 1.0f;
      const float w_row = EPI == kEpiDown && p.row_w && real ? p.row_w[grow] : 1.0f;
      if (!mbar_wait(&acc_full_bar, acc_phase, abort_flag)) {
        if constexpr (PAIR) give_up_pair(p.status, abort_flag, peer_abort);
        else give_up(p.status, abort_flag);
        break;
      }
      tc_fence_after();
      if (EPI == kEpiSharedGateUp) {
        // bf16 operands, no global scales: h = silu(gate) * up, stored bf16
        uint32_t rg[64], ru[64];
        tmem_ld32(tacc + half * 64, rg);
        tmem_ld32(tacc + half * 64 + 32, rg + 32);
        tmem_ld32(tacc + 128 + half * 64, ru);
        tmem_ld32(tacc + 128 + half * 64 + 32, ru + 32);
        tmem_ld_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&acc_empty_bar);
        if (real && p.partial) {
          // split K: this part's gate and up sums; the reduction applies SiLU * up
          float4* pg = reinterpret_cast<float4*>(p.partial + ((size_t)tc.ks * p.partial_rows + grow) * (2 * p.I) +
                                                 nt * 128 + half * 64);
          float4* pu = pg + p.I / 4;
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            pg[i] = make_float4(__uint_as_float(rg[4 * i]), __uint_as_float(rg[4 * i + 1]),
                                __uint_as_float(rg[4 * i + 2]), __uint_as_float(rg[4 * i + 3]));
            pu[i] = make_float4(__uint_as_float(ru[4 * i]), __uint_as_float(ru[4 * i + 1]),
                                __uint_as_float(ru[4 * i + 2]), __uint_as_float(ru[4 * i + 3]));
          }
        } else if (real) {
          uint4* dst = reinterpret_cast<uint4*>(p.h_bf16 + (size_t)grow * p.I + nt * 128 + half * 64);
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            uint32_t w[4];
#pragma unroll
            for (int q = 0; q < 4; ++q) {
              const int c = 8 * i + 2 * q;
              w[q] = pack_bf16x2(__fmul_rn(silu(__uint_as_float(rg[c])), __uint_as_float(ru[c])),
                                 __fmul_rn(silu(__uint_as_float(rg[c + 1])), __uint_as_float(ru[c + 1])));
            }
            dst[i] = make_uint4(w[0], w[1], w[2], w[3]);
          }
        }
      } else if (EPI == kEpiGateUp) {
        const float sg = __fmul_rn(g_act, g_b0);
        const float su = __fmul_rn(g_act, g_b1);
        // drain this thread's 64 gate and 64 up columns, then hand the
        // accumulator back before any arithmetic
        uint32_t rg[64], ru[64];
        tmem_ld32(tacc + half * 64, rg);
        tmem_ld32(tacc + half * 64 + 32, rg + 32);
        tmem_ld32(tacc + 128 + half * 64, ru);
        tmem_ld32(tacc + 128 + half * 64 + 32, ru + 32);
        tmem_ld_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) {
          if constexpr (PAIR) mbar_arrive_remote(acce_leader);
          else mbar_arrive(&acc_empty_bar);
        }
        const int hcol0 = nt * 128 + half * 64;
        uint4 cw0 = make_uint4(0, 0, 0, 0), cw1 = make_uint4(0, 0, 0, 0);
        uint32_t sw = 0;
        if (real) {
          float h[64];
#pragma unroll
          for (int i = 0; i < 64; ++i) {
            const float gate = __fmul_rn(__uint_as_float(rg[i]), sg);
            const float up = __fmul_rn(__uint_as_float(ru[i]), su);
            h[i] = __fmul_rn(silu(gate), up);
          }
          const BlockScaler b2 = make_scaler(g_h);
          uint2 c0, c1, c2, c3;
          const uint32_t s0 = quant_block16(h, b2, c0);
          const uint32_t s1 = quant_block16(h + 16, b2, c1);
          const uint32_t s2 = quant_block16(h + 32, b2, c2);
          const uint32_t s3 = quant_block16(h + 48, b2, c3);
          cw0 = make_uint4(c0.x, c0.y, c1.x, c1.y);
          cw1 = make_uint4(c2.x, c2.y, c3.x, c3.y);
          sw = s0 | (s1 << 8) | (s2 << 16) | (s3 << 24);
          if (p.h_f32) {
            float4* dst = reinterpret_cast<float4*>(p.h_f32 + (size_t)grow * p.I + hcol0);
#pragma unroll
            for (int i = 0; i < 16; ++i) dst[i] = make_float4(h[4 * i], h[4 * i + 1], h[4 * i + 2], h[4 * i + 3]);
          }
          if (p.h_amax) {
            float m = 0.0f;
#pragma unroll
            for (int i = 0; i < 64; ++i) m = fmaxf(m, fabsf(h[i]));
            atomicMax(reinterpret_cast<unsigned int*>(p.h_amax + se), __float_as_uint(m));
          }
        }
        // padding rows of a segment get zero codes and scales; a pair CTA
        // without rows of its own stores nothing
        if (tc.valid) {
          uint4* cdst = reinterpret_cast<uint4*>(p.h_codes + (size_t)grow * (p.I / 2) + hcol0 / 2);
          cdst[0] = cw0;
          cdst[1] = cw1;
          *reinterpret_cast<uint32_t*>(p.h_sf + tiled_scale_offset(grow, hcol0 / kQBlock, p.I / 64)) = sw;
        }
      } else {
        const float scale = kBf16 ? 1.0f : __fmul_rn(__fmul_rn(g_act, g_b0), w_row);
        const int col0 = nt * kBN + half * 128;
        // drain this thread's 128 columns, then hand the accumulator back
        uint32_t r[128];
#pragma unroll
        for (int c = 0; c < 4; ++c) tmem_ld32(tacc + half * 128 + 32 * c, r + 32 * c);
        tmem_ld_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) {
          if constexpr (PAIR) mbar_arrive_remote(acce_leader);
          else mbar_arrive(&acc_empty_bar);
        }
        if (kBf16 && real && p.partial) {
          // split K: this part's sums (the bf16 kind has no scale); the
          // reduction adds the parts and rounds to bf16
          float4* pd = reinterpret_cast<float4*>(p.partial + ((size_t)tc.ks * p.partial_rows + grow) * p.H + col0);
#pragma unroll
          for (int i = 0; i < 32; ++i)
            pd[i] = make_float4(__uint_as_float(r[4 * i]), __uint_as_float(r[4 * i + 1]),
                                __uint_as_float(r[4 * i + 2]), __uint_as_float(r[4 * i + 3]));
        }
        if (real && p.y_f32) {
          float4* dst = reinterpret_cast<float4*>(p.y_f32 + (size_t)grow * p.H + col0);
#pragma unroll
          for (int i = 0; i < 32; ++i)
            dst[i] = make_float4(__fmul_rn(__uint_as_float(r[4 * i]), scale),
                                 __fmul_rn(__uint_as_float(r[4 * i + 1]), scale),
                                 __fmul_rn(__uint_as_float(r[4 * i + 2]), scale),
                                 __fmul_rn(__uint_as_float(r[4 * i + 3]), scale));
        }
        if (real && p.y_sq_part) {
          float ss = 0.0f;
#pragma unroll
          for (int i = 0; i < 128; ++i) {
            const float v = __fmul_rn(__uint_as_float(r[i]), scale);
            ss = fmaf(v, v, ss);
          }
          p.y_sq_part[(size_t)grow * (p.H / 128) + nt * 2 + half] = ss;
        }
        // scaled and packed to bf16 pairs right away, which frees r
        uint32_t yw[64];
#pragma unroll
        for (int i = 0; i < 64; ++i)
          yw[i] = pack_bf16x2(__fmul_rn(__uint_as_float(r[2 * i]), scale), __fmul_rn(__uint_as_float(r[2 * i + 1]), scale));
        const uint32_t real_mask = __ballot_sync(0xffffffffu, real);
        if (PAIR && p.y_bf16 && real_mask != 0) {
          // Whole 32-row boxes of 64 columns go out by TMA store from a
          // staging tile in the 128-byte swizzle (16-byte chunk c of row r
          // at chunk c ^ (r % 8)), which lane r writes without bank
          // conflicts.  A box holding padding rows is written back by the
          // warp instead, data rows only, as 128-byte row segments.
          uint8_t* ybuf = smem + kStages * kSB + (warp - 2) * y_stage_bytes_of<EPI, PAIR>();
          const int row0 = mt * kBM + quad * 32;
#pragma unroll
          for (int b = 0; b < 2; ++b) {
            if (lane == 0) bulk_wait_read_all();        // the previous box has left ybuf
            __syncwarp();
#pragma unroll
            for (int c = 0; c < 8; ++c) {
              const int w = b * 32 + c * 4;
              *reinterpret_cast<uint4*>(ybuf + lane * 128 + ((c ^ (lane & 7)) << 4)) =
                  make_uint4(yw[w], yw[w + 1], yw[w + 2], yw[w + 3]);
            }
            if (real_mask == 0xffffffffu) {
              fence_proxy_async();                      // the writes above, before the async proxy reads them
              __syncwarp();
              if (lane == 0) {
                tma_store_2d(&pm->y, ybuf, col0 + b * 64, row0);
                bulk_commit_group();
              }
            } else {
              __syncwarp();
#pragma unroll
              for (int it = 0; it < 8; ++it) {
                const int rr = it * 4 + (lane >> 3), ch = lane & 7;
                const uint4 v = *reinterpret_cast<const uint4*>(ybuf + rr * 128 + ((ch ^ (rr & 7)) << 4));
                if ((real_mask >> rr) & 1u)
                  *reinterpret_cast<uint4*>(p.y_bf16 + (size_t)(row0 + rr) * p.H + col0 + b * 64 + ch * 8) = v;
              }
              __syncwarp();
            }
          }
        } else if (p.y_bf16 && real_mask != 0) {
          // Each lane holds one row.  Stores straight from registers would
          // hit 32 rows per instruction, so the warp stages kYCols columns of
          // its 32 rows in shared memory and writes them back as whole row
          // segments (kYCols * 2 bytes), 32 / kCh rows per instruction.  The
          // 16-byte chunks are XOR-swizzled by row so that every 8-lane phase
          // of a 16-byte access covers the 32 banks once, in both directions.
          constexpr int kYCols = y_pass_cols_of<EPI, PAIR>(), kCh = kYCols / 8, kRowsPer = 32 / kCh;
          uint4* ybuf = reinterpret_cast<uint4*>(smem + kStages * kSB + (warp - 2) * y_stage_bytes_of<EPI, PAIR>());
          const int row0 = mt * kBM + quad * 32;
          auto swz = [](int r) { return (r / (8 / kCh)) % kCh; };
#pragma unroll
          for (int pass = 0; pass < 128 / kYCols; ++pass) {
#pragma unroll
            for (int ch = 0; ch < kCh; ++ch) {
              const int w = pass * (kYCols / 2) + ch * 4;
              ybuf[lane * kCh + (ch ^ swz(lane))] = make_uint4(yw[w], yw[w + 1], yw[w + 2], yw[w + 3]);
            }
            __syncwarp();
#pragma unroll
            for (int it = 0; it < kCh; ++it) {
              const int rr = it * kRowsPer + lane / kCh, ch = lane % kCh;
              const uint4 v = ybuf[rr * kCh + (ch ^ swz(rr))];
              if ((real_mask >> rr) & 1u)
                *reinterpret_cast<uint4*>(p.y_bf16 + (size_t)(row0 + rr) * p.H + col0 + pass * kYCols + ch * 8) = v;
            }
            __syncwarp();
          }
        }
      }
      acc_phase ^= 1u;
    }
    // the CTA's shared memory outlives every TMA store of y it issued
    if (PAIR && EPI == kEpiDown && lane == 0) bulk_wait_all();
  }
  tc_fence_before();
  __syncthreads();
  if constexpr (PAIR) {
    // neither CTA leaves while the other may still arrive on its barriers or
    // the leader's MMAs may still read its shared memory
    cluster_sync_all();
    if (*abort_flag) {
      // after a give-up, copies issued before it may still be landing in
      // this CTA's shared memory: they finish within microseconds
      const uint64_t t0 = globaltimer_ns();
      while (globaltimer_ns() - t0 < 1000000ull) {
      }
    }
  }
  if (warp == 1) {
    tc_fence_after();
    if constexpr (PAIR) tmem_dealloc_pair(tmem, kTmemCols);
    else tmem_dealloc(tmem, kTmemCols);
  }
}

template <int EPI>
__global__ void __launch_bounds__(kThreads, 1)
    grouped_fp4_gemm_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmA32,
                            const __grid_constant__ CUtensorMap tmB0, const __grid_constant__ CUtensorMap tmB1,
                            const GemmParams p) {
  gemm_body<EPI, false>(tmA, tmA32, tmB0, tmB1, nullptr, p);
}

// The CTA-pair form of the FP4 GEMMs: launched in clusters of two.
template <int EPI>
__global__ void __launch_bounds__(kThreads, 1)
    grouped_fp4_gemm_pair_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB0,
                                 const __grid_constant__ CUtensorMap tmB1, const __grid_constant__ PairMaps pm,
                                 const GemmParams p) {
  gemm_body<EPI, true>(tmA, tmA, tmB0, tmB1, &pm, p);
}

// Opts a kernel into the large dynamic shared memory once per device.
static nvfp4_status set_smem_attr(const void* fn, int which, int smem) {
  static std::mutex mu;
  static bool done[6][64] = {};
  int dev = 0;
  NV_CHECK(check_cuda(cudaGetDevice(&dev), "cudaGetDevice"));
  if (dev < 0 || dev >= 64) dev = 63;
  std::lock_guard<std::mutex> lock(mu);
  if (!done[which][dev]) {
    NV_CHECK(check_cuda(cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, smem),
                        "cudaFuncSetAttribute"));
    done[which][dev] = true;
  }
  return NVFP4_OK;
}

// Launches the CTA-pair kernel: clusters of two CTAs, as many clusters as can
// be resident at once (persistent), as a programmatic dependent launch.
template <int EPI>
static nvfp4_status launch_pair(const char* what, const CUtensorMap& tmA, const CUtensorMap& tmB0,
                                const CUtensorMap& tmB1, const PairMaps& pm, const GemmParams& p, int max_pair_tiles,
                                cudaStream_t s) {
  constexpr int smem = smem_bytes_of<EPI, true>();
  NV_CHECK(set_smem_attr((const void*)grouped_fp4_gemm_pair_kernel<EPI>, EPI == kEpiGateUp ? 4 : 5, smem));
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  static std::mutex mu;
  static int clusters[2][64] = {};
  int dev = 0;
  NV_CHECK(check_cuda(cudaGetDevice(&dev), "cudaGetDevice"));
  if (dev < 0 || dev >= 64) dev = 63;
  int n = 0;
  {
    std::lock_guard<std::mutex> lock(mu);
    n = clusters[EPI == kEpiGateUp ? 0 : 1][dev];
    if (n == 0) {
      int sms = 0;
      NV_CHECK(device_sm_count(&sms));
      cfg.gridDim = dim3(2 * (sms / 2));
      NV_CHECK(check_cuda(cudaOccupancyMaxActiveClusters(&n, grouped_fp4_gemm_pair_kernel<EPI>, &cfg),
                          "cudaOccupancyMaxActiveClusters"));
      NV_REQUIRE(n >= 1, NVFP4_ERR_CUDA, "%s: no cluster of two CTAs can be resident", what);
      clusters[EPI == kEpiGateUp ? 0 : 1][dev] = n;
    }
  }
  cfg.gridDim = dim3(2 * std::max(1, std::min(n, max_pair_tiles)));
  cfg.numAttrs = 2;
  return check_cuda(cudaLaunchKernelEx(&cfg, grouped_fp4_gemm_pair_kernel<EPI>, tmA, tmB0, tmB1, pm, p), what);
}

bool gemm_runs_pair(const GroupedGemmArgs& a) {
  const bool fp4 = a.epi == kEpiGateUp || a.epi == kEpiDown;
  const int K = a.epi == kEpiGateUp ? a.H : a.I;
  return a.pair && fp4 && K % kBK == 0;
}

nvfp4_status launch_grouped_gemm(const GroupedGemmArgs& a, cudaStream_t s) {
  int sms = 0;
  NV_CHECK(device_sm_count(&sms));
  const bool gu = a.epi == kEpiGateUp || a.epi == kEpiSharedGateUp;
  const bool bf = a.epi == kEpiSharedGateUp || a.epi == kEpiSharedDown;
  const int K = gu ? a.H : a.I;
  const int Nw = gu ? a.I : a.H;
  // the CTA pair: FP4 kinds with whole 256-element K stages, when asked for
  const bool pair = gemm_runs_pair(a);
  // 128-byte K boxes: 128 packed FP4 bytes, or 64 bf16 elements
  const CUtensorMapDataType dt = bf ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_UINT8;
  const uint64_t inner = bf ? (uint64_t)K : (uint64_t)K / 2;       // elements per row
  const uint64_t pitch = bf ? (uint64_t)K * 2 : (uint64_t)K / 2;   // bytes per row
  const uint32_t box = bf ? 64 : kBKBytes;
  CUtensorMap tmA, tmA32, tmB0, tmB1;
  const uint64_t a_rows = (uint64_t)(a.a_rows > 0 ? a.a_rows : a.rows_capacity);
  NV_CHECK(make_tmap_2d(&tmA, a.a_codes, dt, inner, a_rows, pitch, box, kBM));
  if (!pair) {
    NV_CHECK(make_tmap_2d(&tmA32, a.a_codes, dt, inner, a_rows, pitch, box, 32));
    NV_CHECK(make_tmap_2d(&tmB0, a.b0_codes, dt, inner, (uint64_t)a.E * Nw, pitch, box, gu ? 128 : kBN));
    if (gu) {
      NV_CHECK(make_tmap_2d(&tmB1, a.b1_codes, dt, inner, (uint64_t)a.E * Nw, pitch, box, 128));
    } else {
      tmB1 = tmB0;
    }
  } else if (a.b_staged) {
    // staged codes as rows of 128 bytes: each 128-row, 256-element K tile is
    // 128 consecutive rows, already in the swizzled order
    const uint64_t rows = (uint64_t)a.E * Nw * (K / kBK);
    NV_CHECK(make_tmap_2d(&tmB0, a.b0_codes, CU_TENSOR_MAP_DATA_TYPE_UINT8, 128, rows, 128, 128, 128, false));
    if (gu) {
      NV_CHECK(make_tmap_2d(&tmB1, a.b1_codes, CU_TENSOR_MAP_DATA_TYPE_UINT8, 128, rows, 128, 128, 128, false));
    } else {
      tmB1 = tmB0;
    }
  } else {
    // each CTA of the pair loads 128 weight rows
    NV_CHECK(make_tmap_2d(&tmB0, a.b0_codes, dt, inner, (uint64_t)a.E * Nw, pitch, box, 128));
    if (gu) {
      NV_CHECK(make_tmap_2d(&tmB1, a.b1_codes, dt, inner, (uint64_t)a.E * Nw, pitch, box, 128));
    } else {
      tmB1 = tmB0;
    }
  }
  GemmParams p;
  p.a_sf = a.a_scales;
  p.b0_sf = a.b0_scales;
  p.b1_sf = a.b1_scales;
  p.K = K;
  p.E = a.E;
  p.Nw = Nw;
  p.n_tiles = gu ? a.I / 128 : a.H / kBN;
  p.cap_tiles = a.rows_capacity / kBM;
  p.tile_expert = a.tile_expert;
  p.num_mtiles = a.num_mtiles;
  p.expert_offsets = a.expert_offsets;
  p.expert_counts = a.expert_counts;
  p.g_act = a.act_gscale;
  p.g_b0 = a.b0_gscale;
  p.g_b1 = a.b1_gscale;
  p.g_h = a.h_gscale;
  p.h_codes = a.h_codes;
  p.h_sf = a.h_scales;
  p.h_f32 = a.h_f32;
  p.h_amax = a.h_amax;
  p.I = a.I;
  p.row_w = a.row_w;
  p.y_bf16 = static_cast<uint16_t*>(a.y_bf16);
  p.y_f32 = a.y_f32;
  p.y_sq_part = a.y_sq_part;
  p.h_bf16 = static_cast<uint16_t*>(a.h_bf16);
  p.H = a.H;
  p.per_expert = a.per_expert_scales ? 1 : 0;
  p.b_staged = a.b_staged ? 1 : 0;
  p.b0_codes = a.b0_codes;
  p.b1_codes = a.b1_codes;
  p.status = a.status;
  p.ksplit = std::max(1, a.ksplit);
  p.partial_rows = a.partial_rows;
  p.partial = a.partial;
  NV_REQUIRE(p.ksplit == 1 || (bf && !pair && a.partial && (K / 64) % p.ksplit == 0 && a.partial_rows > 0),
             NVFP4_ERR_INVALID_ARG, "split K needs a bf16 kind, a partial buffer and K / 64 divisible by %d",
             p.ksplit);
  const int max_tiles = a.rows_capacity / kBM * p.n_tiles * p.ksplit;
  if (pair) {
    // scale atoms as rows of 128 32-bit words (512 bytes), four per stage
    const int nblk4 = K / 64;
    PairMaps pm;
    NV_CHECK(make_tmap_2d(&pm.sfa, a.a_scales, CU_TENSOR_MAP_DATA_TYPE_UINT32, 128,
                          (uint64_t)(a.rows_capacity / kBM) * nblk4, kAtomBytes, 128, 4, false));
    NV_CHECK(make_tmap_2d(&pm.sfb0, a.b0_scales, CU_TENSOR_MAP_DATA_TYPE_UINT32, 128,
                          (uint64_t)a.E * Nw / kBM * nblk4, kAtomBytes, 128, 4, false));
    if (gu) {
      NV_CHECK(make_tmap_2d(&pm.sfb1, a.b1_scales, CU_TENSOR_MAP_DATA_TYPE_UINT32, 128,
                            (uint64_t)a.E * Nw / kBM * nblk4, kAtomBytes, 128, 4, false));
    } else {
      pm.sfb1 = pm.sfb0;
    }
    std::memset(&pm.y, 0, sizeof(pm.y));
    if (!gu && a.y_bf16)
      NV_CHECK(make_tmap_2d(&pm.y, a.y_bf16, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, (uint64_t)a.H,
                            (uint64_t)a.rows_capacity, (uint64_t)a.H * 2, 64, 32, true));
    if (a.epi == kEpiGateUp)
      return launch_pair<kEpiGateUp>("grouped_fp4_gemm_pair_kernel<gate_up>", tmA, tmB0, tmB1, pm, p, max_tiles, s);
    return launch_pair<kEpiDown>("grouped_fp4_gemm_pair_kernel<down>", tmA, tmB0, tmB1, pm, p, max_tiles, s);
  }
  const int grid = std::max(1, std::min(sms, max_tiles));
  switch (a.epi) {
    case kEpiGateUp:
      NV_CHECK(set_smem_attr((const void*)grouped_fp4_gemm_kernel<kEpiGateUp>, 0,
                             smem_bytes_of<kEpiGateUp, false>()));
      return launch_dependent("grouped_fp4_gemm_kernel<gate_up>", grouped_fp4_gemm_kernel<kEpiGateUp>, dim3(grid),
                              dim3(kThreads), smem_bytes_of<kEpiGateUp, false>(), s, tmA, tmA32, tmB0, tmB1, p);
    case kEpiDown:
      NV_CHECK(set_smem_attr((const void*)grouped_fp4_gemm_kernel<kEpiDown>, 1, smem_bytes_of<kEpiDown, false>()));
      return launch_dependent("grouped_fp4_gemm_kernel<down>", grouped_fp4_gemm_kernel<kEpiDown>, dim3(grid),
                              dim3(kThreads), smem_bytes_of<kEpiDown, false>(), s, tmA, tmA32, tmB0, tmB1, p);
    case kEpiSharedGateUp:
      NV_CHECK(set_smem_attr((const void*)grouped_fp4_gemm_kernel<kEpiSharedGateUp>, 2,
                             smem_bytes_of<kEpiSharedGateUp, false>()));
      return launch_dependent("grouped_fp4_gemm_kernel<shared_gate_up>", grouped_fp4_gemm_kernel<kEpiSharedGateUp>,
                              dim3(grid), dim3(kThreads), smem_bytes_of<kEpiSharedGateUp, false>(), s, tmA, tmA32,
                              tmB0, tmB1, p);
    default:
      NV_CHECK(set_smem_attr((const void*)grouped_fp4_gemm_kernel<kEpiSharedDown>, 3,
                             smem_bytes_of<kEpiSharedDown, false>()));
      return launch_dependent("grouped_fp4_gemm_kernel<shared_down>", grouped_fp4_gemm_kernel<kEpiSharedDown>,
                              dim3(grid), dim3(kThreads), smem_bytes_of<kEpiSharedDown, false>(), s, tmA, tmA32,
                              tmB0, tmB1, p);
  }
}

// Builds the m-tile -> expert map from caller-supplied segment offsets,
// clamped so that every tile stays inside the row capacity.
__global__ void tiles_from_offsets_kernel(const int32_t* __restrict__ offsets, int E, int cap_tiles,
                                          int32_t* __restrict__ tile_expert, int32_t* __restrict__ num_mtiles) {
  for (int m = threadIdx.x; m < cap_tiles; m += blockDim.x) tile_expert[m] = 0;
  __syncthreads();
  for (int e = threadIdx.x; e < E; e += blockDim.x) {
    const int lo = min(max(offsets[e] / kRowTile, 0), cap_tiles);
    const int hi = min(max(offsets[e + 1] / kRowTile, lo), cap_tiles);
    for (int m = lo; m < hi; ++m) tile_expert[m] = e;
  }
  if (threadIdx.x == 0) *num_mtiles = min(max(offsets[E] / kRowTile, 0), cap_tiles);
}

struct GemmScratch {
  uint32_t* status;
  int32_t* tile_expert;
  int32_t* num_mtiles;
};

static GemmScratch carve_gemm_scratch(Carver& c, int rows_capacity) {
  GemmScratch g;
  g.status = c.take<uint32_t>(64);
  g.tile_expert = c.take<int32_t>((size_t)rows_capacity / kRowTile + 1);
  g.num_mtiles = c.take<int32_t>(1);
  return g;
}

static nvfp4_status check_weights(const moe_nvfp4_weights* W) {
  NV_REQUIRE(W != nullptr, NVFP4_ERR_INVALID_ARG, "weights struct is NULL");
  NV_REQUIRE(W->E >= 1 && W->E <= 256 && W->k >= 1 && W->k <= 16 && W->k <= W->E, NVFP4_ERR_UNSUPPORTED_SHAPE,
             "needs 1 <= k <= 16 and k <= E <= 256 (E=%d k=%d)", W->E, W->k);
  NV_REQUIRE(W->H > 0 && W->H % 256 == 0, NVFP4_ERR_UNSUPPORTED_SHAPE, "H=%d must be a positive multiple of 256",
             W->H);
  NV_REQUIRE(W->I > 0 && W->I % 128 == 0, NVFP4_ERR_UNSUPPORTED_SHAPE, "I=%d must be a positive multiple of 128",
             W->I);
  NV_REQUIRE(W->codes_layout == NVFP4_LAYOUT_CANONICAL || W->codes_layout == NVFP4_LAYOUT_STAGED,
             NVFP4_ERR_INVALID_ARG, "codes_layout=%d: expected NVFP4_LAYOUT_CANONICAL or NVFP4_LAYOUT_STAGED",
             W->codes_layout);
  NV_REQUIRE(W->codes_layout != NVFP4_LAYOUT_STAGED || W->I % 256 == 0, NVFP4_ERR_UNSUPPORTED_SHAPE,
             "staged codes need I %% 256 == 0 (I=%d)", W->I);
  const bool any_shared = W->shared_gate || W->shared_up || W->shared_down || W->I_shared;
  NV_REQUIRE(!any_shared || (W->shared_gate && W->shared_up && W->shared_down && W->I_shared > 0 &&
                             W->I_shared % 128 == 0),
             NVFP4_ERR_INVALID_ARG, "shared expert: all three weights and I_shared %% 128 == 0 (I_shared=%d)",
             W->I_shared);
  NV_REQUIRE(!any_shared || (aligned(W->shared_gate, 16) && aligned(W->shared_up, 16) &&
                             aligned(W->shared_down, 16)),
             NVFP4_ERR_INVALID_ARG, "shared expert weights need 16-byte alignment");
  return NVFP4_OK;
}

}  // namespace nvfp4moe

using namespace nvfp4moe;

nvfp4_status nvfp4moe_check_weights(const moe_nvfp4_weights* W) { return check_weights(W); }

extern "C" size_t moe_nvfp4_gemm_workspace_size(int rows_capacity) {
  if (rows_capacity < 0) return 0;
  Carver c(nullptr);
  carve_gemm_scratch(c, rows_capacity);
  return c.size();
}

static nvfp4_status step_common(const moe_nvfp4_weights* W, const int32_t* expert_offsets, int rows_capacity,
                                void* ws, size_t ws_bytes, const char* name) {
  NV_CHECK(check_weights(W));
  NV_REQUIRE(expert_offsets != nullptr, NVFP4_ERR_INVALID_ARG, "%s: expert_offsets is NULL", name);
  NV_REQUIRE(rows_capacity >= 0 && rows_capacity % 128 == 0, NVFP4_ERR_UNSUPPORTED_SHAPE,
             "%s: rows_capacity=%d must be a non-negative multiple of 128", name, rows_capacity);
  const size_t need = moe_nvfp4_gemm_workspace_size(rows_capacity);
  NV_REQUIRE(ws && ws_bytes >= need && aligned(ws, 256), NVFP4_ERR_WORKSPACE,
             "%s: needs a 256-byte aligned workspace of %zu bytes", name, need);
  return NVFP4_OK;
}

extern "C" nvfp4_status moe_nvfp4_gate_up(const moe_nvfp4_weights* W, const uint8_t* a_codes,
                                          const uint8_t* a_scales, const int32_t* expert_offsets,
                                          const int32_t* expert_counts, int rows_capacity, const float* act_gscale,
                                          const float* h_gscale, uint8_t* h_codes, uint8_t* h_scales, float* h_f32,
                                          float* h_amax, void* ws, size_t ws_bytes, void* stream) {
  NV_CHECK(step_common(W, expert_offsets, rows_capacity, ws, ws_bytes, "moe_nvfp4_gate_up"));
  NV_REQUIRE(a_codes && a_scales && act_gscale && h_gscale && h_codes && h_scales && W->gate_codes &&
                 W->gate_scales && W->gate_gscale && W->up_codes && W->up_scales && W->up_gscale,
             NVFP4_ERR_INVALID_ARG, "moe_nvfp4_gate_up: a required pointer is NULL");
  NV_REQUIRE(aligned(a_codes, 16) && aligned(h_codes, 16) && aligned(a_scales, 16) && aligned(h_scales, 16) &&
                 aligned(W->gate_codes, 16) && aligned(W->up_codes, 16) && aligned(W->gate_scales, 16) &&
                 aligned(W->up_scales, 16) && (!h_f32 || aligned(h_f32, 16)),
             NVFP4_ERR_INVALID_ARG, "moe_nvfp4_gate_up: operands need 16-byte alignment");
  if (rows_capacity == 0) return NVFP4_OK;
  cudaStream_t s = as_stream(stream);
  Carver c(ws);
  GemmScratch g = carve_gemm_scratch(c, rows_capacity);
  NV_CHECK(check_cuda(cudaMemsetAsync(g.status, 0, sizeof(uint32_t), s), "clear status word"));
  tiles_from_offsets_kernel<<<1, 256, 0, s>>>(expert_offsets, W->E, rows_capacity / kRowTile, g.tile_expert,
                                              g.num_mtiles);
  NV_CHECK(check_launch("tiles_from_offsets_kernel"));
  GroupedGemmArgs a;
  a.epi = kEpiGateUp;
  a.E = W->E; a.H = W->H; a.I = W->I;
  a.rows_capacity = rows_capacity;
  a.a_codes = a_codes; a.a_scales = a_scales;
  a.b0_codes = W->gate_codes; a.b0_scales = W->gate_scales; a.b0_gscale = W->gate_gscale;
  a.b1_codes = W->up_codes; a.b1_scales = W->up_scales; a.b1_gscale = W->up_gscale;
  a.b_staged = W->codes_layout == NVFP4_LAYOUT_STAGED;
  a.act_gscale = act_gscale;
  a.tile_expert = g.tile_expert; a.num_mtiles = g.num_mtiles;
  a.expert_offsets = expert_offsets; a.expert_counts = expert_counts;
  a.h_gscale = h_gscale; a.h_codes = h_codes; a.h_scales = h_scales; a.h_f32 = h_f32; a.h_amax = h_amax;
  a.status = g.status;
  a.pair = rows_capacity >= kPairMinRows;
  return launch_grouped_gemm(a, s);
}

extern "C" nvfp4_status moe_nvfp4_down(const moe_nvfp4_weights* W, const uint8_t* h_codes, const uint8_t* h_scales,
                                       const int32_t* expert_offsets, const int32_t* expert_counts, int rows_capacity,
                                       const float* h_gscale, const float* row_weight, void* y_bf16, float* y_f32,
                                       void* ws, size_t ws_bytes, void* stream) {
  NV_CHECK(step_common(W, expert_offsets, rows_capacity, ws, ws_bytes, "moe_nvfp4_down"));
  NV_REQUIRE(h_codes && h_scales && h_gscale && W->down_codes && W->down_scales && W->down_gscale,
             NVFP4_ERR_INVALID_ARG, "moe_nvfp4_down: a required pointer is NULL");
  NV_REQUIRE((y_bf16 != nullptr) != (y_f32 != nullptr), NVFP4_ERR_INVALID_ARG,
             "moe_nvfp4_down: pass exactly one of y_bf16 and y_f32");
  NV_REQUIRE(aligned(h_codes, 16) && aligned(h_scales, 16) && aligned(W->down_codes, 16) &&
                 aligned(W->down_scales, 16) && (!y_bf16 || aligned(y_bf16, 16)) && (!y_f32 || aligned(y_f32, 16)),
             NVFP4_ERR_INVALID_ARG, "moe_nvfp4_down: operands need 16-byte alignment");
  if (rows_capacity == 0) return NVFP4_OK;
  cudaStream_t s = as_stream(stream);
  Carver c(ws);
  GemmScratch g = carve_gemm_scratch(c, rows_capacity);
  NV_CHECK(check_cuda(cudaMemsetAsync(g.status, 0, sizeof(uint32_t), s), "clear status word"));
  tiles_from_offsets_kernel<<<1, 256, 0, s>>>(expert_offsets, W->E, rows_capacity / kRowTile, g.tile_expert,
                                              g.num_mtiles);
  NV_CHECK(check_launch("tiles_from_offsets_kernel"));
  GroupedGemmArgs a;
  a.epi = kEpiDown;
  a.E = W->E; a.H = W->H; a.I = W->I;
  a.rows_capacity = rows_capacity;
  a.a_codes = h_codes; a.a_scales = h_scales;
  a.b0_codes = W->down_codes; a.b0_scales = W->down_scales; a.b0_gscale = W->down_gscale;
  a.b_staged = W->codes_layout == NVFP4_LAYOUT_STAGED;
  a.act_gscale = h_gscale;
  a.tile_expert = g.tile_expert; a.num_mtiles = g.num_mtiles;
  a.expert_offsets = expert_offsets; a.expert_counts = expert_counts;
  a.row_w = row_weight; a.y_bf16 = y_bf16; a.y_f32 = y_f32;
  a.status = g.status;
  a.pair = rows_capacity >= kPairMinRows;
  return launch_grouped_gemm(a, s);
}
