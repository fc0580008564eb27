// Internal interface of the grouped NVFP4 GEMM (used by the layer).
#pragma once

#include "host.cuh"

namespace nvfp4moe {

// 0/1: the routed experts' block-scaled FP4 GEMMs; 2/3: the same tiles on
// bf16 operands for the shared expert (dense, no scale factors)
enum GemmEpilogue { kEpiGateUp = 0, kEpiDown = 1, kEpiSharedGateUp = 2, kEpiSharedDown = 3 };

// One grouped GEMM over the permuted rows: row tile m (128 rows) belongs to
// expert tile_expert[m]; m-tiles beyond *num_mtiles are not computed.
struct GroupedGemmArgs {
  int epi = kEpiGateUp;
  int E = 0, H = 0, I = 0;
  int rows_capacity = 0;
  int a_rows = 0;            // rows the A tensor map covers (0: rows_capacity); TMA reads zeros past them
  // A operand: packed codes [rows][K/2], tiled scales
  const uint8_t* a_codes = nullptr;
  const uint8_t* a_scales = nullptr;
  // B operands (gate and up for kEpiGateUp; down for kEpiDown); b_staged:
  // the FP4 codes are in the staged layout (NVFP4_LAYOUT_STAGED)
  bool b_staged = false;
  const uint8_t* b0_codes = nullptr;
  const uint8_t* b0_scales = nullptr;
  const float* b0_gscale = nullptr;
  const uint8_t* b1_codes = nullptr;
  const uint8_t* b1_scales = nullptr;
  const float* b1_gscale = nullptr;
  const float* act_gscale = nullptr;        // g1 (gate/up) or g2 (down)
  // act_gscale, h_gscale and h_amax hold one value per expert (indexed by the
  // tile's expert) instead of one for the tensor
  bool per_expert_scales = false;
  // row grouping
  const int32_t* tile_expert = nullptr;
  const int32_t* num_mtiles = nullptr;
  const int32_t* expert_offsets = nullptr;
  const int32_t* expert_counts = nullptr;   // nullable: every row of a segment is data
  // gate/up outputs
  const float* h_gscale = nullptr;          // g2
  uint8_t* h_codes = nullptr;
  uint8_t* h_scales = nullptr;
  float* h_f32 = nullptr;
  float* h_amax = nullptr;
  // down outputs
  const float* row_w = nullptr;
  void* y_bf16 = nullptr;
  float* y_f32 = nullptr;
  // nullable [rows][H/128]: sum of squares of each thread's 128 scaled y
  // values (the REAP saliency's row norms are finished from these)
  float* y_sq_part = nullptr;
  // kEpiSharedGateUp output: silu(gate) * up as bf16 [rows][I]
  void* h_bf16 = nullptr;
  uint32_t* status = nullptr;
  // run the FP4 kinds on CTA pairs (clusters of two sharing one 256-row MMA)
  // when K is a multiple of 256; the caller asks for it on large batches
  bool pair = false;
  // split K (bf16 kinds only): ksplit CTAs per (m-tile, n-tile), each over
  // K / ksplit, storing fp32 partial sums of their data rows to partial
  // [ksplit][partial_rows][2I or H] instead of running the epilogue
  int ksplit = 1;
  int partial_rows = 0;
  float* partial = nullptr;
};

// Batches with at least this many (token, expert) rows run the FP4 GEMMs on
// CTA pairs; smaller ones (decode) on one CTA per tile, which loads only a
// tile's data rows.
constexpr int kPairMinRows = 2048;

nvfp4_status launch_grouped_gemm(const GroupedGemmArgs& a, cudaStream_t s);
// Whether launch_grouped_gemm runs these arguments on CTA pairs.
bool gemm_runs_pair(const GroupedGemmArgs& a);

}  // namespace nvfp4moe

// Host-side shape checks of a weights struct.
nvfp4_status nvfp4moe_check_weights(const moe_nvfp4_weights* W);

