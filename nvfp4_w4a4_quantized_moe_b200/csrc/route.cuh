// Internal interface of the router / permutation kernels (used by the layer).
#pragma once

#include "host.cuh"

namespace nvfp4moe {

struct RouteArgs {
  const void* x = nullptr;              // bf16 [T][H]; NULL when logits are given
  const void* router_weight = nullptr;  // bf16 [E][H]
  const float* logit_offset = nullptr;  // [E] or NULL
  const float* bias = nullptr;          // [E]
  int T = 0, H = 0, E = 0, k = 0;
  float rsf = 1.0f;
  float* logits = nullptr;              // [T][E]: written when x is given, read always
  int32_t* topk_idx = nullptr;
  float* topk_w = nullptr;
  int32_t* expert_offsets = nullptr;    // [E+1]
  int32_t* perm = nullptr;              // [capacity]
  int32_t* inv_perm = nullptr;          // [T][k]
  // the router GEMM clears the status word once the previous work on the
  // stream has finished (the caller then issues no memset before it)
  bool clear_status = false;
  // Optional, for small batches (route_fuses_x_quantise): the routing kernel
  // also quantises x under the tensor's g1 (act_gscale[0]) and writes each
  // token's codes and tiled scales to its k permuted rows of a_codes [rows]
  // [H/2] / a_scales, the work the layer's quantise-scatter kernel does
  bool quant_x = false;
  const float* act_gscale = nullptr;
  uint8_t* a_codes = nullptr;
  uint8_t* a_scales = nullptr;
};

// Whether the single-block routing kernel also quantises x and writes it to
// the permuted rows: only for small volumes, since those writes all go
// through one SM (route.cu gives the measured bound).
bool route_fuses_x_quantise(int T, int H, int k);

struct RouteScratch {
  uint32_t* status = nullptr;           // device status word (start of the workspace)
  uint32_t* bm = nullptr;               // [ceil(T/32)][E] tokens of each 32-token block that chose e
  int32_t* blk_counts = nullptr;        // [E][ceil(T/32)] popcounts of bm
  int32_t* counts = nullptr;            // [E] rows routed to each expert
  int32_t* tile_expert = nullptr;       // [capacity / 128] expert of each m-tile
  int32_t* num_mtiles = nullptr;        // [1]
  float* row_w = nullptr;               // [capacity] routing weight of each row (0 on padding)
  float* partial = nullptr;             // [splits][T][E] router GEMM partial sums
};

int route_rows_capacity(int T, int E, int k);
// K splits of the router GEMM (64-column K stages, one CTA per 128 tokens
// and split); a function of the shape only.
int router_splits(int T, int H);
RouteScratch carve_route_scratch(Carver& c, int T, int E, int k);
nvfp4_status check_route_shape(int T, int H, int E, int k);
nvfp4_status launch_route(const RouteArgs& a, const RouteScratch& r, cudaStream_t s);

}  // namespace nvfp4moe
