/*
 * nvfp4_moe.h - C ABI of libnvfp4moe.so: the NVFP4 W4A4 routed-expert MoE
 * layer on NVIDIA B200 (sm_100a).
 *
 * What the layer computes
 *   "K-EXAONE-152B-A23B-REAP-80E-NVFP4" model card, section "Quantization
 *   Setup": routed-expert weights are FP4 E2M1 in groups of 16 with FP8 E4M3
 *   block scales, quantised round-to-nearest per expert Linear; activations
 *   are quantised dynamically to FP4 under calibrated global scales; the
 *   router (mlp.gate) stays BF16.
 *   "[NetsPresso AQ Deep Dive] How to Quantize the K-EXAONE-236B Model to
 *   4-Bit (NVFP4)", section "The Standard NVFP4 Serving Spec": NVFP4 scales a
 *   block by a global scale times a block scale.
 *   "K-EXAONE-152B-A23B-REAP-80E-BF16" model card, section "Pruning Setup",
 *   "Routing behavior": renormalised sigmoid routing with an
 *   e_score_correction_bias and a routed_scaling_factor.
 *
 * Conventions for every call
 *   - Every data pointer is DEVICE memory owned by the caller; the library
 *     never allocates, frees or keeps a pointer after the call returns.
 *   - Work is queued on `stream` (a cudaStream_t passed as void*; NULL is the
 *     legacy default stream) and the call returns without synchronising.
 *     Argument checks happen on the host before anything is queued; a failed
 *     check queues nothing.
 *   - Errors come back as an nvfp4_status; nvfp4_last_error() gives a message
 *     for the calling host thread.  Nothing is thrown across the ABI.
 *   - bf16 tensors are row-major with the last index contiguous.
 *   - Packed codes: two E2M1 codes per byte, the element with the even index
 *     in the low nibble; the sign is bit 3 of a code.
 *   - Scale layouts (one E4M3 byte per 16 consecutive elements of a row):
 *       NVFP4_LAYOUT_CANONICAL: [rows][cols/16] row-major.
 *       NVFP4_LAYOUT_TILED: the layout the tensor-core MMA reads.  Rows are
 *       grouped in tiles of 128 and 16-element blocks in groups of 4; each
 *       (row tile, block group) is a 512-byte atom, atoms ordered row tile
 *       major, and inside an atom row r (0..127), block b (0..3) sits at byte
 *       (r % 32) * 16 + (r / 32) * 4 + b.  The buffer holds
 *       ceil(rows/128) * 128 * cols / 16 bytes; needs cols % 64 == 0.
 *   - Weight code layouts (the packed codes of a weight matrix, rows x cols):
 *       NVFP4_LAYOUT_CANONICAL / NVFP4_LAYOUT_TILED: [rows][cols/2] row-major.
 *       NVFP4_LAYOUT_STAGED (scales TILED as above): the bytes the GEMM
 *       copies to shared memory for one 128-row x 256-column K stage are one
 *       contiguous, pre-swizzled 16 KiB tile.  Tile (i, j) covers rows
 *       [128 i, 128 i + 128) and columns [256 j, 256 j + 256) and starts at
 *       byte (i * cols/256 + j) * 16384.  Inside it, row r (0..127) fills
 *       bytes [128 r, 128 r + 128), and the 16 bytes of its columns
 *       [256 j + 32 c, 256 j + 32 c + 32) sit at byte 128 r + 16 (c ^ (r % 8)):
 *       the image a 128-byte-swizzled TMA box leaves in shared memory.  The
 *       buffer has the canonical size; needs rows % 128 == 0 and
 *       cols % 256 == 0.  Streaming a stage then reads one contiguous range
 *       instead of 128 rows of 128 bytes.
 *   - Workspace: calls that take (ws, ws_bytes) need at least the size their
 *     *_workspace_size() function returns, 256-byte aligned.  Its first word
 *     is a status word: each call clears it when it starts and a device-side
 *     wait that gives up sets it; read it with nvfp4_workspace_status().
 */
#ifndef NVFP4_MOE_H
#define NVFP4_MOE_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define NVFP4_API __attribute__((visibility("default")))
#else
#define NVFP4_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum nvfp4_status {
  NVFP4_OK = 0,
  NVFP4_ERR_INVALID_ARG = 1,       /* null pointer, bad enum, negative size   */
  NVFP4_ERR_UNSUPPORTED_SHAPE = 2, /* a size the kernels do not handle        */
  NVFP4_ERR_CUDA = 3,              /* a CUDA runtime or driver call failed    */
  NVFP4_ERR_TIMEOUT = 4,           /* a device-side wait gave up              */
  NVFP4_ERR_WORKSPACE = 5,         /* workspace missing, misaligned or small  */
  NVFP4_ERR_DEVICE = 6             /* the current device is not an sm_100 GPU */
} nvfp4_status;

enum { NVFP4_LAYOUT_CANONICAL = 0, NVFP4_LAYOUT_TILED = 1, NVFP4_LAYOUT_STAGED = 2 };

/* Message for the last failed call on this host thread ("" if none). */
NVFP4_API const char* nvfp4_last_error(void);

/* Version of this interface (incremented on any signature change). */
NVFP4_API int nvfp4_abi_version(void);

/* Synchronises `stream`, then reads the status word a call left at the start
 * of `ws`: NVFP4_OK, or NVFP4_ERR_TIMEOUT if a device-side wait gave up (the
 * outputs of that call are then undefined).  Resets the word to 0. */
NVFP4_API nvfp4_status nvfp4_workspace_status(void* ws, void* stream);

/* ------------------------------------------------------------------------
 * Offline RTN weight quantiser ("Quantization Setup": round-to-nearest weight
 * quantisation at per-expert Linear granularity).
 *
 * Quantises n_mats independent bf16 matrices w[n_mats][rows][cols].  For each
 * matrix: g = amax|w| / (6 * 448) (fp32 division); for each 16-element block
 * of a row: s = E4M3(amax_block / (6 g)), S = s * g, codes = E2M1(x * (1/S))
 * with round-to-nearest-even and saturation; a zero block or matrix gives
 * scale 0 and codes +-0.
 *   codes        [n_mats][rows][cols/2]; STAGED: each matrix's codes in the
 *                staged layout (its n_mats * rows * cols / 2 bytes)
 *   scales       CANONICAL: [n_mats][rows][cols/16];
 *                TILED, STAGED: n_mats * rows rows in the tiled layout
 *                (rows % 128 == 0)
 *   global_scale [n_mats] fp32
 * Needs cols % 32 == 0 (TILED: cols % 64 == 0, rows % 128 == 0; STAGED:
 * cols % 256 == 0, rows % 128 == 0).
 * Each matrix is read twice (amax pass, then quantise pass) with the second
 * read scheduled while the matrix is still in L2.
 * ---------------------------------------------------------------------- */
NVFP4_API size_t nvfp4_quantize_weights_workspace_size(int n_mats);
NVFP4_API nvfp4_status nvfp4_quantize_weights(const void* w_bf16, int n_mats, int rows, int cols, int layout,
                                    uint8_t* codes, uint8_t* scales, float* global_scale, void* ws,
                                    size_t ws_bytes, void* stream);

/* Same quantiser, for callers that cannot allocate device memory.  The pages
 * have no counterpart to this entry point; it exists for hosts whose device
 * memory is owned by another allocator (a serving engine's arena, a plugin
 * host's fixed pool) so that they cannot provide the workspace above, or that
 * run where device allocation calls are not allowed.  It takes no workspace
 * and allocates nothing: its scratch is a 8448-byte array inside the library,
 * which every GPU that loads the library keeps until the process exits.
 *   - At most 1024 matrices per call; more returns
 *     NVFP4_ERR_UNSUPPORTED_SHAPE (split the call or use the workspace form).
 *   - Every call looks up the array's device address in the current context
 *     (a host-side query, no allocation).  The first call in a context may
 *     also load the library's device code there, so make it before any
 *     stream capture on that device.
 *   - Every call shares the one array and clears it when it starts, so calls
 *     whose work overlaps on the GPU (different streams, or different host
 *     threads on one device) race; serialise them on one stream.
 *   - A device-side wait that gives up sets the status word at the start of
 *     the array: read it with nvfp4_quantize_weights_noalloc_status() before
 *     the next call, which clears it.  The outputs of that call are then
 *     undefined, as with the workspace form.
 * Arguments, layouts and results are those of nvfp4_quantize_weights. */
NVFP4_API nvfp4_status nvfp4_quantize_weights_noalloc(const void* w_bf16, int n_mats, int rows, int cols,
                                                      int layout, uint8_t* codes, uint8_t* scales,
                                                      float* global_scale, void* stream);

/* The status of the last nvfp4_quantize_weights_noalloc call on the current
 * device, the counterpart of nvfp4_workspace_status for the built-in array
 * (no counterpart on the pages either).  Synchronises `stream` (the stream
 * that call used), then reads the status word: NVFP4_OK, or
 * NVFP4_ERR_TIMEOUT if a device-side wait of that call gave up, in which case
 * the word is reset to 0.  Allocates nothing. */
NVFP4_API nvfp4_status nvfp4_quantize_weights_noalloc_status(void* stream);

/* ------------------------------------------------------------------------
 * Dynamic activation quantiser ("Quantization Setup": activations dynamically
 * quantised to FP4 with calibrated global scales).
 *
 * x[rows][cols] bf16 under the caller's calibrated global scale (one fp32 in
 * device memory), same block arithmetic as the weight quantiser.
 *   codes  [rows][cols/2];  scales CANONICAL [rows][cols/16] or TILED
 *   (rows beyond `rows` in the last 128-row tile get scale 0).
 * Needs cols % 32 == 0 (TILED: cols % 64 == 0).
 * ---------------------------------------------------------------------- */
NVFP4_API nvfp4_status nvfp4_quantize_act(const void* x_bf16, int rows, int cols, const float* global_scale,
                                int layout, uint8_t* codes, uint8_t* scales, void* stream);

/* ------------------------------------------------------------------------
 * Router and permutation ("Pruning Setup", "Routing behavior").
 *
 * logits = x W^T + logit_offset (bf16 operands, fp32 accumulation; the
 * optional per-expert logit_offset is a synthetic load-skew knob, not part of
 * the method), or the caller's logits_in when that is non-NULL (then x_bf16,
 * router_weight_bf16 and logit_offset must be NULL).
 * sigma = 1 / (1 + exp(-logit)) with a fixed fp32 exp (Cody-Waite reduction by
 * ln 2, degree-7 Taylor polynomial, IEEE operations only, |logit| clamped to
 * 80); the k experts with the largest sigma + bias are selected (ties to the
 * lower index) in descending order; w_j = (sigma_j / sum_sel sigma) * rsf
 * with the sum taken in fp32 in that order.
 * Permutation: pairs (token t, slot j) ordered by expert, token, slot; each
 * expert's segment padded to a multiple of 128 rows.
 *   logits_out     [T][E] fp32 (nullable)
 *   topk_idx       [T][k] int32;  topk_w [T][k] fp32
 *   expert_offsets [E+1] int32 (row where each expert's segment starts)
 *   perm           [moe_route_rows_capacity(T,E,k)] int32: token of each row,
 *                  -1 on padding rows and beyond expert_offsets[E]
 *   inv_perm       [T][k] int32: row of each (token, slot)
 * Needs 1 <= k <= 16, k <= E <= 256, H % 64 == 0.
 * ---------------------------------------------------------------------- */
NVFP4_API int moe_route_rows_capacity(int T, int E, int k);
NVFP4_API size_t moe_route_workspace_size(int T, int E, int k);
NVFP4_API nvfp4_status moe_route(const void* x_bf16, const void* router_weight_bf16, const float* logits_in,
                       const float* bias, const float* logit_offset, int T, int H, int E, int k,
                       float routed_scaling_factor, float* logits_out, int32_t* topk_idx, float* topk_w,
                       int32_t* expert_offsets, int32_t* perm, int32_t* inv_perm, void* ws, size_t ws_bytes,
                       void* stream);

/* ------------------------------------------------------------------------
 * The layer.
 * ---------------------------------------------------------------------- */
typedef struct moe_nvfp4_weights {
  int E, H, I, k;                 /* experts, hidden, expert intermediate, top-k */
  float routed_scaling_factor;
  const void* router_weight;      /* bf16 [E][H] (kept BF16)                     */
  const float* bias;              /* fp32 [E] e_score_correction_bias            */
  const uint8_t* gate_codes;      /* [E][I][H/2]                                 */
  const uint8_t* gate_scales;     /* TILED, E*I rows x H cols                    */
  const float* gate_gscale;       /* [E]                                         */
  const uint8_t* up_codes;        /* [E][I][H/2]                                 */
  const uint8_t* up_scales;       /* TILED, E*I rows x H cols                    */
  const float* up_gscale;         /* [E]                                         */
  const uint8_t* down_codes;      /* [E][H][I/2]                                 */
  const uint8_t* down_scales;     /* TILED, E*H rows x I cols                    */
  const float* down_gscale;       /* [E]                                         */
  /* The shared expert, kept BF16 (NVFP4 card, "Quantization Setup"; its size
   * is not on the pages): out += down_s(silu(gate_s x) * up_s x) for every
   * token, the intermediate rounded to bf16.  NULL pointers and I_shared 0:
   * no shared expert.  I_shared % 128 == 0. */
  const void* shared_gate;        /* bf16 [I_shared][H]                          */
  const void* shared_up;          /* bf16 [I_shared][H]                          */
  const void* shared_down;        /* bf16 [H][I_shared]                          */
  int I_shared;
  /* Layout of gate_codes, up_codes and down_codes: NVFP4_LAYOUT_CANONICAL
   * (0, row-major as above) or NVFP4_LAYOUT_STAGED (needs H % 256 == 0 and
   * I % 256 == 0).  The scales are TILED either way. */
  int codes_layout;
} moe_nvfp4_weights;

/* Optional copies of intermediate results (every pointer nullable; device
 * memory; row-indexed buffers have moe_route_rows_capacity(T,E,k) rows). */
typedef struct moe_nvfp4_debug {
  float* logits;                  /* [T][E]                                      */
  int32_t* topk_idx;              /* [T][k]                                      */
  float* topk_w;                  /* [T][k]                                      */
  int32_t* expert_offsets;        /* [E+1]                                       */
  int32_t* perm;                  /* [rows]                                      */
  int32_t* inv_perm;              /* [T][k]                                      */
  uint8_t* a_codes;               /* [rows][H/2] quantised x in permuted order   */
  uint8_t* a_scales;              /* TILED, rows x H                             */
  float* h;                       /* [rows][I] silu(gate)*up before requantising */
  float* h_amax;                  /* max |h| over real rows (fp32, caller zeroes);
                                     [E], one per expert, in the per-expert modes */
  uint8_t* h_codes;               /* [rows][I/2]                                 */
  uint8_t* h_scales;              /* TILED, rows x I                             */
  float* y;                       /* [rows][H] weighted down-projection rows     */
  /* cudaEvent_t handles (nullable, each created by the caller): recorded on
   * `stream` at the start and after each stage (0 start, 1 routing and
   * permutation, 2 quantise x, 3 gate/up GEMM, 4 down GEMM, 5 combine), so a
   * caller can time every stage of a call on the device. */
  void* stage_events[6];
  /* REAP saliency accumulators ("K-EXAONE-152B-A23B-REAP-80E-BF16" card,
   * "Pruning Setup": saliency = mean(topk_weight * ||f_e(x)||_2) over routed
   * tokens).  Nullable, [E] each, owned and zeroed by the caller; every call
   * ADDS its batch: saliency_sum[e] += sum over the (token, slot) pairs routed
   * to e of w * ||y||_2, with y the expert's fp32 down output before the
   * routing weight w; saliency_count[e] += their number.  Sum over
   * calibration batches, then divide.  Deterministic: fixed reduction order. */
  double* saliency_sum;
  unsigned long long* saliency_count;
  /* cudaEvent_t (nullable): recorded on `stream` after the shared expert's
   * GEMMs, when the layer has a shared expert (they run between stage events
   * 4 and 5, before the combine). */
  void* shared_event;
} moe_nvfp4_debug;

/* REAP expert retention ("K-EXAONE-152B-A23B-REAP-80E-BF16" card, "Pruning
 * Setup": the routed experts with the lowest saliency are dropped, and the
 * router's gate.weight and e_score_correction_bias are sliced to the ones
 * kept).  From the accumulators of moe_nvfp4_debug (device, [E] each): the
 * mean saliency of expert e is saliency_sum[e] / saliency_count[e] in IEEE
 * fp64 (0 for an expert never routed); the `keep` experts with the highest
 * means are retained, ties to the lower index, and keep_idx[0..keep) (device
 * int32) receives their indices in increasing order.  Needs 1 <= E <= 256,
 * 0 <= keep <= E. */
NVFP4_API nvfp4_status moe_reap_keep(const double* saliency_sum, const unsigned long long* saliency_count, int E,
                                     int keep, int32_t* keep_idx, void* stream);

NVFP4_API size_t moe_nvfp4_workspace_size(int T, int E, int H, int I, int k);
/* The same with a shared expert of intermediate size I_shared (0: none). */
NVFP4_API size_t moe_nvfp4_workspace_size_shared(int T, int E, int H, int I, int k, int I_shared);

/* out[T][H] bf16 = [shared(x) +] sum_j w_j * down_e( quant_g2( silu(gate_e(xq)) * up_e(xq) ) )
 * with xq = x quantised under act_gscale (g1) and the intermediate quantised
 * under h_gscale (g2), both one fp32 in device memory.  Steps: router GEMM ->
 * top-k -> permutation -> quantise x into permuted rows -> grouped FP4 GEMM
 * gate/up with SiLU*up and requantisation fused -> grouped FP4 GEMM down with
 * g2 * g_down * w_j fused -> [shared expert: bf16 GEMMs gate/up with SiLU*up,
 * then down] -> combine: fp32 sum of the shared row and the k rows in slot
 * order, bf16 out.  With a shared expert the workspace comes from
 * moe_nvfp4_workspace_size_shared.
 * Needs H % 256 == 0, I % 128 == 0, 1 <= k <= 16, k <= E <= 256, T >= 1. */
NVFP4_API nvfp4_status moe_nvfp4_forward(const moe_nvfp4_weights* W, const void* x_bf16, int T,
                               const float* act_gscale, const float* h_gscale, const float* logit_offset,
                               void* out_bf16, const moe_nvfp4_debug* dbg, void* ws, size_t ws_bytes,
                               void* stream);

/* ------------------------------------------------------------------------
 * The forward on host buffers, for a caller whose tokens live in host memory
 * (no counterpart on the pages: it is the serving wrapper around the layer).
 * x_host_bf16 [T][H] and out_host_bf16 [T][H] are host pointers, page-locked
 * for the copies to run asynchronously.  The call enqueues, and returns
 * without waiting:
 *   1. the copy of x into a staging buffer at the end of `ws`, on a copy
 *      stream of the library's own;
 *   2. moe_nvfp4_forward (per-tensor scales, no debug outputs) on `stream`,
 *      reading the staged x and writing a staged out;
 *   3. the copy of out back to out_host_bf16, on a second copy stream.
 * Consecutive calls on DIFFERENT workspaces overlap: one call's copies run
 * while another computes.  A call on the same workspace as an earlier one
 * waits for that call's copies before it reuses its staging buffers.  The
 * library keeps three CUDA events per workspace (until
 * moe_nvfp4_host_release) and two copy streams per device.
 * out_host_bf16 holds the result once the work that moe_nvfp4_host_join
 * orders has completed (for example, after join then a synchronize of
 * `stream`).  x_host_bf16 must not change before the copy in has run.  The
 * workspace comes from moe_nvfp4_workspace_size_host.  It belongs to one
 * device, and its status word is read with nvfp4_workspace_status as for
 * moe_nvfp4_forward. */
NVFP4_API size_t moe_nvfp4_workspace_size_host(int T, int E, int H, int I, int k, int I_shared);
NVFP4_API nvfp4_status moe_nvfp4_forward_host(const moe_nvfp4_weights* W, const void* x_host_bf16, int T,
                                    const float* act_gscale, const float* h_gscale, const float* logit_offset,
                                    void* out_host_bf16, void* ws, size_t ws_bytes, void* stream);
/* Makes `stream` wait until the last moe_nvfp4_forward_host call on `ws` has
 * copied its out back (nothing to wait for: returns at once). */
NVFP4_API nvfp4_status moe_nvfp4_host_join(const void* ws, void* stream);
/* Waits for the last call on `ws` to finish its copies, then frees the
 * library's events for that workspace (call before freeing `ws`). */
NVFP4_API nvfp4_status moe_nvfp4_host_release(const void* ws);

/* Activation global-scale modes of moe_nvfp4_forward_scaled.  The pages fix
 * one calibrated fp32 global scale per activation tensor ("Quantization
 * Setup"); the other modes are an extension: one scale per expert, and g1
 * derived on the device from the batch with the weight rule
 * g1 = fl32(amax|x| / 2688), taken over the whole batch or over the tokens
 * routed to each expert (0 for an expert without tokens).
 *   mode                          act_gscale              h_gscale
 *   NVFP4_ACT_SCALE_TENSOR         [1] read                [1]
 *   NVFP4_ACT_SCALE_EXPERT         [E] read                [E]
 *   NVFP4_ACT_SCALE_DYNAMIC        [1] written (batch g1)  [1]
 *   NVFP4_ACT_SCALE_DYNAMIC_EXPERT [E] written (per expert) [E]
 * With one g1 per expert, each of a token's k permuted rows is quantised under
 * its own expert's g1, and expert e's h rows under h_gscale[e]. */
enum {
  NVFP4_ACT_SCALE_TENSOR = 0,
  NVFP4_ACT_SCALE_EXPERT = 1,
  NVFP4_ACT_SCALE_DYNAMIC = 2,
  NVFP4_ACT_SCALE_DYNAMIC_EXPERT = 3
};

/* moe_nvfp4_forward with a choice of activation global-scale mode (above);
 * moe_nvfp4_forward is this call with NVFP4_ACT_SCALE_TENSOR.  Same workspace,
 * layouts and errors; an unknown mode returns NVFP4_ERR_INVALID_ARG. */
NVFP4_API nvfp4_status moe_nvfp4_forward_scaled(const moe_nvfp4_weights* W, const void* x_bf16, int T,
                                                int act_scale_mode, float* act_gscale, const float* h_gscale,
                                                const float* logit_offset, void* out_bf16,
                                                const moe_nvfp4_debug* dbg, void* ws, size_t ws_bytes,
                                                void* stream);

/* Number of kernels one moe_nvfp4_forward_scaled call (act_scale_mode; mode 0
 * is moe_nvfp4_forward) queues for this shape, without the REAP saliency
 * kernel that the debug struct can add; memsets are not kernels.  It depends
 * on the shape only: small batches route in one kernel, and small layers
 * quantise x inside it.  Host-only arithmetic, no CUDA call.  Returns -1 for
 * a shape or mode the forward rejects.  This has no counterpart on the pages:
 * it lets a caller account for the launches it measures. */
NVFP4_API int moe_nvfp4_forward_launches(int T, int E, int H, int I, int k, int I_shared, int act_scale_mode);

/* ------------------------------------------------------------------------
 * The two grouped GEMMs on caller-supplied quantised operands (the same
 * kernels moe_nvfp4_forward runs).  Rows are grouped by expert_offsets
 * ([E+1], each segment a multiple of 128 rows, expert_offsets[E] <=
 * rows_capacity); expert_counts ([E], nullable) gives the rows of each segment
 * that hold data (rows past it are written as zeros / skipped).
 * ---------------------------------------------------------------------- */
NVFP4_API size_t moe_nvfp4_gemm_workspace_size(int rows_capacity);

/* h = silu(g1 g_gate[e] acc_gate) * (g1 g_up[e] acc_up), then quantised under
 * h_gscale into h_codes [rows][I/2] and TILED h_scales.  h_f32 ([rows][I]) and
 * h_amax (one fp32, caller zeroes) are optional outputs. */
NVFP4_API nvfp4_status moe_nvfp4_gate_up(const moe_nvfp4_weights* W, const uint8_t* a_codes, const uint8_t* a_scales,
                               const int32_t* expert_offsets, const int32_t* expert_counts, int rows_capacity,
                               const float* act_gscale, const float* h_gscale, uint8_t* h_codes,
                               uint8_t* h_scales, float* h_f32, float* h_amax, void* ws, size_t ws_bytes,
                               void* stream);

/* y[r] = g2 g_down[e] row_weight[r] acc_down[r]: y_bf16 [rows][H] and/or
 * y_f32 [rows][H] (each nullable, not both).  row_weight nullable (= 1). */
NVFP4_API nvfp4_status moe_nvfp4_down(const moe_nvfp4_weights* W, const uint8_t* h_codes, const uint8_t* h_scales,
                            const int32_t* expert_offsets, const int32_t* expert_counts, int rows_capacity,
                            const float* h_gscale, const float* row_weight, void* y_bf16, float* y_f32,
                            void* ws, size_t ws_bytes, void* stream);

/* ------------------------------------------------------------------------
 * Block-scale distortion statistics (NetsPresso AQ article, section "Why
 * 4-Bit Quantization of MoE Models Is Hard: Outliers in the Final Two
 * Layers": the share of weights with |w| > 0.1, and the way concentrated
 * outliers distort the NVFP4 block scale and the precision of the other
 * weights of their block).
 *
 * For each of n_mats matrices w[m] ([rows][cols] bf16) and its NVFP4 encoding
 * (codes and scales in `layout` as the weight quantiser writes them,
 * global_scale[n_mats]), stats[m] receives:
 *   elements, outliers            elements; elements with |w| > threshold
 *   blocks, outlier_blocks        16-element blocks; blocks holding an outlier
 *   zero_scale_blocks             blocks with scale code 0
 *   subnormal_scale_blocks        blocks with an E4M3 subnormal scale (codes 1..7)
 *   saturated_elements            |fl32(w * fl32(1/S))| > 6, S = fl32(E4M3(s) g):
 *                                 elements the E2M1 conversion clamps
 *   neighbours, clean             non-outlier elements of outlier blocks;
 *                                 elements of blocks without outliers
 *   sum_sq, sse                   sum of w^2 and of (w - dq)^2, where
 *                                 dq = fl32(fl32(E2M1(q) E4M3(s)) g)
 *   *_neighbours, *_clean         the same two sums over those subsets
 * Counts are exact.  The sums are taken in fp32 within a block and in fp64
 * across blocks, which keeps them within about 1e-6 relative.  `stats`
 * is device memory of n_mats entries; the call overwrites it.  Needs
 * cols % 16 == 0 (TILED: cols % 64 == 0, rows % 128 == 0; STAGED:
 * cols % 256 == 0, rows % 128 == 0), w 16-byte and codes and stats 8-byte
 * aligned.  Reads 2.5625 bytes per element.
 * ---------------------------------------------------------------------- */
typedef struct {
  uint64_t elements, outliers, blocks, outlier_blocks, zero_scale_blocks, subnormal_scale_blocks,
      saturated_elements, neighbours, clean;
  double sum_sq, sse, sum_sq_neighbours, sse_neighbours, sum_sq_clean, sse_clean;
} nvfp4_block_stats;

NVFP4_API nvfp4_status nvfp4_block_stats_compute(const void* w_bf16, const uint8_t* codes, const uint8_t* scales,
                                                 const float* global_scale, int n_mats, int rows, int cols,
                                                 int layout, float outlier_threshold, nvfp4_block_stats* stats,
                                                 void* stream);

#ifdef __cplusplus
}
#endif
#endif /* NVFP4_MOE_H */
