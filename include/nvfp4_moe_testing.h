/*
 * nvfp4_moe_testing.h - test hooks of libnvfp4moe.so.
 *
 * These entry points expose the device-side building blocks of the layer so
 * that tests can compare them element by element with an independent CPU
 * implementation: the E2M1 and E4M3 conversions used by every quantiser
 * (element formats of the "K-EXAONE-152B-A23B-REAP-80E-NVFP4" model card,
 * "Quantization Setup") and the fixed fp32 sigmoid of the router
 * ("K-EXAONE-152B-A23B-REAP-80E-BF16" model card, "Routing behavior"), and
 * the router GEMM's split of K, which fixes the logits' fp32 rounding.
 * Same conventions as nvfp4_moe.h: device pointers, asynchronous on `stream`,
 * nvfp4_status results.  They are not needed to run the layer.
 */
#ifndef NVFP4_MOE_TESTING_H
#define NVFP4_MOE_TESTING_H

#include "nvfp4_moe.h"

#ifdef __cplusplus
extern "C" {
#endif

/* For each y[i] (fp32), hw[i] = the E2M1 code the quantisers produce (the
 * hardware conversion, round to nearest even, saturating) and sw[i] = the
 * same rounding written as comparisons against the grid midpoints. */
NVFP4_API nvfp4_status nvfp4_test_e2m1(const float* y, int n, uint8_t* hw, uint8_t* sw, void* stream);

/* Counts, over the fp32 bit patterns [first, first + count) that are not
 * NaN, how many give different hardware and comparison E2M1 codes; adds the
 * count to *mismatches (device uint64) and records one offending pattern in
 * *example (device uint32; left unchanged if none). */
NVFP4_API nvfp4_status nvfp4_test_e2m1_sweep(uint32_t first, uint64_t count, unsigned long long* mismatches,
                                             uint32_t* example, void* stream);

/* codes[i] = E4M3 code of s[i] >= 0 (nearest even, saturating at 448) and
 * value[i] = the value of that code. */
NVFP4_API nvfp4_status nvfp4_test_e4m3(const float* s, int n, uint8_t* codes, float* value, void* stream);

/* FP4 tensor-core rate without memory traffic: `ctas` CTAs (at most one per
 * SM) each issue `iters` x 4 block-scaled 128 x n x 64 MMAs (n = 128 or 256)
 * from fixed shared-memory operands.  with_cp selects what else one issuing
 * thread does per 4 MMAs (one 256-wide K stage):
 *   0 nothing; 1 the stage's 12 scale-factor copies into one set of tensor
 *   memory columns; 2 the same rotating over four sets; 3 copies issued one
 *   stage ahead; 4 six 128-lane x 256-bit copies instead of twelve;
 *   5/6 (without/with copies) a full/empty mbarrier handshake with a second
 *   thread over 4 stages, 9/10 over 8 stages, 7/8 with spinning waits,
 *   11/12 over 8 stages of 2 MMAs; 13 copies and a tcgen05.commit (no wait);
 *   14 a commit only; 15 copies and a tcgen05 after-thread-sync fence;
 *   16 copies and a commit every second stage; 17 split issue: this thread
 *   issues only the MMAs and a second thread the copies, into two
 *   alternating column sets, with mbarrier handshakes; 18 the same plus a
 *   full/empty handshake with a third thread; 19-21 the whole warp runs
 *   the loop and one elected lane issues: 19 copies and MMAs as predicated
 *   instructions, 20 MMAs only, 21 copies and MMAs in a branch.
 * cycles[c] (device uint64) = SM clock cycles CTA c spent; *status (device
 * uint32) is set non-zero if a wait gave up.  INVALID_ARG for with_cp outside
 * [0, 21]. */
NVFP4_API nvfp4_status nvfp4_test_mma_peak(int iters, int n, int with_cp, int ctas, unsigned long long* cycles,
                                           uint32_t* status, void* stream);

/* Makes a bounded device wait run out, to test the give-up path that every
 * wait of the library shares (no counterpart on the pages: it checks the
 * status-word contract of nvfp4_moe.h).  One CTA issues a 4 KiB bulk copy
 * from src (device, 16-byte aligned) and allocates tensor memory, then waits
 * on a barrier that nothing completes, with the library's bounded wait and
 * the limit limit_ns (0 < limit_ns <= 1e9).  When the wait gives up it sets
 * the status word at the start of `ws` (read it with
 * nvfp4_workspace_status), lets the copy land, drains its tensor-core work
 * and frees the tensor memory.  elapsed_ns[0] (device) receives how long the
 * limited wait lasted, elapsed_ns[1] how long a second warp waited before it
 * saw the abort flag; *copied (device) the XOR of the 1024 copied words. */
NVFP4_API nvfp4_status nvfp4_test_wait_timeout(const void* src, uint64_t limit_ns, void* ws, size_t ws_bytes,
                                               unsigned long long* elapsed_ns, uint32_t* copied, void* stream);

/* For each (amax[i] >= 0, g[i] >= 0): q_lib[i] = the block-scale quotient
 * amax / (6 g) as the quantisers compute it (a three-instruction division by
 * Markstein's method where 6 g is in range, else IEEE division; quotients of
 * 464 and more may come out as 464), q_ieee[i] = the same by CUDA's IEEE
 * division, and code_lib[i], code_ieee[i] = their E4M3 codes. */
NVFP4_API nvfp4_status nvfp4_test_block_scale_div(const float* amax, const float* g, int n, float* q_lib,
                                                  float* q_ieee, uint8_t* code_lib, uint8_t* code_ieee,
                                                  void* stream);

/* out[i] = the router's fp32 sigmoid of l[i]. */
NVFP4_API nvfp4_status nvfp4_test_sigmoid(const float* l, int n, float* out, void* stream);

/* Host arithmetic only, no CUDA call: the number of K splits the router GEMM
 * of moe_route and the layer uses for T tokens and hidden size H (one CTA
 * per 128 tokens and split, at most 148 CTAs, at least four 64-column K
 * stages per split where H allows, and no split without stages), with the
 * stages each split takes (the last may take fewer) in *stages_per_split
 * when it is not NULL.  The logits' fp32 rounding follows this split.
 * Returns -1 when T < 1 or H is not a positive multiple of 64. */
NVFP4_API int nvfp4_test_router_splits(int T, int H, int* stages_per_split);

#ifdef __cplusplus
}
#endif
#endif /* NVFP4_MOE_TESTING_H */
