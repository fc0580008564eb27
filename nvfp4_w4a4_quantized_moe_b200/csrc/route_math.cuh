// Fixed fp32 sigmoid of the router (shared by the router kernels and the
// test hooks of the library).
#pragma once

#include "common.cuh"

namespace nvfp4moe {

// ---------------------------------------------------------------------------
// fp32 exp from IEEE operations only, no fused multiply-add: Cody and Waite's
// reduction v = n ln2 + r with ln 2 split into a 16-bit head and its
// remainder, then e^r by the degree-7 Taylor polynomial in Horner form, then
// the exact power of two.  Constants (all rounded to fp32):
//   1/ln2, ln2 to 16 significant bits, ln2 minus that head, 1/j! for j <= 7.
// ---------------------------------------------------------------------------
NVDEV float exp_fixed(float v) {
  const float kLog2e = 0x1.715476p+0f;
  const float kLn2Hi = 0x1.62e4p-1f;
  const float kLn2Lo = 0x1.7f7d1cp-20f;
  const float c[8] = {1.0f, 1.0f, 0.5f, 0x1.555556p-3f, 0x1.555556p-5f, 0x1.111112p-7f, 0x1.6c16c2p-10f,
                      0x1.a01a02p-13f};
  v = fminf(fmaxf(v, -80.0f), 80.0f);
  const float n = rintf(__fmul_rn(v, kLog2e));
  const float r = __fsub_rn(__fsub_rn(v, __fmul_rn(n, kLn2Hi)), __fmul_rn(n, kLn2Lo));
  float p = c[7];
#pragma unroll
  for (int j = 6; j >= 0; --j) p = __fadd_rn(__fmul_rn(p, r), c[j]);
  const float two_n = __int_as_float(((int)n + 127) << 23);
  return __fmul_rn(p, two_n);
}

NVDEV float sigmoid_fixed(float l) { return __fdiv_rn(1.0f, __fadd_rn(1.0f, exp_fixed(-l))); }

}  // namespace nvfp4moe
