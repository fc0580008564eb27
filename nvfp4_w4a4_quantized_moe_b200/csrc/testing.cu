// Test hooks: element-wise access to the device conversions and the router's
// sigmoid, for comparison with an independent CPU implementation.
#include "../../include/nvfp4_moe_testing.h"
#include "common.cuh"
#include "host.cuh"
#include "route_math.cuh"

namespace nvfp4moe {

__global__ void test_e2m1_kernel(const float* y, int n, uint8_t* hw, uint8_t* sw) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= n) return;
  float v[8] = {y[i], 0, 0, 0, 0, 0, 0, 0};
  hw[i] = (uint8_t)(e2m1x8_hw(v) & 0xFu);
  sw[i] = (uint8_t)e2m1_sw(y[i]);
}

__global__ void test_e2m1_sweep_kernel(uint32_t first, uint64_t count, unsigned long long* mismatches,
                                       uint32_t* example) {
  unsigned long long local = 0;
  uint32_t bad = 0;
  bool have_bad = false;
  const uint64_t stride = (uint64_t)gridDim.x * blockDim.x * 8;
  for (uint64_t base = ((uint64_t)blockIdx.x * blockDim.x + threadIdx.x) * 8; base < count; base += stride) {
    float v[8];
    uint32_t sw = 0;
#pragma unroll
    for (int q = 0; q < 8; ++q) {
      const uint64_t idx = base + q;
      const uint32_t bits = (uint32_t)(first + idx);
      float f = __uint_as_float(bits);
      if (idx >= count || (bits & 0x7F800000u) == 0x7F800000u && (bits & 0x7FFFFFu)) f = 0.0f;   // skip NaN
      v[q] = f;
      sw |= e2m1_sw(f) << (4 * q);
    }
    const uint32_t hw = e2m1x8_hw(v);
    if (hw != sw) {
#pragma unroll
      for (int q = 0; q < 8; ++q) {
        if (((hw >> (4 * q)) & 0xF) != ((sw >> (4 * q)) & 0xF)) {
          ++local;
          if (!have_bad) {
            bad = (uint32_t)(first + base + q);
            have_bad = true;
          }
        }
      }
    }
  }
  if (local) {
    atomicAdd(mismatches, local);
    atomicExch(example, bad);
  }
}

__global__ void test_e4m3_kernel(const float* s, int n, uint8_t* codes, float* value) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= n) return;
  const uint32_t c = e4m3_code(s[i]);
  codes[i] = (uint8_t)c;
  value[i] = e4m3_value(c);
}

__global__ void test_sigmoid_kernel(const float* l, int n, float* out) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i < n) out[i] = sigmoid_fixed(l[i]);
}

}  // namespace nvfp4moe

using namespace nvfp4moe;

extern "C" nvfp4_status nvfp4_test_e2m1(const float* y, int n, uint8_t* hw, uint8_t* sw, void* stream) {
  NV_REQUIRE(y && hw && sw && n >= 0, NVFP4_ERR_INVALID_ARG, "nvfp4_test_e2m1: bad arguments");
  int sms = 0;
  NV_CHECK(device_sm_count(&sms));
  if (n == 0) return NVFP4_OK;
  test_e2m1_kernel<<<(n + 255) / 256, 256, 0, as_stream(stream)>>>(y, n, hw, sw);
  return check_launch("test_e2m1_kernel");
}

extern "C" nvfp4_status nvfp4_test_e2m1_sweep(uint32_t first, uint64_t count, unsigned long long* mismatches,
                                              uint32_t* example, void* stream) {
  NV_REQUIRE(mismatches && example, NVFP4_ERR_INVALID_ARG, "nvfp4_test_e2m1_sweep: bad arguments");
  NV_REQUIRE(count <= (1ull << 32) && (uint64_t)first + count <= (1ull << 32), NVFP4_ERR_INVALID_ARG,
             "nvfp4_test_e2m1_sweep: range beyond 2^32");
  int sms = 0;
  NV_CHECK(device_sm_count(&sms));
  if (count == 0) return NVFP4_OK;
  test_e2m1_sweep_kernel<<<sms * 8, 256, 0, as_stream(stream)>>>(first, count, mismatches, example);
  return check_launch("test_e2m1_sweep_kernel");
}

extern "C" nvfp4_status nvfp4_test_e4m3(const float* s, int n, uint8_t* codes, float* value, void* stream) {
  NV_REQUIRE(s && codes && value && n >= 0, NVFP4_ERR_INVALID_ARG, "nvfp4_test_e4m3: bad arguments");
  int sms = 0;
  NV_CHECK(device_sm_count(&sms));
  if (n == 0) return NVFP4_OK;
  test_e4m3_kernel<<<(n + 255) / 256, 256, 0, as_stream(stream)>>>(s, n, codes, value);
  return check_launch("test_e4m3_kernel");
}

extern "C" nvfp4_status nvfp4_test_sigmoid(const float* l, int n, float* out, void* stream) {
  NV_REQUIRE(l && out && n >= 0, NVFP4_ERR_INVALID_ARG, "nvfp4_test_sigmoid: bad arguments");
  int sms = 0;
  NV_CHECK(device_sm_count(&sms));
  if (n == 0) return NVFP4_OK;
  test_sigmoid_kernel<<<(n + 255) / 256, 256, 0, as_stream(stream)>>>(l, n, out);
  return check_launch("test_sigmoid_kernel");
}
