// Error reporting, device checks, tensor maps and the status-word reader.
#include <string.h>

#include <mutex>

#include "host.cuh"

namespace nvfp4moe {

static thread_local char g_last_error[512] = "";

nvfp4_status set_error(nvfp4_status st, const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_last_error, sizeof(g_last_error), fmt, ap);
  va_end(ap);
  return st;
}

nvfp4_status check_cuda(cudaError_t e, const char* what) {
  if (e == cudaSuccess) return NVFP4_OK;
  return set_error(NVFP4_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

nvfp4_status check_launch(const char* what) { return check_cuda(cudaGetLastError(), what); }

nvfp4_status device_sm_count(int* sms) {
  int dev = 0;
  NV_CHECK(check_cuda(cudaGetDevice(&dev), "cudaGetDevice"));
  static int cached_dev = -1, cached_sms = 0, cached_major = 0;
  static std::mutex mu;
  std::lock_guard<std::mutex> lock(mu);
  if (dev != cached_dev) {
    int major = 0, count = 0;
    NV_CHECK(check_cuda(cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev),
                        "cudaDeviceGetAttribute"));
    NV_CHECK(check_cuda(cudaDeviceGetAttribute(&count, cudaDevAttrMultiProcessorCount, dev),
                        "cudaDeviceGetAttribute"));
    cached_dev = dev;
    cached_sms = count;
    cached_major = major;
  }
  if (cached_major != 10)
    return set_error(NVFP4_ERR_DEVICE, "device %d has compute capability %d.x; this library is built for sm_100a",
                     dev, cached_major);
  *sms = cached_sms;
  return NVFP4_OK;
}

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

static EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

nvfp4_status make_tmap_2d(CUtensorMap* map, const void* base, CUtensorMapDataType dtype, uint64_t inner,
                          uint64_t outer, uint64_t pitch_bytes, uint32_t box_inner, uint32_t box_outer,
                          bool swizzle128) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return set_error(NVFP4_ERR_CUDA, "cuTensorMapEncodeTiled is not available from the driver");
  cuuint64_t dims[2] = {inner, outer};
  cuuint64_t strides[1] = {pitch_bytes};
  cuuint32_t box[2] = {box_inner, box_outer};
  cuuint32_t elem_strides[2] = {1, 1};
  CUresult r = fn(map, dtype, 2, const_cast<void*>(base), dims, strides, box, elem_strides,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_NONE,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS)
    return set_error(NVFP4_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d) for a %llu x %llu tensor", (int)r,
                     (unsigned long long)inner, (unsigned long long)outer);
  return NVFP4_OK;
}

}  // namespace nvfp4moe

using namespace nvfp4moe;

extern "C" const char* nvfp4_last_error(void) { return g_last_error; }

extern "C" int nvfp4_abi_version(void) { return 6; }

extern "C" nvfp4_status nvfp4_workspace_status(void* ws, void* stream) {
  NV_REQUIRE(ws != nullptr, NVFP4_ERR_INVALID_ARG, "nvfp4_workspace_status: ws is NULL");
  uint32_t word = 0;
  cudaStream_t s = as_stream(stream);
  NV_CHECK(check_cuda(cudaMemcpyAsync(&word, ws, sizeof(word), cudaMemcpyDeviceToHost, s), "read status"));
  NV_CHECK(check_cuda(cudaStreamSynchronize(s), "cudaStreamSynchronize"));
  if (word != 0) {
    NV_CHECK(check_cuda(cudaMemsetAsync(ws, 0, sizeof(word), s), "reset status"));
    NV_CHECK(check_cuda(cudaStreamSynchronize(s), "cudaStreamSynchronize"));
    return set_error(NVFP4_ERR_TIMEOUT, "a device-side wait gave up (status word %u)", word);
  }
  return NVFP4_OK;
}
