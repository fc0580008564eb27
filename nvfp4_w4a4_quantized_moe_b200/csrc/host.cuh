// Host-side plumbing shared by the entry points: error reporting, checks,
// tensor-map encoding and workspace carving.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdarg.h>
#include <stdint.h>
#include <stdio.h>

#include <utility>

#include "../../include/nvfp4_moe.h"

namespace nvfp4moe {

nvfp4_status set_error(nvfp4_status st, const char* fmt, ...);
nvfp4_status check_cuda(cudaError_t e, const char* what);
nvfp4_status check_launch(const char* what);
// Confirms the current device is sm_100 and returns its SM count.
nvfp4_status device_sm_count(int* sms);

inline cudaStream_t as_stream(void* s) { return reinterpret_cast<cudaStream_t>(s); }

// 2-D row-major tensor of bytes or bf16 for TMA: `inner` elements per row,
// `outer` rows, a row pitch of `pitch_bytes`, loaded in boxes of
// box_inner x box_outer with the 128-byte swizzle.
nvfp4_status make_tmap_2d(CUtensorMap* map, const void* base, CUtensorMapDataType dtype, uint64_t inner,
                          uint64_t outer, uint64_t pitch_bytes, uint32_t box_inner, uint32_t box_outer,
                          bool swizzle128 = true);

// Sequential carving of a workspace: every slice 256-byte aligned.
struct Carver {
  uint8_t* base;
  size_t used = 0;
  explicit Carver(void* b) : base(static_cast<uint8_t*>(b)) {}
  template <class T>
  T* take(size_t count) {
    used = (used + 255) & ~size_t(255);
    T* p = base ? reinterpret_cast<T*>(base + used) : nullptr;
    used += count * sizeof(T);
    return p;
  }
  size_t size() const { return (used + 255) & ~size_t(255); }
};

inline bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

// Launches `kernel` as a programmatic dependent of the stream's previous
// kernel: its blocks may start once every block of that kernel has signalled
// (griddepcontrol.launch_dependents), and the kernel itself waits for the
// previous one to finish (griddepcontrol.wait) before it touches memory that
// kernel wrote.  Every kernel launched this way calls griddep_wait() first.
template <typename... Params, typename... Args>
nvfp4_status launch_dependent(const char* what, void (*kernel)(Params...), dim3 grid, dim3 block, size_t smem,
                              cudaStream_t s, Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return check_cuda(cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...), what);
}

}  // namespace nvfp4moe

#define NV_CHECK(expr)                      \
  do {                                      \
    nvfp4_status _st = (expr);              \
    if (_st != NVFP4_OK) return _st;        \
  } while (0)

#define NV_REQUIRE(cond, code, ...)                                 \
  do {                                                              \
    if (!(cond)) return ::nvfp4moe::set_error(code, __VA_ARGS__);   \
  } while (0)
