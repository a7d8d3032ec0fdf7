// Shared device helpers for libgptq_b200 (sm_100a).
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <cuda_fp16.h>
#include <cuda_bf16.h>
#include <stdint.h>

#include "../../include/gptq.h"

#define GPTQ_CHECK_LAUNCH()                              \
  do {                                                   \
    cudaError_t e_ = cudaPeekAtLastError();              \
    if (e_ != cudaSuccess) return GPTQ_ERR_CUDA;         \
  } while (0)

namespace gptq {

constexpr int kWarp = 32;

// Programmatic dependent launch.  A kernel launched with launch_pdl may start
// while the kernel before it in the stream is still running: it must call
// pdl_wait() before touching anything an earlier kernel wrote (the wait
// returns once the previous grid has completed and its memory is visible),
// and it calls pdl_trigger() to let the next kernel start early in turn.
// Both are no-ops in a kernel launched the ordinary way.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_trigger() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

template <typename... KArgs, typename... Args>
inline cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                              cudaStream_t s, Args... args) {
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
  return cudaLaunchKernelEx(&cfg, kernel, static_cast<KArgs>(args)...);
}

// Process-wide runtime helpers (runtime.cu); all thread-safe.
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
// The driver's cuTensorMapEncodeTiled, or nullptr when the driver lacks it.
EncodeTiledFn tensormap_encoder();
// Opt the kernel `func` into `bytes` of dynamic shared memory on the current
// device (once per device and size; the error of a failed opt-in is returned).
cudaError_t smem_optin(const void* func, size_t bytes);
// SM count of the current device.
int sm_count();
// Polls after which a pipeline wait of a tensor-core kernel gives up
// (gptq_set_wait_limit); passed to each kernel at launch.
uint32_t wait_limit();

__host__ __device__ inline int64_t cdiv(int64_t a, int64_t b) { return (a + b - 1) / b; }
__host__ __device__ inline size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

template <typename T> __device__ __forceinline__ float to_f32(T v);
template <> __device__ __forceinline__ float to_f32<float>(float v) { return v; }
template <> __device__ __forceinline__ float to_f32<__half>(__half v) { return __half2float(v); }
template <> __device__ __forceinline__ float to_f32<__nv_bfloat16>(__nv_bfloat16 v) {
  return __bfloat162float(v);
}

// The quantization decision of the grid: c = clamp(rint(w / scale) + zero, 0, maxq),
// with an IEEE fp32 division and round-half-to-even, as the fp32 reference does.
__device__ __forceinline__ float quant_code(float w, float scale, float zero, float maxq) {
  float c = rintf(__fdiv_rn(w, scale)) + zero;
  return fminf(fmaxf(c, 0.0f), maxq);
}

// Grid parameters of one group from its min and max, lo = min(0, min),
// hi = max(0, max):
//   asymmetric: scale = max(hi - lo, 1e-8) / maxq, zero = rint(-lo / scale);
//   symmetric:  a = max(-lo, hi), scale = max(2a, 1e-8) / maxq,
//               zero = (maxq + 1) / 2 (the grid's middle code).
__device__ __forceinline__ void grid_from_range(float mn, float mx, float maxq, float& scale,
                                                float& zero, bool sym = false) {
  float lo = fminf(mn, 0.0f), hi = fmaxf(mx, 0.0f);
  if (sym) {
    const float a = fmaxf(-lo, hi);
    scale = __fdiv_rn(fmaxf(__fadd_rn(a, a), 1e-8f), maxq);
    zero = (maxq + 1.0f) * 0.5f;
    return;
  }
  scale = __fdiv_rn(fmaxf(__fsub_rn(hi, lo), 1e-8f), maxq);
  zero = rintf(__fdiv_rn(-lo, scale));
}

}  // namespace gptq
