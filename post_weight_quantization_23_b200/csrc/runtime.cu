// Process-wide runtime state of libgptq_b200, kept thread-safe and per device:
//   * the driver's tensor-map encoder (one entry point for the process);
//   * each kernel's dynamic shared-memory opt-in, which CUDA records per
//     function and per device context -- so it is tracked per (device,
//     kernel), under a lock, and a failed opt-in is reported, not cached;
//   * the number of polls after which a pipeline wait inside a tensor-core
//     kernel gives up (gptq_set_wait_limit), read at each launch.
#include <atomic>
#include <map>
#include <mutex>
#include <utility>

#include "common.cuh"
#include "tc_ptx.cuh"

namespace gptq {

EncodeTiledFn tensormap_encoder() {
  static const EncodeTiledFn fn = []() -> EncodeTiledFn {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      return (EncodeTiledFn)p;
    return nullptr;
  }();
  return fn;
}

namespace {
std::mutex g_optin_mu;
std::map<std::pair<int, const void*>, size_t> g_optin;  // (device, kernel) -> bytes opted in
std::atomic<uint32_t> g_wait_limit{tc::kSpinLimit};
}  // namespace

cudaError_t smem_optin(const void* func, size_t bytes) {
  if (bytes <= 48 * 1024) return cudaSuccess;  // the default limit needs no opt-in
  int dev = -1;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  std::lock_guard<std::mutex> lock(g_optin_mu);
  size_t& have = g_optin[std::make_pair(dev, func)];
  if (have >= bytes) return cudaSuccess;
  e = cudaFuncSetAttribute(func, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
  if (e == cudaSuccess) have = bytes;
  return e;
}

int sm_count() {
  int dev = 0, nsm = 0;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || nsm <= 0)
    return 148;
  return nsm;
}

uint32_t wait_limit() { return g_wait_limit.load(std::memory_order_relaxed); }

}  // namespace gptq

extern "C" void gptq_set_wait_limit(uint32_t polls) {
  gptq::g_wait_limit.store(polls == 0xFFFFFFFFu ? gptq::tc::kSpinLimit : polls,
                           std::memory_order_relaxed);
}
