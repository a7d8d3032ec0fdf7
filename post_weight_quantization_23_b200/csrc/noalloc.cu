// gptq_prepare_hinv_noalloc: the inverse-Hessian factor for callers that
// cannot allocate device memory.
//
// Some callers of this library cannot call cudaMalloc or hand over a
// workspace: a plugin whose host framework passes it only its input and
// output buffers, a process that has carved all device memory into its own
// arena up front (so a new allocation would fail or fragment it), or a
// runtime that forbids allocation after start-up.  This entry point runs the
// same computation as gptq_prepare_hinv, but its scratch lives in a file-scope
// __device__ array that the CUDA runtime creates when the library's device
// code is loaded, so the call itself allocates nothing.
//
// The array is `kScratchBytes` (4 MiB) on every device that loads the
// library and is held until the process exits; it covers k up to
// kNoAllocMaxK = 12288.  Up to k = 4076 the tensor-core rank updates' operand
// splits for one 64-column block fit beside the rest (one-level updates, where
// gptq_prepare_hinv batches 8 blocks); above, the fp32 CUDA-core rank update
// runs instead (slower).  Either way U equals gptq_prepare_hinv's within fp32
// rounding.  All calls share it and it keeps the previous call's
// contents; the Cholesky stages write every scratch word before reading it,
// so nothing needs clearing.  Calls whose work overlaps on the GPU (two
// streams, or two host threads) race on the array: serialise them.
//
// Host code cannot pass the array's name to a kernel (on the host it is only
// a stand-in for the device symbol).  The device address comes from
// cudaGetSymbolAddress with the device current, on every call made outside
// stream capture (so a device reset or a context re-created since the last
// call gets the fresh address); a call made while its stream is capturing
// reuses the address of the last call on that device, so the first call on a
// device must come before any capture.
#include <mutex>

#include "common.cuh"

namespace gptq {
size_t hinv_workspace_min_bytes(int64_t k);
gptq_status prepare_hinv_impl(const float* H, int64_t k, const gptq_config* cfg, float* U,
                              int32_t* perm, int32_t* invperm, uint8_t* dead, int32_t* d_info,
                              void* ws, size_t ws_bytes, cudaStream_t s);
}  // namespace gptq

namespace {

constexpr int64_t kNoAllocMaxK = 12288;
constexpr size_t kScratchBytes = (size_t)4 << 20;

__device__ __align__(256) unsigned char g_hinv_scratch[kScratchBytes];

constexpr int kMaxDevices = 128;
void* g_scratch_addr[kMaxDevices] = {};
std::mutex g_scratch_mu;

gptq_status scratch_address(cudaStream_t stream, void** out) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) return GPTQ_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return GPTQ_ERR_UNSUPPORTED;
  cudaStreamCaptureStatus cap = cudaStreamCaptureStatusNone;
  if (cudaStreamIsCapturing(stream, &cap) != cudaSuccess) return GPTQ_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  if (cap == cudaStreamCaptureStatusNone) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_hinv_scratch) != cudaSuccess || p == nullptr)
      return GPTQ_ERR_CUDA;
    g_scratch_addr[dev] = p;
  } else if (g_scratch_addr[dev] == nullptr) {
    return GPTQ_ERR_CUDA;  // first call on this device inside a capture
  }
  *out = g_scratch_addr[dev];
  return GPTQ_OK;
}

}  // namespace

extern "C" gptq_status gptq_prepare_hinv_noalloc(const float* H, int64_t k,
                                                 const gptq_config* cfg, float* U,
                                                 int32_t* perm, int32_t* invperm, uint8_t* dead,
                                                 int32_t* d_info, gptq_stream_t stream) {
  if (k <= 0) return GPTQ_ERR_INVALID_ARG;
  if (H == nullptr || U == nullptr || perm == nullptr || invperm == nullptr || dead == nullptr ||
      d_info == nullptr || cfg == nullptr)
    return GPTQ_ERR_INVALID_ARG;
  if (!(cfg->percdamp >= 0.0f) || !isfinite(cfg->percdamp)) return GPTQ_ERR_INVALID_ARG;
  if ((const void*)H == (const void*)U) return GPTQ_ERR_INVALID_ARG;
  // sizes beyond the built-in scratch
  if (k > kNoAllocMaxK || gptq::hinv_workspace_min_bytes(k) > kScratchBytes) return GPTQ_ERR_WORKSPACE;
  void* ws = nullptr;
  gptq_status st = scratch_address((cudaStream_t)stream, &ws);
  if (st != GPTQ_OK) return st;
  return gptq::prepare_hinv_impl(H, k, cfg, U, perm, invperm, dead, d_info, ws, kScratchBytes,
                                 (cudaStream_t)stream);
}
