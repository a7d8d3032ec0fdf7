// Measured peak rates of the two arithmetic units the inverse factor and the
// sweep's updates run on, for their roofline fractions (the copy bandwidth and
// the dense bf16 rate come from elsewhere):
//   * fp32 FMA on the CUDA cores: every thread runs 8 independent chains of
//     packed fp32x2 FMAs (16 FMAs per iteration), one CTA of 256 threads per
//     scheduler-filling slot, 4 CTAs per SM;
//   * kind::tf32 MMAs on the tensor cores: one thread per SM issues M = 128,
//     N = 256, K = 8 MMAs back to back on one resident operand pair (zeroed
//     shared memory, K-major, 128-byte swizzle: the layout of the 3xTF32
//     update), accumulating into TMEM, and waits (bounded) for them.
// Each is timed with CUDA events around one launch after a warm-up launch.
// Nothing is allocated: the kernels' only outputs are two file-scope device
// words (a sink that keeps the FMA chains alive, and a timeout flag).
#include "common.cuh"
#include "tc_ptx.cuh"

namespace gptq {
namespace {

__device__ float g_pk_sink;
__device__ int32_t g_pk_status;

constexpr int PK_FMA_ITERS = 4096;
constexpr int PK_THREADS = 256;

__global__ void __launch_bounds__(PK_THREADS)
fp32_fma_rate_kernel(float a, float b) {
  float2 acc[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) acc[i] = make_float2(threadIdx.x * 1e-7f + i, (float)blockIdx.x);
  const float2 av = make_float2(a, a), bv = make_float2(b, b);
  for (int it = 0; it < PK_FMA_ITERS; ++it) {
#pragma unroll
    for (int i = 0; i < 8; ++i) acc[i] = __ffma2_rn(acc[i], av, bv);
  }
  float s = 0.f;
#pragma unroll
  for (int i = 0; i < 8; ++i) s += acc[i].x + acc[i].y;
  if (s == 12345.678f) g_pk_sink = s;  // keeps the chains alive
}

constexpr int PK_MMA_REPS = 2048;
constexpr int PK_A_BYTES = 128 * 32 * 4;   // 128 rows x 32 fp32, K-major swizzled
constexpr int PK_B_BYTES = 256 * 32 * 4;
// more than half an SM's shared memory: one CTA per SM
constexpr size_t PK_SMEM = 120 * 1024;

__global__ void __launch_bounds__(128, 1) tf32_mma_rate_kernel() {
  extern __shared__ uint8_t pk_raw[];
  uint8_t* smem = (uint8_t*)(((uintptr_t)pk_raw + 1023) & ~(uintptr_t)1023);
  uint64_t* done = (uint64_t*)(smem + PK_A_BYTES + PK_B_BYTES);
  uint32_t* tmem_slot = (uint32_t*)(done + 1);
  const int warp = threadIdx.x / 32;
  for (int e = threadIdx.x; e < (PK_A_BYTES + PK_B_BYTES) / 16; e += blockDim.x)
    reinterpret_cast<uint4*>(smem)[e] = make_uint4(0u, 0u, 0u, 0u);
  if (threadIdx.x == 0) {
    tc::mbar_init(done, 1);
    tc::fence_barrier_init();
  }
  tc::fence_proxy_async_smem();  // the MMAs (async proxy) read the zeroed operands
  if (warp == 1) tc::tmem_alloc(tmem_slot, 256);
  tc::tc_fence_before();
  __syncthreads();
  tc::tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  if (threadIdx.x == 0) {
    const uint32_t idesc = tc::instr_desc(2, 128, 256, 0, 0);
    const uint32_t sa = tc::smem_u32(smem), sb = sa + PK_A_BYTES;
    for (int r = 0; r < PK_MMA_REPS; ++r) {
#pragma unroll
      for (int kk = 0; kk < 4; ++kk) {
        const uint64_t da = tc::smem_desc_sw128(sa + kk * 32, 16, 1024);
        const uint64_t db = tc::smem_desc_sw128(sb + kk * 32, 16, 1024);
        tc::mma_tf32_ss(tmem, da, db, idesc, (r > 0 || kk > 0) ? 1u : 0u);
      }
    }
    tc::mma_commit(done);
    bool ok = false;
    for (uint32_t i = 0; i < tc::kSpinLimit && !ok; ++i) ok = tc::mbar_try_wait(done, 0);
    if (!ok) atomicExch(&g_pk_status, 1);
  }
  tc::tc_fence_before();
  __syncthreads();
  tc::tc_fence_after();
  if (warp == 1) tc::tmem_dealloc(tmem, 256);
}

float time_ms(cudaEvent_t e0, cudaEvent_t e1) {
  // (events of the legacy default stream, around one launch)
  float ms = 0.f;
  cudaEventElapsedTime(&ms, e0, e1);
  return ms;
}

}  // namespace
}  // namespace gptq

using namespace gptq;

extern "C" gptq_status gptq_measure_peaks(double* fp32_tflops, double* tf32_tflops) {
  if (fp32_tflops == nullptr || tf32_tflops == nullptr) return GPTQ_ERR_INVALID_ARG;
  const int nsm = sm_count();
  gptq_status st = GPTQ_OK;
  const int32_t zero = 0;
  if (cudaMemcpyToSymbol(g_pk_status, &zero, sizeof(zero)) != cudaSuccess) return GPTQ_ERR_CUDA;
  if (smem_optin((const void*)tf32_mma_rate_kernel, PK_SMEM) != cudaSuccess) return GPTQ_ERR_CUDA;
  cudaEvent_t e0, e1;
  if (cudaEventCreate(&e0) != cudaSuccess) return GPTQ_ERR_CUDA;
  if (cudaEventCreate(&e1) != cudaSuccess) {
    cudaEventDestroy(e0);
    return GPTQ_ERR_CUDA;
  }
  for (int rep = 0; rep < 2 && st == GPTQ_OK; ++rep) {  // a warm-up launch, then the timed one
    cudaEventRecord(e0);
    fp32_fma_rate_kernel<<<4 * nsm, PK_THREADS>>>(0.999f, 1e-3f);
    cudaEventRecord(e1);
    if (cudaEventSynchronize(e1) != cudaSuccess) st = GPTQ_ERR_CUDA;
    const double flop = 2.0 * 16.0 * PK_FMA_ITERS * PK_THREADS * 4.0 * nsm;
    *fp32_tflops = flop / (time_ms(e0, e1) * 1e-3) / 1e12;
  }
  for (int rep = 0; rep < 2 && st == GPTQ_OK; ++rep) {
    cudaEventRecord(e0);
    tf32_mma_rate_kernel<<<nsm, 128, PK_SMEM>>>();
    cudaEventRecord(e1);
    if (cudaEventSynchronize(e1) != cudaSuccess) st = GPTQ_ERR_CUDA;
    const double flop = 2.0 * 128.0 * 256.0 * 8.0 * 4.0 * PK_MMA_REPS * nsm;
    *tf32_tflops = flop / (time_ms(e0, e1) * 1e-3) / 1e12;
  }
  int32_t h = 0;
  if (st == GPTQ_OK && cudaMemcpyFromSymbol(&h, g_pk_status, sizeof(h)) == cudaSuccess && h != 0)
    st = GPTQ_ERR_TIMEOUT;
  cudaEventDestroy(e0);
  cudaEventDestroy(e1);
  return st;
}
