// Hessian accumulation on the CUDA cores (fp32 inputs; also the fallback-free
// reference path of the f16/bf16 inputs at sizes the tensor-core kernel does
// not take).  H += alpha * X^T X, [GPTQ-tool] "GPTQ" How it works Step 3.
//
// Tiles of 64 x 64 of the upper triangle, 256 threads with 4 x 4 outputs each,
// split over tokens (grid.z) so that each fp32 running sum covers at most
// HS_SPLIT_TOKENS tokens; the partial sums are added into H with atomics and a
// final pass mirrors the upper triangle into the lower one.
#include "common.cuh"

namespace gptq {

constexpr int HS_T = 64, HS_KT = 16, HS_THREADS = 256;
constexpr int HS_SPLIT_TOKENS = 2048;

__device__ __forceinline__ void tri_tile_decode(int id, int nt, int& ti, int& tj) {
  int t = 0;
  while (id >= nt - t) {
    id -= nt - t;
    ++t;
  }
  ti = t;
  tj = t + id;
}

template <typename T>
__global__ void __launch_bounds__(HS_THREADS)
hessian_simt_kernel(const T* __restrict__ X, int64_t n, int k, int64_t ldx, float alpha,
                    float* __restrict__ H, int nt, int64_t tok_per_split) {
  int ti, tj;
  tri_tile_decode(blockIdx.x, nt, ti, tj);
  const int i0 = ti * HS_T, j0 = tj * HS_T;
  const int64_t t_beg = (int64_t)blockIdx.y * tok_per_split;
  const int64_t t_end = min(n, t_beg + tok_per_split);
  __shared__ float sI[HS_KT][HS_T + 4];
  __shared__ float sJ[HS_KT][HS_T + 4];
  const int tid = threadIdx.x, tx = tid % 16, ty = tid / 16;
  float acc[4][4] = {};
  for (int64_t t0 = t_beg; t0 < t_end; t0 += HS_KT) {
    // 16 tokens x 64 columns for each operand: 1024 elements, 4 per thread
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      int e = tid + q * HS_THREADS;
      int tt = e / HS_T, cc = e % HS_T;
      int64_t gt = t0 + tt;
      float vi = 0.f, vj = 0.f;
      if (gt < t_end) {
        if (i0 + cc < k) vi = to_f32(X[gt * ldx + i0 + cc]);
        if (j0 + cc < k) vj = to_f32(X[gt * ldx + j0 + cc]);
      }
      sI[tt][cc] = vi;
      sJ[tt][cc] = vj;
    }
    __syncthreads();
#pragma unroll
    for (int tt = 0; tt < HS_KT; ++tt) {
      float a[4], b[4];
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        a[q] = sI[tt][ty * 4 + q];
        b[q] = sJ[tt][tx * 4 + q];
      }
#pragma unroll
      for (int p = 0; p < 4; ++p)
#pragma unroll
        for (int q = 0; q < 4; ++q) acc[p][q] = fmaf(a[p], b[q], acc[p][q]);
    }
    __syncthreads();
  }
#pragma unroll
  for (int p = 0; p < 4; ++p) {
    int gi = i0 + ty * 4 + p;
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      int gj = j0 + tx * 4 + q;
      if (gi < k && gj < k && gj >= gi) atomicAdd(&H[(int64_t)gi * k + gj], alpha * acc[p][q]);
    }
  }
}

// H[j][i] = H[i][j] for j > i.  A nonzero *poison_flag (a device-side wait
// of the tensor-core pass gave up) writes NaN into H[0][0] instead, so the
// Cholesky of the next stage reports the failure.
// Copies the upper triangle of H into the lower one.  status (may be NULL):
// the tensor-core kernel's workspace words; when its per-call flag status[0]
// is set (a bounded wait gave up), H[0][0] becomes NaN and the caller's
// status word status[1] GPTQ_ERR_TIMEOUT instead.
__global__ void mirror_upper_kernel(float* __restrict__ H, int k, int32_t* status) {
  __shared__ float tile[32][33];
  int bi = blockIdx.y, bj = blockIdx.x;
  if (status != nullptr && status[0] != 0) {
    if (bi == 0 && bj == 0 && threadIdx.x == 0 && threadIdx.y == 0) {
      H[0] = __int_as_float(0x7fc00000);
      status[1] = (int32_t)GPTQ_ERR_TIMEOUT;
    }
    return;
  }
  if (bj < bi) return;
  int tx = threadIdx.x, ty = threadIdx.y;  // 32 x 8
  for (int r = ty; r < 32; r += 8) {
    int gi = bi * 32 + r, gj = bj * 32 + tx;
    tile[r][tx] = (gi < k && gj < k) ? H[(int64_t)gi * k + gj] : 0.f;
  }
  __syncthreads();
  for (int r = ty; r < 32; r += 8) {
    int gi = bj * 32 + r, gj = bi * 32 + tx;  // lower element (gi, gj) = upper (gj, gi)
    if (gi < k && gj < k && gi > gj) H[(int64_t)gi * k + gj] = tile[tx][r];
  }
}

gptq_status hessian_simt(const void* X, gptq_dtype dt, int64_t n, int64_t k, int64_t ldx,
                         float alpha, float* H, cudaStream_t s) {
  int nt = (int)cdiv(k, HS_T);
  int64_t splits = cdiv(n, HS_SPLIT_TOKENS);
  if (splits > 65535) splits = 65535;
  int64_t per = cdiv(cdiv(n, splits), HS_KT) * HS_KT;
  splits = cdiv(n, per);
  dim3 grid((unsigned)(nt * (nt + 1) / 2), (unsigned)splits);
  switch (dt) {
    case GPTQ_F32:
      hessian_simt_kernel<float><<<grid, HS_THREADS, 0, s>>>((const float*)X, n, (int)k, ldx,
                                                             alpha, H, nt, per);
      break;
    case GPTQ_F16:
      hessian_simt_kernel<__half><<<grid, HS_THREADS, 0, s>>>((const __half*)X, n, (int)k, ldx,
                                                              alpha, H, nt, per);
      break;
    case GPTQ_BF16:
      hessian_simt_kernel<__nv_bfloat16><<<grid, HS_THREADS, 0, s>>>(
          (const __nv_bfloat16*)X, n, (int)k, ldx, alpha, H, nt, per);
      break;
  }
  GPTQ_CHECK_LAUNCH();
  int nb = (int)cdiv(k, 32);
  mirror_upper_kernel<<<dim3(nb, nb), dim3(32, 8), 0, s>>>(H, (int)k, nullptr);
  GPTQ_CHECK_LAUNCH();
  return GPTQ_OK;
}

}  // namespace gptq
