// FP32 CUDA-core GEMM used by the inverse-factor and loss stages:
//   C = beta * C + alpha * op(A) * op(B)
// A row-major (M x K, lda), or with TRANS_A the transpose of a row-major
// (K x M) matrix; B row-major (K x N, ldb), or with TRANS_B the transpose of a
// row-major (N x K) matrix.  TRI_A: only the upper triangle of op(A) is used
// (entries below the diagonal are read as 0, whatever memory holds there), so
// a row tile's K loop starts at its first row.  TRI_B: only the upper triangle
// of op(B) is used, so a column tile's K loop ends at its last column.  UPPER_ONLY: tiles that lie entirely below the diagonal are
// skipped (the caller only reads C's upper triangle).  A nonzero *abort_flag
// (device) makes every CTA return at once; it carries an earlier failure.
#pragma once

#include "common.cuh"

namespace gptq {

constexpr int SG_BM = 128, SG_BN = 128, SG_BK = 8, SG_THREADS = 256;

template <bool TRANS_A, bool TRANS_B, bool TRI_A, bool TRI_B, bool UPPER_ONLY>
__global__ void __launch_bounds__(SG_THREADS)
sgemm_kernel(int M, int N, int K, float alpha, const float* __restrict__ A, int64_t lda,
             const float* __restrict__ B, int64_t ldb, float beta, float* __restrict__ C,
             int64_t ldc, const int32_t* __restrict__ abort_flag) {
  if (abort_flag != nullptr && *abort_flag != 0) return;
  const int bm = blockIdx.y, bn = blockIdx.x;
  if (UPPER_ONLY && bn < bm) return;
  const int m0 = bm * SG_BM, n0 = bn * SG_BN;
  __shared__ float sA[2][SG_BK][SG_BM + 4];
  __shared__ float sB[2][SG_BK][SG_BN + 4];
  const int tid = threadIdx.x;
  const int tx = tid % 16, ty = tid / 16;  // 16 x 16 threads, 8 x 8 outputs each

  float acc[8][8];
#pragma unroll
  for (int i = 0; i < 8; ++i)
#pragma unroll
    for (int j = 0; j < 8; ++j) acc[i][j] = 0.f;

  const int kbeg = TRI_A ? (m0 / SG_BK) * SG_BK : 0;
  const int kend = TRI_B ? min(K, n0 + SG_BN) : K;
  // A tile: 128 rows x 8 k; thread loads rows (tid/2) and k (tid%2)*4 .. +3
  const int a_row = tid / 2, a_k = (tid % 2) * 4;
  // B tile (no trans): 8 k x 128 n; thread loads k = tid/32, n = (tid%32)*4 .. +3
  // B tile (trans): element (kk, n) = B[n*ldb + kk]; thread loads n = tid/2, kk = (tid%2)*4..+3
  float ra[4], rb[4];

  auto load_tile = [&](int k0) {
    if (!TRANS_A) {
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        int gm = m0 + a_row, gk = k0 + a_k + q;
        bool ok = gm < M && gk < kend && (!TRI_A || gk >= gm);
        ra[q] = ok ? A[(int64_t)gm * lda + gk] : 0.f;
      }
    } else {
      // element (m, kk) = A[kk * lda + m]: thread loads kk = tid / 32, m = (tid % 32) * 4 .. +3
      int kk = tid / 32, mm = (tid % 32) * 4;
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        int gk = k0 + kk, gm = m0 + mm + q;
        bool ok = gk < kend && gm < M && (!TRI_A || gk >= gm);
        ra[q] = ok ? A[(int64_t)gk * lda + gm] : 0.f;
      }
    }
    if (!TRANS_B) {
      int kk = tid / 32, nn = (tid % 32) * 4;
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        int gk = k0 + kk, gn = n0 + nn + q;
        bool ok = gk < kend && gn < N && (!TRI_B || gk <= gn);
        rb[q] = ok ? B[(int64_t)gk * ldb + gn] : 0.f;
      }
    } else {
      int nn = tid / 2, kk = (tid % 2) * 4;
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        int gk = k0 + kk + q, gn = n0 + nn;
        bool ok = gk < kend && gn < N && (!TRI_B || gk <= gn);
        rb[q] = ok ? B[(int64_t)gn * ldb + gk] : 0.f;
      }
    }
  };
  auto store_tile = [&](int buf) {
    if (!TRANS_A) {
#pragma unroll
      for (int q = 0; q < 4; ++q) sA[buf][a_k + q][a_row] = ra[q];
    } else {
      int kk = tid / 32, mm = (tid % 32) * 4;
#pragma unroll
      for (int q = 0; q < 4; ++q) sA[buf][kk][mm + q] = ra[q];
    }
    if (!TRANS_B) {
      int kk = tid / 32, nn = (tid % 32) * 4;
#pragma unroll
      for (int q = 0; q < 4; ++q) sB[buf][kk][nn + q] = rb[q];
    } else {
      int nn = tid / 2, kk = (tid % 2) * 4;
#pragma unroll
      for (int q = 0; q < 4; ++q) sB[buf][kk + q][nn] = rb[q];
    }
  };

  int buf = 0;
  if (kbeg < kend) {
    load_tile(kbeg);
    store_tile(0);
  }
  __syncthreads();
  for (int k0 = kbeg; k0 < kend; k0 += SG_BK) {
    const bool more = k0 + SG_BK < kend;
    if (more) load_tile(k0 + SG_BK);
#pragma unroll
    for (int kk = 0; kk < SG_BK; ++kk) {
      float a[8], b[8];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        a[i] = sA[buf][kk][ty * 4 + i];
        a[i + 4] = sA[buf][kk][64 + ty * 4 + i];
        b[i] = sB[buf][kk][tx * 4 + i];
        b[i + 4] = sB[buf][kk][64 + tx * 4 + i];
      }
#pragma unroll
      for (int i = 0; i < 8; ++i)
#pragma unroll
        for (int j = 0; j < 8; ++j) acc[i][j] = fmaf(a[i], b[j], acc[i][j]);
    }
    if (more) store_tile(buf ^ 1);
    __syncthreads();
    buf ^= 1;
  }

#pragma unroll
  for (int i = 0; i < 8; ++i) {
    int gm = m0 + (i < 4 ? ty * 4 + i : 64 + ty * 4 + (i - 4));
    if (gm >= M) continue;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      int gn = n0 + (j < 4 ? tx * 4 + j : 64 + tx * 4 + (j - 4));
      if (gn >= N) continue;
      float* c = C + (int64_t)gm * ldc + gn;
      float v = alpha * acc[i][j];
      *c = (beta == 0.f) ? v : fmaf(beta, *c, v);
    }
  }
}

template <bool TRANS_A, bool TRANS_B, bool TRI_A, bool TRI_B, bool UPPER_ONLY>
inline void sgemm(int M, int N, int K, float alpha, const float* A, int64_t lda, const float* B,
                  int64_t ldb, float beta, float* C, int64_t ldc, const int32_t* abort_flag,
                  cudaStream_t s) {
  if (M <= 0 || N <= 0) return;
  dim3 grid((unsigned)cdiv(N, SG_BN), (unsigned)cdiv(M, SG_BM));
  sgemm_kernel<TRANS_A, TRANS_B, TRI_A, TRI_B, UPPER_ONLY>
      <<<grid, SG_THREADS, 0, s>>>(M, N, K, alpha, A, lda, B, ldb, beta, C, ldc, abort_flag);
}

}  // namespace gptq
