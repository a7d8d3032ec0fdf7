// Inverse-Hessian factor: dead columns, act-order, damping and the upper
// Cholesky factor of the inverse ([GPTQ-tool] "GPTQ" How it works Steps 4
// and 6, Optional refinements).
//
// U (upper, U^T U = Hp^-1) is computed without forming Hp^-1: factor
// Hp = V V^T with V upper triangular by a bottom-up ("backward") blocked
// Cholesky, then U = V^-1 (the inverse of an upper triangular matrix is upper
// and U^T U = V^-T V^-1 = (V V^T)^-1; uniqueness of the Cholesky factor makes
// this the factor the pages' three-call recipe produces).  fp32 throughout;
// ~2/3 k^3 + 1/3 k^3 flops instead of the recipe's ~4/3 k^3.
//
// Work matrix: U itself.  Stage order on the stream:
//   prep (diag, dead mask, damping lambda) -> rank (act-order) -> gather
//   (Hp + lambda I into U) -> for each block from the bottom: diagonal block
//   factor, panel solve, trailing update -> zero the lower triangle ->
//   for each block from the top: invert diagonal block, triangular multiply,
//   scale by the inverted diagonal block.
#include "common.cuh"
#include "sgemm.cuh"

namespace gptq {

constexpr int HV_B = 64;  // panel width

struct HinvScratch {
  double* sum_diag;  // [1]
  float* lambda;     // [1]
  float* diag;       // [k] diag(H) after the dead-column fix
  float* dinv;       // [HV_B * HV_B] inverse of the current diagonal block
  float* panel;      // [k * HV_B] triangular-multiply result
};

size_t hinv_workspace_bytes(int64_t k) {
  size_t b = 0;
  b += align256(sizeof(double));
  b += align256(sizeof(float));
  b += align256(sizeof(float) * (size_t)k);
  b += align256(sizeof(float) * HV_B * HV_B);
  b += align256(sizeof(float) * (size_t)k * HV_B);
  return b;
}

static HinvScratch carve(void* ws, int64_t k) {
  char* p = (char*)ws;
  HinvScratch s;
  s.sum_diag = (double*)p; p += align256(sizeof(double));
  s.lambda = (float*)p; p += align256(sizeof(float));
  s.diag = (float*)p; p += align256(sizeof(float) * (size_t)k);
  s.dinv = (float*)p; p += align256(sizeof(float) * HV_B * HV_B);
  s.panel = (float*)p;
  return s;
}

// diag, dead mask, lambda = percdamp * mean(diag after the dead fix).  One CTA.
__global__ void hinv_prep_kernel(const float* __restrict__ H, int k, float percdamp,
                                 uint8_t* __restrict__ dead, float* __restrict__ diag,
                                 double* __restrict__ sum_diag, float* __restrict__ lambda,
                                 int32_t* __restrict__ d_info) {
  __shared__ double red[1024 / kWarp];
  double acc = 0.0;
  for (int i = threadIdx.x; i < k; i += blockDim.x) {
    float d = H[(int64_t)i * k + i];
    bool is_dead = (d == 0.0f);
    dead[i] = is_dead ? 1 : 0;
    d = is_dead ? 1.0f : d;
    diag[i] = d;
    acc += (double)d;
  }
  for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x / 32] = acc;
  __syncthreads();
  if (threadIdx.x == 0) {
    double s = 0.0;
    for (int w = 0; w < (int)(blockDim.x / 32); ++w) s += red[w];
    *sum_diag = s;
    *lambda = (float)((double)percdamp * (s / (double)k));
    *d_info = 0;
  }
}

// Stable descending rank of diag: rank(i) = #{j : d_j > d_i} + #{j < i : d_j == d_i}.
__global__ void hinv_rank_kernel(const float* __restrict__ diag, int k, int act_order,
                                 int32_t* __restrict__ perm, int32_t* __restrict__ invperm) {
  __shared__ float sd[1024];
  // NaN keys sort last (as -inf) so the ranks always form a permutation; the
  // factorisation then reports the non-finite pivot through d_info.
  int i = blockIdx.x * blockDim.x + threadIdx.x;
  float di = (i < k) ? diag[i] : 0.f;
  di = isnan(di) ? -INFINITY : di;
  int rank = 0;
  if (!act_order) {
    rank = i;
  } else {
    for (int j0 = 0; j0 < k; j0 += 1024) {
      __syncthreads();
      for (int q = threadIdx.x; q < 1024; q += blockDim.x)
        sd[q] = (j0 + q < k) ? (isnan(diag[j0 + q]) ? -INFINITY : diag[j0 + q]) : 0.f;
      __syncthreads();
      int jn = min(1024, k - j0);
      for (int q = 0; q < jn; ++q) {
        float dj = sd[q];
        rank += (dj > di) || (dj == di && (j0 + q) < i);
      }
    }
  }
  if (i < k) {
    perm[rank] = i;
    invperm[i] = rank;
  }
}

// U[a][b] = H[perm[a]][perm[b]] for b >= a, with the diagonal replaced by
// diag (dead fix) + lambda.
__global__ void hinv_gather_kernel(const float* __restrict__ H, int k,
                                   const int32_t* __restrict__ perm,
                                   const float* __restrict__ diag,
                                   const float* __restrict__ lambda, float* __restrict__ U) {
  int a = blockIdx.y;
  int pa = perm[a];
  float lam = *lambda;
  for (int b = a + blockIdx.x * blockDim.x + threadIdx.x; b < k; b += gridDim.x * blockDim.x) {
    float v;
    if (b == a) {
      v = diag[pa] + lam;
    } else {
      v = H[(int64_t)pa * k + perm[b]];
    }
    U[(int64_t)a * k + b] = v;
  }
}

__device__ __forceinline__ void set_info(int32_t* d_info, int idx) {
  atomicCAS(d_info, 0, idx + 1);
}

// Bottom-up Cholesky of the diagonal block A[j0:j1, j0:j1] (upper part):
// for c = b-1 .. 0: d = sqrt(a_cc); V[i][c] = a_ic / d (i < c);
// a_ij -= V[i][c] V[j][c] (i <= j < c).  One CTA of 256 threads.
__global__ void chol_diag_kernel(float* __restrict__ A, int k, int j0, int b,
                                 int32_t* __restrict__ d_info) {
  if (*d_info != 0) return;
  __shared__ float S[HV_B][HV_B + 1];
  __shared__ int fail;
  for (int e = threadIdx.x; e < b * b; e += blockDim.x) {
    int i = e / b, j = e % b;
    S[i][j] = (j >= i) ? A[(int64_t)(j0 + i) * k + j0 + j] : 0.f;
  }
  if (threadIdx.x == 0) fail = -1;
  __syncthreads();
  for (int c = b - 1; c >= 0; --c) {
    if (threadIdx.x == 0) {
      float p = S[c][c];
      if (!(p > 0.f) || !isfinite(p)) {
        fail = c;
      } else {
        S[c][c] = sqrtf(p);
      }
    }
    __syncthreads();
    if (fail >= 0) break;
    float d = S[c][c];
    for (int i = threadIdx.x; i < c; i += blockDim.x) S[i][c] = S[i][c] / d;
    __syncthreads();
    for (int e = threadIdx.x; e < c * c; e += blockDim.x) {
      int i = e / c, j = e % c;
      if (i <= j) S[i][j] -= S[i][c] * S[j][c];
    }
    __syncthreads();
  }
  if (fail >= 0) {
    if (threadIdx.x == 0) set_info(d_info, j0 + fail);
    return;
  }
  for (int e = threadIdx.x; e < b * b; e += blockDim.x) {
    int i = e / b, j = e % b;
    if (j >= i) A[(int64_t)(j0 + i) * k + j0 + j] = S[i][j];
  }
}

// Panel: rows i in [0, j0): V[i][J] solves x V22^T = a with V22 = V[J][J]
// upper: x_c = (a_c - sum_{m > c} x_m V22[c][m]) / V22[c][c], c = b-1 .. 0.
template <int B>
__global__ void __launch_bounds__(128)
chol_panel_kernel(float* __restrict__ A, int k, int j0, const int32_t* __restrict__ d_info) {
  if (*d_info != 0) return;
  __shared__ float V22[B][B + 1];
  __shared__ float rdiag[B];
  for (int e = threadIdx.x; e < B * B; e += blockDim.x) {
    int i = e / B, j = e % B;
    V22[i][j] = (j >= i) ? A[(int64_t)(j0 + i) * k + j0 + j] : 0.f;
  }
  __syncthreads();
  for (int c = threadIdx.x; c < B; c += blockDim.x) rdiag[c] = 1.0f / V22[c][c];
  __syncthreads();
  int row = blockIdx.x * blockDim.x + threadIdx.x;
  if (row >= j0) return;
  float* a = A + (int64_t)row * k + j0;
  float x[B];
#pragma unroll
  for (int c = 0; c < B; ++c) x[c] = a[c];
#pragma unroll
  for (int c = B - 1; c >= 0; --c) {
    float v = x[c];
#pragma unroll
    for (int m = c + 1; m < B; ++m) v = fmaf(-x[m], V22[c][m], v);
    x[c] = v * rdiag[c];
  }
#pragma unroll
  for (int c = 0; c < B; ++c) a[c] = x[c];
}

// Generic-width panel (the short top block when k % HV_B != 0): same
// recurrence, runtime width b <= HV_B.
__global__ void __launch_bounds__(128)
chol_panel_small_kernel(float* __restrict__ A, int k, int j0, int b,
                        const int32_t* __restrict__ d_info) {
  if (*d_info != 0) return;
  __shared__ float V22[HV_B][HV_B + 1];
  for (int e = threadIdx.x; e < b * b; e += blockDim.x) {
    int i = e / b, j = e % b;
    V22[i][j] = (j >= i) ? A[(int64_t)(j0 + i) * k + j0 + j] : 0.f;
  }
  __syncthreads();
  int row = blockIdx.x * blockDim.x + threadIdx.x;
  if (row >= j0) return;
  float* a = A + (int64_t)row * k + j0;
  for (int c = b - 1; c >= 0; --c) {
    float v = a[c];
    for (int m = c + 1; m < b; ++m) v = fmaf(-a[m], V22[c][m], v);
    a[c] = v / V22[c][c];
  }
}

// Zero the strict lower triangle of U.
__global__ void zero_lower_kernel(float* __restrict__ U, int k, const int32_t* __restrict__ d_info) {
  if (*d_info != 0) return;
  int i = blockIdx.y;
  for (int j = blockIdx.x * blockDim.x + threadIdx.x; j < i; j += gridDim.x * blockDim.x)
    U[(int64_t)i * k + j] = 0.f;
}

// Inverse of the upper triangular diagonal block V[J][J] (b x b): thread c
// computes column c by back substitution; the result goes to dinv (b x b).
__global__ void tri_inv_diag_kernel(const float* __restrict__ A, int k, int j0, int b,
                                    float* __restrict__ dinv, const int32_t* __restrict__ d_info) {
  if (*d_info != 0) return;
  __shared__ float V[HV_B][HV_B + 1];
  __shared__ float Y[HV_B][HV_B + 1];
  for (int e = threadIdx.x; e < b * b; e += blockDim.x) {
    int i = e / b, j = e % b;
    V[i][j] = (j >= i) ? A[(int64_t)(j0 + i) * k + j0 + j] : 0.f;
    Y[i][j] = 0.f;
  }
  __syncthreads();
  int c = threadIdx.x;
  if (c < b) {
    Y[c][c] = 1.0f / V[c][c];
    for (int i = c - 1; i >= 0; --i) {
      float s = 0.f;
      for (int m = i + 1; m <= c; ++m) s = fmaf(V[i][m], Y[m][c], s);
      Y[i][c] = -s / V[i][i];
    }
  }
  __syncthreads();
  for (int e = threadIdx.x; e < b * b; e += blockDim.x) dinv[e] = Y[e / b][e % b];
}

// Write dinv into U[J][J] (upper part; lower part zero).
__global__ void put_diag_block_kernel(float* __restrict__ U, int k, int j0, int b,
                                      const float* __restrict__ dinv,
                                      const int32_t* __restrict__ d_info) {
  if (*d_info != 0) return;
  for (int e = threadIdx.x; e < b * b; e += blockDim.x) {
    int i = e / b, j = e % b;
    U[(int64_t)(j0 + i) * k + j0 + j] = (j >= i) ? dinv[e] : 0.f;
  }
}

gptq_status prepare_hinv_impl(const float* H, int64_t k64, const gptq_config* cfg, float* U,
                              int32_t* perm, int32_t* invperm, uint8_t* dead, int32_t* d_info,
                              void* ws, cudaStream_t s) {
  const int k = (int)k64;
  HinvScratch sc = carve(ws, k);
  hinv_prep_kernel<<<1, 1024, 0, s>>>(H, k, cfg->percdamp, dead, sc.diag, sc.sum_diag, sc.lambda,
                                      d_info);
  GPTQ_CHECK_LAUNCH();
  hinv_rank_kernel<<<(unsigned)cdiv(k, 256), 256, 0, s>>>(sc.diag, k, cfg->act_order, perm,
                                                          invperm);
  GPTQ_CHECK_LAUNCH();
  {
    dim3 grid((unsigned)cdiv(k, 1024), (unsigned)k);
    hinv_gather_kernel<<<grid, 256, 0, s>>>(H, k, perm, sc.diag, sc.lambda, U);
    GPTQ_CHECK_LAUNCH();
  }
  // bottom-up blocked Cholesky: blocks [j0, j1) from the bottom; the short
  // block (if any) is the top one.
  for (int j1 = k; j1 > 0; j1 -= HV_B) {
    int j0 = j1 > HV_B ? j1 - HV_B : 0;
    int b = j1 - j0;
    chol_diag_kernel<<<1, 256, 0, s>>>(U, k, j0, b, d_info);
    GPTQ_CHECK_LAUNCH();
    if (j0 == 0) break;
    if (b == HV_B) {
      chol_panel_kernel<HV_B><<<(unsigned)cdiv(j0, 128), 128, 0, s>>>(U, k, j0, d_info);
    } else {
      chol_panel_small_kernel<<<(unsigned)cdiv(j0, 128), 128, 0, s>>>(U, k, j0, b, d_info);
    }
    GPTQ_CHECK_LAUNCH();
    // A[0:j0, 0:j0] (upper) -= P P^T, P = A[0:j0, j0:j1]
    sgemm<true, false, true>(j0, j0, b, -1.0f, U + j0, k, U + j0, k, 1.0f, U, k, d_info, s);
    GPTQ_CHECK_LAUNCH();
  }
  {
    dim3 grid((unsigned)cdiv(k, 1024), (unsigned)k);
    zero_lower_kernel<<<grid, 256, 0, s>>>(U, k, d_info);
    GPTQ_CHECK_LAUNCH();
  }
  // in-place inverse of the upper triangular V, block columns left to right:
  // U[0:j0, J] = -U[0:j0, 0:j0] V[0:j0, J] V[J, J]^-1 ; U[J, J] = V[J, J]^-1.
  // Same block boundaries as the factorisation (short block first).
  int first = k % HV_B == 0 ? HV_B : k % HV_B;
  for (int j0 = 0; j0 < k;) {
    int b = (j0 == 0) ? first : HV_B;
    tri_inv_diag_kernel<<<1, 64, 0, s>>>(U, k, j0, b, sc.dinv, d_info);
    GPTQ_CHECK_LAUNCH();
    if (j0 > 0) {
      // panel = U[0:j0, 0:j0] (upper, inverted) * V[0:j0, J]
      sgemm<false, true, false>(j0, b, j0, 1.0f, U, k, U + j0, k, 0.0f, sc.panel, HV_B, d_info,
                                s);
      GPTQ_CHECK_LAUNCH();
      // U[0:j0, J] = -panel * dinv
      sgemm<false, false, false>(j0, b, b, -1.0f, sc.panel, HV_B, sc.dinv, b, 0.0f, U + j0, k,
                                 d_info, s);
      GPTQ_CHECK_LAUNCH();
    }
    put_diag_block_kernel<<<1, 256, 0, s>>>(U, k, j0, b, sc.dinv, d_info);
    GPTQ_CHECK_LAUNCH();
    j0 += b;
  }
  return GPTQ_OK;
}

}  // namespace gptq
