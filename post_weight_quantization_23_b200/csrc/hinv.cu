// Inverse-Hessian factor: dead columns, act-order, damping and the upper
// Cholesky factor of the inverse ([GPTQ-tool] "GPTQ" How it works Steps 4
// and 6, Optional refinements).
//
// U (upper, U^T U = Hp^-1) is computed without forming Hp^-1.  Factor
// Hp = L^T L with L lower triangular (a Cholesky that starts from the last
// index); then V = L^T is upper with Hp = V V^T, and U = V^-1 is the upper
// triangular matrix with U^T U = V^-T V^-1 = Hp^-1 -- by uniqueness of the
// Cholesky factor, the factor the pages' three-call recipe produces, for
// about half its flops.  fp32 throughout.
//
// One k x k work matrix (the output U) holds both factors: L grows in the
// LOWER triangle while U is built in the UPPER one, so the inverse never
// reads what it writes.
// Factor, blocks of HV_B = 64 indices from the last one up, step J = [j0, j1):
//   K1 diag    L_JJ from the Schur-updated diagonal block (lower part) and
//              U_JJ = (L_JJ^T)^-1, written to A[J, J] (upper) and the scratch.
//   K2 panel   L[J, 0:j0] = U_JJ * Hp[J, 0:j0]   (in place, lower part).
//   K3 update  A[0:j0, 0:j0] (lower) -= L[J, 0:j0]^T L[J, 0:j0].
// Inverse, recursively over halves of the block range (leaves = the U_JJ):
//   with V = [[V11, V12], [0, V22]], U12 = -U11 V12 U22 and V12 = L21^T:
//   S = U11 * L21^T into the free upper-right block, then U12 = -S * U22 in
//   place (row by row, columns right to left).
// A final pass zeroes the strict lower triangle.
#include "common.cuh"
#include "sgemm.cuh"

namespace gptq {

constexpr int HV_B = 64;  // block width

struct HinvScratch {
  double* sum_diag;  // [1]
  float* lambda;     // [1]
  float* diag;       // [k] diag(H) after the dead-column fix
  float* ujj;        // [HV_B * HV_B] U_JJ of the current step
};

size_t hinv_workspace_bytes(int64_t k) {
  size_t b = 0;
  b += align256(sizeof(double));
  b += align256(sizeof(float));
  b += align256(sizeof(float) * (size_t)k);
  b += align256(sizeof(float) * HV_B * HV_B);
  return b;
}

static HinvScratch carve(void* ws, int64_t k) {
  char* p = (char*)ws;
  HinvScratch s;
  s.sum_diag = (double*)p; p += align256(sizeof(double));
  s.lambda = (float*)p; p += align256(sizeof(float));
  s.diag = (float*)p; p += align256(sizeof(float) * (size_t)k);
  s.ujj = (float*)p;
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
// NaN keys sort last (as -inf) so the ranks always form a permutation; the
// factorisation then reports the non-finite pivot through d_info.
__global__ void hinv_rank_kernel(const float* __restrict__ diag, int k, int act_order,
                                 int32_t* __restrict__ perm, int32_t* __restrict__ invperm) {
  __shared__ float sd[1024];
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

// A[a][b] = H[perm[a]][perm[b]] for b <= a (lower part), the diagonal replaced
// by diag (dead fix) + lambda.
__global__ void hinv_gather_lower_kernel(const float* __restrict__ H, int k,
                                         const int32_t* __restrict__ perm,
                                         const float* __restrict__ diag,
                                         const float* __restrict__ lambda, float* __restrict__ A) {
  int a = blockIdx.y;
  int pa = perm[a];
  float lam = *lambda;
  const float* hrow = H + (int64_t)pa * k;
  for (int b = blockIdx.x * blockDim.x + threadIdx.x; b <= a; b += gridDim.x * blockDim.x) {
    float v = (b == a) ? diag[pa] + lam : hrow[perm[b]];
    A[(int64_t)a * k + b] = v;
  }
}

__device__ __forceinline__ void set_info(int32_t* d_info, int idx) { atomicCAS(d_info, 0, idx + 1); }

// K1: factor the diagonal block (lower storage, A_JJ = L^T L with L lower)
// and invert V = L^T: U_JJ = V^-1 (upper), written to the scratch and to the
// upper part of A[J, J] (the block was read into shared memory first).  One
// CTA of 256 threads.
//   factor, c = b-1 .. 0:  a_ij -= a_ci a_cj / a_cc  (j <= i < c), then
//   L_cj = a_cj / sqrt(a_cc) (j < c), L_cc = sqrt(a_cc);
//   inverse, i = b-1 .. 0: U_ii = 1 / V_ii, U_ic = -(sum_{m=i+1..c} V_im U_mc) / V_ii,
//   with V_im = L_mi.
__global__ void __launch_bounds__(256)
chol_inv_diag_kernel(float* __restrict__ A, int k, int j0, int b,
                     float* __restrict__ ujj, int32_t* __restrict__ d_info) {
  if (*d_info != 0) return;
  __shared__ float S[HV_B][HV_B + 1];
  __shared__ float Y[HV_B][HV_B + 1];
  __shared__ float dg[HV_B];
  const int t = threadIdx.x;
  for (int e = t; e < HV_B * HV_B; e += 256) {
    int i = e / HV_B, j = e % HV_B;
    S[i][j] = (i < b && j <= i) ? A[(int64_t)(j0 + i) * k + j0 + j] : 0.f;
    Y[i][j] = 0.f;
  }
  __syncthreads();
  const int ri = t >> 2, jq = t & 3;  // row ri, columns jq, jq+4, ...
  int fail = -1;
  for (int c = b - 1; c >= 0; --c) {
    const float p = S[c][c];
    if (!(p > 0.f) || !isfinite(p)) {
      fail = c;  // every thread reads the same pivot: the exit is uniform
      break;
    }
    if (ri < c) {
      const float f = S[c][ri] / p;
#pragma unroll
      for (int q = 0; q < HV_B / 4; ++q) {
        const int j = jq + 4 * q;
        if (j <= ri) S[ri][j] = fmaf(-f, S[c][j], S[ri][j]);
      }
    }
    __syncthreads();
  }
  if (fail >= 0) {
    if (t == 0) set_info(d_info, j0 + fail);
    return;
  }
  if (t < b) dg[t] = sqrtf(S[t][t]);
  __syncthreads();
  // scale to L: L_ij = a_ij / sqrt(a_ii) below the diagonal, L_ii = sqrt(a_ii)
  if (ri < b) {
    const float rd = 1.0f / dg[ri];
#pragma unroll
    for (int q = 0; q < HV_B / 4; ++q) {
      const int j = jq + 4 * q;
      if (j < ri) S[ri][j] *= rd;
    }
  }
  __syncthreads();
  if (t < b) S[t][t] = dg[t];
  __syncthreads();
  // inverse of V = L^T, rows from the bottom; thread (c = t / 4, part = t % 4)
  const int c = t >> 2, part = t & 3;
  for (int i = b - 1; i >= 0; --i) {
    float s = 0.f;
    if (c > i && c < b)
      for (int m = i + 1 + part; m <= c; m += 4) s = fmaf(S[m][i], Y[m][c], s);
    s += __shfl_xor_sync(0xffffffffu, s, 1);
    s += __shfl_xor_sync(0xffffffffu, s, 2);
    if (part == 0 && c < b) {
      const float rv = 1.0f / S[i][i];
      if (c == i) Y[i][i] = rv;
      else if (c > i) Y[i][c] = -s * rv;
    }
    __syncthreads();
  }
  for (int e = t; e < HV_B * HV_B; e += 256) {
    const int i = e / HV_B, j = e % HV_B;
    const float y = Y[i][j];
    ujj[e] = y;
    if (i < b && j < b && j >= i) A[(int64_t)(j0 + i) * k + j0 + j] = y;
  }
}

// K2: L[J, c] = U_JJ * A[J, c] for columns c in [c0, c0 + 64) of [0, j0), in
// place.  Thread (r = t / 4, cq = t % 4) computes row r, columns cq + 4q.
__global__ void __launch_bounds__(256)
chol_panel_kernel(float* __restrict__ A, int k, int j0, int b, const float* __restrict__ ujj,
                  const int32_t* __restrict__ d_info) {
  if (*d_info != 0) return;
  __shared__ float Us[HV_B][HV_B + 1];
  __shared__ float Hs[HV_B][HV_B + 1];
  const int t = threadIdx.x;
  const int c0 = blockIdx.x * HV_B;
  for (int e = t; e < HV_B * HV_B; e += 256) {
    int i = e / HV_B, j = e % HV_B;
    Us[i][j] = ujj[e];
    Hs[i][j] = (i < b && c0 + j < j0) ? A[(int64_t)(j0 + i) * k + c0 + j] : 0.f;
  }
  __syncthreads();
  const int r = t >> 2, cq = t & 3;
  if (r >= b) return;
  float acc[HV_B / 4];
#pragma unroll
  for (int q = 0; q < HV_B / 4; ++q) acc[q] = 0.f;
  for (int m = r; m < b; ++m) {
    const float u = Us[r][m];
#pragma unroll
    for (int q = 0; q < HV_B / 4; ++q) acc[q] = fmaf(u, Hs[m][cq + 4 * q], acc[q]);
  }
#pragma unroll
  for (int q = 0; q < HV_B / 4; ++q) {
    const int cc = c0 + cq + 4 * q;
    if (cc < j0) A[(int64_t)(j0 + r) * k + cc] = acc[q];
  }
}

// K3: A[0:n, 0:n] (lower) -= P^T P with P = A[j0:j0+b, 0:n] (b x n): 128 x 128
// tiles on or below the diagonal, 256 threads with 8 x 8 outputs.
__global__ void __launch_bounds__(256)
syrk_lower_tn_kernel(float* __restrict__ A, int k, int n, int j0, int b,
                     const int32_t* __restrict__ d_info) {
  if (*d_info != 0) return;
  const int bi = blockIdx.y, bj = blockIdx.x;
  if (bj > bi) return;
  const int i0 = bi * 128, jj0 = bj * 128;
  __shared__ float Pi[16][128 + 4];
  __shared__ float Pj[16][128 + 4];
  const int t = threadIdx.x, tx = t % 16, ty = t / 16;
  float acc[8][8];
#pragma unroll
  for (int p = 0; p < 8; ++p)
#pragma unroll
    for (int q = 0; q < 8; ++q) acc[p][q] = 0.f;
  for (int m0 = 0; m0 < b; m0 += 16) {
    for (int e = t; e < 16 * 128; e += 256) {
      int mm = e / 128, cc = e % 128;
      const float* prow = A + (int64_t)(j0 + m0 + mm) * k;
      bool okm = m0 + mm < b;
      Pi[mm][cc] = (okm && i0 + cc < n) ? prow[i0 + cc] : 0.f;
      Pj[mm][cc] = (okm && jj0 + cc < n) ? prow[jj0 + cc] : 0.f;
    }
    __syncthreads();
#pragma unroll
    for (int mm = 0; mm < 16; ++mm) {
      float a[8], bb[8];
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        a[q] = Pi[mm][ty * 4 + q];
        a[q + 4] = Pi[mm][64 + ty * 4 + q];
        bb[q] = Pj[mm][tx * 4 + q];
        bb[q + 4] = Pj[mm][64 + tx * 4 + q];
      }
#pragma unroll
      for (int p = 0; p < 8; ++p)
#pragma unroll
        for (int q = 0; q < 8; ++q) acc[p][q] = fmaf(a[p], bb[q], acc[p][q]);
    }
    __syncthreads();
  }
#pragma unroll
  for (int p = 0; p < 8; ++p) {
    const int gi = i0 + (p < 4 ? ty * 4 + p : 64 + ty * 4 + p - 4);
    if (gi >= n) continue;
#pragma unroll
    for (int q = 0; q < 8; ++q) {
      const int gj = jj0 + (q < 4 ? tx * 4 + q : 64 + tx * 4 + q - 4);
      if (gj <= gi && gj < n) A[(int64_t)gi * k + gj] -= acc[p][q];
    }
  }
}

// C[0:M, 0:N] := alpha * C * Uu, Uu (N x N) upper triangular, in place.
// Row a of the result needs only row a of C, and column c needs C[a][0..c]:
// each CTA owns TM rows and walks column tiles from right to left, so the
// entries it still has to read are never overwritten.  256 threads: thread
// (ty = t / 64, tx = t % 64) owns rows 4ty..4ty+3 of the tile, column tx.
constexpr int TR_TM = 16, TR_TN = 64, TR_KC = 32;
__global__ void __launch_bounds__(256)
trmm_right_upper_inplace_kernel(float* __restrict__ C, int64_t ldc, int M, int N,
                                const float* __restrict__ Uu, int64_t ldu, float alpha,
                                const int32_t* __restrict__ d_info) {
  if (*d_info != 0) return;
  __shared__ float Cs[TR_TM][TR_KC + 1];
  __shared__ float Us[TR_KC][TR_TN + 4];
  const int t = threadIdx.x, ty = t >> 6, tx = t & 63;
  const int a0 = blockIdx.x * TR_TM;
  if (a0 >= M) return;
  const int ntiles = (N + TR_TN - 1) / TR_TN;
  for (int tile = ntiles - 1; tile >= 0; --tile) {
    const int c0 = tile * TR_TN;
    const int kend = min(N, c0 + TR_TN);
    float acc[4] = {0.f, 0.f, 0.f, 0.f};
    for (int m0 = 0; m0 < kend; m0 += TR_KC) {
      for (int q = t; q < TR_TM * TR_KC; q += 256) {
        const int aa = q / TR_KC, mm = q % TR_KC;
        const int gr = a0 + aa, gm = m0 + mm;
        Cs[aa][mm] = (gr < M && gm < kend) ? C[(int64_t)gr * ldc + gm] : 0.f;
      }
      for (int q = t; q < TR_KC * TR_TN; q += 256) {
        const int mm = q / TR_TN, cc = q % TR_TN;
        const int gm = m0 + mm, gc = c0 + cc;
        Us[mm][cc] = (gm < kend && gc < N && gm <= gc) ? Uu[(int64_t)gm * ldu + gc] : 0.f;
      }
      __syncthreads();
#pragma unroll 8
      for (int mm = 0; mm < TR_KC; ++mm) {
        const float u = Us[mm][tx];
#pragma unroll
        for (int p = 0; p < 4; ++p) acc[p] = fmaf(Cs[4 * ty + p][mm], u, acc[p]);
      }
      __syncthreads();
    }
    const int gc = c0 + tx;
    if (gc < N) {
#pragma unroll
      for (int p = 0; p < 4; ++p) {
        const int gr = a0 + 4 * ty + p;
        if (gr < M) C[(int64_t)gr * ldc + gc] = alpha * acc[p];
      }
    }
    __syncthreads();
  }
}

// Zero the strict lower triangle of U.
__global__ void zero_lower_kernel(float* __restrict__ U, int k, const int32_t* __restrict__ d_info) {
  if (*d_info != 0) return;
  int i = blockIdx.y;
  for (int j = blockIdx.x * blockDim.x + threadIdx.x; j < i; j += gridDim.x * blockDim.x)
    U[(int64_t)i * k + j] = 0.f;
}

// Start of block `blk` when blocks of HV_B are laid from the bottom (the
// short block, if any, is block 0 at the top).
static int block_start(int k, int blk) {
  const int nb = (int)cdiv(k, HV_B);
  return std::max(0, k - (nb - blk) * HV_B);
}

// Upper inverse of the blocks [lo, hi): both halves first, then the coupling
// block U12 = -U11 * L21^T * U22.
static gptq_status trtri_range(float* A, int k, int lo, int hi, const int32_t* d_info,
                               cudaStream_t s) {
  if (hi - lo <= 1) return GPTQ_OK;  // leaf: U_JJ written by the diagonal kernel
  const int mid = (lo + hi) / 2;
  gptq_status st = trtri_range(A, k, lo, mid, d_info, s);
  if (st != GPTQ_OK) return st;
  st = trtri_range(A, k, mid, hi, d_info, s);
  if (st != GPTQ_OK) return st;
  const int r1 = block_start(k, lo), r2 = block_start(k, mid);
  const int e = (hi == (int)cdiv(k, HV_B)) ? k : block_start(k, hi);
  const int k1 = r2 - r1, k2 = e - r2;
  // S = U11 * L21^T  (U11 upper; L21 = A[r2:e, r1:r2]) into A[r1:r2, r2:e]
  sgemm<false, true, true, false, false>(k1, k2, k1, 1.0f, A + (int64_t)r1 * k + r1, k,
                                         A + (int64_t)r2 * k + r1, k, 0.0f,
                                         A + (int64_t)r1 * k + r2, k, d_info, s);
  GPTQ_CHECK_LAUNCH();
  trmm_right_upper_inplace_kernel<<<(unsigned)cdiv(k1, TR_TM), 256, 0, s>>>(
      A + (int64_t)r1 * k + r2, k, k1, k2, A + (int64_t)r2 * k + r2, k, -1.0f, d_info);
  GPTQ_CHECK_LAUNCH();
  return GPTQ_OK;
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
    hinv_gather_lower_kernel<<<grid, 256, 0, s>>>(H, k, perm, sc.diag, sc.lambda, U);
    GPTQ_CHECK_LAUNCH();
  }
  // blocks from the bottom; the short block (if any) is the top one
  for (int j1 = k; j1 > 0; j1 -= HV_B) {
    const int j0 = j1 > HV_B ? j1 - HV_B : 0;
    const int b = j1 - j0;
    chol_inv_diag_kernel<<<1, 256, 0, s>>>(U, k, j0, b, sc.ujj, d_info);
    GPTQ_CHECK_LAUNCH();
    if (j0 > 0) {
      chol_panel_kernel<<<(unsigned)cdiv(j0, HV_B), 256, 0, s>>>(U, k, j0, b, sc.ujj, d_info);
      GPTQ_CHECK_LAUNCH();
      const int nt = (int)cdiv(j0, 128);
      syrk_lower_tn_kernel<<<dim3(nt, nt), 256, 0, s>>>(U, k, j0, j0, b, d_info);
      GPTQ_CHECK_LAUNCH();
    }
  }
  {
    gptq_status st = trtri_range(U, k, 0, (int)cdiv(k, HV_B), d_info, s);
    if (st != GPTQ_OK) return st;
  }
  {
    dim3 grid((unsigned)cdiv(k, 1024), (unsigned)k);
    zero_lower_kernel<<<grid, 256, 0, s>>>(U, k, d_info);
    GPTQ_CHECK_LAUNCH();
  }
  return GPTQ_OK;
}

}  // namespace gptq
