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
// LOWER triangle; the UPPER triangle first holds Y = V[0:e, e:] U[e:, e:]
// (rows above the processed part) and turns into U row block by row block.
// Blocks of HV_B = 64 indices, from the last one up; step J = [j0, j1), e = j1:
//   K1 diag    L_JJ from the Schur-updated diagonal block (lower part) and
//              U_JJ = (L_JJ^T)^-1, written to A[J, J] (upper part; blocked in
//              16 x 16 pieces inside one CTA).
//   K2 panel   P = L[J, 0:j0] = U_JJ * Hp[J, 0:j0]   (in place, lower part),
//      and     U[J, e:] = -U_JJ * Y[J, e:]          (in place, upper part):
//              V = [[V_JJ, V_J*], [0, V_**]] gives U_J* = -V_JJ^-1 V_J* U_**.
//              K1 and K2 also write row block J transposed and split into
//              tf32 hi / lo, the operand of the tensor-core update.
//   K3 one rank-64 update of rows [0, j0) (K = the 64 rows of block J), on
//      the tensor cores in fp32-accurate 3xTF32 when the workspace holds the
//      operand splits (tf32x3.cu), else on the CUDA cores:
//              A[0:j0, 0:j0] (lower) -= P^T P        (Schur complement)
//              Y[0:j0, j0:]          += P^T U[J, j0:] (V[0:j0, J] = P^T)
//      The tensor-core form updates the whole square [0, j0)^2 (tiles that
//      lie entirely above its diagonal excepted), so the strip
//      A[0:j0, j0:j1] is cleared by K2 before Y's block-J columns start.
// On the tensor-core path the update has two levels: outer blocks O =
// [o0, o1) of HV_O = 512 indices (8 blocks).  Block J's update goes at once
// only to the band of rows [o0, j0) -- everything the later blocks of O read
// (their diagonal blocks, panels and Y rows) -- and the rows [0, o0) above O
// get the contributions of all of O's blocks in one K = 512 product at O's
// end.  Its operand holds the 8 row blocks side by side; the Schur part of a
// block inside O (columns [o0, j0)) is zeroed once its band update has used
// it, so that only Y contributions reach those columns of the rows above.
// Adds are reordered, nothing else: the result is that of the one-level
// scheme up to fp32 rounding, and the k x k matrix (larger than L2 for the
// widest layers) is streamed 8 times less often.
// A final pass zeroes the strict lower triangle.
#include "common.cuh"

namespace gptq {

constexpr int HV_B = 64;   // block width
constexpr int HV_O = 512;  // outer block width of the two-level tensor-core path

bool tc_update_supported(int64_t k);
gptq_status tc_rank_update(float* A, int k, int row0, int row1, int split, int K, int ld_s,
                           const float* s_hi, const float* s_lo, const float* r_hi,
                           const float* r_lo, int32_t* d_info, cudaStream_t s);

struct HinvScratch {
  double* sum_diag;  // [1]
  float* lambda;     // [1]
  float* diag;       // [k] diag(H) after the dead-column fix
  float* s_hi;       // [k * HV_O] signed splits of the outer block's row blocks, transposed
  float* s_lo;       //   (tensor-core path; row block J at column j0 - o0)
  float* r_hi;       // [k * HV_O] unsigned splits (columns < j0 only)
  float* r_lo;
};

// Scratch of the CUDA-core path.
size_t hinv_workspace_min_bytes(int64_t k) {
  size_t b = 0;
  b += align256(sizeof(double));
  b += align256(sizeof(float));
  b += align256(sizeof(float) * (size_t)k);
  return b;
}

// Scratch of the tensor-core path with outer blocks of `outer` columns.
static size_t hinv_workspace_tc_bytes(int64_t k, int outer) {
  return hinv_workspace_min_bytes(k) + 4 * align256(sizeof(float) * (size_t)outer * (size_t)k);
}

// Scratch the call asks for (gptq_workspace_size): the two-level tensor-core
// path where it applies.
size_t hinv_workspace_bytes(int64_t k) {
  return tc_update_supported(k) ? hinv_workspace_tc_bytes(k, HV_O) : hinv_workspace_min_bytes(k);
}

static HinvScratch carve(void* ws, int64_t k, int outer) {
  char* p = (char*)ws;
  HinvScratch s;
  s.sum_diag = (double*)p; p += align256(sizeof(double));
  s.lambda = (float*)p; p += align256(sizeof(float));
  s.diag = (float*)p; p += align256(sizeof(float) * (size_t)k);
  float* t[4] = {nullptr, nullptr, nullptr, nullptr};
  for (int i = 0; i < 4 && outer > 0; ++i) {
    t[i] = (float*)p;
    p += align256(sizeof(float) * (size_t)outer * (size_t)k);
  }
  s.s_hi = t[0], s.s_lo = t[1], s.r_hi = t[2], s.r_lo = t[3];
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
// by diag (dead fix) + lambda; the strict upper part (Y) starts at 0.
__global__ void hinv_gather_lower_kernel(const float* __restrict__ H, int k,
                                         const int32_t* __restrict__ perm,
                                         const float* __restrict__ diag,
                                         const float* __restrict__ lambda, float* __restrict__ A) {
  int a = blockIdx.y;
  int pa = perm[a];
  float lam = *lambda;
  const float* hrow = H + (int64_t)pa * k;
  for (int b = blockIdx.x * blockDim.x + threadIdx.x; b < k; b += gridDim.x * blockDim.x) {
    float v = (b == a) ? diag[pa] + lam : (b < a ? hrow[perm[b]] : 0.f);
    A[(int64_t)a * k + b] = v;
  }
}

// hi = x rounded to tf32 (nearest, ties away), lo = x - hi
__device__ __forceinline__ void hv_split_tf32(float x, float& hi, float& lo) {
  uint32_t h;
  asm("cvt.rna.tf32.f32 %0, %1;" : "=r"(h) : "f"(x));
  hi = __uint_as_float(h);
  lo = x - hi;
}

__device__ __forceinline__ void set_info(int32_t* d_info, int idx) { atomicCAS(d_info, 0, idx + 1); }

// K1: the diagonal block: U_JJ with U_JJ^T U_JJ = A_JJ^-1, from the lower
// part of the Schur-updated A_JJ.  One CTA of 256 threads.
// With B = P A_JJ P (P reverses the indices), A_JJ = L^T L (L lower, the
// factorisation that starts from the last index) becomes the ordinary lower
// Cholesky B = M M^T with M = P L^T P, and U_JJ = (L^T)^-1 = P M^-1 P.  The
// kernel factors B and inverts M together, in 16 x 16 blocks (rows and
// columns past b padded with the identity), block column kb = 0..3, with two
// roles so that the serial chain of diagonal blocks runs at the speed of one
// warp:
//   warp 0 (diagonal): M_kk = chol(B_kk) and N_kk = M_kk^-1, lane i holding
//     row i in registers, the pivots' columns passed along by shuffles; then
//     it hands N_kk over and waits for the next diagonal block;
//   warps 1-7 (bulk): M_ik = B_ik N_kk^T for block row kb+1 first, the rank-16
//     update of diagonal block kb+1 (handed to warp 0 at once), then the
//     rest: M_ik for the rows further down, their rank-16 update, and the
//     inverse's block row N_km = -N_kk sum_{l=m}^{kb-1} M_kl N_lm (m < kb), so
//     that N = M^-1 is complete when the loop ends.
// The hand-overs are named barriers (arrive by the producer, sync by the
// consumer); every thread takes the same sequence of barriers whatever the
// data (a failed pivot only marks the result).  U_JJ goes to the upper part of
// A[J, J]; the panel kernel reads it from there.
constexpr int K1_BS = 16;                 // block size
constexpr int K1_NB = HV_B / K1_BS;       // blocks per side
constexpr int K1_LD = HV_B + 1;
constexpr int K1_BULK = 224;              // threads of warps 1-7

__device__ __forceinline__ void k1_bar_sync(uint32_t id, uint32_t n) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(n) : "memory");
}
__device__ __forceinline__ void k1_bar_arrive(uint32_t id, uint32_t n) {
  asm volatile("bar.arrive %0, %1;" ::"r"(id), "r"(n) : "memory");
}

// Pivot C of chol16_rows and the ones after it, unrolled at compile time by
// template recursion (so that a[] stays in registers).
template <int C>
struct Chol16Rows {
  __device__ __forceinline__ static void run(float (&a)[16], int i, float& myr, int& bad) {
    const float p = __shfl_sync(0xffffffffu, a[C], C);
    if ((!(p > 0.f) || !isfinite(p)) && bad < 0) bad = C;
    const float r = rsqrtf(p);  // 1 / sqrt(p), within 2 ulp
    if (i == C) myr = r;
    if (i >= C) a[C] *= r;      // column C of M (the pivot row gets sqrt(p))
#pragma unroll
    for (int j = C + 1; j < 16; ++j) {
      const float lj = __shfl_sync(0xffffffffu, a[C], j);
      if (i >= j) a[j] = fmaf(-a[C], lj, a[j]);
    }
    Chol16Rows<C + 1>::run(a, i, myr, bad);
  }
};
template <>
struct Chol16Rows<16> {
  __device__ __forceinline__ static void run(float (&)[16], int, float&, int&) {}
};

__device__ __forceinline__ int chol16_rows(float (*S)[K1_LD], float* rd, int c0, int lane) {
  const int i = lane & 15;
  float a[16];
#pragma unroll
  for (int j = 0; j < 16; ++j) a[j] = (j <= i) ? S[c0 + i][c0 + j] : 0.f;
  int bad = -1;
  float myr = 0.f;
  Chol16Rows<0>::run(a, i, myr, bad);
  if (lane < 16) {
#pragma unroll
    for (int j = 0; j < 16; ++j)
      if (j <= i) S[c0 + i][c0 + j] = a[j];
    rd[c0 + i] = myr;
  }
  return bad;
}

// N = M^-1 of the 16 x 16 lower block at (c0, c0) of S, into T: lane j < 16
// solves for column j (x_j = 1 / M_jj, x_i = -(sum_{m=j}^{i-1} M_im x_m) / M_ii),
// every lane reading the same row of M at a time (broadcast).
__device__ __forceinline__ void inv16_cols(const float (*S)[K1_LD], float (*T)[K1_LD],
                                           const float* rd, int c0, int lane) {
  if (lane >= 16) return;
  const int j = lane;
  float x[16];
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    float acc = 0.f;
#pragma unroll
    for (int m = 0; m < i; ++m) acc = fmaf(S[c0 + i][c0 + m], x[m], acc);
    const float r = rd[c0 + i];
    x[i] = (i < j) ? 0.f : (i == j ? r : -acc * r);
  }
#pragma unroll
  for (int i = 0; i < 16; ++i)
    if (i >= j) T[c0 + i][c0 + j] = x[i];
}

__global__ void __launch_bounds__(256)
chol_inv_diag_kernel(float* __restrict__ A, int k, int j0, int b, int32_t* __restrict__ d_info) {
  __shared__ float S[HV_B][K1_LD];                  // B, then M (lower part)
  __shared__ float T[HV_B][K1_LD];                  // N = M^-1 (lower part)
  __shared__ float Mt[HV_B - K1_BS][K1_BS + 1];     // M_ik of the current block column
  __shared__ float Xs[K1_NB - 1][K1_BS][K1_BS + 1];  // X_m of the current block row
  __shared__ float rdg[HV_B];                        // 1 / M_ii
  __shared__ int fail;
  const int t = threadIdx.x, warp = t >> 5, lane = t & 31;
  // the padding and the zeros go in while the previous kernel finishes
  for (int e = t; e < HV_B * HV_B; e += 256) {
    const int i = e / HV_B, j = e % HV_B;
    S[i][j] = (i == j && i >= b) ? 1.f : 0.f;
    T[i][j] = 0.f;
  }
  if (t == 0) fail = -1;
  pdl_wait();
  pdl_trigger();
  if (*d_info != 0) return;  // the same word for every thread: the whole CTA leaves
  // B[b-1-ca][b-1-ra] = A[ra][ca] for ca <= ra < b (coalesced along ca; the
  // loads are in flight across the barrier that orders them after the zeros)
  {
    float v[HV_B * HV_B / 256];
#pragma unroll
    for (int q = 0; q < HV_B * HV_B / 256; ++q) {
      const int e = t + 256 * q, ra = e / HV_B, ca = e % HV_B;
      v[q] = (ra < b && ca <= ra) ? A[(int64_t)(j0 + ra) * k + j0 + ca] : 0.f;
    }
    __syncthreads();
#pragma unroll
    for (int q = 0; q < HV_B * HV_B / 256; ++q) {
      const int e = t + 256 * q, ra = e / HV_B, ca = e % HV_B;
      if (ra < b && ca <= ra) S[b - 1 - ca][b - 1 - ra] = v[q];
    }
  }
  __syncthreads();

  if (warp == 0) {
    for (int kb = 0; kb < K1_NB; ++kb) {
      const int c0 = kb * K1_BS;
      if (kb > 0) k1_bar_sync(2, 256);  // diagonal block kb updated by the bulk warps
      const int bad = chol16_rows(S, rdg, c0, lane);
      if (lane == 0 && bad >= 0 && fail < 0) fail = c0 + bad;
      __syncwarp();
      inv16_cols(S, T, rdg, c0, lane);
      __syncwarp();
      k1_bar_arrive(1, 256);            // M_kk, N_kk ready
    }
  } else {
    const int u = t - 32;  // 0 .. K1_BULK - 1
    for (int kb = 0; kb < K1_NB; ++kb) {
      const int c0 = kb * K1_BS, r0 = c0 + K1_BS, nr = HV_B - r0;
      k1_bar_sync(1, 256);
      if (kb + 1 < K1_NB) {
        // block row kb + 1 first: M_{kb+1,kb} = B_{kb+1,kb} N_kk^T ...
        for (int e = u; e < K1_BS * K1_BS; e += K1_BULK) {
          const int ii = e / K1_BS, j = e % K1_BS;
          float acc = 0.f;
#pragma unroll
          for (int m = 0; m < K1_BS; ++m)
            if (m <= j) acc = fmaf(S[r0 + ii][c0 + m], T[c0 + j][c0 + m], acc);
          Mt[ii][j] = acc;
        }
        k1_bar_sync(3, K1_BULK);
        // ... and the rank-16 update of diagonal block kb + 1
        for (int e = u; e < K1_BS * K1_BS; e += K1_BULK) {
          const int ii = e / K1_BS, jj = e % K1_BS;
          if (jj <= ii) {
            float acc = S[r0 + ii][r0 + jj];
#pragma unroll
            for (int m = 0; m < K1_BS; ++m) acc = fmaf(-Mt[ii][m], Mt[jj][m], acc);
            S[r0 + ii][r0 + jj] = acc;
          }
          S[r0 + ii][c0 + jj] = Mt[ii][jj];
        }
        k1_bar_arrive(2, 256);  // diagonal block kb + 1 ready
      }
      // the rows below block row kb + 1, and X_m for the inverse's block row kb
      const int nr2 = nr > K1_BS ? nr - K1_BS : 0;
      for (int e = u; e < nr2 * K1_BS + kb * K1_BS * K1_BS; e += K1_BULK) {
        if (e < nr2 * K1_BS) {
          const int ii = K1_BS + e / K1_BS, j = e % K1_BS;
          float acc = 0.f;
#pragma unroll
          for (int m = 0; m < K1_BS; ++m)
            if (m <= j) acc = fmaf(S[r0 + ii][c0 + m], T[c0 + j][c0 + m], acc);
          Mt[ii][j] = acc;
        } else {
          const int f = e - nr2 * K1_BS, mb = f / (K1_BS * K1_BS);
          const int q = (f / K1_BS) % K1_BS, c = f % K1_BS;
          float acc = 0.f;
          for (int l = mb; l < kb; ++l) {
#pragma unroll
            for (int p = 0; p < K1_BS; ++p)
              acc = fmaf(S[c0 + q][l * K1_BS + p], T[l * K1_BS + p][mb * K1_BS + c], acc);
          }
          Xs[mb][q][c] = acc;
        }
      }
      k1_bar_sync(3, K1_BULK);
      // M_ik back into B, the rank-16 update below block row kb + 1 (rows and
      // columns from r0 + 16 down, and block column kb + 1 of those rows),
      // the inverse's block row kb
      for (int e = u; e < nr2 * K1_BS; e += K1_BULK) {
        const int ii = K1_BS + e / K1_BS, j = e % K1_BS;
        S[r0 + ii][c0 + j] = Mt[ii][j];
      }
      for (int e = u; e < nr2 * nr; e += K1_BULK) {
        const int ii = K1_BS + e / nr, jj = e % nr;
        if (jj <= ii) {
          float acc = S[r0 + ii][r0 + jj];
#pragma unroll
          for (int m = 0; m < K1_BS; ++m) acc = fmaf(-Mt[ii][m], Mt[jj][m], acc);
          S[r0 + ii][r0 + jj] = acc;
        }
      }
      for (int e = u; e < kb * K1_BS * K1_BS; e += K1_BULK) {
        const int mb = e / (K1_BS * K1_BS), r = (e / K1_BS) % K1_BS, c = e % K1_BS;
        float acc = 0.f;
#pragma unroll
        for (int q = 0; q < K1_BS; ++q)
          if (q <= r) acc = fmaf(T[c0 + r][c0 + q], Xs[mb][q][c], acc);
        T[c0 + r][mb * K1_BS + c] = -acc;
      }
      k1_bar_sync(3, K1_BULK);
    }
  }
  __syncthreads();
  if (fail >= 0) {
    if (t == 0) set_info(d_info, j0 + (b - 1 - fail));
    return;
  }
  // U_JJ[iu][cu] = N[b-1-iu][b-1-cu] (iu <= cu < b) into the upper part of A[J, J]
  for (int e = t; e < HV_B * HV_B; e += 256) {
    const int iu = e / HV_B, cu = e % HV_B;
    if (iu <= cu && cu < b) A[(int64_t)(j0 + iu) * k + j0 + cu] = T[b - 1 - iu][b - 1 - cu];
  }
}

// K2, one launch, three independent roles (16-column tiles, so that the launch
// fills the GPU; each CTA reads U_JJ from the upper part of A[J, J] and its
// whole 64 x 16 tile before writing it):
//   CTAs [0, n_pan): columns c0 .. c0+15 of [0, j0): P[:, c] = U_JJ * A[J, c]
//     (lower part of row block J, in place).
//   CTAs [n_pan, n_pan + n_row): columns c0 .. c0+15 of [e, k): U[J, c] =
//     -U_JJ * Y[J, c] (upper part of row block J, in place).
//   With st_hi given, cdiv(b, 16) more CTAs: block J's own columns of the
//     operand, st[j0 + c][s_off + m] = U_JJ[m][c] (0 below the diagonal), and
//     the s_prev slice cleared there.
//   With the tensor-core update (st_hi given) each panel CTA also zeroes rows
//     [c0, c0 + 16) of the strip A[0:j0, j0:j1], where Y's columns of block J
//     start accumulating in this step's update (the tensor-core Schur update
//     writes the whole square [0, j0)^2 and leaves values above its diagonal).
// Thread (r = t / 4, cq = t % 4) computes row r, columns 4 cq .. 4 cq + 3.  When
// st_hi is given, the new row-block tile also goes out transposed and split
// into tf32 hi / lo in the rank update's operand layout (row stride ld_s,
// this block's slice at column s_off): st[c][m] = -R[m][c] for c < j0 and
// +R[m][c] above, rt[c][m] = R[m][c] for c < j0.  With two-level blocking the
// panel CTAs also zero the slice s_prev of the block below (same outer block
// [o0, ...)) at columns [o0, j0): that block's Schur part inside the outer
// block has been applied by its band update and must not reach the outer one.
constexpr int K2_W = 16;  // columns per CTA

__global__ void __launch_bounds__(256)
panel_rowblock_kernel(float* __restrict__ A, int k, int j0, int b, int n_pan, int n_row,
                      float* __restrict__ st_hi, float* __restrict__ st_lo,
                      float* __restrict__ rt_hi, float* __restrict__ rt_lo, int ld_s, int s_off,
                      int o0, int s_prev, const int32_t* __restrict__ d_info) {
  pdl_wait();
  pdl_trigger();
  if (*d_info != 0) return;
  __shared__ __align__(16) float Us[HV_B][HV_B + 4];  // row stride 68: conflict-free row reads
  __shared__ __align__(16) float Hs[HV_B][K2_W + 4];  // row stride 20: aligned float4 rows
  __shared__ float Os[HV_B][K2_W + 1];                // results; stride 17: conflict-free columns
  const int t = threadIdx.x;
  const bool vec = (k % 4 == 0);
  if ((int)blockIdx.x >= n_pan + n_row) {
    // block J's own columns of the operand: U_JJ (upper triangle) transposed and split
    const int d0 = ((int)blockIdx.x - n_pan - n_row) * K2_W;
#pragma unroll
    for (int q = 0; q < K2_W * HV_B / 256; ++q) {
      const int e = t + 256 * q, cc = d0 + e / HV_B, m = e % HV_B;
      if (cc < b) {
        const float u = (m <= cc) ? A[(int64_t)(j0 + m) * k + j0 + cc] : 0.f;
        float h, l;
        hv_split_tf32(u, h, l);
        const int64_t o = (int64_t)(j0 + cc) * ld_s + s_off + m;
        st_hi[o] = h;
        st_lo[o] = l;
        if (s_prev >= 0) {
          st_hi[o - s_off + s_prev] = 0.f;
          st_lo[o - s_off + s_prev] = 0.f;
        }
      }
    }
    return;
  }
  const bool pan = (int)blockIdx.x < n_pan;
  const int c0 = pan ? blockIdx.x * K2_W : j0 + b + (blockIdx.x - n_pan) * K2_W;
  const int cend = pan ? j0 : k;
  const float sign = pan ? 1.0f : -1.0f;
  const int r = t >> 2, j = (t & 3) * 4;  // this thread's row and first column in the tile
  {
    // U_JJ from the upper part of A[J, J]; only entries (row, col >= row) are
    // used below, so the lower part's contents do not matter
    float4 uv[4];
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const int e4 = t + 256 * q, ur = e4 >> 4, uc = (e4 & 15) * 4;
      const float* us = A + (int64_t)(j0 + ur) * k + j0 + uc;
      if (ur < b && vec && uc + 3 < b) {
        uv[q] = *reinterpret_cast<const float4*>(us);
      } else {
        uv[q].x = (ur < b && uc < b) ? us[0] : 0.f;
        uv[q].y = (ur < b && uc + 1 < b) ? us[1] : 0.f;
        uv[q].z = (ur < b && uc + 2 < b) ? us[2] : 0.f;
        uv[q].w = (ur < b && uc + 3 < b) ? us[3] : 0.f;
      }
    }
    float4 hv;
    const float* src = A + (int64_t)(j0 + r) * k + c0 + j;
    if (r < b && vec && c0 + j + 3 < cend) {
      hv = *reinterpret_cast<const float4*>(src);
    } else {
      hv.x = (r < b && c0 + j < cend) ? src[0] : 0.f;
      hv.y = (r < b && c0 + j + 1 < cend) ? src[1] : 0.f;
      hv.z = (r < b && c0 + j + 2 < cend) ? src[2] : 0.f;
      hv.w = (r < b && c0 + j + 3 < cend) ? src[3] : 0.f;
    }
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const int e4 = t + 256 * q;
      *reinterpret_cast<float4*>(&Us[e4 >> 4][(e4 & 15) * 4]) = uv[q];
    }
    *reinterpret_cast<float4*>(&Hs[r][j]) = hv;
  }
  __syncthreads();
  float a0 = 0.f, a1 = 0.f, a2 = 0.f, a3 = 0.f;
  if (r < b) {
    for (int m = r; m < b; ++m) {
      const float u = Us[r][m];
      const float4 h = *reinterpret_cast<const float4*>(&Hs[m][j]);
      a0 = fmaf(u, h.x, a0);
      a1 = fmaf(u, h.y, a1);
      a2 = fmaf(u, h.z, a2);
      a3 = fmaf(u, h.w, a3);
    }
  }
  Os[r][j] = sign * a0, Os[r][j + 1] = sign * a1, Os[r][j + 2] = sign * a2, Os[r][j + 3] = sign * a3;
  if (r < b) {
    float* dst = A + (int64_t)(j0 + r) * k + c0 + j;
    const float o[4] = {sign * a0, sign * a1, sign * a2, sign * a3};
    if (vec && c0 + j + 3 < cend) {
      *reinterpret_cast<float4*>(dst) = make_float4(o[0], o[1], o[2], o[3]);
    } else {
#pragma unroll
      for (int jj = 0; jj < 4; ++jj)
        if (c0 + j + jj < cend) dst[jj] = o[jj];
    }
  }
  if (st_hi == nullptr) return;
  if (pan) {
    // rows c0 .. c0+15 of the strip A[0:j0, j0:j0+b)
#pragma unroll
    for (int q = 0; q < K2_W * HV_B / 256; ++q) {
      const int e = t + 256 * q, i = c0 + e / HV_B, c = j0 + e % HV_B;
      if (i < j0 && c < j0 + b) A[(int64_t)i * k + c] = 0.f;
    }
  }
  __syncthreads();
#pragma unroll
  for (int q = 0; q < K2_W * HV_B / 256; ++q) {
    const int e = t + 256 * q, cc = e / HV_B, m = e % HV_B;
    if (c0 + cc < cend) {
      const float x = m < b ? Os[m][cc] : 0.f;  // the new row block R
      float h, l;
      hv_split_tf32(pan ? -x : x, h, l);  // st = -R for c < j0, +R for c >= j1
      const int64_t o = (int64_t)(c0 + cc) * ld_s + s_off + m;
      st_hi[o] = h;
      st_lo[o] = l;
      if (pan) {
        rt_hi[o] = -h;
        rt_lo[o] = -l;
        if (s_prev >= 0 && c0 + cc >= o0) {
          st_hi[o - s_off + s_prev] = 0.f;
          st_lo[o - s_off + s_prev] = 0.f;
        }
      }
    }
  }
}

// K3: rows [0, j0) += P^T Q with P = A[j0:j0+b, 0:j0] (the panel) and
//   Q[m][c] = -P[m][c]            for c < j0 (lower-triangle tiles only),
//   Q[m][c] = U[j0 + m][c]        for c >= j0 (U_JJ read as upper triangular).
// 128 x 128 output tiles; the K = b rows are taken in chunks of 16, double
// buffered; thread (ty = t / 16, tx = t % 16) owns 8 x 8 outputs.
constexpr int RU_KC = 16, RU_LD = 128 + 4;

__global__ void __launch_bounds__(256)
rank_update_kernel(float* __restrict__ A, int k, int j0, int b, int n_low,
                   const int32_t* __restrict__ d_info) {
  if (*d_info != 0) return;
  __shared__ float Pi[2][RU_KC][RU_LD];
  __shared__ float Qc[2][RU_KC][RU_LD];
  const int x = blockIdx.x;
  int bi, c0;
  bool low;
  if (x < n_low) {
    low = true;
    bi = (int)((sqrtf(8.0f * x + 1.0f) - 1.0f) * 0.5f);
    while (bi * (bi + 1) / 2 > x) --bi;
    while ((bi + 1) * (bi + 2) / 2 <= x) ++bi;
    c0 = (x - bi * (bi + 1) / 2) * 128;
  } else {
    low = false;
    const int nt = (j0 + 127) / 128;
    const int y = x - n_low;
    bi = y % nt;
    c0 = j0 + (y / nt) * 128;
  }
  const int i0 = bi * 128;
  const int j1 = j0 + b;
  const int t = threadIdx.x, tx = t % 16, ty = t / 16;
  const int lm = t / 16, lc = (t % 16) * 8;
  float acc[8][8];
#pragma unroll
  for (int p = 0; p < 8; ++p)
#pragma unroll
    for (int q = 0; q < 8; ++q) acc[p][q] = 0.f;
  float ri[8], rq[8];
  auto gload = [&](int m0) {
    const int m = m0 + lm;
    const bool okm = m < b;
    const float* prow = A + (int64_t)(j0 + m) * k;
#pragma unroll
    for (int q = 0; q < 8; ++q) {
      const int i = i0 + lc + q, c = c0 + lc + q;
      ri[q] = (okm && i < j0) ? prow[i] : 0.f;
      bool okq;
      if (low) okq = okm && c < j0;
      else okq = okm && c < k && (c >= j1 || m <= c - j0);
      rq[q] = okq ? prow[c] : 0.f;
    }
  };
  auto sstore = [&](int buf) {
#pragma unroll
    for (int q = 0; q < 8; ++q) {
      Pi[buf][lm][lc + q] = ri[q];
      Qc[buf][lm][lc + q] = rq[q];
    }
  };
  gload(0);
  sstore(0);
  __syncthreads();
  int buf = 0;
  for (int m0 = 0; m0 < b; m0 += RU_KC) {
    const bool more = m0 + RU_KC < b;
    if (more) gload(m0 + RU_KC);
#pragma unroll
    for (int mm = 0; mm < RU_KC; ++mm) {
      float a[8], bb[8];
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        a[q] = Pi[buf][mm][ty * 4 + q];
        a[q + 4] = Pi[buf][mm][64 + ty * 4 + q];
        bb[q] = Qc[buf][mm][tx * 4 + q];
        bb[q + 4] = Qc[buf][mm][64 + tx * 4 + q];
      }
#pragma unroll
      for (int p = 0; p < 8; ++p)
#pragma unroll
        for (int q = 0; q < 8; ++q) acc[p][q] = fmaf(a[p], bb[q], acc[p][q]);
    }
    if (more) sstore(buf ^ 1);
    __syncthreads();
    buf ^= 1;
  }
  const float sign = low ? -1.0f : 1.0f;
  const int cend = low ? j0 : k;
  const bool vec = (k % 4 == 0) && (!low || c0 + 127 < i0);
#pragma unroll
  for (int p = 0; p < 8; ++p) {
    const int gi = i0 + (p < 4 ? ty * 4 + p : 64 + ty * 4 + p - 4);
    if (gi >= j0) continue;
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int gc = c0 + h * 64 + tx * 4;
      float* dst = A + (int64_t)gi * k + gc;
      if (vec && gc + 3 < cend) {
        float4 v = *reinterpret_cast<float4*>(dst);
        v.x = fmaf(sign, acc[p][h * 4 + 0], v.x);
        v.y = fmaf(sign, acc[p][h * 4 + 1], v.y);
        v.z = fmaf(sign, acc[p][h * 4 + 2], v.z);
        v.w = fmaf(sign, acc[p][h * 4 + 3], v.w);
        *reinterpret_cast<float4*>(dst) = v;
      } else {
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const int c = gc + q;
          if (c < cend && (!low || c <= gi)) dst[q] = fmaf(sign, acc[p][h * 4 + q], dst[q]);
        }
      }
    }
  }
}

// Zero the strict lower triangle of U.
__global__ void zero_lower_kernel(float* __restrict__ U, int k, const int32_t* __restrict__ d_info) {
  if (*d_info != 0) return;
  int i = blockIdx.y;
  for (int j = blockIdx.x * blockDim.x + threadIdx.x; j < i; j += gridDim.x * blockDim.x)
    U[(int64_t)i * k + j] = 0.f;
}

gptq_status prepare_hinv_impl(const float* H, int64_t k64, const gptq_config* cfg, float* U,
                              int32_t* perm, int32_t* invperm, uint8_t* dead, int32_t* d_info,
                              void* ws, size_t ws_bytes, cudaStream_t s) {
  const int k = (int)k64;
  // tensor-core rank updates when the workspace holds their operand splits:
  // two-level (outer blocks of HV_O) when it holds HV_O columns of them per
  // row, one level (outer = HV_B) when it holds HV_B; else CUDA-core updates
  int outer = 0;
  if (tc_update_supported(k)) {
    if (ws_bytes >= hinv_workspace_tc_bytes(k, HV_O)) outer = HV_O;
    else if (ws_bytes >= hinv_workspace_tc_bytes(k, HV_B)) outer = HV_B;
  }
  const bool tc = outer > 0;
  HinvScratch sc = carve(ws, k, outer);
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
  // blocks from the bottom; the short block (if any) is the top one.  Outer
  // blocks [o0, o1) of `outer` columns (whole blocks; the top one may be
  // shorter).  Per block J = [j0, j1) of an outer block: K1, K2, then the
  // band update of rows [o0, j0) (everything the outer block's later blocks
  // read); after the outer block's top block, the outer update of rows
  // [0, o0) with K = o1 - o0.  One level (outer = HV_B) has no band updates.
  const int ob = tc ? outer : HV_B;
  for (int o1 = k; o1 > 0; o1 -= ob) {
    const int o0 = o1 > ob ? o1 - ob : 0;
    for (int j1 = o1; j1 > o0; j1 -= HV_B) {
      const int j0 = j1 - HV_B > o0 ? j1 - HV_B : o0;
      const int b = j1 - j0;
      // the tensor-core updates take row block J transposed and split into
      // tf32 hi / lo, written by K1 (diagonal columns) and K2 (the rest) at
      // column j0 - o0 of the outer block's slices; their Schur part leaves
      // values above the diagonal of the square they update, so K2 also
      // clears the strip where block J's Y columns start accumulating
      const bool tcs = tc && j0 > 0;
      const int s_off = j0 - o0;
      const int s_prev = (tcs && j1 < o1) ? j1 - o0 : -1;  // the block below, same outer block
      launch_pdl(chol_inv_diag_kernel, dim3(1), dim3(256), 0, s, U, k, j0, b, d_info);
      GPTQ_CHECK_LAUNCH();
      const int n_pan = (int)cdiv(j0, K2_W);
      const int n_row = (int)cdiv(k - j1, K2_W);
      const int n_diag = tcs ? (int)cdiv(b, K2_W) : 0;
      if (n_pan + n_row + n_diag > 0) {
        launch_pdl(panel_rowblock_kernel, dim3((unsigned)(n_pan + n_row + n_diag)), dim3(256), 0,
                   s, U, k, j0, b, n_pan, n_row, tcs ? sc.s_hi : nullptr,
                   tcs ? sc.s_lo : nullptr, tcs ? sc.r_hi : nullptr, tcs ? sc.r_lo : nullptr,
                   outer, s_off, o0, s_prev, (const int32_t*)d_info);
        GPTQ_CHECK_LAUNCH();
      }
      if (j0 == 0) continue;
      if (!tc) {
        const int nt = (int)cdiv(j0, 128);
        const int n_low = nt * (nt + 1) / 2;
        const int n_right = nt * (int)cdiv(k - j0, 128);
        rank_update_kernel<<<(unsigned)(n_low + n_right), 256, 0, s>>>(U, k, j0, b, n_low,
                                                                       d_info);
        GPTQ_CHECK_LAUNCH();
      } else if (j0 > o0) {
        // band: rows [o0, j0) += (block J's panel)^T (its signed row block)
        gptq_status st = tc_rank_update(U, k, o0, j0, j0, b, outer, sc.s_hi + s_off,
                                        sc.s_lo + s_off, sc.r_hi + s_off, sc.r_lo + s_off,
                                        d_info, s);
        if (st != GPTQ_OK) return st;
      }
    }
    if (tc && o0 > 0) {
      // outer: rows [0, o0) += (the outer block's panels)^T (its row blocks,
      // without their Schur parts inside the outer block)
      gptq_status st = tc_rank_update(U, k, 0, o0, o0, o1 - o0, outer, sc.s_hi, sc.s_lo,
                                      sc.r_hi, sc.r_lo, d_info, s);
      if (st != GPTQ_OK) return st;
    }
  }
  {
    dim3 grid((unsigned)cdiv(k, 1024), (unsigned)k);
    zero_lower_kernel<<<grid, 256, 0, s>>>(U, k, d_info);
    GPTQ_CHECK_LAUNCH();
  }
  return GPTQ_OK;
}

}  // namespace gptq
