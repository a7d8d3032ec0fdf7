// Lazy-blocked GPTQ column sweep ([GPTQ-tool] "GPTQ" How it works Steps 5, 7
// and 8; A minimal Python sketch; [What-is-GPTQ] Step 3 groups).
//
// Rows of W are independent given U, so the sweep is parallel over rows and
// sequential over columns.  Per lazy block [s, e) of processing-order columns:
//   (group kernel)  when a group starts at s and is wider than the block, its
//                   per-row grid comes from the row's current weights;
//   (block kernel)  four threads per row: the block's slice of 32 rows and the
//                   block's U tile (transposed) sit in shared memory; columns
//                   are taken in sub-blocks of SB held in registers (in-sub-
//                   block compensation immediately), and the remaining columns
//                   of the block get the sub-block's errors as one rank-SB
//                   update, each thread of the row taking every fourth column;
//   (trailing)      W[:, e:] -= Err * U[s:e, e:]: on the tensor cores in
//                   fp32-accurate 3xTF32 (tf32x3.cu) when k % 4 == 0, else an
//                   fp32 CUDA-core GEMM.
// On the tensor-core path the lazy batching has two levels: blocks of B
// columns inside outer blocks of WO = 512 columns.  A block's errors update
// only the rest of its outer block at once (W[:, e:o1] -= Err_b U[s:e, e:o1]);
// the outer block's errors (r x WO) update everything beyond it in one
// K = WO product at its end (W[:, o1:] -= Err_O U[o0:o1, o1:]).  Every column
// still receives every earlier column's compensation before its own turn, so
// the result is that of the one-level sweep (and of the column-by-column
// sweep) up to fp32 summation order, while the trailing matrix, which is
// larger than L2 for the big layers, is streamed WO / B = 4 times less often.
// The layer loss is accumulated inside the block kernel through the Optimal
// Brain Surgeon accounting: fixing column i and compensating the later ones
// raises (w - q) Hd (w - q)^T by err_i^2, so per row
//   (w0 - q) H0 (w0 - q)^T = sum_i err_i^2 - lambda * sum_i (w0_i - q_i)^2
// (H0 = Hd - lambda I, dead columns count with w0 = 0); no k x k product.
// The fp32 working copy Wt (processing order) lives in the workspace.
#include <algorithm>

#include "common.cuh"
#include "sgemm.cuh"
#include "tc_ptx.cuh"

namespace gptq {

constexpr int SW_MAX_B = 128;
constexpr int SW_ROWS = 32;           // rows per CTA (4 warps x 8 rows)
constexpr int SW_THREADS = 128;
constexpr int SW_LDW = 40;            // sW column stride: 32 rows + 8 pad (conflict-free quads)
constexpr int SW_LDU = SW_MAX_B + 4;  // UtS column stride
constexpr size_t SW_SMEM = sizeof(float) * ((size_t)SW_MAX_B * SW_LDU + (size_t)SW_MAX_B * SW_LDW +
                                            SW_MAX_B) +
                           sizeof(int32_t) * SW_MAX_B;

// Layout of the lane kernel for L lanes per row (L = 4 or 8): S = 128 / L
// slots per lane, record segments of S + 4 floats (the pad spreads the lanes'
// float4 reads over distinct banks).
template <int L> struct SqLayout {
  static constexpr int S = SW_MAX_B / L;             // slots (columns) per lane
  static constexpr int SEG = S + 4;                  // floats per (column, lane) segment
  static constexpr int LDI = L * SEG;                // floats per column of Uq
  static constexpr int UQ = SW_MAX_B * LDI;
  static constexpr int UD = (SW_MAX_B / L) * L * L;  // diagonal L x L tiles
  static constexpr size_t REC_BYTES =
      sizeof(float) * ((size_t)UQ + UD + SW_MAX_B) + sizeof(int32_t) * SW_MAX_B;
  static constexpr size_t SMEM = REC_BYTES + 64;
  static constexpr int ROWS_PER_WARP = 32 / L;
};
constexpr int SQ_MAX_WARPS = 12;
constexpr uint32_t SQ_COPY_CHUNK = 16384;
constexpr size_t SQ_REC_MAX = SqLayout<8>::REC_BYTES > SqLayout<4>::REC_BYTES
                                  ? SqLayout<8>::REC_BYTES
                                  : SqLayout<4>::REC_BYTES;

// per-block records of the lane kernel (one per lazy block)
static size_t sweep_records_bytes(int64_t k, int B) { return (size_t)cdiv(k, B) * SQ_REC_MAX; }

bool tc_update_supported(int64_t k);
gptq_status tc_split_transpose(const float* src, int64_t lds, int rows, int cols, float sign,
                               int upper_only, float* hi, float* lo, int64_t ldo, cudaStream_t s);
gptq_status tc_sweep_trailing(const float* err_hi, const float* err_lo, int ldE, int K,
                              const float* nut_hi, const float* nut_lo, float* Wt, int r, int k,
                              int s0, int c0, int c1, int32_t* d_status, cudaStream_t s);

constexpr int SW_OUTER = 512;  // outer lazy block of the tensor-core path

// Outer block width: SW_OUTER when every dynamic grid wider than a block
// still sees all of its group's columns up to date at the group's start
// (groups inside a block, static grids, one grid per row, or groups that
// nest with the outer blocks), else B (one level).
static int sweep_outer_width(int64_t k, int B, int G, bool static_groups, bool tc) {
  if (!tc || B >= SW_OUTER || SW_OUTER % B != 0) return B;
  if (static_groups || G <= B || G >= k || SW_OUTER % G == 0 || G % SW_OUTER == 0) return SW_OUTER;
  return B;
}

struct SweepScratch {
  float* Wt;      // [r * k] working weights, processing order
  float* Err;     // [r * WO] errors of the current outer block (tf32 high part on the tensor-core path)
  float* Err_lo;  // [r * WO] tf32 low part (tensor-core path)
  float* U_hi;    // [k * k] tf32 split of -U^T (tensor-core path)
  float* U_lo;    // [k * k]
  float* lambda;  // [1] damping added to the Hessian diagonal (for the loss)
  uint8_t* rec;   // per-block records of the 4-lanes-per-row kernel
};

size_t sweep_workspace_bytes(int64_t r, int64_t k, int B, int G, bool static_groups) {
  const bool tc = tc_update_supported(k);
  const int WO = sweep_outer_width(k, B, G == -1 ? (int)k : G, static_groups, tc);
  size_t b = align256(sizeof(float) * (size_t)r * k) + 2 * align256(sizeof(float) * (size_t)r * WO) +
             align256(sizeof(float)) + align256(sweep_records_bytes(k, B));
  if (tc) b += 2 * align256(sizeof(float) * (size_t)k * k);
  return b;
}

static SweepScratch carve_sweep(void* ws, int64_t r, int64_t k, int B, int WO, bool tc) {
  char* p = (char*)ws;
  SweepScratch s;
  s.Wt = (float*)p; p += align256(sizeof(float) * (size_t)r * k);
  s.Err = (float*)p; p += align256(sizeof(float) * (size_t)r * WO);
  s.Err_lo = (float*)p; p += align256(sizeof(float) * (size_t)r * WO);
  s.lambda = (float*)p; p += align256(sizeof(float));
  s.rec = (uint8_t*)p; p += align256(sweep_records_bytes(k, B));
  s.U_hi = tc ? (float*)p : nullptr;
  if (tc) p += align256(sizeof(float) * (size_t)k * k);
  s.U_lo = tc ? (float*)p : nullptr;
  return s;
}

// hi = x rounded to tf32 (nearest, ties away), lo = x - hi
__device__ __forceinline__ void split_tf32(float x, float& hi, float& lo) {
  uint32_t h;
  asm("cvt.rna.tf32.f32 %0, %1;" : "=r"(h) : "f"(x));
  hi = __uint_as_float(h);
  lo = x - hi;
}

// vec: four positions per thread (perm read and Wt written as 16-byte vectors;
// k % 4 == 0 and perm 16-byte aligned).
template <typename T>
__global__ void sweep_init_kernel(const T* __restrict__ W, int64_t ldw, int r, int k,
                                  const int32_t* __restrict__ perm,
                                  const uint8_t* __restrict__ dead, int G, int static_groups,
                                  int vec, float* __restrict__ Wt, int32_t* __restrict__ g_idx,
                                  double* __restrict__ loss, int32_t* __restrict__ d_status) {
  int row = blockIdx.y;
  const T* wrow = W + (int64_t)row * ldw;
  if (vec) {
    for (int j4 = 4 * (blockIdx.x * blockDim.x + threadIdx.x); j4 < k;
         j4 += 4 * gridDim.x * blockDim.x) {
      const int4 c4 = *reinterpret_cast<const int4*>(perm + j4);
      const int cc[4] = {c4.x, c4.y, c4.z, c4.w};
      float v[4];
#pragma unroll
      for (int q = 0; q < 4; ++q) v[q] = dead[cc[q]] ? 0.f : to_f32(wrow[cc[q]]);
      *reinterpret_cast<float4*>(Wt + (int64_t)row * k + j4) = make_float4(v[0], v[1], v[2], v[3]);
      if (row == 0) {
#pragma unroll
        for (int q = 0; q < 4; ++q) g_idx[cc[q]] = (static_groups ? cc[q] : j4 + q) / G;
      }
    }
  } else {
    for (int j = blockIdx.x * blockDim.x + threadIdx.x; j < k; j += gridDim.x * blockDim.x) {
      int c = perm[j];
      float v = dead[c] ? 0.f : to_f32(wrow[c]);
      Wt[(int64_t)row * k + j] = v;
      // dynamic groups are runs of processing positions; static ones keep the
      // original columns together
      if (row == 0) g_idx[c] = (static_groups ? c : j) / G;
    }
  }
  if (blockIdx.x == 0 && threadIdx.x == 0) {
    if (loss != nullptr) {
      loss[row] = 0.0;
      if (row == 0) loss[r] = 0.0;
    }
    if (row == 0 && d_status != nullptr) *d_status = 0;
  }
}

// lambda = percdamp * mean(diag H0), dead diagonal entries (0) counted as 1,
// exactly as the inverse factor damped the Hessian.  One CTA.
__global__ void sweep_lambda_kernel(const float* __restrict__ H0, int k, float percdamp,
                                    float* __restrict__ lambda) {
  __shared__ double red[32];
  double acc = 0.0;
  for (int i = threadIdx.x; i < k; i += blockDim.x) {
    float d = H0[(int64_t)i * k + i];
    acc += (double)(d == 0.0f ? 1.0f : d);
  }
  for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x / 32] = acc;
  __syncthreads();
  if (threadIdx.x == 0) {
    double sm = 0.0;
    for (int w = 0; w < (int)(blockDim.x / 32); ++w) sm += red[w];
    *lambda = (float)((double)percdamp * (sm / (double)k));
  }
}

// Per-row grid of a group [s, s+gw) wider than the lazy block: one warp per row.
__global__ void group_grid_kernel(const float* __restrict__ Wt, int r, int k, int s, int gw,
                                  int gidx, int ngroups, float maxq, int sym,
                                  float* __restrict__ scales, int32_t* __restrict__ zeros) {
  int warp = (blockIdx.x * blockDim.x + threadIdx.x) / kWarp;
  int lane = threadIdx.x % kWarp;
  if (warp >= r) return;
  const float* w = Wt + (int64_t)warp * k + s;
  float mn = INFINITY, mx = -INFINITY;
  for (int j = lane; j < gw; j += kWarp) {
    float v = w[j];
    mn = fminf(mn, v);
    mx = fmaxf(mx, v);
  }
  for (int o = 16; o > 0; o >>= 1) {
    mn = fminf(mn, __shfl_xor_sync(0xffffffffu, mn, o));
    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
  }
  if (lane == 0) {
    float sc, z;
    grid_from_range(mn, mx, maxq, sc, z, sym != 0);
    scales[(int64_t)warp * ngroups + gidx] = sc;
    zeros[(int64_t)warp * ngroups + gidx] = (int32_t)z;
  }
}

// Static groups: the grid of every (row, group), fitted before the sweep to
// the original weights of the original columns [g G, g G + G) (dead columns
// count as 0).  One warp per (row, group).
template <typename T>
__global__ void static_grid_kernel(const T* __restrict__ W, int64_t ldw, int r, int k,
                                   const uint8_t* __restrict__ dead, int G, int ngroups,
                                   float maxq, int sym, float* __restrict__ scales,
                                   int32_t* __restrict__ zeros) {
  const int64_t warp = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) / kWarp;
  const int lane = threadIdx.x % kWarp;
  if (warp >= (int64_t)r * ngroups) return;
  const int row = (int)(warp / ngroups), g = (int)(warp % ngroups);
  const int c0 = g * G, c1 = min(k, c0 + G);
  const T* w = W + (int64_t)row * ldw;
  float mn = INFINITY, mx = -INFINITY;
  for (int c = c0 + lane; c < c1; c += kWarp) {
    const float v = dead[c] ? 0.f : to_f32(w[c]);
    mn = fminf(mn, v);
    mx = fmaxf(mx, v);
  }
  for (int o = 16; o > 0; o >>= 1) {
    mn = fminf(mn, __shfl_xor_sync(0xffffffffu, mn, o));
    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
  }
  if (lane == 0) {
    float sc, z;
    grid_from_range(mn, mx, maxq, sc, z, sym != 0);
    scales[warp] = sc;
    zeros[warp] = (int32_t)z;
  }
}

// One lazy block [s, s + bw) for 32 rows.  Thread (rr = row in CTA, q = lane
// % 4): all four threads of a row run the column chain (identical values, so
// SIMT issues it once); the rank-SB updates of the rest of the block and the
// outputs are split by q.  SB divides the group size when groups are smaller
// than the block, so a group always starts at a sub-block boundary.
template <int SB>
__global__ void __launch_bounds__(SW_THREADS)
sweep_block_kernel(const float* __restrict__ Wt, float* __restrict__ Err,
                   float* __restrict__ Err_lo, const float* __restrict__ U,
                   const int32_t* __restrict__ perm, int r, int k, int s, int bw, int B, int ldE,
                   int G, int ngroups, float maxq, int sym, float* __restrict__ scales,
                   int32_t* __restrict__ zeros, uint8_t* __restrict__ codes,
                   double* __restrict__ loss, int32_t* __restrict__ d_status) {
  extern __shared__ float sm_sweep[];
  float* UtS = sm_sweep;                           // UtS[j * LDU + i] = U[s+i][s+j], i <= j
  float* sW = UtS + SW_MAX_B * SW_LDU;             // sW[j * LDW + rr] = W[r0+rr][s+j]
  float* rdg = sW + SW_MAX_B * SW_LDW;             // 1 / U[s+i][s+i]
  int32_t* pcol = (int32_t*)(rdg + SW_MAX_B);      // perm[s + i]
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int q = lane & 3;
  const int rr = warp * 8 + (lane >> 2);
  const int r0 = blockIdx.x * SW_ROWS;
  const int row = r0 + rr;
  const bool valid = row < r;
  for (int e = tid; e < bw * bw; e += SW_THREADS) {
    const int i = e / bw, j = e % bw;
    UtS[j * SW_LDU + i] = (j >= i) ? U[(int64_t)(s + i) * k + s + j] : 0.f;
  }
  for (int e = tid; e < SW_ROWS * bw; e += SW_THREADS) {
    const int r2 = e / bw, j = e % bw;
    const int gr = r0 + r2;
    sW[j * SW_LDW + r2] = (gr < r) ? Wt[(int64_t)gr * k + s + j] : 0.f;
  }
  for (int i = tid; i < bw; i += SW_THREADS) {
    rdg[i] = 1.0f / U[(int64_t)(s + i) * k + s + i];
    pcol[i] = perm[s + i];
  }
  __syncthreads();

  float scale = 1.f, zero = 0.f;
  if (G > B && valid) {  // the group started at or before s and spans the block
    const int g = s / G;
    scale = scales[(int64_t)row * ngroups + g];
    zero = (float)zeros[(int64_t)row * ngroups + g];
  }
  double e2 = 0.0;
  bool nonfinite = false;

  for (int c0 = 0; c0 < bw; c0 += SB) {
    float w[SB];
#pragma unroll
    for (int jj = 0; jj < SB; ++jj) w[jj] = (c0 + jj < bw) ? sW[(c0 + jj) * SW_LDW + rr] : 0.f;
    if (G <= B && (s + c0) % G == 0) {
      const int gw = min(G, bw - c0);
      float mn = INFINITY, mx = -INFINITY;
#pragma unroll
      for (int jj = 0; jj < SB; ++jj)
        if (jj < gw) mn = fminf(mn, w[jj]), mx = fmaxf(mx, w[jj]);
      for (int j = c0 + SB + q; j < c0 + gw; j += 4) {
        const float v = sW[j * SW_LDW + rr];
        mn = fminf(mn, v);
        mx = fmaxf(mx, v);
      }
      mn = fminf(mn, __shfl_xor_sync(0xffffffffu, mn, 1));
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
      mn = fminf(mn, __shfl_xor_sync(0xffffffffu, mn, 2));
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
      grid_from_range(mn, mx, maxq, scale, zero, sym != 0);
      if (valid && q == 0) {
        scales[(int64_t)row * ngroups + (s + c0) / G] = scale;
        zeros[(int64_t)row * ngroups + (s + c0) / G] = (int32_t)zero;
      }
    }
    float errs[SB];
#pragma unroll
    for (int ii = 0; ii < SB; ++ii) {
      const int col = c0 + ii;
      float err = 0.f;
      if (col < bw) {
        const float wv = w[ii];
        float c;
        if (isfinite(wv)) {
          c = quant_code(wv, scale, zero, maxq);
        } else {
          nonfinite = true;
          c = zero;
        }
        const float qv = scale * (c - zero);
        err = (wv - qv) * rdg[col];
        if (valid && (ii & 3) == q) {
          const int oc = pcol[col];
          codes[(int64_t)row * k + oc] = (uint8_t)c;
          if (loss != nullptr) e2 += (double)err * (double)err;
        }
      }
      errs[ii] = err;
#pragma unroll
      for (int jj = ii + 1; jj < SB; ++jj)
        w[jj] = fmaf(-err, UtS[(c0 + jj) * SW_LDU + col], w[jj]);
    }
    // rank-SB update of the block's remaining columns
    for (int j = c0 + SB + q; j < bw; j += 4) {
      float v = sW[j * SW_LDW + rr];
      const float* ucol = UtS + j * SW_LDU + c0;
#pragma unroll
      for (int ii = 0; ii < SB; ++ii) v = fmaf(-errs[ii], ucol[ii], v);
      sW[j * SW_LDW + rr] = v;
    }
    if (valid) {
#pragma unroll
      for (int ii = 0; ii < SB; ++ii)
        if ((ii & 3) == q && c0 + ii < bw) {
          if (Err_lo != nullptr) {
            float h, l;
            split_tf32(errs[ii], h, l);
            Err[(int64_t)row * ldE + c0 + ii] = h;
            Err_lo[(int64_t)row * ldE + c0 + ii] = l;
          } else {
            Err[(int64_t)row * ldE + c0 + ii] = errs[ii];
          }
        }
    }
    __syncwarp();
  }
  if (loss != nullptr) {
    e2 += __shfl_xor_sync(0xffffffffu, e2, 1);
    e2 += __shfl_xor_sync(0xffffffffu, e2, 2);
    if (valid && q == 0) loss[row] += e2;
  }
  if (nonfinite && valid && d_status != nullptr) atomicCAS(d_status, 0, (int32_t)GPTQ_ERR_NONFINITE);
}

// rint(w / scale) with the IEEE quotient.
__device__ __noinline__ float rint_exact_div(float w, float scale) {
  return rintf(__fdiv_rn(w, scale));
}

// ---- the lane block kernel ----------------------------------------------------
//
// L lanes per row (L = 8 or 4).  Lane l owns the block columns l + L j
// (j = 0 .. S-1, S = 128 / L), held in registers w[]; after each sub-block of L
// columns the registers shift down by one, so w[0] is always the current
// sub-block and the loop body is the same for every sub-block.  The
// sub-block's L columns are gathered into x[0..L-1] of the row's lanes by
// shuffles and quantized there (every lane of the row runs the same column
// chain); then each lane applies the L errors to its later columns (a rank-L
// update with packed fp32x2 FMAs, in column order).  The block runs in four
// phases whose register windows (S, 3S/4, S/2, S/4 slots) cover the columns
// still ahead, so little update work is spent on dead slots.
//
// The quantization decision takes rint(w * (1/scale)).  Where that product
// lies within 1e-6 (relative) of a half-integer -- the only place where it
// can round differently from the correctly rounded quotient -- the warp redoes
// the sub-block with rint(w / scale) throughout, so every code equals
// clamp(rint(w / scale) + zero, 0, maxq) with the IEEE quotient.
//
// Per lazy block, a record built once per layer from U and perm holds, in
// the order the kernel reads them:
//   Uq[i][l][j] = U[s+i][s + l + L (i/L + j)]  (j = 1..S-1; 0 for j = 0, past
//                  the block, and in the pad)
//   Ud[m][o][o2] = U[s+Lm+o][s+Lm+o2]           (o2 > o; the L x L diagonal tiles)
//   rdg[i] = 1 / U[s+i][s+i],  pcol[i] = perm[s+i]
// and one bulk copy brings it into shared memory.
template <int L>
__global__ void sweep_records_kernel(const float* __restrict__ U, const int32_t* __restrict__ perm,
                                     int k, int B, uint8_t* __restrict__ rec_all) {
  using Ly = SqLayout<L>;
  const int b = blockIdx.x;
  const int s = b * B, bw = min(B, k - s);
  float* Uq = (float*)(rec_all + (size_t)b * SQ_REC_MAX);
  float* Ud = Uq + Ly::UQ;
  float* rdg = Ud + Ly::UD;
  int32_t* pcol = (int32_t*)(rdg + SW_MAX_B);
  // blockIdx.y splits the record's elements between CTAs
  const int tid = blockIdx.y * blockDim.x + threadIdx.x, nth = gridDim.y * blockDim.x;
  for (int e = tid; e < Ly::UQ; e += nth) {
    const int i = e / Ly::LDI, rem = e % Ly::LDI, l = rem / Ly::SEG, j = rem % Ly::SEG;
    const int col = l + L * (i / L + j);
    Uq[e] = (j >= 1 && j < Ly::S && i < bw && col < bw) ? U[(int64_t)(s + i) * k + s + col] : 0.f;
  }
  for (int e = tid; e < Ly::UD; e += nth) {
    const int m = e / (L * L), o = (e / L) % L, o2 = e % L;
    Ud[e] = (o2 > o && L * m + o2 < bw) ? U[(int64_t)(s + L * m + o) * k + s + L * m + o2] : 0.f;
  }
  for (int i = tid; i < SW_MAX_B; i += nth) {
    rdg[i] = (i < bw) ? 1.0f / U[(int64_t)(s + i) * k + s + i] : 0.f;
    pcol[i] = (i < bw) ? perm[s + i] : 0;
  }
}

struct SqArgs {
  const float* Wt;
  float* Err;
  float* Err_lo;
  const uint8_t* rec;  // this block's record
  int r, k, s, bw, B, G, ngroups;
  int ldE;  // row stride of Err / Err_lo (Err points at this block's first column)
  float maxq;
  int sym;  // symmetric grid
  float* scales;
  int32_t* zeros;
  uint8_t* codes;
  double* loss;
  int32_t* d_status;
  uint32_t spin;  // polls before the record wait gives up
};

template <int L>
struct SqState {
  float w[SqLayout<L>::S];
  float scale, zero, inv_s, lo_d, hi_d;
  float next_scale, next_zero;  // MODE 2: this lane's column of the next sub-block
  double e2;
  bool nonfinite;
};

// MODE 2 (static groups): fetch the fixed grid of this lane's column in
// sub-block m, i.e. group perm[s + c] / G of the row.
template <int L>
__device__ __forceinline__ void sq_fetch_static(SqState<L>& st, int m, const SqArgs& a,
                                                const int32_t* pcol, int l, int row, bool valid) {
  const int c = L * m + l;
  st.next_scale = 1.f, st.next_zero = 0.f;
  if (valid && c < a.bw) {
    const int64_t idx = (int64_t)row * a.ngroups + pcol[c] / a.G;
    st.next_scale = a.scales[idx];
    st.next_zero = (float)a.zeros[idx];
  }
}

// One sub-block (columns L m .. L m + L - 1) with a register window of W + 1 slots.
template <int L, int W, int MODE>
__device__ __forceinline__ void sq_sub_block(SqState<L>& st, int m, const SqArgs& a,
                                             const float* Uq, const float* Ud, const float* rdg,
                                             const int32_t* pcol, int l, int row, bool valid) {
  using Ly = SqLayout<L>;
  float x[L];
#pragma unroll
  for (int o = 0; o < L; ++o) x[o] = __shfl_sync(0xffffffffu, st.w[0], o, L);
  if (MODE == 1 && (L * m) % a.G == 0) {
    // a group starts here: its grid from the current weights of its columns
    // [Lm, Lm + G) (slots past the block hold 0, which min(., 0) / max(., 0) absorb)
    float mn = x[0], mx = x[0];
#pragma unroll
    for (int o = 1; o < L; ++o) mn = fminf(mn, x[o]), mx = fmaxf(mx, x[o]);
    const int gq = a.G / L;
    float pn = INFINITY, px = -INFINITY;
#pragma unroll
    for (int j = 1; j <= W; ++j)
      if (j < gq) pn = fminf(pn, st.w[j]), px = fmaxf(px, st.w[j]);
#pragma unroll
    for (int o = 1; o < L; o <<= 1) {
      pn = fminf(pn, __shfl_xor_sync(0xffffffffu, pn, o, L));
      px = fmaxf(px, __shfl_xor_sync(0xffffffffu, px, o, L));
    }
    grid_from_range(fminf(mn, pn), fmaxf(mx, px), a.maxq, st.scale, st.zero, a.sym != 0);
    st.inv_s = 1.0f / st.scale;
    st.lo_d = -st.zero;
    st.hi_d = a.maxq - st.zero;
    if (valid && l == 0) {
      const int g = (a.s + L * m) / a.G;
      a.scales[(int64_t)row * a.ngroups + g] = st.scale;
      a.zeros[(int64_t)row * a.ngroups + g] = (int32_t)st.zero;
    }
  }
  // MODE 2: every column has its own fixed grid; lane o holds column o's
  // (fetched one sub-block ahead) and the row's lanes share them by shuffles
  float own_zero = st.zero;
  float gs[L], gi[L], gz[L];
  if (MODE == 2) {
    const float own_scale = st.next_scale;
    own_zero = st.next_zero;
    sq_fetch_static(st, m + 1, a, pcol, l, row, valid);
    const float own_inv = 1.0f / own_scale;
#pragma unroll
    for (int o = 0; o < L; ++o) {
      gs[o] = __shfl_sync(0xffffffffu, own_scale, o, L);
      gi[o] = __shfl_sync(0xffffffffu, own_inv, o, L);
      gz[o] = __shfl_sync(0xffffffffu, own_zero, o, L);
    }
  }
  float rd[L];
#pragma unroll
  for (int v = 0; v < L / 4; ++v) {
    const float4 r4 = *(const float4*)(rdg + L * m + 4 * v);
    rd[4 * v] = r4.x, rd[4 * v + 1] = r4.y, rd[4 * v + 2] = r4.z, rd[4 * v + 3] = r4.w;
  }
  float x0[L];
#pragma unroll
  for (int o = 0; o < L; ++o) x0[o] = x[o];
  float err[L], dq[L];
  bool tie = false;
#pragma unroll
  for (int o = 0; o < L; ++o) {
    const float sc = MODE == 2 ? gs[o] : st.scale;
    const float lo_d = MODE == 2 ? -gz[o] : st.lo_d;
    const float hi_d = MODE == 2 ? a.maxq - gz[o] : st.hi_d;
    const float t = x[o] * (MODE == 2 ? gi[o] : st.inv_s);
    const float rq = rintf(t);
    tie |= fabsf(fabsf(t - rq) - 0.5f) <= 1e-6f * fabsf(t);
    const float d = fminf(fmaxf(rq, lo_d), hi_d);  // code - zero
    const float e = (x[o] - sc * d) * rd[o];
    err[o] = e;
    dq[o] = d;
    if (o + 1 < L) {
      const float* ur = Ud + (m * L + o) * L;
#pragma unroll
      for (int o2 = o + 1; o2 < L; ++o2) x[o2] = fmaf(-e, ur[o2], x[o2]);
    }
  }
  if (__any_sync(0xffffffffu, tie)) {
#pragma unroll
    for (int o = 0; o < L; ++o) x[o] = x0[o];
#pragma unroll
    for (int o = 0; o < L; ++o) {
      const float sc = MODE == 2 ? gs[o] : st.scale;
      const float lo_d = MODE == 2 ? -gz[o] : st.lo_d;
      const float hi_d = MODE == 2 ? a.maxq - gz[o] : st.hi_d;
      const float d = fminf(fmaxf(rint_exact_div(x[o], sc), lo_d), hi_d);
      const float e = (x[o] - sc * d) * rd[o];
      err[o] = e;
      dq[o] = d;
      if (o + 1 < L) {
        const float* ur = Ud + (m * L + o) * L;
#pragma unroll
        for (int o2 = o + 1; o2 < L; ++o2) x[o2] = fmaf(-e, ur[o2], x[o2]);
      }
    }
  }
  // rank-L update of the later columns, one column's error at a time
#pragma unroll
  for (int o = 0; o < L; ++o) {
    const float4* up = (const float4*)(Uq + (L * m + o) * Ly::LDI + l * Ly::SEG);
    const float2 ne = make_float2(-err[o], -err[o]);
#pragma unroll
    for (int v = 0; v < (W + 1) / 4; ++v) {
      const float4 u4 = up[v];
      float2 p0 = make_float2(st.w[4 * v], st.w[4 * v + 1]);
      float2 p1 = make_float2(st.w[4 * v + 2], st.w[4 * v + 3]);
      p0 = __ffma2_rn(ne, make_float2(u4.x, u4.y), p0);
      p1 = __ffma2_rn(ne, make_float2(u4.z, u4.w), p1);
      st.w[4 * v] = p0.x, st.w[4 * v + 1] = p0.y;
      st.w[4 * v + 2] = p1.x, st.w[4 * v + 3] = p1.y;
    }
  }
  // this lane's column of the sub-block
  float e_own = err[0], d_own = dq[0];
#pragma unroll
  for (int o = 1; o < L; ++o)
    if (l == o) e_own = err[o], d_own = dq[o];
  const int c = L * m + l;
  if (valid && c < a.bw) {
    a.codes[(int64_t)row * a.k + pcol[c]] = (uint8_t)(d_own + own_zero);
    if (a.Err_lo != nullptr) {
      float h, lo;
      split_tf32(e_own, h, lo);
      a.Err[(int64_t)row * a.ldE + c] = h;
      a.Err_lo[(int64_t)row * a.ldE + c] = lo;
    } else {
      a.Err[(int64_t)row * a.ldE + c] = e_own;
    }
    st.nonfinite |= !isfinite(e_own);
    st.e2 += (double)e_own * (double)e_own;
  }
#pragma unroll
  for (int j = 0; j < W; ++j) st.w[j] = st.w[j + 1];
  st.w[W] = 0.f;
}

// One lazy block [s, s + bw) for 32 / L rows per warp.  MODE 1: groups start
// inside the block (G <= B, G % L == 0); MODE 0: the block lies inside one
// group whose grid is already in scales / zeros; MODE 2: static groups, each
// column's grid read from scales / zeros (group perm[col] / G).  Adds
// sum_i err_i^2 of the block to loss[row] (the Optimal Brain Surgeon part of
// the layer loss).
template <int L, int MODE>
__global__ void __launch_bounds__(SQ_MAX_WARPS * 32, 1) sweep_block_lane_kernel(SqArgs a) {
  using Ly = SqLayout<L>;
  extern __shared__ __align__(128) uint8_t smq[];
  float* Uq = (float*)smq;
  float* Ud = Uq + Ly::UQ;
  float* rdg = Ud + Ly::UD;
  const int32_t* pcol = (const int32_t*)(rdg + SW_MAX_B);
  uint64_t* bar = (uint64_t*)(smq + Ly::REC_BYTES);
  volatile int* abort_flag = (volatile int*)(bar + 1);
  const int tid = threadIdx.x, lane = tid & 31, l = lane % L;
  const int row = (blockIdx.x * (blockDim.x / 32) + (tid >> 5)) * Ly::ROWS_PER_WARP + lane / L;
  const bool valid = row < a.r;
  if (tid == 0) {
    tc::mbar_init(bar, 1);
    *abort_flag = 0;
    tc::fence_barrier_init();
  }
  __syncthreads();
  if (tid == 0) {
    tc::mbar_arrive_expect_tx(bar, (uint32_t)Ly::REC_BYTES);
    for (uint32_t off = 0; off < Ly::REC_BYTES; off += SQ_COPY_CHUNK) {
      const uint32_t n = min(SQ_COPY_CHUNK, (uint32_t)Ly::REC_BYTES - off);
      asm volatile(
          "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
              tc::smem_u32(smq + off)),
          "l"(a.rec + off), "r"(n), "r"(tc::smem_u32(bar))
          : "memory");
    }
  }
  // the record comes from a kernel that finished before the previous one
  // started; the weights (and a group grid) come from the previous kernels
  pdl_wait();
  pdl_trigger();
  SqState<L> st;
#pragma unroll
  for (int j = 0; j < Ly::S; ++j) {
    const int c = l + L * j;
    st.w[j] = (valid && c < a.bw) ? a.Wt[(int64_t)row * a.k + a.s + c] : 0.f;
  }
  st.scale = 1.f, st.zero = 0.f;
  if (MODE == 0 && valid) {
    const int g = a.s / a.G;
    st.scale = a.scales[(int64_t)row * a.ngroups + g];
    st.zero = (float)a.zeros[(int64_t)row * a.ngroups + g];
  }
  st.inv_s = 1.0f / st.scale;
  st.lo_d = -st.zero;
  st.hi_d = a.maxq - st.zero;
  st.e2 = 0.0;
  st.nonfinite = false;
  if (!tc::mbar_wait(bar, 0, abort_flag, a.spin)) {
    // the record never arrived: let the copy land (bounded) and report
    for (uint32_t i = 0; i < tc::kSpinLimit; ++i)
      if (tc::mbar_try_wait(bar, 0)) break;
    if (tid == 0 && a.d_status != nullptr) atomicCAS(a.d_status, 0, (int32_t)GPTQ_ERR_TIMEOUT);
    return;
  }
  if (MODE == 2) sq_fetch_static(st, 0, a, pcol, l, row, valid);  // needs pcol from the record
  constexpr int S = Ly::S;
  const int nsb = (a.bw + L - 1) / L;
  int m = 0;
  for (; m < min(nsb, S / 4); ++m)
    sq_sub_block<L, S - 1, MODE>(st, m, a, Uq, Ud, rdg, pcol, l, row, valid);
  for (; m < min(nsb, S / 2); ++m)
    sq_sub_block<L, 3 * S / 4 - 1, MODE>(st, m, a, Uq, Ud, rdg, pcol, l, row, valid);
  for (; m < min(nsb, 3 * S / 4); ++m)
    sq_sub_block<L, S / 2 - 1, MODE>(st, m, a, Uq, Ud, rdg, pcol, l, row, valid);
  for (; m < nsb; ++m)
    sq_sub_block<L, S / 4 - 1, MODE>(st, m, a, Uq, Ud, rdg, pcol, l, row, valid);
  double e2 = st.e2;
#pragma unroll
  for (int o = 1; o < L; o <<= 1) e2 += __shfl_xor_sync(0xffffffffu, e2, o, L);
  if (a.loss != nullptr && valid && l == 0) a.loss[row] += e2;
  if (st.nonfinite && a.d_status != nullptr) atomicCAS(a.d_status, 0, (int32_t)GPTQ_ERR_NONFINITE);
}

// Four consecutive weights as fp32 (8- or 16-byte aligned load).
__device__ __forceinline__ void load4_f32(const float* p, float (&o)[4]) {
  const float4 v = *reinterpret_cast<const float4*>(p);
  o[0] = v.x, o[1] = v.y, o[2] = v.z, o[3] = v.w;
}
__device__ __forceinline__ void load4_f32(const __half* p, float (&o)[4]) {
  const uint2 v = *reinterpret_cast<const uint2*>(p);
  const float2 a = __half22float2(*reinterpret_cast<const __half2*>(&v.x));
  const float2 b = __half22float2(*reinterpret_cast<const __half2*>(&v.y));
  o[0] = a.x, o[1] = a.y, o[2] = b.x, o[3] = b.y;
}
__device__ __forceinline__ void load4_f32(const __nv_bfloat16* p, float (&o)[4]) {
  const uint2 v = *reinterpret_cast<const uint2*>(p);
  const float2 a = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&v.x));
  const float2 b = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&v.y));
  o[0] = a.x, o[1] = a.y, o[2] = b.x, o[3] = b.y;
}

// Layer loss, second part: loss[row] -= lambda * sum_c (w0_c - q_c)^2 over the
// original columns, q = scale * (code - zero) of the column's group (dead
// columns count with w0 = 0).  One warp per row; with vec (k % 4 == 0, the
// row starts aligned) each lane takes four adjacent columns per load.
template <typename T>
__global__ void loss_finish_kernel(const T* __restrict__ W0, int64_t ldw, int r, int k, int vec,
                                   const uint8_t* __restrict__ dead,
                                   const uint8_t* __restrict__ codes,
                                   const float* __restrict__ scales,
                                   const int32_t* __restrict__ zeros,
                                   const int32_t* __restrict__ g_idx, int ngroups,
                                   const float* __restrict__ lambda, double* __restrict__ loss) {
  const int row = (blockIdx.x * blockDim.x + threadIdx.x) / kWarp;
  const int lane = threadIdx.x % kWarp;
  if (row >= r) return;
  double acc = 0.0;
  const uint8_t* crow = codes + (int64_t)row * k;
  const T* wrow = W0 + (int64_t)row * ldw;
  const float* srow = scales + (int64_t)row * ngroups;
  const int32_t* zrow = zeros + (int64_t)row * ngroups;
  if (vec) {
#pragma unroll 2
    for (int c = 4 * lane; c < k; c += 4 * kWarp) {
      const int4 g4 = *reinterpret_cast<const int4*>(g_idx + c);
      const uchar4 q4 = *reinterpret_cast<const uchar4*>(crow + c);
      const uchar4 d4 = *reinterpret_cast<const uchar4*>(dead + c);
      float w4[4];
      load4_f32(wrow + c, w4);
      const int gg[4] = {g4.x, g4.y, g4.z, g4.w};
      const uint8_t qq[4] = {q4.x, q4.y, q4.z, q4.w}, de[4] = {d4.x, d4.y, d4.z, d4.w};
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const float q = srow[gg[i]] * ((float)qq[i] - (float)zrow[gg[i]]);
        const float w0 = de[i] ? 0.f : w4[i];
        const double dd = (double)w0 - (double)q;
        acc += dd * dd;
      }
    }
  } else {
#pragma unroll 4
    for (int c = lane; c < k; c += kWarp) {
      const int g = g_idx[c];
      const float q = srow[g] * ((float)crow[c] - (float)zrow[g]);
      const float w0 = dead[c] ? 0.f : to_f32(wrow[c]);
      const double dd = (double)w0 - (double)q;
      acc += dd * dd;
    }
  }
  for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
  if (lane == 0) loss[row] -= (double)(*lambda) * acc;
}

__global__ void loss_total_kernel(double* __restrict__ loss, int r) {
  __shared__ double red[32];
  double acc = 0.0;
  for (int i = threadIdx.x; i < r; i += blockDim.x) acc += loss[i];
  for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x / 32] = acc;
  __syncthreads();
  if (threadIdx.x == 0) {
    double s = 0.0;
    for (int w = 0; w < (int)(blockDim.x / 32); ++w) s += red[w];
    loss[r] = s;
  }
}

template <int SB>
static gptq_status launch_block(unsigned grid, cudaStream_t s, const float* Wt, float* Err,
                                float* Err_lo, const float* U, const int32_t* perm, int r, int k,
                                int s0, int bw, int B, int ldE, int G, int ngroups, float maxq,
                                int sym, float* scales, int32_t* zeros, uint8_t* codes,
                                double* loss, int32_t* d_status) {
  if (smem_optin((const void*)sweep_block_kernel<SB>, SW_SMEM) != cudaSuccess) return GPTQ_ERR_CUDA;
  sweep_block_kernel<SB><<<grid, SW_THREADS, SW_SMEM, s>>>(Wt, Err, Err_lo, U, perm, r, k, s0, bw,
                                                           B, ldE, G, ngroups, maxq, sym, scales,
                                                           zeros, codes, loss, d_status);
  return GPTQ_OK;
}

// pdl: launch early behind the previous kernel (every block but the first,
// whose record may still be in flight from the kernel right before it)
template <int L, int MODE>
static gptq_status launch_lane(unsigned grid, int threads, cudaStream_t s, const SqArgs& a,
                               bool pdl) {
  if (smem_optin((const void*)sweep_block_lane_kernel<L, MODE>, SqLayout<L>::SMEM) != cudaSuccess)
    return GPTQ_ERR_CUDA;
  if (pdl)
    launch_pdl(sweep_block_lane_kernel<L, MODE>, dim3(grid), dim3(threads), SqLayout<L>::SMEM, s,
               a);
  else
    sweep_block_lane_kernel<L, MODE><<<grid, threads, SqLayout<L>::SMEM, s>>>(a);
  return GPTQ_OK;
}

template <typename T>
static gptq_status quantize_typed(const T* W, int64_t ldw, int r, int k, const float* U,
                                  const int32_t* perm, const uint8_t* dead, const float* H0,
                                  const gptq_config* cfg, uint8_t* codes, float* scales,
                                  int32_t* zeros, int32_t* g_idx, double* loss,
                                  int32_t* d_status, void* ws, cudaStream_t s) {
  const int B = cfg->block_size;
  const int G = cfg->group_size == -1 ? k : cfg->group_size;
  const int ngroups = (int)cdiv(k, G);
  const float maxq = (float)((1 << cfg->bits) - 1);
  const bool tc = tc_update_supported(k);
  const bool stat = cfg->static_groups != 0;
  const int WO = sweep_outer_width(k, B, G, stat, tc);
  SweepScratch sc = carve_sweep(ws, r, k, B, WO, tc);
  const bool want_loss = (H0 != nullptr && loss != nullptr);
  double* lossp = want_loss ? loss : nullptr;
  {
    dim3 grid((unsigned)cdiv(k, 1024), (unsigned)r);
    const int ivec = (k % 4 == 0 && (uintptr_t)perm % 16 == 0) ? 1 : 0;
    sweep_init_kernel<T><<<grid, 256, 0, s>>>(W, ldw, r, k, perm, dead, G, cfg->static_groups,
                                              ivec, sc.Wt, g_idx, lossp, d_status);
    GPTQ_CHECK_LAUNCH();
  }
  if (stat) {
    static_grid_kernel<T><<<(unsigned)cdiv((int64_t)r * ngroups * kWarp, 256), 256, 0, s>>>(
        W, ldw, r, k, dead, G, ngroups, maxq, cfg->sym, scales, zeros);
    GPTQ_CHECK_LAUNCH();
  }
  if (want_loss) {
    sweep_lambda_kernel<<<1, 1024, 0, s>>>(H0, k, cfg->percdamp, sc.lambda);
    GPTQ_CHECK_LAUNCH();
  }
  if (tc) {
    // the trailing updates read -U^T only at (c, i) with c > i
    gptq_status st = tc_split_transpose(U, k, k, k, -1.0f, 1, sc.U_hi, sc.U_lo, k, s);
    if (st != GPTQ_OK) return st;
  }
  // block kernel: the lane kernel when the groups inside a block have a
  // multiple of 4 columns (or the block lies inside one group) -- 8 lanes per
  // row unless the rows alone fill the SMs with 2 warps per scheduler, or the
  // groups need 4 -- else the 4-threads-per-row kernel
  int lane_mode = -1, lanes = 8;
  if (stat) lane_mode = 2;  // any group size: grids are looked up per column
  else if (G > B) lane_mode = 0;
  else if (G % 4 == 0) lane_mode = 1;
  const int nblocks = (int)cdiv(k, B);
  int q_warps = 1;
  unsigned q_grid = 0;
  if (lane_mode >= 0) {
    const int nsm = sm_count();
    if ((lane_mode == 1 && G % 8 != 0) || cdiv(r, 8) >= (int64_t)nsm * 8) lanes = 4;
    const int64_t warps = cdiv(r, 32 / lanes);
    q_warps = (int)std::min<int64_t>(SQ_MAX_WARPS, std::max<int64_t>(1, cdiv(warps, nsm)));
    q_grid = (unsigned)cdiv(warps, q_warps);
    const dim3 rgrid((unsigned)nblocks, 16);
    if (lanes == 8) sweep_records_kernel<8><<<rgrid, 256, 0, s>>>(U, perm, k, B, sc.rec);
    else sweep_records_kernel<4><<<rgrid, 256, 0, s>>>(U, perm, k, B, sc.rec);
    GPTQ_CHECK_LAUNCH();
  }
  int SB = 16;
  if (G < B) {
    SB = 1;
    while (SB < 16 && G % (SB * 2) == 0) SB *= 2;
  }
  const unsigned grid = (unsigned)cdiv(r, SW_ROWS);
  for (int s0 = 0, b = 0; s0 < k; s0 += B, ++b) {
    const int bw = min(B, k - s0);
    const int o0 = (s0 / WO) * WO, o1 = min(o0 + WO, k);  // the outer block of this block
    float* err_b = sc.Err + (s0 - o0);                     // this block's columns of Err
    float* err_lo_b = tc ? sc.Err_lo + (s0 - o0) : nullptr;
    if (!stat && G > B && s0 % G == 0) {
      int gw = min(G, k - s0);
      group_grid_kernel<<<(unsigned)cdiv((int64_t)r * kWarp, 256), 256, 0, s>>>(
          sc.Wt, r, k, s0, gw, s0 / G, ngroups, maxq, cfg->sym, scales, zeros);
      GPTQ_CHECK_LAUNCH();
    }
    if (lane_mode >= 0) {
      SqArgs a;
      a.Wt = sc.Wt;
      a.Err = err_b;
      a.Err_lo = err_lo_b;
      a.ldE = WO;
      a.rec = sc.rec + (size_t)b * SQ_REC_MAX;
      a.r = r, a.k = k, a.s = s0, a.bw = bw, a.B = B, a.G = G, a.ngroups = ngroups;
      a.maxq = maxq;
      a.sym = cfg->sym;
      a.scales = scales;
      a.zeros = zeros;
      a.codes = codes;
      a.loss = lossp;
      a.d_status = d_status;
      a.spin = wait_limit();
      // right behind a trailing update (not behind a group grid launch)
      const bool pdl = b > 0 && !(!stat && G > B && s0 % G == 0);
      gptq_status st;
      if (lanes == 8) {
        if (lane_mode == 0) st = launch_lane<8, 0>(q_grid, 32 * q_warps, s, a, pdl);
        else if (lane_mode == 1) st = launch_lane<8, 1>(q_grid, 32 * q_warps, s, a, pdl);
        else st = launch_lane<8, 2>(q_grid, 32 * q_warps, s, a, pdl);
      } else {
        if (lane_mode == 0) st = launch_lane<4, 0>(q_grid, 32 * q_warps, s, a, pdl);
        else if (lane_mode == 1) st = launch_lane<4, 1>(q_grid, 32 * q_warps, s, a, pdl);
        else st = launch_lane<4, 2>(q_grid, 32 * q_warps, s, a, pdl);
      }
      if (st != GPTQ_OK) return st;
    } else {
      gptq_status st = GPTQ_OK;
#define GPTQ_SWEEP_BLOCK(SBV)                                                                   \
  st = launch_block<SBV>(grid, s, sc.Wt, err_b, err_lo_b, U, perm, r, k, s0, bw, B, WO, G, ngroups, \
                         maxq, cfg->sym, scales, zeros, codes, lossp, d_status)
      switch (SB) {
        case 16: GPTQ_SWEEP_BLOCK(16); break;
        case 8: GPTQ_SWEEP_BLOCK(8); break;
        case 4: GPTQ_SWEEP_BLOCK(4); break;
        case 2: GPTQ_SWEEP_BLOCK(2); break;
        default: GPTQ_SWEEP_BLOCK(1); break;
      }
#undef GPTQ_SWEEP_BLOCK
      if (st != GPTQ_OK) return st;
    }
    GPTQ_CHECK_LAUNCH();
    const int e0 = s0 + bw;
    if (e0 >= k) continue;
    if (tc) {
      gptq_status st = GPTQ_OK;
      if (e0 < o1) {
        // the rest of the outer block: W[:, e0:o1] -= Err_b U[s0:e0, e0:o1]
        st = tc_sweep_trailing(err_b, err_lo_b, WO, bw, sc.U_hi, sc.U_lo, sc.Wt, r, k, s0, e0, o1,
                               d_status, s);
      } else {
        // everything beyond the outer block: W[:, o1:] -= Err_O U[o0:o1, o1:]
        st = tc_sweep_trailing(sc.Err, sc.Err_lo, WO, o1 - o0, sc.U_hi, sc.U_lo, sc.Wt, r, k, o0,
                               o1, k, d_status, s);
      }
      if (st != GPTQ_OK) return st;
    } else {  // one level (WO == B)
      sgemm<false, false, false, false, false>(r, k - e0, bw, -1.0f, sc.Err, WO,
                                               U + (int64_t)s0 * k + e0, k, 1.0f, sc.Wt + e0, k,
                                               nullptr, s);
      GPTQ_CHECK_LAUNCH();
    }
  }
  if (want_loss) {
    const int lvec = (k % 4 == 0 && ldw % 4 == 0 && (uintptr_t)W % (4 * sizeof(T)) == 0 &&
                      (uintptr_t)codes % 4 == 0 && (uintptr_t)g_idx % 16 == 0 &&
                      (uintptr_t)dead % 4 == 0)
                         ? 1
                         : 0;
    loss_finish_kernel<T><<<(unsigned)cdiv((int64_t)r * kWarp, 256), 256, 0, s>>>(
        W, ldw, r, k, lvec, dead, codes, scales, zeros, g_idx, ngroups, sc.lambda, loss);
    GPTQ_CHECK_LAUNCH();
    loss_total_kernel<<<1, 1024, 0, s>>>(loss, r);
    GPTQ_CHECK_LAUNCH();
  }
  return GPTQ_OK;
}

gptq_status quantize_layer_impl(const void* W, gptq_dtype dt, int64_t r, int64_t k, int64_t ldw,
                                const float* U, const int32_t* perm, const uint8_t* dead,
                                const float* H0, const gptq_config* cfg, uint8_t* codes,
                                float* scales, int32_t* zeros, int32_t* g_idx, double* loss,
                                int32_t* d_status, void* ws, cudaStream_t s) {
  switch (dt) {
    case GPTQ_F32:
      return quantize_typed<float>((const float*)W, ldw, (int)r, (int)k, U, perm, dead, H0, cfg,
                                   codes, scales, zeros, g_idx, loss, d_status, ws, s);
    case GPTQ_F16:
      return quantize_typed<__half>((const __half*)W, ldw, (int)r, (int)k, U, perm, dead, H0, cfg,
                                    codes, scales, zeros, g_idx, loss, d_status, ws, s);
    case GPTQ_BF16:
      return quantize_typed<__nv_bfloat16>((const __nv_bfloat16*)W, ldw, (int)r, (int)k, U, perm,
                                           dead, H0, cfg, codes, scales, zeros, g_idx, loss,
                                           d_status, ws, s);
  }
  return GPTQ_ERR_INVALID_ARG;
}

}  // namespace gptq
