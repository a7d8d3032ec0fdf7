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
// The layer loss is accumulated inside the block kernel through the Optimal
// Brain Surgeon accounting: fixing column i and compensating the later ones
// raises (w - q) Hd (w - q)^T by err_i^2, so per row
//   (w0 - q) H0 (w0 - q)^T = sum_i err_i^2 - lambda * sum_i (w0_i - q_i)^2
// (H0 = Hd - lambda I, dead columns count with w0 = 0); no k x k product.
// The fp32 working copy Wt (processing order) lives in the workspace.
#include "common.cuh"
#include "sgemm.cuh"

namespace gptq {

constexpr int SW_MAX_B = 128;
constexpr int SW_ROWS = 32;           // rows per CTA (4 warps x 8 rows)
constexpr int SW_THREADS = 128;
constexpr int SW_LDW = 40;            // sW column stride: 32 rows + 8 pad (conflict-free quads)
constexpr int SW_LDU = SW_MAX_B + 4;  // UtS column stride
constexpr size_t SW_SMEM = sizeof(float) * ((size_t)SW_MAX_B * SW_LDU + (size_t)SW_MAX_B * SW_LDW +
                                            SW_MAX_B) +
                           sizeof(int32_t) * SW_MAX_B;

bool tc_update_supported(int64_t k);
gptq_status tc_split_transpose(const float* src, int64_t lds, int rows, int cols, float* hi,
                               float* lo, int64_t ldo, cudaStream_t s);
gptq_status tc_sweep_trailing(const float* err_hi, const float* err_lo, int B, const float* u_hi,
                              const float* u_lo, float* Wt, int r, int k, int s0, int e,
                              int32_t* d_status, cudaStream_t s);

struct SweepScratch {
  float* Wt;      // [r * k] working weights, processing order
  float* Err;     // [r * B] errors of the current block (tf32 high part on the tensor-core path)
  float* Err_lo;  // [r * B] tf32 low part (tensor-core path)
  float* U_hi;    // [k * k] tf32 split of U^T (tensor-core path)
  float* U_lo;    // [k * k]
  float* lambda;  // [1] damping added to the Hessian diagonal (for the loss)
};

size_t sweep_workspace_bytes(int64_t r, int64_t k, int B) {
  size_t b = align256(sizeof(float) * (size_t)r * k) + 2 * align256(sizeof(float) * (size_t)r * B) +
             align256(sizeof(float));
  if (tc_update_supported(k)) b += 2 * align256(sizeof(float) * (size_t)k * k);
  return b;
}

static SweepScratch carve_sweep(void* ws, int64_t r, int64_t k, int B, bool tc) {
  char* p = (char*)ws;
  SweepScratch s;
  s.Wt = (float*)p; p += align256(sizeof(float) * (size_t)r * k);
  s.Err = (float*)p; p += align256(sizeof(float) * (size_t)r * B);
  s.Err_lo = (float*)p; p += align256(sizeof(float) * (size_t)r * B);
  s.lambda = (float*)p; p += align256(sizeof(float));
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

template <typename T>
__global__ void sweep_init_kernel(const T* __restrict__ W, int64_t ldw, int r, int k,
                                  const int32_t* __restrict__ perm,
                                  const uint8_t* __restrict__ dead, int G, float* __restrict__ Wt,
                                  int32_t* __restrict__ g_idx, double* __restrict__ loss,
                                  int32_t* __restrict__ d_status) {
  int row = blockIdx.y;
  for (int j = blockIdx.x * blockDim.x + threadIdx.x; j < k; j += gridDim.x * blockDim.x) {
    int c = perm[j];
    float v = dead[c] ? 0.f : to_f32(W[(int64_t)row * ldw + c]);
    Wt[(int64_t)row * k + j] = v;
    if (row == 0) g_idx[c] = j / G;
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
                                  int gidx, int ngroups, float maxq, float* __restrict__ scales,
                                  int32_t* __restrict__ zeros) {
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
    grid_from_range(mn, mx, maxq, sc, z);
    scales[(int64_t)warp * ngroups + gidx] = sc;
    zeros[(int64_t)warp * ngroups + gidx] = (int32_t)z;
  }
}

// One lazy block [s, s + bw) for 32 rows.  Thread (rr = row in CTA, q = lane
// % 4): all four threads of a row run the column chain (identical values, so
// SIMT issues it once); the rank-SB updates of the rest of the block and the
// outputs are split by q.  SB divides the group size when groups are smaller
// than the block, so a group always starts at a sub-block boundary.
template <int SB, typename T>
__global__ void __launch_bounds__(SW_THREADS)
sweep_block_kernel(const float* __restrict__ Wt, float* __restrict__ Err,
                   float* __restrict__ Err_lo, const float* __restrict__ U,
                   const int32_t* __restrict__ perm,
                   const uint8_t* __restrict__ dead, const T* __restrict__ W0, int64_t ldw, int r,
                   int k, int s, int bw, int B, int G, int ngroups, float maxq,
                   const float* __restrict__ lambda, float* __restrict__ scales,
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
  const float lam = (lambda != nullptr) ? *lambda : 0.f;
  double e2 = 0.0, d2 = 0.0;
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
      grid_from_range(mn, mx, maxq, scale, zero);
      if (valid && q == 0) {
        scales[(int64_t)row * ngroups + (s + c0) / G] = scale;
        zeros[(int64_t)row * ngroups + (s + c0) / G] = (int32_t)zero;
      }
    }
    // original weights of the columns this thread reports (ii % 4 == q),
    // fetched before the column chain so their latency overlaps it
    constexpr int NQ = (SB + 3) / 4;
    float w0r[NQ];
#pragma unroll
    for (int u = 0; u < NQ; ++u) {
      const int ii = 4 * u + q;
      w0r[u] = 0.f;
      if (loss != nullptr && valid && ii < SB && c0 + ii < bw) {
        const int oc = pcol[c0 + ii];
        w0r[u] = dead[oc] ? 0.f : to_f32(W0[(int64_t)row * ldw + oc]);
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
          if (loss != nullptr) {
            const double dd = (double)w0r[ii >> 2] - (double)qv;
            d2 += dd * dd;
            e2 += (double)err * (double)err;
          }
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
            Err[(int64_t)row * B + c0 + ii] = h;
            Err_lo[(int64_t)row * B + c0 + ii] = l;
          } else {
            Err[(int64_t)row * B + c0 + ii] = errs[ii];
          }
        }
    }
    __syncwarp();
  }
  if (loss != nullptr) {
    e2 += __shfl_xor_sync(0xffffffffu, e2, 1);
    d2 += __shfl_xor_sync(0xffffffffu, d2, 1);
    e2 += __shfl_xor_sync(0xffffffffu, e2, 2);
    d2 += __shfl_xor_sync(0xffffffffu, d2, 2);
    if (valid && q == 0) atomicAdd(&loss[row], e2 - (double)lam * d2);
  }
  if (nonfinite && valid && d_status != nullptr) atomicCAS(d_status, 0, (int32_t)GPTQ_ERR_NONFINITE);
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

template <int SB, typename T>
static void launch_block(unsigned grid, cudaStream_t s, const float* Wt, float* Err,
                         float* Err_lo, const float* U, const int32_t* perm, const uint8_t* dead, const T* W0,
                         int64_t ldw, int r, int k, int s0, int bw, int B, int G, int ngroups,
                         float maxq, const float* lambda, float* scales, int32_t* zeros,
                         uint8_t* codes, double* loss, int32_t* d_status) {
  static bool attr = false;
  if (!attr) {
    cudaFuncSetAttribute(sweep_block_kernel<SB, T>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                         (int)SW_SMEM);
    attr = true;
  }
  sweep_block_kernel<SB, T><<<grid, SW_THREADS, SW_SMEM, s>>>(
      Wt, Err, Err_lo, U, perm, dead, W0, ldw, r, k, s0, bw, B, G, ngroups, maxq, lambda, scales, zeros,
      codes, loss, d_status);
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
  SweepScratch sc = carve_sweep(ws, r, k, B, tc);
  const bool want_loss = (H0 != nullptr && loss != nullptr);
  double* lossp = want_loss ? loss : nullptr;
  {
    dim3 grid((unsigned)cdiv(k, 1024), (unsigned)r);
    sweep_init_kernel<T><<<grid, 256, 0, s>>>(W, ldw, r, k, perm, dead, G, sc.Wt, g_idx, lossp,
                                              d_status);
    GPTQ_CHECK_LAUNCH();
  }
  if (want_loss) {
    sweep_lambda_kernel<<<1, 1024, 0, s>>>(H0, k, cfg->percdamp, sc.lambda);
    GPTQ_CHECK_LAUNCH();
  }
  if (tc) {
    gptq_status st = tc_split_transpose(U, k, k, k, sc.U_hi, sc.U_lo, k, s);
    if (st != GPTQ_OK) return st;
  }
  // sub-block width: 16, or the largest power of two dividing a smaller group
  int SB = 16;
  if (G < B) {
    SB = 1;
    while (SB < 16 && G % (SB * 2) == 0) SB *= 2;
  }
  const unsigned grid = (unsigned)cdiv(r, SW_ROWS);
  for (int s0 = 0; s0 < k; s0 += B) {
    int bw = min(B, k - s0);
    if (G > B && s0 % G == 0) {
      int gw = min(G, k - s0);
      group_grid_kernel<<<(unsigned)cdiv((int64_t)r * kWarp, 256), 256, 0, s>>>(
          sc.Wt, r, k, s0, gw, s0 / G, ngroups, maxq, scales, zeros);
      GPTQ_CHECK_LAUNCH();
    }
    const float* lam = want_loss ? sc.lambda : nullptr;
#define GPTQ_SWEEP_BLOCK(SBV)                                                                     \
  launch_block<SBV, T>(grid, s, sc.Wt, sc.Err, tc ? sc.Err_lo : nullptr, U, perm, dead, W, ldw, r, k, s0, bw, B, G, ngroups, \
                       maxq, lam, scales, zeros, codes, lossp, d_status)
    switch (SB) {
      case 16: GPTQ_SWEEP_BLOCK(16); break;
      case 8: GPTQ_SWEEP_BLOCK(8); break;
      case 4: GPTQ_SWEEP_BLOCK(4); break;
      case 2: GPTQ_SWEEP_BLOCK(2); break;
      default: GPTQ_SWEEP_BLOCK(1); break;
    }
#undef GPTQ_SWEEP_BLOCK
    GPTQ_CHECK_LAUNCH();
    int e0 = s0 + bw;
    if (e0 < k) {
      if (tc) {
        gptq_status st = tc_sweep_trailing(sc.Err, sc.Err_lo, B, sc.U_hi, sc.U_lo, sc.Wt, r, k,
                                           s0, e0, d_status, s);
        if (st != GPTQ_OK) return st;
      } else {
        sgemm<false, false, false, false, false>(r, k - e0, bw, -1.0f, sc.Err, B,
                                                 U + (int64_t)s0 * k + e0, k, 1.0f, sc.Wt + e0, k,
                                                 nullptr, s);
        GPTQ_CHECK_LAUNCH();
      }
    }
  }
  if (want_loss) {
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
