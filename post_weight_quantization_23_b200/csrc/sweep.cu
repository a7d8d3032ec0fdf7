// Lazy-blocked GPTQ column sweep ([GPTQ-tool] "GPTQ" How it works Steps 5, 7
// and 8; A minimal Python sketch; [What-is-GPTQ] Step 3 groups).
//
// Rows of W are independent given U, so the sweep is parallel over rows and
// sequential over columns.  Per lazy block [s, e) of processing-order columns:
//   (group kernel)  when a group starts at s and is wider than the block, its
//                   per-row grid comes from the row's current weights;
//   (block kernel)  one lane per row, the block's slice of the row in shared
//                   memory: group grids that start inside the block, codes,
//                   err = (w - q) / U[i][i], in-block compensation, Err out;
//   (trailing)      W[:, e:] -= Err * U[s:e, e:]  (fp32 GEMM).
// The fp32 working copy Wt (processing order) lives in the workspace.
#include "common.cuh"
#include "sgemm.cuh"

namespace gptq {

constexpr int SW_MAX_B = 128;

struct SweepScratch {
  float* Wt;   // [r * k] working weights, processing order
  float* Err;  // [r * B]
  float* D;    // [r * k] w0 - q in original order (loss)
};

size_t sweep_workspace_bytes(int64_t r, int64_t k, int B) {
  return align256(sizeof(float) * (size_t)r * k) + align256(sizeof(float) * (size_t)r * B) +
         align256(sizeof(float) * (size_t)r * k);
}

static SweepScratch carve_sweep(void* ws, int64_t r, int64_t k, int B) {
  char* p = (char*)ws;
  SweepScratch s;
  s.Wt = (float*)p; p += align256(sizeof(float) * (size_t)r * k);
  s.Err = (float*)p; p += align256(sizeof(float) * (size_t)r * B);
  s.D = (float*)p;
  return s;
}

// Wt[row][j] = dead[perm[j]] ? 0 : W[row][perm[j]];  g_idx[perm[j]] = j / G.
template <typename T>
__global__ void sweep_init_kernel(const T* __restrict__ W, int64_t ldw, int r, int k,
                                  const int32_t* __restrict__ perm,
                                  const uint8_t* __restrict__ dead, int G, float* __restrict__ Wt,
                                  int32_t* __restrict__ g_idx, int32_t* __restrict__ d_status) {
  int row = blockIdx.y;
  for (int j = blockIdx.x * blockDim.x + threadIdx.x; j < k; j += gridDim.x * blockDim.x) {
    int c = perm[j];
    float v = dead[c] ? 0.f : to_f32(W[(int64_t)row * ldw + c]);
    Wt[(int64_t)row * k + j] = v;
    if (row == 0) g_idx[c] = j / G;
  }
  if (row == 0 && blockIdx.x == 0 && threadIdx.x == 0 && d_status != nullptr) *d_status = 0;
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

// One lazy block for 32 rows (one warp per CTA).
template <typename T>
__global__ void __launch_bounds__(32)
sweep_block_kernel(float* __restrict__ Wt, float* __restrict__ Err, const float* __restrict__ U,
                   const int32_t* __restrict__ perm, const T* __restrict__ W0, int64_t ldw, int r,
                   int k, int s, int bw, int B, int G, int ngroups, float maxq,
                   float* __restrict__ scales, int32_t* __restrict__ zeros,
                   uint8_t* __restrict__ codes, float* __restrict__ D,
                   int32_t* __restrict__ d_status) {
  __shared__ float sW[SW_MAX_B][33];
  __shared__ float sE[SW_MAX_B][33];
  const int lane = threadIdx.x;
  const int r0 = blockIdx.x * 32;
  const int row = r0 + lane;
  const bool valid = row < r;
  // cooperative, row-contiguous load of the block slice
  for (int rr = 0; rr < 32; ++rr) {
    int gr = r0 + rr;
    for (int j = lane; j < bw; j += 32) sW[j][rr] = (gr < r) ? Wt[(int64_t)gr * k + s + j] : 0.f;
  }
  __syncwarp();
  float scale = 1.f, zero = 0.f;
  bool nonfinite = false;
  if (G > B) {  // group started at or before s and spans the block
    int g = s / G;
    if (valid) {
      scale = scales[(int64_t)row * ngroups + g];
      zero = (float)zeros[(int64_t)row * ngroups + g];
    }
  }
  for (int i = 0; i < bw; ++i) {
    const int gi = s + i;
    if (G <= B && gi % G == 0) {
      int gw = min(G, bw - i);
      float mn = INFINITY, mx = -INFINITY;
      for (int j = 0; j < gw; ++j) {
        float v = sW[i + j][lane];
        mn = fminf(mn, v);
        mx = fmaxf(mx, v);
      }
      grid_from_range(mn, mx, maxq, scale, zero);
      if (valid) {
        scales[(int64_t)row * ngroups + gi / G] = scale;
        zeros[(int64_t)row * ngroups + gi / G] = (int32_t)zero;
      }
    }
    float w = sW[i][lane];
    float c;
    if (isfinite(w)) {
      c = quant_code(w, scale, zero, maxq);
    } else {
      nonfinite = true;
      c = zero;
    }
    float q = scale * (c - zero);
    float err = (w - q) / U[(int64_t)gi * k + gi];
    sE[i][lane] = err;
    if (valid) {
      int oc = perm[gi];
      codes[(int64_t)row * k + oc] = (uint8_t)c;
      if (D != nullptr) D[(int64_t)row * k + oc] = to_f32(W0[(int64_t)row * ldw + oc]) - q;
    }
    const float* urow = U + (int64_t)gi * k + s;
    for (int j = i + 1; j < bw; ++j) sW[j][lane] = fmaf(-err, __ldg(urow + j), sW[j][lane]);
  }
  __syncwarp();
  for (int rr = 0; rr < 32; ++rr) {
    int gr = r0 + rr;
    if (gr < r)
      for (int j = lane; j < bw; j += 32) Err[(int64_t)gr * B + j] = sE[j][rr];
  }
  if (nonfinite && valid && d_status != nullptr) atomicCAS(d_status, 0, (int32_t)GPTQ_ERR_NONFINITE);
}

// loss[row] = sum_c Y[row][c] * D[row][c] (fp64), one warp per row.
__global__ void rowdot_kernel(const float* __restrict__ Y, const float* __restrict__ D, int r,
                              int k, double* __restrict__ loss) {
  int warp = (blockIdx.x * blockDim.x + threadIdx.x) / kWarp;
  int lane = threadIdx.x % kWarp;
  if (warp >= r) return;
  double acc = 0.0;
  for (int c = lane; c < k; c += kWarp)
    acc += (double)Y[(int64_t)warp * k + c] * (double)D[(int64_t)warp * k + c];
  for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
  if (lane == 0) loss[warp] = acc;
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
  SweepScratch sc = carve_sweep(ws, r, k, B);
  const bool want_loss = (H0 != nullptr && loss != nullptr);
  {
    dim3 grid((unsigned)cdiv(k, 1024), (unsigned)r);
    sweep_init_kernel<T><<<grid, 256, 0, s>>>(W, ldw, r, k, perm, dead, G, sc.Wt, g_idx, d_status);
    GPTQ_CHECK_LAUNCH();
  }
  for (int s0 = 0; s0 < k; s0 += B) {
    int bw = min(B, k - s0);
    if (G > B && s0 % G == 0) {
      int gw = min(G, k - s0);
      group_grid_kernel<<<(unsigned)cdiv((int64_t)r * kWarp, 256), 256, 0, s>>>(
          sc.Wt, r, k, s0, gw, s0 / G, ngroups, maxq, scales, zeros);
      GPTQ_CHECK_LAUNCH();
    }
    sweep_block_kernel<T><<<(unsigned)cdiv(r, 32), 32, 0, s>>>(
        sc.Wt, sc.Err, U, perm, W, ldw, r, k, s0, bw, B, G, ngroups, maxq, scales, zeros, codes,
        want_loss ? sc.D : nullptr, d_status);
    GPTQ_CHECK_LAUNCH();
    int e0 = s0 + bw;
    if (e0 < k) {
      sgemm<false, false, false, false, false>(r, k - e0, bw, -1.0f, sc.Err, B, U + (int64_t)s0 * k + e0, k,
                                 1.0f, sc.Wt + e0, k, nullptr, s);
      GPTQ_CHECK_LAUNCH();
    }
  }
  if (want_loss) {
    // Y = D * H0 into the (now free) working copy, then per-row dot with D.
    sgemm<false, false, false, false, false>(r, k, k, 1.0f, sc.D, k, H0, k, 0.0f, sc.Wt, k, nullptr, s);
    GPTQ_CHECK_LAUNCH();
    rowdot_kernel<<<(unsigned)cdiv((int64_t)r * kWarp, 256), 256, 0, s>>>(sc.Wt, sc.D, r, k, loss);
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
