// Hessian accumulation on the 5th-generation tensor cores (sm_100a):
//   H += alpha * X^T X,  X (n, k) row-major f16 / bf16, H (k, k) fp32.
// [GPTQ-tool] "GPTQ" How it works Step 3 and the sketch (H = 2 X^T X / n).
//
// Both MMA operands are column panels of the same row-major X, i.e. MN-major
// tiles: A = X[t0:t0+64, i0:i0+128]^T (M = 128 features), B = X[t0:t0+64,
// j0:j0+256] (N = 256 features), K = tokens.  TMA brings 64-token x 64-feature
// boxes (128-byte swizzle) into a 4-stage shared-memory ring; one thread issues
// tcgen05.mma (kind::f16, fp32 accumulate in TMEM); eight epilogue warps drain
// the accumulator.
//
// Only tiles that reach the upper triangle are computed (j0 + 256 > i0); for
// tiles on the diagonal A is a sub-panel of B and is not loaded twice.
//
// Accuracy: the tensor core accumulates at most 256 tokens (16 MMAs) in TMEM;
// the epilogue then adds that partial into fp32 registers (TMEM is double
// buffered, so the next 256 tokens accumulate meanwhile) and flushes the
// register sum into H once per unit of up to 65536 tokens, by TMA reduce-adds
// of 32 x 32 chunks staged through one shared-memory slot per epilogue warp.
// A plain fp32 running sum over all n tokens would miss the 1e-5 relative
// Frobenius target at n = 262144.
//
// Work units are (tile, token chunk) pairs taken token-major, strided over a
// persistent grid of one CTA per SM, so all CTAs stream through the same
// token rows of X at the same time; tiles are numbered in blocks (see
// decode_tile) so that the CTAs of one wave share their feature panels.
//
// Every mbarrier wait is bounded.  If one gives up, the CTA stops, waits for
// its own copies and MMAs in flight, frees TMEM and raises a flag in the
// workspace; the mirror pass then sets the caller's status word (the
// workspace's second int32) to GPTQ_ERR_TIMEOUT and writes NaN into H[0][0],
// so that a caller who never reads the word still sees the failure in the next
// stage (the Cholesky in gptq_prepare_hinv).
#include "common.cuh"
#include "tc_ptx.cuh"

namespace gptq {

__global__ void mirror_upper_kernel(float* __restrict__ H, int k, int32_t* status);

namespace {

constexpr int HT_M = 128, HT_N = 256, HT_KT = 64;       // tile rows, cols, tokens per stage
constexpr int HT_STAGES = 4;
constexpr int HT_SUB_STAGES = 4;                        // stages per TMEM partial (256 tokens)
constexpr int HT_BOX_BYTES = 64 * 64 * 2;               // one 64x64 16-bit box
constexpr int HT_B_BYTES = 4 * HT_BOX_BYTES;            // 32 KB
constexpr int HT_A_BYTES = 2 * HT_BOX_BYTES;            // 16 KB
constexpr int HT_STAGE_BYTES = HT_B_BYTES + HT_A_BYTES; // 48 KB
constexpr int HT_THREADS = 320;                         // TMA warp, MMA warp, 8 epilogue warps
constexpr int HT_TMEM_COLS = 512;                       // 2 accumulators x 256 columns
constexpr int HT_MAX_CHUNK = 65536;
constexpr int HT_SLOT_BYTES = 32 * 32 * 4;              // one warp's 32 x 32 flush chunk
constexpr int HT_EPI_WARPS = 8;
constexpr size_t HT_SMEM = (size_t)HT_STAGES * HT_STAGE_BYTES +
                           (size_t)HT_EPI_WARPS * HT_SLOT_BYTES + 1024 + 256;

struct HtArgs {
  int k;
  int64_t n;
  int nI, nJ, ntiles;
  int64_t chunk;
  int64_t nunits;
  float alpha;
  float* H;
  int32_t* status;
  uint32_t spin;  // polls before a pipeline wait gives up
};

// Tiles (I, J) reaching the upper triangle: J >= I / 2 (rows of 128, columns
// of 256).  They are numbered block by block, blocks of HT_BI x HT_BJ tiles in
// row-major block order, so that the CTAs running at the same time work on one
// block: together they read HT_BI * 128 + HT_BJ * 256 = 4096 features of each
// token row, which L2 keeps while the token range is streamed (numbering the
// tiles row by row made each wave read whole rows, and wide layers read X from
// DRAM once per wave).
constexpr int HT_BI = 16, HT_BJ = 8;

__device__ __forceinline__ int tiles_in_row(int I, int J0, int J1, int nJ) {
  const int lo = max(J0, I / 2), hi = min(J1, nJ);
  return hi > lo ? hi - lo : 0;
}

__device__ __forceinline__ void decode_tile(int t, int nI, int nJ, int& I, int& J) {
  const int nbI = (nI + HT_BI - 1) / HT_BI, nbJ = (nJ + HT_BJ - 1) / HT_BJ;
  for (int bi = 0; bi < nbI; ++bi) {
    const int I0 = bi * HT_BI, I1 = min(nI, I0 + HT_BI);
    for (int bj = 0; bj < nbJ; ++bj) {
      const int J0 = bj * HT_BJ, J1 = J0 + HT_BJ;
      if (J1 <= I0 / 2) continue;  // block entirely below the triangle
      for (int i = I0; i < I1; ++i) {
        const int cnt = tiles_in_row(i, J0, J1, nJ);
        if (t < cnt) {
          I = i;
          J = max(J0, i / 2) + t;
          return;
        }
        t -= cnt;
      }
    }
  }
  I = nI;  // past the last tile (never reached for t < ntiles)
  J = nJ;
}

__global__ void __launch_bounds__(HT_THREADS, 1)
hessian_tc_kernel(const __grid_constant__ CUtensorMap xmap, const __grid_constant__ CUtensorMap hmap,
                  HtArgs a, int fmt_bf16) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  uint8_t* stages = smem;
  uint8_t* slots = smem + HT_STAGES * HT_STAGE_BYTES;  // [8] flush chunks, 1024-byte aligned
  uint64_t* bars = (uint64_t*)(slots + HT_EPI_WARPS * HT_SLOT_BYTES);
  uint64_t* full = bars;                      // [HT_STAGES]
  uint64_t* empty = bars + HT_STAGES;         // [HT_STAGES]
  uint64_t* tfull = bars + 2 * HT_STAGES;     // [2]
  uint64_t* tempty = bars + 2 * HT_STAGES + 2;  // [2]
  uint64_t* done = bars + 2 * HT_STAGES + 4;  // [1]
  uint32_t* tmem_slot = (uint32_t*)(bars + 2 * HT_STAGES + 5);
  volatile int* abort_flag = (volatile int*)(tmem_slot + 1);

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  if (threadIdx.x == 0) {
    for (int s = 0; s < HT_STAGES; ++s) {
      tc::mbar_init(&full[s], 1);
      tc::mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      tc::mbar_init(&tfull[b], 1);
      tc::mbar_init(&tempty[b], 8);
    }
    tc::mbar_init(done, 1);
    *abort_flag = 0;
    tc::fence_barrier_init();
    tc::prefetch_tensormap(&xmap);
    tc::prefetch_tensormap(&hmap);
  }
  if (warp == 1) tc::tmem_alloc(tmem_slot, HT_TMEM_COLS);
  tc::tc_fence_before();
  __syncthreads();
  tc::tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  const uint32_t idesc = tc::instr_desc(fmt_bf16 ? 1 : 0, HT_M, HT_N, 1, 1);

  if (warp == 0) {
    // ---------------- TMA producer ----------------
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      uint32_t issued_parity[HT_STAGES];
      bool issued[HT_STAGES];
      for (int s = 0; s < HT_STAGES; ++s) issued[s] = false, issued_parity[s] = 0;
      bool ok = true;
      for (int64_t u = blockIdx.x; u < a.nunits && ok; u += gridDim.x) {
        const int t = (int)(u % a.ntiles);
        const int64_t c = u / a.ntiles;
        int I, J;
        decode_tile(t, a.nI, a.nJ, I, J);
        const int i0 = I * HT_M, j0 = J * HT_N;
        const bool a_in_b = (i0 >= j0) && (i0 < j0 + HT_N);
        const int64_t t_beg = c * a.chunk;
        const int64_t t_end = min(a.n, t_beg + a.chunk);
        const int nst = (int)((t_end - t_beg + HT_KT - 1) / HT_KT);
        for (int st = 0; st < nst; ++st) {
          if (!tc::mbar_wait(&empty[stage], phase ^ 1u, abort_flag, a.spin)) { ok = false; break; }
          uint8_t* sb = stages + (size_t)stage * HT_STAGE_BYTES;
          tc::mbar_arrive_expect_tx(&full[stage], a_in_b ? HT_B_BYTES : HT_STAGE_BYTES);
          const int32_t tok = (int32_t)(t_beg + (int64_t)st * HT_KT);
#pragma unroll
          for (int q = 0; q < 4; ++q)
            tc::tma_load_2d(sb + q * HT_BOX_BYTES, &xmap, &full[stage], j0 + q * 64, tok);
          if (!a_in_b) {
#pragma unroll
            for (int q = 0; q < 2; ++q)
              tc::tma_load_2d(sb + HT_B_BYTES + q * HT_BOX_BYTES, &xmap, &full[stage],
                              i0 + q * 64, tok);
          }
          issued[stage] = true;
          issued_parity[stage] = phase;
          if (++stage == HT_STAGES) stage = 0, phase ^= 1u;
        }
      }
      if (!ok || *abort_flag) {
        // let every copy this thread issued land before the CTA goes away
        for (int s = 0; s < HT_STAGES; ++s)
          if (issued[s]) {
            for (uint32_t i = 0; i < tc::kSpinLimit; ++i)
              if (tc::mbar_try_wait(&full[s], issued_parity[s])) break;
          }
      }
    }
  } else if (warp == 1) {
    // ---------------- MMA issuer ----------------
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      int tb = 0;
      uint32_t tphase = 0;
      bool ok = true;
      for (int64_t u = blockIdx.x; u < a.nunits && ok; u += gridDim.x) {
        const int t = (int)(u % a.ntiles);
        const int64_t c = u / a.ntiles;
        int I, J;
        decode_tile(t, a.nI, a.nJ, I, J);
        const int i0 = I * HT_M, j0 = J * HT_N;
        const bool a_in_b = (i0 >= j0) && (i0 < j0 + HT_N);
        const int64_t t_beg = c * a.chunk;
        const int64_t t_end = min(a.n, t_beg + a.chunk);
        const int nst = (int)((t_end - t_beg + HT_KT - 1) / HT_KT);
        for (int s0 = 0; s0 < nst && ok; s0 += HT_SUB_STAGES) {
          if (!tc::mbar_wait(&tempty[tb], tphase ^ 1u, abort_flag, a.spin)) { ok = false; break; }
          tc::tc_fence_after();
          const uint32_t dcol = tmem + (uint32_t)(tb * HT_N);
          const int s1 = min(nst, s0 + HT_SUB_STAGES);
          for (int st = s0; st < s1; ++st) {
            if (!tc::mbar_wait(&full[stage], phase, abort_flag, a.spin)) { ok = false; break; }
            tc::tc_fence_after();
            const uint32_t sb = tc::smem_u32(stages + (size_t)stage * HT_STAGE_BYTES);
            const uint32_t a_base = a_in_b ? sb + (uint32_t)((i0 - j0) / 64) * HT_BOX_BYTES
                                           : sb + HT_B_BYTES;
#pragma unroll
            for (int kk = 0; kk < HT_KT / 16; ++kk) {
              const uint64_t ad = tc::smem_desc_sw128(a_base + kk * 2048, HT_BOX_BYTES, 1024);
              const uint64_t bd = tc::smem_desc_sw128(sb + kk * 2048, HT_BOX_BYTES, 1024);
              tc::mma_f16_ss(dcol, ad, bd, idesc, (st > s0 || kk > 0) ? 1u : 0u);
            }
            tc::mma_commit(&empty[stage]);
            if (++stage == HT_STAGES) stage = 0, phase ^= 1u;
          }
          if (!ok) break;
          tc::mma_commit(&tfull[tb]);
          if (++tb == 2) tb = 0, tphase ^= 1u;
        }
      }
      // all MMAs issued by this thread have completed once `done` flips
      tc::mma_commit(done);
      for (uint32_t i = 0; i < tc::kSpinLimit; ++i)
        if (tc::mbar_try_wait(done, 0)) break;
    }
  } else {
    // ---------------- epilogue: 8 warps ----------------
    const int ew = warp - 2;
    const int quarter = warp & 3;        // TMEM lane quarter this warp may access
    const int half = ew >> 2;            // column half of the 256-wide tile
    int tb = 0;
    uint32_t tphase = 0;
    bool ok = true;
    for (int64_t u = blockIdx.x; u < a.nunits && ok; u += gridDim.x) {
      const int t = (int)(u % a.ntiles);
      const int64_t c = u / a.ntiles;
      int I, J;
      decode_tile(t, a.nI, a.nJ, I, J);
      const int i0 = I * HT_M, j0 = J * HT_N;
      const int64_t t_beg = c * a.chunk;
      const int64_t t_end = min(a.n, t_beg + a.chunk);
      const int nst = (int)((t_end - t_beg + HT_KT - 1) / HT_KT);
      const int nsub = (nst + HT_SUB_STAGES - 1) / HT_SUB_STAGES;
      float acc[128];
#pragma unroll
      for (int q = 0; q < 128; ++q) acc[q] = 0.f;
      for (int sub = 0; sub < nsub; ++sub) {
        if (!tc::mbar_wait_warp(&tfull[tb], tphase, abort_flag, a.spin)) { ok = false; break; }
        tc::tc_fence_after();
        const uint32_t base =
            tmem + ((uint32_t)(quarter * 32) << 16) + (uint32_t)(tb * HT_N + half * 128);
#pragma unroll
        for (int cc = 0; cc < 4; ++cc) {
          float v[32];
          tc::tmem_ld_32x32b_x32(base + cc * 32, v);
          tc::tmem_ld_wait();
#pragma unroll
          for (int q = 0; q < 32; ++q) acc[cc * 32 + q] += v[q];
        }
        tc::tc_fence_before();
        __syncwarp();
        if (lane == 0) tc::mbar_arrive(&tempty[tb]);
        if (++tb == 2) tb = 0, tphase ^= 1u;
      }
      if (!ok) break;
      // flush: alpha * the unit's sums into H, 32 x 32 chunks reduce-added by
      // TMA (L2 adds them; rows and columns past k are clipped).  Entries
      // below the diagonal are added as well: the mirror pass overwrites them.
      uint8_t* slot = slots + ew * HT_SLOT_BYTES;
      const int jb = j0 + half * 128;
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        if (lane == 0) tc::bulk_wait_read_all();  // the slot's previous reduce has read it
        __syncwarp();
        uint8_t* rowp = slot + lane * 128;
#pragma unroll
        for (int u = 0; u < 8; ++u)
          *(float4*)(rowp + ((u ^ (lane & 7)) << 4)) =
              make_float4(a.alpha * acc[c * 32 + 4 * u], a.alpha * acc[c * 32 + 4 * u + 1],
                          a.alpha * acc[c * 32 + 4 * u + 2], a.alpha * acc[c * 32 + 4 * u + 3]);
        tc::fence_proxy_async_smem();  // the reduce reads what this thread wrote
        __syncwarp();
        if (lane == 0) {
          tc::tma_reduce_add_2d(&hmap, slot, jb + c * 32, i0 + quarter * 32);
          tc::bulk_commit_group();
        }
      }
    }
    if (lane == 0) tc::bulk_wait_all();  // every reduce of this warp has completed
  }

  __syncthreads();
  if (*abort_flag && threadIdx.x == 0) atomicExch(a.status, 1);
  tc::tc_fence_after();
  if (warp == 1) tc::tmem_dealloc(tmem, HT_TMEM_COLS);
}

}  // namespace

bool hessian_tc_supported(gptq_dtype dt, int64_t n, int64_t k, int64_t ldx, const void* X,
                          const float* H) {
  if (dt != GPTQ_F16 && dt != GPTQ_BF16) return false;
  if (k < 64 || k % 8 != 0 || ldx % 8 != 0 || ((uintptr_t)X % 16) != 0) return false;
  if (((uintptr_t)H % 16) != 0) return false;  // H is reduce-added by TMA
  if (n <= 0 || n > ((int64_t)1 << 31) - HT_MAX_CHUNK) return false;
  return tensormap_encoder() != nullptr;
}

size_t hessian_tc_workspace_bytes(int64_t, int64_t) { return 256; }

gptq_status hessian_tc(const void* X, gptq_dtype dt, int64_t n, int64_t k, int64_t ldx,
                       float alpha, float* H, void* ws, cudaStream_t s) {
  EncodeTiledFn enc = tensormap_encoder();
  if (enc == nullptr) return GPTQ_ERR_UNSUPPORTED;
  CUtensorMap map;
  cuuint64_t gdim[2] = {(cuuint64_t)k, (cuuint64_t)n};
  cuuint64_t gstride[1] = {(cuuint64_t)ldx * 2};
  cuuint32_t box[2] = {64, 64};
  cuuint32_t estride[2] = {1, 1};
  CUresult r = enc(&map, dt == GPTQ_BF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16
                                         : CU_TENSOR_MAP_DATA_TYPE_FLOAT16,
                   2, const_cast<void*>(X), gdim, gstride, box, estride,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return GPTQ_ERR_INVALID_ARG;
  CUtensorMap hmap;
  {
    cuuint64_t hdim[2] = {(cuuint64_t)k, (cuuint64_t)k};
    cuuint64_t hstride[1] = {(cuuint64_t)k * 4};
    cuuint32_t hbox[2] = {32, 32};
    if (enc(&hmap, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, H, hdim, hstride, hbox, estride,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return GPTQ_ERR_INVALID_ARG;
  }

  const int nsm = sm_count();
  if (smem_optin((const void*)hessian_tc_kernel, HT_SMEM) != cudaSuccess) return GPTQ_ERR_CUDA;
  HtArgs a;
  a.k = (int)k;
  a.n = n;
  a.nI = (int)cdiv(k, HT_M);
  a.nJ = (int)cdiv(k, HT_N);
  a.ntiles = 0;
  for (int i = 0; i < a.nI; ++i) a.ntiles += max(0, a.nJ - i / 2);
  // token chunk per unit: enough units for ~4 per SM, 256..65536 tokens
  int64_t want = cdiv(n * a.ntiles, 4 * (int64_t)nsm);
  int64_t chunk = cdiv(want, 256) * 256;
  chunk = std::min<int64_t>(std::max<int64_t>(chunk, 256), HT_MAX_CHUNK);
  a.chunk = chunk;
  a.nunits = cdiv(n, chunk) * a.ntiles;
  a.alpha = alpha;
  a.H = H;
  a.status = (int32_t*)ws;
  a.spin = wait_limit();
  // word 0: this call's give-up flag; word 1 (the caller's status) is only ever set
  if (cudaMemsetAsync(ws, 0, sizeof(int32_t), s) != cudaSuccess) return GPTQ_ERR_CUDA;
  const int grid = (int)std::min<int64_t>(a.nunits, nsm);
  hessian_tc_kernel<<<grid, HT_THREADS, HT_SMEM, s>>>(map, hmap, a, dt == GPTQ_BF16 ? 1 : 0);
  GPTQ_CHECK_LAUNCH();
  int nb = (int)cdiv(k, 32);
  mirror_upper_kernel<<<dim3(nb, nb), dim3(32, 8), 0, s>>>(H, (int)k, (int32_t*)ws);
  GPTQ_CHECK_LAUNCH();
  return GPTQ_OK;
}

}  // namespace gptq
