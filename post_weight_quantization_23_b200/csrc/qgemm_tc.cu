// The inference product Y = X W_hat^T on the 5th-generation tensor cores,
// for token counts where the multiply, not the weight stream, is the cost
// (prefill): the 4-bit codes are expanded just in time, one 128 x 64 tile at
// a time, into a shared-memory operand of the MMA ("GPTQ",
// ozercemkelahmet.com/tools/gptq: What the output looks like -- the kernel
// dequantizes inside the matrix multiply; "What Is GPTQ?", ai-tldr.dev, How
// it works: each group expanded just in time for the multiply).
//
// One CTA per tile of 128 weight rows x 256 tokens, K in stages of 64:
//   warp 0      TMA: the packed words of the 128 rows (128 x 32 bytes) and
//               the 256 x 64 activation box (128-byte swizzle), one barrier;
//   warps 2..5  thread = weight row: read its 8 packed words, w = s (c - z)
//               in fp32 (exact c - z, one rounding by the scale), rounded
//               once to the activations' type, written as the A operand in
//               the 128-byte-swizzled K-major layout; then, after the last
//               stage, the epilogue (TMEM lane = weight row, column = token);
//   warp 1      one thread issues kind::f16 MMAs D[128 x 256] += A B^T into
//               TMEM (fp32), one commit per stage frees it.
// Rows past n and tokens past m are zero-filled by TMA and not stored.  Every
// wait is bounded; a CTA that gives up drains its own copies and MMAs, frees
// TMEM and writes NaN over its outputs.
#include "common.cuh"
#include "tc_ptx.cuh"

namespace gptq {

namespace {

constexpr int QT_M = 128, QT_N = 256, QT_K = 64;     // weight rows, tokens, K per stage
constexpr int QT_STAGES = 4;
constexpr int QT_A_BYTES = QT_M * QT_K * 2;          // 16 KB dequantized W tile
constexpr int QT_B_BYTES = QT_N * QT_K * 2;          // 32 KB activation tile
constexpr int QT_P_BYTES = QT_M * QT_K / 2;          // 4 KB packed 4-bit tile
constexpr int QT_STAGE_BYTES = QT_A_BYTES + QT_B_BYTES + QT_P_BYTES;  // 52 KB, 1024-aligned
constexpr int QT_THREADS = 192;
constexpr int QT_TMEM_COLS = 256;
constexpr size_t QT_SMEM = (size_t)QT_STAGES * QT_STAGE_BYTES + 1024 + 256;

struct QtArgs {
  const float* scales;
  const int32_t* zeros;
  void* Y;
  int64_t ldy;
  int n, m, k, G, ngroups;
  int bf16;
};

__device__ __forceinline__ uint32_t pack2_f16(float a, float b) {
  uint32_t r;
  asm("cvt.rn.f16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(b), "f"(a));  // a in the low half
  return r;
}
__device__ __forceinline__ uint32_t pack2_bf16(float a, float b) {
  uint32_t r;
  asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(b), "f"(a));
  return r;
}

__global__ void __launch_bounds__(QT_THREADS, 1)
qgemm_tc_kernel(const __grid_constant__ CUtensorMap xmap, const __grid_constant__ CUtensorMap pmap,
                QtArgs a) {
  extern __shared__ uint8_t qt_raw[];
  uint8_t* smem = (uint8_t*)(((uintptr_t)qt_raw + 1023) & ~(uintptr_t)1023);
  uint64_t* bars = (uint64_t*)(smem + QT_STAGES * QT_STAGE_BYTES);
  uint64_t* full_tma = bars;                  // packed + activation boxes landed
  uint64_t* full_a = bars + QT_STAGES;        // the 4 dequant warps wrote the A tile
  uint64_t* empty = bars + 2 * QT_STAGES;     // the stage's MMAs completed
  uint64_t* done = bars + 3 * QT_STAGES;      // all MMAs completed
  uint32_t* tmem_slot = (uint32_t*)(done + 1);
  volatile int* abort_flag = (volatile int*)(tmem_slot + 1);

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int n0 = blockIdx.x * QT_M, t0 = blockIdx.y * QT_N;
  const int nk = (a.k + QT_K - 1) / QT_K;
  auto stage_a = [&](int s) { return smem + (size_t)s * QT_STAGE_BYTES; };
  auto stage_b = [&](int s) { return smem + (size_t)s * QT_STAGE_BYTES + QT_A_BYTES; };
  auto stage_p = [&](int s) { return smem + (size_t)s * QT_STAGE_BYTES + QT_A_BYTES + QT_B_BYTES; };

  if (threadIdx.x == 0) {
    for (int s = 0; s < QT_STAGES; ++s) {
      tc::mbar_init(&full_tma[s], 1);
      tc::mbar_init(&full_a[s], 4);
      tc::mbar_init(&empty[s], 1);
    }
    tc::mbar_init(done, 1);
    *abort_flag = 0;
    tc::fence_barrier_init();
    tc::prefetch_tensormap(&xmap);
    tc::prefetch_tensormap(&pmap);
  }
  if (warp == 1) tc::tmem_alloc(tmem_slot, QT_TMEM_COLS);
  tc::tc_fence_before();
  __syncthreads();
  tc::tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    if (lane == 0) {
      bool ok = true;
      int issued = 0;
      for (int kc = 0; kc < nk && ok; ++kc) {
        const int s = kc % QT_STAGES;
        const uint32_t ph = (uint32_t)(kc / QT_STAGES) & 1u;
        if (!tc::mbar_wait(&empty[s], ph ^ 1u, abort_flag)) { ok = false; break; }
        tc::mbar_arrive_expect_tx(&full_tma[s], QT_P_BYTES + QT_B_BYTES);
        tc::tma_load_2d(stage_p(s), &pmap, &full_tma[s], kc * (QT_K / 8), n0);
        tc::tma_load_2d(stage_b(s), &xmap, &full_tma[s], kc * QT_K, t0);
        issued = kc + 1;
      }
      if (!ok) {  // let the copies in flight land before the CTA exits
        for (int kc = issued - QT_STAGES < 0 ? 0 : issued - QT_STAGES; kc < issued; ++kc)
          for (uint32_t i = 0; i < tc::kSpinLimit; ++i)
            if (tc::mbar_try_wait(&full_tma[kc % QT_STAGES], (uint32_t)(kc / QT_STAGES) & 1u))
              break;
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      const uint32_t idesc = tc::instr_desc(a.bf16 ? 1 : 0, QT_M, QT_N, 0, 0);  // both K-major
      for (int kc = 0; kc < nk; ++kc) {
        const int s = kc % QT_STAGES;
        const uint32_t ph = (uint32_t)(kc / QT_STAGES) & 1u;
        if (!tc::mbar_wait(&full_tma[s], ph, abort_flag)) break;
        if (!tc::mbar_wait(&full_a[s], ph, abort_flag)) break;
        tc::tc_fence_after();
        const uint32_t sa = tc::smem_u32(stage_a(s)), sb = tc::smem_u32(stage_b(s));
#pragma unroll
        for (int kk = 0; kk < QT_K / 16; ++kk) {
          // K-major, 128-byte swizzle: 8-row groups 1024 B apart, K step of 16 = 32 B
          const uint64_t da = tc::smem_desc_sw128(sa + kk * 32, 16, 1024);
          const uint64_t db = tc::smem_desc_sw128(sb + kk * 32, 16, 1024);
          tc::mma_f16_ss(tmem, da, db, idesc, (kc > 0 || kk > 0) ? 1u : 0u);
        }
        tc::mma_commit(&empty[s]);
      }
      tc::mma_commit(done);  // also after a give-up: fires once the issued MMAs finish
    }
  } else {
    // warps 2..5: thread = tile row (= its TMEM lane in the epilogue)
    const int quarter = warp & 3;
    const int r = quarter * 32 + lane;
    const int row = n0 + r;
    const bool rv = row < a.n;
    const float* srow = a.scales + (int64_t)(rv ? row : 0) * a.ngroups;
    const int32_t* zrow = a.zeros + (int64_t)(rv ? row : 0) * a.ngroups;
    // the grids of a stage's two 32-column halves (a group holds whole
    // halves), fetched one stage ahead so no load waits inside the loop
    auto fetch = [&](int kc, float (&sc)[2], float (&zb)[2]) {
#pragma unroll
      for (int hf = 0; hf < 2; ++hf) {
        const int col = kc * QT_K + 32 * hf;
        const bool ok = rv && kc < nk && col < a.k;
        const int g = ok ? col / a.G : 0;
        sc[hf] = ok ? srow[g] : 0.f;
        zb[hf] = 8388608.f + (ok ? (float)zrow[g] : 0.f);  // 2^23 + zero, exact
      }
    };
    float sc[2], zb[2], sc_n[2], zb_n[2];
    fetch(0, sc, zb);
    for (int kc = 0; kc < nk; ++kc) {
      const int s = kc % QT_STAGES;
      const uint32_t ph = (uint32_t)(kc / QT_STAGES) & 1u;
      fetch(kc + 1, sc_n, zb_n);
      if (!tc::mbar_wait(&full_tma[s], ph, abort_flag)) break;
      const uint4* pr = reinterpret_cast<const uint4*>(stage_p(s) + r * 32);
      const uint4 p0 = pr[0], p1 = pr[1];
      const uint32_t words[8] = {p0.x, p0.y, p0.z, p0.w, p1.x, p1.y, p1.z, p1.w};
      uint8_t* arow = stage_a(s) + r * 128;
#pragma unroll
      for (int wi = 0; wi < 8; ++wi) {
        const float s_w = sc[wi / 4], zb_w = zb[wi / 4];
        float w[8];
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          // 2^23 + c exactly, minus 2^23 + zero: c - zero exactly; times the scale
          const float f = __uint_as_float(0x4B000000u | ((words[wi] >> (4 * j)) & 0xFu));
          w[j] = (f - zb_w) * s_w;
        }
        uint4 o;
        if (a.bf16) {
          o = make_uint4(pack2_bf16(w[0], w[1]), pack2_bf16(w[2], w[3]), pack2_bf16(w[4], w[5]),
                         pack2_bf16(w[6], w[7]));
        } else {
          o = make_uint4(pack2_f16(w[0], w[1]), pack2_f16(w[2], w[3]), pack2_f16(w[4], w[5]),
                         pack2_f16(w[6], w[7]));
        }
        *reinterpret_cast<uint4*>(arow + ((wi ^ (r & 7)) << 4)) = o;
      }
      tc::fence_proxy_async_smem();  // the MMA (async proxy) reads what this thread wrote
      __syncwarp();
      if (lane == 0) tc::mbar_arrive(&full_a[s]);
#pragma unroll
      for (int hf = 0; hf < 2; ++hf) sc[hf] = sc_n[hf], zb[hf] = zb_n[hf];
    }
    // epilogue
    const bool ok = tc::mbar_wait(done, 0, abort_flag) && !*abort_flag;
    tc::tc_fence_after();
    const uint32_t tbase = tmem + ((uint32_t)(quarter * 32) << 16);
    for (int c = 0; c < QT_N / 32; ++c) {
      float v[32];
      tc::tmem_ld_32x32b_x32(tbase + (uint32_t)(c * 32), v);
      tc::tmem_ld_wait();
      if (!rv) continue;
#pragma unroll
      for (int t = 0; t < 32; ++t) {
        const int tok = t0 + c * 32 + t;
        if (tok < a.m) {
          const float y = ok ? v[t] : __int_as_float(0x7fc00000);
          if (a.bf16)
            reinterpret_cast<__nv_bfloat16*>(a.Y)[(int64_t)tok * a.ldy + row] =
                __float2bfloat16_rn(y);
          else
            reinterpret_cast<__half*>(a.Y)[(int64_t)tok * a.ldy + row] = __float2half_rn(y);
        }
      }
    }
  }
  // a give-up anywhere: wait (bounded) for every MMA this CTA issued before freeing TMEM
  if (warp == 1 && lane == 0 && *abort_flag)
    for (uint32_t i = 0; i < tc::kSpinLimit; ++i)
      if (tc::mbar_try_wait(done, 0)) break;
  tc::tc_fence_before();
  __syncthreads();
  tc::tc_fence_after();
  if (warp == 1) tc::tmem_dealloc(tmem, QT_TMEM_COLS);
}

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn qt_encode_fn() {
  static EncodeTiledFn fn = nullptr;
  if (fn == nullptr) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = (EncodeTiledFn)p;
  }
  return fn;
}

}  // namespace

// The tensor-core path takes 4-bit codes, groups of whole 32-column runs (or
// one per row), 16-byte aligned X and qweight and an X row stride that is a
// multiple of 8 elements (the TMA rules).
bool qgemm_tc_supported(const void* X, int64_t ldx, const int32_t* qw, int bits, int64_t k,
                        int G, bool has_gidx) {
  return bits == 4 && !has_gidx && (G >= k || G % 32 == 0) && ((uintptr_t)X % 16) == 0 &&
         ((uintptr_t)qw % 16) == 0 && ldx % 8 == 0 && qt_encode_fn() != nullptr;
}

gptq_status qgemm_tc(const void* X, bool bf16, int64_t m, int64_t k, int64_t ldx,
                     const int32_t* qw, const float* scales, const int32_t* zeros, int64_t n,
                     int G, int64_t ngroups, void* Y, int64_t ldy, cudaStream_t s) {
  EncodeTiledFn enc = qt_encode_fn();
  if (enc == nullptr) return GPTQ_ERR_CUDA;
  CUtensorMap xmap, pmap;
  {
    cuuint64_t gdim[2] = {(cuuint64_t)k, (cuuint64_t)m};
    cuuint64_t gstride[1] = {(cuuint64_t)ldx * 2};
    cuuint32_t box[2] = {QT_K, QT_N};
    cuuint32_t es[2] = {1, 1};
    if (enc(&xmap, bf16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2,
            const_cast<void*>(X), gdim, gstride, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE,
            CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return GPTQ_ERR_CUDA;
  }
  {
    cuuint64_t gdim[2] = {(cuuint64_t)(k / 8), (cuuint64_t)n};
    cuuint64_t gstride[1] = {(cuuint64_t)(k / 8) * 4};
    cuuint32_t box[2] = {QT_K / 8, QT_M};
    cuuint32_t es[2] = {1, 1};
    if (enc(&pmap, CU_TENSOR_MAP_DATA_TYPE_INT32, 2, const_cast<int32_t*>(qw), gdim, gstride, box,
            es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return GPTQ_ERR_CUDA;
  }
  static bool attr = false;
  if (!attr) {
    if (cudaFuncSetAttribute(qgemm_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)QT_SMEM) != cudaSuccess)
      return GPTQ_ERR_CUDA;
    attr = true;
  }
  QtArgs a;
  a.scales = scales;
  a.zeros = zeros;
  a.Y = Y;
  a.ldy = ldy;
  a.n = (int)n, a.m = (int)m, a.k = (int)k, a.G = G, a.ngroups = (int)ngroups;
  a.bf16 = bf16 ? 1 : 0;
  const dim3 grid((unsigned)cdiv(n, QT_M), (unsigned)cdiv(m, QT_N));
  qgemm_tc_kernel<<<grid, QT_THREADS, QT_SMEM, s>>>(xmap, pmap, a);
  GPTQ_CHECK_LAUNCH();
  return GPTQ_OK;
}

}  // namespace gptq
