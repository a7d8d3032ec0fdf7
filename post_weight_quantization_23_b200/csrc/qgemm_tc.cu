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
//   warps 2..9  thread = (weight row, 32-column half of the stage): its 4
//               packed words become 32 weights in the activations' 16-bit
//               type, two at a time: a byte permute and a mask put codes
//               c_2i, c_2i+1 into the mantissas of a half2 holding M + c (M =
//               1024 for f16, 128 for bf16: exact), one packed subtract of
//               M + zero leaves c - zero exactly, one packed multiply by the
//               scale (itself rounded to the type) gives the weight; written
//               as the A operand in the 128-byte-swizzled K-major layout.
//               After the last stage the same warps are the epilogue (TMEM
//               lane = weight row, column = token; two warps per lane quarter
//               split the tokens);
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
constexpr int QT_DQ_WARPS = 8;                        // dequantizing / epilogue warps
constexpr int QT_THREADS = 64 + 32 * QT_DQ_WARPS;     // + TMA and MMA warps
constexpr int QT_TMEM_COLS = 256;
constexpr size_t QT_SMEM = (size_t)QT_STAGES * QT_STAGE_BYTES + 1024 + 256;

struct QtArgs {
  const float* scales;
  const int32_t* zeros;
  void* Y;
  int64_t ldy;
  int n, m, k, G, ngroups;
  uint32_t spin;  // polls before a pipeline wait gives up
};

// The 16-bit activation type T and its packed pair T2.
template <bool BF16> struct QtType;
template <> struct QtType<false> {
  using T = __half;
  using T2 = __half2;
  static constexpr uint32_t MAGIC = 0x64006400u;  // 1024 in both halves: ulp 1 on [1024, 2048)
  static constexpr float BASE = 1024.f;
  __device__ static T2 pair(float v) { return __float2half2_rn(v); }
  __device__ static T out(float v) { return __float2half_rn(v); }
};
template <> struct QtType<true> {
  using T = __nv_bfloat16;
  using T2 = __nv_bfloat162;
  static constexpr uint32_t MAGIC = 0x43004300u;  // 128 in both halves: ulp 1 on [128, 256)
  static constexpr float BASE = 128.f;
  __device__ static T2 pair(float v) { return __float2bfloat162_rn(v); }
  __device__ static T out(float v) { return __float2bfloat16_rn(v); }
};

template <typename T2> __device__ __forceinline__ T2 as_t2(uint32_t u) {
  return *reinterpret_cast<T2*>(&u);
}
template <typename T2> __device__ __forceinline__ uint32_t as_u32(T2 v) {
  return *reinterpret_cast<uint32_t*>(&v);
}

template <bool BF16>
__global__ void __launch_bounds__(QT_THREADS, 1)
qgemm_tc_kernel(const __grid_constant__ CUtensorMap xmap, const __grid_constant__ CUtensorMap pmap,
                QtArgs a) {
  using Ty = QtType<BF16>;
  using T2 = typename Ty::T2;
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
      tc::mbar_init(&full_a[s], QT_DQ_WARPS);
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
        if (!tc::mbar_wait(&empty[s], ph ^ 1u, abort_flag, a.spin)) { ok = false; break; }
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
      const uint32_t idesc = tc::instr_desc(BF16 ? 1 : 0, QT_M, QT_N, 0, 0);  // both K-major
      for (int kc = 0; kc < nk; ++kc) {
        const int s = kc % QT_STAGES;
        const uint32_t ph = (uint32_t)(kc / QT_STAGES) & 1u;
        if (!tc::mbar_wait(&full_tma[s], ph, abort_flag, a.spin)) break;
        if (!tc::mbar_wait(&full_a[s], ph, abort_flag, a.spin)) break;
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
    // warps 2..9: thread = (tile row = its TMEM lane, 32-column half of each stage)
    const int dq = warp - 2;
    const int quarter = warp & 3;
    const int r = quarter * 32 + lane;
    const int hf = dq >> 2;
    const int row = n0 + r;
    const bool rv = row < a.n;
    const float* srow = a.scales + (int64_t)(rv ? row : 0) * a.ngroups;
    const int32_t* zrow = a.zeros + (int64_t)(rv ? row : 0) * a.ngroups;
    // the grid of this thread's half of stage kc, as (scale, scale) and
    // (M + zero, M + zero) pairs; fetched two stages ahead
    auto fetch = [&](int kc, uint32_t& s2, uint32_t& z2) {
      const int col = kc * QT_K + 32 * hf;
      const bool ok = rv && kc < nk && col < a.k;
      const int g = ok ? col / a.G : 0;
      s2 = as_u32(Ty::pair(ok ? srow[g] : 0.f));
      z2 = as_u32(Ty::pair(Ty::BASE + (ok ? (float)zrow[g] : 0.f)));  // exact
    };
    uint32_t s_c, z_c, s_1, z_1, s_2, z_2;
    fetch(0, s_c, z_c);
    fetch(1, s_1, z_1);
    for (int kc = 0; kc < nk; ++kc) {
      const int s = kc % QT_STAGES;
      const uint32_t ph = (uint32_t)(kc / QT_STAGES) & 1u;
      fetch(kc + 2, s_2, z_2);
      if (!tc::mbar_wait_warp(&full_tma[s], ph, abort_flag, a.spin)) break;
      const uint4 pw = reinterpret_cast<const uint4*>(stage_p(s) + r * 32)[hf];
      const uint32_t words[4] = {pw.x, pw.y, pw.z, pw.w};
      const T2 sc2 = as_t2<T2>(s_c), zz2 = as_t2<T2>(z_c);
      uint8_t* arow = stage_a(s) + r * 128;
#pragma unroll
      for (int wi = 0; wi < 4; ++wi) {
        const uint32_t w = words[wi], w4 = w >> 4;
        uint32_t o[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          // byte i of w (c_2i low) into half 0, byte i of w >> 4 (c_2i+1 low) into half 1
          const uint32_t v = __byte_perm(w, w4, (uint32_t)(i | (i << 4) | ((4 + i) << 8) | (i << 12)));
          const T2 h = as_t2<T2>((v & 0x000F000Fu) | Ty::MAGIC);     // M + c, exact
          o[i] = as_u32(__hmul2(__hsub2(h, zz2), sc2));              // (c - z) exact, times s
        }
        *reinterpret_cast<uint4*>(arow + (((4 * hf + wi) ^ (r & 7)) << 4)) =
            make_uint4(o[0], o[1], o[2], o[3]);
      }
      tc::fence_proxy_async_smem();  // the MMA (async proxy) reads what this thread wrote
      __syncwarp();
      if (lane == 0) tc::mbar_arrive(&full_a[s]);
      s_c = s_1, z_c = z_1, s_1 = s_2, z_1 = z_2;
    }
    // epilogue: this warp's lane quarter, tokens [128 hf, 128 hf + 128)
    const bool ok = tc::mbar_wait_warp(done, 0, abort_flag, a.spin) && !*abort_flag;
    tc::tc_fence_after();
    const uint32_t tbase = tmem + ((uint32_t)(quarter * 32) << 16);
    for (int c = 4 * hf; c < 4 * hf + 4; ++c) {
      float v[32];
      tc::tmem_ld_32x32b_x32(tbase + (uint32_t)(c * 32), v);
      tc::tmem_ld_wait();
      if (!rv) continue;
#pragma unroll
      for (int t = 0; t < 32; ++t) {
        const int tok = t0 + c * 32 + t;
        if (tok < a.m)
          reinterpret_cast<typename Ty::T*>(a.Y)[(int64_t)tok * a.ldy + row] =
              Ty::out(ok ? v[t] : __int_as_float(0x7fc00000));
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


}  // namespace

// The tensor-core path takes 4-bit codes, at least one full K stage (k >= 64),
// groups of whole 32-column runs (or one per row), 16-byte aligned X and
// qweight and an X row stride that is a multiple of 8 elements (the TMA rules).
bool qgemm_tc_supported(const void* X, int64_t ldx, const int32_t* qw, int bits, int64_t k,
                        int G, bool has_gidx) {
  return bits == 4 && !has_gidx && k >= QT_K && (G >= k || G % 32 == 0) && ((uintptr_t)X % 16) == 0 &&
         ((uintptr_t)qw % 16) == 0 && ldx % 8 == 0 && tensormap_encoder() != nullptr;
}

gptq_status qgemm_tc(const void* X, bool bf16, int64_t m, int64_t k, int64_t ldx,
                     const int32_t* qw, const float* scales, const int32_t* zeros, int64_t n,
                     int G, int64_t ngroups, void* Y, int64_t ldy, cudaStream_t s) {
  EncodeTiledFn enc = tensormap_encoder();
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
  if (smem_optin(bf16 ? (const void*)qgemm_tc_kernel<true> : (const void*)qgemm_tc_kernel<false>,
                 QT_SMEM) != cudaSuccess)
    return GPTQ_ERR_CUDA;
  QtArgs a;
  a.scales = scales;
  a.zeros = zeros;
  a.Y = Y;
  a.ldy = ldy;
  a.n = (int)n, a.m = (int)m, a.k = (int)k, a.G = G, a.ngroups = (int)ngroups;
  a.spin = wait_limit();
  const dim3 grid((unsigned)cdiv(n, QT_M), (unsigned)cdiv(m, QT_N));
  if (bf16)
    qgemm_tc_kernel<true><<<grid, QT_THREADS, QT_SMEM, s>>>(xmap, pmap, a);
  else
    qgemm_tc_kernel<false><<<grid, QT_THREADS, QT_SMEM, s>>>(xmap, pmap, a);
  GPTQ_CHECK_LAUNCH();
  return GPTQ_OK;
}

}  // namespace gptq
