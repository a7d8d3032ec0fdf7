// fp32-accurate short-K updates on the 5th-generation tensor cores:
//   D[row][c] += sum_k R[row][k] C[c][k]                          (K <= 128)
// with every fp32 operand split as x = hi + lo, hi = x rounded to tf32 and
// lo = x - hi (exact), and three kind::tf32 MMAs per K step,
//   A B ~= A_hi B_hi + A_hi B_lo + A_lo B_hi,
// which keeps fp32-level accuracy (the dropped A_lo B_lo term and the tf32
// rounding of lo are ~2^-21 relative).  The splits are written to global
// memory K-major (K contiguous) for both operands -- a transposing split
// where the source is stored the other way -- so TMA brings hi and lo boxes
// straight into shared memory in the 128-byte-swizzled K-major layout.  Any
// sign of the update is folded into the C operand by whoever writes it, so
// the whole tile is a plain D += R C^T.
//
// Two uses:
//   mode 0, lazy-batch trailing update of the GPTQ sweep ([GPTQ-tool]
//     "GPTQ" How it works Step 7): W[:, e:] -= Err * U[s:s+B, e:], with
//     R = Err (rows x B) and C = -U^T (the negated transposed split).
//   mode 1, rank-b update of the inverse factor: rows [0, j0) of the work
//     matrix += R^T S, R = A[j0:j0+b, 0:j0] and S = the row block with its
//     columns c < j0 negated (Schur complement) and c >= j0 kept (Y update);
//     tiles that lie entirely right of the diagonal inside [0, j0)^2 are
//     skipped, the others are updated whole.
//
// Tiles of 128 x 256 (128 x 128 for updates with fewer tiles than SMs) on a
// persistent grid; warp 0 issues the
// operand TMA loads, warp 1 the MMAs (one thread), warps 2..5 are the
// epilogue.  TMEM holds two accumulators, so a tile's epilogue overlaps the
// next tile's MMAs.  D is never read by the kernel: the epilogue writes the
// accumulator of a 128 x 32 chunk into a two-slot shared-memory ring
// (128-byte swizzle, conflict-free) and one thread sends it to D with a TMA
// tensor reduce-add, which L2 applies as D = fl(D + v) and which clips at the
// tensor's extent.  A slot is rewritten once its reduce has read it.  Every
// mbarrier wait is bounded; on a timeout the CTA drains its own copies and
// MMAs, frees TMEM and raises *status.
#include "common.cuh"
#include "tc_ptx.cuh"

namespace gptq {

namespace {

constexpr int TX_M = 128, TX_KC = 32;                // tile rows, K per stage
constexpr int TX_STAGES = 2;
constexpr int TX_A_BYTES = TX_M * TX_KC * 4;         // 16 KB
constexpr int TX_THREADS = 192;                      // TMA, MMA, 4 epilogue warps
constexpr int TX_DC = 32;                             // D chunk columns (one 128-byte row)
constexpr int TX_D_BYTES = TX_M * TX_DC * 4;          // 16 KB per D chunk
constexpr int TX_D_SLOTS = 2;

// Tile width TN = 256 (large updates: more reuse of each operand byte) or 128
// (updates with fewer tiles than SMs: twice the CTAs, half the chain of MMAs
// and epilogue chunks per CTA).
template <int TN>
struct TxTile {
  static constexpr int B_BYTES = TN * TX_KC * 4;                        // 32 / 16 KB
  static constexpr int STAGE_BYTES = 2 * TX_A_BYTES + 2 * B_BYTES;      // hi + lo of both
  static constexpr int TMEM_COLS = 2 * TN;                              // two accumulators
  static constexpr size_t SMEM =
      (size_t)TX_STAGES * STAGE_BYTES + (size_t)TX_D_SLOTS * TX_D_BYTES + 1024 + 256;
};

struct TxArgs {
  float* D;
  int64_t ldd;
  int M, N;        // output extent from (row0, col0)
  int row0, col0;  // output offsets in D
  int K;           // inner extent
  int a_k0, a_r0;  // A map coordinates of (k = 0, output row 0)
  int b_k0, b_r0;  // B map coordinates of (k = 0, output column 0)
  int ntm, ntiles;
  int mode, split;
  int32_t* status;
  int32_t status_code;
  uint32_t spin;  // polls before a pipeline wait gives up
};

template <int TN>
__device__ __forceinline__ bool tile_skipped(const TxArgs& a, int m0, int n0) {
  // mode 1: a tile whose columns all lie in [0, split) and strictly right of
  // the diagonal of its rows (row0 + m0 ...) has nothing the factorisation reads
  return a.mode == 1 && n0 + TN <= a.split && n0 >= a.row0 + m0 + TX_M;
}

// Next tile of this CTA after t (t = -1: the first) that has work, or ntiles.
template <int TN>
__device__ __forceinline__ int next_tile(const TxArgs& a, int t) {
  for (t = (t < 0) ? (int)blockIdx.x : t + (int)gridDim.x; t < a.ntiles; t += gridDim.x) {
    const int m0 = (t % a.ntm) * TX_M, n0 = (t / a.ntm) * TN;
    if (!tile_skipped<TN>(a, m0, n0)) return t;
  }
  return a.ntiles;
}

template <int TN>
__global__ void __launch_bounds__(TX_THREADS, 1)
tf32x3_update_kernel(const __grid_constant__ CUtensorMap a_hi, const __grid_constant__ CUtensorMap a_lo,
                     const __grid_constant__ CUtensorMap b_hi, const __grid_constant__ CUtensorMap b_lo,
                     const __grid_constant__ CUtensorMap d_map, TxArgs a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  uint8_t* ring = smem + TX_STAGES * TxTile<TN>::STAGE_BYTES;  // D chunks, 1024-byte aligned
  uint64_t* bars = (uint64_t*)(ring + TX_D_SLOTS * TX_D_BYTES);
  uint64_t* full = bars;
  uint64_t* empty = bars + TX_STAGES;
  uint64_t* tfull = bars + 2 * TX_STAGES;
  uint64_t* tempty = bars + 2 * TX_STAGES + 2;
  uint64_t* done = bars + 2 * TX_STAGES + 4;
  uint64_t* dfree = bars + 2 * TX_STAGES + 5;     // slot read by its reduce
  uint64_t* dwritten = dfree + TX_D_SLOTS;        // the 4 epilogue warps wrote it
  uint32_t* tmem_slot = (uint32_t*)(dwritten + TX_D_SLOTS);
  volatile int* abort_flag = (volatile int*)(tmem_slot + 1);

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  if (threadIdx.x == 0) {
    for (int s = 0; s < TX_STAGES; ++s) {
      tc::mbar_init(&full[s], 1);
      tc::mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      tc::mbar_init(&tfull[b], 1);
      tc::mbar_init(&tempty[b], 4);
    }
    tc::mbar_init(done, 1);
    for (int d = 0; d < TX_D_SLOTS; ++d) {
      tc::mbar_init(&dfree[d], 1);
      tc::mbar_init(&dwritten[d], 4);  // one arrival per epilogue warp
    }
    *abort_flag = 0;
    tc::fence_barrier_init();
    tc::prefetch_tensormap(&a_hi);
    tc::prefetch_tensormap(&a_lo);
    tc::prefetch_tensormap(&b_hi);
    tc::prefetch_tensormap(&b_lo);
    tc::prefetch_tensormap(&d_map);
  }
  if (warp == 1) tc::tmem_alloc(tmem_slot, TxTile<TN>::TMEM_COLS);
  tc::tc_fence_before();
  __syncthreads();
  tc::tc_fence_after();
  // set-up above overlaps the previous kernel; its outputs are read below
  pdl_wait();
  pdl_trigger();
  const uint32_t tmem = *tmem_slot;
  const int nkc = (a.K + TX_KC - 1) / TX_KC;
  const uint32_t idesc = tc::instr_desc(2, TX_M, TN, 0, 0);  // both operands K-major

  if (warp == 0) {
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      bool issued[TX_STAGES];
      uint32_t issued_parity[TX_STAGES];
      for (int s = 0; s < TX_STAGES; ++s) issued[s] = false, issued_parity[s] = 0;
      bool ok = true;
      for (int t = blockIdx.x; t < a.ntiles && ok; t += gridDim.x) {
        const int m0 = (t % a.ntm) * TX_M, n0 = (t / a.ntm) * TN;
        if (tile_skipped<TN>(a, m0, n0)) continue;
        for (int kc = 0; kc < nkc; ++kc) {
          if (!tc::mbar_wait(&empty[stage], phase ^ 1u, abort_flag, a.spin)) { ok = false; break; }
          uint8_t* sb = smem + (size_t)stage * TxTile<TN>::STAGE_BYTES;
          tc::mbar_arrive_expect_tx(&full[stage], TxTile<TN>::STAGE_BYTES);
          const int k0 = kc * TX_KC;
          tc::tma_load_2d(sb, &a_hi, &full[stage], a.a_k0 + k0, a.a_r0 + m0);
          tc::tma_load_2d(sb + TX_A_BYTES, &a_lo, &full[stage], a.a_k0 + k0, a.a_r0 + m0);
          uint8_t* bb = sb + 2 * TX_A_BYTES;
          tc::tma_load_2d(bb, &b_hi, &full[stage], a.b_k0 + k0, a.b_r0 + n0);
          tc::tma_load_2d(bb + TxTile<TN>::B_BYTES, &b_lo, &full[stage], a.b_k0 + k0, a.b_r0 + n0);
          issued[stage] = true;
          issued_parity[stage] = phase;
          if (++stage == TX_STAGES) stage = 0, phase ^= 1u;
        }
      }
      if (!ok || *abort_flag) {
        for (int s = 0; s < TX_STAGES; ++s)
          if (issued[s])
            for (uint32_t i = 0; i < tc::kSpinLimit; ++i)
              if (tc::mbar_try_wait(&full[s], issued_parity[s])) break;
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      int tb = 0;
      uint32_t tphase = 0;
      bool ok = true;
      for (int t = blockIdx.x; t < a.ntiles && ok; t += gridDim.x) {
        const int m0 = (t % a.ntm) * TX_M, n0 = (t / a.ntm) * TN;
        if (tile_skipped<TN>(a, m0, n0)) continue;
        if (!tc::mbar_wait(&tempty[tb], tphase ^ 1u, abort_flag, a.spin)) { ok = false; break; }
        tc::tc_fence_after();
        const uint32_t dcol = tmem + (uint32_t)(tb * TN);
        for (int kc = 0; kc < nkc; ++kc) {
          if (!tc::mbar_wait(&full[stage], phase, abort_flag, a.spin)) { ok = false; break; }
          tc::tc_fence_after();
          const uint32_t sb = tc::smem_u32(smem + (size_t)stage * TxTile<TN>::STAGE_BYTES);
          const uint32_t ah = sb, al = sb + TX_A_BYTES;
          const uint32_t bh = sb + 2 * TX_A_BYTES, bl = bh + TxTile<TN>::B_BYTES;
#pragma unroll
          for (int kk = 0; kk < TX_KC / 8; ++kk) {
            // K-major, 128-byte swizzle: 8-row groups 1024 B apart, K step 32 B
            const uint64_t dah = tc::smem_desc_sw128(ah + kk * 32, 16, 1024);
            const uint64_t dal = tc::smem_desc_sw128(al + kk * 32, 16, 1024);
            const uint64_t dbh = tc::smem_desc_sw128(bh + kk * 32, 16, 1024);
            const uint64_t dbl = tc::smem_desc_sw128(bl + kk * 32, 16, 1024);
            const uint32_t acc0 = (kc > 0 || kk > 0) ? 1u : 0u;
            tc::mma_tf32_ss(dcol, dal, dbh, idesc, acc0);  // small terms first
            tc::mma_tf32_ss(dcol, dah, dbl, idesc, 1u);
            tc::mma_tf32_ss(dcol, dah, dbh, idesc, 1u);
          }
          tc::mma_commit(&empty[stage]);
          if (++stage == TX_STAGES) stage = 0, phase ^= 1u;
        }
        if (!ok) break;
        tc::mma_commit(&tfull[tb]);
        if (++tb == 2) tb = 0, tphase ^= 1u;
      }
      tc::mma_commit(done);
      for (uint32_t i = 0; i < tc::kSpinLimit; ++i)
        if (tc::mbar_try_wait(done, 0)) break;
    }
  } else {
    // epilogue: warp w reads TMEM lanes 32 * (w % 4) .. +31, i.e. tile rows
    const int quarter = warp & 3;
    const int trow = quarter * 32 + lane;
    const bool dprod = (threadIdx.x == 64);  // issues the reduce-adds
    int tb = 0, g = 0;
    uint32_t tphase = 0;
    bool ok = true;
    for (int t = next_tile<TN>(a, -1); t < a.ntiles && ok; t = next_tile<TN>(a, t)) {
      const int m0 = (t % a.ntm) * TX_M, n0 = (t / a.ntm) * TN;
      if (!tc::mbar_wait_warp(&tfull[tb], tphase, abort_flag, a.spin)) { ok = false; break; }
      tc::tc_fence_after();
      const uint32_t tbase = tmem + ((uint32_t)(quarter * 32) << 16) + (uint32_t)(tb * TN);
      float v[32];
      tc::tmem_ld_32x32b_x32(tbase, v);
      for (int cc = 0; cc < TN / TX_DC; ++cc, ++g) {
        tc::tmem_ld_wait();
        const int slot = g % TX_D_SLOTS;
        if (g >= TX_D_SLOTS) {
          // the slot's previous reduce must have read it
          if (!tc::mbar_wait_warp(&dfree[slot], (uint32_t)((g / TX_D_SLOTS) - 1) & 1u, abort_flag,
                                  a.spin)) {
            ok = false;
            break;
          }
        }
        uint8_t* rowp = ring + slot * TX_D_BYTES + trow * 128;
#pragma unroll
        for (int u = 0; u < 8; ++u)
          *(float4*)(rowp + ((u ^ (trow & 7)) << 4)) =
              make_float4(v[4 * u], v[4 * u + 1], v[4 * u + 2], v[4 * u + 3]);
        if (cc + 1 < TN / TX_DC) {
          tc::tmem_ld_32x32b_x32(tbase + (uint32_t)((cc + 1) * TX_DC), v);
        } else {  // accumulator fully read: hand it back to the MMA warp
          tc::tc_fence_before();
          __syncwarp();
          if (lane == 0) tc::mbar_arrive(&tempty[tb]);
        }
        tc::fence_proxy_async_smem();  // the reduce reads what this thread wrote
        __syncwarp();
        if (lane == 0) tc::mbar_arrive(&dwritten[slot]);
        bool gave_up = false;
        if (dprod) {
          if (tc::mbar_wait(&dwritten[slot], (uint32_t)(g / TX_D_SLOTS) & 1u, abort_flag, a.spin)) {
            tc::tma_reduce_add_2d(&d_map, ring + slot * TX_D_BYTES, a.col0 + n0 + cc * TX_DC,
                                  a.row0 + m0);
            tc::bulk_commit_group();
            // free the other slot for the chunk after next once its reduce has read it
            tc::bulk_wait_read_1();
            if (g >= 1) tc::mbar_arrive(&dfree[(g - 1) % TX_D_SLOTS]);
          } else {
            gave_up = true;
          }
        }
        // the reduce thread's warp leaves the loop together with it
        if (__shfl_sync(0xffffffffu, gave_up, 0)) {
          ok = false;
          break;
        }
      }
      if (++tb == 2) tb = 0, tphase ^= 1u;
    }
    if (dprod) tc::bulk_wait_all();
  }

  __syncthreads();
  if (*abort_flag && threadIdx.x == 0 && a.status != nullptr) atomicCAS(a.status, 0, a.status_code);
  tc::tc_fence_after();
  if (warp == 1) tc::tmem_dealloc(tmem, TxTile<TN>::TMEM_COLS);
}


// fp32 2-D map (cols inner, rows outer), row stride ld floats, box {32, box_rows}.
bool make_map(CUtensorMap* m, const float* base, int64_t cols, int64_t rows, int64_t ld,
              uint32_t box_rows) {
  EncodeTiledFn enc = tensormap_encoder();
  if (enc == nullptr) return false;
  cuuint64_t gdim[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
  cuuint64_t gstride[1] = {(cuuint64_t)ld * 4};
  cuuint32_t box[2] = {32, box_rows};
  cuuint32_t es[2] = {1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, const_cast<float*>(base), gdim, gstride, box,
             es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int TN>
gptq_status launch(const CUtensorMap& ah, const CUtensorMap& al, const CUtensorMap& bh,
                   const CUtensorMap& bl, const CUtensorMap& dm, TxArgs& a, cudaStream_t s) {
  if (smem_optin((const void*)tf32x3_update_kernel<TN>, TxTile<TN>::SMEM) != cudaSuccess)
    return GPTQ_ERR_CUDA;
  a.spin = wait_limit();
  const int nsm = sm_count();
  const int grid = std::min(a.ntiles, nsm);
  if (grid <= 0) return GPTQ_OK;
  launch_pdl(tf32x3_update_kernel<TN>, dim3(grid), dim3(TX_THREADS), TxTile<TN>::SMEM, s, ah, al,
             bh, bl, dm, a);
  GPTQ_CHECK_LAUNCH();
  return GPTQ_OK;
}

// The tile width for an update of M x N outputs: 128 when 256-wide tiles
// would leave SMs idle.
int pick_tn(int M, int N) {
  return cdiv(M, TX_M) * cdiv(N, 256) < (int64_t)sm_count() ? 128 : 256;
}


// hi = x rounded to tf32 (nearest, ties away), lo = x - hi
__device__ __forceinline__ void split_tf32(float x, float& hi, float& lo) {
  uint32_t h;
  asm("cvt.rna.tf32.f32 %0, %1;" : "=r"(h) : "f"(x));
  hi = __uint_as_float(h);
  lo = x - hi;
}

// dst[c][r] = split(sign * src[r][c]) for r < rows, c < cols (32 x 32 tiles
// through shared memory, so both the reads and the writes are coalesced).
// upper_only: src is upper triangular and only dst[c][r] with c >= r is
// wanted; tiles with every c < r are left unwritten.
__global__ void split_transpose_kernel(const float* __restrict__ src, int64_t lds, int rows,
                                       int cols, float sign, int upper_only,
                                       float* __restrict__ hi, float* __restrict__ lo,
                                       int64_t ldo) {
  __shared__ float tile[32][33];
  const int r0 = blockIdx.y * 32, c0 = blockIdx.x * 32;
  if (upper_only && c0 + 31 < r0) return;
  const int tx = threadIdx.x, ty = threadIdx.y;  // 32 x 8
  for (int y = ty; y < 32; y += 8) {
    const int r = r0 + y, c = c0 + tx;
    tile[y][tx] = (r < rows && c < cols) ? src[(int64_t)r * lds + c] : 0.f;
  }
  __syncthreads();
  for (int y = ty; y < 32; y += 8) {
    const int c = c0 + y, r = r0 + tx;
    if (c < cols && r < rows) {
      float h, l;
      split_tf32(sign * tile[tx][y], h, l);
      hi[(int64_t)c * ldo + r] = h;
      lo[(int64_t)c * ldo + r] = l;
    }
  }
}

}  // namespace

bool tc_update_supported(int64_t k) { return k % 4 == 0 && tensormap_encoder() != nullptr; }

gptq_status tc_split_transpose(const float* src, int64_t lds, int rows, int cols, float sign,
                               int upper_only, float* hi, float* lo, int64_t ldo, cudaStream_t s) {
  if (rows <= 0 || cols <= 0) return GPTQ_OK;
  dim3 grid((unsigned)cdiv(cols, 32), (unsigned)cdiv(rows, 32));
  split_transpose_kernel<<<grid, dim3(32, 8), 0, s>>>(src, lds, rows, cols, sign, upper_only, hi,
                                                      lo, ldo);
  GPTQ_CHECK_LAUNCH();
  return GPTQ_OK;
}

// Wt[0:r, c0:c1] -= Err[0:r, 0:K] * U[s0:s0+K, c0:c1]   (Err_hi/lo: r x K at
// row stride ldE, 16-byte aligned; nut_hi/lo: the split of -U^T, k x k).  The
// output map ends at column c1 and Err's at column K (a K that is not a
// multiple of the 32-wide stage reads zeros past it), so nothing outside
// [c0, c1) is touched.  A timeout sets *d_status = GPTQ_ERR_TIMEOUT.
gptq_status tc_sweep_trailing(const float* err_hi, const float* err_lo, int ldE, int K,
                              const float* nut_hi, const float* nut_lo, float* Wt, int r, int k,
                              int s0, int c0, int c1, int32_t* d_status, cudaStream_t s) {
  if (c1 <= c0 || K <= 0) return GPTQ_OK;
  const int tn = pick_tn(r, c1 - c0);
  CUtensorMap ah, al, bh, bl, dm;
  if (!make_map(&ah, err_hi, K, r, ldE, TX_M) || !make_map(&al, err_lo, K, r, ldE, TX_M) ||
      !make_map(&bh, nut_hi, k, k, k, tn) || !make_map(&bl, nut_lo, k, k, k, tn) ||
      !make_map(&dm, Wt, c1, r, k, TX_M))
    return GPTQ_ERR_INVALID_ARG;
  TxArgs a;
  a.D = Wt;
  a.ldd = k;
  a.M = r;
  a.N = c1 - c0;
  a.row0 = 0;
  a.col0 = c0;
  a.K = K;
  a.a_k0 = 0;
  a.a_r0 = 0;
  a.b_k0 = s0;
  a.b_r0 = c0;
  a.ntm = (int)cdiv(r, TX_M);
  a.ntiles = a.ntm * (int)cdiv(c1 - c0, tn);
  a.mode = 0;
  a.split = 0;
  a.status = d_status;
  a.status_code = GPTQ_ERR_TIMEOUT;
  return tn == 128 ? launch<128>(ah, al, bh, bl, dm, a, s) : launch<256>(ah, al, bh, bl, dm, a, s);
}

// Rows [row0, row1) of the k x k work matrix A += R^T S (see the file
// comment): r_hi / r_lo = row blocks transposed and split, r[c][m] =
// A[j0 + m][c] for the K = K rows m of the update, read for the output rows c;
// s_hi / s_lo = the same with the Schur columns (c < split) negated, read for
// every column c.  Both have row stride ld_s and start at the update's first
// K column (16-byte aligned); written by the caller.  The output map ends at
// row row1 and the operands' at column K.  A timeout sets *d_info = k + 1.
gptq_status tc_rank_update(float* A, int k, int row0, int row1, int split, int K, int ld_s,
                           const float* s_hi, const float* s_lo, const float* r_hi,
                           const float* r_lo, int32_t* d_info, cudaStream_t s) {
  if (row1 <= row0 || K <= 0) return GPTQ_OK;
  const int tn = pick_tn(row1 - row0, k);
  CUtensorMap ah, al, bh, bl, dm;
  if (!make_map(&ah, r_hi, K, row1, ld_s, TX_M) || !make_map(&al, r_lo, K, row1, ld_s, TX_M) ||
      !make_map(&bh, s_hi, K, k, ld_s, tn) || !make_map(&bl, s_lo, K, k, ld_s, tn) ||
      !make_map(&dm, A, k, row1, k, TX_M))
    return GPTQ_ERR_INVALID_ARG;
  TxArgs a;
  a.D = A;
  a.ldd = k;
  a.M = row1 - row0;
  a.N = k;
  a.row0 = row0;
  a.col0 = 0;
  a.K = K;
  a.a_k0 = 0;
  a.a_r0 = row0;
  a.b_k0 = 0;
  a.b_r0 = 0;
  a.ntm = (int)cdiv(row1 - row0, TX_M);
  a.ntiles = a.ntm * (int)cdiv(k, tn);
  a.mode = 1;
  a.split = split;
  a.status = d_info;
  a.status_code = k + 1;
  return tn == 128 ? launch<128>(ah, al, bh, bl, dm, a, s) : launch<256>(ah, al, bh, bl, dm, a, s);
}

}  // namespace gptq
