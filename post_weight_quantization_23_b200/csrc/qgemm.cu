// The inference product of a GPTQ-quantized layer, Y = X W_hat^T with
// W_hat[j, c] = scale[j, g(c)] * (code[j, c] - zero[j, g(c)]), read straight
// from the packed codes ("GPTQ", ozercemkelahmet.com/tools/gptq: What the
// output looks like -- a GPU kernel reads the packed data and dequantizes
// inside the matrix multiply; How it works, Step 8; "What Is GPTQ?",
// ai-tldr.dev, How it works: each group is expanded just in time).
//
// Small token counts (decode) are bound by the bytes of the packed weights,
// so the decode kernel streams them once with coalesced 16-byte loads and
// does the arithmetic on the CUDA cores.  Each code c is turned into a float
// by one logic op: a code sitting at bit b j of a 16-bit half word (b = bits,
// j = its slot) is kept in place and given the exponent of 2^(23 - b j), which
// makes the float 2^(23 - b j) + c exactly; subtracting 2^(23 - b j) and the
// zero point leaves c - zero exactly, so every product x (c - zero) is exact
// in fp32.  The products are summed in fp32 per 16-byte piece (one group) and
// multiplied by the group's scale once.
#include "common.cuh"

#include <type_traits>

namespace gptq {

bool qgemm_tc_supported(const void* X, int64_t ldx, const int32_t* qw, int bits, int64_t k,
                        int G, bool has_gidx);
gptq_status qgemm_tc(const void* X, bool bf16, int64_t m, int64_t k, int64_t ldx,
                     const int32_t* qw, const float* scales, const int32_t* zeros, int64_t n,
                     int G, int64_t ngroups, void* Y, int64_t ldy, cudaStream_t s);

// Token counts above this use the tensor-core kernel when it applies.
constexpr int QG_TC_MIN_TOKENS = 17;
// From this token count up to 16 the small-batch mma.sync kernel, when it applies
// (measured on 28 7B-shaped layers per pass: 3 and 4 tokens 522 us against the
// decode kernel's 557, 8 tokens 539 against 985, 16 tokens 573 against 1994;
// two tokens stay on the decode kernel, 316 us).
constexpr int QM_MIN_TOKENS = 3;

namespace {

template <typename T> __device__ __forceinline__ T qg_out(float v);
template <> __device__ __forceinline__ __half qg_out<__half>(float v) { return __float2half_rn(v); }
template <> __device__ __forceinline__ __nv_bfloat16 qg_out<__nv_bfloat16>(float v) {
  return __float2bfloat16_rn(v);
}

__device__ __forceinline__ uint4 ld_stream_u4(const void* p) {
  uint4 v;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}

constexpr int QV_WARPS = 8;     // warps per CTA, each a share of the slabs
constexpr int QV_RPL = 4;       // rows per lane
constexpr int QV_ROWS = 4 * QV_RPL;  // rows of W per CTA (4 rows per load instruction)
constexpr int QV_KC = 8192;     // columns of X staged in shared memory per pass

template <int BITS>
struct QvShape {
  static constexpr int CPW = 32 / BITS;   // codes per 32-bit word
  static constexpr int HC = CPW / 2;      // codes per 16-bit half word
  static constexpr int CH = 4 * CPW;      // columns per 16-byte piece
  static constexpr int SLAB = 8 * CH;     // columns one warp covers per step (8 lanes per row)
  static constexpr int PAD = 4;           // floats of padding after every CH staged columns
  static constexpr uint32_t MASK = (1u << BITS) - 1u;
};

// Columns of X staged per pass for M tokens (the staging buffer stays under
// 150 KB of shared memory).
constexpr int qv_kc_max(int M) { return M <= 4 ? QV_KC : QV_KC / 2; }

inline int qv_kc(int k, int slab, int M) {
  const int kc = k < qv_kc_max(M) ? k : qv_kc_max(M);
  return (int)(cdiv(kc, slab) * slab);
}

template <int BITS>
inline size_t qv_smem_bytes(int M, int KC) {
  using Sh = QvShape<BITS>;
  const int XS = KC + Sh::PAD * (KC / Sh::CH);
  return sizeof(float) * ((size_t)M * XS + (size_t)QV_WARPS * M * QV_ROWS);
}

// One warp-slab of packed words: lane (q, p) holds piece p of rows 4 i + q.
template <int BITS>
struct QvSlab {
  uint4 d[QV_RPL];
  float sc[QV_RPL];
  float nz[QV_RPL];  // -zero
};

template <int BITS>
__device__ __forceinline__ void qv_load(QvSlab<BITS>& S, const int32_t* __restrict__ qw,
                                        const float* __restrict__ scales,
                                        const int32_t* __restrict__ zeros, int64_t wpr, int r0,
                                        int q, int n, int c, bool have, int G, int ngroups) {
  using Sh = QvShape<BITS>;
  const int g = c / G;
#pragma unroll
  for (int i = 0; i < QV_RPL; ++i) {
    const int row = r0 + 4 * i + q;
    const bool ok = have && row < n;
    S.d[i] = ok ? ld_stream_u4(qw + (int64_t)row * wpr + c / Sh::CPW) : make_uint4(0u, 0u, 0u, 0u);
    S.sc[i] = ok ? scales[(int64_t)row * ngroups + g] : 0.f;
    S.nz[i] = ok ? -(float)zeros[(int64_t)row * ngroups + g] : 0.f;
  }
}

// y[i][t] += scale_i * sum over the lane's piece of x_t (code - zero).
template <int BITS, int M>
__device__ __forceinline__ void qv_compute(const QvSlab<BITS>& S, const float* xb, int XS,
                                           float (&y)[QV_RPL][M]) {
  using Sh = QvShape<BITS>;
  float2 acc[QV_RPL][M];
#pragma unroll
  for (int i = 0; i < QV_RPL; ++i)
#pragma unroll
    for (int t = 0; t < M; ++t) acc[i][t] = make_float2(0.f, 0.f);
#pragma unroll
  for (int wi = 0; wi < 4; ++wi) {
#pragma unroll
    for (int h = 0; h < 2; ++h) {
#pragma unroll
      for (int j = 0; j < Sh::HC; j += 2) {
        const int col = wi * Sh::CPW + h * Sh::HC + j;
        float2 x2[M];
#pragma unroll
        for (int t = 0; t < M; ++t) x2[t] = *reinterpret_cast<const float2*>(xb + t * XS + col);
        // -2^(23 - b j) for the two slots (compile-time constants)
        const float2 nmag = make_float2(-(float)(1 << (23 - BITS * j)),
                                        -(float)(1 << (23 - BITS * (j + 1))));
        const float2 one = make_float2(1.f, 1.f);
#pragma unroll
        for (int i = 0; i < QV_RPL; ++i) {
          const uint32_t word = wi == 0 ? S.d[i].x : wi == 1 ? S.d[i].y : wi == 2 ? S.d[i].z : S.d[i].w;
          const uint32_t hw = h ? (word >> 16) : word;
          // 2^(23 - b j) + c, exactly
          const float f0 = __uint_as_float((0x4B000000u - ((uint32_t)(BITS * j) << 23)) |
                                           (hw & (Sh::MASK << (BITS * j))));
          const float f1 = __uint_as_float((0x4B000000u - ((uint32_t)(BITS * (j + 1)) << 23)) |
                                           (hw & (Sh::MASK << (BITS * (j + 1)))));
          const float2 c2 = __ffma2_rn(make_float2(f0, f1), one, nmag);                 // c, exact
          const float2 dd = __ffma2_rn(c2, one, make_float2(S.nz[i], S.nz[i]));        // c - zero
#pragma unroll
          for (int t = 0; t < M; ++t) acc[i][t] = __ffma2_rn(x2[t], dd, acc[i][t]);
        }
      }
    }
  }
#pragma unroll
  for (int i = 0; i < QV_RPL; ++i)
#pragma unroll
    for (int t = 0; t < M; ++t) y[i][t] = fmaf(S.sc[i], acc[i][t].x + acc[i][t].y, y[i][t]);
}

// Decode kernel: CTA = 16 rows x M tokens (M = 1, 2, 4 or 8), 8 warps sharing
// the column slabs.  The CTAs of one row block are consecutive (the block index
// runs over the token groups first), so a second token group finds the row
// block's packed words in L2.  Launched with programmatic dependent launch:
// the first slabs of packed words are requested before waiting for the
// previous kernel (only X depends on it; the weights must not be written by a
// kernel that lets this one start early).
// Lane (q = lane / 8, p = lane % 8) loads, for i = 0..3, the 16-byte piece p
// of row 4 i + q in its warp's slab, so each load instruction reads four whole
// 128-byte row segments.  The first AHEAD slabs' words (two for M = 1, one
// otherwise) are requested before the activations are staged, and each later
// slab's AHEAD slabs before it is computed.  Needs k % CH == 0 and a group size that is a multiple of CH (or
// one group per row), so a piece lies in one group.
template <int BITS, int M, typename T>
__global__ void __launch_bounds__(QV_WARPS * 32, M <= 2 ? 2 : 1)  // decode: 2 CTAs per SM
qgemv_kernel(const T* __restrict__ X, int64_t ldx, int m, int k,
             const int32_t* __restrict__ qw, const float* __restrict__ scales,
             const int32_t* __restrict__ zeros, int n, int G, int ngroups, int KC,
             int xvec, T* __restrict__ Y, int64_t ldy) {
  using Sh = QvShape<BITS>;
  extern __shared__ __align__(16) float qv_smem[];
  const int XS = KC + Sh::PAD * (KC / Sh::CH);
  float* xs = qv_smem;            // [M][XS] staged activations (fp32)
  float* red = xs + M * XS;       // [QV_WARPS][M][QV_ROWS] per-warp row sums
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int q = lane >> 3, p = lane & 7;
  const int ntg = (m + M - 1) / M;
  const int r0 = (int)(blockIdx.x / ntg) * QV_ROWS;
  const int t0 = (int)(blockIdx.x % ntg) * M;
  const int64_t wpr = (int64_t)k / Sh::CPW;  // words per row
  constexpr int STEP = QV_WARPS * Sh::SLAB;  // columns per round of the 8 warps
  // slabs in flight beyond the one being computed: two for one token (whose
  // few slabs per warp are then all requested early; measured 290 -> 273 us
  // for the 28-layer decode pass, while two tokens ran 316 -> 325 us)
  constexpr int AHEAD = M == 1 ? 2 : 1;

  float y[QV_RPL][M];
#pragma unroll
  for (int i = 0; i < QV_RPL; ++i)
#pragma unroll
    for (int t = 0; t < M; ++t) y[i][t] = 0.f;

  for (int kc0 = 0; kc0 < k; kc0 += KC) {
    const int kcw = min(KC, k - kc0);
    // this warp's first AHEAD slabs of the chunk, requested before the staging
    int sl = warp * Sh::SLAB;
    QvSlab<BITS> cur, nxt;
    {
      const int cl = sl + p * Sh::CH;
      qv_load<BITS>(cur, qw, scales, zeros, wpr, r0, q, n, kc0 + cl, cl < kcw, G, ngroups);
      if (AHEAD == 2) {
        const int cn = sl + STEP + p * Sh::CH;
        qv_load<BITS>(nxt, qw, scales, zeros, wpr, r0, q, n, kc0 + cn, cn < kcw, G, ngroups);
      }
    }
    if (kc0 == 0) {
      // X comes from the previous kernel
      pdl_wait();
      pdl_trigger();
    }
    __syncthreads();  // the previous pass is done with xs
    if (xvec) {
      // 8 activations per 16-byte load, all of a thread's loads in flight
      // together (kcw is a multiple of 8; 8 columns never straddle a pad)
      const int nv = kcw / 8;
#pragma unroll 4
      for (int e = tid; e < M * nv; e += blockDim.x) {
        const int t = e / nv, c = 8 * (e - t * nv);
        uint4 u = make_uint4(0u, 0u, 0u, 0u);
        if (t0 + t < m) u = *reinterpret_cast<const uint4*>(X + (int64_t)(t0 + t) * ldx + kc0 + c);
        const T* h = reinterpret_cast<const T*>(&u);
        float4* dst = reinterpret_cast<float4*>(xs + t * XS + c + Sh::PAD * (c / Sh::CH));
        dst[0] = make_float4(to_f32(h[0]), to_f32(h[1]), to_f32(h[2]), to_f32(h[3]));
        dst[1] = make_float4(to_f32(h[4]), to_f32(h[5]), to_f32(h[6]), to_f32(h[7]));
      }
    } else {
#pragma unroll 8
      for (int e = tid; e < M * kcw; e += blockDim.x) {
        const int t = e / kcw, c = e - t * kcw;
        float v = 0.f;
        if (t0 + t < m) v = to_f32(X[(int64_t)(t0 + t) * ldx + kc0 + c]);
        xs[t * XS + c + Sh::PAD * (c / Sh::CH)] = v;
      }
    }
    __syncthreads();
    for (; sl < kcw; sl += STEP) {
      const int cl = sl + p * Sh::CH;  // this lane's piece, local column
      const bool have = cl < kcw;
      QvSlab<BITS> nn;
      const int sa = sl + AHEAD * STEP;  // the slab requested now
      if (sa < kcw) {
        const int ca = sa + p * Sh::CH;
        qv_load<BITS>(nn, qw, scales, zeros, wpr, r0, q, n, kc0 + ca, ca < kcw, G, ngroups);
      }
      // lanes past the chunk's end have zero words and scale 0; they read
      // (and discard) the chunk's first columns instead of past the buffer
      const int clx = have ? cl : 0;
      qv_compute<BITS, M>(cur, xs + clx + Sh::PAD * (clx / Sh::CH), XS, y);
      if (AHEAD == 2) {
        cur = nxt;
        if (sa < kcw) nxt = nn;
      } else if (sa < kcw) {
        cur = nn;
      }
    }
  }
  // sum the 8 pieces of each row, then the warps
#pragma unroll
  for (int i = 0; i < QV_RPL; ++i)
#pragma unroll
    for (int t = 0; t < M; ++t) {
      float v = y[i][t];
      v += __shfl_xor_sync(0xffffffffu, v, 1);
      v += __shfl_xor_sync(0xffffffffu, v, 2);
      v += __shfl_xor_sync(0xffffffffu, v, 4);
      y[i][t] = v;
    }
  if (p == 0) {
#pragma unroll
    for (int i = 0; i < QV_RPL; ++i)
#pragma unroll
      for (int t = 0; t < M; ++t) red[(warp * M + t) * QV_ROWS + 4 * i + q] = y[i][t];
  }
  __syncthreads();
  for (int e = tid; e < M * QV_ROWS; e += blockDim.x) {
    const int t = e / QV_ROWS, rr = e % QV_ROWS;
    float v = 0.f;
#pragma unroll
    for (int w = 0; w < QV_WARPS; ++w) v += red[(w * M + t) * QV_ROWS + rr];
    if (t0 + t < m && r0 + rr < n) Y[(int64_t)(t0 + t) * ldy + r0 + rr] = qg_out<T>(v);
  }
}

// General kernel: any bit width (3-bit codes straddle words), any g_idx, any
// group size.  One warp per (row, 8 tokens); lanes stride over the columns;
// W_hat = scale * (code - zero) in fp32 per element.  A g_idx entry outside
// [0, ngroups) is not read through: it makes the row's outputs NaN.
template <typename T>
__global__ void __launch_bounds__(256)
qgemm_general_kernel(const T* __restrict__ X, int64_t ldx, int m, int k,
                     const int32_t* __restrict__ qw, int bits, const float* __restrict__ scales,
                     const int32_t* __restrict__ zeros, const int32_t* __restrict__ g_idx, int G,
                     int ngroups, int n, T* __restrict__ Y, int64_t ldy) {
  const int lane = threadIdx.x & 31;
  const int row = blockIdx.x * 8 + (threadIdx.x >> 5);
  const int t0 = blockIdx.y * 8;
  if (row >= n) return;
  const int64_t wpr = (int64_t)k * bits / 32;
  const uint32_t* wr = reinterpret_cast<const uint32_t*>(qw) + (int64_t)row * wpr;
  const uint32_t mask = (1u << bits) - 1u;
  float acc[8];
#pragma unroll
  for (int t = 0; t < 8; ++t) acc[t] = 0.f;
  bool bad = false;
  for (int c = lane; c < k; c += 32) {
    const int64_t bit = (int64_t)c * bits;
    const int64_t w = bit >> 5;
    const int sh = (int)(bit & 31);
    uint32_t v = wr[w] >> sh;
    if (sh + bits > 32) v |= wr[w + 1] << (32 - sh);
    const int code = (int)(v & mask);
    const int g = g_idx != nullptr ? g_idx[c] : c / G;
    if (g < 0 || g >= ngroups) {
      bad = true;
      continue;
    }
    const float wv = scales[(int64_t)row * ngroups + g] *
                     (float)(code - zeros[(int64_t)row * ngroups + g]);
#pragma unroll
    for (int t = 0; t < 8; ++t)
      if (t0 + t < m) acc[t] = fmaf(to_f32(X[(int64_t)(t0 + t) * ldx + c]), wv, acc[t]);
  }
  bad = __any_sync(0xffffffffu, bad);
#pragma unroll
  for (int t = 0; t < 8; ++t) {
    float v = acc[t];
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    if (lane == 0 && t0 + t < m)
      Y[(int64_t)(t0 + t) * ldy + row] = qg_out<T>(bad ? __int_as_float(0x7fc00000) : v);
  }
}

// Small-batch kernel (3 to 16 tokens, 4-bit codes, groups of a multiple of 128
// columns or one group per row): the tokens are one 16-row A operand of the
// legacy mma.sync m16n8k16 (fp32 accumulate), the weights its B operand,
// expanded in registers from the packed words.  The weight stream, which
// bounds these token counts as it bounds decode, is read once for all tokens.
// CTA = 16 weight rows (two 8-row MMA tiles) x all tokens, 8 warps splitting k
// in slabs of 256 columns as in the decode kernel (same coalesced 16-byte
// loads, the next pass's slab requested before the current one is computed);
// each warp parks its slab's packed words in shared memory so that every lane can
// pick its fragment's codes: lane (g, t) needs, for row g of a tile and k-step
// s, codes 2t, 2t+1 of word 2s and of word 2s+1 -- one byte of each.  A code
// pair becomes one packed pair of M + c exactly (M = 1024 for f16, 128 for
// bf16, the nibbles put in the low mantissa bits); a packed subtract of M + z
// leaves c - z exactly and one packed multiply by the scale (rounded to the
// activations' type) gives the weight, rounded once: the tensor-core kernel's
// weights.  Each warp stages its own slab's columns of the activations in
// shared memory (tokens past m as zeros) and reads A fragments with ldmatrix.
constexpr int QM_WARPS = 8;
constexpr int QM_ROWS = 16;             // weight rows per CTA
constexpr int QM_SLAB = 256;            // columns per warp-step (8 lanes x 32 codes)
constexpr int QM_STEP = QM_WARPS * QM_SLAB;
constexpr int QM_KC = 2048;             // columns of X per pass
static_assert(QM_KC == QM_STEP, "one slab per warp and pass");
constexpr int QM_XLD = QM_KC + 8;       // row stride of the staged X (16-byte aligned rows)
constexpr int QM_WLD = 36;              // words per row of a parked slab (conflict-free reads)
constexpr size_t QM_SMEM = sizeof(uint16_t) * 16 * QM_XLD +
                           sizeof(uint32_t) * QM_WARPS * QM_ROWS * QM_WLD +
                           sizeof(float) * QM_WARPS * 16 * QM_ROWS;

template <bool BF16> struct QmType;
template <> struct QmType<false> {
  using T = __half;
  using T2 = __half2;
  static constexpr uint32_t MAGIC = 0x64006400u;  // 1024 in both halves
  static constexpr float BASE = 1024.f;
  __device__ static T2 pair(float v) { return __float2half2_rn(v); }
};
template <> struct QmType<true> {
  using T = __nv_bfloat16;
  using T2 = __nv_bfloat162;
  static constexpr uint32_t MAGIC = 0x43004300u;  // 128 in both halves
  static constexpr float BASE = 128.f;
  __device__ static T2 pair(float v) { return __float2bfloat162_rn(v); }
};

template <bool BF16>
__device__ __forceinline__ void qm_mma(float (&d)[4], const uint32_t (&a)[4], uint32_t b0,
                                       uint32_t b1) {
  if (BF16)
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, "
        "{%4, %5, %6, %7}, {%8, %9}, {%0, %1, %2, %3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
  else
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0, %1, %2, %3}, "
        "{%4, %5, %6, %7}, {%8, %9}, {%0, %1, %2, %3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// byte x = two codes (low nibble first) -> the weights of that pair in T
template <bool BF16>
__device__ __forceinline__ uint32_t qm_weights(uint32_t x, typename QmType<BF16>::T2 zb,
                                               typename QmType<BF16>::T2 sc) {
  using Q = QmType<BF16>;
  const uint32_t h = (x & 0x0Fu) | ((x & 0xF0u) << 12) | Q::MAGIC;  // M + c, exactly
  typename Q::T2 v = *reinterpret_cast<const typename Q::T2*>(&h);
  v = __hmul2(__hsub2(v, zb), sc);
  return *reinterpret_cast<const uint32_t*>(&v);
}

template <bool BF16>
__global__ void __launch_bounds__(QM_WARPS * 32, 2)
qgemm_mma_kernel(const typename QmType<BF16>::T* __restrict__ X, int64_t ldx, int m, int k,
                 const int32_t* __restrict__ qw, const float* __restrict__ scales,
                 const int32_t* __restrict__ zeros, int n, int G, int ngroups, int xvec,
                 typename QmType<BF16>::T* __restrict__ Y, int64_t ldy) {
  using Q = QmType<BF16>;
  using T = typename Q::T;
  extern __shared__ __align__(16) uint8_t qm_smem[];
  T* xs = reinterpret_cast<T*>(qm_smem);                                   // [16][QM_XLD]
  uint32_t* wpark = reinterpret_cast<uint32_t*>(xs + 16 * QM_XLD);         // [8][16][QM_WLD]
  float* red = reinterpret_cast<float*>(wpark + QM_WARPS * QM_ROWS * QM_WLD);  // [8][16][16]
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int q = lane >> 3, p = lane & 7;   // load layout: piece p of rows 4 i + q
  const int g = lane >> 2, t = lane & 3;   // fragment layout
  const int r0 = (int)blockIdx.x * QM_ROWS;
  const int64_t wpr = (int64_t)k / 8;      // words per row
  uint32_t* park = wpark + warp * QM_ROWS * QM_WLD;
  float acc[2][4];
#pragma unroll
  for (int nt = 0; nt < 2; ++nt)
#pragma unroll
    for (int e = 0; e < 4; ++e) acc[nt][e] = 0.f;
  const uint32_t xs_base = (uint32_t)__cvta_generic_to_shared(xs);
  // ldmatrix row address of this lane: matrix lane / 8, row lane % 8
  const int lm_row = (lane & 7) + ((lane >> 3) & 1) * 8, lm_col = (lane >> 4) * 8;

  // each pass of QM_KC = 8 x 256 columns gives every warp at most one slab, and
  // the warp stages only its own slab's activations (no CTA-wide barrier); the
  // next pass's packed words are requested before this pass is computed
  const int sl = warp * QM_SLAB;
  uint4 cur[4];
#define QM_LOAD_SLAB(d, kc0_, kcw_)                                                            \
  _Pragma("unroll") for (int i = 0; i < 4; ++i) {                                               \
    const int row_ = r0 + 4 * i + q, cl_ = sl + p * 32;                                          \
    d[i] = (row_ < n && cl_ < (kcw_)) ? ld_stream_u4(qw + (int64_t)row_ * wpr + ((kc0_) + cl_) / 8) \
                                      : make_uint4(0u, 0u, 0u, 0u);                              \
  }
  QM_LOAD_SLAB(cur, 0, min(QM_KC, k))
  // X comes from the previous kernel
  pdl_wait();
  pdl_trigger();
  for (int kc0 = 0; kc0 < k; kc0 += QM_KC) {
    const int kcw = min(QM_KC, k - kc0);
    uint4 nxt[4];
    const bool more = kc0 + QM_KC < k;
    if (more) {
      QM_LOAD_SLAB(nxt, kc0 + QM_KC, min(QM_KC, k - kc0 - QM_KC))
    }
    if (sl < kcw) {
      const int ncol = min(QM_SLAB, kcw - sl);  // a multiple of 32
      __syncwarp();  // this warp's reads of its columns of xs and of its parking rows are done
      if (xvec) {
        const int nv = ncol / 8;
        for (int e = lane; e < 16 * nv; e += 32) {
          const int tk = e / nv, c = sl + 8 * (e - tk * nv);
          uint4 u = make_uint4(0u, 0u, 0u, 0u);
          if (tk < m) u = *reinterpret_cast<const uint4*>(X + (int64_t)tk * ldx + kc0 + c);
          *reinterpret_cast<uint4*>(xs + tk * QM_XLD + c) = u;
        }
      } else {
        for (int e = lane; e < 16 * ncol; e += 32) {
          const int tk = e / ncol, c = sl + (e - tk * ncol);
          xs[tk * QM_XLD + c] = tk < m ? X[(int64_t)tk * ldx + kc0 + c] : Q::pair(0.f).x;
        }
      }
#pragma unroll
      for (int i = 0; i < 4; ++i)
        *reinterpret_cast<uint4*>(park + (4 * i + q) * QM_WLD + 4 * p) = cur[i];
      __syncwarp();
      // the group grids of this lane's two rows in the slab's two 128-column halves
      typename Q::T2 zb[2][2], sc[2][2];
#pragma unroll
      for (int nt = 0; nt < 2; ++nt) {
        const int row = r0 + 8 * nt + g;
#pragma unroll
        for (int hf = 0; hf < 2; ++hf) {
          const int c = kc0 + sl + 128 * hf;
          const int grp = min(c, k - 1) / G;
          float sv = 0.f, zv = 0.f;
          if (row < n) {
            sv = scales[(int64_t)row * ngroups + grp];
            zv = (float)zeros[(int64_t)row * ngroups + grp];
          }
          zb[nt][hf] = Q::pair(Q::BASE + zv);
          sc[nt][hf] = Q::pair(sv);
        }
      }
#pragma unroll
      for (int hf = 0; hf < 2; ++hf) {
#pragma unroll 4
        for (int s8 = 0; s8 < QM_SLAB / 32; ++s8) {
          const int s = 8 * hf + s8;
          if (16 * s >= ncol) break;  // the same for every lane
          uint32_t a[4];
          const uint32_t addr =
              xs_base + (uint32_t)((lm_row * QM_XLD + sl + 16 * s + lm_col) * (int)sizeof(T));
          asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
                       : "=r"(a[0]), "=r"(a[1]), "=r"(a[2]), "=r"(a[3])
                       : "r"(addr));
#pragma unroll
          for (int nt = 0; nt < 2; ++nt) {
            const uint2 w = *reinterpret_cast<const uint2*>(park + (8 * nt + g) * QM_WLD + 2 * s);
            const uint32_t b0 =
                qm_weights<BF16>((w.x >> (8 * t)) & 0xFFu, zb[nt][hf], sc[nt][hf]);
            const uint32_t b1 =
                qm_weights<BF16>((w.y >> (8 * t)) & 0xFFu, zb[nt][hf], sc[nt][hf]);
            qm_mma<BF16>(acc[nt], a, b0, b1);
          }
        }
      }
    }
    if (more) {
#pragma unroll
      for (int i = 0; i < 4; ++i) cur[i] = nxt[i];
    }
  }
  // lane (g, t) holds, per tile nt, (token g | g + 8, row 8 nt + 2 t | + 1)
#pragma unroll
  for (int nt = 0; nt < 2; ++nt) {
    float* rw = red + warp * 16 * QM_ROWS;
    rw[g * QM_ROWS + 8 * nt + 2 * t] = acc[nt][0];
    rw[g * QM_ROWS + 8 * nt + 2 * t + 1] = acc[nt][1];
    rw[(g + 8) * QM_ROWS + 8 * nt + 2 * t] = acc[nt][2];
    rw[(g + 8) * QM_ROWS + 8 * nt + 2 * t + 1] = acc[nt][3];
  }
  __syncthreads();
  {
    const int tk = tid / QM_ROWS, rr = tid % QM_ROWS;  // 256 threads = 16 tokens x 16 rows
    float v = 0.f;
#pragma unroll
    for (int w = 0; w < QM_WARPS; ++w) v += red[(w * 16 + tk) * QM_ROWS + rr];
    if (tk < m && r0 + rr < n) Y[(int64_t)tk * ldy + r0 + rr] = qg_out<T>(v);
  }
}

#undef QM_LOAD_SLAB

template <bool BF16>
gptq_status launch_qgemm_mma(const void* X, int64_t ldx, int m, int k, const int32_t* qw,
                             const float* scales, const int32_t* zeros, int n, int G, int ngroups,
                             void* Y, int64_t ldy, cudaStream_t s) {
  using T = typename QmType<BF16>::T;
  if (smem_optin((const void*)qgemm_mma_kernel<BF16>, QM_SMEM) != cudaSuccess) return GPTQ_ERR_CUDA;
  const int xvec = ((uintptr_t)X % 16) == 0 && ldx % 8 == 0;
  launch_pdl(qgemm_mma_kernel<BF16>, dim3((unsigned)cdiv(n, QM_ROWS)), dim3(QM_WARPS * 32),
             QM_SMEM, s, (const T*)X, ldx, m, k, qw, scales, zeros, n, G, ngroups, xvec, (T*)Y,
             ldy);
  GPTQ_CHECK_LAUNCH();
  return GPTQ_OK;
}

template <int BITS, int M, typename T>
gptq_status launch_qgemv(const T* X, int64_t ldx, int m, int k, const int32_t* qw,
                         const float* scales, const int32_t* zeros, int n, int G, int ngroups,
                         T* Y, int64_t ldy, cudaStream_t s) {
  using Sh = QvShape<BITS>;
  const int KC = qv_kc(k, Sh::SLAB, M);
  const size_t smem = qv_smem_bytes<BITS>(M, KC);
  // opt in once per device to the most this instantiation can ask for
  if (smem > 48 * 1024 &&
      smem_optin((const void*)qgemv_kernel<BITS, M, T>,
                 qv_smem_bytes<BITS>(M, (int)(cdiv(qv_kc_max(M), Sh::SLAB) * Sh::SLAB))) !=
          cudaSuccess)
    return GPTQ_ERR_CUDA;
  const int64_t nblk = cdiv(n, QV_ROWS) * cdiv(m, M);
  if (nblk > (int64_t)INT32_MAX) return GPTQ_ERR_INVALID_ARG;
  // 16-byte activation loads when every row of X starts on a 16-byte boundary
  const int xvec = ((uintptr_t)X % 16) == 0 && ldx % 8 == 0;
  launch_pdl(qgemv_kernel<BITS, M, T>, dim3((unsigned)nblk), dim3(QV_WARPS * 32), smem, s, X, ldx,
             m, k, qw, scales, zeros, n, G, ngroups, KC, xvec, Y, ldy);
  GPTQ_CHECK_LAUNCH();
  return GPTQ_OK;
}

template <int BITS, typename T>
gptq_status qgemv_bits(const T* X, int64_t ldx, int m, int k, const int32_t* qw,
                       const float* scales, const int32_t* zeros, int n, int G, int ngroups, T* Y,
                       int64_t ldy, cudaStream_t s) {
  // up to 8 tokens per CTA; more tokens take several CTAs per row block,
  // which find its packed words in L2
  if (m == 1) return launch_qgemv<BITS, 1, T>(X, ldx, m, k, qw, scales, zeros, n, G, ngroups, Y, ldy, s);
  if (m == 2) return launch_qgemv<BITS, 2, T>(X, ldx, m, k, qw, scales, zeros, n, G, ngroups, Y, ldy, s);
  if (m <= 4) return launch_qgemv<BITS, 4, T>(X, ldx, m, k, qw, scales, zeros, n, G, ngroups, Y, ldy, s);
  return launch_qgemv<BITS, 8, T>(X, ldx, m, k, qw, scales, zeros, n, G, ngroups, Y, ldy, s);
}

template <typename T>
gptq_status qgemm_typed(const T* X, int64_t ldx, int m, int k, const int32_t* qw,
                        const float* scales, const int32_t* zeros, const int32_t* g_idx, int n,
                        int bits, int G, int ngroups, T* Y, int64_t ldy, cudaStream_t s) {
  const bool pow2 = bits == 2 || bits == 4 || bits == 8;
  if (m >= QG_TC_MIN_TOKENS && k > 0 &&
      qgemm_tc_supported(X, ldx, qw, bits, k, G, g_idx != nullptr))
    return qgemm_tc(X, std::is_same<T, __nv_bfloat16>::value, m, k, ldx, qw, scales, zeros, n, G,
                    ngroups, Y, ldy, s);
  if (m >= QM_MIN_TOKENS && m <= 16 && bits == 4 && g_idx == nullptr && k > 0 && k % 32 == 0 &&
      (G >= k || G % 128 == 0) && ((uintptr_t)qw % 16) == 0)
    return launch_qgemm_mma<std::is_same<T, __nv_bfloat16>::value>(X, ldx, m, k, qw, scales,
                                                                    zeros, n, G, ngroups, Y, ldy, s);
  if (pow2 && g_idx == nullptr && ((uintptr_t)qw % 16) == 0 && k > 0) {
    const int CH = 4 * (32 / bits);
    if (k % CH == 0 && (G >= k || G % CH == 0)) {
      switch (bits) {
        case 2: return qgemv_bits<2, T>(X, ldx, m, k, qw, scales, zeros, n, G, ngroups, Y, ldy, s);
        case 4: return qgemv_bits<4, T>(X, ldx, m, k, qw, scales, zeros, n, G, ngroups, Y, ldy, s);
        default: return qgemv_bits<8, T>(X, ldx, m, k, qw, scales, zeros, n, G, ngroups, Y, ldy, s);
      }
    }
  }
  const dim3 grid((unsigned)cdiv(n, 8), (unsigned)cdiv(m, 8));
  qgemm_general_kernel<T><<<grid, 256, 0, s>>>(X, ldx, m, k, qw, bits, scales, zeros, g_idx, G,
                                               ngroups, n, Y, ldy);
  GPTQ_CHECK_LAUNCH();
  return GPTQ_OK;
}

}  // namespace

gptq_status gemm_impl(const void* X, gptq_dtype dt, int64_t m, int64_t k, int64_t ldx,
                      const int32_t* qweight, const float* scales, const int32_t* zeros,
                      const int32_t* g_idx, int64_t n, int bits, int group_size, int64_t ngroups,
                      void* Y, int64_t ldy, cudaStream_t s) {
  const int G = group_size == -1 ? (int)k : group_size;
  if (dt == GPTQ_F16)
    return qgemm_typed<__half>((const __half*)X, ldx, (int)m, (int)k, qweight, scales, zeros,
                               g_idx, (int)n, bits, G, (int)ngroups, (__half*)Y, ldy, s);
  return qgemm_typed<__nv_bfloat16>((const __nv_bfloat16*)X, ldx, (int)m, (int)k, qweight, scales,
                                    zeros, g_idx, (int)n, bits, G, (int)ngroups,
                                    (__nv_bfloat16*)Y, ldy, s);
}

}  // namespace gptq
