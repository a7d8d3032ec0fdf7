// Packing and dequantization of GPTQ codes ([GPTQ-tool] "GPTQ" How it works
// Step 8: eight 4-bit codes per 32-bit word; sketch dequantization
// scale * (q - zero); [What-is-GPTQ] Step 3, groups expanded just in time).
//
// Layout: each row's codes form an LSB-first bit stream, code j in stream bits
// [j*bits, (j+1)*bits), stream bit m in bit m%32 of word m/32.  32 codes fill
// exactly `bits` words for every bit width, so one thread handles one run of
// 32 codes <-> `bits` words: reads and writes are contiguous per thread and
// adjacent threads touch adjacent runs.
#include "common.cuh"

namespace gptq {

template <int BITS>
__global__ void pack_kernel(const uint8_t* __restrict__ codes, int64_t r, int64_t k,
                            int32_t* __restrict__ qweight) {
  const int64_t runs_per_row = k / 32;
  const int64_t nruns = r * runs_per_row;
  for (int64_t t = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; t < nruns;
       t += (int64_t)gridDim.x * blockDim.x) {
    const int64_t row = t / runs_per_row, run = t % runs_per_row;
    const uint4* src = reinterpret_cast<const uint4*>(codes + row * k + run * 32);
    uint4 a = src[0], b = src[1];
    uint32_t in[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
    uint32_t out[BITS];
#pragma unroll
    for (int w = 0; w < BITS; ++w) out[w] = 0u;
#pragma unroll
    for (int j = 0; j < 32; ++j) {
      uint32_t c = (in[j / 4] >> (8 * (j % 4))) & ((1u << BITS) - 1u);
      const int bit = j * BITS;  // compile-time after unrolling
      out[bit / 32] |= c << (bit % 32);
      if ((bit % 32) + BITS > 32) out[bit / 32 + 1] |= c >> (32 - bit % 32);
    }
    int32_t* dst = qweight + row * (k * BITS / 32) + run * BITS;
#pragma unroll
    for (int w = 0; w < BITS; ++w) dst[w] = (int32_t)out[w];
  }
}

template <typename OutT> __device__ __forceinline__ OutT cvt_out(float v);
template <> __device__ __forceinline__ float cvt_out<float>(float v) { return v; }
template <> __device__ __forceinline__ __half cvt_out<__half>(float v) { return __float2half_rn(v); }
template <> __device__ __forceinline__ __nv_bfloat16 cvt_out<__nv_bfloat16>(float v) {
  return __float2bfloat16_rn(v);
}

// Store 32 consecutive outputs of one run: with `vec` as 16-byte vectors (the
// run's outputs are contiguous and, for an aligned `out` and k % 32 == 0,
// 16-byte aligned), else one by one.
template <typename OutT>
__device__ __forceinline__ void store_run(OutT* dst, const float (&v)[32], bool vec) {
  if (vec) {
    if constexpr (sizeof(OutT) == 4) {
#pragma unroll
      for (int q = 0; q < 8; ++q)
        reinterpret_cast<float4*>(dst)[q] =
            make_float4(v[4 * q], v[4 * q + 1], v[4 * q + 2], v[4 * q + 3]);
    } else {
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        uint32_t w[4];
#pragma unroll
        for (int h = 0; h < 4; ++h) {
          const OutT lo = cvt_out<OutT>(v[8 * q + 2 * h]), hi = cvt_out<OutT>(v[8 * q + 2 * h + 1]);
          w[h] = (uint32_t)(*reinterpret_cast<const uint16_t*>(&lo)) |
                 ((uint32_t)(*reinterpret_cast<const uint16_t*>(&hi)) << 16);
        }
        reinterpret_cast<uint4*>(dst)[q] = make_uint4(w[0], w[1], w[2], w[3]);
      }
    }
  } else {
#pragma unroll
    for (int j = 0; j < 32; ++j) dst[j] = cvt_out<OutT>(v[j]);
  }
}

// One thread per run of 32 codes (`bits` words): the run's g_idx entries come
// in as 16-byte vectors, each code becomes scale[g] * (code - zero[g]) in fp32
// and the 32 outputs leave as 16-byte vectors (vec: out and g_idx 16-byte
// aligned).
template <int BITS, typename OutT>
__global__ void dequant_kernel(const int32_t* __restrict__ qweight,
                               const float* __restrict__ scales,
                               const int32_t* __restrict__ zeros,
                               const int32_t* __restrict__ g_idx, int64_t r, int64_t k,
                               int64_t ngroups, int vec, OutT* __restrict__ out) {
  const int64_t runs_per_row = k / 32;
  const int64_t nruns = r * runs_per_row;
  for (int64_t t = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; t < nruns;
       t += (int64_t)gridDim.x * blockDim.x) {
    const int64_t row = t / runs_per_row, run = t % runs_per_row;
    const int32_t* src = qweight + row * (k * BITS / 32) + run * BITS;
    uint32_t in[BITS];
#pragma unroll
    for (int w = 0; w < BITS; ++w) in[w] = (uint32_t)src[w];
    int gi[32];
    if (vec) {
      const int4* gsrc = reinterpret_cast<const int4*>(g_idx + run * 32);
#pragma unroll
      for (int q = 0; q < 8; ++q) {
        const int4 g4 = gsrc[q];
        gi[4 * q] = g4.x, gi[4 * q + 1] = g4.y, gi[4 * q + 2] = g4.z, gi[4 * q + 3] = g4.w;
      }
    } else {
#pragma unroll
      for (int j = 0; j < 32; ++j) gi[j] = g_idx[run * 32 + j];
    }
    const float* srow = scales + row * ngroups;
    const int32_t* zrow = zeros + row * ngroups;
    float v[32];
#pragma unroll
    for (int j = 0; j < 32; ++j) {
      const int bit = j * BITS;
      uint32_t c = in[bit / 32] >> (bit % 32);
      if ((bit % 32) + BITS > 32) c |= in[bit / 32 + 1] << (32 - bit % 32);
      c &= (1u << BITS) - 1u;
      const int g = gi[j];
      v[j] = srow[g] * (float)((int32_t)c - zrow[g]);
    }
    store_run<OutT>(out + row * k + run * 32, v, vec != 0);
  }
}

static unsigned grid_for(int64_t work) {
  int64_t g = cdiv(work, 256);
  if (g > 148 * 64) g = 148 * 64;
  return (unsigned)(g > 0 ? g : 1);
}

gptq_status pack_impl(const uint8_t* codes, int64_t r, int64_t k, int bits, int32_t* qweight,
                      cudaStream_t s) {
  const int64_t work = r * (k / 32);
  if (work == 0) return GPTQ_OK;
  const unsigned g = grid_for(work);
  switch (bits) {
    case 2: pack_kernel<2><<<g, 256, 0, s>>>(codes, r, k, qweight); break;
    case 3: pack_kernel<3><<<g, 256, 0, s>>>(codes, r, k, qweight); break;
    case 4: pack_kernel<4><<<g, 256, 0, s>>>(codes, r, k, qweight); break;
    case 8: pack_kernel<8><<<g, 256, 0, s>>>(codes, r, k, qweight); break;
    default: return GPTQ_ERR_UNSUPPORTED;
  }
  GPTQ_CHECK_LAUNCH();
  return GPTQ_OK;
}

template <typename OutT>
static gptq_status dequant_typed(const int32_t* qweight, const float* scales, const int32_t* zeros,
                                 const int32_t* g_idx, int64_t r, int64_t k, int bits,
                                 int64_t ngroups, OutT* out, cudaStream_t s) {
  const int64_t work = r * (k / 32);
  if (work == 0) return GPTQ_OK;
  const unsigned g = grid_for(work);
  const int vec = ((uintptr_t)out % 16 == 0 && (uintptr_t)g_idx % 16 == 0) ? 1 : 0;
  switch (bits) {
    case 2: dequant_kernel<2, OutT><<<g, 256, 0, s>>>(qweight, scales, zeros, g_idx, r, k, ngroups, vec, out); break;
    case 3: dequant_kernel<3, OutT><<<g, 256, 0, s>>>(qweight, scales, zeros, g_idx, r, k, ngroups, vec, out); break;
    case 4: dequant_kernel<4, OutT><<<g, 256, 0, s>>>(qweight, scales, zeros, g_idx, r, k, ngroups, vec, out); break;
    case 8: dequant_kernel<8, OutT><<<g, 256, 0, s>>>(qweight, scales, zeros, g_idx, r, k, ngroups, vec, out); break;
    default: return GPTQ_ERR_UNSUPPORTED;
  }
  GPTQ_CHECK_LAUNCH();
  return GPTQ_OK;
}

gptq_status dequant_impl(const int32_t* qweight, const float* scales, const int32_t* zeros,
                         const int32_t* g_idx, int64_t r, int64_t k, int bits, int64_t ngroups,
                         gptq_dtype out_dt, void* out, cudaStream_t s) {
  switch (out_dt) {
    case GPTQ_F32:
      return dequant_typed<float>(qweight, scales, zeros, g_idx, r, k, bits, ngroups, (float*)out, s);
    case GPTQ_F16:
      return dequant_typed<__half>(qweight, scales, zeros, g_idx, r, k, bits, ngroups, (__half*)out, s);
    case GPTQ_BF16:
      return dequant_typed<__nv_bfloat16>(qweight, scales, zeros, g_idx, r, k, bits, ngroups,
                                          (__nv_bfloat16*)out, s);
  }
  return GPTQ_ERR_INVALID_ARG;
}

}  // namespace gptq
