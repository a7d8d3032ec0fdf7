// Rotation preprocessing ("GPTQ", ozercemkelahmet.com/tools/gptq, Variants
// and extensions: weights and activations multiplied by an orthogonal matrix
// before quantizing, so that outliers spread out).  Each row x becomes
//   x Q = (x * s) H_b / sqrt(b)        (inverse: x Q^T = (x H_b / sqrt(b)) * s)
// with s a vector of random signs and H_b the block-diagonal Sylvester
// Hadamard matrix of order b: a fast Walsh-Hadamard transform of every b
// columns.  The work is a stream over the rows (bound by HBM), so it runs on
// the CUDA cores: one CTA per (row, block of b columns), 8 contiguous
// elements per thread (one 16-byte load for 16-bit types); the butterflies of
// the lowest 3 index bits run in registers, the next 5 across the lanes of a
// warp (shuffles), the rest across warps through one shared-memory transpose
// (every one of the 256 positions of a warp's chunk takes its W values).
#include "common.cuh"

namespace gptq {

namespace {

template <typename T> __device__ __forceinline__ void load8(const T* p, float (&v)[8]);
template <> __device__ __forceinline__ void load8<float>(const float* p, float (&v)[8]) {
  const float4 a = reinterpret_cast<const float4*>(p)[0], b = reinterpret_cast<const float4*>(p)[1];
  v[0] = a.x, v[1] = a.y, v[2] = a.z, v[3] = a.w, v[4] = b.x, v[5] = b.y, v[6] = b.z, v[7] = b.w;
}
template <> __device__ __forceinline__ void load8<__half>(const __half* p, float (&v)[8]) {
  const uint4 u = *reinterpret_cast<const uint4*>(p);
  const __half2* h = reinterpret_cast<const __half2*>(&u);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float2 f = __half22float2(h[i]);
    v[2 * i] = f.x, v[2 * i + 1] = f.y;
  }
}
template <> __device__ __forceinline__ void load8<__nv_bfloat16>(const __nv_bfloat16* p, float (&v)[8]) {
  const uint4 u = *reinterpret_cast<const uint4*>(p);
  const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&u);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float2 f = __bfloat1622float2(h[i]);
    v[2 * i] = f.x, v[2 * i + 1] = f.y;
  }
}

template <typename T> __device__ __forceinline__ void store8(T* p, const float (&v)[8]);
template <> __device__ __forceinline__ void store8<float>(float* p, const float (&v)[8]) {
  reinterpret_cast<float4*>(p)[0] = make_float4(v[0], v[1], v[2], v[3]);
  reinterpret_cast<float4*>(p)[1] = make_float4(v[4], v[5], v[6], v[7]);
}
template <> __device__ __forceinline__ void store8<__half>(__half* p, const float (&v)[8]) {
  uint4 u;
  __half2* h = reinterpret_cast<__half2*>(&u);
#pragma unroll
  for (int i = 0; i < 4; ++i) h[i] = __floats2half2_rn(v[2 * i], v[2 * i + 1]);
  *reinterpret_cast<uint4*>(p) = u;
}
template <> __device__ __forceinline__ void store8<__nv_bfloat16>(__nv_bfloat16* p, const float (&v)[8]) {
  uint4 u;
  __nv_bfloat162* h = reinterpret_cast<__nv_bfloat162*>(&u);
#pragma unroll
  for (int i = 0; i < 4; ++i) h[i] = __floats2bfloat162_rn(v[2 * i], v[2 * i + 1]);
  *reinterpret_cast<uint4*>(p) = u;
}

// W warps per CTA: a block of b = 256 W columns.
template <typename T, int W>
__global__ void __launch_bounds__(W * 32)
rotate_kernel(const T* __restrict__ in, int64_t ld_in, const int8_t* __restrict__ signs,
              int nblk, int inverse, float scale, T* __restrict__ out, int64_t ld_out) {
  constexpr int B = W * 256;
  __shared__ __align__(16) float sm[W > 1 ? B : 4];
  const int64_t row = blockIdx.x / nblk;
  const int blk = blockIdx.x % nblk;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int c0 = blk * B + tid * 8;
  float v[8];
  load8<T>(in + row * ld_in + c0, v);
  const uint2 sb = *reinterpret_cast<const uint2*>(signs + c0);
  float sg[8];
#pragma unroll
  for (int e = 0; e < 8; ++e) {
    const int8_t sv = (int8_t)(((e < 4 ? sb.x : sb.y) >> (8 * (e & 3))) & 0xFF);
    sg[e] = sv < 0 ? -1.f : 1.f;
  }
  if (!inverse) {
#pragma unroll
    for (int e = 0; e < 8; ++e) v[e] *= sg[e];
  }
  // index bits 0..2: inside the thread
#pragma unroll
  for (int h = 1; h < 8; h <<= 1)
#pragma unroll
    for (int e = 0; e < 8; ++e)
      if ((e & h) == 0) {
        const float a = v[e], b = v[e + h];
        v[e] = a + b;
        v[e + h] = a - b;
      }
  // index bits 3..7: lane bits 0..4
#pragma unroll
  for (int m = 1; m < 32; m <<= 1) {
    const bool upper = (lane & m) != 0;
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      const float u = __shfl_xor_sync(0xffffffffu, v[e], m);
      v[e] = upper ? u - v[e] : v[e] + u;
    }
  }
  // index bits 8 and up: warp bits, through shared memory
  if (W > 1) {
    float4* s4 = reinterpret_cast<float4*>(sm + warp * 256 + lane * 8);
    s4[0] = make_float4(v[0], v[1], v[2], v[3]);
    s4[1] = make_float4(v[4], v[5], v[6], v[7]);
    __syncthreads();
    // 256 positions (lane 8 + e), each with its W values; fewer than 256
    // threads (W < 8) take several positions
    for (int pos = tid; pos < 256; pos += W * 32) {
      float u[W];
#pragma unroll
      for (int w = 0; w < W; ++w) u[w] = sm[w * 256 + pos];
#pragma unroll
      for (int h = 1; h < W; h <<= 1)
#pragma unroll
        for (int w = 0; w < W; ++w)
          if ((w & h) == 0) {
            const float a = u[w], b = u[w + h];
            u[w] = a + b;
            u[w + h] = a - b;
          }
#pragma unroll
      for (int w = 0; w < W; ++w) sm[w * 256 + pos] = u[w];
    }
    __syncthreads();
    const float4 a = s4[0], b = s4[1];
    v[0] = a.x, v[1] = a.y, v[2] = a.z, v[3] = a.w, v[4] = b.x, v[5] = b.y, v[6] = b.z, v[7] = b.w;
  }
#pragma unroll
  for (int e = 0; e < 8; ++e) {
    v[e] *= scale;
    if (inverse) v[e] *= sg[e];
  }
  store8<T>(out + row * ld_out + c0, v);
}

template <typename T, int W>
gptq_status launch_rotate(const T* in, int64_t ld_in, const int8_t* signs, int64_t rows,
                          int64_t k, int inverse, T* out, int64_t ld_out, cudaStream_t s) {
  constexpr int B = W * 256;
  const int nblk = (int)(k / B);
  const float scale = 1.0f / sqrtf((float)B);
  rotate_kernel<T, W><<<(unsigned)(rows * nblk), W * 32, 0, s>>>(in, ld_in, signs, nblk, inverse,
                                                                   scale, out, ld_out);
  GPTQ_CHECK_LAUNCH();
  return GPTQ_OK;
}

template <typename T>
gptq_status rotate_typed(const T* in, int64_t ld_in, const int8_t* signs, int64_t rows, int64_t k,
                         int block, int inverse, T* out, int64_t ld_out, cudaStream_t s) {
  switch (block) {
    case 256: return launch_rotate<T, 1>(in, ld_in, signs, rows, k, inverse, out, ld_out, s);
    case 512: return launch_rotate<T, 2>(in, ld_in, signs, rows, k, inverse, out, ld_out, s);
    case 1024: return launch_rotate<T, 4>(in, ld_in, signs, rows, k, inverse, out, ld_out, s);
    case 2048: return launch_rotate<T, 8>(in, ld_in, signs, rows, k, inverse, out, ld_out, s);
    case 4096: return launch_rotate<T, 16>(in, ld_in, signs, rows, k, inverse, out, ld_out, s);
    case 8192: return launch_rotate<T, 32>(in, ld_in, signs, rows, k, inverse, out, ld_out, s);
  }
  return GPTQ_ERR_UNSUPPORTED;
}

}  // namespace

gptq_status rotate_impl(const void* in, gptq_dtype dt, int64_t rows, int64_t k, int64_t ld_in,
                        const int8_t* signs, int block, int inverse, void* out, int64_t ld_out,
                        cudaStream_t s) {
  switch (dt) {
    case GPTQ_F32:
      return rotate_typed<float>((const float*)in, ld_in, signs, rows, k, block, inverse,
                                 (float*)out, ld_out, s);
    case GPTQ_F16:
      return rotate_typed<__half>((const __half*)in, ld_in, signs, rows, k, block, inverse,
                                  (__half*)out, ld_out, s);
    case GPTQ_BF16:
      return rotate_typed<__nv_bfloat16>((const __nv_bfloat16*)in, ld_in, signs, rows, k, block,
                                         inverse, (__nv_bfloat16*)out, ld_out, s);
  }
  return GPTQ_ERR_INVALID_ARG;
}

}  // namespace gptq
