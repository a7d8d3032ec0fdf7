// extern "C" entry points of libgptq_b200: argument checks, workspace
// carving and dispatch to the kernels.  Every check here runs on the host,
// before anything is enqueued.
#include "common.cuh"

#include <algorithm>

namespace gptq {
gptq_status hessian_simt(const void* X, gptq_dtype dt, int64_t n, int64_t k, int64_t ldx,
                         float alpha, float* H, cudaStream_t s);
gptq_status hessian_tc(const void* X, gptq_dtype dt, int64_t n, int64_t k, int64_t ldx,
                       float alpha, float* H, void* ws, cudaStream_t s);
bool hessian_tc_supported(gptq_dtype dt, int64_t n, int64_t k, int64_t ldx, const void* X,
                          const float* H);
size_t hessian_tc_workspace_bytes(int64_t k, int64_t n);
size_t hinv_workspace_bytes(int64_t k);
gptq_status prepare_hinv_impl(const float* H, int64_t k, const gptq_config* cfg, float* U,
                              int32_t* perm, int32_t* invperm, uint8_t* dead, int32_t* d_info,
                              void* ws, size_t ws_bytes, cudaStream_t s);
size_t sweep_workspace_bytes(int64_t r, int64_t k, int B, int G, bool static_groups);
gptq_status quantize_layer_impl(const void* W, gptq_dtype dt, int64_t r, int64_t k, int64_t ldw,
                                const float* U, const int32_t* perm, const uint8_t* dead,
                                const float* H0, const gptq_config* cfg, uint8_t* codes,
                                float* scales, int32_t* zeros, int32_t* g_idx, double* loss,
                                int32_t* d_status, void* ws, cudaStream_t s);
gptq_status pack_impl(const uint8_t* codes, int64_t r, int64_t k, int bits, int32_t* qweight,
                      cudaStream_t s);
gptq_status dequant_impl(const int32_t* qweight, const float* scales, const int32_t* zeros,
                         const int32_t* g_idx, int64_t r, int64_t k, int bits, int64_t ngroups,
                         gptq_dtype out_dt, void* out, cudaStream_t s);
gptq_status gemm_impl(const void* X, gptq_dtype dt, int64_t m, int64_t k, int64_t ldx,
                      const int32_t* qweight, const float* scales, const int32_t* zeros,
                      const int32_t* g_idx, int64_t n, int bits, int group_size, int64_t ngroups,
                      void* Y, int64_t ldy, cudaStream_t s);
gptq_status rotate_impl(const void* in, gptq_dtype dt, int64_t rows, int64_t k, int64_t ld_in,
                        const int8_t* signs, int block, int inverse, void* out, int64_t ld_out,
                        cudaStream_t s);
}  // namespace gptq

using namespace gptq;

namespace {

constexpr int64_t kMaxDim = (int64_t)1 << 20;  // k and r limit (int indexing inside kernels)
constexpr int64_t kGemmMaxTokens = (int64_t)65535 * 2;  // token pairs on the grid's y axis

bool valid_dtype(gptq_dtype dt) { return dt == GPTQ_F32 || dt == GPTQ_F16 || dt == GPTQ_BF16; }

bool valid_bits(int b) { return b == 2 || b == 3 || b == 4 || b == 8; }

// Checks a config against k; returns GPTQ_OK, INVALID_ARG or UNSUPPORTED.
gptq_status check_config(const gptq_config* cfg, int64_t k) {
  if (cfg == nullptr) return GPTQ_ERR_INVALID_ARG;
  if (!valid_bits(cfg->bits)) return GPTQ_ERR_UNSUPPORTED;
  if (cfg->sym != 0 && cfg->sym != 1) return GPTQ_ERR_INVALID_ARG;
  if (cfg->static_groups != 0 && cfg->static_groups != 1) return GPTQ_ERR_INVALID_ARG;
  if (!(cfg->percdamp >= 0.0f) || !isfinite(cfg->percdamp)) return GPTQ_ERR_INVALID_ARG;
  const int B = cfg->block_size;
  if (B < 16 || B > 128 || B % 16 != 0) return GPTQ_ERR_UNSUPPORTED;
  const int G = cfg->group_size;
  if (G != -1) {
    if (G <= 0) return GPTQ_ERR_INVALID_ARG;
    // dynamic grids are fitted at a group's start inside one lazy block
    if (!cfg->static_groups && !(B % G == 0 || G % B == 0)) return GPTQ_ERR_INVALID_ARG;
  }
  (void)k;
  return GPTQ_OK;
}

bool aligned(const void* p, size_t a) { return ((uintptr_t)p % a) == 0; }

size_t dtype_bytes(gptq_dtype dt) { return dt == GPTQ_F32 ? 4 : 2; }

}  // namespace

extern "C" {

const char* gptq_status_string(gptq_status s) {
  switch (s) {
    case GPTQ_OK: return "GPTQ_OK";
    case GPTQ_ERR_INVALID_ARG: return "GPTQ_ERR_INVALID_ARG";
    case GPTQ_ERR_NOT_PD: return "GPTQ_ERR_NOT_PD";
    case GPTQ_ERR_CUDA: return "GPTQ_ERR_CUDA";
    case GPTQ_ERR_UNSUPPORTED: return "GPTQ_ERR_UNSUPPORTED";
    case GPTQ_ERR_WORKSPACE: return "GPTQ_ERR_WORKSPACE";
    case GPTQ_ERR_TIMEOUT: return "GPTQ_ERR_TIMEOUT";
    case GPTQ_ERR_NONFINITE: return "GPTQ_ERR_NONFINITE";
  }
  return "GPTQ_ERR_UNKNOWN";
}

size_t gptq_workspace_size(int op, int64_t r, int64_t k, int64_t n, const gptq_config* cfg) {
  if (k < 0 || r < 0 || n < 0 || k > kMaxDim || r > kMaxDim) return 0;
  switch (op) {
    case GPTQ_OP_HESSIAN:
      return hessian_tc_workspace_bytes(k, n);
    case GPTQ_OP_PREPARE_HINV:
      return hinv_workspace_bytes(k);
    case GPTQ_OP_QUANTIZE:
      if (cfg == nullptr) return 0;
      return sweep_workspace_bytes(r, k, cfg->block_size, cfg->group_size, cfg->static_groups != 0);
  }
  return 0;
}

gptq_status gptq_hessian_accumulate(const void* X, gptq_dtype dt, int64_t n, int64_t k,
                                    int64_t ldx, float alpha, float* H, void* ws,
                                    size_t ws_bytes, gptq_stream_t stream) {
  if (!valid_dtype(dt)) return GPTQ_ERR_INVALID_ARG;
  if (n < 0 || k < 0 || k > kMaxDim || ldx < k) return GPTQ_ERR_INVALID_ARG;
  if (n == 0 || k == 0) return GPTQ_OK;
  if (X == nullptr || H == nullptr) return GPTQ_ERR_INVALID_ARG;
  if (!aligned(X, dtype_bytes(dt)) || !aligned(H, 4)) return GPTQ_ERR_INVALID_ARG;
  cudaStream_t s = (cudaStream_t)stream;
  if (hessian_tc_supported(dt, n, k, ldx, X, H)) {
    size_t need = hessian_tc_workspace_bytes(k, n);
    if (need > 0 && (ws == nullptr || ws_bytes < need || !aligned(ws, 256)))
      return GPTQ_ERR_WORKSPACE;
    return hessian_tc(X, dt, n, k, ldx, alpha, H, ws, s);
  }
  return hessian_simt(X, dt, n, k, ldx, alpha, H, s);
}

gptq_status gptq_prepare_hinv(const float* H, int64_t k, const gptq_config* cfg, float* U,
                              int32_t* perm, int32_t* invperm, uint8_t* dead, int32_t* d_info,
                              void* ws, size_t ws_bytes, gptq_stream_t stream) {
  if (k <= 0 || k > kMaxDim) return GPTQ_ERR_INVALID_ARG;
  if (H == nullptr || U == nullptr || perm == nullptr || invperm == nullptr || dead == nullptr ||
      d_info == nullptr || cfg == nullptr)
    return GPTQ_ERR_INVALID_ARG;
  if (!(cfg->percdamp >= 0.0f) || !isfinite(cfg->percdamp)) return GPTQ_ERR_INVALID_ARG;
  if ((const void*)H == (const void*)U) return GPTQ_ERR_INVALID_ARG;
  size_t need = hinv_workspace_bytes(k);
  if (ws == nullptr || ws_bytes < need || !aligned(ws, 256)) return GPTQ_ERR_WORKSPACE;
  return prepare_hinv_impl(H, k, cfg, U, perm, invperm, dead, d_info, ws, ws_bytes,
                           (cudaStream_t)stream);
}

gptq_status gptq_quantize_layer(const void* W, gptq_dtype dt, int64_t r, int64_t k, int64_t ldw,
                                const float* U, const int32_t* perm, const uint8_t* dead,
                                const float* H0, const gptq_config* cfg, uint8_t* codes,
                                float* scales, int32_t* zeros, int32_t* g_idx, double* loss,
                                int32_t* d_status, void* ws, size_t ws_bytes,
                                gptq_stream_t stream) {
  if (!valid_dtype(dt)) return GPTQ_ERR_INVALID_ARG;
  if (r <= 0 || k <= 0 || r > kMaxDim || k > kMaxDim || ldw < k) return GPTQ_ERR_INVALID_ARG;
  if ((int64_t)r * k > ((int64_t)1 << 34)) return GPTQ_ERR_UNSUPPORTED;
  gptq_status st = check_config(cfg, k);
  if (st != GPTQ_OK) return st;
  if (W == nullptr || U == nullptr || perm == nullptr || dead == nullptr || codes == nullptr ||
      scales == nullptr || zeros == nullptr || g_idx == nullptr)
    return GPTQ_ERR_INVALID_ARG;
  if (!aligned(W, dtype_bytes(dt))) return GPTQ_ERR_INVALID_ARG;
  size_t need = sweep_workspace_bytes(r, k, cfg->block_size, cfg->group_size,
                                      cfg->static_groups != 0);
  if (ws == nullptr || ws_bytes < need || !aligned(ws, 256)) return GPTQ_ERR_WORKSPACE;
  return quantize_layer_impl(W, dt, r, k, ldw, U, perm, dead, H0, cfg, codes, scales, zeros, g_idx,
                             loss, d_status, ws, (cudaStream_t)stream);
}

gptq_status gptq_pack(const uint8_t* codes, int64_t r, int64_t k, int bits, int32_t* qweight,
                      gptq_stream_t stream) {
  if (!valid_bits(bits)) return GPTQ_ERR_UNSUPPORTED;
  if (r < 0 || k < 0 || k % 32 != 0) return GPTQ_ERR_INVALID_ARG;
  if (r == 0 || k == 0) return GPTQ_OK;
  if (codes == nullptr || qweight == nullptr) return GPTQ_ERR_INVALID_ARG;
  if (!aligned(codes, 16) || !aligned(qweight, 4)) return GPTQ_ERR_INVALID_ARG;
  return pack_impl(codes, r, k, bits, qweight, (cudaStream_t)stream);
}

gptq_status gptq_dequant(const int32_t* qweight, const float* scales, const int32_t* zeros,
                         const int32_t* g_idx, int64_t r, int64_t k, int bits, int64_t ngroups,
                         gptq_dtype out_dt, void* out, gptq_stream_t stream) {
  if (!valid_bits(bits)) return GPTQ_ERR_UNSUPPORTED;
  if (!valid_dtype(out_dt)) return GPTQ_ERR_INVALID_ARG;
  if (r < 0 || k < 0 || k % 32 != 0 || ngroups < 0) return GPTQ_ERR_INVALID_ARG;
  if (r == 0 || k == 0) return GPTQ_OK;
  if (ngroups == 0 || qweight == nullptr || scales == nullptr || zeros == nullptr ||
      g_idx == nullptr || out == nullptr)
    return GPTQ_ERR_INVALID_ARG;
  if (!aligned(out, dtype_bytes(out_dt))) return GPTQ_ERR_INVALID_ARG;
  return dequant_impl(qweight, scales, zeros, g_idx, r, k, bits, ngroups, out_dt, out,
                      (cudaStream_t)stream);
}

gptq_status gptq_gemm(const void* X, gptq_dtype dt, int64_t m, int64_t k, int64_t ldx,
                      const int32_t* qweight, const float* scales, const int32_t* zeros,
                      const int32_t* g_idx, int64_t n, int bits, int group_size, int64_t ngroups,
                      void* Y, int64_t ldy, gptq_stream_t stream) {
  if (!valid_bits(bits)) return GPTQ_ERR_UNSUPPORTED;
  if (dt == GPTQ_F32) return GPTQ_ERR_UNSUPPORTED;
  if (!valid_dtype(dt)) return GPTQ_ERR_INVALID_ARG;
  if (m < 0 || n < 0 || k < 0 || k % 32 != 0 || k > kMaxDim || n > kMaxDim) return GPTQ_ERR_INVALID_ARG;
  if (m > kGemmMaxTokens) return GPTQ_ERR_INVALID_ARG;
  if (group_size != -1 && group_size <= 0) return GPTQ_ERR_INVALID_ARG;
  if (m == 0 || n == 0) return GPTQ_OK;
  if (ldx < k || ldy < n) return GPTQ_ERR_INVALID_ARG;
  if (X == nullptr || Y == nullptr || qweight == nullptr || scales == nullptr ||
      zeros == nullptr || ngroups <= 0)
    return GPTQ_ERR_INVALID_ARG;
  if (g_idx == nullptr) {
    const int64_t G = group_size == -1 ? std::max<int64_t>(k, 1) : group_size;
    if (ngroups != std::max<int64_t>(cdiv(k, G), 1)) return GPTQ_ERR_INVALID_ARG;
  }
  if (!aligned(X, 2) || !aligned(Y, 2) || !aligned(qweight, 4)) return GPTQ_ERR_INVALID_ARG;
  return gemm_impl(X, dt, m, k, ldx, qweight, scales, zeros, g_idx, n, bits, group_size, ngroups,
                   Y, ldy, (cudaStream_t)stream);
}

gptq_status gptq_rotate(const void* in, gptq_dtype dt, int64_t rows, int64_t k, int64_t ld_in,
                        const int8_t* signs, int block, int inverse, void* out, int64_t ld_out,
                        gptq_stream_t stream) {
  if (!valid_dtype(dt)) return GPTQ_ERR_INVALID_ARG;
  if (block < 256 || block > 8192 || (block & (block - 1)) != 0) return GPTQ_ERR_UNSUPPORTED;
  if (rows < 0 || k <= 0 || k % block != 0 || k > kMaxDim) return GPTQ_ERR_INVALID_ARG;
  if (rows == 0) return GPTQ_OK;
  if (in == nullptr || out == nullptr || signs == nullptr) return GPTQ_ERR_INVALID_ARG;
  if (ld_in < k || ld_out < k) return GPTQ_ERR_INVALID_ARG;
  const size_t es = dtype_bytes(dt);
  if (!aligned(in, 16) || !aligned(out, 16) || !aligned(signs, 8) ||
      ((size_t)ld_in * es) % 16 != 0 || ((size_t)ld_out * es) % 16 != 0)
    return GPTQ_ERR_INVALID_ARG;
  if (rows * (k / block) > (int64_t)INT32_MAX) return GPTQ_ERR_INVALID_ARG;
  if (in != out || ld_in != ld_out) {  // distinct buffers must not overlap
    const char* a = (const char*)in;
    const char* b = (const char*)out;
    const size_t na = ((size_t)(rows - 1) * ld_in + k) * es, nb = ((size_t)(rows - 1) * ld_out + k) * es;
    if (a < b + nb && b < a + na) return GPTQ_ERR_INVALID_ARG;
  }
  return rotate_impl(in, dt, rows, k, ld_in, signs, block, inverse != 0, out, ld_out,
                     (cudaStream_t)stream);
}

}  // extern "C"
