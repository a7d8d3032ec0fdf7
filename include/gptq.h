/*
 * gptq.h — C ABI of libgptq_b200, a B200 (sm_100a) implementation of GPTQ
 * layer-wise weight quantization.
 *
 * Sources (web pages on GPTQ, cited by title and section):
 *   [GPTQ-tool]  "GPTQ", ozercemkelahmet.com/tools/gptq — How it works,
 *                Steps 1-9; Optional refinements; A minimal Python sketch;
 *                Memory arithmetic; Glossary.
 *   [GPTQ-guide] "GPTQ Quantization: Complete Technical Guide",
 *                notes.jayaprakash.net — Quantization Equation; Computing the
 *                Hessian; Configuration Deep Dive.
 *   [GPTQ-breakdown] "GPTQ", ai360xpert.com/papers/gptq — How It Works.
 *   [What-is-GPTQ] "What Is GPTQ? Classic 4-Bit LLM Quantization",
 *                ai-tldr.dev — How it works, Step 3.
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 * Pointers.   Every array argument is a DEVICE pointer (memory the caller
 *             allocated with cudaMalloc or a caching allocator on the device
 *             the call runs on) unless its comment says otherwise.  The
 *             library allocates no memory and keeps no per-call state;
 *             scratch memory is the caller's workspace `ws` of at least
 *             gptq_workspace_size(...) bytes, 256-byte aligned.  Process-
 *             wide it only caches the driver's tensor-map encoder entry
 *             point, each kernel's shared-memory opt-in (per device, under a
 *             lock, set on first use) and the wait limit of
 *             gptq_set_wait_limit; gptq_prepare_hinv_noalloc alone uses a
 *             file-scope device scratch array (see there).  Calls may come
 *             from several host threads and for several devices.
 * Layout.     Row-major.  W is (r, k): r = out-features (rows), k =
 *             in-features (columns); X is (n, k): n calibration tokens.
 *             Leading dimensions are in elements.
 * Streams.    Every call enqueues its kernels on `stream` (0 = legacy
 *             default stream) and returns without synchronising.
 * Errors.     Argument errors are detected on the host and returned before
 *             anything is enqueued.  GPTQ_ERR_CUDA means a launch failed
 *             (the CUDA error is left for cudaGetLastError to report).
 *             Failures that only the device can see are written to device
 *             status words (`d_info`, `d_status`) that the caller reads after
 *             synchronising; no kernel traps, asserts or waits without bound.
 * Inputs.     W and X are never modified (gptq_rotate writes `out`, which
 *             is `in` only when the caller asks for an in-place rotation);
 *             H is written only by gptq_hessian_accumulate (H += ...).
 */
#ifndef GPTQ_B200_H
#define GPTQ_B200_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define GPTQ_API __attribute__((visibility("default")))
#else
#define GPTQ_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st* gptq_stream_t; /* == cudaStream_t */

typedef enum {
  GPTQ_OK = 0,
  GPTQ_ERR_INVALID_ARG = 1, /* null pointer, bad size, leading dimension, alignment */
  GPTQ_ERR_NOT_PD = 2,      /* damped Hessian not positive definite (device: d_info) */
  GPTQ_ERR_CUDA = 3,        /* a kernel launch failed */
  GPTQ_ERR_UNSUPPORTED = 4, /* valid request the library does not implement (bits, dtype) */
  GPTQ_ERR_WORKSPACE = 5,   /* workspace null, too small or misaligned */
  GPTQ_ERR_TIMEOUT = 6,     /* a bounded device-side wait gave up */
  GPTQ_ERR_NONFINITE = 7    /* NaN/Inf met in the weights being quantized (device: d_status) */
} gptq_status;

typedef enum { GPTQ_F32 = 0, GPTQ_F16 = 1, GPTQ_BF16 = 2 } gptq_dtype;

/* Quantization settings ([GPTQ-guide] Configuration Deep Dive; [GPTQ-tool]
 * Optional refinements).
 *   bits        2, 3, 4 or 8: codes are 0 .. 2^bits-1 on an asymmetric grid.
 *   group_size  columns (in processing order) sharing one scale/zero per row;
 *               -1 = one group per row.  Must divide block_size or be a
 *               multiple of it, so a group never straddles a lazy block
 *               (any positive size when static_groups is set).
 *   block_size  lazy-batch width B ([GPTQ-tool] Step 7), 16..128, multiple of 16.
 *   percdamp    damping fraction of mean(diag H) ([GPTQ-tool] Step 4), >= 0.
 *   act_order   nonzero: process columns by descending diag(H).
 *   sym         0: asymmetric grid, zero point fitted per group (rint(-min/scale));
 *               1: symmetric grid about 0, scale = 2 max(|min|, |max|) / maxq and
 *               zero point (maxq + 1) / 2 for every group ("GPTQ",
 *               ozercemkelahmet.com/tools/gptq, Optional refinements).
 *               Other values: GPTQ_ERR_INVALID_ARG.
 *   static_groups  0: each group's grid is fitted when the sweep reaches the
 *               group, to the already-compensated weights (groups of
 *               consecutive processing positions; g_idx[c] = position / G).
 *               1: every grid is fitted before the sweep to the original
 *               weights (dead columns as 0) of the original columns
 *               [g G, (g+1) G); a column keeps its original group under
 *               act_order, so g_idx[c] = c / G.  (The static_groups flag of
 *               the AutoGPTQ configuration in "GPTQ Quantization: Complete
 *               Technical Guide", Configuration Deep Dive; its meaning there
 *               is not spelled out and this is the plain reading of the name.)
 *               Other values: GPTQ_ERR_INVALID_ARG. */
typedef struct {
  int bits;
  int group_size;
  int block_size;
  float percdamp;
  int act_order;
  int sym;
  int static_groups;
} gptq_config;

typedef enum {
  GPTQ_OP_HESSIAN = 0,
  GPTQ_OP_PREPARE_HINV = 1,
  GPTQ_OP_QUANTIZE = 2
} gptq_op;

/* Bytes of workspace `op` needs for the given sizes (n is ignored except by
 * GPTQ_OP_HESSIAN; cfg may be NULL for GPTQ_OP_HESSIAN).  0 means none. */
GPTQ_API size_t gptq_workspace_size(int op, int64_t r, int64_t k, int64_t n, const gptq_config* cfg);

/* Human-readable name of a status code (static storage). */
GPTQ_API const char* gptq_status_string(gptq_status s);

/* Hessian accumulation: H += alpha * X^T X.
 * [GPTQ-tool] Step 3 and A minimal Python sketch (H = 2 X^T X / n);
 * [GPTQ-guide] Computing the Hessian.  Call once per chunk of calibration
 * tokens with alpha = 2 / n_total (n_total = tokens over all chunks).
 *   X      (n, k) row-major, dtype `dt`, leading dimension ldx >= k.
 *          F16 / BF16 are accumulated on the tensor cores (exact products,
 *          fp32 accumulation over short token runs, re-accumulated in fp32);
 *          F32 on the CUDA cores in fp32.  F16/BF16 need k % 8 == 0,
 *          ldx % 8 == 0 and a 16-byte aligned X.
 *   H      (k, k) fp32, symmetric on entry (zero it before the first chunk);
 *          both triangles are updated.  Must not alias X.
 *   ws     GPTQ_OP_HESSIAN workspace (256 bytes, 256-byte aligned).  Its
 *          second int32, ((int32_t*)ws)[1], is a device status word the
 *          library only ever sets: GPTQ_ERR_TIMEOUT once a bounded wait of
 *          the tensor-core kernel gave up in this call or an earlier one on
 *          the same workspace (H[0][0] is then NaN as well, so a caller who
 *          never reads the word meets the failure in gptq_prepare_hinv).
 *          Zero it with H before the first chunk; read it after
 *          synchronising.  The first int32 is the library's own.
 * Returns GPTQ_OK, GPTQ_ERR_INVALID_ARG, GPTQ_ERR_WORKSPACE, GPTQ_ERR_CUDA.
 * n == 0 or k == 0 is a no-op. */
GPTQ_API gptq_status gptq_hessian_accumulate(const void* X, gptq_dtype dt, int64_t n, int64_t k,
                                    int64_t ldx, float alpha, float* H, void* ws,
                                    size_t ws_bytes, gptq_stream_t stream);

/* Inverse-Hessian factor with dead columns, act-order and damping.
 * [GPTQ-tool] Steps 4 and 6, Optional refinements (act-order), and the
 * sketch's factor cholesky(cholesky_inverse(cholesky(H)), upper=True).
 *   H       (k, k) fp32 undamped Hessian (read only).
 *   Steps:  dead = {i : H_ii == 0} (those get H_ii := 1; the sweep zeroes
 *           their weights); perm = stable sort of columns by descending
 *           diag(H) if cfg->act_order, else identity; Hp = H[perm][:, perm];
 *           Hp += percdamp * mean(diag Hp) * I; U = upper Cholesky factor of
 *           Hp^-1 (U^T U = Hp^-1), computed as U = V^-1 with Hp = V V^T,
 *           V upper (a bottom-up Cholesky), never forming Hp^-1.
 *   U       (k, k) fp32 out, row-major, in PROCESSING order; lower triangle
 *           written as 0.
 *   perm    int32[k] out: perm[j] = original column processed j-th.
 *   invperm int32[k] out: invperm[perm[j]] = j.
 *   dead    uint8[k] out (original column order): 1 = dead column.
 *   d_info  int32 device scalar out: 0, or 1 + the processing-order index
 *           of the first pivot found non-positive or non-finite (then U is
 *           unspecified; retry with a larger percdamp), or k + 1 when a
 *           bounded wait of a tensor-core update gave up (GPTQ_ERR_TIMEOUT;
 *           U is unspecified).
 *   ws      GPTQ_OP_PREPARE_HINV workspace.
 * Returns GPTQ_OK (the device may still report NOT_PD in d_info),
 * GPTQ_ERR_INVALID_ARG, GPTQ_ERR_WORKSPACE, GPTQ_ERR_CUDA. */
GPTQ_API gptq_status gptq_prepare_hinv(const float* H, int64_t k, const gptq_config* cfg, float* U,
                              int32_t* perm, int32_t* invperm, uint8_t* dead,
                              int32_t* d_info, void* ws, size_t ws_bytes,
                              gptq_stream_t stream);

/* Test hook: the number of polls after which a pipeline wait inside the
 * tensor-core kernels (Hessian, factor and sweep updates, lane sweep, the
 * tensor-core inference product) gives up and takes its error path.  It
 * applies to launches made after the call, from any thread; the waits that
 * let a CTA's own copies and MMAs land before it exits keep their full bound.
 * 0 makes every such wait give up at once (each stage then reports
 * GPTQ_ERR_TIMEOUT as its comment says); GPTQ_WAIT_LIMIT_DEFAULT restores the
 * default (2^26 polls, far beyond any correct wait).  Not for production use:
 * a small limit turns slow waits into failures. */
#define GPTQ_WAIT_LIMIT_DEFAULT 0xFFFFFFFFu
GPTQ_API void gptq_set_wait_limit(uint32_t polls);

/* gptq_prepare_hinv without a workspace, for callers that cannot allocate
 * device memory (the pages have no counterpart: this is an interface
 * convenience, not part of the method).
 * Some callers cannot call cudaMalloc or hand over a workspace: a plugin
 * whose host passes it only its input and output buffers, a process that has
 * carved all device memory into its own arena, or a runtime that forbids
 * allocation after start-up.  This call takes the arguments of
 * gptq_prepare_hinv minus ws / ws_bytes and keeps its scratch in a 4 MiB
 * array of the library's device code, which every device that loads the
 * library holds until the process exits.
 *   k        1 .. 12288; a larger k returns GPTQ_ERR_WORKSPACE (the built-in
 *            scratch is too small) before anything is enqueued.
 *   Result.  perm, invperm, dead and d_info are those of
 *            gptq_prepare_hinv; U agrees with its U within fp32 rounding
 *            (1e-5 relative to max |U|), not bit for bit, because the array
 *            holds less of the rank updates' operand splits than the
 *            workspace does: up to k = 4076 the tensor-core updates run with
 *            one level of 64-column blocks (gptq_prepare_hinv batches 8 of
 *            them per update), and from k = 4080 to 12288 the fp32 CUDA-core
 *            rank update runs instead, which is slower (at k = 4096 about 4x).
 *   Setup.   Host code cannot hand the array's name to a kernel; its device
 *            address comes from cudaGetSymbolAddress, looked up with the
 *            device current on every call made outside stream capture (so a
 *            device reset or a new context is picked up).  A call made while
 *            `stream` is capturing reuses the address of the last call on that
 *            device: make the first call on a device before any capture.
 *   Sharing. All calls share the array and it keeps the last call's
 *            contents (every word is written before it is read, nothing needs
 *            clearing).  Calls whose work overlaps on the GPU (other streams,
 *            other host threads) race on it: serialise them.
 * Returns as gptq_prepare_hinv, with GPTQ_ERR_WORKSPACE for k > 12288. */
GPTQ_API gptq_status gptq_prepare_hinv_noalloc(const float* H, int64_t k, const gptq_config* cfg,
                                               float* U, int32_t* perm, int32_t* invperm,
                                               uint8_t* dead, int32_t* d_info,
                                               gptq_stream_t stream);

/* Lazy-blocked GPTQ column sweep of one layer.
 * [GPTQ-tool] Steps 5, 7 and 8, A minimal Python sketch; [What-is-GPTQ]
 * Step 3 (groups); [GPTQ-breakdown] How It Works (lazy batching).
 * Per block of B = cfg->block_size processing-order columns [s, e): at each
 * group start the row's grid is taken from the current weights of the group
 * (lo = min(0, min w), hi = max(0, max w), scale = max(hi-lo, 1e-8)/maxq,
 * zero = rint(-lo/scale)); each column is coded c = clamp(rint(w/scale) +
 * zero, 0, maxq) (fp32 decisions, ties to even), err = (w - q)/U[i,i] with
 * q = scale*(c - zero), later in-block columns get w_j -= err*U[i,j], and at
 * the block end W[:, e:] -= Err * U[s:e, e:].
 *   W       (r, k) dtype `dt` (F32/F16/BF16), leading dimension ldw >= k,
 *           ORIGINAL column order (read only).
 *   U, perm, dead  as produced by gptq_prepare_hinv for this layer.
 *   H0      (k, k) fp32 undamped Hessian for the layer loss, or NULL.
 *   codes   uint8 (r, k) out, ORIGINAL column order.
 *   scales  fp32 (r, ngroups) out, group index in processing order;
 *           ngroups = ceil(k / group_size) (1 when group_size == -1).
 *   zeros   int32 (r, ngroups) out.
 *   g_idx   int32[k] out: group of each ORIGINAL column.
 *   loss    fp64 device array of r+1 out (may be NULL; ignored when H0 is
 *           NULL): loss[0..r-1] = per-row (w0-q) H0 (w0-q)^T, loss[r] = their
 *           sum ([GPTQ-tool] Step 2 objective; Reading a quantization log).
 *   d_status int32 device scalar out (may be NULL): 0, GPTQ_ERR_NONFINITE
 *           if a non-finite weight was met (its code is then the zero point),
 *           or GPTQ_ERR_TIMEOUT if a bounded device wait gave up (the outputs
 *           are then unspecified).
 *   ws      GPTQ_OP_QUANTIZE workspace (holds the fp32 working copy of W).
 * Returns GPTQ_OK, GPTQ_ERR_INVALID_ARG, GPTQ_ERR_UNSUPPORTED,
 * GPTQ_ERR_WORKSPACE, GPTQ_ERR_CUDA. */
GPTQ_API gptq_status gptq_quantize_layer(const void* W, gptq_dtype dt, int64_t r, int64_t k,
                                int64_t ldw, const float* U, const int32_t* perm,
                                const uint8_t* dead, const float* H0,
                                const gptq_config* cfg, uint8_t* codes, float* scales,
                                int32_t* zeros, int32_t* g_idx, double* loss,
                                int32_t* d_status, void* ws, size_t ws_bytes,
                                gptq_stream_t stream);

/* Pack codes into 32-bit words ([GPTQ-tool] Step 8: eight 4-bit codes per
 * 32-bit word).  Each row's codes form an LSB-first bit stream: code j
 * occupies stream bits [j*bits, (j+1)*bits), stream bit m is bit m%32 of
 * word m/32 (3-bit codes straddle words).
 *   codes   uint8 (r, k), values < 2^bits (higher bits are masked off),
 *           16-byte aligned.
 *   qweight int32 (r, k*bits/32) out.  Needs k % 32 == 0 (then every row
 *           is a whole number of 32-code runs of `bits` words each).
 * Returns GPTQ_OK, GPTQ_ERR_INVALID_ARG, GPTQ_ERR_UNSUPPORTED, GPTQ_ERR_CUDA. */
GPTQ_API gptq_status gptq_pack(const uint8_t* codes, int64_t r, int64_t k, int bits, int32_t* qweight,
                      gptq_stream_t stream);

/* Dequantize packed codes: out[i, c] = scales[i, g] * (code - zeros[i, g]),
 * g = g_idx[c] ([GPTQ-tool] sketch dequantization; [What-is-GPTQ] Step 3).
 * The product is formed in fp32 and rounded to out_dt (F32/F16/BF16).
 *   qweight int32 (r, k*bits/32); scales fp32 / zeros int32 (r, ngroups);
 *   g_idx int32[k] with 0 <= g_idx[c] < ngroups; out (r, k) row-major.
 *   Needs k % 32 == 0.
 * Returns GPTQ_OK, GPTQ_ERR_INVALID_ARG, GPTQ_ERR_UNSUPPORTED, GPTQ_ERR_CUDA. */
GPTQ_API gptq_status gptq_dequant(const int32_t* qweight, const float* scales, const int32_t* zeros,
                         const int32_t* g_idx, int64_t r, int64_t k, int bits,
                         int64_t ngroups, gptq_dtype out_dt, void* out,
                         gptq_stream_t stream);

/* The inference product of a quantized layer, read straight from the packed
 * codes ("GPTQ", ozercemkelahmet.com/tools/gptq: What the output looks like --
 * a GPU kernel reads the packed data and dequantizes inside the matrix
 * multiply; How it works, Step 8; "What Is GPTQ?", ai-tldr.dev, How it works:
 * each group is expanded just in time):
 *   Y[t, j] = sum_c X[t, c] * scales[j, g] * (code[j, c] - zeros[j, g]),
 *   g = g_idx[c], or c / group_size when g_idx is NULL,
 * summed in fp32 and rounded once to dt.
 *   X       (m, k) f16 or bf16 (dt), row-major, leading dimension ldx >= k.
 *   qweight int32 (n, k*bits/32) as written by gptq_pack; n = rows of W
 *           (output features).  k % 32 == 0.
 *   scales  fp32 (n, ngroups); zeros int32 (n, ngroups).
 *   g_idx   int32[k] with 0 <= g_idx[c] < ngroups (an entry outside makes the
 *           affected outputs NaN), or NULL: then group_size (-1 = one group)
 *           defines the groups and ngroups must be ceil(k / group_size).
 *   Y       (m, n) out, dt, row-major, leading dimension ldy >= n.
 *   m <= 131070 tokens.  The library allocates nothing.
 * Kernel choice (all results within the same bounds of the exact product):
 *   m >= 17, 4-bit, g_idx NULL, k >= 64, group_size a multiple of 32 (or one
 *     group per row), X and qweight 16-byte aligned, ldx % 8 == 0: the
 *     tensor-core kernel (each weight formed in dt: the scale rounded to dt
 *     times the exact code - zero, rounded once more; fp32 accumulation);
 *   3 <= m <= 16, 4-bit, g_idx NULL, group_size a multiple of 128 (or one
 *     group per row), qweight 16-byte aligned: the small-batch kernel
 *     (mma.sync, weights streamed once for all tokens and formed in dt as in
 *     the tensor-core kernel; fp32 accumulation);
 *   else g_idx NULL, bits 2/4/8 and group_size a multiple of 128/bits (or one
 *     group per row): the decode kernel (weights streamed once per 8 tokens,
 *     each product x (code - zero) exact in fp32);
 *   every other case: the general kernel (fp32 weights per element).
 * Returns GPTQ_OK, GPTQ_ERR_INVALID_ARG, GPTQ_ERR_UNSUPPORTED (bits, f32 X),
 * GPTQ_ERR_CUDA. */
GPTQ_API gptq_status gptq_gemm(const void* X, gptq_dtype dt, int64_t m, int64_t k, int64_t ldx,
                      const int32_t* qweight, const float* scales, const int32_t* zeros,
                      const int32_t* g_idx, int64_t n, int bits, int group_size,
                      int64_t ngroups, void* Y, int64_t ldy, gptq_stream_t stream);

/* Rotation preprocessing ("GPTQ", ozercemkelahmet.com/tools/gptq, Variants
 * and extensions: weights and activations multiplied by an orthogonal matrix
 * before quantizing so that outliers spread out).  Every row x of `in`
 * becomes
 *   x Q = (x * s) H_b / sqrt(b),  or with inverse != 0,  x Q^T = (x H_b / sqrt(b)) * s,
 * Q = diag(s) H_b / sqrt(b) orthogonal, s[c] = -1 where signs[c] < 0 and +1
 * elsewhere, H_b the block-diagonal Sylvester Hadamard matrix of order b
 * (block).  Rotating W (r, k) and X (n, k) alike keeps X W^T; the Hessian of
 * the rotated X is Q^T H Q.  Arithmetic in fp32, rounded once to dt.
 *   in, out  (rows, k) dt (F32/F16/BF16), row strides ld_in, ld_out >= k
 *            (elements; rows 16-byte aligned).  in == out with ld_in ==
 *            ld_out rotates in place; other overlaps are rejected.
 *   signs    int8[k] device array, 8-byte aligned.
 *   block    b: a power of two from 256 to 8192 dividing k (else
 *            GPTQ_ERR_UNSUPPORTED / GPTQ_ERR_INVALID_ARG).
 * Returns GPTQ_OK, GPTQ_ERR_INVALID_ARG, GPTQ_ERR_UNSUPPORTED, GPTQ_ERR_CUDA. */
GPTQ_API gptq_status gptq_rotate(const void* in, gptq_dtype dt, int64_t rows, int64_t k,
                        int64_t ld_in, const int8_t* signs, int block, int inverse, void* out,
                        int64_t ld_out, gptq_stream_t stream);

/* Measured peak rates of the current device, for roofline fractions (a
 * calibration utility, not part of the method): fp32 FMA on the CUDA cores
 * (packed fp32x2 FMA chains on every SM) and kind::tf32 MMAs on the tensor
 * cores (M = 128, N = 256, K = 8 back to back, one issuing thread per SM), in
 * TFLOP/s (2 flops per multiply-add), each from one launch timed with events
 * after a warm-up launch.  Runs on the legacy default stream and waits for it.
 * Allocates nothing (two file-scope device words).
 *   fp32_tflops, tf32_tflops  host pointers, written on GPTQ_OK.
 * Returns GPTQ_OK, GPTQ_ERR_INVALID_ARG, GPTQ_ERR_CUDA, GPTQ_ERR_TIMEOUT (an
 * MMA wait gave up). */
GPTQ_API gptq_status gptq_measure_peaks(double* fp32_tflops, double* tf32_tflops);

#ifdef __cplusplus
}
#endif

#endif /* GPTQ_B200_H */
