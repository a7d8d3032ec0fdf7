"""ctypes binding of libgptq_b200.so: argument marshalling only.

Each function here takes torch tensors (device memory owned by the caller),
passes their pointers, sizes and the current CUDA stream to the C ABI entry of
the same name (declared in include/gptq.h), and turns a non-OK status into a
``GptqError``.  No arithmetic of the method happens in Python, and there is no
CPU fallback: if the library or a CUDA device is missing, every call raises.
"""

from __future__ import annotations

import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libgptq_b200.so")

GPTQ_OK = 0
GPTQ_ERR_INVALID_ARG = 1
GPTQ_ERR_NOT_PD = 2
GPTQ_ERR_CUDA = 3
GPTQ_ERR_UNSUPPORTED = 4
GPTQ_ERR_WORKSPACE = 5
GPTQ_ERR_TIMEOUT = 6
GPTQ_ERR_NONFINITE = 7

GPTQ_F32, GPTQ_F16, GPTQ_BF16 = 0, 1, 2
OP_HESSIAN, OP_PREPARE_HINV, OP_QUANTIZE = 0, 1, 2

EXPORTED = (
    "gptq_workspace_size",
    "gptq_status_string",
    "gptq_hessian_accumulate",
    "gptq_prepare_hinv",
    "gptq_prepare_hinv_noalloc",
    "gptq_quantize_layer",
    "gptq_pack",
    "gptq_dequant",
    "gptq_gemm",
    "gptq_rotate",
    "gptq_set_wait_limit",
    "gptq_measure_peaks",
)

WAIT_LIMIT_DEFAULT = 0xFFFFFFFF

_DTYPES = {torch.float32: GPTQ_F32, torch.float16: GPTQ_F16, torch.bfloat16: GPTQ_BF16}


class GptqError(RuntimeError):
    def __init__(self, status: int, where: str, detail: str = ""):
        self.status = int(status)
        name = _status_name(status)
        super().__init__(f"{where}: {name}" + (f" ({detail})" if detail else ""))


class NotPositiveDefinite(GptqError):
    pass


class GptqConfig(ctypes.Structure):
    _fields_ = [
        ("bits", ctypes.c_int),
        ("group_size", ctypes.c_int),
        ("block_size", ctypes.c_int),
        ("percdamp", ctypes.c_float),
        ("act_order", ctypes.c_int),
        ("sym", ctypes.c_int),
        ("static_groups", ctypes.c_int),
    ]


def make_config(bits=4, group_size=128, block_size=128, percdamp=0.01, act_order=False,
                sym=False, static_groups=False):
    return GptqConfig(int(bits), int(group_size), int(block_size), float(percdamp),
                      int(bool(act_order)), int(bool(sym)), int(bool(static_groups)))


_lib = None


def load(path: str = LIB_PATH):
    """Load the shared library (once).  Raises if it has not been built."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise ImportError(f"libgptq_b200.so not built at {path}; run "
                          "`python -m post_weight_quantization_23_b200.build`")
    lib = ctypes.CDLL(path)
    vp, i64, sz, i32 = ctypes.c_void_p, ctypes.c_int64, ctypes.c_size_t, ctypes.c_int
    cfgp = ctypes.POINTER(GptqConfig)
    lib.gptq_workspace_size.restype = sz
    lib.gptq_workspace_size.argtypes = [i32, i64, i64, i64, cfgp]
    lib.gptq_status_string.restype = ctypes.c_char_p
    lib.gptq_status_string.argtypes = [i32]
    lib.gptq_hessian_accumulate.restype = i32
    lib.gptq_hessian_accumulate.argtypes = [vp, i32, i64, i64, i64, ctypes.c_float, vp, vp, sz, vp]
    lib.gptq_prepare_hinv.restype = i32
    lib.gptq_prepare_hinv.argtypes = [vp, i64, cfgp, vp, vp, vp, vp, vp, vp, sz, vp]
    lib.gptq_prepare_hinv_noalloc.restype = i32
    lib.gptq_prepare_hinv_noalloc.argtypes = [vp, i64, cfgp, vp, vp, vp, vp, vp, vp]
    lib.gptq_quantize_layer.restype = i32
    lib.gptq_quantize_layer.argtypes = [vp, i32, i64, i64, i64, vp, vp, vp, vp, cfgp, vp, vp, vp,
                                        vp, vp, vp, vp, sz, vp]
    lib.gptq_pack.restype = i32
    lib.gptq_pack.argtypes = [vp, i64, i64, i32, vp, vp]
    lib.gptq_dequant.restype = i32
    lib.gptq_dequant.argtypes = [vp, vp, vp, vp, i64, i64, i32, i64, i32, vp, vp]
    lib.gptq_gemm.restype = i32
    lib.gptq_gemm.argtypes = [vp, i32, i64, i64, i64, vp, vp, vp, vp, i64, i32, i32, i64, vp, i64,
                              vp]
    lib.gptq_rotate.restype = i32
    lib.gptq_rotate.argtypes = [vp, i32, i64, i64, i64, vp, i32, i32, vp, i64, vp]
    lib.gptq_set_wait_limit.restype = None
    lib.gptq_set_wait_limit.argtypes = [ctypes.c_uint32]
    lib.gptq_measure_peaks.restype = i32
    lib.gptq_measure_peaks.argtypes = [ctypes.POINTER(ctypes.c_double),
                                       ctypes.POINTER(ctypes.c_double)]
    _lib = lib
    return lib


def _status_name(st: int) -> str:
    try:
        return load().gptq_status_string(int(st)).decode()
    except Exception:  # pragma: no cover - library missing
        return f"status {st}"


def _check(st: int, where: str):
    if st != GPTQ_OK:
        raise GptqError(st, where)


def _ptr(t):
    if t is None:
        return None
    if not t.is_cuda:
        raise GptqError(GPTQ_ERR_INVALID_ARG, "binding", "tensor not on a CUDA device")
    return ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def dtype_code(dt: torch.dtype) -> int:
    if dt not in _DTYPES:
        raise GptqError(GPTQ_ERR_INVALID_ARG, "binding", f"dtype {dt}")
    return _DTYPES[dt]


def workspace_size(op: int, r: int, k: int, n: int, cfg: GptqConfig | None) -> int:
    return int(load().gptq_workspace_size(op, r, k, n, ctypes.byref(cfg) if cfg is not None else None))


def hessian_accumulate(X, H, alpha, ws=None, stream=None):
    n, k = X.shape
    ldx = X.stride(0)
    if X.stride(1) != 1:
        raise GptqError(GPTQ_ERR_INVALID_ARG, "gptq_hessian_accumulate", "X rows must be contiguous")
    st = load().gptq_hessian_accumulate(_ptr(X), dtype_code(X.dtype), n, k, ldx, float(alpha),
                                        _ptr(H), _ptr(ws), ws.numel() * ws.element_size() if ws is not None else 0,
                                        _stream(stream))
    _check(st, "gptq_hessian_accumulate")


def prepare_hinv(H, cfg, U, perm, invperm, dead, d_info, ws, stream=None):
    k = H.shape[0]
    st = load().gptq_prepare_hinv(_ptr(H), k, ctypes.byref(cfg), _ptr(U), _ptr(perm), _ptr(invperm),
                                  _ptr(dead), _ptr(d_info), _ptr(ws), ws.numel() * ws.element_size(),
                                  _stream(stream))
    _check(st, "gptq_prepare_hinv")


def set_wait_limit(polls: int):
    """Test hook (gptq_set_wait_limit): polls before a pipeline wait of the
    tensor-core kernels gives up; WAIT_LIMIT_DEFAULT restores the default."""
    load().gptq_set_wait_limit(int(polls) & 0xFFFFFFFF)


def measure_peaks() -> dict:
    """Measured fp32-FMA and kind::tf32 peak rates (TFLOP/s) of the current
    device (gptq_measure_peaks)."""
    a, b = ctypes.c_double(0.0), ctypes.c_double(0.0)
    _check(load().gptq_measure_peaks(ctypes.byref(a), ctypes.byref(b)), "gptq_measure_peaks")
    return {"fp32_tflops": a.value, "tf32_tflops": b.value}


def prepare_hinv_noalloc(H, cfg, U, perm, invperm, dead, d_info, stream=None):
    """gptq_prepare_hinv without a workspace (scratch in the library's own
    device array; see include/gptq.h)."""
    k = H.shape[0]
    st = load().gptq_prepare_hinv_noalloc(_ptr(H), k, ctypes.byref(cfg), _ptr(U), _ptr(perm),
                                          _ptr(invperm), _ptr(dead), _ptr(d_info), _stream(stream))
    _check(st, "gptq_prepare_hinv_noalloc")


def quantize_layer(W, U, perm, dead, H0, cfg, codes, scales, zeros, g_idx, loss, d_status, ws,
                   stream=None):
    r, k = W.shape
    if W.stride(1) != 1:
        raise GptqError(GPTQ_ERR_INVALID_ARG, "gptq_quantize_layer", "W rows must be contiguous")
    st = load().gptq_quantize_layer(_ptr(W), dtype_code(W.dtype), r, k, W.stride(0), _ptr(U),
                                    _ptr(perm), _ptr(dead), _ptr(H0), ctypes.byref(cfg),
                                    _ptr(codes), _ptr(scales), _ptr(zeros), _ptr(g_idx),
                                    _ptr(loss), _ptr(d_status), _ptr(ws),
                                    ws.numel() * ws.element_size(), _stream(stream))
    _check(st, "gptq_quantize_layer")


def pack(codes, bits, qweight, stream=None):
    r, k = codes.shape
    st = load().gptq_pack(_ptr(codes), r, k, int(bits), _ptr(qweight), _stream(stream))
    _check(st, "gptq_pack")


def dequant(qweight, scales, zeros, g_idx, k, bits, out, stream=None):
    r = qweight.shape[0]
    st = load().gptq_dequant(_ptr(qweight), _ptr(scales), _ptr(zeros), _ptr(g_idx), r, k, int(bits),
                             scales.shape[1], dtype_code(out.dtype), _ptr(out), _stream(stream))
    _check(st, "gptq_dequant")


def gemm(X, qweight, scales, zeros, g_idx, bits, group_size, Y, stream=None):
    """Y = X W_hat^T from the packed weights (gptq_gemm).  X (m, k) and Y (m, n)
    f16/bf16 with unit column stride; g_idx None means groups of group_size."""
    m, k = X.shape
    n = qweight.shape[0]
    if X.stride(1) != 1 or Y.stride(1) != 1 or Y.dtype != X.dtype:
        raise GptqError(GPTQ_ERR_INVALID_ARG, "gptq_gemm", "X, Y: unit column stride, same dtype")
    st = load().gptq_gemm(_ptr(X), dtype_code(X.dtype), m, k, X.stride(0), _ptr(qweight),
                          _ptr(scales), _ptr(zeros), _ptr(g_idx), n, int(bits), int(group_size),
                          scales.shape[1], _ptr(Y), Y.stride(0), _stream(stream))
    _check(st, "gptq_gemm")


def rotate(x, signs, block, out, inverse=False, stream=None):
    """Each row of x (rows, k) times Q (or Q^T when inverse), into out (gptq_rotate)."""
    rows, k = x.shape
    if x.stride(1) != 1 or out.stride(1) != 1 or out.dtype != x.dtype or signs.dtype != torch.int8:
        raise GptqError(GPTQ_ERR_INVALID_ARG, "gptq_rotate", "unit column stride, same dtype, int8 signs")
    st = load().gptq_rotate(_ptr(x), dtype_code(x.dtype), rows, k, x.stride(0), _ptr(signs),
                            int(block), int(bool(inverse)), _ptr(out), out.stride(0),
                            _stream(stream))
    _check(st, "gptq_rotate")
