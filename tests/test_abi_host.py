"""CPU checks of the C ABI library: it loads, exports every function that
include/gptq.h declares, and rejects bad arguments on the host before any
device work (no compute call is made here)."""

import ctypes
import os
import re

import pytest

import post_weight_quantization_23_b200 as P
from post_weight_quantization_23_b200 import _lib

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    src = open(os.path.join(ROOT, "include", "gptq.h")).read()
    return sorted(set(re.findall(r"GPTQ_API\s+[\w\s\*]+?\b(gptq_\w+)\s*\(", src)))


@pytest.fixture(scope="module")
def lib():
    if not os.path.exists(_lib.LIB_PATH):
        from post_weight_quantization_23_b200 import build
        build.build()
    return _lib.load()


def test_header_declares_the_abi():
    assert _declared() == sorted(_lib.EXPORTED)


def test_library_exports_every_declared_symbol(lib):
    for name in _declared():
        assert hasattr(lib, name), name


def test_status_strings(lib):
    for code, name in [(0, "GPTQ_OK"), (2, "GPTQ_ERR_NOT_PD"), (7, "GPTQ_ERR_NONFINITE")]:
        assert lib.gptq_status_string(code).decode() == name


def test_workspace_sizes(lib):
    cfg = _lib.make_config(4, 128, 128, 0.01, False)
    q = _lib.workspace_size(_lib.OP_QUANTIZE, 4096, 4096, 0, cfg)
    # the fp32 working copy and the error block dominate
    assert q >= 4 * 4096 * 4096 + 4 * 4096 * 128
    p = _lib.workspace_size(_lib.OP_PREPARE_HINV, 0, 4096, 0, cfg)
    assert p >= 4 * 4096
    assert _lib.workspace_size(_lib.OP_QUANTIZE, -1, 4096, 0, cfg) == 0


def test_host_argument_checks(lib):
    cfgp = ctypes.byref(_lib.make_config(4, 128, 128, 0.01, False))
    bad_bits = ctypes.byref(_lib.make_config(5, 128, 128, 0.01, False))
    bad_group = ctypes.byref(_lib.make_config(4, 96, 128, 0.01, False))
    bad_block = ctypes.byref(_lib.make_config(4, 128, 512, 0.01, False))
    neg_damp = ctypes.byref(_lib.make_config(4, 128, 128, -0.1, False))
    fake = ctypes.c_void_p(256)  # never dereferenced: every call below fails a host check
    # pack / dequant
    assert lib.gptq_pack(fake, 4, 32, 5, fake, None) == _lib.GPTQ_ERR_UNSUPPORTED
    assert lib.gptq_pack(fake, 4, 40, 4, fake, None) == _lib.GPTQ_ERR_INVALID_ARG
    assert lib.gptq_pack(None, 4, 32, 4, fake, None) == _lib.GPTQ_ERR_INVALID_ARG
    assert lib.gptq_pack(fake, 0, 32, 4, fake, None) == _lib.GPTQ_OK  # empty: no-op
    assert lib.gptq_dequant(fake, fake, fake, fake, 4, 32, 4, 0, 0, fake, None) == _lib.GPTQ_ERR_INVALID_ARG
    assert lib.gptq_dequant(fake, fake, fake, fake, 4, 32, 4, 1, 9, fake, None) == _lib.GPTQ_ERR_INVALID_ARG
    # hessian
    assert lib.gptq_hessian_accumulate(fake, 0, 0, 64, 64, 1.0, fake, None, 0, None) == _lib.GPTQ_OK
    assert lib.gptq_hessian_accumulate(fake, 0, 10, 64, 32, 1.0, fake, None, 0, None) == _lib.GPTQ_ERR_INVALID_ARG
    assert lib.gptq_hessian_accumulate(None, 0, 10, 64, 64, 1.0, fake, None, 0, None) == _lib.GPTQ_ERR_INVALID_ARG
    assert lib.gptq_hessian_accumulate(fake, 7, 10, 64, 64, 1.0, fake, None, 0, None) == _lib.GPTQ_ERR_INVALID_ARG
    # prepare_hinv
    args = [fake, 64, cfgp, ctypes.c_void_p(512), fake, fake, fake, fake]
    assert lib.gptq_prepare_hinv(*args, None, 0, None) == _lib.GPTQ_ERR_WORKSPACE
    assert lib.gptq_prepare_hinv(fake, 0, cfgp, fake, fake, fake, fake, fake, fake, 1 << 20, None) == _lib.GPTQ_ERR_INVALID_ARG
    assert lib.gptq_prepare_hinv(fake, 64, neg_damp, ctypes.c_void_p(512), fake, fake, fake, fake, fake, 1 << 20, None) == _lib.GPTQ_ERR_INVALID_ARG
    assert lib.gptq_prepare_hinv(fake, 64, cfgp, fake, fake, fake, fake, fake, fake, 1 << 20, None) == _lib.GPTQ_ERR_INVALID_ARG  # H aliases U
    # quantize_layer
    q = lambda c, ws=fake, nbytes=1 << 30, ldw=64: lib.gptq_quantize_layer(  # noqa: E731
        fake, 1, 16, 64, ldw, fake, fake, fake, None, c, fake, fake, fake, fake, None, None, ws, nbytes, None)
    assert q(bad_bits) == _lib.GPTQ_ERR_UNSUPPORTED
    assert q(bad_group) == _lib.GPTQ_ERR_INVALID_ARG
    assert q(bad_block) == _lib.GPTQ_ERR_UNSUPPORTED
    assert q(cfgp, ldw=32) == _lib.GPTQ_ERR_INVALID_ARG
    assert q(cfgp, ws=None) == _lib.GPTQ_ERR_WORKSPACE
    assert q(cfgp, nbytes=16) == _lib.GPTQ_ERR_WORKSPACE
    assert q(cfgp, ws=ctypes.c_void_p(257)) == _lib.GPTQ_ERR_WORKSPACE
    bad_sym = _lib.make_config(4, 128, 128, 0.01, False)
    bad_sym.sym = 2
    assert q(ctypes.byref(bad_sym)) == _lib.GPTQ_ERR_INVALID_ARG
    bad_static = _lib.make_config(4, 128, 128, 0.01, False)
    bad_static.static_groups = 2
    assert q(ctypes.byref(bad_static)) == _lib.GPTQ_ERR_INVALID_ARG
    # groups that straddle lazy blocks are fine once the grids are static: the
    # call then gets past the config check to the workspace check
    static_g96 = ctypes.byref(_lib.make_config(4, 96, 128, 0.01, False, static_groups=True))
    assert q(static_g96, ws=None) == _lib.GPTQ_ERR_WORKSPACE


def test_gemm_host_checks(lib):
    fake = ctypes.c_void_p(256)  # never dereferenced: every call below fails a host check
    F16, F32, BF16 = _lib.GPTQ_F16, _lib.GPTQ_F32, _lib.GPTQ_BF16

    def g(dt=F16, m=2, k=256, ldx=256, bits=4, gs=128, ng=2, gidx=None, n=8, ldy=8, X=fake):
        return lib.gptq_gemm(X, dt, m, k, ldx, fake, fake, fake, gidx, n, bits, gs, ng, fake,
                             ldy, None)

    assert g(bits=5) == _lib.GPTQ_ERR_UNSUPPORTED
    assert g(dt=F32) == _lib.GPTQ_ERR_UNSUPPORTED
    assert g(dt=9) == _lib.GPTQ_ERR_INVALID_ARG
    assert g(k=250, ldx=250) == _lib.GPTQ_ERR_INVALID_ARG          # k % 32
    assert g(m=0) == _lib.GPTQ_OK and g(n=0) == _lib.GPTQ_OK       # empty: no-op
    assert g(ldx=128) == _lib.GPTQ_ERR_INVALID_ARG                 # ldx < k
    assert g(ldy=4) == _lib.GPTQ_ERR_INVALID_ARG                   # ldy < n
    assert g(ng=3) == _lib.GPTQ_ERR_INVALID_ARG                    # ngroups != ceil(k / G)
    assert g(gs=0) == _lib.GPTQ_ERR_INVALID_ARG
    assert g(gs=-1, ng=2) == _lib.GPTQ_ERR_INVALID_ARG             # one group per row
    assert g(X=None) == _lib.GPTQ_ERR_INVALID_ARG
    assert g(m=131071) == _lib.GPTQ_ERR_INVALID_ARG                # token limit
    assert g(X=ctypes.c_void_p(257)) == _lib.GPTQ_ERR_INVALID_ARG  # misaligned X


def test_rotate_host_checks(lib):
    fake = ctypes.c_void_p(256)  # never dereferenced: every call below fails a host check
    F16 = _lib.GPTQ_F16

    def r(rows=4, k=512, ld_in=512, block=256, ld_out=512, inp=fake, out=ctypes.c_void_p(1 << 30),
          signs=fake, dt=F16):
        return lib.gptq_rotate(inp, dt, rows, k, ld_in, signs, block, 0, out, ld_out, None)

    assert r(block=128) == _lib.GPTQ_ERR_UNSUPPORTED
    assert r(block=384) == _lib.GPTQ_ERR_UNSUPPORTED
    assert r(block=16384) == _lib.GPTQ_ERR_UNSUPPORTED
    assert r(k=640, ld_in=640, ld_out=640) == _lib.GPTQ_ERR_INVALID_ARG   # k % block
    assert r(rows=0) == _lib.GPTQ_OK
    assert r(ld_in=256) == _lib.GPTQ_ERR_INVALID_ARG
    assert r(ld_in=516) == _lib.GPTQ_ERR_INVALID_ARG                      # row not 16-byte aligned
    assert r(signs=None) == _lib.GPTQ_ERR_INVALID_ARG
    assert r(signs=ctypes.c_void_p(260)) == _lib.GPTQ_ERR_INVALID_ARG     # signs not 8-byte aligned
    assert r(out=ctypes.c_void_p(256 + 512)) == _lib.GPTQ_ERR_INVALID_ARG  # overlapping buffers
    assert r(dt=9) == _lib.GPTQ_ERR_INVALID_ARG


def test_hadamard_block_choice():
    from post_weight_quantization_23_b200 import hadamard_block
    assert hadamard_block(4096) == 4096 and hadamard_block(11008) == 256
    assert hadamard_block(12288) == 4096 and hadamard_block(16384) == 8192
    assert hadamard_block(4160) == 0 and hadamard_block(0) == 0


def test_binding_refuses_cpu_tensors():
    import torch
    with pytest.raises(P.GptqError):
        _lib.pack(torch.zeros(4, 32, dtype=torch.uint8), 4, torch.zeros(4, 4, dtype=torch.int32))
