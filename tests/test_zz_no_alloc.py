"""The allocation-free entry point gptq_prepare_hinv_noalloc, for callers
that cannot allocate device memory (a plugin handed only its input and output
buffers, a process whose device memory is all in its own arena).

Called through the C ABI, twice in a row with different layers, its output
must match the workspace-taking gptq_prepare_hinv on the same input within
the tolerance the GPU parity tests use for fp32 matrices (1e-5 relative); the
integer outputs (order, dead mask, status) must be equal.  It must also refuse
a k beyond its built-in scratch before doing anything.  This file is collected
last so that a failure here leaves every other test already run.
"""

import ctypes

import numpy as np
import pytest
import torch

import synth

pytestmark = pytest.mark.gpu

TOL_REL = 1e-5


def _hessian(spec, seed, dead_cols=()):
    X = synth.make_x(spec, seed).double()
    if dead_cols:
        X[:, list(dead_cols)] = 0
    H = (2.0 / X.shape[0]) * (X.T @ X)
    return H.float().cuda()


def _both(H, cfg):
    from post_weight_quantization_23_b200 import _lib
    k = H.shape[0]
    dev = H.device
    outs = []
    for noalloc in (False, True):
        U = torch.full((k, k), float("nan"), device=dev)
        perm = torch.full((k,), -1, dtype=torch.int32, device=dev)
        invperm = torch.full((k,), -1, dtype=torch.int32, device=dev)
        dead = torch.full((k,), 7, dtype=torch.uint8, device=dev)
        d_info = torch.full((1,), -5, dtype=torch.int32, device=dev)
        if noalloc:
            _lib.prepare_hinv_noalloc(H, cfg, U, perm, invperm, dead, d_info)
        else:
            nbytes = _lib.workspace_size(_lib.OP_PREPARE_HINV, 0, k, 0, cfg)
            ws = torch.empty(nbytes, dtype=torch.uint8, device=dev)
            _lib.prepare_hinv(H, cfg, U, perm, invperm, dead, d_info, ws)
        torch.cuda.synchronize()
        outs.append((U.cpu(), perm.cpu(), invperm.cpu(), dead.cpu(), d_info.cpu()))
    return outs


def _assert_match(ref, got):
    U0, p0, ip0, d0, i0 = ref
    U1, p1, ip1, d1, i1 = got
    assert int(i0.item()) == 0 and int(i1.item()) == 0
    assert torch.equal(p0, p1) and torch.equal(ip0, ip1) and torch.equal(d0, d1)
    assert torch.isfinite(U1).all()
    rel = (U1.double() - U0.double()).abs().max() / U0.double().abs().max()
    assert float(rel) <= TOL_REL
    assert torch.equal(torch.tril(U1, -1), torch.zeros_like(U1))


def test_noalloc_matches_workspace_entry_two_calls_in_a_row():
    from post_weight_quantization_23_b200 import _lib
    # first call: a q_proj-like layer, natural order
    spec1 = synth.CONFIGS["q_proj"].scaled(r=64, k=1024, n=8192)
    H1 = _hessian(spec1, 11)
    cfg1 = _lib.make_config(4, 128, 128, 0.01, False)
    ref1, got1 = _both(H1, cfg1)
    _assert_match(ref1, got1)
    # second call right after, different size, act-order and dead columns:
    # the shared scratch still holds the first call's contents
    spec2 = synth.CONFIGS["down_proj"].scaled(r=64, k=768, n=8192)
    H2 = _hessian(spec2, 12, dead_cols=(5, 400))
    cfg2 = _lib.make_config(4, 128, 128, 0.01, True)
    ref2, got2 = _both(H2, cfg2)
    _assert_match(ref2, got2)
    assert list(np.flatnonzero(got2[3].numpy())) == [5, 400]


def _gpu_hessian(spec, seed):
    """H of a seeded layer from the library's own Hessian call (both entry
    points under test then factor the same bytes)."""
    from post_weight_quantization_23_b200 import _lib
    X = synth.make_x(spec, seed).cuda()
    H = torch.zeros(spec.k, spec.k, device="cuda")
    ws = torch.zeros(_lib.workspace_size(_lib.OP_HESSIAN, 0, spec.k, spec.n, None),
                     dtype=torch.uint8, device="cuda")
    _lib.hessian_accumulate(X, H, 2.0 / spec.n, ws)
    torch.cuda.synchronize()
    return H


@pytest.mark.parametrize("name,k", [("q_proj", 4096), ("opt175_width", 12288)])
def test_noalloc_cuda_core_update_at_full_width(name, k):
    """From k = 4080 the operand splits of the tensor-core rank update no
    longer fit in the built-in scratch, so the call takes the fp32 CUDA-core
    rank update (a triangular tile schedule over several row tiles): at the
    q_proj width and at the OPT-175B width, twice in a row, against the
    workspace entry point's tensor-core result."""
    from post_weight_quantization_23_b200 import _lib
    spec = synth.CONFIGS[name].scaled(r=64, k=k, n=16384)
    H = _gpu_hessian(spec, 21)
    for act_order in (False, True):
        cfg = _lib.make_config(spec.bits, spec.group_size, spec.block_size, 0.01, act_order)
        ref, got = _both(H, cfg)
        rel = float((got[0].double() - ref[0].double()).abs().max() / ref[0].double().abs().max())
        print(f"k={k} act_order={act_order}: max |dU| / max |U| = {rel:.3e}")
        _assert_match(ref, got)
    print(f"k={k}: device ms workspace / no-alloc = {_time_both(H, cfg)}")


def _time_both(H, cfg):
    """Device time of one call of each entry point (for the record)."""
    from post_weight_quantization_23_b200 import _lib
    k = H.shape[0]
    U = torch.empty(k, k, device="cuda")
    i32 = dict(dtype=torch.int32, device="cuda")
    perm, invperm, d_info = torch.empty(k, **i32), torch.empty(k, **i32), torch.empty(1, **i32)
    dead = torch.empty(k, dtype=torch.uint8, device="cuda")
    ws = torch.empty(_lib.workspace_size(_lib.OP_PREPARE_HINV, 0, k, 0, cfg), dtype=torch.uint8,
                     device="cuda")
    out = []
    for noalloc in (False, True):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        if noalloc:
            _lib.prepare_hinv_noalloc(H, cfg, U, perm, invperm, dead, d_info)
        else:
            _lib.prepare_hinv(H, cfg, U, perm, invperm, dead, d_info, ws)
        e1.record()
        torch.cuda.synchronize()
        out.append(round(e0.elapsed_time(e1), 2))
    return out


def test_noalloc_rejects_k_beyond_its_scratch():
    from post_weight_quantization_23_b200 import _lib
    lib = _lib.load()
    cfg = _lib.make_config(4, 128, 128, 0.01, False)
    fake = ctypes.c_void_p(256)  # never dereferenced: the size check comes first
    st = lib.gptq_prepare_hinv_noalloc(fake, 12289, ctypes.byref(cfg), ctypes.c_void_p(512),
                                       fake, fake, fake, fake, None)
    assert st == _lib.GPTQ_ERR_WORKSPACE
