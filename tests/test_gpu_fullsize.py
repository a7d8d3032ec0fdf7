"""Full-size parity of the pages' layer shapes, in the launch configuration
bench.py times (all calibration tokens resident on the device, one Hessian
call):

* q_proj        W 4096 x 4096,   X 262144 x 4096,  int4 g128;
* down_proj     W 4096 x 11008,  X 262144 x 11008 (silu-gated), int4 g128, act-order;
* opt175_width  W 12288 x 12288, X 131072 x 12288 (x50 outliers), 3-bit per row;
* stack_gate_up the 7B stack's gate and up projections stacked on one shared
                Hessian: W 22016 x 4096, X 65536 x 4096, int4 g128, act-order.

The oracle computes the whole fp64 Hessian from the same tokens (in chunks),
its own inverse factor at full k, and sweeps a seeded sample of rows (rows are
independent given U); codes, scales, zeros, g_idx, loss and packing of those
rows are compared, and the GPU's fp32 factor U is checked against the
oracle's at a bound derived from the fp32 arithmetic (``u_bound``).  The whole-
layer loss is checked against the oracle's evaluation of the GPU's own codes.
"""

import math

import numpy as np
import pytest
import torch
from scipy.linalg import lapack

import oracle as O
import synth
from _parity import TOL_LOSS_REL, compare

pytestmark = [pytest.mark.gpu, pytest.mark.slow]

FULL = {
    "q_proj": synth.CONFIGS["q_proj"],
    "down_proj": synth.CONFIGS["down_proj"],
    "opt175_width": synth.CONFIGS["opt175_width"],
    "stack_gate_up": synth.stack_spec("gate_up"),
}

U32 = 2.0 ** -24


def scaled_condition(Hd):
    """1-norm condition estimate (LAPACK dpocon) of the damped Hessian scaled
    to unit diagonal, S = D^-1/2 Hd D^-1/2: a Cholesky factor's relative
    accuracy is governed by the scaled matrix, not by Hd itself."""
    d = 1.0 / np.sqrt(np.diag(Hd))
    S = Hd * d[:, None] * d[None, :]
    c, info = lapack.dpotrf(S, lower=0)
    assert info == 0
    rc, info = lapack.dpocon(c, float(np.abs(S).sum(axis=0).max()))
    assert info == 0 and rc > 0
    return 1.0 / rc


def u_bound(kappa, k, h_rel):
    """Bound on max|U_gpu - U| / max|U| for the fp32 factor: first-order
    perturbation of a Cholesky factor multiplies a relative perturbation of
    the scaled matrix by at most its condition number kappa; the
    perturbation is the GPU Hessian's own error h_rel (twice: H enters the
    damping and the factor) plus the fp32 rounding of a k-long factorisation,
    whose errors grow like sqrt(k) u in practice (u = 2^-24), with a factor 8
    of margin."""
    return kappa * (2.0 * h_rel + 8.0 * math.sqrt(k) * U32)


def _oracle_hessian(X, n, chunk=16384):
    return O.hessian((X[a:a + chunk].numpy() for a in range(0, n, chunk)), n_total=n)


@pytest.mark.parametrize("name", list(FULL))
def test_fullsize_sampled_rows(name):
    from post_weight_quantization_23_b200 import GptqPlan, QuantConfig
    spec = FULL[name]
    W = synth.make_w(spec, 0)
    X = torch.empty(spec.n, spec.k, dtype=synth.dtype_of(spec.x_dtype), pin_memory=True)
    synth.make_x(spec, 0, out=X)
    cfg = QuantConfig(spec.bits, spec.group_size, spec.block_size, spec.percdamp, spec.act_order)
    plan = GptqPlan(spec.r, spec.k, cfg, "cuda", deq_dtype=torch.float16,
                    hessian_tokens_hint=spec.n)
    plan.hessian_add(X.cuda(), spec.n)
    plan.run_after_hessian(W.cuda())
    plan.check()
    gpu = {key: v.detach().cpu() for key, v in plan.result().items() if torch.is_tensor(v)}
    del plan
    torch.cuda.empty_cache()
    H = _oracle_hessian(X, spec.n)
    rows = np.sort(np.random.default_rng(0).choice(spec.r, 48, replace=False))
    a = compare(gpu, W.numpy(), None, cfg, rows=rows, H=H)
    # the factor: the oracle's damped Hessian in the GPU's processing order
    perm = gpu["perm"].numpy().astype(np.int64)
    Hf = O.fix_dead_columns(H, W.numpy()[:1])[0]
    kappa = scaled_condition(O.damp(Hf[np.ix_(perm, perm)], spec.percdamp))
    bound = u_bound(kappa, spec.k, a.h_rel_fro)
    print(f"{name} full size {a}; scaled condition {kappa:.3g}, U bound {bound:.3g}")
    a.assert_ok()
    assert a.u_rel_max <= bound, (a.u_rel_max, bound)
    # pack / dequant of the sampled rows, bit exact
    codes = gpu["codes"].numpy().astype(np.int64)[rows]
    assert np.array_equal(gpu["qweight"].numpy()[rows], O.pack(codes, spec.bits))
    deq = O.dequant(codes, gpu["scales"].numpy()[rows], gpu["zeros"].numpy()[rows],
                    gpu["g_idx"].numpy(), np.float16)
    assert np.array_equal(gpu["deq"].numpy()[rows], deq)
    # whole-layer loss against the oracle's loss of the GPU's own codes
    # (a property at any size: the loss kernel evaluates tr(D H0 D^T))
    qhat = O.dequant(gpu["codes"].numpy(), gpu["scales"].numpy(), gpu["zeros"].numpy(),
                     gpu["g_idx"].numpy(), np.float32).astype(np.float64)
    D = W.double().numpy() - qhat
    loss_ref = float(np.einsum("ij,ij->", D @ H, D))
    assert abs(float(gpu["loss"]) - loss_ref) <= TOL_LOSS_REL * loss_ref
