"""Bounded device waits that run out ("GPTQ", ozercemkelahmet.com/tools/gptq,
When the method breaks down: a failure must surface as an error, never as a
hang).

gptq_set_wait_limit(0) makes every pipeline wait of the tensor-core kernels
give up at its first poll -- deterministically, before any data could have
arrived -- while the drain waits that let a CTA's own copies and MMAs land keep
their full bound.  Each stage must then report GPTQ_ERR_TIMEOUT through its
device status word (the Hessian workspace's status word, d_info = k + 1 of the
factor, d_status of the sweep), nothing may trap or hang, and with the default
limit restored the same plan must produce oracle-matching results again (the
context stays usable).
"""

import math

import numpy as np
import pytest
import torch

import oracle as O
import synth

pytestmark = pytest.mark.gpu

SPEC = synth.CONFIGS["q_proj"].scaled(r=256, k=512, n=8192)


def _setup():
    from post_weight_quantization_23_b200 import GptqPlan, QuantConfig
    W = synth.make_w(SPEC, 3)
    X = synth.make_x(SPEC, 3)
    cfg = QuantConfig(4, 128, 128, 0.01, False)
    plan = GptqPlan(SPEC.r, SPEC.k, cfg, "cuda", deq_dtype=torch.float32,
                    hessian_tokens_hint=SPEC.n)
    return plan, W, X, W.cuda(), X.cuda()


class _Limit:
    def __init__(self, polls):
        self.polls = polls

    def __enter__(self):
        from post_weight_quantization_23_b200 import _lib
        _lib.set_wait_limit(self.polls)

    def __exit__(self, *exc):
        from post_weight_quantization_23_b200 import _lib
        _lib.set_wait_limit(_lib.WAIT_LIMIT_DEFAULT)


def _healthy_run(plan, W, X, Wd, Xd):
    """The whole layer with the default limit, against the oracle."""
    plan.hessian_reset()
    plan.hessian_add(Xd, SPEC.n)
    plan.run_after_hessian(Wd)
    plan.check()
    H = O.hessian(X.numpy())
    Hg = plan.H.double().cpu().numpy()
    assert np.linalg.norm(Hg - H) / np.linalg.norm(H) <= 1e-5
    ref = O.gptq(W.numpy(), H, 4, 128, 128, 0.01, False)
    codes = plan.codes.cpu().numpy().astype(np.int64)
    assert (codes == ref["codes"]).mean() >= 0.999


def test_hessian_wait_gives_up_with_timeout_status():
    from post_weight_quantization_23_b200 import GptqError, _lib
    plan, W, X, Wd, Xd = _setup()
    plan.hessian_reset()
    with _Limit(0):
        plan.hessian_add(Xd, SPEC.n)
        st = plan.status()
    assert st["hessian"] == _lib.GPTQ_ERR_TIMEOUT
    assert math.isnan(float(plan.H[0, 0]))  # the poison a status-blind caller meets
    with pytest.raises(GptqError) as e:
        plan.check()
    assert e.value.status == _lib.GPTQ_ERR_TIMEOUT
    _healthy_run(plan, W, X, Wd, Xd)
    assert plan.status()["hessian"] == 0


def test_factor_update_wait_gives_up_with_timeout_status():
    from post_weight_quantization_23_b200 import GptqError, _lib
    plan, W, X, Wd, Xd = _setup()
    plan.hessian_reset()
    plan.hessian_add(Xd, SPEC.n)
    with _Limit(0):
        plan.prepare()
        st = plan.status()
    assert st["hessian"] == 0
    assert st["d_info"] == SPEC.k + 1  # a timeout, not a pivot
    with pytest.raises(GptqError) as e:
        plan.check()
    assert e.value.status == _lib.GPTQ_ERR_TIMEOUT
    _healthy_run(plan, W, X, Wd, Xd)


def test_sweep_waits_give_up_with_timeout_status():
    from post_weight_quantization_23_b200 import GptqError, _lib
    plan, W, X, Wd, Xd = _setup()
    plan.hessian_reset()
    plan.hessian_add(Xd, SPEC.n)
    plan.prepare()
    with _Limit(0):
        plan.quantize(Wd)
        st = plan.status()
    assert st["d_info"] == 0
    assert st["d_status"] == _lib.GPTQ_ERR_TIMEOUT
    with pytest.raises(GptqError) as e:
        plan.check()
    assert e.value.status == _lib.GPTQ_ERR_TIMEOUT
    _healthy_run(plan, W, X, Wd, Xd)


def test_inference_product_wait_gives_up_with_nan_outputs():
    """gptq_gemm has no status word: a tensor-core CTA that gives up writes NaN
    over its outputs (never a silently wrong number)."""
    from post_weight_quantization_23_b200 import quant_matmul
    g = torch.Generator().manual_seed(5)
    n, k, G, m = 256, 512, 128, 64
    codes = torch.randint(0, 16, (n, k), generator=g)
    qw = torch.from_numpy(O.pack(codes.numpy(), 4)).cuda()
    sc = (torch.rand(n, k // G, generator=g) * 0.02 + 1e-3).cuda()
    z = torch.randint(0, 16, (n, k // G), generator=g, dtype=torch.int32).cuda()
    X = torch.randn(m, k, generator=g).half().cuda()
    with _Limit(0):
        Y = quant_matmul(X, qw, sc, z, 4, G)
        torch.cuda.synchronize()
    assert torch.isnan(Y).all()
    Y = quant_matmul(X, qw, sc, z, 4, G)
    ref = O.dequant_matmul(X.double().cpu().numpy(), qw.cpu().numpy(), sc.cpu().numpy(),
                           z.cpu().numpy().astype(np.int64), np.arange(k) // G, 4, k)
    assert np.abs(Y.double().cpu().numpy() - ref).max() <= 4e-3 * np.abs(ref).max()
