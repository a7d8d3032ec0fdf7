"""Full-size parity of the Llama-7B-shaped q_proj layer (W 4096 x 4096 fp16,
X 262144 x 4096 fp16, int4 g128 B128) in the launch configuration bench.py
times (all tokens in one Hessian call).  The oracle computes the whole fp64
Hessian (in token chunks) and its own inverse factor, then sweeps a seeded
sample of rows (rows are independent given U); codes, scales, zeros, loss
and packing of those rows are compared."""

import numpy as np
import pytest
import torch

import oracle as O
import synth
from _parity import TOL_LOSS_REL, compare

pytestmark = [pytest.mark.gpu, pytest.mark.slow]


def test_q_proj_fullsize_sampled_rows():
    from post_weight_quantization_23_b200 import GptqPlan, QuantConfig
    spec = synth.CONFIGS["q_proj"]
    W = synth.make_w(spec, 0)
    X = torch.empty(spec.n, spec.k, dtype=torch.float16, pin_memory=True)
    synth.make_x(spec, 0, out=X)
    cfg = QuantConfig(spec.bits, spec.group_size, spec.block_size, spec.percdamp, spec.act_order)
    plan = GptqPlan(spec.r, spec.k, cfg, "cuda", deq_dtype=torch.float16,
                    hessian_tokens_hint=spec.n)
    plan.hessian_add(X.cuda(), spec.n)
    plan.run_after_hessian(W.cuda())
    plan.check()
    gpu = {key: v.detach().cpu() for key, v in plan.result().items() if torch.is_tensor(v)}
    # oracle Hessian in fp64, chunked over tokens
    H = None
    for a in range(0, spec.n, 16384):
        Xc = X[a:a + 16384].double().numpy()
        G = Xc.T @ Xc
        H = G if H is None else H + G
    H *= 2.0 / spec.n
    rows = np.sort(np.random.default_rng(0).choice(spec.r, 48, replace=False))
    a = compare(gpu, W.numpy(), None, cfg, rows=rows, H=H)
    print("q_proj full size", a)
    a.assert_ok()
    # pack / dequant of the sampled rows, bit exact
    codes = gpu["codes"].numpy().astype(np.int64)[rows]
    assert np.array_equal(gpu["qweight"].numpy()[rows], O.pack(codes, 4))
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
