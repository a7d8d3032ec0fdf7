"""GPU parity of the inference product Y = X W_hat^T read from packed codes
(gptq_gemm), against the oracle's fp64 product on the same seeded inputs.

Inputs: seeded random codes, scales and zero points, packed by the oracle's
pack(); activations from the layer generators.  Tolerance, from the
arithmetic: every product x * (code - zero) is exact or once rounded in
fp32, the sums are fp32 (at most k + 2 roundings on any path, |error| <=
(k + 2) 2^-24 sum_c |x_c w_c|), and Y is rounded once to its dtype
(2^-11 relative for f16, 2^-8 for bf16, and half the f16 subnormal spacing).
"""

import numpy as np
import pytest
import torch

import oracle as O
import synth

pytestmark = pytest.mark.gpu

U_OUT = {torch.float16: 2.0 ** -11, torch.bfloat16: 2.0 ** -8}


def _inputs(n, k, bits, G, m, dtype, seed, act_perm=False):
    g = torch.Generator().manual_seed(seed)
    ng = (k + G - 1) // G
    codes = torch.randint(0, 2 ** bits, (n, k), generator=g, dtype=torch.int64)
    scales = (torch.rand(n, ng, generator=g) * 0.02 + 1e-3).float()
    zeros = torch.randint(0, 2 ** bits, (n, ng), generator=g, dtype=torch.int32)
    if act_perm:
        g_idx = (torch.arange(k) // G)[torch.randperm(k, generator=g)].to(torch.int32)
    else:
        g_idx = (torch.arange(k) // G).to(torch.int32)
    spec = synth.CONFIGS["q_proj"].scaled(r=n, k=k, n=max(m, 1))
    X = synth.make_x(spec, seed)[:m].to(dtype)
    qw = torch.from_numpy(O.pack(codes.numpy(), bits))
    return codes, scales, zeros, g_idx, X, qw


def _tc_path(bits, G, k, m, pass_gidx):
    """Whether gptq_gemm forms each weight in the activations' 16-bit type
    (contiguous inputs): the tensor-core kernel from 17 tokens, the
    small-batch mma.sync kernel for 3 to 16 tokens."""
    if bits != 4 or pass_gidx:
        return False
    if m >= 17:
        return k >= 64 and (G >= k or G % 32 == 0)
    return m >= 3 and k % 32 == 0 and (G >= k or G % 128 == 0)


def _check(Y, X, qw, scales, zeros, g_idx, bits, k, dtype, tc=False):
    Xn = X.float().numpy().astype(np.float64)
    ref = O.dequant_matmul(Xn, qw.numpy(), scales.numpy(), zeros.numpy().astype(np.int64),
                           g_idx.numpy(), bits, k)
    codes = O.unpack(qw.numpy(), k, bits)
    gi = g_idx.numpy().astype(np.int64)
    W_abs = np.abs(scales.numpy().astype(np.float64)[:, gi] *
                   (codes - zeros.numpy().astype(np.int64)[:, gi]))
    # |fl(Y32) - ref| <= u |ref| + (1 + u) |Y32 - ref|, plus half the f16
    # subnormal spacing for outputs that round into the subnormal range
    fp32_err = (k + 2) * 2.0 ** -24 * (np.abs(Xn) @ W_abs.T)
    if tc:
        # tensor cores: each weight is the scale rounded to the activations'
        # type times the exact (code - zero), rounded once more (relative error
        # at most 2u + u^2), exact products, fp32 sums (counted twice over in
        # case the adder truncates)
        u = U_OUT[dtype]
        fp32_err = (2 * u + u * u) * (np.abs(Xn) @ W_abs.T) + 2 * fp32_err
    bound = U_OUT[dtype] * np.abs(ref) + (1 + U_OUT[dtype]) * fp32_err + 2.0 ** -25
    got = Y.float().cpu().numpy().astype(np.float64)
    err = np.abs(got - ref)
    assert np.all(np.isfinite(got))
    assert np.all(err <= bound), (float((err / bound).max()), np.argwhere(err > bound)[:5])
    return float((err / bound).max())


CASES = [
    # (n, k, bits, G, m, dtype, g_idx passed, act-order g_idx)
    (256, 1024, 4, 128, 1, torch.float16, False, False),   # decode kernel, one token
    (256, 1024, 4, 128, 2, torch.float16, False, False),   # decode kernel, a token pair
    (100, 4352, 4, 128, 3, torch.bfloat16, False, False),  # small-batch kernel: ragged rows, 3 passes, odd m
    (64, 8192, 4, 32, 5, torch.float16, False, False),     # smallest 4-bit group, 2 passes
    (50, 4352, 4, 128, 8, torch.float16, False, False),    # 8 tokens per CTA, 2 passes over X
    (100, 2048, 2, 64, 12, torch.bfloat16, False, False),  # 2-bit, two 8-token groups
    (70, 1024, 8, 32, 20, torch.float16, False, False),    # 8-bit past 16 tokens: decode kernel
    (96, 1536, 2, 64, 1, torch.float16, False, False),     # 2-bit decode
    (96, 1536, 8, 16, 2, torch.bfloat16, False, False),    # 8-bit decode, 16-column groups
    (33, 2048, 4, 2048, 1, torch.float16, False, False),   # one group per row
    (64, 1024, 4, 16, 2, torch.float16, False, False),     # group below a 16-byte piece: general
    (64, 1024, 3, 128, 3, torch.float16, False, False),    # 3-bit codes straddle words: general
    (80, 1024, 4, 128, 9, torch.bfloat16, True, True),     # act-order g_idx: general kernel
    (48, 512, 4, 128, 17, torch.float16, True, False),     # trivial g_idx passed explicitly
    # small-batch mma.sync kernel (3 to 16 tokens, 4-bit, groups of 128k columns or per row)
    (272, 4096, 4, 128, 16, torch.float16, False, False),   # two passes over X
    (50, 2112, 4, 2112, 9, torch.bfloat16, False, False),   # one group per row, a short last pass
    (33, 1024, 4, 256, 5, torch.float16, False, False),     # groups of 256, ragged rows
    # tensor-core kernel (17 tokens and more)
    (256, 1024, 4, 128, 64, torch.float16, False, False),
    (300, 4128, 4, 128, 300, torch.bfloat16, False, False),  # ragged rows, tokens, last K stage
    (128, 2048, 4, 32, 17, torch.float16, False, False),      # two groups per K stage
    (96, 2048, 4, 2048, 513, torch.float16, False, False),    # one group per row
]


@pytest.mark.parametrize("case", CASES, ids=[f"n{c[0]}_k{c[1]}_b{c[2]}_g{c[3]}_m{c[4]}"
                                              f"{'_gidx' if c[6] else ''}{'_act' if c[7] else ''}"
                                              for c in CASES])
def test_qgemm_parity(case):
    from post_weight_quantization_23_b200 import quant_matmul
    n, k, bits, G, m, dtype, pass_gidx, act = case
    codes, scales, zeros, g_idx, X, qw = _inputs(n, k, bits, G, m, dtype, seed=n + k + m,
                                                 act_perm=act)
    dev = "cuda"
    Y = quant_matmul(X.to(dev), qw.to(dev), scales.to(dev), zeros.to(dev), bits, G,
                     g_idx.to(dev) if pass_gidx else None)
    torch.cuda.synchronize()
    r = _check(Y, X, qw, scales, zeros, g_idx, bits, k, dtype, _tc_path(bits, G, k, m, pass_gidx))
    print(case, "max err / bound", r)


@pytest.mark.parametrize("m", [1, 2, 16, 512])
def test_qgemm_full_size_q_proj(m):
    # the full q_proj layer (4096 x 4096, int4 g128), every output compared
    from post_weight_quantization_23_b200 import quant_matmul
    n = k = 4096
    codes, scales, zeros, g_idx, X, qw = _inputs(n, k, 4, 128, m, torch.float16, seed=m)
    Y = quant_matmul(X.cuda(), qw.cuda(), scales.cuda(), zeros.cuda(), 4, 128)
    torch.cuda.synchronize()
    _check(Y, X, qw, scales, zeros, g_idx, 4, k, torch.float16, _tc_path(4, 128, k, m, False))


def test_qgemm_small_batch_strided():
    # the small-batch kernel with X rows off 16-byte boundaries (scalar staging)
    # and a padded output
    from post_weight_quantization_23_b200 import quant_matmul
    n, k, m = 40, 768, 6
    codes, scales, zeros, g_idx, X, qw = _inputs(n, k, 4, 128, m, torch.bfloat16, seed=11)
    Xo = torch.zeros(m, k + 3, dtype=torch.bfloat16, device="cuda")
    Xo[:, :k] = X.cuda()
    Yp = torch.full((m, n + 8), 7.0, dtype=torch.bfloat16, device="cuda")
    quant_matmul(Xo[:, :k], qw.cuda(), scales.cuda(), zeros.cuda(), 4, 128, out=Yp[:, :n])
    torch.cuda.synchronize()
    _check(Yp[:, :n], X, qw, scales, zeros, g_idx, 4, k, torch.bfloat16, True)
    assert torch.all(Yp[:, n:] == 7.0)


def test_qgemm_strided_and_empty():
    from post_weight_quantization_23_b200 import quant_matmul
    n, k = 64, 512
    codes, scales, zeros, g_idx, X, qw = _inputs(n, k, 4, 128, 2, torch.float16, seed=3)
    # X and Y rows with padding (leading dimensions above k and n)
    Xp = torch.zeros(2, k + 64, dtype=torch.float16, device="cuda")
    Xp[:, :k] = X.cuda()
    Yp = torch.full((2, n + 8), 7.0, dtype=torch.float16, device="cuda")
    quant_matmul(Xp[:, :k], qw.cuda(), scales.cuda(), zeros.cuda(), 4, 128, out=Yp[:, :n])
    torch.cuda.synchronize()
    _check(Yp[:, :n], X, qw, scales, zeros, g_idx, 4, k, torch.float16)
    assert torch.all(Yp[:, n:] == 7.0)  # the padding is not written
    # rows of X that do not start on 16-byte boundaries: the scalar staging path
    Xo = torch.zeros(2, k + 3, dtype=torch.float16, device="cuda")
    Xo[:, :k] = X.cuda()
    Yo = quant_matmul(Xo[:, :k], qw.cuda(), scales.cuda(), zeros.cuda(), 4, 128)
    torch.cuda.synchronize()
    _check(Yo, X, qw, scales, zeros, g_idx, 4, k, torch.float16)
    # no tokens: nothing to do
    Y0 = quant_matmul(torch.empty(0, k, dtype=torch.float16, device="cuda"), qw.cuda(),
                      scales.cuda(), zeros.cuda(), 4, 128)
    assert Y0.shape == (0, n)


def test_qgemm_bad_g_idx_gives_nan_not_a_fault():
    # a g_idx entry outside [0, ngroups) is never read through
    from post_weight_quantization_23_b200 import quant_matmul
    n, k = 16, 256
    codes, scales, zeros, g_idx, X, qw = _inputs(n, k, 4, 128, 1, torch.float16, seed=5)
    bad = g_idx.clone()
    bad[17] = 1000
    Y = quant_matmul(X.cuda(), qw.cuda(), scales.cuda(), zeros.cuda(), 4, 128, bad.cuda())
    torch.cuda.synchronize()
    assert torch.all(torch.isnan(Y.float()))


@pytest.mark.parametrize("act,static,m", [(True, False, 3), (True, True, 1), (False, False, 32)])
def test_plan_matmul_matches_its_own_dequantized_weights(act, static, m):
    # A consistency property of the plan's glue (which g_idx it passes): Y from
    # the packed codes equals X W_hat^T with the plan's own fp32 dequantized
    # weights, up to the kernels' rounding (bounds as in _check).
    from post_weight_quantization_23_b200 import GptqPlan, QuantConfig
    spec = synth.CONFIGS["q_proj"].scaled(r=256, k=512, n=4096)
    W = synth.make_w(spec, 8).cuda()
    X = synth.make_x(spec, 8).cuda()
    cfg = QuantConfig(4, 128, 128, 0.01, act, static_groups=static)
    plan = GptqPlan(spec.r, spec.k, cfg, "cuda", deq_dtype=torch.float32)
    plan.hessian_add(X, spec.n)
    plan.run_after_hessian(W)
    plan.check()
    Xm = X[:m].contiguous()
    Y = plan.matmul(Xm)
    torch.cuda.synchronize()
    Wd = plan.deq.double().cpu().numpy()
    Xn = Xm.double().cpu().numpy()
    ref = Xn @ Wd.T
    k = spec.k
    u = U_OUT[torch.float16]
    # + 2 roundings: the plan's fp32 weights are themselves rounded s (c - z)
    e = (k + 4) * 2.0 ** -24 * (np.abs(Xn) @ np.abs(Wd).T)
    if _tc_path(4, 128, k, m, cfg.act_order and not cfg.static_groups):
        e = (2 * u + u * u) * (np.abs(Xn) @ np.abs(Wd).T) + 2 * e
    bound = u * np.abs(ref) + (1 + u) * e + 2.0 ** -25
    err = np.abs(Y.double().cpu().numpy() - ref)
    assert np.all(err <= bound), float((err / bound).max())


@pytest.mark.parametrize("n,k", [(11008, 4096), (4096, 11008)])
@pytest.mark.parametrize("m", [1, 2048])
def test_qgemm_full_size_7b_mlp_shapes(n, k, m):
    # The other layer shapes the bench times (gate/up and down of a 7B block),
    # int4 g128, in full on the device (decode kernel at 1 token, tensor cores
    # at 2048).  The packed words are seeded random int32 (every code pattern),
    # and the oracle checks 512 sampled output features.
    from post_weight_quantization_23_b200 import quant_matmul
    G = 128
    g = torch.Generator().manual_seed(n + m)
    qw = torch.randint(-2 ** 31, 2 ** 31 - 1, (n, k // 8), generator=g, dtype=torch.int32)
    scales = (torch.rand(n, k // G, generator=g) * 0.02 + 1e-3).float()
    zeros = torch.randint(0, 16, (n, k // G), generator=g, dtype=torch.int32)
    g_idx = (torch.arange(k) // G).to(torch.int32)
    spec = synth.CONFIGS["q_proj"].scaled(r=n, k=k, n=m)
    X = synth.make_x(spec, n + m)[:m].to(torch.float16)
    Y = quant_matmul(X.cuda(), qw.cuda(), scales.cuda(), zeros.cuda(), 4, G)
    torch.cuda.synchronize()
    rows = torch.randperm(n, generator=g)[:512]
    _check(Y.cpu()[:, rows], X, qw[rows], scales[rows], zeros[rows], g_idx, 4, k, torch.float16,
           _tc_path(4, G, k, m, False))
