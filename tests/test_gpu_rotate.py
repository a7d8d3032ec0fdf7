"""GPU parity of the rotation preprocessing (gptq_rotate) against the oracle's
explicit Q = diag(s) H_b / sqrt(b) in fp64, on seeded inputs.

Tolerance, from the arithmetic: a butterfly network of log2(b) fp32 additions
per output and one fp32 scaling gives |error| <= (log2(b) + 2) 2^-24 *
sum_block |x| / sqrt(b); the result is then rounded once to its dtype
(2^-11 relative for f16, 2^-8 for bf16, 2^-24 for f32), plus half the f16
subnormal spacing.
"""

import math

import numpy as np
import pytest
import torch

import oracle as O
import synth

pytestmark = pytest.mark.gpu

U_OUT = {torch.float16: 2.0 ** -11, torch.bfloat16: 2.0 ** -8, torch.float32: 2.0 ** -24}


def _check(got, x, signs, block, inverse, dtype):
    xn = x.double().numpy()
    ref = O.rotate(xn, signs.numpy(), block, inverse)
    rows, k = xn.shape
    blk_abs = np.abs(xn).reshape(rows, k // block, block).sum(axis=2)
    e32 = (math.log2(block) + 2) * 2.0 ** -24 * np.repeat(blk_abs, block, axis=1) / math.sqrt(block)
    bound = U_OUT[dtype] * np.abs(ref) + (1 + U_OUT[dtype]) * e32 + 2.0 ** -25
    g = got.double().cpu().numpy()
    err = np.abs(g - ref)
    assert np.all(np.isfinite(g))
    assert np.all(err <= bound), float((err / bound).max())
    return float((err / bound).max())


def _inputs(rows, k, dtype, seed):
    spec = synth.CONFIGS["q_proj"].scaled(r=rows, k=k, n=rows)
    x = synth.make_x(spec, seed).float().to(dtype)  # lognormal with outlier channels
    g = torch.Generator().manual_seed(seed)
    signs = (torch.randint(0, 2, (k,), generator=g) * 2 - 1).to(torch.int8)
    return x, signs


CASES = [
    (37, 256, 256, torch.float16, False),
    (64, 4096, 4096, torch.float16, False),
    (100, 11008, 256, torch.bfloat16, False),
    (16, 12288, 4096, torch.float32, False),
    (8, 8192, 8192, torch.float16, False),
    (5, 1536, 512, torch.float32, True),
    (33, 2048, 1024, torch.bfloat16, True),
    (7, 4096, 2048, torch.float16, True),
]


@pytest.mark.parametrize("case", CASES, ids=[f"r{c[0]}_k{c[1]}_b{c[2]}_{str(c[3])[6:]}"
                                              f"{'_inv' if c[4] else ''}" for c in CASES])
def test_rotate_parity(case):
    from post_weight_quantization_23_b200 import rotate
    rows, k, block, dtype, inverse = case
    x, signs = _inputs(rows, k, dtype, seed=rows + k)
    out = rotate(x.cuda(), signs.cuda(), block, inverse)
    torch.cuda.synchronize()
    print(case, _check(out, x, signs, block, inverse, dtype))


def test_rotate_in_place_strided_and_round_trip():
    from post_weight_quantization_23_b200 import rotate
    rows, k, block = 24, 2048, 2048
    x, signs = _inputs(rows, k, torch.float32, seed=9)
    buf = torch.zeros(rows, k + 64, dtype=torch.float32, device="cuda")
    buf[:, :k] = x.cuda()
    view = buf[:, :k]
    rotate(view, signs.cuda(), block, out=view)  # in place, padded rows
    torch.cuda.synchronize()
    _check(view, x, signs, block, False, torch.float32)
    assert torch.all(buf[:, k:] == 0)
    back = rotate(view.clone(), signs.cuda(), block, inverse=True)
    torch.cuda.synchronize()
    assert torch.allclose(back.cpu(), x, rtol=0, atol=1e-5 * float(x.abs().max()))


def test_rotate_full_size_activations_sampled_rows():
    # the full q_proj calibration matrix (262144 x 4096 f16), rotated on the
    # device in one launch; 64 sampled rows compared with the oracle
    from post_weight_quantization_23_b200 import rotate
    spec = synth.CONFIGS["q_proj"]
    X = synth.make_x(spec, 0)
    g = torch.Generator().manual_seed(1)
    signs = (torch.randint(0, 2, (spec.k,), generator=g) * 2 - 1).to(torch.int8)
    Xd = X.cuda()
    out = rotate(Xd, signs.cuda(), 4096)
    torch.cuda.synchronize()
    rows = torch.randint(0, spec.n, (64,), generator=g)
    _check(out[rows.cuda()].cpu(), X[rows], signs, 4096, False, torch.float16)
