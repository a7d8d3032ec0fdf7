"""Pins of the fp64 oracle against what the GPTQ pages and the mathematics fix.

CPU only.  Each test names the passage or fact it pins; together they are
chosen so that a plausible slip in the oracle (a dropped term, a wrong sign,
a transposed operand, an off-by-one group index) fails at least one of them.
"""

import itertools
import math
import os

import numpy as np
import pytest
import torch

import oracle as O
import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "worked_examples.txt")


def _golden():
    out = {}
    for line in open(GOLDEN):
        line = line.strip()
        if not line or line.startswith("#"):
            continue
        name, inputs, expected, cite = [p.strip() for p in line.split("|")]
        kv = lambda s: dict(x.split("=") for x in s.split())  # noqa: E731
        out[name] = (kv(inputs), kv(expected), cite)
    return out


G = _golden()


def _rand_layer(seed, r, k, n=None, corr=True):
    rng = np.random.default_rng(seed)
    n = n or 4 * k
    Z = rng.standard_normal((n, k))
    if corr:
        L = np.eye(k) + np.tril(rng.standard_normal((k, k)) / math.sqrt(k), -1)
        Z = Z @ L
    W = rng.normal(0, 0.02, (r, k))
    return W, Z, O.hessian(Z)


# ---------------------------------------------------------------- worked numbers

def test_quantization_equation_worked_example():
    # "GPTQ Quantization: Complete Technical Guide", Quantization Equation.
    inp, exp, _ = G["quant_eq"]
    v, s = float(inp["value"]), float(inp["scale"])
    for dt in (np.float32, np.float64):
        c = O.quantize_codes(np.array([v]), s, 0.0, None, dt)[0]
        assert c == int(exp["code"])
        deq = s * c
        assert deq == pytest.approx(float(exp["deq"]), abs=1e-12)
        assert abs(v - deq) == pytest.approx(float(exp["abs_err"]), abs=1e-12)


def test_single_weight_worked_example():
    # same page, "Example: Quantizing a Single Weight" (int4 range -8..7).
    inp, exp, _ = G["single_weight"]
    v, s = float(inp["value"]), float(inp["scale"])
    c = O.quantize_codes(np.array([v]), s, 0.0, None)[0]
    assert c == int(exp["code"]) and -8 <= c <= 7
    assert s * c == pytest.approx(float(exp["deq"]))
    assert v - s * c == pytest.approx(float(exp["err"]), abs=1e-9)


@pytest.mark.parametrize("rho", [0.5, 0.9, 0.99, 0.999])
def test_two_weight_compensation_closed_form(rho):
    # "GPTQ" (ozercemkelahmet.com), A worked example: w = (0.40, 0.31) on a 0.25
    # grid, H = [[1, rho], [rho, 1]], no damping.  Column 1 rounds to 0.50 (error
    # +0.10); the compensated second weight is 0.31 - 0.10*rho in closed form
    # (U = chol(H^-1) upper: U11 = 1/sqrt(1-rho^2), U12 = -rho/sqrt(1-rho^2)),
    # about 0.21 as rho -> 1, and it still rounds to 0.25.
    inp, exp, _ = G["two_weights"]
    w = np.array([[float(x) for x in inp["w"].split(",")]])
    s = float(inp["scale"])
    H = np.array([[1.0, rho], [rho, 1.0]])
    U = O.hinv_upper_factor(O.damp(H, 0.0))
    assert U[1, 0] == 0.0
    assert U[0, 0] == pytest.approx(1 / math.sqrt(1 - rho * rho), rel=1e-12)
    assert U[0, 1] == pytest.approx(-rho / math.sqrt(1 - rho * rho), rel=1e-10)
    res = O.sweep_unblocked(w, U, 8, -1, fixed_grid=(s, 0.0))
    rtn_q = [float(x) for x in exp["rtn"].split(",")]
    rtn_err = [float(x) for x in exp["rtn_err"].split(",")]
    assert res["qhat"][0, 0] == pytest.approx(rtn_q[0])
    assert res["qhat"][0, 0] - w[0, 0] == pytest.approx(rtn_err[0], abs=1e-12)
    assert rtn_q[1] - w[0, 1] == pytest.approx(rtn_err[1], abs=1e-12)
    w2 = res["w_at"][0, 1]
    assert w2 == pytest.approx(0.31 - 0.10 * rho, abs=1e-12)
    assert res["qhat"][0, 1] == pytest.approx(float(exp["q2"]))
    if rho == 0.999:
        assert w2 == pytest.approx(float(exp["w2_near_one"]), abs=5e-4)
    # the blocked sweep and the OBS-downdate sweep agree on the same example
    rb = O.sweep_blocked(w, U, 8, -1, 1, fixed_grid=(s, 0.0))
    ro = O.sweep_obs(w, H, 8, -1, fixed_grid=(s, 0.0))
    assert rb["w_at"][0, 1] == pytest.approx(w2, abs=1e-14)
    assert np.array_equal(ro["codes"], res["codes"])


def test_bits_per_weight_memory_arithmetic():
    # "GPTQ" (ozercemkelahmet.com), Memory arithmetic.
    inp, exp, _ = G["bits_per_weight"]
    b = O.storage_bits_per_weight(int(inp["bits"]), int(inp["group"]), 4096,
                                  int(inp["scale_bits"]), int(inp["zero_bits"]))
    assert round(b, 2) == float(exp["approx"])
    over128 = O.storage_bits_per_weight(4, 128, 4096, 16, 4) - 4
    over32 = O.storage_bits_per_weight(4, 32, 4096, 16, 4) - 4
    assert over32 / over128 == pytest.approx(float(exp["overhead_g32_over_g128"]))


# ---------------------------------------------------------------- Hessian

def test_hessian_closed_form_and_chunking():
    # H = (2/n) X^T X on a hand-checkable X; chunked accumulation normalises by
    # the total token count (READING R1).
    X = np.array([[1.0, 0.0], [0.0, 1.0], [1.0, 1.0]])
    H = O.hessian(X)
    assert np.allclose(H, (2.0 / 3.0) * np.array([[2.0, 1.0], [1.0, 2.0]]), rtol=0, atol=1e-15)
    rng = np.random.default_rng(0)
    X = rng.standard_normal((100, 7)).astype(np.float32)
    H1 = O.hessian(X)
    H2 = O.hessian([X[:13], X[13:60], X[60:]])
    assert np.allclose(H1, H2, rtol=1e-13, atol=1e-13)
    assert np.allclose(H1, H1.T)
    assert np.linalg.eigvalsh(H1).min() > 0
    # brute force single entry
    i, j = 2, 5
    assert H1[i, j] == pytest.approx(2.0 / 100 * sum(float(X[t, i]) * float(X[t, j]) for t in range(100)),
                                     rel=1e-12)


def test_hessian_exact_on_fp16_inputs():
    # the oracle reads f16/bf16 values exactly
    x16 = torch.tensor([[0.1, 3.0], [-2.5, 0.125]], dtype=torch.float16)
    H = O.hessian(x16.numpy())
    xv = x16.double().numpy()
    assert H[0, 1] == (2.0 / 2) * (xv[0, 0] * xv[0, 1] + xv[1, 0] * xv[1, 1])


# ---------------------------------------------------------------- inverse factor

def test_hinv_factor_definition_and_reversed_route():
    # U^T U = H^-1 with U upper; and the reversed-order route used by the CUDA
    # library (H = V V^T with V upper, U = V^-1, V from the lower Cholesky of
    # the index-reversed H) is the same matrix.
    _, _, H = _rand_layer(1, 4, 40)
    Hd = O.damp(H, 0.01)
    U = O.hinv_upper_factor(Hd)
    assert np.allclose(np.tril(U, -1), 0)
    assert np.all(np.diag(U) > 0)
    assert np.allclose(U.T @ U, np.linalg.inv(Hd), rtol=1e-10, atol=1e-12)
    J = np.arange(40)[::-1]
    Lr = np.linalg.cholesky(Hd[np.ix_(J, J)])
    V = Lr[np.ix_(J, J)]
    assert np.allclose(V @ V.T, Hd, atol=1e-12)
    assert np.allclose(np.linalg.inv(V), U, rtol=1e-10, atol=1e-12)


def test_not_positive_definite_raises():
    rng = np.random.default_rng(3)
    X = rng.standard_normal((4, 10))  # rank 4 < 10, no dead column
    H = O.hessian(X)
    with pytest.raises(O.NotPositiveDefinite):
        O.hinv_upper_factor(O.damp(H, 0.0))
    O.hinv_upper_factor(O.damp(H, 0.01))  # damping fixes it


def test_damping_uses_mean_of_diagonal():
    H = np.diag([1.0, 2.0, 3.0, 6.0])
    Hd = O.damp(H, 0.1)
    assert np.allclose(np.diag(Hd) - np.diag(H), 0.1 * 3.0)


# ---------------------------------------------------------------- grid

def test_grid_properties():
    rng = np.random.default_rng(5)
    w = rng.normal(0, 0.02, (50, 32))
    for bits in (2, 3, 4, 8):
        maxq = 2 ** bits - 1
        s, z = O.grid_params(w, maxq)
        assert np.all((z >= 0) & (z <= maxq))
        c = O.quantize_codes(w, s[:, None], z[:, None], maxq)
        q = s[:, None].astype(np.float64) * (c - z[:, None])
        assert np.all((c >= 0) & (c <= maxq))
        # round to nearest: error at most half a step (plus fp32 slack)
        assert np.all(np.abs(w - q) <= s[:, None] * (0.5 + 1e-5) + 1e-12)
        # the range spans the grid: max -> top code, min -> bottom code (+-1 from rounding z)
        assert np.all(c.max(axis=1) >= maxq - 1) and np.all(c.min(axis=1) <= 1)
    # all-zero group: scale is the 1e-8 floor, everything codes to the zero point 0
    s, z = O.grid_params(np.zeros((1, 8)), 15)
    assert s[0] == np.float32(1e-8) / np.float32(15) and z[0] == 0


def test_symmetric_grid_closed_form_and_properties():
    # READING R14 (symmetric grid: range [-a, a], zero point (maxq + 1) / 2).
    # Exact binary values, 2 bits: a = 0.75, scale = 1.5 / 3 = 0.5, zero = 2;
    # w / s = -1.5, 0.5, 1.0 round half to even to -2, 0, 1 -> codes 0, 2, 3.
    w = np.array([[-0.75, 0.25, 0.5]])
    s, z = O.grid_params(w, 3, sym=True)
    assert s[0] == np.float32(0.5) and z[0] == 2
    c = O.quantize_codes(w, s[:, None], z[:, None], 3)
    assert c.tolist() == [[0.0, 2.0, 3.0]]
    assert (s[0] * (c - z[0])).tolist() == [[-1.0, 0.0, 0.5]]
    rng = np.random.default_rng(7)
    x = rng.normal(0, 0.02, (40, 32)) + rng.normal(0, 0.01, (40, 1))  # skewed groups
    for bits in (2, 3, 4, 8):
        maxq = 2 ** bits - 1
        s, z = O.grid_params(x, maxq, sym=True)
        assert np.all(z == (maxq + 1) // 2)
        a = np.maximum(np.abs(x.astype(np.float32)).max(axis=1), 0)
        assert np.array_equal(s, ((a + a) / np.float32(maxq)).astype(np.float32))
        c = O.quantize_codes(x, s[:, None], z[:, None], maxq)
        assert np.all((c >= 0) & (c <= maxq))
    # all-positive group: only the upper half of the codes is used
    s, z = O.grid_params(np.abs(x), 15, sym=True)
    c = O.quantize_codes(np.abs(x), s[:, None], z[:, None], 15)
    assert np.all(c >= z[:, None])


@pytest.mark.parametrize("gs,bs,act", [(32, 32, False), (-1, 32, False), (64, 32, True)])
def test_symmetric_invariants(gs, bs, act):
    # R14 with the pinned invariants: diagonal H == RTN, blocked == unblocked,
    # Cholesky sweep == OBS downdate.
    rng = np.random.default_rng(12)
    W = rng.normal(0, 0.02, (16, 96))
    H = np.diag(rng.lognormal(0, 1, 96))
    res = O.gptq(W, H, bits=4, group_size=gs, block_size=bs, act_order=act, sym=True)
    ref = O.rtn(W[:, res["perm"]], 4, gs, sym=True)
    assert np.array_equal(res["codes"][:, res["perm"]], ref["codes"])
    assert np.array_equal(res["scales"], ref["scales"])
    W2, _, H2 = _rand_layer(8, 12, 96)
    U = O.hinv_upper_factor(O.damp(H2, 0.01))
    a = O.sweep_unblocked(W2, U, 3, gs, sym=True)
    b = O.sweep_blocked(W2, U, 3, gs, bs, sym=True)
    assert np.array_equal(a["codes"], b["codes"])
    assert np.all(a["zeros"] == 4)
    c = O.sweep_obs(W2, O.damp(H2, 0.01), 3, gs, sym=True)
    assert np.array_equal(a["codes"], c["codes"])


# ---------------------------------------------------------------- static groups (R15)

def test_static_grid_closed_form():
    # READING R15: a static grid is fitted to the ORIGINAL columns of its group.
    # 2 bits (maxq 3), G = 2: group 1 holds 0.75 and 0.25 (exact binary values),
    # so lo = min(0, 0.25) = 0, hi = 0.75, scale = 0.75 / 3 = 0.25, zero = 0.
    # Column 0 (0.6 on a grid of step ~0.25, zero 1) is rounded with an error,
    # and a strongly correlated H moves columns 2 and 3 before they are
    # quantized, so the dynamic grid of group 1 (fitted after compensation)
    # differs while the first group's grid is the same either way.
    W = np.array([[0.6, -0.15, 0.75, 0.25]])
    C = np.array([[1.0, 0.9, 0.8, 0.7], [0.9, 1.0, 0.9, 0.8], [0.8, 0.9, 1.0, 0.9],
                  [0.7, 0.8, 0.9, 1.0]])
    st = O.gptq(W, C, bits=2, group_size=2, block_size=2, percdamp=0.01, static_groups=True)
    assert st["scales"][0, 1] == 0.25 and st["zeros"][0, 1] == 0
    dy = O.gptq(W, C, bits=2, group_size=2, block_size=2, percdamp=0.01)
    assert dy["scales"][0, 0] == st["scales"][0, 0] and dy["zeros"][0, 0] == 1
    assert dy["scales"][0, 1] != 0.25
    # column 0 is quantized first on either grid: rint(0.6 / 0.25) + 1 = 3
    assert st["codes"][0, 0] == 3 and dy["codes"][0, 0] == 3


@pytest.mark.parametrize("gs,bs", [(32, 32), (48, 32), (-1, 64), (16, 64)])
def test_static_groups_diagonal_hessian_is_rtn_in_original_order(gs, bs):
    # A diagonal H means no compensation, so every column is rounded on its
    # grid alone; with static groups those grids are RTN's on the ORIGINAL
    # columns, whatever order act-order imposes.  Processing-order groups (the
    # dynamic rule) would fail this under act-order.  Dead column 7 counts as 0.
    rng = np.random.default_rng(21)
    r, k = 12, 96
    W = rng.normal(0, 0.02, (r, k))
    d = rng.lognormal(0, 1, k)
    d[7] = 0.0
    H = np.diag(d)
    res = O.gptq(W, H, bits=3, group_size=gs, block_size=bs, act_order=True,
                 static_groups=True)
    assert not np.array_equal(res["perm"], np.arange(k))
    W0 = W.copy()
    W0[:, 7] = 0.0
    ref = O.rtn(W0, 3, gs)
    assert np.array_equal(res["codes"], ref["codes"])
    assert np.array_equal(res["scales"], ref["scales"])
    assert np.array_equal(res["zeros"], ref["zeros"])
    G = k if gs == -1 else gs
    assert np.array_equal(res["g_idx"], np.arange(k) // G)


@pytest.mark.parametrize("gs,B,act", [(48, 32, True), (32, 32, False), (8, 96, True),
                                      (100, 64, False)])
def test_static_groups_blocked_unblocked_obs_agree(gs, B, act):
    # With grids fixed before the sweep, the lazy blocks cannot change a grid,
    # so the blocked sweep equals the column-by-column one for ANY group and
    # block sizes (no alignment needed), and both equal the OBS downdate.
    W, _, H = _rand_layer(31, 10, 192)
    k = W.shape[1]
    G = k if gs == -1 else gs
    Hf, Wf, _ = O.fix_dead_columns(H, W)
    perm = O.act_order_perm(Hf) if act else np.arange(k)
    Wp, Hd = Wf[:, perm], O.damp(Hf[np.ix_(perm, perm)], 0.01)
    U = O.hinv_upper_factor(Hd)
    ss, zz = O.static_grids(Wf, 4, gs)
    st = (ss, zz, perm // G)
    a = O.sweep_unblocked(Wp, U, 4, gs, static=st)
    b = O.sweep_blocked(Wp, U, 4, gs, B, static=st)
    c = O.sweep_obs(Wp, Hd, 4, gs, static=st)
    assert np.array_equal(a["codes"], b["codes"]) and np.array_equal(a["codes"], c["codes"])
    assert np.allclose(a["qhat"], b["qhat"], rtol=0, atol=1e-15)
    res = O.gptq(W, H, 4, gs, B, 0.01, act, static_groups=True)
    assert np.array_equal(res["codes"][:, perm], b["codes"])


@pytest.mark.parametrize("act", [False, True])
def test_static_equals_dynamic_for_one_group_per_row(act):
    # group_size = -1: the dynamic rule already takes the row's one grid from
    # the original row before the first column (READING R5), so static and
    # dynamic groups are the same computation.
    W, _, H = _rand_layer(5, 8, 64)
    a = O.gptq(W, H, 4, -1, 32, 0.01, act)
    b = O.gptq(W, H, 4, -1, 32, 0.01, act, static_groups=True)
    assert np.array_equal(a["codes"], b["codes"])
    assert np.array_equal(a["scales"], b["scales"]) and np.array_equal(a["zeros"], b["zeros"])
    assert a["loss"] == b["loss"]


def test_static_groups_loss_identity_and_sym():
    # The OBS accounting (loss = sum err^2 - lambda ||W0 - Q||^2) does not depend
    # on how the grids were chosen; checked with static groups, act-order, dead
    # columns and both grid kinds.  Static symmetric grids keep zero = (maxq+1)/2.
    spec = synth.CONFIGS["q_proj"].scaled(r=16, k=128, n=2000)
    W = synth.make_w(spec, 4).numpy().astype(np.float64)
    X = synth.make_x(spec, 4).numpy()
    X[:, 9] = 0
    H = O.hessian(X)
    for sym in (False, True):
        res = O.gptq(W, H, 4, 32, 64, 0.01, True, sym=sym, static_groups=True)
        Hf, Wf, _ = O.fix_dead_columns(H, W)
        perm = res["perm"]
        lam = 0.01 * np.mean(np.diag(Hf))
        ss, zz = O.static_grids(Wf, 4, 32, sym=sym)
        sw = O.sweep_blocked(Wf[:, perm], res["U"], 4, 32, 64, sym=sym, static=(ss, zz, perm // 32))
        e2 = (sw["err"] ** 2).sum(axis=1)
        d2 = ((Wf[:, perm] - sw["qhat"]) ** 2).sum(axis=1)
        assert np.allclose(e2 - lam * d2, res["loss_rows"], rtol=1e-10, atol=0)
        if sym:
            assert np.all(res["zeros"] == 8)


def test_half_to_even_rounding():
    c = O.quantize_codes(np.array([6.5, 7.5, -0.5, 2.4999]), 1.0, 0.0, None)
    assert list(c) == [6, 8, 0, 2]


# ---------------------------------------------------------------- sweeps: invariants

@pytest.mark.parametrize("gs,bs,act", [(32, 32, False), (16, 64, False), (-1, 32, False),
                                       (32, 32, True), (64, 32, True)])
def test_diagonal_hessian_reduces_to_rtn(gs, bs, act):
    # "GPTQ" (ozercemkelahmet.com), A worked example: independent features do
    # not share blame.  A diagonal H gives a diagonal U, no compensation, and
    # GPTQ equals round-to-nearest exactly (codes, scales, zeros).
    rng = np.random.default_rng(11)
    r, k = 24, 128
    W = rng.normal(0, 0.02, (r, k))
    H = np.diag(rng.lognormal(0, 1, k))
    res = O.gptq(W, H, bits=4, group_size=gs, block_size=bs, percdamp=0.01, act_order=act)
    perm = res["perm"]
    ref = O.rtn(W[:, perm], 4, gs)
    assert np.array_equal(res["codes"][:, perm], ref["codes"])
    assert np.array_equal(res["scales"], ref["scales"])
    assert np.array_equal(res["zeros"], ref["zeros"])
    if act:
        assert np.all(np.diff(np.diag(H)[perm]) <= 0)


@pytest.mark.parametrize("c", [4.0, 0.25, 3.0])
def test_scale_invariance(c):
    # Scaling H by c > 0 scales U by 1/sqrt(c) and err by sqrt(c): the
    # compensation err*U is unchanged, so are the codes (exactly for powers of 4).
    W, _, H = _rand_layer(2, 16, 64)
    a = O.gptq(W, H, bits=3, group_size=32, block_size=32)
    b = O.gptq(W, c * H, bits=3, group_size=32, block_size=32)
    if c in (4.0, 0.25):
        assert np.array_equal(a["codes"], b["codes"])
        assert np.array_equal(a["scales"], b["scales"])
    else:
        assert (a["codes"] != b["codes"]).mean() < 1e-3
    assert b["loss"] == pytest.approx(c * a["loss"], rel=1e-6 if c != 3.0 else 1e-2)


@pytest.mark.parametrize("gs", [8, -1, 5])
def test_cholesky_sweep_equals_obs_downdate(gs):
    # "GPTQ" (ozercemkelahmet.com) Step 6: the rows of the Cholesky factor hold
    # the numbers the explicit inverse-Hessian downdate of the guide's Detailed
    # Algorithm would produce; the two sweeps agree to fp64 round-off.
    W, _, H = _rand_layer(4, 12, 24)
    Hd = O.damp(H, 0.01)
    U = O.hinv_upper_factor(Hd)
    a = O.sweep_unblocked(W, U, 3, gs)
    b = O.sweep_obs(W, Hd, 3, gs)
    assert np.array_equal(a["codes"], b["codes"])
    assert np.allclose(a["qhat"], b["qhat"], atol=1e-14)
    assert np.array_equal(a["zeros"], b["zeros"])


@pytest.mark.parametrize("B", [1, 8, 32, 128, 96, 200])
@pytest.mark.parametrize("gs", [8, -1])
def test_blocked_equals_unblocked(B, gs):
    # "GPTQ" (ozercemkelahmet.com) Step 7: lazy batching must not change the result.
    W, _, H = _rand_layer(6, 20, 96)
    U = O.hinv_upper_factor(O.damp(H, 0.01))
    a = O.sweep_unblocked(W, U, 4, gs)
    b = O.sweep_blocked(W, U, 4, gs, B)
    assert np.array_equal(a["codes"], b["codes"])
    assert np.array_equal(a["scales"], b["scales"])
    assert np.allclose(a["w_at"], b["w_at"], rtol=0, atol=1e-13)


def test_blocked_equals_unblocked_ragged():
    # k not a multiple of the group or block size: last group and block are short
    W, _, H = _rand_layer(7, 9, 100)
    U = O.hinv_upper_factor(O.damp(H, 0.01))
    a = O.sweep_unblocked(W, U, 4, 32)
    b = O.sweep_blocked(W, U, 4, 32, 64)
    assert a["scales"].shape == (9, 4)
    assert np.array_equal(a["codes"], b["codes"])


def test_group_alignment_is_enforced():
    W, _, H = _rand_layer(7, 4, 48)
    U = O.hinv_upper_factor(O.damp(H, 0.01))
    with pytest.raises(ValueError):
        O.sweep_blocked(W, U, 4, 24, 32)


def test_per_row_equals_group_of_k():
    W, _, H = _rand_layer(8, 10, 64)
    a = O.gptq(W, H, bits=4, group_size=-1, block_size=32)
    b = O.gptq(W, H, bits=4, group_size=64, block_size=32)
    assert np.array_equal(a["codes"], b["codes"]) and np.array_equal(a["scales"], b["scales"])
    assert np.all(a["g_idx"] == 0)


# ---------------------------------------------------------------- loss

def test_layer_loss_equals_direct_output_error():
    # READING R11: tr(D H0 D^T) with H0 = (2/n) X^T X equals (2/n)||D X^T||^2.
    W, X, H = _rand_layer(9, 6, 16, n=50)
    res = O.gptq(W, H, bits=3, group_size=8, block_size=8)
    D = W - res["qhat"]
    direct = 2.0 / X.shape[0] * np.sum((D @ X.T) ** 2)
    assert res["loss"] == pytest.approx(direct, rel=1e-12)
    assert np.allclose(res["loss_rows"], 2.0 / X.shape[0] * np.sum((D @ X.T) ** 2, axis=1))


@pytest.mark.parametrize("gs,bs,act,bits", [(32, 32, False, 4), (128, 128, True, 3),
                                             (-1, 64, False, 2), (16, 64, True, 8)])
def test_loss_equals_obs_error_sum(gs, bs, act, bits):
    # Optimal Brain Surgeon accounting ("GPTQ" page, Where it came from; the
    # guide's Detailed Algorithm): fixing column i and compensating the rest
    # raises (w - q)^T Hd (w - q) by err_i^2 = (w_i - q_i)^2 / U_ii^2, so the
    # damped layer error is the sum of err^2 and the undamped one subtracts
    # lambda * ||W0 - Q||^2.  Holds row by row, with groups, act-order and dead
    # columns (whose original weights count as 0).
    spec = synth.CONFIGS["q_proj"].scaled(r=24, k=192, n=3000)
    W = synth.make_w(spec, bits).numpy().astype(np.float64)
    X = synth.make_x(spec, bits).numpy()
    X[:, [5, 77]] = 0
    H = O.hessian(X)
    res = O.gptq(W, H, bits, gs, bs, 0.01, act)
    Hf, Wf, dead = O.fix_dead_columns(H, W)
    perm = res["perm"]
    lam = 0.01 * np.mean(np.diag(Hf))
    sw = O.sweep_blocked(Wf[:, perm], res["U"], bits, gs, bs)
    e2 = (sw["err"] ** 2).sum(axis=1)
    d2 = ((Wf[:, perm] - sw["qhat"]) ** 2).sum(axis=1)
    assert np.allclose(e2 - lam * d2, res["loss_rows"], rtol=1e-10, atol=0)


@pytest.mark.parametrize("seed", range(5))
def test_gptq_beats_rtn_on_tiny_layer(seed):
    # "GPTQ" (ozercemkelahmet.com), sketch remark: compare the output error with
    # plain rounding on correlated random data.  Per seed, GPTQ <= RTN; the
    # absolute gap grows as the bit width falls.
    spec = synth.CONFIGS["tiny"]
    W = synth.make_w(spec, seed).numpy()
    X = synth.make_x(spec, seed).numpy()
    H = O.hessian(X)
    gaps = []
    for bits in (4, 3, 2):
        g = O.gptq(W, H, bits=bits, group_size=32, block_size=32)
        r = O.rtn(W, bits, 32)
        lr, _ = O.layer_loss(W, r["qhat"], H)
        assert g["loss"] <= lr
        gaps.append(lr - g["loss"])
    assert gaps[0] < gaps[1] < gaps[2]


def test_brute_force_optimum_bounds_both():
    # r = 1, k = 6, 2-bit, one grid per row taken from the original weights (what
    # GPTQ uses with group_size = -1): enumerating all 4^6 code vectors gives the
    # true optimum, which neither GPTQ nor RTN can beat; on this correlated
    # example GPTQ is at least as good as RTN.
    rng = np.random.default_rng(12)
    k = 6
    W, X, H = _rand_layer(13, 1, k, n=40)
    s, z = O.grid_params(W, 3)
    best = math.inf
    for codes in itertools.product(range(4), repeat=k):
        q = s[0].astype(np.float64) * (np.array(codes, dtype=np.float64) - z[0])
        best = min(best, O.layer_loss(W, q[None, :], H)[0])
    g = O.gptq(W, H, bits=2, group_size=-1, block_size=k, percdamp=0.0)
    r = O.rtn(W, 2, -1)
    lr = O.layer_loss(W, r["qhat"], H)[0]
    assert best <= g["loss"] + 1e-15 and best <= lr + 1e-15
    assert g["loss"] <= lr
    del rng


# ---------------------------------------------------------------- dead columns / act-order

def test_dead_columns():
    # READING R2: a feature that is always zero gives H_ii = 0; it is marked
    # dead, its weights are zeroed (code = zero point) and its original weight
    # values change nothing else.
    W, X, _ = _rand_layer(14, 8, 32, n=200)
    X[:, [3, 17]] = 0.0
    H = O.hessian(X)
    a = O.gptq(W, H, bits=4, group_size=16, block_size=16)
    W2 = W.copy()
    W2[:, [3, 17]] = 123.0
    b = O.gptq(W2, H, bits=4, group_size=16, block_size=16)
    assert list(np.flatnonzero(a["dead"])) == [3, 17]
    Hf, Wf, dead = O.fix_dead_columns(H, W)
    assert Hf[3, 3] == 1.0 and Hf[17, 17] == 1.0 and np.all(Wf[:, [3, 17]] == 0)
    assert np.array_equal(a["codes"], b["codes"])
    assert a["loss"] == pytest.approx(b["loss"], rel=1e-12)
    zp = a["zeros"][:, a["g_idx"][3]]
    assert np.array_equal(a["codes"][:, 3], zp.astype(np.int64))


def test_act_order_permutation_and_gidx():
    # "GPTQ" (ozercemkelahmet.com), Optional refinements: act-order processes
    # columns by descending diag(H); g_idx maps each original column to the
    # group (in processing order) whose scale/zero it uses.  Ties: READING R3.
    H = np.diag([1.0, 5.0, 5.0, 2.0, 9.0, 1.0, 0.5, 5.0])
    perm = O.act_order_perm(H)
    assert list(perm) == [4, 1, 2, 7, 3, 0, 5, 6]
    W = np.random.default_rng(15).normal(0, 0.02, (3, 8))
    res = O.gptq(W, H, bits=4, group_size=4, block_size=4, act_order=True)
    assert list(res["g_idx"]) == [1, 0, 0, 1, 0, 1, 1, 0]
    res2 = O.gptq(W, H, bits=4, group_size=4, block_size=4, act_order=False)
    assert list(res2["g_idx"]) == [0, 0, 0, 0, 1, 1, 1, 1]


def test_act_order_candidate_accepted_only_at_ties():
    # a candidate order may swap columns whose diagonals agree within the
    # tolerance, nothing else
    d = np.array([1.0, 5.0, 5.0 * (1 + 1e-7), 2.0, 9.0])
    H = np.diag(d)
    assert list(O.act_order_perm(H)) == [4, 2, 1, 3, 0]
    assert list(O.act_order_perm(H, [4, 1, 2, 3, 0], 1e-5)) == [4, 1, 2, 3, 0]
    with pytest.raises(ValueError):
        O.act_order_perm(H, [4, 1, 2, 0, 3], 1e-5)
    with pytest.raises(ValueError):
        O.act_order_perm(H, [4, 1, 1, 3, 0], 1e-5)


# ---------------------------------------------------------------- the sketch

def _sketch_in_my_words(W, X, bits, damp_frac):
    """What the minimal Python sketch on the "GPTQ" page computes, re-expressed
    with torch fp64 on the CPU: one grid per row from the raw min/max (no zero
    inclusion), H = 2 X^T X / n damped by the mean diagonal, the three-call
    factor, and the unblocked column loop."""
    Wt = torch.tensor(W, dtype=torch.float64)
    Xt = torch.tensor(X, dtype=torch.float64)
    H = 2.0 * Xt.T @ Xt / Xt.shape[0]
    H = H + damp_frac * torch.diagonal(H).mean() * torch.eye(H.shape[0], dtype=torch.float64)
    U = torch.linalg.cholesky(torch.cholesky_inverse(torch.linalg.cholesky(H)), upper=True)
    top = 2 ** bits - 1
    lo = Wt.min(dim=1, keepdim=True).values
    hi = Wt.max(dim=1, keepdim=True).values
    step = (hi - lo).clamp(min=1e-8) / top
    zp = torch.round(-lo / step)
    out = torch.zeros_like(Wt)
    for i in range(Wt.shape[1]):
        col = Wt[:, i:i + 1].clone()
        qc = step * (torch.clamp(torch.round(col / step) + zp, 0, top) - zp)
        out[:, i:i + 1] = qc
        Wt[:, i + 1:] -= ((col - qc) / U[i, i]) @ U[i:i + 1, i + 1:]
    return out.numpy()


def test_oracle_reproduces_page_sketch():
    # "GPTQ" (ozercemkelahmet.com), A minimal Python sketch: with one group per
    # row, the sketch's raw range and fp64 decisions, the oracle's sweep gives
    # the sketch's result.
    W, X, _ = _rand_layer(16, 10, 48, n=300)
    ref = _sketch_in_my_words(W, X, 4, 0.01)
    H = O.hessian(X)
    res = O.gptq(W, H, bits=4, group_size=-1, block_size=48, percdamp=0.01,
                 include_zero=False, decide_dtype=np.float64, blocked=False)
    assert np.allclose(res["qhat"], ref, rtol=0, atol=1e-12)


# ---------------------------------------------------------------- pack / dequant

@pytest.mark.parametrize("bits", [2, 3, 4, 8])
def test_pack_unpack_identity(bits):
    rng = np.random.default_rng(bits)
    k = 96 if bits == 3 else 64
    codes = rng.integers(0, 2 ** bits, (7, k))
    q = O.pack(codes, bits)
    assert q.dtype == np.int32 and q.shape == (7, k * bits // 32)
    assert np.array_equal(O.unpack(q, k, bits), codes)


def test_pack_four_bit_layout():
    # "GPTQ" (ozercemkelahmet.com) Step 8: eight 4-bit codes per 32-bit word;
    # READING R9 puts code j of a word in bits [4j, 4j+4).
    codes = np.array([[1, 2, 3, 4, 5, 6, 7, 8, 15, 0, 0, 0, 0, 0, 0, 9]])
    q = O.pack(codes, 4).view(np.uint32)
    assert q[0, 0] == 0x87654321 and q[0, 1] == 0x9000000F


def test_pack_three_bit_straddles_words():
    codes = np.zeros((1, 32), dtype=np.int64)
    codes[0, 10] = 7  # stream bits 30..32 straddle words 0 and 1
    q = O.pack(codes, 3).view(np.uint32)
    assert q[0, 0] == 0xC0000000 and q[0, 1] == 0x1 and q[0, 2] == 0


def test_dequant_matches_grid():
    rng = np.random.default_rng(17)
    codes = rng.integers(0, 16, (5, 64))
    scales = rng.uniform(1e-3, 1e-2, (5, 2)).astype(np.float32)
    zeros = rng.integers(0, 16, (5, 2))
    g_idx = np.arange(64) // 32
    out = O.dequant(codes, scales, zeros, g_idx)
    exp = scales[:, g_idx] * (codes - zeros[:, g_idx]).astype(np.float32)
    assert out.dtype == np.float32 and np.array_equal(out, exp)
    assert np.array_equal(O.dequant(codes, scales, zeros, g_idx, np.float16), exp.astype(np.float16))


# ---------------------------------------------------------------- replay

def test_tie_replay_accepts_only_ties():
    # The replay takes a candidate's code only at a rounding tie; a planted
    # off-by-one away from a tie is still reported as a mismatch.
    W, _, H = _rand_layer(18, 8, 64)
    ref = O.gptq(W, H, bits=4, group_size=32, block_size=32)
    cand = ref["codes"].copy()
    rep = O.gptq(W, H, bits=4, group_size=32, block_size=32, force_codes=cand,
                 force_zeros=ref["zeros"])
    assert rep["n_forced"] == 0 and np.array_equal(rep["codes"], cand)
    cand[2, 5] = cand[2, 5] + 1 if cand[2, 5] < 15 else cand[2, 5] - 1
    rep = O.gptq(W, H, bits=4, group_size=32, block_size=32, force_codes=cand,
                 force_zeros=ref["zeros"], tau=1e-9)
    assert rep["codes"][2, 5] != cand[2, 5]


# ---------------------------------------------------------------- inference product

def test_dequant_matmul_worked_word():
    # One packed word, LSB first: codes 0..7 -> 0x76543210.  scale 0.5, zero 3
    # gives W_hat = 0.5 * (c - 3) = -1.5, -1, ..., 2.  A token of ones sums it
    # (0.5 * (28 - 24) = 2.0); the token 1..8 gives 0.5 * sum_i (i + 1)(i - 3)
    # = 0.5 * (140 - 56 - 24) = 30.
    qw = np.array([[0x76543210]], dtype=np.int64).astype(np.uint32).view(np.int32)
    assert O.unpack(qw, 8, 4).tolist() == [list(range(8))]
    X = np.array([np.ones(8), np.arange(1, 9)], dtype=np.float64)
    Y = O.dequant_matmul(X, qw, np.array([[0.5]]), np.array([[3]]), np.zeros(8, int), 4, 8)
    assert Y.tolist() == [[2.0], [30.0]]


@pytest.mark.parametrize("bits", [2, 3, 4, 8])
def test_dequant_matmul_identity_and_brute_force(bits):
    # X = I recovers W_hat^T, exact in fp64, so rounding it to fp32 gives
    # dequant() of the unpacked codes (one fp32 product, correctly rounded);
    # a triple loop over plain Python numbers gives the same product.
    rng = np.random.default_rng(bits)
    n, k, G = 5, 64, 16
    codes = rng.integers(0, 2 ** bits, (n, k))
    scales = (rng.random((n, k // G)) * 0.01 + 1e-3).astype(np.float32)
    zeros = rng.integers(0, 2 ** bits, (n, k // G))
    g_idx = rng.permutation(np.arange(k) // G)  # an act-order style g_idx
    qw = O.pack(codes, bits)
    Y = O.dequant_matmul(np.eye(k), qw, scales, zeros, g_idx, bits, k)
    assert np.array_equal(Y.T.astype(np.float32), O.dequant(codes, scales, zeros, g_idx))
    X = rng.standard_normal((3, k)).astype(np.float16)
    Y = O.dequant_matmul(X, qw, scales, zeros, g_idx, bits, k)
    for t in range(3):
        for j in range(n):
            acc = 0.0
            for c in range(k):
                g = int(g_idx[c])
                acc += float(X[t, c]) * float(scales[j, g]) * (int(codes[j, c]) - int(zeros[j, g]))
            assert abs(acc - Y[t, j]) <= 1e-12 * max(1.0, abs(acc))


@pytest.mark.parametrize("act,static", [(False, False), (True, False), (True, True)])
def test_dequant_matmul_of_gptq_output_equals_sweep_weights(act, static):
    # The packed output of a GPTQ run, multiplied through the inference
    # product, gives X Qhat^T with the sweep's own dequantized weights (a
    # different route: the sweep's scale * (code - zero) at quantization time).
    W, Z, H = _rand_layer(41, 12, 128)
    res = O.gptq(W, H, 4, 32, 32, 0.01, act, static_groups=static)
    qw = O.pack(res["codes"], 4)
    X = Z[:7].astype(np.float16).astype(np.float64)
    Y = O.dequant_matmul(X, qw, res["scales"], res["zeros"].astype(np.int64), res["g_idx"], 4, 128)
    assert np.allclose(Y, X @ res["qhat"].T, rtol=1e-13, atol=1e-15)


# ---------------------------------------------------------------- rotation (R16)

def test_rotation_worked_values_and_outlier_spread():
    # b = 4, all signs +1: e_0 Q is the first row of H_4 / 2 = [1, 1, 1, 1] / 2;
    # e_1 Q = [1, -1, 1, -1] / 2.  One outlier of size A spreads to A / sqrt(b)
    # in every coordinate ("GPTQ", Variants and extensions: outliers spread out).
    s = np.ones(4)
    assert O.rotate(np.eye(4)[:2], s, 4).tolist() == [[0.5, 0.5, 0.5, 0.5],
                                                      [0.5, -0.5, 0.5, -0.5]]
    # the signs act on the input coordinates (Q = diag(s) H / sqrt(b)): with s_1 = -1,
    # e_1 Q = -[1, -1, 1, -1] / 2, while signs on the outputs would give
    # [1, -1, 1, -1] / 2 * s = [0.5, 0.5, 0.5, -0.5]
    s = np.array([1, -1, 1, 1])
    assert O.rotate(np.eye(4)[1:2], s, 4).tolist() == [[-0.5, 0.5, -0.5, 0.5]]
    assert O.rotate(np.array([[-0.5, 0.5, -0.5, 0.5]]), s, 4, inverse=True).tolist() == [[0, 1, 0, 0]]
    x = np.zeros((1, 256))
    x[0, 37] = 100.0
    y = O.rotate(x, np.random.default_rng(0).choice([-1, 1], 256), 256)
    assert np.allclose(np.abs(y), 100.0 / 16.0)


@pytest.mark.parametrize("k,b", [(256, 256), (768, 256), (1024, 512), (4096, 4096)])
def test_rotation_is_orthogonal_and_keeps_the_layer_function(k, b):
    rng = np.random.default_rng(k + b)
    s = rng.choice([-1, 1], k)
    Q = O.rotation_matrix(s, b)
    assert np.allclose(Q @ Q.T, np.eye(k), atol=1e-12)
    X = rng.standard_normal((6, k))
    W = rng.standard_normal((5, k))
    Xr, Wr = O.rotate(X, s, b), O.rotate(W, s, b)
    assert np.allclose(Xr @ Wr.T, X @ W.T, atol=1e-10)           # X W^T = X' W'^T
    assert np.allclose(O.rotate(Xr, s, b, inverse=True), X, atol=1e-12)
    assert np.allclose(O.hessian(Xr), Q.T @ O.hessian(X) @ Q, atol=1e-10)
    # a sign flip or a missing 1/sqrt(b) would break these; so would H_b^T != H_b
    assert not np.allclose(O.rotate(X, -s, b), Xr)


def test_gptq_in_the_rotated_basis_measures_the_same_loss():
    # Quantizing W' = W Q against H' = Q^T H Q and rotating the result back
    # (Q_hat = Q_hat' Q^T) gives the same layer loss in the original basis:
    # tr((W - Q_hat) H (W - Q_hat)^T) = tr((W' - Q_hat') H' (W' - Q_hat')^T).
    W, Z, H = _rand_layer(51, 8, 256)
    s = np.random.default_rng(3).choice([-1, 1], 256)
    Hr = O.rotate(O.rotate(H, s, 256).T, s, 256).T  # Q^T H Q
    assert np.allclose(Hr, O.hessian(O.rotate(Z, s, 256)), atol=1e-10)
    res = O.gptq(O.rotate(W, s, 256), Hr, 4, 64, 64, 0.01)
    back = O.rotate(res["qhat"], s, 256, inverse=True)
    loss, _ = O.layer_loss(W, back, H)
    assert abs(loss - res["loss"]) <= 1e-9 * res["loss"]
