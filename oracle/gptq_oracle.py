"""fp64 CPU oracle for GPTQ layer-wise quantization (test infrastructure only).

Page tags ([GPTQ-tool], [GPTQ-guide], [GPTQ-breakdown], [What-is-GPTQ]) are
defined in ``oracle/__init__.py``.  Floating point work is fp64 except where a
floating-point value decides an integer (a quantization code or a zero point):
those decisions are taken in fp32, the precision of [GPTQ-tool] *A minimal
Python sketch*, which converts W with ``.float()`` before quantizing.  The CUDA
path takes the same decisions in fp32, so the two sides only disagree where
their (fp64 vs fp32) inputs to a decision straddle a rounding tie.

READINGS (places where the pages are silent, ambiguous or disagree):

R1  Hessian normalisation: ``n`` is the total token count over all chunks.
R2  Dead columns: a column whose Hessian diagonal is exactly 0 gets H_ii := 1
    and W[:, i] := 0, before act-order and damping.
R3  Act-order ties: stable sort of descending diag(H), equal values keep
    ascending column index.
R4  Damping uses the MEAN of diag(H) ([GPTQ-tool] Step 4 and the sketch), not
    the trace of [GPTQ-guide] *Configuration Deep Dive*.
R5  Group parameters are taken at each group start from the current, already
    error-compensated weights (dynamic groups); group_size = -1 means one group
    per row, taken before the first column.
R6  The grid range includes 0 (lo = min(0, min w), hi = max(0, max w)), so the
    zero point is an integer in [0, maxq] ([GPTQ-tool] *Glossary*: the zero
    point is the integer that represents real zero).  ``include_zero=False``
    gives the sketch's literal range.
R7  Rounding is round-half-to-even (``torch.round`` in the sketch).
R8  Error compensation divides by the inverse-Hessian diagonal ([GPTQ-tool]
    Step 5); the [GPTQ-guide] pseudocode omits that division and is not
    followed.
R9  Packing: codes form an LSB-first bit stream along the input dimension of
    each row; code j occupies bits [j*bits, (j+1)*bits) of the row's stream,
    32-bit words little-end first.  Only "eight 4-bit codes per 32-bit word"
    is fixed by [GPTQ-tool] Step 8.
R10 Groups and lazy blocks are aligned: group_size divides block_size or
    block_size divides group_size, so a group never straddles a block end and
    the lazy-blocked sweep equals the column-by-column sweep exactly.
R11 Layer loss = tr((W0 - Qhat) H0 (W0 - Qhat)^T) with the undamped H0, i.e.
    (2/n)·||(W0 - Qhat) X^T||_F^2 ([GPTQ-tool] Step 2 objective and *Reading a
    quantization log*).
R14 Symmetric grid ([GPTQ-tool] *Optional refinements*: "simpler", no fitted
    zero point; nothing else is said): the range is made symmetric about 0,
    [-a, a] with a = max(|min|, |max|) (0 included), scale = max(2a, 1e-8) /
    maxq, and every group's zero point is the grid's middle code
    (maxq + 1) / 2, so codes cover [-(maxq+1)/2, (maxq-1)/2] steps.
R15 Static groups (the ``static_groups`` flag of the AutoGPTQ configuration
    listed by [GPTQ-guide] *Configuration Deep Dive*; its meaning is not
    given): every group's grid is fixed before the sweep, from the
    dead-column-fixed ORIGINAL weights of the group's original columns
    [g G, (g+1) G) (the grid RTN would use); the sweep never refits a grid.
    Under act-order a column keeps its original group, so g_idx[c] = c // G,
    and each column is quantized on that group's grid when its turn comes.
    Because no grid depends on the sweep, groups need not align with the
    lazy blocks (READING R10 is not needed).
R16 Rotation preprocessing ([GPTQ-tool] *Variants and extensions*: weights
    and activations are multiplied by an orthogonal matrix before quantizing
    so that outliers spread out; the matrix is not named): Q = D_s H_b / sqrt(b),
    D_s = diag(s) with random signs s (an input), H_b the block-diagonal
    Sylvester-Hadamard matrix with blocks of b columns (b a power of two
    dividing k).  W' = W Q and X' = X Q keep X W^T = X' W'^T, and the
    Hessian of X' is Q^T H Q.
"""

from __future__ import annotations

import math

import numpy as np
from scipy.linalg import solve_triangular

F64 = np.float64
F32 = np.float32


class NotPositiveDefinite(ValueError):
    """The damped Hessian is not positive definite (Cholesky failed)."""


# ---------------------------------------------------------------------------
# Hessian, dead columns, act-order, damping, inverse factor
# ---------------------------------------------------------------------------

def hessian(x_chunks, n_total=None):
    """H = (2/n) * sum_t x_t x_t^T in fp64.

    [GPTQ-tool] *How it works*, Step 3 (the Hessian of the squared layer error
    w.r.t. one row of W is proportional to X X^T and is shared by every row)
    and *A minimal Python sketch* (``H = 2.0 * X.T @ X / X.shape[0]``), with
    X laid out (n_samples, in_features).  The factor 2 of the sketch is kept;
    [GPTQ-guide] *Computing the Hessian* writes E[x x^T] without it.

    ``x_chunks`` is one (n, k) array or an iterable of (n_c, k) arrays of any
    float dtype; each is converted exactly to fp64.  READING R1: ``n`` is the
    total token count over all chunks unless ``n_total`` is given.
    """
    if isinstance(x_chunks, np.ndarray) or hasattr(x_chunks, "numpy"):
        x_chunks = [x_chunks]
    H = None
    n = 0
    for X in x_chunks:
        Xd = np.asarray(X, dtype=F64)
        G = Xd.T @ Xd
        H = G if H is None else H + G
        n += Xd.shape[0]
    if n_total is None:
        n_total = n
    return H * (2.0 / n_total)


def fix_dead_columns(H, W):
    """READING R2.  [GPTQ-tool] Step 4 notes that features which are always
    zero make H singular, without giving a rule.  A column i with H_ii == 0
    (exactly) gets H_ii := 1 and W[:, i] := 0; such a column never reaches the
    layer output, so its code is loss-neutral and W = 0 makes it the zero
    point.  Returns (H', W', dead mask)."""
    H = np.array(H, dtype=F64, copy=True)
    W = np.array(W, dtype=F64, copy=True)
    dead = np.diag(H) == 0.0
    idx = np.flatnonzero(dead)
    H[idx, idx] = 1.0
    W[:, idx] = 0.0
    return H, W, dead


def act_order_perm(H, force_perm=None, tau_rel=1e-5):
    """[GPTQ-tool] *Optional refinements*, Act-order: process columns in
    descending order of the Hessian diagonal.  READING R3: stable, so equal
    diagonal values keep ascending column index.

    The order is an integer result decided by floating-point values: two
    diagonals that agree within the Hessian's tolerance may come out in
    either order from an fp32 Hessian.  ``force_perm`` (a candidate order)
    is accepted when it is a permutation whose every out-of-order pair lies
    within ``tau_rel`` (relative) of a tie, i.e. d[perm[j]] >=
    (1 - tau_rel) * max_{m > j} d[perm[m]] for all j; otherwise ValueError.
    """
    d = np.diag(np.asarray(H, dtype=F64))
    if force_perm is None:
        return np.argsort(-d, kind="stable").astype(np.int64)
    p = np.asarray(force_perm, dtype=np.int64)
    k = d.shape[0]
    if p.shape != (k,) or not np.array_equal(np.sort(p), np.arange(k)):
        raise ValueError("candidate order is not a permutation")
    dp = d[p]
    suffix_max = np.maximum.accumulate(dp[::-1])[::-1]
    later = np.append(suffix_max[1:], -np.inf)
    bad = dp < (1.0 - tau_rel) * later
    if bad.any():
        j = int(np.flatnonzero(bad)[0])
        raise ValueError(f"candidate order breaks descending diag at position {j}")
    return p


def damp(H, percdamp):
    """[GPTQ-tool] Step 4 and the sketch: H + percdamp * mean(diag H) * I.
    READING R4 (mean, not the trace of [GPTQ-guide])."""
    H = np.asarray(H, dtype=F64)
    lam = percdamp * np.mean(np.diag(H))
    return H + lam * np.eye(H.shape[0])


def hinv_upper_factor(H):
    """Upper Cholesky factor U of H^-1 (U^T U = H^-1).

    [GPTQ-tool] Step 6 (Cholesky factor of the inverse Hessian, computed once;
    its rows hold the numbers each column step needs) and the sketch, which
    forms it as cholesky(cholesky_inverse(cholesky(H)), upper=True).  Written
    out: L = chol(H) lower; H^-1 = (L L^T)^-1 = L^-T L^-1; U = upper chol of
    H^-1.  Raises NotPositiveDefinite when either factorisation fails.
    """
    H = np.asarray(H, dtype=F64)
    k = H.shape[0]
    try:
        L = np.linalg.cholesky(H)
    except np.linalg.LinAlgError as e:
        raise NotPositiveDefinite(str(e)) from None
    Linv = solve_triangular(L, np.eye(k), lower=True)
    Hinv = Linv.T @ Linv
    try:
        Lh = np.linalg.cholesky(Hinv)
    except np.linalg.LinAlgError as e:
        raise NotPositiveDefinite(str(e)) from None
    return Lh.T.copy()


# ---------------------------------------------------------------------------
# Quantization grid
# ---------------------------------------------------------------------------

def grid_params(wg, maxq, include_zero=True, decide_dtype=F32, sym=False):
    """Min/max grid for each row of ``wg`` (r, g).

    [GPTQ-tool] sketch: scale = clamp(max - min, min=1e-8) / maxq and
    zero = round(-min / scale); *Optional refinements* (asymmetric grids use a
    zero point); *Glossary* (zero point = the integer that represents real
    zero).  READING R6: the range includes 0 unless ``include_zero`` is False.
    Computed in ``decide_dtype`` (fp32, as the sketch) because the zero point
    is an integer decision.  Returns (scale, zero) as arrays of decide_dtype.

    ``sym`` ([GPTQ-tool] *Optional refinements*: symmetric grids, no fitted
    zero point; READING R14): the range is made symmetric, [-a, a] with
    a = max(|lo|, |hi|), so scale = max(2a, 1e-8) / maxq, and the zero point is
    the grid's middle code (maxq + 1) / 2 for every group.
    """
    dt = decide_dtype
    w = np.asarray(wg, dtype=F64).astype(dt)
    lo = w.min(axis=1)
    hi = w.max(axis=1)
    if include_zero or sym:
        lo = np.minimum(lo, dt(0))
        hi = np.maximum(hi, dt(0))
    if sym:
        a = np.maximum(-lo, hi)
        scale = np.maximum(a + a, dt(1e-8)) / dt(maxq)
        zero = np.full(scale.shape, (maxq + 1) // 2, dtype=dt)
        return scale.astype(dt), zero
    scale = np.maximum(hi - lo, dt(1e-8)) / dt(maxq)
    zero = np.rint(-lo / scale)
    return scale.astype(dt), zero.astype(dt)


def quantize_codes(w, scale, zero, maxq, decide_dtype=F32):
    """[GPTQ-tool] sketch ``quantize_to_grid``: code = clamp(round(w / scale)
    + zero, 0, maxq), decided in fp32 (READING R7: half-to-even).  Also the
    quantization equation of [GPTQ-guide] (round(value / scale)) when
    zero = 0 and no clamp is wanted (pass maxq=None)."""
    dt = decide_dtype
    x = np.asarray(w, dtype=F64).astype(dt) / np.asarray(scale, dtype=dt)
    c = np.rint(x) + np.asarray(zero, dtype=dt)
    if maxq is not None:
        c = np.clip(c, 0, maxq)
    return c.astype(F64)


def _dequant_f64(codes, scale, zero):
    """scale * (code - zero) in fp64 (exact: fp32 scale times a small int)."""
    return np.asarray(scale, dtype=F64) * (np.asarray(codes, dtype=F64) - np.asarray(zero, dtype=F64))


def group_count(k, group_size):
    """Number of groups along k; group_size = -1 means one group per row."""
    G = k if group_size == -1 else group_size
    return int(math.ceil(k / G)) if k > 0 else 0


def _check_groups(k, group_size, block_size=None):
    if group_size != -1 and group_size <= 0:
        raise ValueError("group_size must be -1 or positive")
    G = k if group_size == -1 else group_size
    if block_size is not None and group_size != -1:
        if not (block_size % G == 0 or G % block_size == 0):
            raise ValueError("READING R10: group_size and block_size must divide one another")
    return max(G, 1)


def static_grids(W, bits, group_size, include_zero=True, decide_dtype=F32, sym=False):
    """READING R15: the grid of every group g, fitted once to the original
    columns [g G, (g+1) G) of ``W`` (r, k), before any error compensation.
    Returns (scales, zeros), each (r, ngroups) in decide_dtype."""
    W = np.asarray(W, dtype=F64)
    r, k = W.shape
    maxq = 2 ** bits - 1
    G = _check_groups(k, group_size)
    ng = group_count(k, group_size)
    scales = np.zeros((r, ng), dtype=decide_dtype)
    zeros = np.zeros((r, ng), dtype=decide_dtype)
    for g in range(ng):
        scales[:, g], zeros[:, g] = grid_params(W[:, g * G:min((g + 1) * G, k)], maxq,
                                                include_zero, decide_dtype, sym)
    return scales, zeros


# ---------------------------------------------------------------------------
# Column sweeps
# ---------------------------------------------------------------------------

def sweep_unblocked(W, U, bits, group_size, include_zero=True, decide_dtype=F32,
                    fixed_grid=None, sym=False, static=None):
    """Column-by-column GPTQ sweep (no lazy batching).

    [GPTQ-tool] *How it works*, Step 5 and the sketch's loop: for each column
    i in order, quantize it, err = (w - q) / U[i, i], and subtract
    err * U[i, i+1:] from every later column.  Generalised by groups
    ([What-is-GPTQ] Step 3; READING R5: parameters from the current weights at
    each group start; group_size = -1: one group per row, taken at column 0).

    ``W`` (r, k) is already dead-fixed and in sweep order; ``U`` is the upper
    factor with U^T U = H^-1 in the same order.  Returns a dict with codes
    (r, k), scales / zeros (r, ngroups), qhat (r, k) dequantized weights,
    err (r, k) scaled errors and w_at (r, k), each column's value at the
    moment it is quantized, all in sweep order.  ``fixed_grid`` = (scale,
    zero) replaces the min/max grid by a fixed one (the worked examples of the
    pages use a fixed step).  ``static`` = (scales, zeros, gcol) gives every
    column a grid fixed before the sweep (READING R15): column i uses group
    gcol[i] of the (r, ngroups) tables, which are returned unchanged.
    """
    W = np.array(W, dtype=F64, copy=True)
    U = np.asarray(U, dtype=F64)
    r, k = W.shape
    maxq = 2 ** bits - 1
    G = _check_groups(k, group_size)
    ng = group_count(k, group_size)
    codes = np.zeros((r, k))
    qhat = np.zeros((r, k))
    errs = np.zeros((r, k))
    w_at = np.zeros((r, k))
    scales = np.zeros((r, ng), dtype=decide_dtype)
    zeros = np.zeros((r, ng), dtype=decide_dtype)
    s = z = None
    for i in range(k):
        if static is not None:
            s, z = _static_grid(static, i)
        elif i % G == 0:
            s, z = _group_grid(W[:, i:i + G], maxq, include_zero, decide_dtype, fixed_grid, r, sym)
            scales[:, i // G] = s
            zeros[:, i // G] = z
        w = W[:, i].copy()
        c = quantize_codes(w, s, z, maxq, decide_dtype)
        q = _dequant_f64(c, s, z)
        err = (w - q) / U[i, i]
        W[:, i + 1:] -= np.outer(err, U[i, i + 1:])
        codes[:, i] = c
        qhat[:, i] = q
        errs[:, i] = err
        w_at[:, i] = w
    if static is not None:
        scales, zeros = static[0], static[1]
    return dict(codes=codes, scales=scales, zeros=zeros, qhat=qhat, err=errs, w_at=w_at)


def _static_grid(static, i):
    """Column i's fixed grid (READING R15)."""
    sc, zc, gcol = static
    return sc[:, gcol[i]], zc[:, gcol[i]]


def _group_grid(wg, maxq, include_zero, dt, fixed_grid, r, sym=False):
    if fixed_grid is None:
        return grid_params(wg, maxq, include_zero, dt, sym)
    s, z = fixed_grid
    return np.full(r, s, dtype=dt), np.full(r, z, dtype=dt)


def sweep_blocked(W, U, bits, group_size, block_size, include_zero=True,
                  decide_dtype=F32, force_codes=None, force_zeros=None, tau=None,
                  fixed_grid=None, sym=False, static=None):
    """Lazy-batch GPTQ sweep.

    [GPTQ-tool] Step 7 (blocks of ``block_size`` columns: updates inside the
    block are applied at once, updates to later columns are collected and
    applied once at the block end) and [GPTQ-breakdown] *How It Works* (lazy
    batching turns the trailing updates into matrix multiplications).  Per
    block [s, e): the column loop of ``sweep_unblocked`` restricted to the
    block, err collected in Err (r, e-s); then W[:, e:] -= Err @ U[s:e, e:].
    By READING R10 this equals ``sweep_unblocked`` up to fp64 rounding.

    ``force_codes`` / ``force_zeros`` (sweep order) turn this into the
    tie-aware replay of ``sweep_replay``; leave them None otherwise.
    ``fixed_grid`` and ``static`` as in ``sweep_unblocked``; with ``static``
    the groups need not align with the blocks (READING R15).
    """
    W = np.array(W, dtype=F64, copy=True)
    U = np.asarray(U, dtype=F64)
    r, k = W.shape
    maxq = 2 ** bits - 1
    B = int(block_size)
    if B <= 0:
        raise ValueError("block_size must be positive")
    G = _check_groups(k, group_size, None if static is not None else B)
    ng = group_count(k, group_size)
    codes = np.zeros((r, k))
    qhat = np.zeros((r, k))
    errs = np.zeros((r, k))
    w_at = np.zeros((r, k))
    scales = np.zeros((r, ng), dtype=decide_dtype)
    zeros = np.zeros((r, ng), dtype=decide_dtype)
    n_forced = 0
    s = z = None
    for s0 in range(0, k, B):
        e0 = min(s0 + B, k)
        Err = np.zeros((r, e0 - s0))
        for i in range(s0, e0):
            if static is not None:
                s, z = _static_grid(static, i)
            elif i % G == 0:
                s, z = _group_grid(W[:, i:i + G], maxq, include_zero, decide_dtype, fixed_grid, r,
                                   sym)
                if force_zeros is not None and not sym:  # a symmetric grid's zero is fixed
                    z, nf = _force_ties(-np.minimum(W[:, i:i + G].astype(decide_dtype).min(axis=1), 0)
                                        if include_zero else
                                        -W[:, i:i + G].astype(decide_dtype).min(axis=1),
                                        s, z, np.asarray(force_zeros[:, i // G]), tau, decide_dtype)
                    n_forced += nf
                scales[:, i // G] = s
                zeros[:, i // G] = z
            w = W[:, i].copy()
            c = quantize_codes(w, s, z, maxq, decide_dtype)
            if force_codes is not None:
                c, nf = _force_code_ties(w, s, z, c, np.asarray(force_codes[:, i], dtype=F64),
                                         maxq, tau, decide_dtype)
                n_forced += nf
            q = _dequant_f64(c, s, z)
            err = (w - q) / U[i, i]
            W[:, i + 1:e0] -= np.outer(err, U[i, i + 1:e0])
            Err[:, i - s0] = err
            codes[:, i] = c
            qhat[:, i] = q
            errs[:, i] = err
            w_at[:, i] = w
        if e0 < k:
            W[:, e0:] -= Err @ U[s0:e0, e0:]
    if static is not None:
        scales, zeros = static[0], static[1]
    return dict(codes=codes, scales=scales, zeros=zeros, qhat=qhat, err=errs, w_at=w_at,
                n_forced=n_forced)


def _near_tie(x, tau):
    return np.abs((x - np.floor(x)) - 0.5) < tau


def _force_code_ties(w, s, z, c, forced, maxq, tau, dt):
    """Take ``forced`` where it differs by exactly 1 from ``c`` and w/s sits
    within ``tau`` (in grid steps) of a rounding tie."""
    x = np.asarray(w, dtype=F64).astype(dt) / s
    take = _near_tie(x.astype(F64), tau) & (np.abs(forced - c) == 1)
    c = np.where(take, forced, c)
    return c, int(take.sum())


def _force_ties(neg_lo, s, z, forced, tau, dt):
    x = (np.asarray(neg_lo, dtype=dt) / s).astype(F64)
    take = _near_tie(x, tau) & (np.abs(forced.astype(F64) - z.astype(F64)) == 1)
    z = np.where(take, forced.astype(dt), z).astype(dt)
    return z, int(take.sum())


def sweep_replay(W, U, bits, group_size, block_size, force_codes, force_zeros,
                 tau=1e-3, include_zero=True, decide_dtype=F32, sym=False, static=None):
    """Tie-aware replay: the lazy-blocked sweep in fp64, except that wherever
    a candidate result (``force_codes``, ``force_zeros``, sweep order) differs
    from the oracle's decision by exactly one step AND the oracle's value
    (w/s for a code, -lo/s for a zero point) lies within ``tau`` grid steps of
    a rounding tie, the candidate's decision is taken.  Both decisions are
    valid there (the fp32 and fp64 inputs straddle the tie); every other
    decision must then agree exactly.  Returns the same dict as
    ``sweep_blocked`` with ``n_forced``.  Static grids (``static``) are
    fixed before the sweep from the same fp32 inputs, so only codes are
    replayed there."""
    return sweep_blocked(W, U, bits, group_size, block_size, include_zero,
                         decide_dtype, force_codes, force_zeros, tau, sym=sym, static=static)


def sweep_obs(W, Hd, bits, group_size, include_zero=True, decide_dtype=F32,
              fixed_grid=None, sym=False, static=None):
    """Column sweep with an explicit inverse Hessian and the Optimal Brain
    Surgeon downdate.

    [GPTQ-guide] *Detailed Algorithm* (compensate with H_inv x error, then
    remove the quantized weight from the inverse Hessian) and [GPTQ-tool]
    *Where it came from* / [GPTQ-breakdown] (OBS lineage).  With READING R8
    (divide by the diagonal, [GPTQ-tool] Step 5): for the first remaining
    column i, d = (w_i - q_i) / Hinv[i, i]; W[:, j] -= d * Hinv[i, j] for the
    remaining j; then Hinv -= Hinv[:, i] Hinv[i, :] / Hinv[i, i].  [GPTQ-tool]
    Step 6 says the rows of the Cholesky factor hold exactly these numbers, so
    this equals ``sweep_unblocked`` up to rounding (a pin, not a product path).
    ``Hd`` is the damped Hessian in sweep order; ``fixed_grid`` and
    ``static`` as in ``sweep_unblocked``.
    """
    W = np.array(W, dtype=F64, copy=True)
    r, k = W.shape
    maxq = 2 ** bits - 1
    G = _check_groups(k, group_size)
    ng = group_count(k, group_size)
    Hinv = np.linalg.inv(np.asarray(Hd, dtype=F64))
    codes = np.zeros((r, k))
    qhat = np.zeros((r, k))
    scales = np.zeros((r, ng), dtype=decide_dtype)
    zeros = np.zeros((r, ng), dtype=decide_dtype)
    s = z = None
    for i in range(k):
        if static is not None:
            s, z = _static_grid(static, i)
        elif i % G == 0:
            s, z = _group_grid(W[:, i:i + G], maxq, include_zero, decide_dtype, fixed_grid, r, sym)
            scales[:, i // G] = s
            zeros[:, i // G] = z
        w = W[:, i].copy()
        c = quantize_codes(w, s, z, maxq, decide_dtype)
        q = _dequant_f64(c, s, z)
        d = (w - q) / Hinv[i, i]
        W[:, i + 1:] -= np.outer(d, Hinv[i, i + 1:])
        Hinv = Hinv - np.outer(Hinv[:, i], Hinv[i, :]) / Hinv[i, i]
        codes[:, i] = c
        qhat[:, i] = q
    if static is not None:
        scales, zeros = static[0], static[1]
    return dict(codes=codes, scales=scales, zeros=zeros, qhat=qhat)


def rtn(W, bits, group_size, include_zero=True, decide_dtype=F32, sym=False):
    """Round-to-nearest baseline ([GPTQ-breakdown] *The Problem*; [GPTQ-tool]
    *A worked example*, "plain rounding"; *Glossary*): every weight is rounded
    on its group's grid independently, with no error compensation.  Group
    parameters come from the original weights."""
    W = np.asarray(W, dtype=F64)
    r, k = W.shape
    maxq = 2 ** bits - 1
    G = _check_groups(k, group_size)
    ng = group_count(k, group_size)
    codes = np.zeros((r, k))
    qhat = np.zeros((r, k))
    scales = np.zeros((r, ng), dtype=decide_dtype)
    zeros = np.zeros((r, ng), dtype=decide_dtype)
    for g in range(ng):
        a, b = g * G, min((g + 1) * G, k)
        s, z = grid_params(W[:, a:b], maxq, include_zero, decide_dtype, sym)
        c = quantize_codes(W[:, a:b], s[:, None], z[:, None], maxq, decide_dtype)
        codes[:, a:b] = c
        qhat[:, a:b] = _dequant_f64(c, s[:, None], z[:, None])
        scales[:, g] = s
        zeros[:, g] = z
    return dict(codes=codes, scales=scales, zeros=zeros, qhat=qhat)


def layer_loss(W0, qhat, H0):
    """READING R11: per-row and total tr((W0 - Qhat) H0 (W0 - Qhat)^T).
    [GPTQ-tool] Step 2 (minimise the squared difference between W X and Q X)
    and *Reading a quantization log* (the squared output error per layer).
    With H0 = (2/n) X^T X this is (2/n) * ||(W0 - Qhat) X^T||_F^2."""
    D = np.asarray(W0, dtype=F64) - np.asarray(qhat, dtype=F64)
    per_row = np.einsum("ij,jk,ik->i", D, np.asarray(H0, dtype=F64), D)
    return float(per_row.sum()), per_row


# ---------------------------------------------------------------------------
# Whole layer
# ---------------------------------------------------------------------------

def gptq(W, H, bits=4, group_size=128, block_size=128, percdamp=0.01,
         act_order=False, include_zero=True, decide_dtype=F32, blocked=True, sym=False,
         force_codes=None, force_zeros=None, tau=1e-3, force_perm=None, tau_perm=1e-5,
         static_groups=False):
    """GPTQ for one linear layer, given W (r, k) and the undamped Hessian H.

    Order of steps ([GPTQ-tool] *How it works* Steps 3-8): dead columns
    (READING R2), act-order permutation ([GPTQ-tool] *Optional refinements*),
    damping (Step 4), inverse factor (Step 6), column sweep (Steps 5 and 7),
    then outputs in the original column order: codes, scales and zeros per
    (row, group in sweep order), g_idx (group of each original column) and the
    layer loss against the undamped H (READING R11).

    ``force_codes`` / ``force_zeros`` (original column order) request the
    tie-aware replay (``sweep_replay``); ``force_perm`` a candidate act-order
    permutation, accepted only where it is a valid order within ``tau_perm``
    (see ``act_order_perm``).

    ``static_groups`` (READING R15): grids fixed before the sweep from the
    dead-column-fixed weights in their original column order; scales / zeros
    are then per (row, original group) and g_idx[c] = c // G.
    """
    W0 = np.asarray(W, dtype=F64)
    H0 = np.asarray(H, dtype=F64)
    r, k = W0.shape
    Hf, Wf, dead = fix_dead_columns(H0, W0)
    if act_order:
        perm = act_order_perm(Hf, force_perm, tau_perm)
    else:
        perm = np.arange(k, dtype=np.int64)
    Wp = Wf[:, perm]
    Hp = Hf[np.ix_(perm, perm)]
    Hd = damp(Hp, percdamp)
    U = hinv_upper_factor(Hd)
    G = k if group_size == -1 else group_size
    static = None
    if static_groups:
        ss, zz = static_grids(Wf, bits, group_size, include_zero, decide_dtype, sym)
        static = (ss, zz, perm // G)
    if force_codes is not None:
        fc = np.asarray(force_codes)[:, perm]
        res = sweep_replay(Wp, U, bits, group_size, block_size, fc,
                           None if static_groups else force_zeros,
                           tau, include_zero, decide_dtype, sym, static)
    elif blocked:
        res = sweep_blocked(Wp, U, bits, group_size, block_size, include_zero, decide_dtype,
                            sym=sym, static=static)
    else:
        res = sweep_unblocked(Wp, U, bits, group_size, include_zero, decide_dtype, sym=sym,
                              static=static)
    codes = np.zeros((r, k))
    qhat = np.zeros((r, k))
    codes[:, perm] = res["codes"]
    qhat[:, perm] = res["qhat"]
    if static_groups:
        g_idx = np.arange(k, dtype=np.int64) // G
    else:
        g_idx = np.zeros(k, dtype=np.int64)
        g_idx[perm] = np.arange(k) // G
    loss, per_row = layer_loss(W0, qhat, H0)
    return dict(codes=codes.astype(np.int64), scales=res["scales"], zeros=res["zeros"],
                g_idx=g_idx, perm=perm, dead=dead, U=U, qhat=qhat, loss=loss,
                loss_rows=per_row, n_forced=res.get("n_forced", 0), Hd=Hd)


# ---------------------------------------------------------------------------
# Packing and dequantization
# ---------------------------------------------------------------------------

def pack(codes, bits):
    """READING R9 ([GPTQ-tool] Step 8: eight 4-bit codes per 32-bit word, the
    only layout the pages fix): each row's codes form an LSB-first bit stream;
    bit b of code j is stream bit j*bits + b; stream bit m is bit (m mod 32) of
    word m // 32.  Needs k*bits % 32 == 0.  Returns int32 (r, k*bits/32)."""
    codes = np.asarray(codes, dtype=np.int64)
    r, k = codes.shape
    if (k * bits) % 32:
        raise ValueError("k*bits must be a multiple of 32")
    if codes.min(initial=0) < 0 or codes.max(initial=0) >= (1 << bits):
        raise ValueError("code out of range")
    stream = np.zeros((r, k * bits), dtype=np.uint64)
    for b in range(bits):
        stream[:, b::bits] = (codes >> b) & 1
    words = np.zeros((r, k * bits // 32), dtype=np.uint64)
    for b in range(32):
        words |= stream[:, b::32] << np.uint64(b)
    return words.astype(np.uint32).view(np.int32)


def unpack(qweight, k, bits):
    """Inverse of ``pack``: reads code j back from stream bits
    [j*bits, (j+1)*bits)."""
    words = np.asarray(qweight).view(np.uint32).astype(np.uint64)
    r = words.shape[0]
    stream = np.zeros((r, words.shape[1] * 32), dtype=np.uint64)
    for b in range(32):
        stream[:, b::32] = (words >> np.uint64(b)) & np.uint64(1)
    codes = np.zeros((r, k), dtype=np.int64)
    for b in range(bits):
        codes |= (stream[:, b:k * bits:bits].astype(np.int64) << b)
    return codes


def dequant(codes, scales, zeros, g_idx, out_dtype=F32):
    """w = scale[g] * (code - zero[g]) with g = g_idx[column] ([GPTQ-tool]
    sketch dequantization and *Glossary*; [What-is-GPTQ] Step 3, each group
    expanded just in time).  The product is taken in fp32 and rounded to
    ``out_dtype``."""
    codes = np.asarray(codes, dtype=np.int64)
    g_idx = np.asarray(g_idx, dtype=np.int64)
    s = np.asarray(scales, dtype=F32)[:, g_idx]
    z = np.asarray(zeros, dtype=np.int64)[:, g_idx]
    v = s * (codes - z).astype(F32)
    return v.astype(out_dtype)


def rotation_matrix(signs, block):
    """READING R16: Q = diag(signs) * blockdiag(H_b, ..., H_b) / sqrt(b), with
    H_b the Sylvester Hadamard matrix of order b (scipy.linalg.hadamard).
    Orthogonal: Q Q^T = I."""
    from scipy.linalg import block_diag, hadamard
    s = np.where(np.asarray(signs) < 0, -1.0, 1.0)
    k = s.shape[0]
    b = int(block)
    if b <= 0 or b & (b - 1) or k % b:
        raise ValueError("block must be a power of two dividing k")
    Hb = hadamard(b).astype(F64) / math.sqrt(b)
    return s[:, None] * block_diag(*([Hb] * (k // b)))


def rotate(x, signs, block, inverse=False):
    """[GPTQ-tool] *Variants and extensions*, rotation-based preprocessing
    (READING R16): each row x of ``x`` becomes x Q (``inverse``: x Q^T, which
    undoes it).  fp64."""
    Q = rotation_matrix(signs, block)
    x = np.asarray(x, dtype=F64)
    return x @ (Q.T if inverse else Q)


def dequant_matmul(X, qweight, scales, zeros, g_idx, bits, k):
    """The inference product of a quantized layer: Y = X W_hat^T with
    W_hat[j, c] = scale[j, g_c] * (code[j, c] - zero[j, g_c]), the codes read
    from the packed words ([GPTQ-tool] *What the output looks like*: a GPU
    kernel reads the packed data and dequantizes inside the matrix multiply;
    Step 8: the fused kernel unpacks, scales and multiplies; [What-is-GPTQ]
    *How it works*: each group is expanded just in time for the multiply).
    X (m, k), qweight int32 (n, k*bits/32), scales / zeros (n, ngroups),
    g_idx (k).  Exact fp64 arithmetic on the exact input values (an fp32
    scale times a small integer is exact in fp64), then one fp64 matrix
    product.  Returns (m, n) fp64."""
    codes = unpack(qweight, k, bits)
    g_idx = np.asarray(g_idx, dtype=np.int64)
    s = np.asarray(scales, dtype=F32).astype(F64)[:, g_idx]
    z = np.asarray(zeros, dtype=np.int64)[:, g_idx]
    W_hat = s * (codes - z).astype(F64)
    return np.asarray(X, dtype=F64) @ W_hat.T


def storage_bits_per_weight(bits, group_size, k, scale_bits=16, zero_bits=None):
    """[GPTQ-tool] *Memory arithmetic*: code bits plus one scale and one zero
    point per group, spread over the group's weights."""
    zb = bits if zero_bits is None else zero_bits
    ng = group_count(k, group_size)
    return bits + ng * (scale_bits + zb) / k
