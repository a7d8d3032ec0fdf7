"""Property-based checks of the oracle (hypothesis), on small random shapes:
facts that hold at any size and that a slip in indexing or layout breaks."""

import numpy as np
from hypothesis import given, settings, strategies as st

import oracle as O

SETTINGS = settings(max_examples=25, deadline=None)


@SETTINGS
@given(bits=st.sampled_from([2, 3, 4, 8]), r=st.integers(1, 5), runs=st.integers(1, 4),
       seed=st.integers(0, 2 ** 31 - 1))
def test_pack_unpack_round_trip(bits, r, runs, seed):
    k = 32 * runs
    codes = np.random.default_rng(seed).integers(0, 2 ** bits, (r, k))
    qw = O.pack(codes, bits)
    assert qw.shape == (r, k * bits // 32)
    assert np.array_equal(O.unpack(qw, k, bits), codes)


@SETTINGS
@given(m=st.integers(1, 4), n=st.integers(1, 6), groups=st.integers(1, 4),
       seed=st.integers(0, 2 ** 31 - 1))
def test_dequant_matmul_is_linear_in_x(m, n, groups, seed):
    rng = np.random.default_rng(seed)
    G, k = 32, 32 * groups
    codes = rng.integers(0, 16, (n, k))
    qw = O.pack(codes, 4)
    sc = (rng.random((n, groups)) + 0.5).astype(np.float32)
    z = rng.integers(0, 16, (n, groups))
    g = np.arange(k) // G
    X1, X2 = rng.standard_normal((m, k)), rng.standard_normal((m, k))
    Y = lambda X: O.dequant_matmul(X, qw, sc, z, g, 4, k)  # noqa: E731
    assert np.allclose(Y(2.0 * X1 - 3.0 * X2), 2.0 * Y(X1) - 3.0 * Y(X2), atol=1e-9)


@SETTINGS
@given(logb=st.integers(8, 10), nblk=st.integers(1, 3), seed=st.integers(0, 2 ** 31 - 1))
def test_rotation_inverse_and_norms(logb, nblk, seed):
    rng = np.random.default_rng(seed)
    b = 2 ** logb
    k = b * nblk
    s = rng.choice([-1, 1], k)
    x = rng.standard_normal((3, k))
    y = O.rotate(x, s, b)
    assert np.allclose(np.linalg.norm(y, axis=1), np.linalg.norm(x, axis=1))
    assert np.allclose(O.rotate(y, s, b, inverse=True), x, atol=1e-12)
    # block-diagonal: the first block of x alone determines the first block of y
    x2 = x.copy()
    x2[:, b:] = 0.0
    assert np.allclose(O.rotate(x2, s, b)[:, :b], y[:, :b])


@SETTINGS
@given(r=st.integers(1, 6), groups=st.integers(1, 4), G=st.sampled_from([8, 16, 32]),
       bits=st.sampled_from([2, 3, 4]), sym=st.booleans(), seed=st.integers(0, 2 ** 31 - 1))
def test_static_grids_are_rtn_grids(r, groups, G, bits, sym, seed):
    W = np.random.default_rng(seed).normal(0, 0.02, (r, G * groups))
    ss, zz = O.static_grids(W, bits, G, sym=sym)
    ref = O.rtn(W, bits, G, sym=sym)
    assert np.array_equal(ss, ref["scales"]) and np.array_equal(zz, ref["zeros"])
