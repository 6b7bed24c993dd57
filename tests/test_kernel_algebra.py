"""Host checks of the arithmetic rewrites the tensor-core kernels rely on (not of the
kernels themselves, which the GPU parity tests compare with the oracle):

* the Newton-Schulz step in completed-square form, (c (A + bI/2c)^2 + (a - b^2/4c) I) X,
  equals a X + (b A + c A^2) X;
* the split of fp32 values into bf16 hi + lo keeps them to about 2^-16 relative, and the
  three-term product hi*hi + hi*lo + lo*hi keeps a product to about 2^-15;
* a split-precision operand stored once as [hi | lo] (K padded to a multiple of 64) and
  read third by third through the K-coordinate remap gives the tripled operands
  [hi hi lo] and [hi lo hi] exactly, so the K-tripled product is hi*hi + hi*lo + lo*hi.
"""
import numpy as np

from ttt_inputs import bf16_round

NS = (3.4445, -4.7750, 2.0315)
BK = 64


def _rng(seed):
    return np.random.Generator(np.random.PCG64(seed))


def _ns_plain(X, steps):
    a, b, c = NS
    for _ in range(steps):
        A = X @ X.T
        X = a * X + (b * A + c * A @ A) @ X
    return X


def _ns_completed_square(X, steps):
    a, b, c = NS
    beta, g = b / (2 * c), a - b * b / (4 * c)
    eye = np.eye(X.shape[0])
    for _ in range(steps):
        Abar = X @ X.T + beta * eye
        X = (c * Abar @ Abar.T + g * eye) @ X
    return X


def test_completed_square_newton_schulz_equals_the_plain_iteration():
    for seed, (r, c) in enumerate([(8, 8), (40, 200), (128, 256), (3, 17)]):
        U = _rng(seed).standard_normal((r, c))
        X = U / (np.linalg.norm(U) + 1e-7)
        ref = _ns_plain(X, 5)
        got = _ns_completed_square(X, 5)
        assert np.abs(got - ref).max() <= 1e-12 * np.abs(ref).max()


def test_completed_square_keeps_zero_padding_zero():
    # rows / columns of zeros (the kernel's padding to 128 x 256) stay zero although the
    # diagonal shift touches the padded diagonal
    X = np.zeros((16, 32))
    X[:10, :21] = _rng(7).standard_normal((10, 21)) * 0.05
    got = _ns_completed_square(X, 5)
    assert not got[10:].any() and not got[:, 21:].any()
    ref = _ns_plain(X[:10, :21], 5)
    assert np.abs(got[:10, :21] - ref).max() <= 1e-12 * np.abs(ref).max()


def _split(x32):
    hi = bf16_round(x32)
    lo = bf16_round((x32 - hi).astype(np.float32))
    return hi.astype(np.float64), lo.astype(np.float64)


def test_hi_lo_split_error_bound():
    r = _rng(11)
    x = (r.standard_normal(200000) * np.exp(r.uniform(-20, 20, 200000))).astype(np.float32)
    hi, lo = _split(x)
    xd = x.astype(np.float64)
    assert np.all(np.abs(xd - (hi + lo)) <= 2.0 ** -16 * np.abs(xd))
    y = (r.standard_normal(200000)).astype(np.float32)
    yh, yl = _split(y)
    three = hi * yh + hi * yl + lo * yh
    assert np.all(np.abs(three - xd * y) <= 2.0 ** -15 * np.abs(xd * y) + 1e-300)


def _kcoord(kb, hilo, k0):
    """K coordinate of k-block kb in a [hi | lo] buffer (k0-wide thirds)."""
    k = kb * BK
    third, kk = divmod(k, k0)
    lo = third == 2 if hilo == 1 else third == 1
    return kk + (k0 if lo else 0)


def test_split_operand_thirds_through_the_k_remap():
    r = _rng(3)
    for rows, K in [(136, 256), (64, 136), (5, 64)]:
        k0 = (K + BK - 1) // BK * BK
        x = r.standard_normal((rows, K)).astype(np.float32)
        hi, lo = _split(x)
        buf = np.zeros((rows, 2 * k0))
        buf[:, :K] = hi
        buf[:, k0:k0 + K] = lo
        pad = lambda m: np.pad(m, ((0, 0), (0, k0 - K)))
        want = {1: np.hstack([pad(hi), pad(hi), pad(lo)]),
                2: np.hstack([pad(hi), pad(lo), pad(hi)])}
        for hilo in (1, 2):
            got = np.hstack([buf[:, _kcoord(kb, hilo, k0):_kcoord(kb, hilo, k0) + BK]
                             for kb in range(3 * k0 // BK)])
            assert np.array_equal(got, want[hilo])
        # the K-tripled product of the two remapped operands is hi hi^T + hi lo^T + lo hi^T
        A = np.hstack([buf[:, _kcoord(kb, 1, k0):_kcoord(kb, 1, k0) + BK]
                       for kb in range(3 * k0 // BK)])
        B = np.hstack([buf[:, _kcoord(kb, 2, k0):_kcoord(kb, 2, k0) + BK]
                       for kb in range(3 * k0 // BK)])
        assert np.allclose(A @ B.T, hi @ hi.T + hi @ lo.T + lo @ hi.T, rtol=0, atol=1e-9)
