"""Host checks of the arithmetic rewrites the tensor-core kernels rely on (not of the
kernels themselves, which the GPU parity tests compare with the oracle):

* the Newton-Schulz step in completed-square form, (c (A + bI/2c)^2 + (a - b^2/4c) I) X,
  equals a X + (b A + c A^2) X;
* the split of fp32 values into bf16 hi + lo keeps them to about 2^-16 relative, and the
  three-term product hi*hi + hi*lo + lo*hi keeps a product to about 2^-15 (the one-CTA
  Newton-Schulz kernel);
* Newton-Schulz with every product's operands cut to tf32 (10-bit mantissa, rounded toward
  zero, as kind::tf32 reads fp32 operands) and fp32 results stays within 1e-2 of the fp64
  iteration, while bf16 operands do not (the batched Newton-Schulz GEMMs for matrices too
  large for one CTA use tf32 for that reason).
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


def _tf32(x):
    """fp32 values with the low 13 mantissa bits cleared (rounded toward zero to tf32)."""
    v = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32) & np.uint32(0xFFFFE000)
    return v.view(np.float32).astype(np.float64)


def _f32(x):
    return np.asarray(x, dtype=np.float32).astype(np.float64)


def _ns_rounded(X, steps, rnd):
    """Newton-Schulz as the batched GEMM path computes it: A = X X^T, P = c A A + b A,
    X <- P X + a X, with each product's operands passed through `rnd` and every result
    stored in fp32."""
    a, b, c = NS
    for _ in range(steps):
        A = _f32(rnd(X) @ rnd(X).T)
        P = _f32(c * (rnd(A) @ rnd(A).T) + b * A)
        X = _f32(rnd(P) @ rnd(X) + a * X)
    return X


def test_tf32_operands_keep_newton_schulz_within_tolerance():
    r = _rng(5)
    for shape in [(64, 128), (136, 256), (256, 512)]:
        X = r.standard_normal(shape)
        X = X / np.linalg.norm(X)
        ref = _ns_plain(X, 5)
        err = lambda Y: np.abs(Y - ref).max() / np.abs(ref).max()
        assert err(_ns_rounded(X, 5, _tf32)) <= 1e-2
        assert err(_ns_rounded(X, 5, bf16_round)) > 2e-2
