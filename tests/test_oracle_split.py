"""Pins of the oracle's fractional widths (b - 1/2 bits a coordinate: the
first d/2 rotated coordinates at b bits, the last d/2 at b - 1): an independent
reader of the record layout, agreement of each half with the integer-width
encoders (pinned on their own), the distortion between the two integer widths,
the decode identity, and unbiasedness over the random matrices."""
import math

import numpy as np
import pytest

import synth
from oracle import oracle as O
from tests.test_oracle_encode import _bits_reader

D = 128


@pytest.fixture(scope="module")
def sp():
    return {b: O.SplitParams(D, b, 0) for b in (2, 3, 4)}


@pytest.mark.parametrize("b", [2, 3, 4])
def test_split_layout_independent_reader(sp, b):
    """The record is the first half's blocks in the b-bit layout, then the
    second half's in the (b-1)-bit layout; np.unpackbits reads both halves."""
    P = sp[b]
    x = synth.gaussian_rows(32, D, seed=1).numpy()
    codes, xn, rn, y, p, idx = O.split_encode(P, x, diagnostics=True)
    h = D // 64  # blocks per half
    assert codes.shape == (32, h * b + h * (b - 1))
    assert codes.shape[1] * 32 == D * (2 * b - 1) // 2  # b - 1/2 bits a coordinate
    i_hi, z_hi = _bits_reader(D // 2, b, np.ascontiguousarray(codes[:, :h * b]))
    i_lo, z_lo = _bits_reader(D // 2, b - 1, np.ascontiguousarray(codes[:, h * b:]))
    np.testing.assert_array_equal(np.concatenate([i_hi, i_lo], 1), idx)
    np.testing.assert_array_equal(np.concatenate([z_hi, z_lo], 1), (p >= 0).astype(np.int64))
    i2, z2 = O.split_unpack(D, b, codes)
    np.testing.assert_array_equal(i2, idx)


@pytest.mark.parametrize("b", [2, 3, 4])
def test_split_halves_agree_with_integer_widths(sp, b):
    """Each half's cells are the cells the integer-width encoder of its width
    gives the same coordinates (same Pi, same grid); the rotation and |x| are
    the same."""
    P = sp[b]
    x = synth.gaussian_rows(24, D, seed=2).numpy()
    _, xn, _, y, _, idx = O.split_encode(P, x, diagnostics=True)
    _, xn_hi, _, y_hi, _, idx_hi = O.encode(O.Params(D, b, 0), x, diagnostics=True)
    _, _, _, _, _, idx_lo = O.encode(O.Params(D, b - 1, 0), x, diagnostics=True)
    np.testing.assert_array_equal(y, y_hi)
    np.testing.assert_array_equal(xn, xn_hi)
    np.testing.assert_array_equal(idx[:, :D // 2], idx_hi[:, :D // 2])
    np.testing.assert_array_equal(idx[:, D // 2:], idx_lo[:, D // 2:])


def test_split_distortion_lies_between_the_integer_widths():
    """E|y - yhat|^2 = E|r|^2 ~ (D_(b-1) + D_(b-2)) / 2 for the two halves'
    Lloyd-Max grids (N(0,1/d) marginal), strictly between the integer widths."""
    d = 256
    x = synth.gaussian_rows(1500, d, seed=5).numpy()
    for b in (3, 4):
        _, _, rn = O.split_encode(O.SplitParams(d, b, 1), x)
        e = float((rn.astype(np.float64) ** 2).mean())
        d_hi = O.lloyd_max(1 << (b - 1))[2]
        d_lo = O.lloyd_max(1 << (b - 2))[2]
        assert abs(e / ((d_hi + d_lo) / 2) - 1) < 0.03, (b, e, d_hi, d_lo)
        assert d_hi < e < d_lo


def test_split_one_and_a_half_bits_low_half_has_no_cells(sp):
    """b = 2 (1.5 bits): the second half keeps only signs, so its residual is y."""
    P = sp[2]
    x = synth.gaussian_rows(16, D, seed=6).numpy()
    _, _, rn, y, _, idx = O.split_encode(P, x, diagnostics=True)
    assert np.all(idx[:, D // 2:] == 0)
    c = P.c_hi.astype(np.float64)
    r = np.concatenate([y[:, :D // 2] - c[idx[:, :D // 2]], y[:, D // 2:]], 1)
    np.testing.assert_allclose(rn, np.linalg.norm(r, axis=1), rtol=1e-6)


@pytest.mark.parametrize("b", [2, 3, 4])
def test_split_score_equals_inner_product_with_decode(sp, b):
    P = sp[b]
    x = synth.gaussian_rows(16, D, seed=7).numpy()
    q = synth.gaussian_rows(5, D, seed=8, norm_range=None).numpy().astype(np.float64)
    codes, xn, rn = O.split_encode(P, x)
    s = O.split_score(P, codes, xn, rn, q)
    xhat = O.split_decode(P, codes, xn, rn)
    np.testing.assert_allclose(s, q @ xhat.T, rtol=0, atol=1e-12 * np.abs(s).max())


def test_split_estimator_unbiased_over_seeds():
    """3.5 bits: over 1000 draws of (Pi, S) the estimate's mean error is within
    3 standard errors of zero (the QJL correction of the residual keeps the
    estimate unbiased whatever the MSE stage)."""
    x = synth.gaussian_rows(1, D, seed=21, norm_range=None).numpy().astype(np.float64)[0]
    q = x + 0.5 * synth.gaussian_rows(1, D, seed=22, norm_range=None).numpy().astype(np.float64)[0]
    true = float(q @ x)
    est = []
    for s in range(1000):
        P = O.SplitParams(D, 4, s)
        codes, xn, rn = O.split_encode(P, x[None, :])
        est.append(O.split_score(P, codes, xn, rn, q[None, :])[0, 0])
    err = np.array(est) - true
    se = err.std(ddof=1) / math.sqrt(err.size)
    assert abs(err.mean()) <= 3 * se, (err.mean(), se)
