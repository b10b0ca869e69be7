"""Pins of the oracle's MSE-only quantizer (all b bits on the Lloyd-Max index,
no QJL; quant_prune_distill #674, "MSE-optimised TurboQuant"), stored as a
code.  Each test checks the oracle against something other than itself:
the published Lloyd-Max table, the nearest-centroid definition computed
independently in numpy, the independent layout reader, the oracle's
separately written estimate routine, and the decode identity."""
import numpy as np
import pytest

import synth
from oracle import oracle as O
from tests import parity as PT
from tests.test_oracle_params import _read_lloyd_max

D = 128


def _full_index(d, b, codes):
    idx, z = PT.read_layout(d, b, codes)
    return z if b == 1 else idx | (z << (b - 1))


@pytest.mark.parametrize("b", [1, 2, 3, 4])
def test_mse_tables_are_max_1960_at_b_bits(b):
    table = _read_lloyd_max()
    P = O.MseParams(D, b, 0)
    L = 1 << b
    assert P.c.size == L and P.beta.size == L - 1
    pos = np.sort(P.c[P.c > 0].astype(np.float64)) * np.sqrt(D)
    np.testing.assert_allclose(pos, table[L][0], rtol=1e-3)


@pytest.mark.parametrize("b", [1, 2, 3, 4])
def test_mse_encode_is_nearest_centroid(b):
    """Cell = nearest b-bit centroid of y = Pi x / |x| (numpy, fp64 from the
    fp32 Pi), read back through the independent layout reader."""
    P = O.MseParams(D, b, 3)
    x = synth.gaussian_rows(400, D, seed=21).numpy().astype(np.float64)
    codes, xn, rn, y, idx = O.mse_encode(P, x, diagnostics=True)
    y_np = (x @ P.Pi.astype(np.float64).T) / np.linalg.norm(x, axis=1, keepdims=True)
    np.testing.assert_allclose(y, y_np, rtol=0, atol=1e-12)
    c = P.c.astype(np.float64)
    near = np.argmin(np.abs(y_np[:, :, None] - c[None, None, :]), axis=2)
    mid = 0.5 * (c[1:] + c[:-1])
    tie = np.min(np.abs(y_np[:, :, None] - mid[None, None, :]), axis=2) < 1e-9
    assert np.array_equal(idx[~tie], near[~tie])
    assert np.array_equal(_full_index(D, b, codes), idx)
    np.testing.assert_allclose(xn, np.linalg.norm(x, axis=1), rtol=1e-6)
    r = y_np - c[idx]
    np.testing.assert_allclose(rn, np.linalg.norm(r, axis=1), rtol=1e-5)


@pytest.mark.parametrize("b", [2, 4])
def test_mse_score_matches_separate_estimate_routine(b):
    """Scores from the stored records equal the separately written MSE
    estimate, which quantizes on the fly without any packing."""
    P = O.MseParams(D, b, 5)
    x = synth.gaussian_rows(12, D, seed=22).numpy().astype(np.float64)
    q = synth.gaussian_rows(3, D, seed=23, norm_range=None).numpy().astype(np.float64)
    codes, xn, rn = O.mse_encode(P, x)
    s = O.mse_score(P, codes, xn, q)
    for t in range(q.shape[0]):
        for v in range(x.shape[0]):
            ref = O.mse_estimate(D, b, 5, x[v], q[t])
            # the record stores |x| in fp32 (relative rounding <= 2^-24)
            assert abs(s[t, v] - ref) <= 1.2e-7 * abs(ref) + 1e-12


@pytest.mark.parametrize("b", [1, 3])
def test_mse_score_is_inner_product_with_decoded(b):
    P = O.MseParams(D, b, 6)
    x = synth.gaussian_rows(50, D, seed=24).numpy()
    q = synth.gaussian_rows(4, D, seed=25, norm_range=None).numpy()
    codes, xn, rn = O.mse_encode(P, x)
    s = O.mse_score(P, codes, xn, q)
    xh = O.mse_decode(P, codes, xn)
    np.testing.assert_allclose(s, q.astype(np.float64) @ xh.T, rtol=1e-10, atol=1e-12)


def test_mse_distortion_near_table_and_falling():
    """E|y - c[idx]|^2 over random directions is close to the N(0,1) Lloyd-Max
    distortion D_b (the rotated coordinates are nearly N(0, 1/d)) and falls
    with b."""
    table = _read_lloyd_max()
    x = synth.gaussian_rows(3000, D, seed=26, unit=True).numpy()
    prev = np.inf
    for b in (1, 2, 3, 4):
        P = O.MseParams(D, b, 7)
        codes, xn, rn = O.mse_encode(P, x)
        mse = float(np.mean(rn.astype(np.float64) ** 2))
        assert abs(mse - table[1 << b][2]) < 0.05 * table[1 << b][2], (b, mse)
        assert mse < prev
        prev = mse
