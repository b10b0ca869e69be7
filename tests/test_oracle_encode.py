"""Pins of the oracle's encode, decode, score and top-k: brute force on tiny
inputs, invariants, closed forms and library routines (numpy)."""
import itertools
import math

import numpy as np
import pytest

import synth
from oracle import oracle as O


def _bits_reader(d, b, codes):
    """Independent reader of the documented layout via np.unpackbits (little
    bit order): returns idx [n,d], z [n,d]."""
    n = codes.shape[0]
    k = b - 1
    words = codes.reshape(n, d // 32, b)
    bits = np.unpackbits(words.view(np.uint8).reshape(n, d // 32, b * 4), axis=2,
                         bitorder="little")  # [n, blocks, 32*b]
    idx = np.zeros((n, d), np.int64)
    z = np.zeros((n, d), np.int64)
    for j in range(32):
        if b in (1, 2, 4):
            base = b * j  # fields are b bits wide, contiguous across words
            for t in range(k):
                idx[:, j::32] += bits[:, :, base + t].astype(np.int64) << t
            z[:, j::32] = bits[:, :, base + k]
        else:  # b == 3: 2-bit index fields in words 0..1, sign plane in word 2
            for t in range(2):
                idx[:, j::32] += bits[:, :, 2 * j + t].astype(np.int64) << t
            z[:, j::32] = bits[:, :, 64 + j]
    return idx, z


@pytest.fixture(scope="module")
def p128():
    return {b: O.Params(128, b, 0) for b in (1, 2, 3, 4)}


@pytest.mark.parametrize("b", [1, 2, 3, 4])
def test_layout_roundtrip_and_independent_reader(p128, b):
    P = p128[b]
    x = synth.gaussian_rows(64, 128, seed=1).numpy()
    codes, xn, rn, y, p, idx = O.encode(P, x, diagnostics=True)
    assert codes.shape == (64, b * 4)
    i2, z2 = O.unpack(128, b, codes)
    np.testing.assert_array_equal(i2, idx)
    np.testing.assert_array_equal(z2, (p >= 0).astype(np.int32))
    i3, z3 = _bits_reader(128, b, codes)
    np.testing.assert_array_equal(i3, idx)
    np.testing.assert_array_equal(z3, (p >= 0).astype(np.int32))


@pytest.mark.parametrize("b", [2, 3, 4])
def test_index_is_nearest_codeword_brute_force(p128, b):
    """Rounding each coordinate on the grid equals the argmin over all joint
    codewords of the squared error (checked jointly on 4 coordinates at a
    time, 2^(4k) candidates)."""
    P = p128[b]
    x = synth.gaussian_rows(16, 128, seed=2).numpy()
    _, _, _, y, _, idx = O.encode(P, x, diagnostics=True)
    c = P.c.astype(np.float64)
    L = c.size
    cands = np.array(list(itertools.product(range(L), repeat=4)))  # [L^4, 4]
    for v in range(4):
        for g in range(0, 128, 4):
            yy = y[v, g:g + 4]
            err = ((yy[None, :] - c[cands]) ** 2).sum(1)
            best = cands[np.argmin(err)]
            np.testing.assert_array_equal(best, idx[v, g:g + 4])


def test_sign_bits_maximise_correlation_brute_force(p128):
    P = p128[4]
    x = synth.gaussian_rows(8, 128, seed=3).numpy()
    codes, _, _, _, p, _ = O.encode(P, x, diagnostics=True)
    _, z = O.unpack(128, 4, codes)
    pats = np.array(list(itertools.product([-1.0, 1.0], repeat=4)))
    for v in range(8):
        for g in range(0, 128, 4):
            best = pats[np.argmax(pats @ p[v, g:g + 4])]
            np.testing.assert_array_equal(best, 2 * z[v, g:g + 4] - 1)


def test_rotation_preserves_norm_and_norms_recorded(p128):
    P = p128[3]
    x = synth.gaussian_rows(32, 128, seed=4).numpy()
    codes, xn, rn, y, p, idx = O.encode(P, x, diagnostics=True)
    np.testing.assert_allclose(np.linalg.norm(y, axis=1), 1.0, atol=1e-6)
    np.testing.assert_allclose(xn, np.linalg.norm(x.astype(np.float64), axis=1), rtol=1e-7)
    # |p|^2 averages d |r|^2 for a Gaussian S (E S^T S = d I)
    ratio = (p ** 2).sum(1) / (128 * rn.astype(np.float64) ** 2)
    assert abs(ratio.mean() - 1) < 0.1


def test_mse_falls_with_bits_and_matches_lloyd_max():
    """E|y - yhat|^2 ~ D_k for the N(0,1/d) marginal (within the O(1/d) gap to
    the exact sphere marginal), strictly decreasing in k."""
    d = 256
    x = synth.gaussian_rows(1500, d, seed=5).numpy()
    errs = []
    for b in (2, 3, 4):
        P = O.Params(d, b, 1)
        _, _, rn, _, _, _ = O.encode(P, x, diagnostics=True)
        D = O.lloyd_max(1 << (b - 1))[2]
        e = float((rn.astype(np.float64) ** 2).mean())
        assert abs(e / D - 1) < 0.03, (b, e, D)
        errs.append(e)
    assert errs[0] > errs[1] > errs[2]


def test_one_bit_has_no_index_and_residual_is_y(p128):
    P = p128[1]
    x = synth.gaussian_rows(16, 128, seed=6).numpy()
    codes, xn, rn, y, p, idx = O.encode(P, x, diagnostics=True)
    assert np.all(idx == 0)
    np.testing.assert_allclose(rn, 1.0, atol=1e-6)


def test_zero_vector(p128):
    for b in (1, 2, 3, 4):
        P = p128[b]
        x = np.zeros((2, 128))
        codes, xn, rn, y, p, idx = O.encode(P, x, diagnostics=True)
        assert np.all(xn == 0) and np.all(y == 0)
        L = 1 << (b - 1)
        assert np.all(idx == (L // 2 if b > 1 else 0))
        q = synth.gaussian_rows(3, 128, seed=7).numpy()
        s = O.score(P, codes, xn, rn, q)
        assert np.all(s == 0.0)


@pytest.mark.parametrize("b", [1, 2, 3, 4])
def test_score_equals_inner_product_with_decoded_vector(p128, b):
    """The estimator is <q, xhat> with xhat the dequantized vector (inverse
    rotation and renormalisation): an algebraic identity between the two."""
    P = p128[b]
    x = synth.gaussian_rows(40, 128, seed=8).numpy()
    q = synth.gaussian_rows(5, 128, seed=9, norm_range=None).numpy()
    codes, xn, rn = O.encode(P, x)
    s = O.score(P, codes, xn, rn, q)
    xh = O.decode(P, codes, xn, rn)
    ref = q.astype(np.float64) @ xh.T
    assert np.abs(s - ref).max() < 1e-12 * np.abs(ref).max() * 128


def test_decode_error_matches_distortion():
    """|x - xhat|^2 / |x|^2 is on average D_k + (pi/2 - 1) D_k for the
    QJL-corrected quantizer (QJL adds variance (pi/2 - 1)|r|^2 on average)."""
    d, b = 128, 3
    P = O.Params(d, b, 2)
    x = synth.gaussian_rows(400, d, seed=10).numpy()
    codes, xn, rn = O.encode(P, x)
    xh = O.decode(P, codes, xn, rn)
    rel = ((xh - x) ** 2).sum(1) / (x.astype(np.float64) ** 2).sum(1)
    D = O.lloyd_max(4)[2]
    assert abs(rel.mean() / (D * math.pi / 2) - 1) < 0.1


def test_topk_matches_numpy_order():
    rng = np.random.default_rng(0)
    s = rng.standard_normal((7, 500))
    s[3, 10] = s[3, 11] = s[3, 12] = 9.0  # ties: ids ascending
    vals, ids = O.topk(s, 10)
    for t in range(7):
        order = np.lexsort((np.arange(500), -s[t]))[:10]
        np.testing.assert_array_equal(ids[t], order)
        np.testing.assert_array_equal(vals[t], s[t, order])
    assert list(ids[3, :3]) == [10, 11, 12]


def test_exact_scores_match_numpy():
    x = synth.gaussian_rows(300, 64, seed=11, norm_range=None).numpy().astype(np.float64)
    q = synth.gaussian_rows(9, 64, seed=12, norm_range=None).numpy().astype(np.float64)
    np.testing.assert_allclose(O.exact_scores(x, q), q @ x.T, rtol=1e-12, atol=1e-12)
