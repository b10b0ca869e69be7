"""Pins of the oracle's parameters (random numbers, codebook, Pi, S) against
things other than the oracle itself: published generator outputs, Max's 1960
table, closed forms, numerical quadrature and LAPACK's QR via numpy."""
import math
import os

import numpy as np
import pytest
from scipy import integrate, stats

from oracle import oracle as O

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _read_lloyd_max():
    rows = {}
    with open(os.path.join(GOLDEN, "lloyd_max_gaussian.txt")) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            lev, ys, xs, D = [s.strip() for s in line.split("|")]
            L = int(lev.split("=")[1])
            rows[L] = ([float(v) for v in ys.split()], [float(v) for v in xs.split()], float(D))
    return rows


# --------------------------------------------------------------------------
# random numbers
# --------------------------------------------------------------------------
def test_splitmix64_published_outputs():
    gamma = 0x9E3779B97F4A7C15
    with open(os.path.join(GOLDEN, "splitmix64.txt")) as f:
        for line in f:
            if line.startswith("#") or not line.strip():
                continue
            i, v = line.split()
            state = ((int(i) + 1) * gamma) % (1 << 64)
            assert O.mix64(state) == int(v, 16)


def test_stream_is_counter_based_and_keyed():
    # stream (seed, s) = SplitMix64 sequence from mix64(seed ^ s*gamma)
    a = [O.stream_u64(5, 1, i) for i in range(4)]
    assert len(set(a)) == 4
    assert O.stream_u64(5, 1, 2) == a[2]
    assert O.stream_u64(5, 0, 0) != O.stream_u64(5, 1, 0)
    assert O.stream_u64(6, 1, 0) != O.stream_u64(5, 1, 0)


def test_box_muller_is_standard_normal():
    g = O.gaussian(11, 0, 200_001)
    assert abs(g.mean()) < 5 * (1 / math.sqrt(g.size))
    assert abs(g.var() - 1.0) < 5 * math.sqrt(2 / g.size)
    ks = stats.kstest(g, "norm")
    assert ks.pvalue > 1e-3
    # pairs are independent: correlation of cos/sin halves ~ 0
    c = np.corrcoef(g[0:-1:2], g[1::2])[0, 1]
    assert abs(c) < 5 / math.sqrt(g.size / 2)
    # odd count drops the last sine only
    h = O.gaussian(11, 0, 7)
    np.testing.assert_array_equal(h, g[:7])


# --------------------------------------------------------------------------
# Lloyd-Max codebook
# --------------------------------------------------------------------------
def test_lloyd_max_one_bit_closed_form():
    c, b, D, _ = O.lloyd_max(2)
    assert abs(c[1] - math.sqrt(2 / math.pi)) < 1e-14
    assert c[0] == -c[1] and b[0] == 0.0
    assert abs(D - (1 - 2 / math.pi)) < 1e-13


@pytest.mark.parametrize("L", [2, 4, 8, 16])
def test_lloyd_max_matches_max_1960_table(L):
    ys, xs, D_tab = _read_lloyd_max()[L]
    c, b, D, _ = O.lloyd_max(L)
    np.testing.assert_allclose(c[L // 2:], ys, atol=6e-4, rtol=0)
    np.testing.assert_allclose(b[L // 2 - 1:], xs, atol=6e-4, rtol=0)
    # four printed figures; the 16-level entry of the 1960 table is known to be
    # slightly low in its last digit, so the table is held to 0.1 % here and the
    # quadrature test below pins D to 1e-10.
    assert abs(D - D_tab) < 1e-3 * D_tab
    # symmetric, sorted, spacing growing away from the centre
    np.testing.assert_array_equal(c, -c[::-1])
    assert np.all(np.diff(c) > 0)
    gaps = np.diff(c[L // 2:])
    assert np.all(np.diff(gaps) > 0) if gaps.size > 1 else True


@pytest.mark.parametrize("L", [4, 8, 16])
def test_lloyd_max_optimality_by_quadrature(L):
    """Centroid condition and distortion checked by adaptive quadrature of the
    normal density (scipy), independent of the oracle's closed forms."""
    c, b, D, _ = O.lloyd_max(L)
    pdf = stats.norm.pdf
    edges = [-np.inf] + list(b) + [np.inf]
    total = 0.0
    for j in range(L):
        m0 = integrate.quad(pdf, edges[j], edges[j + 1], epsabs=1e-14, epsrel=1e-13)[0]
        m1 = integrate.quad(lambda t: t * pdf(t), edges[j], edges[j + 1],
                            epsabs=1e-14, epsrel=1e-13)[0]
        assert abs(m1 / m0 - c[j]) < 1e-9
        total += integrate.quad(lambda t: (t - c[j]) ** 2 * pdf(t), edges[j], edges[j + 1],
                                epsabs=1e-14, epsrel=1e-13)[0]
    assert abs(total - D) < 1e-10
    np.testing.assert_allclose(b, 0.5 * (c[:-1] + c[1:]), rtol=0, atol=0)


def test_distortion_falls_with_bits():
    Ds = [O.lloyd_max(1 << k)[2] for k in range(0, 6)]
    assert Ds[0] == 1.0
    assert all(Ds[i + 1] < Ds[i] for i in range(len(Ds) - 1))
    # high-rate (Panter-Dite) asymptote: D ~ (sqrt(3) pi / 2) 4^-k
    k = 5
    assert abs(Ds[k] / (math.sqrt(3) * math.pi / 2 * 4.0 ** -k) - 1) < 0.1


@pytest.mark.parametrize("d,b", [(128, 2), (128, 4), (1536, 3), (3072, 4)])
def test_codebook_scaled_to_dimension(d, b):
    c, beta = O.codebook(d, b)
    L = 1 << (b - 1)
    cd, bd, _, _ = O.lloyd_max(L)
    np.testing.assert_array_equal(c, (cd / math.sqrt(d)).astype(np.float32))
    np.testing.assert_array_equal(beta, (bd / math.sqrt(d)).astype(np.float32))


def test_codebook_one_bit_total_is_empty():
    c, beta = O.codebook(128, 1)
    assert c.size == 0 and beta.size == 0


# --------------------------------------------------------------------------
# Pi and S
# --------------------------------------------------------------------------
@pytest.mark.parametrize("d", [32, 128])
def test_rotation_is_haar_qr_of_gaussian(d):
    seed = 3
    pf, pd, rd = O.rotation(d, seed, want_double=True)
    G = O.gaussian(seed, 0, d * d).reshape(d, d)
    # orthogonal
    assert np.abs(pd.T @ pd - np.eye(d)).max() < 1e-12
    assert np.abs(pf.astype(np.float64).T @ pf.astype(np.float64) - np.eye(d)).max() < 1e-6
    # G = Pi R with R upper triangular, positive diagonal
    R = pd.T @ G
    assert np.abs(np.tril(R, -1)).max() < 1e-10 * np.abs(R).max()
    assert np.all(np.diag(R) > 0)
    np.testing.assert_allclose(np.diag(R), rd, rtol=1e-12)
    # LAPACK's Householder QR with the same sign normalisation
    Q, Rl = np.linalg.qr(G)
    Q = Q * np.sign(np.diag(Rl))[None, :]
    assert np.abs(Q - pd).max() < 1e-11
    # stored fp32 copy is the rounded double
    np.testing.assert_array_equal(pf, pd.astype(np.float32))


def test_rotation_is_dense_not_hadamard():
    d = 128
    pf = O.rotation(d, 0)
    a = np.abs(pf)
    # a (scaled) Hadamard matrix has every |entry| = 1/sqrt(d)
    assert np.std(a * math.sqrt(d)) > 0.3
    # entries of a Haar matrix are ~ N(0, 1/d)
    assert abs((pf.astype(np.float64) ** 2).mean() * d - 1.0) < 1e-6


def test_rotation_deterministic_per_seed():
    a = O.rotation(64, 9)
    b = O.rotation(64, 9)
    c = O.rotation(64, 10)
    np.testing.assert_array_equal(a, b)
    assert np.abs(a - c).max() > 0.1


def test_qjl_matrix_is_gaussian_stream_one():
    d = 128
    S = O.qjl_matrix(d, 4)
    g = O.gaussian(4, 1, d * d).astype(np.float32).reshape(d, d)
    np.testing.assert_array_equal(S, g)
    assert stats.kstest(S.ravel().astype(np.float64), "norm").pvalue > 1e-3
    # independent of Pi's stream
    G0 = O.gaussian(4, 0, d * d).reshape(d, d)
    assert abs(np.corrcoef(G0.ravel(), S.ravel())[0, 1]) < 0.05
