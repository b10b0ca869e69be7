"""Statistical pins of the estimator: the QJL-corrected (b-1)+1-bit estimate
is unbiased over the random matrices, the MSE-only estimate is visibly biased
towards zero by the Lloyd-Max distortion, and the spread of the unbiased
estimate matches the closed-form QJL variance."""
import math

import numpy as np
import pytest

import synth
from oracle import oracle as O

D = 128


@pytest.fixture(scope="module")
def pair():
    x = synth.gaussian_rows(1, D, seed=21, norm_range=None).numpy().astype(np.float64)[0]
    q = x + 0.5 * synth.gaussian_rows(1, D, seed=22, norm_range=None).numpy().astype(np.float64)[0]
    return x, q


def _qjl_estimates(x, q, b, seeds):
    est, pred_var = [], []
    for s in seeds:
        P = O.Params(D, b, s)
        codes, xn, rn, y, p, idx = O.encode(P, x[None, :], diagnostics=True)
        est.append(O.score(P, codes, xn, rn, q[None, :])[0, 0])
        qr, _ = O.query(P, q[None, :])
        r = y[0] - P.c.astype(np.float64)[idx[0]]
        nr2 = float(r @ r)
        pred_var.append(float(xn[0]) ** 2 * (math.pi / 2 * nr2 * float(qr[0] @ qr[0])
                                             - float(r @ qr[0]) ** 2) / D)
    return np.array(est), np.array(pred_var)


@pytest.mark.parametrize("b", [2, 3])
def test_qjl_estimator_unbiased_over_seeds(pair, b):
    x, q = pair
    true = float(q @ x)
    est, pred_var = _qjl_estimates(x, q, b, range(1000))
    err = est - true
    se = err.std(ddof=1) / math.sqrt(err.size)
    assert abs(err.mean()) <= 3 * se, (err.mean(), se)
    # spread = QJL closed form E[|x|^2 ((pi/2)|r|^2 |qr|^2 - <r,qr>^2) / d]
    assert abs(err.var(ddof=1) / pred_var.mean() - 1) < 0.2


@pytest.mark.parametrize("bits", [1, 2, 3])
def test_mse_only_estimator_is_biased(pair, bits):
    x, q = pair
    true = float(q @ x)
    est = np.array([O.mse_estimate(D, bits, s, x, q) for s in range(300)])
    err = est - true
    se = err.std(ddof=1) / math.sqrt(err.size)
    Db = O.lloyd_max(1 << bits)[2]
    assert abs(err.mean()) > 3 * se
    # shrinkage towards zero by ~ the Lloyd-Max distortion: E est = (1 - D_b) <q,x>
    assert abs(err.mean() / (-Db * true) - 1) < 0.25, (err.mean(), -Db * true)
