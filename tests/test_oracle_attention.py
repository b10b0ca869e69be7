"""Pins of the oracle's decode attention over quantized keys and values.

The pages stop at the attention logits (quant_prune_distill #674: the
inner-product estimate; comuna.ru "Google speeds up LLMs 8x": logits from
4-bit keys).  The reading built here is the standard attention those logits
feed: softmax of scale x logits over all keys of the group, applied to the
MSE-dequantized values.  Each test checks the oracle against something other
than its own formula: closed forms with printed numbers, special cases that
reduce to a mean or a single row, the limit of a sharp softmax, invariances
that a wrong axis, sign or index breaks, and bounds."""
import math

import numpy as np
import pytest

import synth
from oracle import oracle as O

D = 128


def _records(n, seed, b_k=4, b_v=4):
    keys = synth.gaussian_rows(n, D, seed=seed).numpy().astype(np.float64)
    vals = synth.gaussian_rows(n, D, seed=seed + 1).numpy().astype(np.float64)
    Pk, Pv = O.Params(D, b_k, 0), O.MseParams(D, b_v, 1)
    kc, kxn, krn = O.encode(Pk, keys)
    vc, vxn, _ = O.mse_encode(Pv, vals)
    return Pk, kc, kxn, krn, Pv, vc, vxn


def test_two_keys_closed_form():
    """logits (0, ln 3) weight the rows 1/4 and 3/4."""
    values = np.array([[1.0, -2.0, 4.0], [5.0, 2.0, 0.0]])
    out = O.softmax_weighted_sum(np.array([[0.0, math.log(3.0)]]), values)
    np.testing.assert_allclose(out[0], [4.0, 1.0, 1.0], rtol=1e-14)


def test_shift_invariance_and_no_overflow():
    """Adding 1000 to every logit changes nothing; exp(1000) alone would
    overflow, so the maximum must be subtracted first."""
    rng = np.random.default_rng(0)
    logits = rng.normal(size=(3, 50))
    values = rng.normal(size=(50, 7))
    a = O.softmax_weighted_sum(logits, values)
    b = O.softmax_weighted_sum(logits + 1000.0, values)
    assert np.all(np.isfinite(b))
    np.testing.assert_allclose(a, b, rtol=1e-12, atol=1e-14)


def test_single_key_returns_its_value():
    Pk, kc, kxn, krn, Pv, vc, vxn = _records(1, 5)
    q = synth.gaussian_rows(3, D, seed=6, norm_range=None).numpy()
    out = O.attention_decode(Pk, kc, kxn, krn, Pv, vc, vxn, q, 1.0 / math.sqrt(D))
    v = O.mse_decode(Pv, vc, vxn)
    for t in range(3):
        np.testing.assert_allclose(out[t], v[0], rtol=1e-12, atol=1e-14)


def test_zero_scale_is_the_mean_value():
    Pk, kc, kxn, krn, Pv, vc, vxn = _records(200, 7)
    q = synth.gaussian_rows(2, D, seed=8, norm_range=None).numpy()
    out = O.attention_decode(Pk, kc, kxn, krn, Pv, vc, vxn, q, 0.0)
    v = O.mse_decode(Pv, vc, vxn)
    np.testing.assert_allclose(out, np.broadcast_to(v.mean(axis=0), out.shape), rtol=1e-10,
                               atol=1e-12)


def test_sharp_softmax_picks_the_best_key():
    """A large scale leaves (nearly) all weight on the key with the largest
    estimated logit: the output is that key's value (not the smallest's)."""
    Pk, kc, kxn, krn, Pv, vc, vxn = _records(64, 9)
    q = synth.gaussian_rows(2, D, seed=10, norm_range=None).numpy()
    s = O.score(Pk, kc, kxn, krn, q)
    v = O.mse_decode(Pv, vc, vxn)
    out = O.attention_decode(Pk, kc, kxn, krn, Pv, vc, vxn, q, 1e4)
    for t in range(2):
        np.testing.assert_allclose(out[t], v[int(np.argmax(s[t]))], rtol=1e-9, atol=1e-9)


def test_joint_permutation_invariance():
    """Permuting keys and values together keeps the output; permuting only
    the values changes it (the j-th weight belongs to the j-th value)."""
    Pk, kc, kxn, krn, Pv, vc, vxn = _records(100, 11)
    q = synth.gaussian_rows(2, D, seed=12, norm_range=None).numpy()
    scale = 1.0 / math.sqrt(D)
    a = O.attention_decode(Pk, kc, kxn, krn, Pv, vc, vxn, q, scale)
    perm = np.random.default_rng(1).permutation(100)
    b = O.attention_decode(Pk, kc[perm], kxn[perm], krn[perm], Pv, vc[perm], vxn[perm], q, scale)
    np.testing.assert_allclose(a, b, rtol=1e-10, atol=1e-12)
    c = O.attention_decode(Pk, kc, kxn, krn, Pv, vc[perm], vxn[perm], q, scale)
    assert np.abs(a - c).max() > 1e-3


@pytest.mark.parametrize("b_k,b_v", [(2, 2), (4, 3)])
def test_output_is_a_convex_combination(b_k, b_v):
    """Every output coordinate lies between the smallest and largest value of
    that coordinate over the keys."""
    Pk, kc, kxn, krn, Pv, vc, vxn = _records(300, 13, b_k, b_v)
    q = synth.gaussian_rows(4, D, seed=14, norm_range=None).numpy()
    out = O.attention_decode(Pk, kc, kxn, krn, Pv, vc, vxn, q, 1.0 / math.sqrt(D))
    v = O.mse_decode(Pv, vc, vxn)
    lo, hi = v.min(axis=0), v.max(axis=0)
    assert np.all(out >= lo - 1e-12) and np.all(out <= hi + 1e-12)
