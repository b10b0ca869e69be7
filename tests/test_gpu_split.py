"""Parity of the fractional widths (b - 1/2 bits a coordinate: the first d/2
rotated coordinates at b bits, the last d/2 at b - 1) between the CUDA path
and the oracle: the two grids, encode (cells, signs, norms), scores, top-k on
both the materialised and the fused path, decode, and the shapes each kernel
meets (several blocks of keys, ragged tails, groups, d = 256)."""
import numpy as np
import pytest
import torch

import synth
from oracle import oracle as O
from tests import parity as PT

pytestmark = pytest.mark.gpu


def _np(t):
    return t.detach().cpu().numpy()


def _f64(t):
    return t.detach().cpu().to(torch.float64).numpy()


@pytest.fixture(scope="module")
def squant(cuda, tq_lib):
    cache = {}

    def get(d, b, groups=1):
        key = (d, b, groups)
        if key not in cache:
            cache[key] = tq_lib.TurboQuant(d, b - 0.5, seed=0, groups=groups, device=cuda)
            torch.cuda.synchronize()
        return cache[key]
    return get


@pytest.fixture(scope="module")
def sparams():
    cache = {}

    def get(d, b, seed=0):
        key = (d, b, seed)
        if key not in cache:
            cache[key] = O.SplitParams(d, b, seed)
        return cache[key]
    return get


def _codes(tq_lib, cuda, recs):
    """Oracle records [(codes, xn, rn)] per group -> device Codes."""
    return tq_lib.Codes(
        torch.stack([torch.from_numpy(r[0].view(np.int32)) for r in recs]).to(cuda),
        torch.stack([torch.from_numpy(r[1]) for r in recs]).to(cuda),
        torch.stack([torch.from_numpy(r[2]) for r in recs]).to(cuda))


@pytest.mark.parametrize("b", [2, 3, 4])
def test_split_grids_match_oracle(squant, sparams, b):
    tq = squant(128, b)
    P = sparams(128, b)
    assert tq.split and tq.b == b and tq.words == 2 * (2 * b - 1)
    cb = tq.cb
    assert cb.split == 1 and cb.levels == 1 << (b - 1) and cb.levels_lo == (1 << (b - 2) if b > 2 else 0)
    np.testing.assert_array_equal(np.array(cb.centroids[:cb.levels], np.float32), P.c_hi)
    np.testing.assert_array_equal(np.array(cb.boundaries[:cb.levels - 1], np.float32), P.beta_hi)
    np.testing.assert_array_equal(np.array(cb.centroids_lo[:cb.levels_lo], np.float32), P.c_lo)
    np.testing.assert_array_equal(np.array(cb.boundaries_lo[:max(cb.levels_lo - 1, 0)], np.float32),
                                  P.beta_lo)


def _encode_both(squant, sparams, x, d, b, groups=1):
    tq = squant(d, b, groups)
    codes = tq.encode(x.cuda())
    torch.cuda.synchronize()
    for g in range(groups):
        P = sparams(d, b, g)
        ora = O.split_encode(P, x[g].to(torch.float64).numpy(), diagnostics=True)
        gpu = (_np(codes.codes[g]).view(np.uint32), _np(codes.xnorm[g]), _np(codes.rnorm[g]))
        yield gpu, ora, P


@pytest.mark.parametrize("b", [2, 3, 4])
def test_split_encode_fp32(squant, sparams, b):
    """4096 x 128 fp32 rows with norms in [0.5, 2]."""
    x = synth.gaussian_rows(4096, 128, seed=1)[None]
    for gpu, ora, P in _encode_both(squant, sparams, x, 128, b):
        rep = PT.compare_encode_split(128, b, P.beta_hi, P.beta_lo, gpu, ora)
        assert rep["codes_identical_fraction"] > 0.98, rep


@pytest.mark.parametrize("d,b,G,n", [(128, 4, 2, 3001), (256, 3, 1, 700), (128, 2, 3, 129)])
def test_split_encode_bf16_groups(squant, sparams, d, b, G, n):
    """bf16 keys with outlier channels, several groups, ragged row counts."""
    x = synth.kv_keys(G, n, d, seed=2)
    for gpu, ora, P in _encode_both(squant, sparams, x, d, b, groups=G):
        PT.compare_encode_split(d, b, P.beta_hi, P.beta_lo, gpu, ora)


def test_split_encode_edge_rows(squant, sparams):
    d, b = 128, 3
    x = synth.gaussian_rows(12, d, seed=3)
    x[2] = 0.0
    x[3, :] = 0.0
    x[3, 70] = 1.5  # axis-aligned, in the second half of the input
    for gpu, ora, P in _encode_both(squant, sparams, x[None], d, b):
        PT.compare_encode_split(d, b, P.beta_hi, P.beta_lo, gpu, ora, bound_flags=False)
    tq = squant(d, b)
    empty = tq.encode(x[:0].cuda()[None])
    torch.cuda.synchronize()
    assert empty.codes.shape == (1, 0, tq.words)


@pytest.mark.parametrize("d,b,G,n,nq", [(128, 4, 1, 4096, 1), (128, 3, 2, 3001, 3),
                                        (128, 2, 1, 1027, 16), (256, 4, 2, 700, 37),
                                        (128, 4, 3, 513, 64)])
def test_split_score(squant, sparams, tq_lib, cuda, d, b, G, n, nq):
    """Scores of oracle records: one to 64 queries a group (query passes of
    the SIMT kernel), key counts that end inside a block."""
    x = synth.gaussian_rows(G * n, d, seed=4).reshape(G, n, d)
    qs = synth.gaussian_rows(G * nq, d, seed=5, norm_range=None).reshape(G, nq, d)
    recs = [O.split_encode(sparams(d, b, g), x[g].to(torch.float64).numpy()) for g in range(G)]
    s_gpu = _np(squant(d, b, G).score(_codes(tq_lib, cuda, recs), qs.cuda()))
    for g in range(G):
        c, xn, rn = recs[g]
        s_ora = O.split_score(sparams(d, b, g), c, xn, rn, _f64(qs[g]))
        PT.compare_scores(s_gpu[g], s_ora, np.linalg.norm(_f64(qs[g]), axis=1),
                          xn.astype(np.float64))


@pytest.mark.parametrize("b,G,n,nq,k", [(4, 1, 4096, 17, 10), (3, 2, 2500, 3, 32),
                                        (2, 1, 33, 2, 32)])
def test_split_topk_materialised(squant, sparams, tq_lib, cuda, b, G, n, nq, k):
    d = 128
    x = synth.gaussian_rows(G * n, d, seed=6).reshape(G, n, d)
    qs = synth.gaussian_rows(G * nq, d, seed=7, norm_range=None).reshape(G, nq, d)
    recs = [O.split_encode(sparams(d, b, g), x[g].to(torch.float64).numpy()) for g in range(G)]
    vals, ids = squant(d, b, G).topk(_codes(tq_lib, cuda, recs), qs.cuda(), k)
    for g in range(G):
        c, xn, rn = recs[g]
        s_ora = O.split_score(sparams(d, b, g), c, xn, rn, _f64(qs[g]))
        PT.compare_topk(_np(vals[g]), _np(ids[g]), s_ora, k, np.linalg.norm(_f64(qs[g]), axis=1),
                        float(xn.max()))


@pytest.mark.parametrize("b,k", [(4, 10), (3, 32)])
def test_split_topk_fused(squant, sparams, tq_lib, cuda, b, k):
    """More than 2^24 scores per call: the fused score + per-range top-k
    kernel and the merge of the ranges' lists."""
    d, n, nq = 128, 300_000, 57
    assert n * nq > 1 << 24
    x = synth.gaussian_rows(n, d, seed=8)
    q = synth.gaussian_rows(nq, d, seed=9, norm_range=None)
    P = sparams(d, b)
    c, xn, rn = O.split_encode(P, x.to(torch.float64).numpy())
    vals, ids = squant(d, b).topk(_codes(tq_lib, cuda, [(c, xn, rn)]), q.cuda()[None], k)
    s_ora = O.split_score(P, c, xn, rn, _f64(q))
    PT.compare_topk(_np(vals[0]), _np(ids[0]), s_ora, k, np.linalg.norm(_f64(q), axis=1),
                    float(xn.max()))


def test_split_score_topk_one_call(squant, sparams, tq_lib, cuda):
    """Scores and top-k of one call equal the two separate calls."""
    d, b, n, nq, k = 128, 4, 5000, 4, 10
    x = synth.gaussian_rows(n, d, seed=10)
    q = synth.gaussian_rows(nq, d, seed=11, norm_range=None).cuda()[None]
    tq = squant(d, b)
    codes = tq.encode(x.cuda()[None])
    s, (v, i) = tq.score_topk(codes, q, k)
    s2 = tq.score(codes, q)
    v2, i2 = tq.topk(codes, q, k)
    torch.cuda.synchronize()
    assert torch.equal(s, s2)
    assert torch.equal(i, i2) and torch.equal(v, v2)


@pytest.mark.parametrize("d,b", [(128, 2), (128, 3), (128, 4), (256, 3)])
def test_split_decode(squant, sparams, tq_lib, cuda, d, b):
    x = synth.gaussian_rows(700, d, seed=12)
    P = sparams(d, b)
    c, xn, rn = O.split_encode(P, x.to(torch.float64).numpy())
    ref = O.split_decode(P, c, xn, rn)
    got = _np(squant(d, b).decode(_codes(tq_lib, cuda, [(c, xn, rn)]))[0]).astype(np.float64)
    err = np.linalg.norm(got - ref, axis=1) / np.linalg.norm(ref, axis=1)
    assert err.max() <= 1e-4, err.max()


def test_split_encode_then_score_end_to_end(squant, sparams, tq_lib, cuda):
    """GPU records scored on the GPU agree with the oracle's score of the same
    GPU records (the records themselves are compared above)."""
    d, b, n, nq = 128, 3, 2000, 8
    x = synth.gaussian_rows(n, d, seed=13)
    q = synth.gaussian_rows(nq, d, seed=14, norm_range=None)
    tq = squant(d, b)
    codes = tq.encode(x.cuda()[None])
    s_gpu = _np(tq.score(codes, q.cuda()[None])[0])
    c = _np(codes.codes[0]).view(np.uint32)
    s_ora = O.split_score(sparams(d, b), c, _np(codes.xnorm[0]), _np(codes.rnorm[0]), _f64(q))
    PT.compare_scores(s_gpu, s_ora, np.linalg.norm(_f64(q), axis=1),
                      _np(codes.xnorm[0]).astype(np.float64))


def test_split_rejected_where_unsupported(squant, tq_lib, cuda):
    """Decode attention takes integer widths only: an error, not a wrong result."""
    tq = squant(128, 3)
    with pytest.raises(ValueError):
        tq_lib.TurboQuant(128, 1.5, variant="mse", device=cuda)
    with pytest.raises(ValueError):
        tq_lib.TurboQuant(128, 2.25, device=cuda)
    v = tq_lib.TurboQuant(128, 2, variant="mse", device=cuda)
    keys = tq.encode(synth.gaussian_rows(64, 128, seed=15).cuda()[None])
    vals = v.encode(synth.gaussian_rows(64, 128, seed=16).cuda()[None])
    with pytest.raises(tq_lib.TQError):
        tq.attention_decode(keys, v, vals, synth.gaussian_rows(1, 128, seed=17).cuda()[None])
