"""Parity of the CUDA path (through the C ABI) with the oracle, at sizes the
oracle finishes in seconds: several tiles and ragged tails, every bit width,
fp32 and bf16 inputs, GQA groups, edge cases."""
import math

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
def quant(cuda, tq_lib):
    cache = {}

    def get(d, b, seed=0, groups=1):
        key = (d, b, seed, groups)
        if key not in cache:
            cache[key] = tq_lib.TurboQuant(d, b, seed=seed, groups=groups, device=cuda)
            torch.cuda.synchronize()
        return cache[key]
    return get


@pytest.fixture(scope="module")
def oparams():
    cache = {}

    def get(d, b, seed):
        key = (d, b, seed)
        if key not in cache:
            cache[key] = O.Params(d, b, seed)
        return cache[key]
    return get


# ---------------------------------------------------------------- parameters
@pytest.mark.parametrize("d,b,G", [(128, 4, 2), (128, 2, 1), (1536, 3, 1)])
def test_parameters_match_oracle(quant, oparams, d, b, G):
    tq = quant(d, b, 0, G)
    for g in range(G):
        P = oparams(d, b, g)
        pi = _np(tq.Pi[g])
        diff = pi.view(np.int32).astype(np.int64) - P.Pi.view(np.int32).astype(np.int64)
        assert np.abs(diff).max() <= 1, "Pi differs by more than one fp32 ulp"
        assert (diff != 0).mean() < 1e-3
        S = _np(tq.S[g])
        sd = S.view(np.int32).astype(np.int64) - P.S.view(np.int32).astype(np.int64)
        assert np.abs(sd).max() <= 1 and (sd != 0).sum() <= 2
    c, beta = O.codebook(d, b)
    np.testing.assert_array_equal(tq.centroids().numpy(), c)
    np.testing.assert_array_equal(tq.boundaries().numpy(), beta)
    pi64 = tq.Pi[0].double()
    assert (pi64.T @ pi64 - torch.eye(d, dtype=torch.float64, device=pi64.device)).abs().max() < 1e-5


# ---------------------------------------------------------------- encode
def _encode_both(quant, oparams, x, d, b, groups=1):
    """x: CPU tensor [G, n, d]; returns list of (gpu, oracle) per group."""
    tq = quant(d, b, 0, groups)
    codes = tq.encode(x.cuda())
    torch.cuda.synchronize()
    out = []
    for g in range(groups):
        P = oparams(d, b, g)
        ora = O.encode(P, x[g].to(torch.float64).numpy(), diagnostics=True)
        gpu = (_np(codes.codes[g]).view(np.uint32), _np(codes.xnorm[g]), _np(codes.rnorm[g]))
        out.append((gpu, ora, P))
    return out


@pytest.mark.parametrize("b", [1, 2, 3, 4])
def test_encode_tiny_config(quant, oparams, b):
    """4096 x 128 fp32 rows, norms U[0.5, 2] (the small workload)."""
    x = synth.gaussian_rows(4096, 128, seed=1)[None]
    for gpu, ora, P in _encode_both(quant, oparams, x, 128, b):
        rep = PT.compare_encode(128, b, P.beta, gpu, ora)
        assert rep["codes_identical_fraction"] > 0.98, rep


@pytest.mark.parametrize("b", [2, 3, 4])
def test_encode_kv_bf16_ragged_groups(quant, oparams, b):
    """bf16 keys with x20 outlier channels, 2 KV heads, a ragged row count."""
    x = synth.kv_keys(2, 3001, 128, seed=1)
    for gpu, ora, P in _encode_both(quant, oparams, x, 128, b, groups=2):
        PT.compare_encode(128, b, P.beta, gpu, ora)


@pytest.mark.parametrize("d,b", [(1536, 2), (1536, 4), (3072, 3)])
def test_encode_large_dims(quant, oparams, d, b):
    x = synth.gaussian_rows(257, d, seed=2, unit=True)[None]
    for gpu, ora, P in _encode_both(quant, oparams, x, d, b):
        PT.compare_encode(d, b, P.beta, gpu, ora)


@pytest.mark.parametrize("d,b,G,n", [(256, 4, 2, 700), (512, 3, 1, 1000), (384, 1, 3, 129)])
def test_encode_tensor_core_gemm_shapes(quant, oparams, d, b, G, n):
    """d >= 256: the rotation and QJL products run as split-precision
    tensor-core GEMMs; bf16 keys (one exact piece) and fp32 rows (three
    pieces), ragged last tiles, several groups."""
    if b == 4:
        x = synth.kv_keys(G, n, d, seed=3)
    else:
        x = synth.gaussian_rows(G * n, d, seed=3).reshape(G, n, d)
    for gpu, ora, P in _encode_both(quant, oparams, x, d, b, groups=G):
        PT.compare_encode(d, b, P.beta, gpu, ora)


def test_encode_edge_rows(quant, oparams):
    d, b = 128, 4
    x = synth.gaussian_rows(40, d, seed=3)
    x[5] = 0.0                 # zero vector
    x[6] = 1e-30               # denormal-scale row
    x[7] = 1e30 / math.sqrt(d)  # very large row
    x[8, :] = 0.0
    x[8, 17] = 2.0              # axis-aligned row
    for gpu, ora, P in _encode_both(quant, oparams, x[None], d, b):
        PT.compare_encode(d, b, P.beta, gpu, ora, bound_flags=False)
    tq = quant(d, b)
    one = tq.encode(x[:1].cuda()[None])
    empty = tq.encode(x[:0].cuda()[None])
    torch.cuda.synchronize()
    assert one.codes.shape == (1, 1, 16) and empty.codes.shape == (1, 0, 16)


# ---------------------------------------------------------------- score / top-k / decode
def _oracle_records(oparams, x, d, b, seed=0):
    P = oparams(d, b, seed)
    codes, xn, rn = O.encode(P, x.to(torch.float64).numpy())
    return P, codes, xn, rn


def _to_codes(tq_lib, codes, xn, rn, device):
    return tq_lib.Codes(torch.from_numpy(codes.view(np.int32)).to(device)[None],
                        torch.from_numpy(xn).to(device)[None],
                        torch.from_numpy(rn).to(device)[None])


@pytest.mark.parametrize("b", [1, 2, 3, 4])
def test_score_tiny_config(quant, oparams, tq_lib, cuda, b):
    d = 128
    x = synth.gaussian_rows(4096, d, seed=1)
    q = synth.gaussian_rows(64, d, seed=2, norm_range=None)
    P, codes, xn, rn = _oracle_records(oparams, x, d, b)
    s_ora = O.score(P, codes, xn, rn, q.numpy())
    tq = quant(d, b)
    s_gpu = _np(tq.score(_to_codes(tq_lib, codes, xn, rn, cuda), q.cuda()[None])[0])
    PT.compare_scores(s_gpu, s_ora, np.linalg.norm(_f64(q), axis=1), xn.astype(np.float64))


def test_score_gqa_bf16_groups(quant, oparams, tq_lib, cuda):
    d, b, G = 128, 4, 2
    keys = synth.kv_keys(G, 1500, d, seed=1)
    qs = synth.kv_queries(2 * G, G, d, seed=2)  # [G, 2, d]
    tq = quant(d, b, 0, G)
    recs = [_oracle_records(oparams, keys[g], d, b, seed=g) for g in range(G)]
    codes = tq_lib.Codes(
        torch.stack([torch.from_numpy(r[1].view(np.int32)) for r in recs]).to(cuda),
        torch.stack([torch.from_numpy(r[2]) for r in recs]).to(cuda),
        torch.stack([torch.from_numpy(r[3]) for r in recs]).to(cuda))
    s_gpu = _np(tq.score(codes, qs.cuda()))
    for g in range(G):
        P, c, xn, rn = recs[g]
        s_ora = O.score(P, c, xn, rn, _f64(qs[g]))
        PT.compare_scores(s_gpu[g], s_ora, np.linalg.norm(_f64(qs[g]), axis=1), xn.astype(np.float64))


@pytest.mark.parametrize("G,n,nq,b", [(160, 300, 2, 4), (160, 300, 16, 4), (3, 1000, 37, 3), (2, 129, 16, 2)])
def test_score_groups_and_query_passes(quant, oparams, tq_lib, cuda, G, n, nq, b):
    """More groups than SMs (whole groups per CTA in turn), several query
    passes per group, a ragged last tile of keys."""
    d = 128
    W = b * d // 32
    qs = synth.gaussian_rows(G * nq, d, seed=50, norm_range=None).reshape(G, nq, d)
    recs = [synth.random_records(n, W, seed=60 + g) for g in range(G)]
    codes = tq_lib.Codes(
        torch.stack([torch.from_numpy(r[0].view(np.int32)) for r in recs]).to(cuda),
        torch.stack([torch.from_numpy(r[1]) for r in recs]).to(cuda),
        torch.stack([torch.from_numpy(r[2]) for r in recs]).to(cuda))
    s_gpu = _np(quant(d, b, 0, G).score(codes, qs.cuda()))
    for g in range(G):
        c, xn, rn = recs[g]
        s_ora = O.score(oparams(d, b, g), c, xn, rn, _f64(qs[g]))
        PT.compare_scores(s_gpu[g], s_ora, np.linalg.norm(_f64(qs[g]), axis=1), xn.astype(np.float64))


@pytest.mark.parametrize("G,n,nq,d", [(3, 2051, 1, 128), (2, 4097, 3, 128), (1, 1027, 4, 128),
                                      (2, 3000, 4, 256), (1, 1024, 2, 128)])
def test_score_few_queries_shapes(quant, oparams, tq_lib, cuda, G, n, nq, d):
    """b = 4 with at most 4 queries per group (the SIMT scoring kernel): 1, 3
    and 4 queries, key counts that are not multiples of the 256 keys of a
    block, d = 256, several groups; scores and top-10."""
    b = 4
    W = b * d // 32
    qs = synth.gaussian_rows(G * nq, d, seed=70, norm_range=None).reshape(G, nq, d)
    recs = [synth.random_records(n, W, seed=80 + g) for g in range(G)]
    codes = tq_lib.Codes(
        torch.stack([torch.from_numpy(r[0].view(np.int32)) for r in recs]).to(cuda),
        torch.stack([torch.from_numpy(r[1]) for r in recs]).to(cuda),
        torch.stack([torch.from_numpy(r[2]) for r in recs]).to(cuda))
    tq = quant(d, b, 0, G)
    s_gpu = _np(tq.score(codes, qs.cuda()))
    vals, ids = tq.topk(codes, qs.cuda(), 10)
    for g in range(G):
        c, xn, rn = recs[g]
        s_ora = O.score(oparams(d, b, g), c, xn, rn, _f64(qs[g]))
        qn = np.linalg.norm(_f64(qs[g]), axis=1)
        PT.compare_scores(s_gpu[g], s_ora, qn, xn.astype(np.float64))
        PT.compare_topk(_np(vals[g]), _np(ids[g]), s_ora, 10, qn, float(xn.max()))


@pytest.mark.parametrize("n,k,nq", [(4096, 10, 17), (2500, 1, 3), (2500, 32, 3), (33, 32, 2)])
def test_topk(quant, oparams, tq_lib, cuda, n, k, nq):
    d, b = 128, 4
    x = synth.gaussian_rows(n, d, seed=4)
    q = synth.gaussian_rows(nq, d, seed=5, norm_range=None)
    P, codes, xn, rn = _oracle_records(oparams, x, d, b)
    s_ora = O.score(P, codes, xn, rn, q.numpy())
    tq = quant(d, b)
    vals, ids = tq.topk(_to_codes(tq_lib, codes, xn, rn, cuda), q.cuda()[None], k)
    PT.compare_topk(_np(vals[0]), _np(ids[0]), s_ora, k, np.linalg.norm(_f64(q), axis=1),
                    float(xn.max()))


@pytest.mark.parametrize("G,n,k,b", [(1, 400_000, 10, 4), (1, 400_000, 32, 2), (3, 150_001, 10, 3)])
def test_topk_long_ranges(quant, oparams, tq_lib, cuda, G, n, k, b):
    """Key ranges of many passes per block: the running threshold and the
    candidate-buffer cuts of the fused score + top-k kernel are exercised."""
    d, nq = 128, 4
    W = b * d // 32
    qs = synth.gaussian_rows(G * nq, d, seed=21, norm_range=None).reshape(G, nq, d)
    recs = [synth.random_records(n, W, seed=30 + g) for g in range(G)]
    codes = tq_lib.Codes(
        torch.stack([torch.from_numpy(r[0].view(np.int32)) for r in recs]).to(cuda),
        torch.stack([torch.from_numpy(r[1]) for r in recs]).to(cuda),
        torch.stack([torch.from_numpy(r[2]) for r in recs]).to(cuda))
    vals, ids = quant(d, b, 0, G).topk(codes, qs.cuda(), k)
    for g in range(G):
        c, xn, rn = recs[g]
        s_ora = O.score(oparams(d, b, g), c, xn, rn, _f64(qs[g]))
        PT.compare_topk(_np(vals[g]), _np(ids[g]), s_ora, k, np.linalg.norm(_f64(qs[g]), axis=1),
                        float(xn.max()))


@pytest.mark.parametrize("copies", [41, 5000])
def test_topk_equal_scores_take_smallest_ids(quant, oparams, tq_lib, cuda, copies):
    """Copies of the best record score exactly alike; the top-k keeps the
    smallest ids among them (ties: id ascending).  5000 copies overflow the
    gathered candidate set and take the full-row selection."""
    d, b, n, nq, k = 128, 4, 300_000, 2, 10
    c, xn, rn = synth.random_records(n, b * d // 32, seed=40)
    q = synth.gaussian_rows(nq, d, seed=41, norm_range=None)
    best = int(np.argmax(O.score(oparams(d, b, 0), c, xn, rn, _f64(q))[0]))
    pos = np.sort(synth.sample_rows(n, copies, seed=42).numpy())
    pos = pos[pos != best]
    c[pos], xn[pos], rn[pos] = c[best], xn[best], rn[best]
    copies = np.sort(np.append(pos, best))
    vals, ids = quant(d, b).topk(_to_codes(tq_lib, c, xn, rn, cuda), q.cuda()[None], k)
    np.testing.assert_array_equal(_np(ids[0])[0], copies[:k])
    assert np.all(_np(vals[0])[0] == _np(vals[0])[0][0])


def test_topk_fused_path(quant, oparams, tq_lib, cuda):
    """More than 2^24 scores: the fused score + running-list kernel and the
    merge of its per-range lists (instead of materialised scores)."""
    d, b, n, nq, k = 128, 2, 2_200_000, 8, 10
    c, xn, rn = synth.random_records(n, b * d // 32, seed=45)
    q = synth.gaussian_rows(nq, d, seed=46, norm_range=None)
    vals, ids = quant(d, b).topk(_to_codes(tq_lib, c, xn, rn, cuda), q.cuda()[None], k)
    s_ora = O.score(oparams(d, b, 0), c, xn, rn, _f64(q))
    PT.compare_topk(_np(vals[0]), _np(ids[0]), s_ora, k, np.linalg.norm(_f64(q), axis=1),
                    float(xn.max()))


def test_exact_topk_many_tiles(tq_lib, cuda):
    """Thousands of partial lists per row through the merge."""
    n, d, nq, k = 200_000, 128, 3, 10
    x = synth.gaussian_rows(n, d, seed=43, unit=True)
    q = synth.gaussian_rows(nq, d, seed=44, unit=True)
    vals, ids = tq_lib.exact_topk(x.cuda()[None], q.cuda()[None], k)
    ex = O.exact_scores(_f64(x), _f64(q))
    PT.compare_topk(_np(vals[0]), _np(ids[0]), ex, k, np.ones(nq), 1.0)


@pytest.mark.parametrize("d,b,G,n,nq,mse", [(256, 4, 2, 3000, 70, False), (384, 2, 1, 1025, 130, False),
                                            (256, 3, 1, 2000, 64, True), (256, 4, 1, 1500, 100, True),
                                            (512, 1, 1, 700, 64, False), (256, 4, 2, 1000, 300, False)])
def test_score_and_topk_decoded_key_gemm(quant, quant_mse, oparams, tq_lib, cuda, d, b, G, n, nq,
                                         mse):
    """d >= 256 with 64+ queries per group: scores as a tensor-core GEMM over
    decoded keys (transposed store, per-tile maxima for the top-k); ragged key
    tiles, padded query tiles, several groups, both variants, every bit width
    of the in-GEMM decode (b = 4 through its byte tables), and 300 queries
    (decoded keys through the workspace)."""
    k = 10
    qs = synth.gaussian_rows(G * nq, d, seed=51, norm_range=None).reshape(G, nq, d)
    W = b * d // 32
    recs = [synth.random_records(n, W, seed=100 + g) for g in range(G)]
    codes = tq_lib.Codes(
        torch.stack([torch.from_numpy(r[0].view(np.int32)) for r in recs]).to(cuda),
        torch.stack([torch.from_numpy(r[1]) for r in recs]).to(cuda),
        torch.stack([torch.from_numpy(r[2]) for r in recs]).to(cuda))
    tq = quant_mse(d, b, 0, G) if mse else quant(d, b, 0, G)
    s_gpu = _np(tq.score(codes, qs.cuda()))
    vals, ids = tq.topk(codes, qs.cuda(), k)
    for g in range(G):
        c, xn, rn = recs[g]
        if mse:
            s_ora = O.mse_score(O.MseParams(d, b, g), c, xn, _f64(qs[g]))
        else:
            s_ora = O.score(oparams(d, b, g), c, xn, rn, _f64(qs[g]))
        qn = np.linalg.norm(_f64(qs[g]), axis=1)
        PT.compare_scores(s_gpu[g], s_ora, qn, xn.astype(np.float64))
        PT.compare_topk(_np(vals[g]), _np(ids[g]), s_ora, k, qn, float(xn.max()))


@pytest.mark.parametrize("b", [1, 3, 4])
def test_decode(quant, oparams, tq_lib, cuda, b):
    d = 128
    x = synth.gaussian_rows(700, d, seed=6)
    P, codes, xn, rn = _oracle_records(oparams, x, d, b)
    ref = O.decode(P, codes, xn, rn)
    got = _np(quant(d, b).decode(_to_codes(tq_lib, codes, xn, rn, cuda))[0]).astype(np.float64)
    err = np.linalg.norm(got - ref, axis=1) / np.linalg.norm(ref, axis=1)
    assert err.max() <= 1e-4, err.max()


def test_logits_fp32(tq_lib, cuda):
    G, n, d = 2, 3000, 128
    keys = synth.gaussian_rows(G * n, d, seed=7, norm_range=None).reshape(G, n, d)
    q = synth.kv_queries(8, G, d, seed=8).float()
    out = _np(tq_lib.logits_fp32(keys.cuda(), q.cuda()))
    ref = np.einsum("gqd,gnd->gqn", _f64(q), _f64(keys))
    tol = 1e-5 * np.linalg.norm(_f64(q), axis=2)[:, :, None] * np.linalg.norm(_f64(keys), axis=2)[:, None, :]
    assert np.all(np.abs(out - ref) <= tol)


def test_exact_topk(tq_lib, cuda):
    n, d, nq, k = 5000, 256, 7, 10
    x = synth.gaussian_rows(n, d, seed=9, unit=True)
    q = synth.gaussian_rows(nq, d, seed=10, unit=True)
    vals, ids = tq_lib.exact_topk(x.cuda()[None], q.cuda()[None], k)
    ex = O.exact_scores(_f64(x), _f64(q))
    PT.compare_topk(_np(vals[0]), _np(ids[0]), ex, k, np.ones(nq), 1.0)


def test_errors_on_device(quant, tq_lib, cuda):
    tq = quant(128, 4)
    B = tq_lib.binding
    x = torch.zeros(1, 10, 128, device=cuda)
    with pytest.raises(B.TQError) as e:
        B.tq_encode(tq.cb, tq.Pi.data_ptr(), tq.S.data_ptr(), 1, 10, x.data_ptr(), B.TQ_F32,
                    x.data_ptr(), x.data_ptr(), x.data_ptr(), x.data_ptr(), 16,
                    torch.cuda.current_stream().cuda_stream)
    assert e.value.status == B.TQ_ERR_WORKSPACE
    with pytest.raises(ValueError):
        tq.encode(torch.zeros(10, 64, device=cuda))
    torch.cuda.synchronize()


def test_device_wait_times_out_and_context_survives(quant, oparams, tq_lib, cuda):
    """The bounded device-side wait gives up on a barrier nothing completes,
    the status word reports TQ_ERR_DEVICE_TIMEOUT, and the next calls on the
    same context run and are correct (status clean again)."""
    B = tq_lib.binding
    stream = torch.cuda.current_stream().cuda_stream
    ws = torch.zeros(256, dtype=torch.uint8, device=cuda)
    B.tq_selftest_wait_timeout(ws.data_ptr(), 20_000_000, stream)  # 20 ms
    assert B.tq_device_status(ws.data_ptr(), stream) == B.TQ_ERR_DEVICE_TIMEOUT
    with pytest.raises(B.TQError):
        B.tq_selftest_wait_timeout(ws.data_ptr(), 0, stream)
    # the context is still usable: an encode through the tensor-core kernel
    x = synth.kv_keys(1, 300, 128, seed=12)
    for gpu, ora, P in _encode_both(quant, oparams, x, 128, 4):
        PT.compare_encode(128, 4, P.beta, gpu, ora)
    assert B.tq_device_status(quant(128, 4).ws.buf.data_ptr(), stream) == B.TQ_OK


# ---------------------------------------------------------------- tensor-core encode (d = 128, bf16)
@pytest.mark.parametrize("G,n,b", [(1, 64, 1), (3, 640, 4), (1, 5, 2), (160, 100, 4), (8, 4097, 3)])
def test_encode_tc_bf16_shapes(quant, oparams, tq_lib, G, n, b):
    """Shapes of the fused tensor-core kernel: exact tiles, a 5-row tile, more
    groups than SMs (whole groups per CTA, weights reloaded into tensor
    memory at each group), ragged tails; device status word stays clean."""
    x = synth.kv_keys(G, n, 128, seed=11)
    tq = quant(128, b, 0, G)
    codes = tq.encode(x.cuda())
    B = tq_lib.binding
    assert B.tq_device_status(tq.ws.buf.data_ptr(), torch.cuda.current_stream().cuda_stream) == 0
    for g in sorted({0, G // 2, G - 1}):
        P = oparams(128, b, g)
        ora = O.encode(P, x[g].to(torch.float64).numpy(), diagnostics=True)
        gpu = (_np(codes.codes[g]).view(np.uint32), _np(codes.xnorm[g]), _np(codes.rnorm[g]))
        PT.compare_encode(128, b, P.beta, gpu, ora, bound_flags=(n * 128 >= 10 ** 5))


@pytest.mark.parametrize("b", [1, 4])
def test_encode_tc_bf16_edge_rows(quant, oparams, tq_lib, b):
    """Edge rows through the tensor-core kernel, which rescales every key by a
    power of two before its fp16 conversion: zero, tiny (1e-30) and huge
    (1e30) rows, an axis-aligned row and a row with one x1000 outlier."""
    d = 128
    x = synth.gaussian_rows(300, d, seed=4)
    x[5] = 0.0
    x[6] = 1e-30
    x[7] = 1e30 / math.sqrt(d)
    x[8, :] = 0.0
    x[8, 17] = 2.0
    x[9, 3] *= 1000.0
    xb = x.to(torch.bfloat16)
    for gpu, ora, P in _encode_both(quant, oparams, xb[None], d, b):
        PT.compare_encode(d, b, P.beta, gpu, ora, bound_flags=False)
    B = tq_lib.binding
    assert B.tq_device_status(quant(d, b).ws.buf.data_ptr(),
                              torch.cuda.current_stream().cuda_stream) == 0


def test_encode_tc_matches_portable_path(quant, tq_lib):
    """The tensor-core kernel (bf16 input) and the SIMT path (the same values
    given as fp32) produce the same records up to boundary flips."""
    G, n, b = 2, 2000, 4
    x = synth.kv_keys(G, n, 128, seed=12)
    tq = quant(128, b, 0, G)
    c_tc = tq.encode(x.cuda())
    c_pt = tq.encode(x.float().cuda())
    torch.cuda.synchronize()
    same = (c_tc.codes == c_pt.codes).all(dim=2).float().mean().item()
    assert same > 0.995
    assert torch.allclose(c_tc.xnorm, c_pt.xnorm, rtol=1e-6)


# ---------------------------------------------------------------- MSE-only variant
@pytest.fixture(scope="module")
def quant_mse(cuda, tq_lib):
    cache = {}

    def get(d, b, seed=0, groups=1):
        key = (d, b, seed, groups)
        if key not in cache:
            cache[key] = tq_lib.TurboQuant(d, b, seed=seed, groups=groups, device=cuda,
                                           variant="mse")
            torch.cuda.synchronize()
        return cache[key]
    return get


def _mse_full_index(d, b, codes):
    idx, z = PT.read_layout(d, b, codes)
    return z if b == 1 else idx | (z << (b - 1))


def _mse_compare(d, b, gpu, ora, beta, bound_flags=True):
    """Cells bit-exact except within 1e-5 sigma of a boundary (counted, at most
    1e-4 of all coordinates); norms to 1e-4; |r| on records whose cells all
    agree."""
    g_codes, g_xn, g_rn = gpu
    o_codes, o_xn, o_rn, y, o_idx = ora
    g_idx = _mse_full_index(d, b, g_codes)
    assert np.array_equal(_mse_full_index(d, b, o_codes), o_idx)
    sigma = 1.0 / math.sqrt(d)
    if beta.size:
        near = np.min(np.abs(y[:, :, None] - beta.astype(np.float64)[None, None, :]), axis=2) \
            < 1e-5 * sigma
    else:
        near = np.zeros_like(y, dtype=bool)
    mism = g_idx != o_idx
    assert not np.any(mism & ~near), int(np.sum(mism & ~near))
    if bound_flags:
        assert near.mean() <= 1e-4, near.mean()
    np.testing.assert_allclose(g_xn, o_xn, rtol=1e-4, atol=1e-30)
    same = ~np.any(mism, axis=1)
    np.testing.assert_allclose(g_rn[same], o_rn[same], rtol=1e-4, atol=1e-6)


def test_mse_and_prod_share_the_rotation(quant, quant_mse):
    a, m = quant(128, 3, 5), quant_mse(128, 3, 5)
    assert torch.equal(a.Pi, m.Pi)
    assert m.S is None and m.cb.variant == 1 and m.cb.levels == 8


@pytest.mark.parametrize("b", [1, 2, 3, 4])
def test_mse_encode_tiny_config(quant_mse, b):
    d = 128
    x = synth.gaussian_rows(4096, d, seed=1)
    P = O.MseParams(d, b, 0)
    codes = quant_mse(d, b).encode(x.cuda()[None])
    ora = O.mse_encode(P, x.numpy(), diagnostics=True)
    gpu = (_np(codes.codes[0]).view(np.uint32), _np(codes.xnorm[0]), _np(codes.rnorm[0]))
    _mse_compare(d, b, gpu, ora, P.beta)


@pytest.mark.parametrize("d,b,G", [(128, 4, 2), (256, 2, 1), (1536, 3, 1)])
def test_mse_encode_bf16_and_large_d(quant_mse, d, b, G):
    x = synth.kv_keys(G, 1001, d, seed=2)
    codes = quant_mse(d, b, 0, G).encode(x.cuda())
    for g in range(G):
        P = O.MseParams(d, b, g)
        ora = O.mse_encode(P, x[g].to(torch.float64).numpy(), diagnostics=True)
        gpu = (_np(codes.codes[g]).view(np.uint32), _np(codes.xnorm[g]), _np(codes.rnorm[g]))
        _mse_compare(d, b, gpu, ora, P.beta)


@pytest.mark.parametrize("b,G,n,kind", [(4, 3, 1024, "kv"), (2, 8, 384, "kv"), (3, 2, 768, "rows"),
                                        (1, 4, 128, "rows")])
def test_mse_encode_groups(quant_mse, b, G, n, kind):
    """d = 128 (the rotation with the bucketize and packing of whole rows in
    its epilogue), several groups with whole 128-row tiles, bf16 keys and fp32
    rows; every group against the oracle."""
    d = 128
    if kind == "kv":
        x = synth.kv_keys(G, n, d, seed=4)
    else:
        x = synth.gaussian_rows(G * n, d, seed=4).reshape(G, n, d)
    codes = quant_mse(d, b, 0, G).encode(x.cuda())
    for g in range(G):
        P = O.MseParams(d, b, g)
        ora = O.mse_encode(P, x[g].to(torch.float64).numpy(), diagnostics=True)
        gpu = (_np(codes.codes[g]).view(np.uint32), _np(codes.xnorm[g]), _np(codes.rnorm[g]))
        _mse_compare(d, b, gpu, ora, P.beta)


@pytest.mark.parametrize("b,nq", [(4, 64), (2, 3), (1, 5)])
def test_mse_score_and_topk(quant_mse, tq_lib, cuda, b, nq):
    d, n, k = 128, 3000, 10
    x = synth.gaussian_rows(n, d, seed=3)
    q = synth.gaussian_rows(nq, d, seed=4, norm_range=None)
    P = O.MseParams(d, b, 0)
    c, xn, rn = O.mse_encode(P, x.numpy())
    codes = _to_codes(tq_lib, c, xn, rn, cuda)
    tq = quant_mse(d, b)
    s_gpu = _np(tq.score(codes, q.cuda()[None])[0])
    s_ora = O.mse_score(P, c, xn, q.numpy())
    qn = np.linalg.norm(_f64(q), axis=1)
    PT.compare_scores(s_gpu, s_ora, qn, xn.astype(np.float64))
    vals, ids = tq.topk(codes, q.cuda()[None], k)
    PT.compare_topk(_np(vals[0]), _np(ids[0]), s_ora, k, qn, float(xn.max()))


@pytest.mark.parametrize("b", [1, 4])
def test_mse_decode(quant_mse, tq_lib, cuda, b):
    d = 128
    x = synth.gaussian_rows(700, d, seed=6)
    P = O.MseParams(d, b, 0)
    c, xn, rn = O.mse_encode(P, x.numpy())
    ref = O.mse_decode(P, c, xn)
    got = _np(quant_mse(d, b).decode(_to_codes(tq_lib, c, xn, rn, cuda))[0]).astype(np.float64)
    err = np.linalg.norm(got - ref, axis=1) / np.linalg.norm(ref, axis=1)
    assert err.max() <= 1e-4, err.max()


# ---------------------------------------------------------------- decode attention
def _records_on(tq_lib, cuda, recs):
    return tq_lib.Codes(
        torch.stack([torch.from_numpy(r[0].view(np.int32)) for r in recs]).to(cuda),
        torch.stack([torch.from_numpy(r[1]) for r in recs]).to(cuda),
        torch.stack([torch.from_numpy(r[2]) for r in recs]).to(cuda))


def _attention_case(quant, quant_mse, oparams, tq_lib, cuda, G, n, nq, b_k, b_v, seed,
                    groups_checked=None):
    d = 128
    krecs = [synth.random_records(n, b_k * d // 32, seed=seed + g) for g in range(G)]
    vrecs = [synth.random_records(n, b_v * d // 32, seed=seed + 100 + g) for g in range(G)]
    if nq % 4 == 0 and G * nq >= G:
        qs = synth.kv_queries(G * nq, G, d, seed=seed + 200)
    else:
        qs = synth.gaussian_rows(G * nq, d, seed=seed + 200, norm_range=None).reshape(G, nq, d)
    tk, tv = quant(d, b_k, 0, G), quant_mse(d, b_v, 1, G)
    out = _np(tk.attention_decode(_records_on(tq_lib, cuda, krecs), tv,
                                  _records_on(tq_lib, cuda, vrecs), qs.cuda()))
    scale = 1.0 / math.sqrt(d)
    for g in (groups_checked if groups_checked is not None else range(G)):
        kc, kxn, krn = krecs[g]
        vc, vxn, _ = vrecs[g]
        Pk, Pv = oparams(d, b_k, g), O.MseParams(d, b_v, 1 + g)
        ora = O.attention_decode(Pk, kc, kxn, krn, Pv, vc, vxn, _f64(qs[g]), scale)
        vmax = np.abs(O.mse_decode(Pv, vc, vxn)).max()
        err = np.abs(out[g] - ora).max()
        assert err <= 1e-4 * vmax, (g, err, vmax)


@pytest.mark.parametrize("G,n,nq,b_k,b_v", [(2, 3001, 4, 4, 4), (1, 5000, 1, 3, 2),
                                            (3, 257, 8, 2, 3), (1, 1, 4, 4, 4),
                                            (2, 70_000, 4, 4, 4), (1, 600, 2, 1, 1)])
def test_attention_decode(quant, quant_mse, oparams, tq_lib, cuda, G, n, nq, b_k, b_v):
    """Softmax attention over key and value records against the oracle: GQA
    groups of 4 queries, one query, two query passes, a single key, splits
    of many tiles with a ragged last tile, every key and value bit width.
    Bound: |out - oracle| <= 1e-4 max |vhat| (the logits agree to ~1e-6
    relative, the fp32 sums over <= 4096 keys per split to ~1e-6)."""
    _attention_case(quant, quant_mse, oparams, tq_lib, cuda, G, n, nq, b_k, b_v, seed=300)


def test_attention_decode_errors(quant, quant_mse, tq_lib, cuda):
    tk, tv = quant(128, 4), quant_mse(128, 4)
    empty = tq_lib.Codes(torch.zeros(1, 0, 16, dtype=torch.int32, device=cuda),
                         torch.zeros(1, 0, device=cuda), torch.zeros(1, 0, device=cuda))
    q = torch.randn(1, 4, 128, device=cuda)
    with pytest.raises(tq_lib.binding.TQError):
        tk.attention_decode(empty, tv, empty, q)
    one = tq_lib.Codes(torch.zeros(1, 1, 16, dtype=torch.int32, device=cuda),
                       torch.ones(1, 1, device=cuda), torch.zeros(1, 1, device=cuda))
    with pytest.raises(tq_lib.binding.TQError):  # keys must be inner-product records
        tv.attention_decode(one, tv, one, q)


# ---------------------------------------------------------------- sharded search merge
@pytest.mark.parametrize("nshards,k", [(3, 10), (5, 32), (1, 4)])
def test_topk_merge_of_shards(quant, oparams, tq_lib, cuda, nshards, k):
    """tq_topk on uneven shards of one record set, ids made global, merged by
    tq_topk_merge: equal to tq_topk over the whole set (same scores, same
    order) and to the oracle; duplicates straddle a shard cut (tie order)."""
    from kv_cache_embedding_b200 import sharded
    d, b, n, G, nq = 128, 4, 20_011, 2, 4
    recs = [list(synth.random_records(n, b * d // 32, seed=700 + g)) for g in range(G)]
    cut = sharded.shard_bounds(n, nshards, 0)[1]
    for r in recs:
        r[0][cut - 5:cut + 5], r[1][cut - 5:cut + 5], r[2][cut - 5:cut + 5] = r[0][3], r[1][3], r[2][3]
    qs = synth.gaussian_rows(G * nq, d, seed=710, norm_range=None).reshape(G, nq, d)
    tq = quant(d, b, 0, G)
    whole = _records_on(tq_lib, cuda, recs)
    wv, wi = tq.topk(whole, qs.cuda(), k)
    lv, li = [], []
    for sh in range(nshards):
        a, e = sharded.shard_bounds(n, nshards, sh)
        part = tq_lib.Codes(whole.codes[:, a:e].contiguous(), whole.xnorm[:, a:e].contiguous(),
                            whole.rnorm[:, a:e].contiguous())
        v, i = tq.topk(part, qs.cuda(), k)
        lv.append(v.reshape(-1, k))
        li.append((i + a).reshape(-1, k))
    mv, mi = sharded.merge_lists(torch.stack(lv), torch.stack(li), k)
    torch.cuda.synchronize()
    assert torch.equal(mi.reshape(wi.shape), wi) and torch.equal(mv.reshape(wv.shape), wv)
    for g in range(G):
        c, xn, rn = recs[g]
        s_ora = O.score(oparams(d, b, g), c, xn, rn, _f64(qs[g]))
        PT.compare_topk(_np(mv.reshape(wv.shape)[g]), _np(mi.reshape(wi.shape)[g]), s_ora, k,
                        np.linalg.norm(_f64(qs[g]), axis=1), float(xn.max()))


# ---------------------------------------------------------------- scores and top-k in one call
@pytest.mark.parametrize("n", [37888 + 64, 2 * 37888 + 200])
def test_decoded_key_topk_ragged_chunks(quant, oparams, tq_lib, cuda, n):
    """256 queries at d = 512: the decoded keys go through chunks of 37,888 keys
    and the CTA-pair GEMM; the last chunk ends inside a 256-key pair tile (one
    CTA of the pair has no live rows).  Every query's top-10 values equal the
    top-10 of its scores; 4 queries against the oracle."""
    d, b, nq, k = 512, 4, 256, 10
    c, xn, rn = synth.random_records(n, b * d // 32, seed=91)
    q = synth.gaussian_rows(nq, d, seed=92, norm_range=None)
    tq = quant(d, b)
    codes = _to_codes(tq_lib, c, xn, rn, cuda)
    s = tq.score(codes, q.cuda()[None])
    vals, ids = tq.topk(codes, q.cuda()[None], k)
    torch.cuda.synchronize()
    tv, _ = torch.topk(s[0], k, dim=1)
    assert torch.equal(vals[0], tv)
    pick = [0, 1, 127, 255]
    qs = _f64(q[pick])
    s_ora = O.score(oparams(d, b, 0), c, xn, rn, qs)
    qn = np.linalg.norm(qs, axis=1)
    PT.compare_scores(_np(s[0, pick]), s_ora, qn, xn.astype(np.float64))
    PT.compare_topk(_np(vals[0, pick]), _np(ids[0, pick]), s_ora, k, qn, float(xn.max()))


@pytest.mark.parametrize("d,b,G,n,nq", [(128, 4, 2, 5000, 4), (128, 4, 1, 3001, 16),
                                        (256, 4, 1, 2000, 70), (128, 2, 1, 2_200_000, 8),
                                        (128, 3, 3, 777, 1)])
def test_score_topk_equals_separate_calls(quant, oparams, tq_lib, cuda, d, b, G, n, nq):
    """tq_score_topk writes exactly tq_score's estimates and tq_topk's lists
    (SIMT, tensor-core and decoded-key GEMM scoring; beyond 2^24 scores, where
    tq_topk takes its fused path); the oracle checks one group."""
    k = 10
    W = b * d // 32
    recs = [synth.random_records(n, W, seed=800 + g) for g in range(G)]
    qs = synth.gaussian_rows(G * nq, d, seed=810, norm_range=None).reshape(G, nq, d)
    tq = quant(d, b, 0, G)
    codes = _records_on(tq_lib, cuda, recs)
    s1 = tq.score(codes, qs.cuda())
    v1, i1 = tq.topk(codes, qs.cuda(), k)
    s2, (v2, i2) = tq.score_topk(codes, qs.cuda(), k)
    torch.cuda.synchronize()
    assert torch.equal(s1, s2)
    assert torch.equal(i1, i2) and torch.equal(v1, v2)
    if n <= 100_000:
        c, xn, rn = recs[0]
        s_ora = O.score(oparams(d, b, 0), c, xn, rn, _f64(qs[0]))
        qn = np.linalg.norm(_f64(qs[0]), axis=1)
        PT.compare_scores(_np(s2[0]), s_ora, qn, xn.astype(np.float64))
        PT.compare_topk(_np(v2[0]), _np(i2[0]), s_ora, k, qn, float(xn.max()))

