"""ctypes wrapper of the plain C oracle (oracle/tq_oracle.c).

TEST INFRASTRUCTURE ONLY: imported by tests/, by the smoke check and by the
CPU-baseline leg of bench.py.  Nothing in the product package imports it.
Every array crossing this boundary is a numpy array; floating-point inputs
are widened exactly to float64 before the call.
"""
import ctypes as C
import os

import numpy as np

from . import build as _build

_lib = None


def lib():
    global _lib
    if _lib is None:
        path = _build.build()
        L = C.CDLL(path)
        u64, i64, i32 = C.c_uint64, C.c_int64, C.c_int
        P = C.c_void_p
        L.tqo_mix64.restype = u64
        L.tqo_mix64.argtypes = [u64]
        L.tqo_stream_key.restype = u64
        L.tqo_stream_key.argtypes = [u64, u64]
        L.tqo_u64.restype = u64
        L.tqo_u64.argtypes = [u64, u64, u64]
        L.tqo_gaussian.restype = None
        L.tqo_gaussian.argtypes = [u64, u64, i64, P]
        L.tqo_lloyd_max.argtypes = [i32, P, P, P, P]
        L.tqo_codebook.argtypes = [i32, i32, P, P]
        L.tqo_rotation.argtypes = [i32, u64, P, P, P]
        L.tqo_qjl_matrix.argtypes = [i32, u64, P]
        L.tqo_words_per_vector.restype = i64
        L.tqo_words_per_vector.argtypes = [i32, i32]
        L.tqo_encode.argtypes = [i32, i32, P, P, P, P, i64, P, P, P, P, P, P, P]
        L.tqo_unpack.argtypes = [i32, i32, i64, P, P, P]
        L.tqo_decode.argtypes = [i32, i32, P, P, P, i64, P, P, P, P]
        L.tqo_query.argtypes = [i32, P, P, i64, P, P, P]
        L.tqo_score.argtypes = [i32, i32, P, i64, P, P, P, i64, P, P, P]
        L.tqo_topk.argtypes = [i64, i64, P, i32, P, P]
        L.tqo_exact_scores.argtypes = [i32, i64, P, i64, P, P]
        L.tqo_mse_estimate.argtypes = [i32, i32, P, P, P, P, P, P]
        L.tqo_mse_encode.argtypes = [i32, i32, P, P, P, i64, P, P, P, P, P, P]
        L.tqo_mse_score.argtypes = [i32, i32, P, i64, P, P, i64, P, P]
        L.tqo_mse_decode.argtypes = [i32, i32, P, P, i64, P, P, P]
        L.tqo_softmax_weighted_sum.argtypes = [i64, i64, i32, P, P, P]
        L.tqo_split_words_per_vector.restype = i64
        L.tqo_split_words_per_vector.argtypes = [i32, i32]
        L.tqo_split_encode.argtypes = [i32, i32, P, P, P, P, P, P, i64, P, P, P, P, P, P, P]
        L.tqo_split_unpack.argtypes = [i32, i32, i64, P, P, P]
        L.tqo_split_decode.argtypes = [i32, i32, P, P, P, P, i64, P, P, P, P]
        L.tqo_split_score.argtypes = [i32, i32, P, P, i64, P, P, P, i64, P, P, P]
        _lib = L
    return _lib


def _p(a):
    return a.ctypes.data_as(C.c_void_p) if a is not None else None


def _f64(a):
    return np.ascontiguousarray(np.asarray(a, dtype=np.float64))


def _f32(a):
    return np.ascontiguousarray(np.asarray(a, dtype=np.float32))


def _check(rc, what):
    if rc != 0:
        raise ValueError(f"oracle {what} rejected its arguments (rc={rc})")


def mix64(z):
    return int(lib().tqo_mix64(z))


def stream_u64(seed, stream, i):
    return int(lib().tqo_u64(seed, stream, i))


def gaussian(seed, stream, count):
    out = np.empty(count, dtype=np.float64)
    lib().tqo_gaussian(seed, stream, count, _p(out))
    return out


def lloyd_max(levels):
    """Lloyd-Max quantizer of N(0,1): (centroids, boundaries, distortion, iters)."""
    c = np.zeros(max(levels, 1), dtype=np.float64)
    b = np.zeros(max(levels - 1, 1), dtype=np.float64)
    D = np.zeros(1, dtype=np.float64)
    it = np.zeros(1, dtype=np.int32)
    _check(lib().tqo_lloyd_max(levels, _p(c), _p(b), _p(D), _p(it)), "lloyd_max")
    return c[:levels], b[: levels - 1], float(D[0]), int(it[0])


def codebook(d, b):
    """fp32 (centroids, boundaries) at scale 1/sqrt(d) for total bit width b."""
    L = 1 << (b - 1)
    c = np.zeros(max(L, 1), dtype=np.float32)
    beta = np.zeros(max(L - 1, 1), dtype=np.float32)
    _check(lib().tqo_codebook(d, b, _p(c), _p(beta)), "codebook")
    if b == 1:
        return np.zeros(0, np.float32), np.zeros(0, np.float32)
    return c[:L], beta[: L - 1]


def rotation(d, seed, want_double=False):
    """Pi (fp32, row-major) from the QR of the seeded Gaussian matrix.
    With want_double also returns Pi in float64 and |diag R|."""
    pf = np.empty((d, d), dtype=np.float32)
    pd = np.empty((d, d), dtype=np.float64) if want_double else None
    rd = np.empty(d, dtype=np.float64) if want_double else None
    _check(lib().tqo_rotation(d, seed, _p(pd), _p(pf), _p(rd)), "rotation")
    return (pf, pd, rd) if want_double else pf


def qjl_matrix(d, seed):
    S = np.empty((d, d), dtype=np.float32)
    _check(lib().tqo_qjl_matrix(d, seed, _p(S)), "qjl_matrix")
    return S


def words_per_vector(d, b):
    return int(lib().tqo_words_per_vector(d, b))


class Params:
    """The oracle's own parameters for (d, b, seed): codebook, Pi, S."""

    def __init__(self, d, b, seed):
        self.d, self.b, self.seed = d, b, seed
        self.c, self.beta = codebook(d, b)
        self.Pi = rotation(d, seed)
        self.S = qjl_matrix(d, seed)


def encode(params, x, diagnostics=False):
    """Encode rows of x ([n, d], any float dtype, widened exactly to float64).
    Returns codes [n, b*d/32] uint32, xnorm [n] f32, rnorm [n] f32 and, with
    diagnostics, y [n,d], p [n,d] (float64) and idx [n,d] (int32)."""
    d, b = params.d, params.b
    x = _f64(x).reshape(-1, d)
    n = x.shape[0]
    codes = np.empty((n, words_per_vector(d, b)), dtype=np.uint32)
    xn = np.empty(n, dtype=np.float32)
    rn = np.empty(n, dtype=np.float32)
    y = np.empty((n, d), np.float64) if diagnostics else None
    p = np.empty((n, d), np.float64) if diagnostics else None
    idx = np.empty((n, d), np.int32) if diagnostics else None
    c = params.c if params.c.size else np.zeros(1, np.float32)
    beta = params.beta if params.beta.size else np.zeros(1, np.float32)
    _check(lib().tqo_encode(d, b, _p(c), _p(beta), _p(params.Pi), _p(params.S), n, _p(x),
                            _p(codes), _p(xn), _p(rn), _p(y), _p(p), _p(idx)), "encode")
    if diagnostics:
        return codes, xn, rn, y, p, idx
    return codes, xn, rn


def unpack(d, b, codes):
    codes = np.ascontiguousarray(codes, dtype=np.uint32).reshape(-1, words_per_vector(d, b))
    n = codes.shape[0]
    idx = np.empty((n, d), np.int32)
    z = np.empty((n, d), np.int32)
    _check(lib().tqo_unpack(d, b, n, _p(codes), _p(idx), _p(z)), "unpack")
    return idx, z


def decode(params, codes, xnorm, rnorm):
    d, b = params.d, params.b
    codes = np.ascontiguousarray(codes, dtype=np.uint32).reshape(-1, words_per_vector(d, b))
    n = codes.shape[0]
    out = np.empty((n, d), np.float64)
    c = params.c if params.c.size else np.zeros(1, np.float32)
    _check(lib().tqo_decode(d, b, _p(c), _p(params.Pi), _p(params.S), n, _p(codes),
                            _p(_f32(xnorm)), _p(_f32(rnorm)), _p(out)), "decode")
    return out


def query(params, q):
    d = params.d
    q = _f64(q).reshape(-1, d)
    nq = q.shape[0]
    qr = np.empty((nq, d), np.float64)
    u = np.empty((nq, d), np.float64)
    _check(lib().tqo_query(d, _p(params.Pi), _p(params.S), nq, _p(q), _p(qr), _p(u)), "query")
    return qr, u


def score(params, codes, xnorm, rnorm, q):
    """Estimated <q_t, x_v> for every query row t and code record v: [nq, n]."""
    d, b = params.d, params.b
    qr, u = query(params, q)
    codes = np.ascontiguousarray(codes, dtype=np.uint32).reshape(-1, words_per_vector(d, b))
    n = codes.shape[0]
    out = np.empty((qr.shape[0], n), np.float64)
    c = params.c if params.c.size else np.zeros(1, np.float32)
    _check(lib().tqo_score(d, b, _p(c), n, _p(codes), _p(_f32(xnorm)), _p(_f32(rnorm)),
                           qr.shape[0], _p(qr), _p(u), _p(out)), "score")
    return out


def topk(scores, k):
    scores = _f64(scores)
    nq, n = scores.shape
    vals = np.empty((nq, k), np.float64)
    ids = np.empty((nq, k), np.int64)
    _check(lib().tqo_topk(nq, n, _p(scores), k, _p(vals), _p(ids)), "topk")
    return vals, ids


def exact_scores(x, q):
    x = _f64(x)
    q = _f64(q)
    d = x.shape[1]
    out = np.empty((q.shape[0], x.shape[0]), np.float64)
    _check(lib().tqo_exact_scores(d, x.shape[0], _p(x), q.shape[0], _p(q), _p(out)), "exact")
    return out


def mse_estimate(d, bits, seed, x, q):
    """MSE-only TurboQuant estimate of <q, x> with a `bits`-bit Lloyd-Max grid
    and the rotation of `seed` (no QJL)."""
    c, beta = codebook(d, bits + 1)
    Pi = rotation(d, seed)
    est = np.zeros(1, np.float64)
    _check(lib().tqo_mse_estimate(d, bits, _p(c), _p(beta), _p(Pi), _p(_f64(x)), _p(_f64(q)),
                                  _p(est)), "mse_estimate")
    return float(est[0])


# ---------------------------------------------------------------- MSE-only variant
class MseParams:
    """The oracle's parameters of the MSE-only quantizer for (d, b, seed): the
    b-bit Lloyd-Max tables (2^b levels) and Pi (the same Pi as the
    inner-product quantizer of that seed)."""

    def __init__(self, d, b, seed):
        self.d, self.b, self.seed = d, b, seed
        self.c, self.beta = codebook(d, b + 1)
        self.Pi = rotation(d, seed)


def mse_encode(params, x, diagnostics=False):
    """Records of the MSE-only quantizer: codes [n, b*d/32] uint32 (R7 layout,
    index top bit in the z position), xnorm, rnorm; with diagnostics also y
    [n, d] float64 and the full b-bit index [n, d] int32."""
    d, b = params.d, params.b
    x = _f64(x).reshape(-1, d)
    n = x.shape[0]
    codes = np.empty((n, words_per_vector(d, b)), dtype=np.uint32)
    xn = np.empty(n, dtype=np.float32)
    rn = np.empty(n, dtype=np.float32)
    y = np.empty((n, d), np.float64) if diagnostics else None
    idx = np.empty((n, d), np.int32) if diagnostics else None
    _check(lib().tqo_mse_encode(d, b, _p(params.c), _p(params.beta), _p(params.Pi), n, _p(x),
                                _p(codes), _p(xn), _p(rn), _p(y), _p(idx)), "mse_encode")
    if diagnostics:
        return codes, xn, rn, y, idx
    return codes, xn, rn


def mse_score(params, codes, xnorm, q):
    """|x| <Pi q, c[idx]> for every query row and record: [nq, n]."""
    d, b = params.d, params.b
    q = _f64(q).reshape(-1, d)
    qr = (q @ params.Pi.astype(np.float64).T)  # Pi q in double from fp32 Pi
    qr = np.ascontiguousarray(qr)
    codes = np.ascontiguousarray(codes, dtype=np.uint32).reshape(-1, words_per_vector(d, b))
    n = codes.shape[0]
    out = np.empty((q.shape[0], n), np.float64)
    _check(lib().tqo_mse_score(d, b, _p(params.c), n, _p(codes), _p(_f32(xnorm)), q.shape[0],
                               _p(qr), _p(out)), "mse_score")
    return out


def mse_decode(params, codes, xnorm):
    d, b = params.d, params.b
    codes = np.ascontiguousarray(codes, dtype=np.uint32).reshape(-1, words_per_vector(d, b))
    n = codes.shape[0]
    out = np.empty((n, d), np.float64)
    _check(lib().tqo_mse_decode(d, b, _p(params.c), _p(params.Pi), n, _p(codes),
                                _p(_f32(xnorm)), _p(out)), "mse_decode")
    return out


# ---------------------------------------------------------------- decode attention
def softmax_weighted_sum(logits, values):
    """out[t] = sum_j softmax(logits[t])_j values[j] in fp64: [nq, d]."""
    logits = np.ascontiguousarray(_f64(logits)).reshape(-1, np.shape(values)[0])
    values = np.ascontiguousarray(_f64(values))
    nq, n = logits.shape
    d = values.shape[1]
    out = np.empty((nq, d), np.float64)
    _check(lib().tqo_softmax_weighted_sum(nq, n, d, _p(logits), _p(values), _p(out)),
           "softmax_weighted_sum")
    return out


def attention_decode(kparams, kcodes, kxnorm, krnorm, vparams, vcodes, vxnorm, q, scale):
    """Decode attention over quantized keys and values: the logits are scale
    times the inner-product estimates of the key records, the values are the
    MSE-only dequantized rows; returns [nq, d]."""
    logits = score(kparams, kcodes, kxnorm, krnorm, q) * float(scale)
    values = mse_decode(vparams, vcodes, vxnorm)
    return softmax_weighted_sum(logits, values)



# ---------------------------------------------------------------- fractional widths
class SplitParams:
    """The oracle's parameters of the fractional width b - 1/2 for (d, b, seed):
    the first d/2 rotated coordinates on the grid of b total bits (c_hi,
    beta_hi: 2^(b-1) levels), the last d/2 on that of b - 1 (c_lo, beta_lo),
    and the Pi and S of the inner-product quantizer of that seed."""

    def __init__(self, d, b, seed):
        self.d, self.b, self.seed = d, b, seed
        self.c_hi, self.beta_hi = codebook(d, b)
        self.c_lo, self.beta_lo = codebook(d, b - 1)
        self.Pi = rotation(d, seed)
        self.S = qjl_matrix(d, seed)


def split_words_per_vector(d, b):
    return int(lib().tqo_split_words_per_vector(d, b))


def _tab(a):
    return a if a.size else np.zeros(1, np.float32)


def split_encode(params, x, diagnostics=False):
    """Records of the fractional width: codes [n, d/64 (2b - 1)] uint32, xnorm,
    rnorm; with diagnostics also y, p [n, d] float64 and idx [n, d] int32."""
    d, b = params.d, params.b
    x = _f64(x).reshape(-1, d)
    n = x.shape[0]
    codes = np.empty((n, split_words_per_vector(d, b)), dtype=np.uint32)
    xn = np.empty(n, dtype=np.float32)
    rn = np.empty(n, dtype=np.float32)
    y = np.empty((n, d), np.float64) if diagnostics else None
    p = np.empty((n, d), np.float64) if diagnostics else None
    idx = np.empty((n, d), np.int32) if diagnostics else None
    _check(lib().tqo_split_encode(d, b, _p(_tab(params.c_hi)), _p(_tab(params.beta_hi)),
                                  _p(_tab(params.c_lo)), _p(_tab(params.beta_lo)), _p(params.Pi),
                                  _p(params.S), n, _p(x), _p(codes), _p(xn), _p(rn), _p(y),
                                  _p(p), _p(idx)), "split_encode")
    if diagnostics:
        return codes, xn, rn, y, p, idx
    return codes, xn, rn


def split_unpack(d, b, codes):
    codes = np.ascontiguousarray(codes, dtype=np.uint32).reshape(-1, split_words_per_vector(d, b))
    n = codes.shape[0]
    idx = np.empty((n, d), np.int32)
    z = np.empty((n, d), np.int32)
    _check(lib().tqo_split_unpack(d, b, n, _p(codes), _p(idx), _p(z)), "split_unpack")
    return idx, z


def split_decode(params, codes, xnorm, rnorm):
    d, b = params.d, params.b
    codes = np.ascontiguousarray(codes, dtype=np.uint32).reshape(-1, split_words_per_vector(d, b))
    n = codes.shape[0]
    out = np.empty((n, d), np.float64)
    _check(lib().tqo_split_decode(d, b, _p(_tab(params.c_hi)), _p(_tab(params.c_lo)),
                                  _p(params.Pi), _p(params.S), n, _p(codes), _p(_f32(xnorm)),
                                  _p(_f32(rnorm)), _p(out)), "split_decode")
    return out


def split_score(params, codes, xnorm, rnorm, q):
    """Estimated <q_t, x_v> from split records: [nq, n]."""
    d, b = params.d, params.b
    qr, u = query(params, q)
    codes = np.ascontiguousarray(codes, dtype=np.uint32).reshape(-1, split_words_per_vector(d, b))
    n = codes.shape[0]
    out = np.empty((qr.shape[0], n), np.float64)
    _check(lib().tqo_split_score(d, b, _p(_tab(params.c_hi)), _p(_tab(params.c_lo)), n,
                                 _p(codes), _p(_f32(xnorm)), _p(_f32(rnorm)), qr.shape[0],
                                 _p(qr), _p(u), _p(out)), "split_score")
    return out
