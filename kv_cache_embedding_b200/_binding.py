"""ctypes binding of libtq.so: one Python function per C entry point, same
names, arguments marshalled as plain integers (device pointers), sizes and
the stream handle.  No computation happens here.

The library must be built (``python kv_cache_embedding_b200/build.py``);
importing this module without it raises, there is no fallback.
"""
import ctypes as C
import os

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libtq.so")

TQ_OK = 0
TQ_ERR_ARG = -1
TQ_ERR_UNSUPPORTED = -2
TQ_ERR_WORKSPACE = -3
TQ_ERR_CUDA = -4
TQ_ERR_DEVICE_TIMEOUT = -5
TQ_ERR_MISMATCH = -6
TQ_ERR_SCRATCH_LIMIT = -7
TQ_NOALLOC_SCRATCH_BYTES = 8 << 20

TQ_F32 = 0
TQ_BF16 = 1
TQ_VARIANT_PROD = 0
TQ_VARIANT_MSE = 1

(TQ_OP_BUILD, TQ_OP_ENCODE, TQ_OP_SCORE, TQ_OP_TOPK, TQ_OP_DECODE, TQ_OP_EXACT,
 TQ_OP_ATTENTION, TQ_OP_SCORE_TOPK) = range(8)

EXPORTS = ("tq_workspace_bytes", "tq_status_str", "tq_build_codebook", "tq_build_codebook_mse",
           "tq_build_codebook_split",
           "tq_encode", "tq_score",
           "tq_topk", "tq_decode", "tq_logits_fp32", "tq_exact_topk", "tq_topk_noalloc",
           "tq_device_status", "tq_selftest_wait_timeout", "tq_attention_decode",
           "tq_topk_merge", "tq_score_topk")


class tq_codebook_t(C.Structure):
    _fields_ = [
        ("d", C.c_int32),
        ("b", C.c_int32),
        ("levels", C.c_int32),
        ("groups", C.c_int32),
        ("seed", C.c_uint64),
        ("centroids", C.c_float * 16),
        ("boundaries", C.c_float * 16),
        ("distortion", C.c_double),
        ("variant", C.c_int32),
        ("reserved", C.c_int32),
        ("split", C.c_int32),
        ("levels_lo", C.c_int32),
        ("centroids_lo", C.c_float * 16),
        ("boundaries_lo", C.c_float * 16),
    ]


class TQError(RuntimeError):
    def __init__(self, fn, status):
        super().__init__(f"{fn} failed: {status} ({tq_status_str(status)})")
        self.status = status


def _load():
    if not os.path.exists(LIB_PATH):
        raise ImportError(
            f"libtq.so not built at {LIB_PATH}; run `python kv_cache_embedding_b200/build.py`")
    L = C.CDLL(LIB_PATH)
    P, i32, i64, u64, sz = C.c_void_p, C.c_int, C.c_int64, C.c_uint64, C.c_size_t
    cbp = C.POINTER(tq_codebook_t)
    L.tq_workspace_bytes.restype = sz
    L.tq_workspace_bytes.argtypes = [i32, i32, i32, i32, i64, i32, i32]
    L.tq_status_str.restype = C.c_char_p
    L.tq_status_str.argtypes = [i32]
    L.tq_build_codebook.restype = i32
    L.tq_build_codebook.argtypes = [i32, i32, u64, i32, cbp, P, P, P, sz, P]
    L.tq_build_codebook_mse.restype = i32
    L.tq_build_codebook_mse.argtypes = [i32, i32, u64, i32, cbp, P, P, sz, P]
    L.tq_build_codebook_split.restype = i32
    L.tq_build_codebook_split.argtypes = [i32, i32, u64, i32, cbp, P, P, P, sz, P]
    L.tq_encode.restype = i32
    L.tq_encode.argtypes = [cbp, P, P, i32, i64, P, i32, P, P, P, P, sz, P]
    L.tq_score.restype = i32
    L.tq_score.argtypes = [cbp, P, P, i32, i64, P, P, P, i32, P, i32, P, P, sz, P]
    L.tq_topk.restype = i32
    L.tq_topk.argtypes = [cbp, P, P, i32, i64, P, P, P, i32, P, i32, i32, P, P, P, sz, P]
    L.tq_topk_noalloc.restype = i32
    L.tq_topk_noalloc.argtypes = [cbp, P, P, i32, i64, P, P, P, i32, P, i32, i32, P, P, P]
    L.tq_device_status.restype = i32
    L.tq_device_status.argtypes = [P, P]
    L.tq_selftest_wait_timeout.restype = i32
    L.tq_selftest_wait_timeout.argtypes = [P, u64, P]
    L.tq_decode.restype = i32
    L.tq_decode.argtypes = [cbp, P, P, i32, i64, P, P, P, P, P, sz, P]
    L.tq_logits_fp32.restype = i32
    L.tq_logits_fp32.argtypes = [i32, i32, i64, P, i32, P, i32, P, P]
    L.tq_exact_topk.restype = i32
    L.tq_exact_topk.argtypes = [i32, i32, i64, P, i32, P, i32, i32, P, P, P, sz, P]
    L.tq_score_topk.restype = i32
    L.tq_score_topk.argtypes = [cbp, P, P, i32, i64, P, P, P, i32, P, i32, i32, P, P, P, P, sz, P]
    L.tq_topk_merge.restype = i32
    L.tq_topk_merge.argtypes = [i64, i32, i32, P, P, P, P, P]
    L.tq_attention_decode.restype = i32
    L.tq_attention_decode.argtypes = [cbp, P, P, cbp, P, i32, i64, P, P, P, P, P, i32, P, i32,
                                      C.c_float, P, P, sz, P]
    return L


lib = _load()


def tq_status_str(status):
    return lib.tq_status_str(status).decode()


def tq_workspace_bytes(op, d, b, G, n, nq, k):
    return int(lib.tq_workspace_bytes(op, d, b, G, n, nq, k))


def _ok(fn, status):
    if status != TQ_OK:
        raise TQError(fn, status)
    return status


def tq_build_codebook(d, b, seed, G, cb, d_Pi, d_S, d_ws, ws_bytes, stream):
    return _ok("tq_build_codebook",
               lib.tq_build_codebook(d, b, seed, G, C.byref(cb), d_Pi, d_S, d_ws, ws_bytes, stream))


def tq_build_codebook_mse(d, b, seed, G, cb, d_Pi, d_ws, ws_bytes, stream):
    return _ok("tq_build_codebook_mse",
               lib.tq_build_codebook_mse(d, b, seed, G, C.byref(cb), d_Pi, d_ws, ws_bytes, stream))


def tq_build_codebook_split(d, b, seed, G, cb, d_Pi, d_S, d_ws, ws_bytes, stream):
    return _ok("tq_build_codebook_split",
               lib.tq_build_codebook_split(d, b, seed, G, C.byref(cb), d_Pi, d_S, d_ws, ws_bytes,
                                           stream))


def tq_encode(cb, d_Pi, d_S, G, n, d_x, x_dtype, d_codes, d_xnorm, d_rnorm, d_ws, ws_bytes,
              stream):
    return _ok("tq_encode", lib.tq_encode(C.byref(cb), d_Pi, d_S, G, n, d_x, x_dtype, d_codes,
                                          d_xnorm, d_rnorm, d_ws, ws_bytes, stream))


def tq_device_status(d_ws, stream):
    """Status word the last tq_encode / tq_score / tq_topk left in d_ws
    (synchronises the stream)."""
    return lib.tq_device_status(d_ws, stream)


def tq_selftest_wait_timeout(d_ws, limit_ns, stream):
    return _ok("tq_selftest_wait_timeout", lib.tq_selftest_wait_timeout(d_ws, limit_ns, stream))


def tq_score(cb, d_Pi, d_S, G, n, d_codes, d_xnorm, d_rnorm, nq, d_q, q_dtype, d_scores, d_ws,
             ws_bytes, stream):
    return _ok("tq_score", lib.tq_score(C.byref(cb), d_Pi, d_S, G, n, d_codes, d_xnorm, d_rnorm,
                                        nq, d_q, q_dtype, d_scores, d_ws, ws_bytes, stream))


def tq_topk(cb, d_Pi, d_S, G, n, d_codes, d_xnorm, d_rnorm, nq, d_q, q_dtype, k, d_vals, d_ids,
            d_ws, ws_bytes, stream):
    return _ok("tq_topk", lib.tq_topk(C.byref(cb), d_Pi, d_S, G, n, d_codes, d_xnorm, d_rnorm,
                                      nq, d_q, q_dtype, k, d_vals, d_ids, d_ws, ws_bytes, stream))


def tq_topk_noalloc(cb, d_Pi, d_S, G, n, d_codes, d_xnorm, d_rnorm, nq, d_q, q_dtype, k, d_vals,
                    d_ids, stream):
    """tq_topk with its scratch in the library's fixed device array (no
    workspace argument, nothing allocated); see include/tq.h."""
    return _ok("tq_topk_noalloc", lib.tq_topk_noalloc(C.byref(cb), d_Pi, d_S, G, n, d_codes,
                                                      d_xnorm, d_rnorm, nq, d_q, q_dtype, k,
                                                      d_vals, d_ids, stream))


def tq_decode(cb, d_Pi, d_S, G, n, d_codes, d_xnorm, d_rnorm, d_xhat, d_ws, ws_bytes, stream):
    return _ok("tq_decode", lib.tq_decode(C.byref(cb), d_Pi, d_S, G, n, d_codes, d_xnorm,
                                          d_rnorm, d_xhat, d_ws, ws_bytes, stream))


def tq_logits_fp32(d, G, n, d_keys, nq, d_q, q_dtype, d_out, stream):
    return _ok("tq_logits_fp32", lib.tq_logits_fp32(d, G, n, d_keys, nq, d_q, q_dtype, d_out,
                                                    stream))


def tq_exact_topk(d, G, n, d_x, nq, d_q, q_dtype, k, d_vals, d_ids, d_ws, ws_bytes, stream):
    return _ok("tq_exact_topk", lib.tq_exact_topk(d, G, n, d_x, nq, d_q, q_dtype, k, d_vals,
                                                  d_ids, d_ws, ws_bytes, stream))


def tq_attention_decode(cb_k, d_Pi_k, d_S_k, cb_v, d_Pi_v, G, n, d_kcodes, d_kxnorm, d_krnorm,
                        d_vcodes, d_vxnorm, nq, d_q, q_dtype, scale, d_out, d_ws, ws_bytes,
                        stream):
    return _ok("tq_attention_decode",
               lib.tq_attention_decode(C.byref(cb_k), d_Pi_k, d_S_k, C.byref(cb_v), d_Pi_v, G, n,
                                       d_kcodes, d_kxnorm, d_krnorm, d_vcodes, d_vxnorm, nq, d_q,
                                       q_dtype, scale, d_out, d_ws, ws_bytes, stream))


def tq_topk_merge(rows, nlists, k, d_vals, d_ids, d_out_vals, d_out_ids, stream):
    return _ok("tq_topk_merge", lib.tq_topk_merge(rows, nlists, k, d_vals, d_ids, d_out_vals,
                                                  d_out_ids, stream))


def tq_score_topk(cb, d_Pi, d_S, G, n, d_codes, d_xnorm, d_rnorm, nq, d_q, q_dtype, k, d_scores,
                  d_vals, d_ids, d_ws, ws_bytes, stream):
    return _ok("tq_score_topk",
               lib.tq_score_topk(C.byref(cb), d_Pi, d_S, G, n, d_codes, d_xnorm, d_rnorm, nq, d_q,
                                 q_dtype, k, d_scores, d_vals, d_ids, d_ws, ws_bytes, stream))

