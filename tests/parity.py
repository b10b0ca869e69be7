"""Helpers of the parity tests: an independent reader of the code layout and
the comparison rules between the CUDA path and the oracle.

Comparison rules (tolerances fixed here, explained in the docstrings):
  * cell indices: bit-exact, except coordinates whose rotated value (oracle,
    fp64) lies within 1e-5*sigma of a Lloyd-Max boundary; those are counted
    and must stay <= 1e-4 of all coordinates;
  * sign bits and |r|: compared on records whose indices all agree; sign
    bits may differ only where |(S r)_i| < 1e-5 |r| (oracle, fp64), counted
    under the same 1e-4 bound;
  * |x|: relative error <= 1e-4; |r|: relative error <= 1e-4;
  * scores on identical records: |s_gpu - s_oracle| <= 1e-4 |q| |x|;
  * top-k: identical id lists for every query whose oracle gap between
    ranks k and k+1 exceeds 1e-5 |q| max|x|.
"""
import math

import numpy as np

BAND = 1e-5
FLAG_FRACTION = 1e-4
NORM_RTOL = 1e-4
SCORE_TOL = 1e-4


def read_layout(d, b, codes):
    """Cell indices and sign bits from packed records (numpy, written from the
    documented layout, independent of the oracle's unpacker)."""
    codes = np.ascontiguousarray(np.asarray(codes)).view(np.uint32).reshape(-1, b * d // 32)
    n = codes.shape[0]
    k = b - 1
    words = codes.reshape(n, d // 32, b)
    bits = np.unpackbits(words.view(np.uint8).reshape(n, d // 32, b * 4), axis=2,
                         bitorder="little")
    idx = np.zeros((n, d), np.int64)
    z = np.zeros((n, d), np.int64)
    for j in range(32):
        if b in (1, 2, 4):
            base = b * j
            for t in range(k):
                idx[:, j::32] += bits[:, :, base + t].astype(np.int64) << t
            z[:, j::32] = bits[:, :, base + k]
        else:
            for t in range(2):
                idx[:, j::32] += bits[:, :, 2 * j + t].astype(np.int64) << t
            z[:, j::32] = bits[:, :, 64 + j]
    return idx, z


class EncodeReport(dict):
    pass


def compare_encode(d, b, beta, gpu, ora, check=True, bound_flags=True):
    """gpu = (codes, xnorm, rnorm) numpy; ora = oracle.encode(..., diagnostics=True).
    Returns a report; with check, asserts the parity rules.  bound_flags=False
    drops the 1e-4 bound on the flagged fraction (for crafted inputs such as a
    zero vector, whose coordinates all sit on the middle boundary)."""
    g_codes = gpu[0]
    o_codes, y, o_idx = ora[0], ora[3], ora[5]
    g_idx, g_z = read_layout(d, b, g_codes)
    o_idx2, o_z = read_layout(d, b, o_codes)
    assert np.array_equal(o_idx2, o_idx)
    return _compare_fields(d, gpu, ora, g_idx, g_z, o_z, _near_boundary(d, y, beta), check,
                           bound_flags)


def _near_boundary(d, y, beta):
    """Coordinates whose rotated value lies within BAND sigma of a boundary."""
    if not beta.size:
        return np.zeros_like(y, dtype=bool)
    dist = np.min(np.abs(y[:, :, None] - beta.astype(np.float64)[None, None, :]), axis=2)
    return dist < BAND / math.sqrt(d)


def compare_encode_split(d, b, beta_hi, beta_lo, gpu, ora, check=True, bound_flags=True):
    """Records of the fractional width b - 1/2: the first d/64 blocks are the
    first d/2 coordinates in the b-bit layout, the rest the last d/2 in the
    (b-1)-bit layout; each half is read with read_layout and flagged against
    its own boundaries, then the rules of compare_encode apply."""
    h = d // 64
    g_codes = np.ascontiguousarray(np.asarray(gpu[0])).view(np.uint32).reshape(-1, h * (2 * b - 1))
    o_codes, y, o_idx = ora[0], ora[3], ora[5]
    gi_hi, gz_hi = read_layout(d // 2, b, np.ascontiguousarray(g_codes[:, :h * b]))
    gi_lo, gz_lo = read_layout(d // 2, b - 1, np.ascontiguousarray(g_codes[:, h * b:]))
    oi_hi, oz_hi = read_layout(d // 2, b, np.ascontiguousarray(o_codes[:, :h * b]))
    oi_lo, oz_lo = read_layout(d // 2, b - 1, np.ascontiguousarray(o_codes[:, h * b:]))
    assert np.array_equal(np.concatenate([oi_hi, oi_lo], 1), o_idx)
    flag = np.concatenate([_near_boundary(d, y[:, :d // 2], beta_hi),
                           _near_boundary(d, y[:, d // 2:], beta_lo)], 1)
    return _compare_fields(d, (g_codes, gpu[1], gpu[2]), ora, np.concatenate([gi_hi, gi_lo], 1),
                           np.concatenate([gz_hi, gz_lo], 1), np.concatenate([oz_hi, oz_lo], 1),
                           flag, check, bound_flags)


def _compare_fields(d, gpu, ora, g_idx, g_z, o_z, flag_idx, check, bound_flags):
    g_codes, g_xn, g_rn = gpu
    o_codes, o_xn, o_rn, y, p, o_idx = ora
    n = o_codes.shape[0]
    rep = EncodeReport(n=n, coords=n * d)
    idx_diff = g_idx != o_idx
    rep["idx_flagged"] = int(flag_idx.sum())
    rep["idx_mismatch"] = int(idx_diff.sum())
    rep["idx_mismatch_unflagged"] = int((idx_diff & ~flag_idx).sum())
    same_rec = ~idx_diff.any(axis=1)
    rnorm_d = o_rn.astype(np.float64)
    flag_z = np.abs(p) < BAND * rnorm_d[:, None]
    z_diff = (g_z != o_z) & same_rec[:, None]
    rep["z_flagged"] = int(flag_z.sum())
    rep["z_mismatch"] = int(z_diff.sum())
    rep["z_mismatch_unflagged"] = int((z_diff & ~flag_z).sum())
    rep["records_exempt"] = int((~same_rec).sum())
    xn_err = np.abs(g_xn.astype(np.float64) - o_xn) / np.maximum(o_xn, 1e-30)
    xn_err[o_xn == 0] = np.abs(g_xn[o_xn == 0])
    rep["xnorm_max_rel"] = float(xn_err.max()) if n else 0.0
    rn_err = np.abs(g_rn.astype(np.float64) - o_rn) / np.maximum(o_rn, 1e-30)
    rn_err[o_rn == 0] = np.abs(g_rn[o_rn == 0])
    rn_err = rn_err[same_rec]
    rep["rnorm_max_rel"] = float(rn_err.max()) if rn_err.size else 0.0
    rep["codes_identical_fraction"] = float((g_codes.view(np.uint32) == o_codes).all(1).mean()) if n else 1.0
    if check:
        assert rep["idx_mismatch_unflagged"] == 0, rep
        assert rep["z_mismatch_unflagged"] == 0, rep
        if bound_flags:
            assert rep["idx_flagged"] <= FLAG_FRACTION * rep["coords"] + 1, rep
            assert rep["z_flagged"] <= FLAG_FRACTION * rep["coords"] + 1, rep
        assert rep["xnorm_max_rel"] <= NORM_RTOL, rep
        assert rep["rnorm_max_rel"] <= NORM_RTOL, rep
    return rep


def compare_scores(s_gpu, s_ora, qnorm, xnorm, check=True):
    """s_*: [nq, n]; tolerance 1e-4 |q| |x| per element."""
    tol = SCORE_TOL * np.outer(qnorm, xnorm) + 1e-30
    err = np.abs(s_gpu.astype(np.float64) - s_ora)
    ratio = float((err / tol).max()) if err.size else 0.0
    big = np.abs(s_ora) > 0.1 * np.outer(qnorm, xnorm)
    rel = float((err[big] / np.abs(s_ora[big])).max()) if big.any() else 0.0
    if check:
        assert ratio <= 1.0, (ratio, rel)
    return {"max_err_over_tol": ratio, "max_rel_err_large": rel}


def compare_topk(g_vals, g_ids, o_scores, k, qnorm, xmax, check=True):
    """o_scores [nq, n] oracle scores; g_* [nq, k]."""
    nq, n = o_scores.shape
    ties = 0
    for t in range(nq):
        order = np.lexsort((np.arange(n), -o_scores[t]))
        top = order[:k]
        gap = (o_scores[t, order[k - 1]] - o_scores[t, order[k]]) if n > k else np.inf
        if gap <= 1e-5 * qnorm[t] * xmax:
            ties += 1
            continue
        if check:
            np.testing.assert_array_equal(np.sort(g_ids[t]), np.sort(top))
            np.testing.assert_allclose(g_vals[t], o_scores[t, g_ids[t]],
                                       atol=SCORE_TOL * qnorm[t] * xmax, rtol=0)
            assert np.all(np.diff(g_vals[t]) <= 0)
    return {"near_tie_queries": ties}
