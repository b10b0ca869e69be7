"""tq_topk_noalloc: the top-k entry point for callers that cannot allocate
device memory (serving engines that own every byte through their own pool,
plugins without access to the host runtime's allocator, paths where an
allocation could stall on device synchronisation).  Its scratch lives in a
fixed 8 MiB array inside libtq instead of a caller workspace.

Checked through the C ABI against tq_topk (which takes a workspace) on two
calls in a row with different queries and k, so that the second call runs on
scratch the first call left behind.  This file is collected last on purpose.
"""
import ctypes

import numpy as np
import pytest
import torch

import synth

pytestmark = pytest.mark.gpu


def _topk_with_workspace(B, tq, codes, q, k):
    G, nq = q.shape[0], q.shape[1]
    vals = torch.empty(G, nq, k, dtype=torch.float32, device=q.device)
    ids = torch.empty(G, nq, k, dtype=torch.int64, device=q.device)
    nbytes = B.tq_workspace_bytes(B.TQ_OP_TOPK, tq.d, tq.b, G, codes.n, nq, k)
    ws = torch.empty(nbytes, dtype=torch.uint8, device=q.device)
    B.tq_topk(tq.cb, tq.Pi.data_ptr(), tq.S.data_ptr(), G, codes.n, codes.codes.data_ptr(),
              codes.xnorm.data_ptr(), codes.rnorm.data_ptr(), nq, q.data_ptr(), B.TQ_BF16, k,
              vals.data_ptr(), ids.data_ptr(), ws.data_ptr(), nbytes,
              torch.cuda.current_stream().cuda_stream)
    return vals, ids


def _topk_noalloc(B, tq, codes, q, k):
    G, nq = q.shape[0], q.shape[1]
    vals = torch.empty(G, nq, k, dtype=torch.float32, device=q.device)
    ids = torch.empty(G, nq, k, dtype=torch.int64, device=q.device)
    B.tq_topk_noalloc(tq.cb, tq.Pi.data_ptr(), tq.S.data_ptr(), G, codes.n,
                      codes.codes.data_ptr(), codes.xnorm.data_ptr(), codes.rnorm.data_ptr(), nq,
                      q.data_ptr(), B.TQ_BF16, k, vals.data_ptr(), ids.data_ptr(),
                      torch.cuda.current_stream().cuda_stream)
    return vals, ids


def _same(ref, got, q, xmax):
    rv, ri = (t.cpu().numpy() for t in ref)
    gv, gi = (t.cpu().numpy() for t in got)
    qn = np.linalg.norm(q.float().cpu().numpy(), axis=2)  # [G, nq]
    tol = 1e-4 * qn[:, :, None] * xmax
    assert np.all(np.abs(gv - rv) <= tol)
    np.testing.assert_array_equal(np.sort(gi, axis=2), np.sort(ri, axis=2))


def test_noalloc_topk_matches_workspace_topk_twice(cuda, tq_lib):
    B = tq_lib.binding
    G, n, d, b = 2, 5000, 128, 4
    tq = tq_lib.TurboQuant(d, b, seed=0, groups=G, device=cuda)
    keys = synth.kv_keys(G, n, d, seed=31, device=cuda)
    codes = tq.encode(keys)
    xmax = float(codes.xnorm.max())
    q1 = synth.kv_queries(4 * G, G, d, seed=32, device=cuda, key_seed=31)
    q2 = synth.kv_queries(3 * G, G, d, seed=33, device=cuda, key_seed=31)

    got1 = _topk_noalloc(B, tq, codes, q1, 10)
    got2 = _topk_noalloc(B, tq, codes, q2, 7)
    ref1 = _topk_with_workspace(B, tq, codes, q1, 10)
    ref2 = _topk_with_workspace(B, tq, codes, q2, 7)
    torch.cuda.synchronize()
    _same(ref1, got1, q1, xmax)
    _same(ref2, got2, q2, xmax)


def test_noalloc_topk_takes_the_second_form_when_scores_do_not_fit(cuda, tq_lib):
    """8 KV heads x 4 query heads x 131072 tokens: the full score matrix (16 MiB)
    does not fit the array, so the call takes the form tq_topk uses beyond
    2^24 scores (key chunks sized to the array).  Two calls in a row, against
    tq_topk with a workspace (which keeps the full score matrix)."""
    B = tq_lib.binding
    G, n, d, b = 8, 131072, 128, 4
    assert (B.tq_workspace_bytes(B.TQ_OP_TOPK, d, b, G, n, 4, 10) >
            B.TQ_NOALLOC_SCRATCH_BYTES)
    tq = tq_lib.TurboQuant(d, b, seed=0, groups=G, device=cuda)
    codes = tq.encode(synth.kv_keys(G, n, d, seed=34, device=cuda))
    xmax = float(codes.xnorm.max())
    q1 = synth.kv_queries(4 * G, G, d, seed=35, device=cuda, key_seed=34)
    q2 = synth.kv_queries(4 * G, G, d, seed=36, device=cuda, key_seed=34)
    got1 = _topk_noalloc(B, tq, codes, q1, 10)
    got2 = _topk_noalloc(B, tq, codes, q2, 5)
    ref1 = _topk_with_workspace(B, tq, codes, q1, 10)
    ref2 = _topk_with_workspace(B, tq, codes, q2, 5)
    torch.cuda.synchronize()
    _same(ref1, got1, q1, xmax)
    _same(ref2, got2, q2, xmax)


def test_noalloc_topk_rejects_sizes_beyond_its_scratch(cuda, tq_lib):
    B = tq_lib.binding
    tq = tq_lib.TurboQuant(128, 4, seed=0, groups=1, device=cuda)
    n, nq, k, d = 1000, 8200, 10, 128
    # every form of the scratch holds the queries' two fp32 transforms, which
    # alone exceed the array: the decision cannot depend on layout details
    assert 2 * nq * d * 4 > B.TQ_NOALLOC_SCRATCH_BYTES
    # sizes alone decide: the call returns before touching any pointer
    rc = B.lib.tq_topk_noalloc(ctypes.byref(tq.cb), tq.Pi.data_ptr(), tq.S.data_ptr(), 1, n, 1, 1,
                               1, nq, 1, B.TQ_BF16, k, 1, 1, None)
    assert rc == B.TQ_ERR_SCRATCH_LIMIT
    assert "8 MiB" in B.tq_status_str(rc)
