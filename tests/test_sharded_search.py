"""Search over a database sharded across ranks, on CPU: two and three gloo
ranks (one process each, as torchrun starts them) hold contiguous shards of
one seeded record set, take their local top-k (the oracle's, in place of
tq_topk), make the ids global, all-gather the lists through the package's
gather_lists and merge them.  The merged lists must equal the oracle's top-k
over the whole record set, ties included (value desc, id asc)."""
import datetime
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as td
import torch.multiprocessing as mp

D, B, N, NQ, K = 128, 4, 3001, 3, 10


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _database():
    import synth
    from oracle import oracle as O
    codes, xn, rn = synth.random_records(N, B * D // 32, seed=90)
    # exact duplicates of one record across the shard cut exercise the id order
    codes[1490:1510] = codes[7]
    xn[1490:1510], rn[1490:1510] = xn[7], rn[7]
    q = synth.gaussian_rows(NQ, D, seed=91, norm_range=None).numpy().astype(np.float64)
    P = O.Params(D, B, 0)
    return P, codes, xn, rn, q


def _merge_lists(vals, ids, k):
    """Best k of [nlists, rows, k] lists by (value desc, id asc)."""
    nl, rows, _ = vals.shape
    out_v = np.empty((rows, k))
    out_i = np.empty((rows, k), dtype=np.int64)
    for r in range(rows):
        v = vals[:, r, :].reshape(-1)
        i = ids[:, r, :].reshape(-1)
        order = np.lexsort((i, -v))[:k]
        out_v[r], out_i[r] = v[order], i[order]
    return out_v, out_i


def _rank_main(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world))
    from kv_cache_embedding_b200 import sharded
    from oracle import oracle as O
    td.init_process_group("gloo", rank=rank, world_size=world,
                          timeout=datetime.timedelta(seconds=60))
    try:
        P, codes, xn, rn, q = _database()
        start, stop = sharded.shard_bounds(N, world, rank)
        s = O.score(P, codes[start:stop], xn[start:stop], rn[start:stop], q)
        v, i = O.topk(s, K)
        gv, gi = sharded.gather_lists(torch.from_numpy(v), torch.from_numpy(i + start))
        out[rank] = _merge_lists(gv.numpy(), gi.numpy(), K)
    finally:
        td.destroy_process_group()


def _rank_main_sharded_topk(rank, world, port, out):
    """sharded_topk itself: the oracle's top-k of this rank's shard in place of
    tq_topk, and a numpy merge in place of tq_topk_merge (both take and return
    torch tensors, as the library calls do); the id offsets, the all-gather
    and the layouts are the package's."""
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world))
    from kv_cache_embedding_b200 import sharded
    from oracle import oracle as O
    td.init_process_group("gloo", rank=rank, world_size=world,
                          timeout=datetime.timedelta(seconds=60))
    try:
        P, codes, xn, rn, q = _database()
        start, stop = sharded.shard_bounds(N, world, rank)

        def local_topk(shard, qq, k):
            c, x, r = shard
            v, i = O.topk(O.score(P, c, x, r, qq[0].numpy()), k)
            return torch.from_numpy(v)[None], torch.from_numpy(i)[None]

        def merge(gv, gi, k):
            v, i = _merge_lists(gv.numpy(), gi.numpy(), k)
            return torch.from_numpy(v), torch.from_numpy(i)

        shard = (codes[start:stop], xn[start:stop], rn[start:stop])
        mv, mi = sharded.sharded_topk(None, shard, torch.from_numpy(q)[None], K, N,
                                      local_topk=local_topk, merge=merge)
        assert mv.shape == (1, NQ, K) and mi.shape == (1, NQ, K)
        out[rank] = (mv[0].numpy(), mi[0].numpy())
    finally:
        td.destroy_process_group()


@pytest.mark.parametrize("world", [2, 3])
def test_sharded_topk_function_equals_whole_database(world):
    """sharded.sharded_topk (the call bench.py makes for the search at N > 1)
    over gloo ranks equals the oracle's top-k over the whole database."""
    from oracle import oracle as O
    port = _free_port()
    out = mp.Manager().dict()
    mp.spawn(_rank_main_sharded_topk, args=(world, port, out), nprocs=world, join=True)
    P, codes, xn, rn, q = _database()
    ev, ei = O.topk(O.score(P, codes, xn, rn, q), K)
    for rank in range(world):
        mv, mi = out[rank]
        np.testing.assert_array_equal(mi, ei)
        np.testing.assert_array_equal(mv, ev)


@pytest.mark.parametrize("world", [2, 3])
def test_sharded_topk_equals_whole_database(world):
    from oracle import oracle as O
    port = _free_port()
    out = mp.Manager().dict()
    mp.spawn(_rank_main, args=(world, port, out), nprocs=world, join=True)
    P, codes, xn, rn, q = _database()
    ev, ei = O.topk(O.score(P, codes, xn, rn, q), K)
    for rank in range(world):
        mv, mi = out[rank]
        np.testing.assert_array_equal(mi, ei)
        np.testing.assert_array_equal(mv, ev)


def test_shard_bounds_cover_the_database():
    from kv_cache_embedding_b200.sharded import shard_bounds
    for n, world in [(10, 3), (7, 7), (5, 8), (1_000_000, 6)]:
        spans = [shard_bounds(n, world, r) for r in range(world)]
        assert spans[0][0] == 0 and spans[-1][1] == n
        assert all(a[1] == b[0] for a, b in zip(spans, spans[1:]))
        sizes = [b - a for a, b in spans]
        assert max(sizes) - min(sizes) <= 1
