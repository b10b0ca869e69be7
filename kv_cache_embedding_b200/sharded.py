"""Search over a database sharded across ranks (one process per GPU): every
rank keeps the records of its contiguous shard, computes its local top-k with
tq_topk, makes the ids global, and one all-gather of the [rows, k] lists
(values fp32, ids int64) feeds tq_topk_merge on every rank.  The pages'
vector search is a top-k over all records; sharding changes where the
records live, not the result."""
import torch
import torch.distributed as dist

from . import _binding as B
from .quantizer import _ptr, _stream


def shard_bounds(n_total, world, rank):
    """Contiguous shard [start, stop) of rank among world (sizes differ by at
    most one record)."""
    base, extra = divmod(n_total, world)
    start = rank * base + min(rank, extra)
    return start, start + base + (1 if rank < extra else 0)


def gather_lists(vals, ids, group=None):
    """All-gather every rank's [..., k] lists: returns [world, rows, k] tensors
    (rank order), rows = the product of the leading dimensions."""
    world = dist.get_world_size(group)
    k = vals.shape[-1]
    v = vals.reshape(-1, k).contiguous()
    i = ids.reshape(-1, k).contiguous()
    gv = [torch.empty_like(v) for _ in range(world)]
    gi = [torch.empty_like(i) for _ in range(world)]
    dist.all_gather(gv, v, group=group)
    dist.all_gather(gi, i, group=group)
    return torch.stack(gv), torch.stack(gi)


def merge_lists(gvals, gids, k):
    """Best k per row of [nlists, rows, k] lists on the device (tq_topk_merge)."""
    nlists, rows, _ = gvals.shape
    out_v = torch.empty(rows, k, dtype=torch.float32, device=gvals.device)
    out_i = torch.empty(rows, k, dtype=torch.int64, device=gvals.device)
    B.tq_topk_merge(rows, nlists, k, _ptr(gvals.contiguous()), _ptr(gids.contiguous()),
                    _ptr(out_v), _ptr(out_i), _stream())
    return out_v, out_i


def sharded_topk(tq, codes, q, k, n_total, group=None, local_topk=None, merge=None):
    """Top-k over a database of n_total records of which this rank holds its
    shard_bounds() slice as `codes` (a Codes of [G, n_shard, ...]); q is the
    same [G, nq, d] on every rank.  Returns the global (vals, ids) [G, nq, k]
    on every rank.

    local_topk(codes, q, k) -> (vals, ids) and merge(gvals, gids, k) -> (vals,
    ids) default to tq.topk and merge_lists (libtq); a caller may pass other
    implementations of the same contract (the CPU tests pass the oracle's)."""
    world, rank = dist.get_world_size(group), dist.get_rank(group)
    start, _ = shard_bounds(n_total, world, rank)
    local_topk = local_topk or tq.topk
    merge = merge or merge_lists
    vals, ids = local_topk(codes, q, k)
    # missing entries (a shard with fewer than k records) keep their marker
    ids = torch.where(ids == torch.iinfo(torch.int64).max, ids, ids + start)
    gv, gi = gather_lists(vals, ids, group)
    mv, mi = merge(gv, gi, k)
    return mv.reshape(vals.shape), mi.reshape(ids.shape)
