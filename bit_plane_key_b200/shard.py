"""Key-range sharding of one layer across GPUs.

One GPU holds the whole problem at the sizes this library is measured on, so
the benchmark scales by giving every rank its own layer (ranks.py).  A single
context longer than one GPU's store can instead be split by key range: every
rank holds a contiguous, 1024-aligned range of the keys, scans it and takes
its local top-k; one all-gather of the (score, global index) pairs per query
head follows, and fathom_topk_merge selects the top-k of all keys on every
rank.  Because the ranges are ascending and each local list is in (score
descending, index ascending) order, ties resolve to the lower global index,
so the result equals the top-k of the unsplit scores.  Attention over the
selected keys then runs on each rank over the rows it holds and writes
per-head partials (o, m, l); one more all-gather and a GPU merge give every
rank the full output.
"""


def shard_range(n, world, rank, granule=1024):
    """[k0, k1): rank's contiguous share of n keys, cut on multiples of granule."""
    per = -(-n // world)
    per = -(-per // granule) * granule
    k0 = min(n, rank * per)
    return k0, min(n, k0 + per)


def gather_candidates(local_scores, local_idx, group=None):
    """All-gather of every rank's [rows][k] (score, global index) lists into
    [rows][world * k], rank by rank."""
    import torch
    import torch.distributed as dist
    world = dist.get_world_size(group)
    scores = [torch.empty_like(local_scores) for _ in range(world)]
    idx = [torch.empty_like(local_idx) for _ in range(world)]
    dist.all_gather(scores, local_scores.contiguous(), group=group)
    dist.all_gather(idx, local_idx.contiguous(), group=group)
    return torch.cat(scores, dim=1).contiguous(), torch.cat(idx, dim=1).contiguous()


def local_topk(store_shard, key0, q, depths, k):
    """The rank's scan + top-k over its keys [key0, key0 + n): [rows][k] lists of
    (score, global index), padded with (-inf, -1) when the shard holds fewer
    than k keys (store_shard None: an empty range)."""
    import torch
    from . import fathom as F
    if store_shard is None or store_shard.n == 0:   # an empty range contributes only padding
        rows = q.shape[0]
        return (torch.full((rows, k), float("-inf"), dtype=torch.float32, device=q.device),
                torch.full((rows, k), -1, dtype=torch.int32, device=q.device))
    kl = min(k, store_shard.n)
    idx, top = F.scan_topk(store_shard, q, depths, kl)
    idx = idx + int(key0)
    if kl < k:
        rows = idx.shape[0]
        idx = torch.cat([idx, torch.full((rows, k - kl), -1, dtype=idx.dtype, device=idx.device)], dim=1)
        top = torch.cat([top, torch.full((rows, k - kl), float("-inf"), dtype=top.dtype, device=top.device)], dim=1)
    return top.contiguous(), idx.contiguous()


def gather_partials(parts, group=None):
    """All-gather of every rank's attention partials [Hq][d + 2] into
    [world][Hq][d + 2], rank by rank."""
    import torch
    import torch.distributed as dist
    world = dist.get_world_size(group)
    out = [torch.empty_like(parts) for _ in range(world)]
    dist.all_gather(out, parts.contiguous(), group=group)
    return torch.stack(out).contiguous()


def sharded_attend(q, K_rows, V_rows, key0, idx, n_kv_heads=None, group=None):
    """Exact attention over the selected keys of a key-range-sharded layer:
    each rank attends over the selected rows it holds (keys [key0, key0 +
    n)), one all-gather of the per-head partials, the GPU merge.  Every rank
    returns the same [Hq][d] output."""
    from . import fathom as F
    if K_rows.shape[1] == 0:   # an empty range: m = -inf, l = 0 for every head
        parts = empty_partials(q.shape[0], q.shape[1], q.device)
    else:
        parts = F.sparse_attend_partial(q, K_rows, V_rows, idx, key0, n_kv_heads)
    return F.attend_merge(gather_partials(parts, group))


def empty_partials(n_q_heads, d, device):
    """The partials of a rank that holds no selected row: o = 0, m = -inf, l = 0."""
    import torch
    parts = torch.zeros((n_q_heads, d + 2), dtype=torch.float32, device=device)
    parts[:, d] = float("-inf")
    return parts


def sharded_scan_topk(store_shard, key0, q, depths, k, group=None):
    """Top-k of all keys of a key-range-sharded layer: local scan + top-k, one
    all-gather, the GPU merge.  Every rank returns the same (idx, scores)."""
    from . import fathom as F
    top, idx = local_topk(store_shard, key0, q, depths, k)
    cand_scores, cand_idx = gather_candidates(top, idx, group)
    return F.topk_merge(cand_scores, cand_idx, k)
