"""The router split by columns across devices (one process per device).

Each rank streams its own contiguous block of the weight's columns with the
window's rows A replicated, so every row still reads each weight byte once and
every logit has the bits of the one-device call.  Each rank takes the top-k of
its shard with global indices (``router_topk_ex``); the ranks all-gather the
candidate lists (``torch.distributed``, NCCL on GPUs) and every rank merges
them under the same total order (``router_topk_merge``).  The global top-k is
contained in the union of the shards' top-k lists, so the merge is exact:
indices and values equal the one-device router's bit for bit, ties across a
shard boundary included (contiguous shards keep the lower index first).

This is the multi-card placement of Strata PR #109 ("Measured": a second card
holding experts; the release comment: an RTX 5080 + RTX 3090 layer split)
applied to the router's columns.  This module holds the host logic only
(shard bounds, candidate layout, the collective); every step of the
arithmetic runs in the library's kernels.
"""
from __future__ import annotations


def shard_columns(n: int, world: int, rank: int) -> tuple[int, int]:
    """Columns [begin, end) of n owned by `rank` of `world` (sizes differ by at most one)."""
    if world < 1 or not 0 <= rank < world or n < world:
        raise ValueError(f"cannot split {n} columns over {world} ranks (rank {rank})")
    return rank * n // world, (rank + 1) * n // world


def local_topk(n_shard: int, topk: int) -> int:
    """Entries each shard contributes: its whole top-k, or all of its columns if fewer."""
    return min(topk, n_shard)


def gather_candidates(mine_idx, mine_val, all_idx, all_val, world: int, group=None):
    """All-gather every rank's [m, topk] candidate lists.

    Rank r's lists land as block r of the first world * m * topk elements of
    the [world, max_m, topk] buffers all_idx / all_val; returns those blocks
    viewed as [world, m, topk] (index and value), the layout router_topk_merge
    reads with ld_row = topk and ld_group = m * topk.  With one rank the
    lists are returned as they are.  Every rank must call this with the same m.
    """
    import torch.distributed as dist
    m, topk = mine_idx.shape
    if world == 1:
        return mine_idx.unsqueeze(0), mine_val.unsqueeze(0)
    flat_idx = all_idx.view(-1)[: world * m * topk]
    flat_val = all_val.view(-1)[: world * m * topk]
    dist.all_gather_into_tensor(flat_idx, mine_idx.contiguous().view(-1), group=group)
    dist.all_gather_into_tensor(flat_val, mine_val.contiguous().view(-1), group=group)
    return flat_idx.view(world, m, topk), flat_val.view(world, m, topk)


class ShardedRouter:
    """One rank's part of the column-split router for windows of up to `max_m` rows.

    ``Wt_shard`` is this rank's [end - begin, k] block of the weight (bf16,
    k contiguous).  Buffers for the logits and candidate lists are allocated
    once here (torch); ``__call__`` only launches kernels and the all-gather
    on the current stream.
    """

    def __init__(self, Wt_shard, n_total: int, topk: int, max_m: int = 16, group=None):
        import torch
        import torch.distributed as dist
        from . import mrgemv_bf16  # noqa: F401  (fails loudly without the library)
        self.world = dist.get_world_size(group) if dist.is_initialized() else 1
        self.rank = dist.get_rank(group) if dist.is_initialized() else 0
        self.group = group
        self.begin, self.end = shard_columns(n_total, self.world, self.rank)
        if Wt_shard.shape[0] != self.end - self.begin:
            raise ValueError(f"rank {self.rank} owns columns [{self.begin}, {self.end}); "
                             f"Wt_shard has {Wt_shard.shape[0]} rows")
        self.Wt = Wt_shard
        self.topk = topk
        self.k_loc = local_topk(self.end - self.begin, topk)
        dev = Wt_shard.device
        self.logits = torch.empty((max_m, self.end - self.begin), dtype=torch.float32, device=dev)
        # This rank's candidates, padded to topk entries (index -1 = empty).
        self.mine_idx = torch.full((max_m, topk), -1, dtype=torch.int32, device=dev)
        self.mine_val = torch.zeros((max_m, topk), dtype=torch.float32, device=dev)
        self.all_idx = torch.empty((self.world, max_m, topk), dtype=torch.int32, device=dev)
        self.all_val = torch.empty((self.world, max_m, topk), dtype=torch.float32, device=dev)

    def __call__(self, A, idx, val=None, flags: int = 0) -> None:
        """idx[m, topk] / val[m, topk] = the global router top-k of A[m, k]."""
        from . import mrgemv_bf16, router_topk_ex, router_topk_merge
        m = A.shape[0]
        logits = self.logits[:m]
        mrgemv_bf16(A, self.Wt, logits, flags=flags)
        router_topk_ex(logits, self.k_loc, self.mine_idx[:m], self.mine_val[:m], index_base=self.begin)
        cand_idx, cand_val = gather_candidates(self.mine_idx[:m], self.mine_val[:m], self.all_idx, self.all_val,
                                               self.world, self.group)
        router_topk_merge(cand_val, cand_idx, self.topk, idx, val)
