"""Memory-parallel routing: the pooled router keys are sharded over ranks.

The pages' deployment (IRMaD reading, "M. Materials & Methods", Memory
Parallel and tiered storage item; EverMind release article 2.3) keeps K̄^R
sharded over the GPUs: the query is broadcast, every GPU scores its own shard,
and a global reduction picks the top-k documents.  Here a shard is a
contiguous range of whole documents (so each document's max over its chunks
stays on one rank), balanced by chunk count.  The exchange step is one
all-gather of the B x k (score, global document id) candidates, a few KB,
followed by the exact merge of ``msa_topk_merge`` on the device; every rank
ends with the same top-k, in the same order as routing the unsharded memory.

The attention follows the same split: every rank attends over the selected
documents it holds (msa_sparse_attend_share; the local keys on one rank), the
ranks all-gather their shares, each the normalised fp32 output and its base-2
log-sum-exp per (query token, head), and msa_attend_merge weighs them into the
softmax over the whole context, in rank order, so every rank ends with the same
output.  Per step that exchange is B x n_q x (head_dim + 1) fp32 per rank (16.5 KB
for one query of 32 heads of 128).

One process per GPU; the collective runs on the default process group (NCCL on
GPUs, gloo in the CPU tests).
"""
from __future__ import annotations

import dataclasses
from typing import Callable, Optional

import numpy as np


@dataclasses.dataclass
class Shard:
    rank: int
    world: int
    doc_lo: int         # first document of this shard (global id)
    doc_hi: int         # one past the last document
    chunk_lo: int       # first chunk (global row of K̄^R)
    chunk_hi: int
    chunk_off: np.ndarray  # [doc_hi - doc_lo + 1] int32, rebased to chunk_lo

    @property
    def n_docs(self) -> int:
        return self.doc_hi - self.doc_lo

    @property
    def n_chunks(self) -> int:
        return self.chunk_hi - self.chunk_lo


def shard_memory(chunk_off, world: int, rank: int) -> Shard:
    """Contiguous document ranges with about C / world chunks each (at least one doc each)."""
    chunk_off = np.asarray(chunk_off, dtype=np.int64)
    n_docs = len(chunk_off) - 1
    if world > n_docs:
        raise ValueError(f"cannot split {n_docs} documents over {world} ranks")
    C = int(chunk_off[-1])
    bounds = [0]
    for r in range(1, world):
        b = int(np.searchsorted(chunk_off[:-1], r * C / world, side="left"))
        b = max(b, bounds[-1] + 1)                 # every shard keeps >= 1 document
        b = min(b, n_docs - (world - r))
        bounds.append(b)
    bounds.append(n_docs)
    d0, d1 = bounds[rank], bounds[rank + 1]
    c0, c1 = int(chunk_off[d0]), int(chunk_off[d1])
    local = (chunk_off[d0:d1 + 1] - c0).astype(np.int32)
    return Shard(rank, world, d0, d1, c0, c1, local)


def exchange_topk(local_idx, local_score, doc_base: int, k: int, group=None,
                  merge: Optional[Callable] = None):
    """Global top-k from every rank's local top-k.

    local_idx [B, k_local] int32 (ids within the shard), local_score [B, k_local] fp32.
    Candidates are padded to k per rank (score -inf), all-gathered as (score, global id)
    and merged; ``merge(cand_score, cand_idx, k)`` defaults to the device merge.
    """
    import torch
    import torch.distributed as dist

    B, kl = local_idx.shape
    world = dist.get_world_size(group)
    sc = torch.full((B, k), float("-inf"), dtype=torch.float32, device=local_score.device)
    gi = torch.full((B, k), np.iinfo(np.int32).max, dtype=torch.int32, device=local_idx.device)
    sc[:, :kl] = local_score
    gi[:, :kl] = local_idx + doc_base
    all_sc = [torch.empty_like(sc) for _ in range(world)]
    all_gi = [torch.empty_like(gi) for _ in range(world)]
    dist.all_gather(all_sc, sc, group=group)
    dist.all_gather(all_gi, gi, group=group)
    cand_s = torch.cat(all_sc, dim=1).contiguous()
    cand_i = torch.cat(all_gi, dim=1).contiguous()
    if merge is None:
        from . import topk_merge

        return topk_merge(cand_s, cand_i, k)
    return merge(cand_s, cand_i, k)


def route_topk_sharded(dims, Hq, W_QR, KR_local, shard: Shard, k: int, group=None, route: Optional[Callable] = None,
                       merge: Optional[Callable] = None):
    """This rank's routing over its shard, then the exchange; returns (topk_idx, topk_score).

    ``route(dims, Hq, W_QR, KR_local, chunk_off, k)`` -> (idx, score, ...) defaults to msa_route_topk
    and ``merge`` to msa_topk_merge (both replaceable so that the protocol runs on CPU ranks)."""
    import torch

    if route is None:
        from . import route_topk as route

    chunk_off = torch.from_numpy(shard.chunk_off).to(KR_local.device)
    kl = min(k, shard.n_docs)
    idx, sc = route(dims, Hq, W_QR, KR_local, chunk_off, kl)[:2]
    return exchange_topk(idx, sc, shard.doc_lo, k, group=group, merge=merge)


def exchange_attention(o_share, lse2_share, group=None, merge: Optional[Callable] = None):
    """All-gather every rank's attention share and merge them (rank order).

    o_share [..., head_dim] fp32, lse2_share [...] fp32 (msa_sparse_attend_share's outputs);
    ``merge(o_shares [R, ...], lse2_shares [R, ...])`` defaults to the device merge."""
    import torch
    import torch.distributed as dist

    world = dist.get_world_size(group)
    all_o = [torch.empty_like(o_share) for _ in range(world)]
    all_l = [torch.empty_like(lse2_share) for _ in range(world)]
    dist.all_gather(all_o, o_share.contiguous(), group=group)
    dist.all_gather(all_l, lse2_share.contiguous(), group=group)
    o = torch.stack(all_o).contiguous()
    l = torch.stack(all_l).contiguous()
    if merge is None:
        from . import attend_merge

        return attend_merge(o, l)
    return merge(o, l)


def attend_sharded(dims, q, K_bar_local, V_bar_local, shard: Shard, topk_idx, K_loc, V_loc, loc_len, pos_offset: int,
                   local_rank: int = 0, k_loc_rotated: bool = False, group=None, share: Optional[Callable] = None,
                   merge: Optional[Callable] = None):
    """This rank's share of the attention over the global top-k (global ids), then the exchange.

    The local keys belong to rank ``local_rank``; every rank passes loc_len (it places the query).
    ``share`` (same arguments as msa_sparse_attend_share's binding) and ``merge`` default to the
    device calls."""
    import torch

    if share is None:
        from . import sparse_attend_share as share

    chunk_off = torch.from_numpy(shard.chunk_off).to(q.device)
    t_loc_max = K_loc.shape[1] if K_loc is not None else 0
    o, l = share(dims, q, K_bar_local, V_bar_local, chunk_off, shard.doc_lo, topk_idx, shard.rank == local_rank, K_loc,
                 V_loc, loc_len, t_loc_max, pos_offset, k_loc_rotated=k_loc_rotated)
    return exchange_attention(o, l, group=group, merge=merge)
