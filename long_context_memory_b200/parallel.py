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


def route_topk_sharded(dims, Hq, W_QR, KR_local, shard: Shard, k: int, group=None):
    """This rank's routing over its shard, then the exchange; returns (topk_idx, topk_score)."""
    import torch

    from . import route_topk

    chunk_off = torch.from_numpy(shard.chunk_off).to(KR_local.device)
    kl = min(k, shard.n_docs)
    idx, sc, _ = route_topk(dims, Hq, W_QR, KR_local, chunk_off, kl)
    return exchange_topk(idx, sc, shard.doc_lo, k, group=group)
