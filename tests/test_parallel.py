"""Memory-parallel routing protocol: world_size-2 gloo ranks on CPU.

Each rank routes its shard of the memory (here with the CPU oracle standing in
for the rank's GPU), the ranks exchange their (score, global id) candidates with
an all-gather, and the merged top-k must equal the oracle's top-k over the
whole memory, on every rank.  The device merge (msa_topk_merge) and the
per-shard GPU routing are covered by test_gpu_parallel.py.
"""
import os
import socket

import numpy as np
import pytest

import oracle as O
from long_context_memory_b200 import parallel as P
from long_context_memory_b200 import workloads as W


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _memory(seed, n_docs=60, B=3, dup=False):
    rng = np.random.default_rng(seed)
    lens = rng.integers(1, 500, size=n_docs)
    co, *_ = O.chunk_layout(W.offsets_from_lengths(lens))
    C = int(co[-1])
    KR = W.normal_bf16(rng, (C, 4, 64))
    QR = W.normal_bf16(rng, (B, 4 * 64))
    if dup:  # identical documents on both sides of the split: ties must go to the lower global id
        first = KR[co[0]:co[1]].copy()
        KR[co[-2]:co[-1]] = first[: co[-1] - co[-2]] if co[-1] - co[-2] <= co[1] - co[0] else KR[co[-2]:co[-1]]
        lens2 = lens.copy()
        lens2[-1] = lens[0]
        co, *_ = O.chunk_layout(W.offsets_from_lengths(lens2))
        KR = np.concatenate([KR[: co[-2]], KR[: co[1]]])
    return co, KR, QR


def oracle_merge(cand_s, cand_i, k):
    import torch

    s = cand_s.numpy().astype(np.float64)
    ids = cand_i.numpy().astype(np.int64)
    out_i, out_s = [], []
    for b in range(s.shape[0]):
        order = np.lexsort((ids[b], -s[b]))[:k]
        out_i.append(ids[b][order])
        out_s.append(s[b][order])
    return torch.tensor(np.array(out_i), dtype=torch.int32), torch.tensor(np.array(out_s), dtype=torch.float32)


def _rank_main(rank, world, port, seed, k, dup, ret, n_docs=60):
    import torch
    import torch.distributed as dist

    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        co, KR, QR = _memory(seed, n_docs=n_docs, dup=dup)
        B = QR.shape[0]
        sh = P.shard_memory(co, world, rank)
        qr = O.bf16_to_f64(QR).reshape(B, 4, 64)
        S = O.chunk_scores(qr, KR[sh.chunk_lo:sh.chunk_hi])
        s_loc = O.doc_scores(S, sh.chunk_off)
        kl = min(k, sh.n_docs)
        li = np.stack([O.topk(s_loc[b], kl)[0] for b in range(B)]).astype(np.int32)
        ls = np.stack([s_loc[b][li[b]] for b in range(B)]).astype(np.float32)
        idx, sc = P.exchange_topk(torch.from_numpy(li), torch.from_numpy(ls), sh.doc_lo, k, merge=oracle_merge)
        ret[rank] = (idx.numpy(), sc.numpy(), (sh.doc_lo, sh.doc_hi, sh.chunk_lo, sh.chunk_hi))
    finally:
        dist.destroy_process_group()


def _run(world, seed, k, dup=False, n_docs=60):
    import torch.multiprocessing as mp

    ctx = mp.get_context("spawn")
    mgr = ctx.Manager()
    ret = mgr.dict()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, seed, k, dup, ret, n_docs)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0, f"rank exited with {p.exitcode}"
    return dict(ret)


def test_shard_memory_covers_every_document_once():
    co, _, _ = _memory(1, n_docs=97)
    for world in (1, 2, 3, 8):
        shards = [P.shard_memory(co, world, r) for r in range(world)]
        assert shards[0].doc_lo == 0 and shards[-1].doc_hi == len(co) - 1
        for a, b in zip(shards, shards[1:]):
            assert a.doc_hi == b.doc_lo and a.chunk_hi == b.chunk_lo
        for s in shards:
            assert s.n_docs >= 1
            assert s.chunk_off[0] == 0 and s.chunk_off[-1] == s.n_chunks
            assert np.array_equal(s.chunk_off, co[s.doc_lo:s.doc_hi + 1] - co[s.doc_lo])
        if world > 1:
            sizes = [s.n_chunks for s in shards]
            assert max(sizes) - min(sizes) <= 2 * max(np.diff(co))   # each boundary is off by < 1 document


@pytest.mark.parametrize("k", [1, 7, 16])
def test_two_rank_exchange_matches_global_topk(k):
    ret = _run(2, seed=11, k=k)
    co, KR, QR = _memory(11)
    B = QR.shape[0]
    s, idx, val = O.route_topk(O.bf16_to_f64(QR).reshape(B, 4, 64), KR, co, k)
    for rank in (0, 1):
        gi, gs, _ = ret[rank]
        assert np.array_equal(gi, idx), (rank, gi, idx)
        assert np.allclose(gs, val, atol=1e-6)


def test_two_rank_ties_go_to_lower_global_id():
    ret = _run(2, seed=5, k=4, dup=True)
    co, KR, QR = _memory(5, dup=True)
    B = QR.shape[0]
    s, idx, val = O.route_topk(O.bf16_to_f64(QR).reshape(B, 4, 64), KR, co, len(co) - 1)
    n = len(co) - 1
    assert np.allclose(s[:, 0], s[:, n - 1])          # the duplicated pair scores the same
    for rank in (0, 1):
        gi, _, _ = ret[rank]
        for b in range(B):
            if 0 in gi[b] and n - 1 in gi[b]:
                assert list(gi[b]).index(0) < list(gi[b]).index(n - 1)
        assert np.array_equal(gi, idx[:, :4])


@pytest.mark.parametrize("k", [5, 8])
def test_three_ranks_with_shards_smaller_than_k(k):
    # 8 documents over 3 ranks: every shard holds fewer than k documents, so each rank pads its
    # candidates (score -inf) before the exchange; k = 8 selects every document
    ret = _run(3, seed=23, k=k, n_docs=8)
    co, KR, QR = _memory(23, n_docs=8)
    B = QR.shape[0]
    _, idx, val = O.route_topk(O.bf16_to_f64(QR).reshape(B, 4, 64), KR, co, k)
    spans = sorted(r[2] for r in ret.values())
    assert all(hi - lo < k for lo, hi, _, _ in spans)
    for rank in range(3):
        gi, gs, _ = ret[rank]
        assert np.array_equal(gi, idx), (rank, gi, idx)
        assert np.allclose(gs, val, atol=1e-6)
