"""Memory-parallel routing protocol: world_size-2 gloo ranks on CPU.

Each rank routes its shard of the memory (here with the CPU oracle standing in
for the rank's GPU), the ranks exchange their (score, global id) candidates with
an all-gather, and the merged top-k must equal the oracle's top-k over the
whole memory, on every rank.  The device merge (msa_topk_merge) and the
per-shard GPU routing are covered by test_gpu_parallel.py.
"""
import math
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


# ----------------------------------------------------------------------------
# the composed functions on CPU ranks: route_topk_sharded, then attend_sharded
# ----------------------------------------------------------------------------
DIMS_CPU = W.Dims(hidden=128, n_q=4, n_kv=2, head_dim=64, n_r=4, d_r=64, rope_base=1e4)


def _bits(t):
    """bf16 torch tensor -> uint16 bit patterns (numpy)."""
    import torch

    return t.view(torch.int16).numpy().view(np.uint16)


def _oracle_route(dims, Hq, W_QR, KR_local, chunk_off, k):
    """Stands in for msa_route_topk on a CPU rank (the oracle's scores of the shard's documents)."""
    import torch

    qr = O.bf16_to_f64(_bits(Hq)).reshape(-1, dims.n_r, dims.d_r)
    s = O.doc_scores(O.chunk_scores(qr, _bits(KR_local)), chunk_off.numpy())
    idx = np.stack([O.topk(s[b], k)[0] for b in range(s.shape[0])]).astype(np.int32)
    sc = np.stack([s[b][idx[b]] for b in range(s.shape[0])]).astype(np.float32)
    return torch.from_numpy(idx), torch.from_numpy(sc)


def _oracle_share(dims, q, K_bar, V_bar, chunk_off, doc_base, topk_idx, local_keys, K_loc, V_loc, loc_len, t_loc_max,
                  pos_offset, k_loc_rotated=False):
    """Stands in for msa_sparse_attend_share on a CPU rank: the softmax over the selected documents this
    shard holds (and the local keys where local_keys), its normalised output and base-2 log-sum-exp."""
    import torch

    qf = O.bf16_to_f64(_bits(q))
    B, n_q, D = qf.shape
    Kb, Vb = O.bf16_to_f64(_bits(K_bar)), O.bf16_to_f64(_bits(V_bar))
    co = chunk_off.numpy()
    G = n_q // dims.n_kv
    o = np.zeros((B, n_q, D))
    l2 = np.full((B, n_q), -np.inf)
    for b in range(B):
        L = int(loc_len[b])
        ks, vs = [], []
        for doc in topk_idx[b].tolist():
            i = doc - doc_base
            if 0 <= i < len(co) - 1:
                ks.append(Kb[co[i]:co[i + 1]])
                vs.append(Vb[co[i]:co[i + 1]])
        if local_keys and L > 0:
            ks.append(O.rope(O.bf16_to_f64(_bits(K_loc[b, :L].contiguous())), (pos_offset + np.arange(L))[:, None], dims.rope_base))
            vs.append(O.bf16_to_f64(_bits(V_loc[b, :L].contiguous())))
        if not ks:
            continue
        K, V = np.concatenate(ks), np.concatenate(vs)
        qr = O.rope(qf[b], pos_offset + L - 1, dims.rope_base)
        for g in range(n_q):
            logits = (K[:, g // G] @ qr[g]) / math.sqrt(D)
            m = logits.max()
            p = np.exp(logits - m)
            o[b, g] = (p[:, None] * V[:, g // G]).sum(0) / p.sum()
            l2[b, g] = (m + math.log(p.sum())) / math.log(2.0)
    return torch.from_numpy(o), torch.from_numpy(l2)


def _numpy_attend_merge(o_sh, l_sh):
    o, l = o_sh.numpy(), l_sh.numpy()
    m = l.max(axis=0)
    w = np.where(np.isfinite(l), np.exp2(l - np.where(np.isfinite(m), m, 0.0)), 0.0)
    import torch

    return torch.from_numpy((w[..., None] * o).sum(0) / np.maximum(w.sum(0), 1e-300)[..., None])


def _composed_rank(rank, world, port, ret):
    import torch
    import torch.distributed as dist

    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        c = _composed_case()
        d, co, k = DIMS_CPU, c["co"], c["k"]
        sh = P.shard_memory(co, world, rank)
        rows = slice(sh.chunk_lo, sh.chunk_hi)
        t = W.to_torch
        idx, sc = P.route_topk_sharded(d, t(c["QR"]), None, t(c["KR"][rows]), sh, k, route=_oracle_route,
                                       merge=oracle_merge)
        out = P.attend_sharded(d, t(c["q"]), t(c["K_bar"][rows]), t(c["V_bar"][rows]), sh, idx, t(c["K_loc"]),
                               t(c["V_loc"]), c["loc_len"], k, share=_oracle_share, merge=_numpy_attend_merge)
        ret[rank] = (idx.numpy(), sc.numpy(), out.numpy())
    finally:
        dist.destroy_process_group()


def _composed_case():
    d = DIMS_CPU
    rng = np.random.default_rng(404)
    lens = rng.integers(1, 400, size=40)
    co, *_ = O.chunk_layout(W.offsets_from_lengths(lens))
    C, B, t_loc = int(co[-1]), 3, 20
    return dict(co=co, k=5, KR=W.normal_bf16(rng, (C, d.n_r, d.d_r)), QR=W.normal_bf16(rng, (B, d.n_r * d.d_r)),
                K_bar=W.normal_bf16(rng, (C, d.n_kv, d.head_dim)), V_bar=W.normal_bf16(rng, (C, d.n_kv, d.head_dim)),
                q=W.normal_bf16(rng, (B, d.n_q, d.head_dim)), K_loc=W.normal_bf16(rng, (B, t_loc, d.n_kv, d.head_dim)),
                V_loc=W.normal_bf16(rng, (B, t_loc, d.n_kv, d.head_dim)), loc_len=np.array([20, 7, 1]))


@pytest.mark.parametrize("world", [2, 3])
def test_composed_route_and_attend_on_gloo_ranks(world):
    # route_topk_sharded then attend_sharded on every rank: the global top-k and the merged attention
    # (the local keys on rank 0 only) equal the oracle over the unsharded memory, on every rank
    import torch.multiprocessing as mp

    ctx = mp.get_context("spawn")
    ret = ctx.Manager().dict()
    port = _free_port()
    procs = [ctx.Process(target=_composed_rank, args=(r, world, port, ret)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(180)
        assert p.exitcode == 0, f"rank exited with {p.exitcode}"
    c, d = _composed_case(), DIMS_CPU
    B = c["q"].shape[0]
    _, idx, val = O.route_topk(O.bf16_to_f64(c["QR"]).reshape(B, d.n_r, d.d_r), c["KR"], c["co"], c["k"])
    ref = O.sparse_attend(c["q"], c["K_bar"], c["V_bar"], c["co"], idx, c["K_loc"], c["V_loc"], c["loc_len"], c["k"],
                          d.rope_base)
    for rank in range(world):
        gi, gs, out = ret[rank]
        assert np.array_equal(gi, idx), rank
        assert np.allclose(gs, val, atol=1e-6)
        assert np.max(np.abs(out - ref)) < 1e-10, np.max(np.abs(out - ref))
