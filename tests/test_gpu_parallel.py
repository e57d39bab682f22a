"""Memory-parallel routing on one GPU: the memory is split into shards, each
shard is routed with msa_route_topk, and msa_topk_merge of the shards'
(score, global id) candidates must equal msa_route_topk over the whole memory
(and the oracle).  No collective runs here; the exchange protocol is covered by
the gloo tests in test_parallel.py."""
import numpy as np
import pytest

import oracle as O
from long_context_memory_b200 import parallel as P
from long_context_memory_b200 import workloads as W
from helpers import check_topk

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("world,B,k", [(2, 1, 16), (3, 5, 16), (4, 32, 8), (8, 2, 64)])
def test_sharded_route_equals_whole_memory(cuda_device, world, B, k):
    import torch

    import long_context_memory_b200 as msa

    rng = np.random.default_rng(100 + world)
    dims = W.Dims(hidden=512, n_q=8, n_kv=2, head_dim=64, n_r=8, d_r=128)
    lens = rng.integers(1, 1500, size=400)
    co, C = msa.chunk_offsets(W.offsets_from_lengths(lens))
    KR = W.normal_bf16(rng, (C, 8, 128))
    QR = W.normal_bf16(rng, (B, 1024))
    dev = cuda_device
    KRd = W.to_torch(KR).to(dev)
    QRd = W.to_torch(QR).to(dev)
    ref_idx, ref_sc, _ = msa.route_topk(dims, QRd, None, KRd, torch.from_numpy(co).to(dev), k)
    cs, ci = [], []
    for r in range(world):
        sh = P.shard_memory(co, world, r)
        kl = min(k, sh.n_docs)
        idx, sc, _ = msa.route_topk(dims, QRd, None, KRd[sh.chunk_lo:sh.chunk_hi],
                                    torch.from_numpy(sh.chunk_off).to(dev), kl)
        pad_s = torch.full((B, k), float("-inf"), device=dev)
        pad_i = torch.full((B, k), 2**31 - 1, dtype=torch.int32, device=dev)
        pad_s[:, :kl] = sc
        pad_i[:, :kl] = idx + sh.doc_lo
        cs.append(pad_s)
        ci.append(pad_i)
    m_idx, m_sc = msa.topk_merge(torch.cat(cs, 1).contiguous(), torch.cat(ci, 1).contiguous(), k)
    torch.cuda.synchronize()
    assert torch.equal(m_idx, ref_idx)
    assert torch.equal(m_sc, ref_sc)
    s, _, _ = O.route_topk(O.bf16_to_f64(QR).reshape(B, 8, 128), KR, co, k)
    for b in range(B):
        check_topk(m_idx[b].cpu().numpy(), m_sc[b].cpu().numpy(), s[b], k, where=f"b={b}")


def test_merge_ties_prefer_lower_global_id(cuda_device):
    import torch

    import long_context_memory_b200 as msa

    sc = torch.tensor([[0.5, 0.9, 0.5, 0.9, 0.1, 0.5]], device=cuda_device)
    ids = torch.tensor([[7, 40, 3, 12, 1, 9]], dtype=torch.int32, device=cuda_device)
    idx, val = msa.topk_merge(sc, ids, 4)
    assert idx.cpu().tolist() == [[12, 40, 3, 7]]
    assert val.cpu().tolist()[0] == pytest.approx([0.9, 0.9, 0.5, 0.5])


@pytest.mark.parametrize("world,B,M,k", [(2, 1, 1, 16), (3, 3, 1, 8), (8, 2, 1, 4), (2, 2, 3, 8)])
def test_sharded_attention_shares_merge_to_whole_memory(cuda_device, world, B, M, k):
    # every shard attends over the selected documents it holds (global ids; the local keys on
    # shard 0 only), msa_attend_merge weighs the shares: the result equals msa_sparse_attend over
    # the unsharded memory and the oracle.  With world 8 and k 4 some shards hold no selected
    # document and no local key (an empty share, log-sum-exp -inf).
    import torch

    import long_context_memory_b200 as msa

    rng = np.random.default_rng(300 + world + B + M)
    dims = W.Dims(hidden=256, n_q=32, n_kv=8, head_dim=128, n_r=4, d_r=64, rope_base=1e6)
    lens = rng.integers(1, 2000, size=60)
    co, C = msa.chunk_offsets(W.offsets_from_lengths(lens))
    t_loc, dev = 40, cuda_device
    Kb = W.normal_bf16(rng, (C, 8, 128))
    Vb = W.normal_bf16(rng, (C, 8, 128))
    q = W.normal_bf16(rng, (B, M, 32, 128) if M > 1 else (B, 32, 128))
    Kl = W.normal_bf16(rng, (B, t_loc, 8, 128))
    Vl = W.normal_bf16(rng, (B, t_loc, 8, 128))
    loc_len = rng.integers(M, t_loc + 1, size=B).astype(np.int32)
    sel = np.stack([rng.permutation(len(lens))[:k] for _ in range(B)]).astype(np.int32)
    t = lambda a: W.to_torch(np.ascontiguousarray(a)).to(dev)
    topk, ll = torch.from_numpy(sel).to(dev), torch.from_numpy(loc_len).to(dev)
    whole = msa.sparse_attend(dims, t(q), t(Kb), t(Vb), torch.from_numpy(co).to(dev), topk, t(Kl), t(Vl), ll, k)
    os_, ls_ = [], []
    for r in range(world):
        sh = P.shard_memory(co, world, r)
        rows = slice(sh.chunk_lo, sh.chunk_hi)
        o, l = msa.sparse_attend_share(dims, t(q), t(Kb[rows]), t(Vb[rows]), torch.from_numpy(sh.chunk_off).to(dev),
                                       sh.doc_lo, topk, r == 0, t(Kl) if r == 0 else None,
                                       t(Vl) if r == 0 else None, ll, t_loc, k)
        os_.append(o)
        ls_.append(l)
    out = msa.attend_merge(torch.stack(os_).contiguous(), torch.stack(ls_).contiguous())
    torch.cuda.synchronize()
    assert msa.check_device_errors() == 0
    assert out.shape == whole.shape
    g, w = out.float().cpu().numpy(), whole.float().cpu().numpy()
    assert np.max(np.abs(g - w)) <= 2 ** -7 * np.max(np.abs(w)) + 1e-3, np.max(np.abs(g - w))
    if world == 8:  # some share saw no key at all
        assert any(bool(torch.isinf(l).any()) for l in ls_)
    from helpers import check_attention

    co_o, *_ = O.chunk_layout(W.offsets_from_lengths(lens))
    if M == 1:
        ref = O.sparse_attend(q, Kb, Vb, co_o, sel, Kl, Vl, loc_len, k, 1e6)
    else:
        ref = O.sparse_attend_tokens(q, Kb, Vb, co_o, sel, Kl, Vl, loc_len, k, 1e6)
    check_attention(g, ref, where=f"world={world}")


def test_attend_merge_weights_by_log_sum_exp(cuda_device):
    # two shares of one row: lse2 0 and 1 -> weights 1/3 and 2/3; an empty share (-inf) counts 0
    import torch

    import long_context_memory_b200 as msa

    o = torch.zeros((3, 1, 64), dtype=torch.float32, device=cuda_device)
    o[0] += 1.0
    o[1] += 4.0
    o[2] += 100.0
    l = torch.tensor([[0.0], [1.0], [float("-inf")]], device=cuda_device)
    out = msa.attend_merge(o, l)
    torch.cuda.synchronize()
    assert torch.allclose(out.float(), torch.full((1, 64), 3.0, device=cuda_device), atol=1e-2)
