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
