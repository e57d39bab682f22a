"""GPU parity of multi-token queries (the query-prefill step) against the CPU oracle.

Routing: a query of M tokens scores a chunk by the largest, over its tokens, of
the head-mean cosine (the max over t of the routing formula), then aggregates
per document as usual.  Attention: the M query tokens are the last M local
tokens; token t sits at pos_offset + loc_len - M + t and sees every gathered
chunk and the local tokens up to its own position.
"""
import numpy as np
import pytest

import oracle as O
from long_context_memory_b200 import workloads as W
from helpers import SCORE_ATOL, check_attention, check_topk

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def msa(cuda_device):
    import long_context_memory_b200 as m

    return m


def _dev(a, device):
    return W.to_torch(np.ascontiguousarray(a)).to(device)


# ----------------------------------------------------------------------------
# routing with M query tokens
# ----------------------------------------------------------------------------
@pytest.mark.parametrize("B,M", [(1, 2), (4, 3), (13, 3), (2, 16), (5, 7)])
@pytest.mark.parametrize("agg", [0, 1])
def test_route_multi_token_direct_query(msa, cuda_device, B, M, agg):
    import torch

    rng = np.random.default_rng(500 + 7 * B + M + agg)
    n_r, d_r = 4, 64
    lens = rng.integers(1, 600, size=150)
    doc_off = W.offsets_from_lengths(lens)
    co, C = msa.chunk_offsets(doc_off)
    KR = W.normal_bf16(rng, (C, n_r, d_r))
    QR = W.normal_bf16(rng, (B * M, n_r * d_r))
    dims = W.Dims(hidden=256, n_q=8, n_kv=2, head_dim=64, n_r=n_r, d_r=d_r)
    k = 10
    idx, sc, ds = msa.route_topk(dims, _dev(QR, cuda_device), None, _dev(KR, cuda_device),
                                 torch.from_numpy(co).to(cuda_device), k, agg=agg, want_doc_scores=True,
                                 q_tokens=M)
    torch.cuda.synchronize()
    assert msa.check_device_errors() == 0
    ds, idx, sc = ds.cpu().numpy(), idx.cpu().numpy(), sc.cpu().numpy()
    s, _, _ = O.route_topk(O.bf16_to_f64(QR).reshape(B, M, n_r, d_r), KR, co, k, "max" if agg == 0 else "mean")
    assert np.max(np.abs(ds - s)) < SCORE_ATOL, np.max(np.abs(ds - s))
    for b in range(B):
        check_topk(idx[b], sc[b], s[b], k, where=f"B={B} M={M} b={b}")


def test_route_multi_token_projection_and_single_token_equivalence(msa, cuda_device):
    import torch

    rng = np.random.default_rng(77)
    B, M, hidden = 3, 5, 512
    lens = rng.integers(1, 900, size=200)
    co, C = msa.chunk_offsets(W.offsets_from_lengths(lens))
    KR = W.normal_bf16(rng, (C, 8, 128))
    Hq = W.normal_bf16(rng, (B * M, hidden))
    Wqr = W.normal_bf16(rng, (hidden, 1024), hidden ** -0.5)
    dims = W.Dims(hidden=hidden, n_q=8, n_kv=2, head_dim=64, n_r=8, d_r=128)
    co_d = torch.from_numpy(co).to(cuda_device)
    idx, sc, ds = msa.route_topk(dims, _dev(Hq, cuda_device), _dev(Wqr, cuda_device), _dev(KR, cuda_device), co_d,
                                 16, want_doc_scores=True, q_tokens=M)
    QR = O.router_query(Hq, Wqr, 8, 128).reshape(B, M, 8, 128)
    s, _, _ = O.route_topk(QR, KR, co, 16)
    ds = ds.cpu().numpy()
    assert np.max(np.abs(ds - s)) < SCORE_ATOL
    for b in range(B):
        check_topk(idx[b].cpu().numpy(), sc[b].cpu().numpy(), s[b], 16, where=f"b={b}")
    # the same rows routed as B*M one-token queries: a query's doc score is the max over its tokens
    _, _, ds1 = msa.route_topk(dims, _dev(Hq, cuda_device), _dev(Wqr, cuda_device), _dev(KR, cuda_device), co_d,
                               16, want_doc_scores=True)
    torch.cuda.synchronize()
    ds1 = ds1.cpu().numpy().reshape(B, M, -1)
    assert np.array_equal(ds, ds1.max(axis=1))


# ----------------------------------------------------------------------------
# attention with M query tokens
# ----------------------------------------------------------------------------
def _case(seed, B, M, n_q, n_kv, D, n_docs, k, t_loc, loc_len):
    rng = np.random.default_rng(seed)
    lens = rng.integers(1, 700, size=n_docs)
    doc_off = W.offsets_from_lengths(lens)
    co, *_ = O.chunk_layout(doc_off)
    C = int(co[-1])
    topk = np.stack([rng.permutation(n_docs)[:k] for _ in range(B)])
    return dict(doc_off=doc_off, chunk_off=co, q=W.normal_bf16(rng, (B, M, n_q, D)),
                K_bar=W.normal_bf16(rng, (C, n_kv, D)), V_bar=W.normal_bf16(rng, (C, n_kv, D)),
                K_loc=W.normal_bf16(rng, (B, t_loc, n_kv, D)), V_loc=W.normal_bf16(rng, (B, t_loc, n_kv, D)),
                loc_len=np.asarray(loc_len), topk=topk)


def _run(msa, dims, c, device, pos_offset, rotated=False):
    import torch

    co, C = msa.chunk_offsets(c["doc_off"])
    K_loc = _dev(c["K_loc"], device)
    if rotated:
        B, T = c["K_loc"].shape[:2]
        pos = (pos_offset + torch.arange(T, dtype=torch.int32, device=device)).repeat(B)
        msa.rope_rows(dims, K_loc.view(B * T, dims.n_kv, dims.head_dim), pos)
    out = msa.sparse_attend(dims, _dev(c["q"], device), _dev(c["K_bar"], device), _dev(c["V_bar"], device),
                            torch.from_numpy(co).to(device), torch.from_numpy(c["topk"].astype(np.int32)).to(device),
                            K_loc, _dev(c["V_loc"], device), torch.from_numpy(c["loc_len"].astype(np.int32)).to(device),
                            pos_offset, k_loc_rotated=rotated)
    torch.cuda.synchronize()
    assert msa.check_device_errors() == 0
    assert tuple(out.shape) == c["q"].shape
    return out.float().cpu().numpy()


def _oracle(c, pos_offset, base=1e6):
    return O.sparse_attend_tokens(c["q"], c["K_bar"], c["V_bar"], c["chunk_off"], c["topk"], c["K_loc"], c["V_loc"],
                                  c["loc_len"], pos_offset, base)


# G = n_q / n_kv; tokens per CTA = 16 / G: G = 4 packs 4 tokens, G = 16 one, G = 1 sixteen
@pytest.mark.parametrize("M", [1, 3, 4, 7])
@pytest.mark.parametrize("D,n_q,n_kv", [(128, 32, 8), (64, 8, 2), (128, 16, 1), (64, 4, 4)])
def test_attend_multi_token_parity(msa, cuda_device, M, D, n_q, n_kv):
    c = _case(900 + M + D + n_q, 3, M, n_q, n_kv, D, n_docs=25, k=4, t_loc=160, loc_len=[160, 37, M])
    dims = W.Dims(hidden=256, n_q=n_q, n_kv=n_kv, head_dim=D, n_r=4, d_r=64, rope_base=1e6)
    out = _run(msa, dims, c, cuda_device, pos_offset=4)
    check_attention(out, _oracle(c, 4), where=f"M={M} D={D} G={n_q // n_kv}")


def test_attend_multi_token_rotated_cache_and_short_local(msa, cuda_device):
    # rotated local cache; one query with fewer local tokens than query tokens (its first
    # tokens see the gathered chunks only) and M = 18 spanning several token groups
    M = 18
    c = _case(77, 2, M, 32, 8, 128, n_docs=20, k=3, t_loc=64, loc_len=[64, 5])
    dims = W.Dims(hidden=256, n_q=32, n_kv=8, head_dim=128, n_r=4, d_r=64, rope_base=1e6)
    out = _run(msa, dims, c, cuda_device, pos_offset=3, rotated=True)
    check_attention(out, _oracle(c, 3), where="rotated M=18")


def test_attend_multi_token_decode_equivalence(msa, cuda_device):
    # token t of an M-token call equals a one-token call whose loc_len is loc_len - M + t + 1
    import torch

    M = 5
    c = _case(31, 2, M, 32, 8, 128, n_docs=30, k=6, t_loc=300, loc_len=[300, 120])
    dims = W.Dims(hidden=256, n_q=32, n_kv=8, head_dim=128, n_r=4, d_r=64, rope_base=1e6)
    out = _run(msa, dims, c, cuda_device, pos_offset=6)
    for t in range(M):
        c1 = dict(c)
        c1["q"] = np.ascontiguousarray(c["q"][:, t])
        c1["loc_len"] = c["loc_len"] - M + t + 1
        one = _run(msa, dims, c1, cuda_device, pos_offset=6)
        # same keys, same rows, same splits: only the accumulation order within a split can differ
        assert np.max(np.abs(one - out[:, t])) < 2e-2, t
