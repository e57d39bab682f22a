"""GPU parity of the tiered decode (routing, host-tier gather and attention of several layers in one
call) and of routing and attention over a 100M-token memory, through the C ABI."""
import math

import numpy as np
import pytest

import oracle as O
from long_context_memory_b200 import workloads as W
from helpers import SCORE_ATOL, TOPK_GAP, check_attention, check_topk, torch_bits

pytestmark = pytest.mark.gpu

DIMS = W.Dims(hidden=512, n_q=32, n_kv=8, head_dim=128, n_r=8, d_r=128, rope_base=1e6)


@pytest.fixture(scope="module")
def msa(cuda_device):
    import long_context_memory_b200 as m

    return m


def _dev(a, device):
    return W.to_torch(np.ascontiguousarray(a)).to(device)


def _layer(rng, d, C, B, t_loc):
    """One layer instance's inputs (bf16 bits): memory, router weights, query, local KV before RoPE, new token."""
    return dict(KR=W.normal_bf16(rng, (C, d.n_r, d.d_r)), K_bar=W.normal_bf16(rng, (C, d.n_kv, d.head_dim)),
                V_bar=W.normal_bf16(rng, (C, d.n_kv, d.head_dim)), Hq=W.normal_bf16(rng, (B, d.hidden)),
                W_QR=W.normal_bf16(rng, (d.hidden, d.n_r * d.d_r), 1 / math.sqrt(d.hidden)),
                q=W.normal_bf16(rng, (B, d.n_q, d.head_dim)),
                K_loc=W.normal_bf16(rng, (B, t_loc, d.n_kv, d.head_dim)),
                V_loc=W.normal_bf16(rng, (B, t_loc, d.n_kv, d.head_dim)),
                k_new=W.normal_bf16(rng, (B, d.n_kv, d.head_dim)), v_new=W.normal_bf16(rng, (B, d.n_kv, d.head_dim)))


def _rotated_cache(msa, d, K_loc_bits, pos_offset, device):
    """The local cache the tiered call reads: every key rotated at its global position."""
    import torch

    B, T = K_loc_bits.shape[:2]
    K = _dev(K_loc_bits, device)
    pos = (pos_offset + torch.arange(T, dtype=torch.int32, device=device)).repeat(B)
    msa.rope_rows(d, K.view(B * T, d.n_kv, d.head_dim), pos)
    return K


# Few documents: the transfers are the longer part and the gather of each layer starts as soon as
# its routing is done.  5,000 short documents at B = 1: the scans are the longer part, so the router
# queries of every layer run first, the scans follow one another, and the selections (two slices
# of documents, merged by the last slice CTA), gathers and attentions run on the copy stream; the
# two routing workspaces are reused and cleared between layers.
@pytest.mark.parametrize("B,n_layers,copy,n_docs,max_len", [(1, 3, True, 120, 3000), (3, 4, True, 120, 3000),
                                                             (2, 3, False, 120, 3000), (1, 5, True, 5000, 600)])
def test_tiered_decode_equals_single_calls_and_oracle(msa, cuda_device, B, n_layers, copy, n_docs, max_len):
    import torch

    dev, d, k, t_loc = cuda_device, DIMS, 16, 300
    rng = np.random.default_rng(500 + 10 * B + n_layers)
    lens = rng.integers(1, max_len, size=n_docs)
    doc_off = W.offsets_from_lengths(lens)
    co, *_ = O.chunk_layout(doc_off)
    C, n_docs = int(co[-1]), len(lens)
    loc_len = rng.integers(1, t_loc + 1, size=B).astype(np.int32)
    loc_len[0] = t_loc
    chunk_off = torch.from_numpy(co.astype(np.int32)).to(dev)
    ll = torch.from_numpy(loc_len).to(dev)
    cap = B * k * int(np.max(co[1:] - co[:-1]))
    layers = [_layer(rng, d, C, B, t_loc) for _ in range(n_layers)]
    tl, single = [], []
    for x in layers:
        base = dict(Hq=_dev(x["Hq"], dev), W_QR=_dev(x["W_QR"], dev), KR_bar=_dev(x["KR"], dev),
                    K_bar_host=W.to_torch(x["K_bar"]).pin_memory(), V_bar_host=W.to_torch(x["V_bar"]).pin_memory(),
                    q=_dev(x["q"], dev), k_new=_dev(x["k_new"], dev), v_new=_dev(x["v_new"], dev))
        base["kr_inv_norm"] = msa.router_key_norms(d, base["KR_bar"])
        Krot = _rotated_cache(msa, d, x["K_loc"], k, dev)
        a = dict(base, K_loc=Krot.clone(), V_loc=_dev(x["V_loc"], dev),
                 topk_idx=torch.empty((B, k), dtype=torch.int32, device=dev),
                 topk_score=torch.empty((B, k), dtype=torch.float32, device=dev),
                 out=torch.empty((B, d.n_q, d.head_dim), dtype=torch.bfloat16, device=dev))
        tl.append(a)
        single.append(dict(a, K_loc=Krot.clone(), V_loc=_dev(x["V_loc"], dev)))
    S = torch.cuda.Stream(device=dev)
    Cs = torch.cuda.Stream(device=dev) if copy else None
    torch.cuda.synchronize()
    msa.tiered_decode(d, tl, B, chunk_off, C, k, ll, t_loc, k, cap, stream=S, copy_stream=Cs)
    torch.cuda.synchronize()
    assert msa.check_device_errors() == 0
    for l, (x, a, s1) in enumerate(zip(layers, tl, single)):
        # the same results as the single calls, bit for bit
        idx, sc, _ = msa.route_topk(d, s1["Hq"], s1["W_QR"], s1["KR_bar"], chunk_off, k, kr_inv_norm=s1["kr_inv_norm"])
        Ks, Vs, soff, sidx = msa.gather_kv(d, s1["K_bar_host"], s1["V_bar_host"], chunk_off, idx, cap)
        out = msa.sparse_attend(d, s1["q"], Ks, Vs, soff, sidx, s1["K_loc"], s1["V_loc"], ll, k,
                                k_loc_rotated=True, k_new=s1["k_new"], v_new=s1["v_new"])
        torch.cuda.synchronize()
        assert msa.check_device_errors() == 0
        assert torch.equal(a["topk_idx"], idx) and torch.equal(a["topk_score"], sc), f"layer {l}"
        assert torch.equal(a["out"], out), f"layer {l}"
        assert torch.equal(a["K_loc"], s1["K_loc"]) and torch.equal(a["V_loc"], s1["V_loc"]), f"layer {l}"
        # and the oracle's: routing over every document, attention over the selected ones
        s, _, _ = O.route_topk(O.router_query(x["Hq"], x["W_QR"], d.n_r, d.d_r), x["KR"], co, k)
        g_idx, g_sc = a["topk_idx"].cpu().numpy(), a["topk_score"].cpu().numpy()
        for b in range(B):
            check_topk(g_idx[b], g_sc[b], s[b], k, where=f"layer {l} b={b}")
        K_or, V_or = x["K_loc"].copy(), x["V_loc"].copy()
        for b in range(B):  # the appended token sits at the query's own slot, loc_len - 1
            K_or[b, loc_len[b] - 1] = x["k_new"][b]
            V_or[b, loc_len[b] - 1] = x["v_new"][b]
        ref = O.sparse_attend(x["q"], x["K_bar"], x["V_bar"], co, g_idx, K_or, V_or, loc_len, k, d.rope_base)
        check_attention(a["out"].float().cpu().numpy(), ref, where=f"tiered layer {l}")


def test_tiered_decode_rejects_bad_layers(msa, cuda_device):
    import torch

    d, dev = DIMS, cuda_device
    co = torch.tensor([0, 4, 8], dtype=torch.int32, device=dev)
    ll = torch.tensor([4], dtype=torch.int32, device=dev)
    x = dict(Hq=torch.zeros((1, d.hidden), dtype=torch.bfloat16, device=dev),
             KR_bar=torch.zeros((8, d.n_r, d.d_r), dtype=torch.bfloat16, device=dev),
             K_bar_host=torch.zeros((8, d.n_kv, d.head_dim), dtype=torch.bfloat16),  # pageable: refused
             V_bar_host=torch.zeros((8, d.n_kv, d.head_dim), dtype=torch.bfloat16),
             q=torch.zeros((1, d.n_q, d.head_dim), dtype=torch.bfloat16, device=dev),
             K_loc=torch.zeros((1, 4, d.n_kv, d.head_dim), dtype=torch.bfloat16, device=dev),
             V_loc=torch.zeros((1, 4, d.n_kv, d.head_dim), dtype=torch.bfloat16, device=dev),
             topk_idx=torch.zeros((1, 1), dtype=torch.int32, device=dev),
             topk_score=torch.zeros((1, 1), dtype=torch.float32, device=dev),
             out=torch.zeros((1, d.n_q, d.head_dim), dtype=torch.bfloat16, device=dev))
    with pytest.raises(msa.MSAError) as e:
        msa.tiered_decode(d, [x], 1, co, 8, 1, ll, 4, 1, 8)
    assert e.value.code == 1 and "pinned" in str(e.value)
    y = dict(x, K_bar_host=x["K_bar_host"].pin_memory(), V_bar_host=x["V_bar_host"].pin_memory(), k_new=x["q"])
    with pytest.raises(msa.MSAError) as e:
        msa.tiered_decode(d, [y], 1, co, 8, 1, ll, 4, 1, 8)
    assert e.value.code == 1 and "k_new and v_new" in str(e.value)


# ----------------------------------------------------------------------------
# the 100M-token memory (lognormal documents, median 4096): routing and the host tier at full size
# ----------------------------------------------------------------------------
T100M = 100_000_000
PLANT_COS = 0.25 + 0.01 * np.arange(16)   # per-head cosines of the planted chunks: ~0.06 above the
                                          # background maximum (about 0.03125 * sqrt(2 ln C) = 0.167)


@pytest.fixture(scope="module")
def mem100m(msa, cuda_device):
    """Router keys of a 100M-token layer on the device (torch's seeded generator), with 16 planted
    documents for each of 16 queries, and those queries' router vectors Q^R (bf16 bits)."""
    import torch

    d = W.QWEN3_4B_DIMS
    rng = np.random.default_rng(W.BASE_SEED + 4)
    lens = W.doc_lengths_lognormal(rng, T100M, 4096)
    doc_off = W.offsets_from_lengths(lens)
    co, *_ = O.chunk_layout(doc_off)
    C, N = int(co[-1]), len(lens)
    g = torch.Generator(device=cuda_device)
    g.manual_seed(W.BASE_SEED + 4)
    KR = torch.empty((C, d.n_r, d.d_r), dtype=torch.bfloat16, device=cuda_device)
    flat = KR.view(-1)
    for i in range(0, flat.numel(), 1 << 26):
        e = min(flat.numel(), i + (1 << 26))
        flat[i:e] = torch.randn(e - i, generator=g, device=cuda_device).to(torch.bfloat16)
    B = 16
    planted = rng.permutation(N)[:B * 16].reshape(B, 16)
    QR = np.zeros((B, d.n_r * d.d_r), dtype=np.uint16)
    for b in range(B):
        u = W._unit(rng, d.n_r, d.d_r)
        QR[b] = W.f32_to_bf16_bits((u * rng.uniform(0.5, 2.0, (d.n_r, 1)) * math.sqrt(d.d_r)).astype(np.float32)
                                   ).reshape(-1)
        for p in range(16):
            doc = int(planted[b, p])
            ch = int(co[doc] + rng.integers(0, co[doc + 1] - co[doc]))
            rows = W._planted_rows(rng, u, np.full(d.n_r, PLANT_COS[p]), d.d_r)
            KR[ch] = W.to_torch(W.f32_to_bf16_bits(rows.astype(np.float32))).to(cuda_device)
    torch.cuda.synchronize()
    return dict(d=d, co=co, C=C, N=N, KR=KR, QR=QR, planted=planted, doc_off=doc_off,
                chunk_off=torch.from_numpy(co.astype(np.int32)).to(cuda_device))


def _oracle_doc_scores(m, QR_b, docs):
    """The oracle's document scores of `docs` for router queries QR_b [B, n_r, d_r] (float64), from
    the documents' own router-key rows (a document's score depends on its chunks alone)."""
    import torch

    co = m["co"]
    docs = np.asarray(docs)
    rows = np.concatenate([np.arange(co[i], co[i + 1]) for i in docs])
    KR = torch_bits(m["KR"][torch.from_numpy(rows).to(m["KR"].device)])
    sub = np.concatenate([[0], np.cumsum(co[docs + 1] - co[docs])])
    s, _, _ = O.route_topk(QR_b, KR, sub, 1)
    return s


def test_route_100m_b1_every_document(msa, cuda_device, mem100m):
    # the headline configuration's routing: every document score and the top-16 against the oracle
    import torch

    m, d, k = mem100m, mem100m["d"], 16
    inv = msa.router_key_norms(d, m["KR"])
    idx, sc, ds = msa.route_topk(d, _dev(m["QR"][:1], cuda_device), None, m["KR"], m["chunk_off"], k,
                                 want_doc_scores=True, kr_inv_norm=inv)
    torch.cuda.synchronize()
    assert msa.check_device_errors() == 0
    QR = O.bf16_to_f64(m["QR"][:1]).reshape(1, d.n_r, d.d_r)
    s = np.empty((1, m["N"]))
    step = 1500  # documents per oracle call (about 100K chunks)
    for a in range(0, m["N"], step):
        docs = np.arange(a, min(m["N"], a + step))
        s[:, docs] = _oracle_doc_scores(m, QR, docs)
    ds = ds.cpu().numpy()
    assert np.max(np.abs(ds - s)) < SCORE_ATOL, np.max(np.abs(ds - s))
    check_topk(idx.cpu().numpy()[0], sc.cpu().numpy()[0], s[0], k, where="100M b=0")
    # the planted documents are the top-16, strongest first
    assert idx.cpu().numpy()[0].tolist() == m["planted"][0][::-1].tolist()


def test_route_100m_b16_sampled(msa, cuda_device, mem100m):
    # 16 queries routed together: the planted documents exactly, ~600 sampled document scores
    import torch

    m, d, k, B = mem100m, mem100m["d"], 16, 16
    idx, sc, ds = msa.route_topk(d, _dev(m["QR"], cuda_device), None, m["KR"], m["chunk_off"], k,
                                 want_doc_scores=True)
    torch.cuda.synchronize()
    assert msa.check_device_errors() == 0
    idx, sc, ds = idx.cpu().numpy(), sc.cpu().numpy(), ds.cpu().numpy()
    QR = O.bf16_to_f64(m["QR"]).reshape(B, d.n_r, d.d_r)
    rng = np.random.default_rng(7)
    sample = np.unique(np.concatenate([rng.choice(m["N"], 600, replace=False), m["planted"].reshape(-1)]))
    s = _oracle_doc_scores(m, QR, sample)
    assert np.max(np.abs(ds[:, sample] - s)) < SCORE_ATOL, np.max(np.abs(ds[:, sample] - s))
    pos = {int(doc): i for i, doc in enumerate(sample)}
    for b in range(B):
        want = m["planted"][b][::-1]
        assert idx[b].tolist() == want.tolist(), f"b={b}"
        o = s[b, [pos[int(x)] for x in want]]
        assert np.all(np.abs(sc[b] - o) < SCORE_ATOL)
        assert np.all(o[:-1] - o[1:] > TOPK_GAP)
        # every other document scores below the weakest planted one by more than the gap
        others = np.delete(ds[b], want)
        assert others.max() < o[-1] - TOPK_GAP


def test_tiered_decode_100m_host_tier(msa, cuda_device, mem100m):
    # the bench's layer at full size: K̄/V̄ of the whole 100M-token memory in pinned host memory,
    # the 16 routed documents (~64 chunks each) gathered and attended with an 8K-token local cache
    import torch

    m, d, k, B, t_loc = mem100m, mem100m["d"], 16, 1, 8192
    dev = cuda_device
    C = m["C"]
    g = torch.Generator(device=dev)
    g.manual_seed(11)
    shape = (C, d.n_kv, d.head_dim)
    host = []
    for _ in range(2):
        h = torch.empty(shape, dtype=torch.bfloat16, pin_memory=True)
        for a in range(0, C, 1 << 16):
            e = min(C, a + (1 << 16))
            h[a:e].copy_(torch.randn((e - a,) + shape[1:], generator=g, device=dev).to(torch.bfloat16))
        host.append(h)
    rng = np.random.default_rng(12)
    q = W.normal_bf16(rng, (B, d.n_q, d.head_dim))
    K_loc = W.normal_bf16(rng, (B, t_loc, d.n_kv, d.head_dim))
    V_loc = W.normal_bf16(rng, (B, t_loc, d.n_kv, d.head_dim))
    k_new, v_new = W.normal_bf16(rng, (B, d.n_kv, d.head_dim)), W.normal_bf16(rng, (B, d.n_kv, d.head_dim))
    L = dict(Hq=_dev(m["QR"][:B], dev), W_QR=None, KR_bar=m["KR"], kr_inv_norm=None, K_bar_host=host[0],
             V_bar_host=host[1], q=_dev(q, dev), K_loc=_rotated_cache(msa, d, K_loc, k, dev), V_loc=_dev(V_loc, dev),
             k_new=_dev(k_new, dev), v_new=_dev(v_new, dev),
             topk_idx=torch.empty((B, k), dtype=torch.int32, device=dev),
             topk_score=torch.empty((B, k), dtype=torch.float32, device=dev),
             out=torch.empty((B, d.n_q, d.head_dim), dtype=torch.bfloat16, device=dev))
    ll = torch.full((B,), t_loc, dtype=torch.int32, device=dev)
    co = m["co"]
    cap = B * k * int(np.max(co[1:] - co[:-1]))
    S, Cs = torch.cuda.Stream(device=dev), torch.cuda.Stream(device=dev)
    torch.cuda.synchronize()
    msa.tiered_decode(d, [L], B, m["chunk_off"], C, k, ll, t_loc, k, cap, stream=S, copy_stream=Cs)
    torch.cuda.synchronize()
    assert msa.check_device_errors() == 0
    sel = L["topk_idx"].cpu().numpy()
    assert sel[0].tolist() == m["planted"][0][::-1].tolist()
    # the oracle over the selected documents' rows (read from the host tier) and the local cache
    rows = np.concatenate([np.arange(co[i], co[i + 1]) for i in sel[0]])
    Kb = torch_bits(host[0][torch.from_numpy(rows)])
    Vb = torch_bits(host[1][torch.from_numpy(rows)])
    sub = np.concatenate([[0], np.cumsum(co[sel[0] + 1] - co[sel[0]])])
    assert 300 <= sub[-1] <= 16 * 512, sub[-1]  # ~64 chunks per routed document
    K_or, V_or = K_loc.copy(), V_loc.copy()
    K_or[0, t_loc - 1], V_or[0, t_loc - 1] = k_new[0], v_new[0]
    ref = O.sparse_attend(q, Kb, Vb, sub, np.arange(k)[None], K_or, V_or, np.full(B, t_loc), k, d.rope_base)
    check_attention(L["out"].float().cpu().numpy(), ref, where="100M host tier")
