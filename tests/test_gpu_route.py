"""GPU parity of stage 2 (routing + top-k) against the CPU oracle, through the C ABI."""
import numpy as np
import pytest

import oracle as O
from long_context_memory_b200 import workloads as W
from helpers import SCORE_ATOL, bf16_of, check_topk


def LAYOUT(doc_off):
    """The oracle's chunk layout (the generator takes the layout from its caller)."""
    return O.chunk_layout(doc_off)[0]


pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def msa(cuda_device):
    import long_context_memory_b200 as m

    return m


def _dev(a, device):
    import torch

    return W.to_torch(np.ascontiguousarray(a)).to(device)


def _route_case(seed, n_docs, B, n_r, d_r, lo=1, hi=700, hidden=256):
    rng = np.random.default_rng(seed)
    lens = rng.integers(lo, hi + 1, size=n_docs)
    doc_off = W.offsets_from_lengths(lens)
    chunk_off, C = None, None
    dims = W.Dims(hidden=hidden, n_q=8, n_kv=2, head_dim=64, n_r=n_r, d_r=d_r)
    co, *_ = O.chunk_layout(doc_off)
    C = int(co[-1])
    KR = W.normal_bf16(rng, (C, n_r, d_r))
    QR = W.normal_bf16(rng, (B, n_r * d_r))
    Hq = W.normal_bf16(rng, (B, hidden))
    Wqr = W.normal_bf16(rng, (hidden, n_r * d_r), 1 / np.sqrt(hidden))
    return dims, doc_off, KR, QR, Hq, Wqr, rng


def _run(msa, dims, Hq, Wqr, KR, doc_off, k, agg, device, head_major=False):
    import torch

    co, C = msa.chunk_offsets(doc_off)
    kr = np.ascontiguousarray(KR.transpose(1, 0, 2)) if head_major else KR
    idx, sc, ds = msa.route_topk(dims, _dev(Hq, device), None if Wqr is None else _dev(Wqr, device),
                                 _dev(kr, device), torch.from_numpy(co).to(device), k, agg=agg, want_doc_scores=True,
                                 kr_head_major=head_major)
    torch.cuda.synchronize()
    assert msa.check_device_errors() == 0
    return idx.cpu().numpy(), sc.cpu().numpy(), ds.cpu().numpy()


@pytest.mark.parametrize("B", [1, 3, 8, 13, 32, 40])
@pytest.mark.parametrize("n_r,d_r", [(8, 128), (4, 64), (3, 128)])
def test_route_direct_query_parity(msa, cuda_device, B, n_r, d_r):
    dims, doc_off, KR, QR, Hq, Wqr, _ = _route_case(100 + B + n_r, 300, B, n_r, d_r)
    k = 16
    idx, sc, ds = _run(msa, dims, QR, None, KR, doc_off, k, msa.AGG_MAX, cuda_device)
    co, *_ = O.chunk_layout(doc_off)
    s, _, _ = O.route_topk(O.bf16_to_f64(QR).reshape(B, n_r, d_r), KR, co, k)
    assert np.max(np.abs(ds - s)) < SCORE_ATOL, np.max(np.abs(ds - s))
    for b in range(B):
        check_topk(idx[b], sc[b], s[b], k, where=f"b={b}")


@pytest.mark.parametrize("norms", [False, True])
def test_route_zero_norm_heads(msa, cuda_device, norms):
    # zero router-key head rows, a zero query head and an all-zero query: the clamped norms make
    # every cosine with a zero vector 0 (scan norms, precomputed norms, query normalisation)
    import torch

    B, k = 3, 16
    dims, doc_off, KR, QR, Hq, Wqr, rng = _route_case(31 + norms, 200, B, 8, 128)
    co, C = msa.chunk_offsets(doc_off)
    KR, QR = KR.copy(), QR.copy().reshape(B, 8, 128)
    for j in rng.choice(C, 300, replace=False):
        KR[j, rng.integers(0, 8)] = 0
    KR[5] = 0          # a chunk with every head zero
    QR[1, 2] = 0       # one zero head of query 1
    QR[2] = 0          # query 2 entirely zero: every document scores 0, ties to the lower ids
    kr = _dev(KR, cuda_device)
    inv = msa.router_key_norms(dims, kr) if norms else None
    idx, sc, ds = msa.route_topk(dims, _dev(QR.reshape(B, -1), cuda_device), None, kr,
                                 torch.from_numpy(co).to(cuda_device), k, want_doc_scores=True, kr_inv_norm=inv)
    torch.cuda.synchronize()
    assert msa.check_device_errors() == 0
    idx, sc, ds = idx.cpu().numpy(), sc.cpu().numpy(), ds.cpu().numpy()
    co_o, *_ = O.chunk_layout(doc_off)
    s, _, _ = O.route_topk(O.bf16_to_f64(QR), KR, co_o, k)
    assert np.all(np.isfinite(ds))
    assert np.max(np.abs(ds - s)) < SCORE_ATOL, np.max(np.abs(ds - s))
    for b in range(B):
        check_topk(idx[b], sc[b], s[b], k, where=f"b={b}")
    assert np.all(ds[2] == 0.0) and idx[2].tolist() == list(range(k))
    # the projection path: a zero hidden state gives a zero router query in every head
    Hz = Hq.copy()
    Hz[1] = 0
    idx2, _, ds2 = msa.route_topk(dims, _dev(Hz, cuda_device), _dev(Wqr, cuda_device), kr,
                                  torch.from_numpy(co).to(cuda_device), k, want_doc_scores=True, kr_inv_norm=inv)
    torch.cuda.synchronize()
    assert np.all(ds2.cpu().numpy()[1] == 0.0) and idx2.cpu().numpy()[1].tolist() == list(range(k))


@pytest.mark.parametrize("agg", [0, 1])
def test_route_projection_and_aggregation(msa, cuda_device, agg):
    B = 5
    dims, doc_off, KR, QR, Hq, Wqr, _ = _route_case(7, 257, B, 8, 128, hidden=512)
    k = 9
    idx, sc, ds = _run(msa, dims, Hq, Wqr, KR, doc_off, k, agg, cuda_device)
    co, *_ = O.chunk_layout(doc_off)
    QRo = O.router_query(Hq, Wqr, 8, 128)
    S = O.chunk_scores(QRo, KR)
    s = O.doc_scores(S, co, "max" if agg == 0 else "mean")
    assert np.max(np.abs(ds - s)) < SCORE_ATOL
    for b in range(B):
        check_topk(idx[b], sc[b], s[b], k, where=f"agg={agg} b={b}")


@pytest.mark.parametrize("B", [1, 13, 40])
@pytest.mark.parametrize("n_r,d_r", [(8, 128), (3, 128), (4, 64)])
def test_route_head_major_keys(msa, cuda_device, B, n_r, d_r):
    # K̄^R stored [n_r, C, d_r]: same products in the same order, so the scores are the chunk-major ones, bit for bit
    dims, doc_off, KR, QR, Hq, Wqr, _ = _route_case(300 + B + n_r, 211, B, n_r, d_r)
    k = 12
    idx, sc, ds = _run(msa, dims, QR, None, KR, doc_off, k, msa.AGG_MAX, cuda_device, head_major=True)
    co, *_ = O.chunk_layout(doc_off)
    s, _, _ = O.route_topk(O.bf16_to_f64(QR).reshape(B, n_r, d_r), KR, co, k)
    assert np.max(np.abs(ds - s)) < SCORE_ATOL, np.max(np.abs(ds - s))
    for b in range(B):
        check_topk(idx[b], sc[b], s[b], k, where=f"b={b}")
    idx0, sc0, ds0 = _run(msa, dims, QR, None, KR, doc_off, k, msa.AGG_MAX, cuda_device)
    assert np.array_equal(ds, ds0) and np.array_equal(idx, idx0) and np.array_equal(sc, sc0)


@pytest.mark.parametrize("agg", [0, 1])
def test_route_fused_topk_matches_separate_kernels(msa, cuda_device, agg):
    # up to 4 queries over one slice of documents take the top-k inside the scan's last CTA;
    # 5 queries take the separate top-k kernel: the first 4 queries' results must agree exactly
    dims, doc_off, KR, QR, Hq, Wqr, _ = _route_case(41 + agg, 500, 5, 8, 128)
    i4, s4, d4 = _run(msa, dims, QR[:4], None, KR, doc_off, 16, agg, cuda_device)
    i5, s5, d5 = _run(msa, dims, QR, None, KR, doc_off, 16, agg, cuda_device)
    assert np.array_equal(i4, i5[:4]) and np.array_equal(s4, s5[:4]) and np.array_equal(d4, d5[:4])
    co, *_ = O.chunk_layout(doc_off)
    s, _, _ = O.route_topk(O.bf16_to_f64(QR).reshape(5, 8, 128), KR, co, 16, "max" if agg == 0 else "mean")
    for b in range(4):
        check_topk(i4[b], s4[b], s[b], 16, where=f"b={b}")


@pytest.mark.parametrize("head_major", [False, True])
@pytest.mark.parametrize("B,n_r,d_r", [(1, 8, 128), (13, 4, 64), (32, 3, 128)])
def test_route_with_precomputed_key_norms(msa, cuda_device, head_major, B, n_r, d_r):
    # inverse norms computed once (msa_router_key_norms) and passed to the scan
    import torch

    dims, doc_off, KR, QR, *_ = _route_case(700 + B + n_r, 400, B, n_r, d_r)
    co, C = msa.chunk_offsets(doc_off)
    kr = np.ascontiguousarray(KR.transpose(1, 0, 2)) if head_major else KR
    krd = _dev(kr, cuda_device)
    inv = msa.router_key_norms(dims, krd, kr_head_major=head_major)
    co_d = torch.from_numpy(co).to(cuda_device)
    idx, sc, ds = msa.route_topk(dims, _dev(QR, cuda_device), None, krd, co_d, 12, want_doc_scores=True,
                                 kr_head_major=head_major, kr_inv_norm=inv)
    _, _, ds0 = msa.route_topk(dims, _dev(QR, cuda_device), None, krd, co_d, 12, want_doc_scores=True,
                               kr_head_major=head_major)
    torch.cuda.synchronize()
    assert msa.check_device_errors() == 0
    want = 1.0 / np.maximum(np.sqrt((O.bf16_to_f64(KR) ** 2).sum(-1)), O.EPS)   # [C, n_r]
    assert np.allclose(inv.cpu().numpy(), want, rtol=2e-6, atol=0)
    ds, ds0 = ds.cpu().numpy(), ds0.cpu().numpy()
    assert np.max(np.abs(ds - ds0)) < 1e-5          # the same norms up to fp32 summation order
    s, _, _ = O.route_topk(O.bf16_to_f64(QR).reshape(B, n_r, d_r), KR, co, 12)
    assert np.max(np.abs(ds - s)) < SCORE_ATOL
    idx, sc = idx.cpu().numpy(), sc.cpu().numpy()
    for b in range(B):
        check_topk(idx[b], sc[b], s[b], 12, where=f"b={b}")


def test_route_edge_shapes(msa, cuda_device):
    # one-chunk docs, k = n_docs, chunk count not a multiple of the tile, single doc
    for seed, n_docs, lo, hi, k in [(1, 17, 1, 64, 17), (2, 1, 5, 5, 1), (3, 40, 1, 1, 40), (4, 33, 60, 70, 1)]:
        dims, doc_off, KR, QR, *_ = _route_case(seed, n_docs, 2, 8, 128, lo=lo, hi=hi)
        idx, sc, ds = _run(msa, dims, QR, None, KR, doc_off, k, 0, cuda_device)
        co, *_ = O.chunk_layout(doc_off)
        s, _, _ = O.route_topk(O.bf16_to_f64(QR).reshape(2, 8, 128), KR, co, k)
        for b in range(2):
            check_topk(idx[b], sc[b], s[b], k, where=f"case {seed} b={b}")


def test_route_many_docs_two_pass_merge(msa, cuda_device):
    # > 4096 docs forces slice top-k + merge
    dims, doc_off, KR, QR, *_ = _route_case(11, 9000, 3, 4, 64, lo=1, hi=130)
    idx, sc, ds = _run(msa, dims, QR, None, KR, doc_off, 32, 0, cuda_device)
    co, *_ = O.chunk_layout(doc_off)
    s, _, _ = O.route_topk(O.bf16_to_f64(QR).reshape(3, 4, 64), KR, co, 32)
    assert np.max(np.abs(ds - s)) < SCORE_ATOL
    for b in range(3):
        check_topk(idx[b], sc[b], s[b], 32, where=f"b={b}")


def test_route_ties_prefer_lower_id(msa, cuda_device):
    # identical documents -> identical scores -> ids ascending
    rng = np.random.default_rng(5)
    dims = W.Dims(hidden=256, n_q=8, n_kv=2, head_dim=64, n_r=8, d_r=128)
    one = W.normal_bf16(rng, (3, 8, 128))
    KR = np.concatenate([one] * 50)
    doc_off = W.offsets_from_lengths(np.full(50, 150))        # 3 chunks each
    QR = W.normal_bf16(rng, (1, 1024))
    idx, sc, ds = _run(msa, dims, QR, None, KR, doc_off, 10, 0, cuda_device)
    assert list(idx[0]) == list(range(10))
    assert np.all(sc[0] == sc[0][0])


@pytest.mark.parametrize("n_docs,k", [(600, 32), (3000, 20), (4000, 1)])
def test_route_all_ties_every_selection_path(msa, cuda_device, n_docs, k):
    # every document identical: every score ties, the ids must come out ascending.  With
    # thousands of tied keys the warp-threshold selection sees too many candidates and hands
    # over to the sorting fallback; k = 32 fills a whole warp list
    rng = np.random.default_rng(6 + n_docs)
    dims = W.Dims(hidden=256, n_q=8, n_kv=2, head_dim=64, n_r=4, d_r=64)
    KR = np.concatenate([W.normal_bf16(rng, (1, 4, 64))] * n_docs)
    doc_off = W.offsets_from_lengths(np.full(n_docs, 64))        # one chunk each
    QR = W.normal_bf16(rng, (2, 256))
    idx, sc, ds = _run(msa, dims, QR, None, KR, doc_off, k, 0, cuda_device)
    for b in range(2):
        assert list(idx[b]) == list(range(k)), idx[b]
        assert np.all(sc[b] == sc[b][0])


@pytest.mark.parametrize("k", [31, 32, 33])
def test_route_k_at_the_selection_boundaries(msa, cuda_device, k):
    # k = 32 is the largest warp-list selection, 33 the smallest radix one
    dims, doc_off, KR, QR, *_ = _route_case(40 + k, 700, 3, 8, 128, lo=1, hi=300)
    idx, sc, ds = _run(msa, dims, QR, None, KR, doc_off, k, 0, cuda_device)
    co, *_ = O.chunk_layout(doc_off)
    s, _, _ = O.route_topk(O.bf16_to_f64(QR).reshape(3, 8, 128), KR, co, k)
    for b in range(3):
        check_topk(idx[b], sc[b], s[b], k, where=f"k={k} b={b}")


def test_route_planted_equal_key_scores_one(msa, cuda_device):
    dims, doc_off, KR, QR, *_ = _route_case(21, 100, 2, 8, 128)
    co, *_ = O.chunk_layout(doc_off)
    KR[co[37] + 0] = QR[0].reshape(8, 128)
    KR[co[81] + 0] = QR[1].reshape(8, 128)
    idx, sc, ds = _run(msa, dims, QR, None, KR, doc_off, 4, 0, cuda_device)
    assert idx[0, 0] == 37 and idx[1, 0] == 81
    assert abs(sc[0, 0] - 1.0) < 1e-5 and abs(sc[1, 0] - 1.0) < 1e-5
    assert np.all(np.abs(ds) <= 1.0 + 1e-5)


def test_route_tiny_config_full_pipeline(msa, cuda_device):
    c = W.tiny_config()
    d = c["dims"]
    _, _, KRb = O.encode_memory(c["H"], c["doc_off"], c["W_K"], c["W_V"], c["W_KR"], d.n_kv, d.head_dim, d.n_r, d.d_r)
    KR = bf16_of(KRb)
    idx, sc, ds = _run(msa, d, c["Hq"], c["W_QR"], KR, c["doc_off"], c["k"], 0, cuda_device)
    co, *_ = O.chunk_layout(c["doc_off"])
    s, _, _ = O.route_topk(O.router_query(c["Hq"], c["W_QR"], d.n_r, d.d_r), KR, co, c["k"])
    check_topk(idx[0], sc[0], s[0], c["k"])
    assert set(idx[0, :2].tolist()) == set(c["planted"])


def test_route_mem1m_full_size(msa, cuda_device):
    c = W.mem1m_config(LAYOUT, with_kv=False)
    d = c["dims"]
    idx, sc, ds = _run(msa, d, c["QR"], None, c["KR"], c["doc_off"], 16, 0, cuda_device)
    co, *_ = O.chunk_layout(c["doc_off"])
    s, _, _ = O.route_topk(O.bf16_to_f64(c["QR"]).reshape(1, d.n_r, d.d_r), c["KR"], co, 16)
    assert np.max(np.abs(ds - s)) < SCORE_ATOL
    check_topk(idx[0], sc[0], s[0], 16)
    assert set(idx[0].tolist()) == set(c["planted_docs"][0].tolist())
    # the projection path at full size
    idx2, sc2, ds2 = _run(msa, d, c["Hq"], c["W_QR"], c["KR"], c["doc_off"], 16, 0, cuda_device)
    s2, _, _ = O.route_topk(O.router_query(c["Hq"], c["W_QR"], d.n_r, d.d_r), c["KR"], co, 16)
    assert np.max(np.abs(ds2 - s2)) < SCORE_ATOL
    check_topk(idx2[0], sc2[0], s2[0], 16)


def test_route_mem16m_batch32_sampled(msa, cuda_device):
    c = W.mem16m_config(LAYOUT, with_kv=False)
    d = c["dims"]
    B = c["B"]
    idx, sc, ds = _run(msa, d, c["QR"], None, c["KR"], c["doc_off"], 16, 0, cuda_device)
    co, *_ = O.chunk_layout(c["doc_off"])
    rng = np.random.default_rng(0)
    sample = np.unique(np.concatenate([c["planted_docs"].ravel(), rng.choice(len(co) - 1, 600, replace=False)]))
    rows = np.concatenate([np.arange(co[i], co[i + 1]) for i in sample])
    S = O.chunk_scores(O.bf16_to_f64(c["QR"]).reshape(B, d.n_r, d.d_r), c["KR"], rows=rows)
    pos = 0
    for i in sample:
        n = co[i + 1] - co[i]
        s_i = S[:, pos:pos + n].max(axis=1)
        pos += n
        assert np.max(np.abs(ds[:, i] - s_i)) < SCORE_ATOL
    for b in range(B):
        # planted cosines 0.21 + 0.01 p: the top-16 are the planted docs, strongest first
        want = c["planted_docs"][b][::-1]
        assert list(idx[b]) == list(want), (b, idx[b], want)
        others = np.setdiff1d(np.arange(len(co) - 1), c["planted_docs"][b])
        assert ds[b, others].max() < sc[b, -1] - 2e-3


@pytest.mark.parametrize("projection", [True, False])
@pytest.mark.parametrize("B", [1, 5])
def test_route_early_inputs_behind_another_call(msa, cuda_device, projection, B):
    # routing launched right behind another library call with MSA_ROUTE_EARLY_INPUTS (the router
    # query multiplies and the scan streams before that call's kernel finishes): the same top-k,
    # scores and document scores, bit for bit, as the ordinary call
    import torch

    dims, doc_off, KR, QR, Hq, Wqr, rng = _route_case(300 + B, 900, B, 8, 128, lo=64, hi=4000, hidden=512)
    dev = cuda_device
    co, C = msa.chunk_offsets(doc_off)
    KR_d, co_d = _dev(KR, dev), torch.from_numpy(co).to(dev)
    inv = msa.router_key_norms(dims, KR_d)
    q_in = _dev(Hq, dev) if projection else _dev(QR, dev)
    w_in = _dev(Wqr, dev) if projection else None
    other = _dev(W.normal_bf16(rng, (20000, 8, 128)), dev)  # a busy preceding call on unrelated data
    res = []
    for early in (False, True, True):
        msa.router_key_norms(dims, other)
        res.append(msa.route_topk(dims, q_in, w_in, KR_d, co_d, 12, want_doc_scores=True, kr_inv_norm=inv,
                                  early_inputs=early))
    torch.cuda.synchronize()
    assert msa.check_device_errors() == 0
    for r in res[1:]:
        for a, b in zip(res[0], r):
            assert torch.equal(a, b)
