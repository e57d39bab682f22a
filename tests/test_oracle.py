"""Pins of the CPU oracle against things other than itself.

Closed forms, invariants, brute force on tiny inputs and hand-derived values
(tests/golden).  Each test is chosen so that a plausible mistake in the oracle
(a dropped term, a wrong sign or index, a transposed operand, a global instead
of a document-wise position) fails at least one of them.
"""
import json
import math
import os

import numpy as np
import pytest

import oracle as O
from long_context_memory_b200 import workloads as W

GOLD = os.path.join(os.path.dirname(__file__), "golden")


def _bits(x):
    return W.f32_to_bf16_bits(np.asarray(x, dtype=np.float32))


# ----------------------------------------------------------------------------
# bf16 widening
# ----------------------------------------------------------------------------
def test_bf16_widening_exact():
    vals = np.array([0.0, 1.0, -2.5, 3.140625, 65280.0, -1.0 / 128], dtype=np.float32)
    bits = _bits(vals)       # all exactly representable in bf16
    assert np.array_equal(O.bf16_to_f64(bits), vals.astype(np.float64))
    assert O.bf16_to_f64(np.array([0x3F80], dtype=np.uint16))[0] == 1.0
    assert O.bf16_to_f64(np.array([0xC000], dtype=np.uint16))[0] == -2.0


# ----------------------------------------------------------------------------
# chunk layout: brute force by walking every token
# ----------------------------------------------------------------------------
@pytest.mark.parametrize("lens", [[1, 63, 64, 65, 127, 128, 129, 200], [64], [5, 1, 3000]])
def test_chunk_layout_brute_force(lens):
    doc_off = W.offsets_from_lengths(np.asarray(lens))
    chunk_off, tok0, clen, owner = O.chunk_layout(doc_off, 64)
    # brute force: token t of doc i belongs to chunk number (t - start) // 64 of doc i
    counts = {}
    first = {}
    for i in range(len(lens)):
        for t in range(int(doc_off[i]), int(doc_off[i + 1])):
            key = (i, (t - int(doc_off[i])) // 64)
            counts[key] = counts.get(key, 0) + 1
            first.setdefault(key, t)
    keys = sorted(counts)
    assert len(keys) == len(tok0)
    for c, key in enumerate(keys):
        assert owner[c] == key[0]
        assert clen[c] == counts[key]
        assert tok0[c] == first[key]
    for i in range(len(lens)):
        assert chunk_off[i + 1] - chunk_off[i] == math.ceil(lens[i] / 64)
    assert chunk_off[-1] == len(tok0)


# ----------------------------------------------------------------------------
# RoPE
# ----------------------------------------------------------------------------
def test_rope_theta_endpoints():
    th = O.rope_theta(128, 1.0e6)
    assert th[0] == 1.0
    assert math.isclose(th[-1], 1.0e6 ** (-126 / 128), rel_tol=1e-14)
    assert np.all(np.diff(th) < 0)


def test_rope_matches_complex_multiplication():
    # rotate-half RoPE == multiplying z_i = x_i + i*x_{i+d/2} by exp(i*pos*theta_i)
    rng = np.random.default_rng(0)
    d = 64
    x = rng.standard_normal((5, d))
    pos = np.array([0, 1, 7, 1000, 123456])
    z = x[:, : d // 2] + 1j * x[:, d // 2:]
    theta = 10000.0 ** (-np.arange(0, d, 2) / d)
    zr = z * np.exp(1j * pos[:, None] * theta[None, :])
    want = np.concatenate([zr.real, zr.imag], axis=1)
    got = O.rope(x, pos, 10000.0)
    assert np.allclose(got, want, atol=1e-12)


def test_rope_invariants():
    rng = np.random.default_rng(1)
    x = rng.standard_normal((4, 128))
    assert np.array_equal(O.rope(x, np.zeros(4), 1e6), x)  # position 0 is the identity
    y = O.rope(x, np.array([3, 50, 999, 31999]), 1e6)
    assert np.allclose(np.linalg.norm(y, axis=1), np.linalg.norm(x, axis=1), rtol=1e-13)
    q, k = rng.standard_normal(128), rng.standard_normal(128)
    a = O.rope(q, 17, 1e6) @ O.rope(k, 5, 1e6)
    b = O.rope(q, 112, 1e6) @ O.rope(k, 100, 1e6)  # same offset m - n = 12
    assert math.isclose(a, b, rel_tol=1e-10, abs_tol=1e-10)


# ----------------------------------------------------------------------------
# encode
# ----------------------------------------------------------------------------
def _small_encode_case(seed=3, lens=(1, 63, 64, 65, 130, 7)):
    rng = np.random.default_rng(seed)
    lens = np.asarray(lens)
    doc_off = W.offsets_from_lengths(lens)
    T, hid = int(doc_off[-1]), 32
    H = W.normal_bf16(rng, (T, hid))
    WK = W.normal_bf16(rng, (hid, 2 * 16), 0.2)
    WV = W.normal_bf16(rng, (hid, 2 * 16), 0.2)
    WKR = W.normal_bf16(rng, (hid, 2 * 8), 0.2)
    return doc_off, H, WK, WV, WKR


def test_encode_pooling_matches_membership_matrix():
    # Brute force: build the 0/1 token->chunk membership matrix by walking tokens,
    # then V̄ = (M H / n) W_V and K̄^R = (M H / n) W^KR (pool first; exact by linearity).
    doc_off, H, WK, WV, WKR = _small_encode_case()
    Kb, Vb, KRb = O.encode_memory(H, doc_off, WK, WV, WKR, 2, 16, 2, 8, rope_base=1e4)
    T = int(doc_off[-1])
    rows = []
    for i in range(len(doc_off) - 1):
        s, e = int(doc_off[i]), int(doc_off[i + 1])
        for c0 in range(s, e, 64):
            r = np.zeros(T)
            r[c0:min(c0 + 64, e)] = 1.0
            rows.append(r / r.sum())
    M = np.asarray(rows)
    Hf = O.bf16_to_f64(H)
    assert np.allclose(Vb.reshape(len(M), -1), M @ Hf @ O.bf16_to_f64(WV), atol=1e-12)
    assert np.allclose(KRb.reshape(len(M), -1), M @ Hf @ O.bf16_to_f64(WKR), atol=1e-12)


def test_encode_k_uses_document_positions():
    # K̄ of chunk c = mean over its tokens of complex-rotated K rows at doc-relative position.
    doc_off, H, WK, WV, WKR = _small_encode_case()
    base = 1e4
    Kb, _, _ = O.encode_memory(H, doc_off, WK, WV, WKR, 2, 16, 2, 8, rope_base=base)
    Hf, Wk = O.bf16_to_f64(H), O.bf16_to_f64(WK)
    theta = base ** (-np.arange(0, 16, 2) / 16)
    c = 0
    for i in range(len(doc_off) - 1):
        s, e = int(doc_off[i]), int(doc_off[i + 1])
        for c0 in range(s, e, 64):
            acc = np.zeros((2, 16))
            n = 0
            for t in range(c0, min(c0 + 64, e)):
                k = (Hf[t] @ Wk).reshape(2, 16)
                z = (k[:, :8] + 1j * k[:, 8:]) * np.exp(1j * (t - s) * theta)
                acc += np.concatenate([z.real, z.imag], axis=1)
                n += 1
            assert np.allclose(Kb[c], acc / n, atol=1e-12)
            c += 1
    assert c == len(Kb)


def test_encode_single_token_doc_is_unrotated_projection():
    doc_off, H, WK, WV, WKR = _small_encode_case()
    Kb, Vb, KRb = O.encode_memory(H, doc_off, WK, WV, WKR, 2, 16, 2, 8)
    h0 = O.bf16_to_f64(H)[0]
    assert np.allclose(Kb[0].ravel(), h0 @ O.bf16_to_f64(WK), atol=1e-13)
    assert np.allclose(Vb[0].ravel(), h0 @ O.bf16_to_f64(WV), atol=1e-13)


def test_encode_doc_order_invariance():
    # positions reset per document, so permuting documents permutes their chunks only
    rng = np.random.default_rng(4)
    lens = np.array([70, 5, 130, 64])
    doc_off = W.offsets_from_lengths(lens)
    hid = 16
    Hd = [W.normal_bf16(rng, (int(L), hid)) for L in lens]
    WK, WV, WKR = (W.normal_bf16(rng, (hid, 32), 0.3) for _ in range(3))
    H = np.concatenate(Hd)
    K1, V1, R1 = O.encode_memory(H, doc_off, WK, WV, WKR, 2, 16, 2, 16)
    perm = [2, 0, 3, 1]
    H2 = np.concatenate([Hd[i] for i in perm])
    off2 = W.offsets_from_lengths(lens[perm])
    K2, V2, R2 = O.encode_memory(H2, off2, WK, WV, WKR, 2, 16, 2, 16)
    co1, *_ = O.chunk_layout(doc_off)
    co2, *_ = O.chunk_layout(off2)
    for new_i, old_i in enumerate(perm):
        a1, b1 = co1[old_i], co1[old_i + 1]
        a2, b2 = co2[new_i], co2[new_i + 1]
        assert np.allclose(K1[a1:b1], K2[a2:b2], atol=1e-12)
        assert np.allclose(V1[a1:b1], V2[a2:b2], atol=1e-12)
        assert np.allclose(R1[a1:b1], R2[a2:b2], atol=1e-12)


# ----------------------------------------------------------------------------
# routing
# ----------------------------------------------------------------------------
def test_route_hand_derived_golden():
    g = json.load(open(os.path.join(GOLD, "route_hand.json")))
    QR = np.asarray(g["query"])[None]               # [B=1, n_r=1, d_r=2]
    chunks, off = [], [0]
    for d in g["docs"]:
        chunks += d["chunks"]
        off.append(len(chunks))
    KR = np.asarray(chunks)[:, None, :]              # [C, 1, 2] float64 (exact)
    S = O.chunk_scores(QR, KR)
    assert np.allclose(S[0], g["chunk_scores"], atol=1e-15)
    smax = O.doc_scores(S, off, "max")[0]
    smean = O.doc_scores(S, off, "mean")[0]
    assert np.allclose(smax, g["doc_scores_max"], atol=1e-15)
    assert np.allclose(smean, g["doc_scores_mean"], atol=1e-15)
    assert list(O.topk(smax, 2)[0]) == g["top2_max"]
    assert list(O.topk(smean, 3)[0]) == g["top3_mean"]


def test_router_query_one_hot_rows_and_head_columns():
    # Q^R = H_q W^QR: a one-hot hidden state picks one row of W^QR; a sum of rows gives the
    # sum; router head h holds the columns [h d_r, (h + 1) d_r).  W^QR is not symmetric, so
    # a transposed operand or a head-major reshape gives other numbers.
    W_QR = np.arange(16, dtype=np.float64).reshape(4, 4)
    Hq = np.array([[0.0, 1.0, 0.0, 0.0], [1.0, 2.0, 0.0, 0.0]])
    QR = O.router_query(Hq, W_QR, 2, 2)
    assert QR.shape == (2, 2, 2)
    assert np.array_equal(QR[0], [[4.0, 5.0], [6.0, 7.0]])
    assert np.array_equal(QR[1], [[8.0, 11.0], [14.0, 17.0]])


def test_cosine_closed_forms_and_range():
    rng = np.random.default_rng(5)
    x = rng.standard_normal((10, 64))
    assert np.allclose(O.cosine(x, 3.5 * x), 1.0, atol=1e-14)
    assert np.allclose(O.cosine(x, -0.25 * x), -1.0, atol=1e-14)
    assert np.all(O.cosine(x, np.zeros_like(x)) == 0.0)
    y = rng.standard_normal((10, 64))
    c = O.cosine(x, y)
    assert np.all(np.abs(c) <= 1.0)
    # orthogonal pair
    e0, e1 = np.eye(64)[0], np.eye(64)[1]
    assert O.cosine(e0, e1) == 0.0


def test_planted_equal_key_scores_one_and_is_selected():
    rng = np.random.default_rng(6)
    n_r, d_r, C = 4, 32, 200
    QR = rng.standard_normal((1, n_r, d_r))
    KR = W.normal_bf16(rng, (C, n_r, d_r))
    off = np.arange(0, C + 1, 5)          # 40 docs of 5 chunks
    qbits = _bits(QR[0])
    KR[123] = qbits                        # planted: router key equal to the (bf16) query
    s, idx, val = O.route_topk(O.bf16_to_f64(qbits)[None], KR, off, k=3)
    assert abs(val[0, 0] - 1.0) < 1e-14
    assert idx[0, 0] == 123 // 5
    assert np.all(np.abs(s) <= 1.0 + 1e-15)


def test_head_mean_not_head_max():
    # two heads: cos 1 on head 0 and cos -1 on head 1 -> head mean 0
    QR = np.array([[[1.0, 0.0], [1.0, 0.0]]])
    KR = np.array([[[2.0, 0.0], [-1.0, 0.0]], [[0.0, 1.0], [1.0, 1.0]]])
    S = O.chunk_scores(QR, KR)
    assert np.allclose(S[0], [0.0, (0.0 + 1 / math.sqrt(2)) / 2], atol=1e-15)


def test_max_over_query_tokens():
    rng = np.random.default_rng(7)
    QR = rng.standard_normal((2, 3, 2, 16))          # B=2, M=3 tokens
    KR = rng.standard_normal((11, 2, 16))
    S = O.chunk_scores(QR, KR)
    per_t = np.stack([O.chunk_scores(QR[:, t], KR) for t in range(3)])
    assert np.array_equal(S, per_t.max(axis=0))


def test_max_vs_mean_aggregation_discriminates():
    # doc 0: one strong chunk among weak ones; doc 1: uniformly medium chunks
    QR = np.array([[[1.0, 0.0]]])
    KR = np.array([[[1.0, 0.0]], [[-1.0, 0.1]], [[-1.0, 0.1]], [[0.6, 0.8]], [[0.6, 0.8]]])
    off = [0, 3, 5]
    assert list(O.topk(O.doc_scores(O.chunk_scores(QR, KR), off, "max")[0], 1)[0]) == [0]
    assert list(O.topk(O.doc_scores(O.chunk_scores(QR, KR), off, "mean")[0], 1)[0]) == [1]


def test_route_topk_per_query_and_aggregation_by_hand():
    # the chunks of the aggregation case, two queries: (1, 0) and (0, 1).  Hand values:
    # query 0 scores the chunks 1, -1/sqrt(1.01) twice, 0.6 twice; query 1 scores them
    # 0, 0.1/sqrt(1.01) twice, 0.8 twice.
    QR = np.array([[[1.0, 0.0]], [[0.0, 1.0]]])
    KR = np.array([[[1.0, 0.0]], [[-1.0, 0.1]], [[-1.0, 0.1]], [[0.6, 0.8]], [[0.6, 0.8]]])
    off = [0, 3, 5]
    r = 1.0 / math.sqrt(1.01)
    s, idx, val = O.route_topk(QR, KR, off, 1, "max")
    assert np.allclose(s, [[1.0, 0.6], [0.1 * r, 0.8]], atol=1e-15)
    assert idx.tolist() == [[0], [1]] and np.allclose(val, [[1.0], [0.8]], atol=1e-15)
    s, idx, val = O.route_topk(QR, KR, off, 1, "mean")
    assert np.allclose(s, [[(1.0 - 2 * r) / 3, 0.6], [0.2 * r / 3, 0.8]], atol=1e-15)
    assert idx.tolist() == [[1], [1]]
    s, idx, _ = O.route_topk(QR, KR, off, 2, "max")
    assert idx.tolist() == [[0, 1], [1, 0]]


@pytest.mark.parametrize("seed", [0, 1, 2])
def test_topk_matches_pure_python_sort(seed):
    rng = np.random.default_rng(seed)
    s = np.round(rng.standard_normal(300), 1)        # many exact ties
    for k in (1, 5, 16, 64, 300):
        want = sorted(range(len(s)), key=lambda i: (-s[i], i))[:k]
        idx, val = O.topk(s, k)
        assert list(idx) == want
        assert np.array_equal(val, s[want])


# ----------------------------------------------------------------------------
# attention
# ----------------------------------------------------------------------------
def test_attention_closed_forms():
    rng = np.random.default_rng(8)
    d = 16
    q = rng.standard_normal(d)
    K1, V1 = rng.standard_normal((1, d)), rng.standard_normal((1, d))
    assert np.allclose(O.attention(q, K1, V1, 0.3), V1[0], atol=1e-15)
    Kc = np.repeat(rng.standard_normal((1, d)), 7, axis=0)
    V7 = rng.standard_normal((7, d))
    assert np.allclose(O.attention(q, Kc, V7, 0.3), V7.mean(axis=0), atol=1e-14)
    # two keys: weight of key 0 is the logistic of the logit difference
    K2 = rng.standard_normal((2, d))
    V2 = np.array([[1.0] + [0.0] * (d - 1), [0.0] * d])
    delta = 0.25 * (K2[0] - K2[1]) @ q
    w0 = 1.0 / (1.0 + math.exp(-delta))
    assert math.isclose(O.attention(q, K2, V2, 0.25)[0], w0, rel_tol=1e-13)
    # key permutation invariance
    K5, V5 = rng.standard_normal((5, d)), rng.standard_normal((5, d))
    p = [3, 1, 4, 0, 2]
    assert np.allclose(O.attention(q, K5, V5, 0.2), O.attention(q, K5[p], V5[p], 0.2), atol=1e-14)


def _attend_case(seed=9, n_q=8, n_kv=2, d=16, L=6, k=2):
    rng = np.random.default_rng(seed)
    lens = np.array([70, 3, 150, 64])
    chunk_off, *_ = O.chunk_layout(W.offsets_from_lengths(lens))
    C = int(chunk_off[-1])
    return dict(
        q=W.normal_bf16(rng, (1, n_q, d)), K_bar=W.normal_bf16(rng, (C, n_kv, d)),
        V_bar=W.normal_bf16(rng, (C, n_kv, d)), chunk_off=chunk_off,
        topk_idx=np.array([[2, 0]])[:, :k], K_loc=W.normal_bf16(rng, (1, 8, n_kv, d)),
        V_loc=W.normal_bf16(rng, (1, 8, n_kv, d)), loc_len=np.array([L]))


def test_attend_gqa_head_mapping():
    c = _attend_case()
    # V of KV head h is the constant h + 1 everywhere -> q head g must output g // 4 + 1
    c["V_bar"] = _bits(np.broadcast_to(np.array([1.0, 2.0])[None, :, None], c["V_bar"].shape))
    c["V_loc"] = _bits(np.broadcast_to(np.array([1.0, 2.0])[None, None, :, None], c["V_loc"].shape))
    out = O.sparse_attend(pos_offset=2, rope_base=1e4, **c)
    for g in range(8):
        assert np.allclose(out[0, g], g // 4 + 1.0, atol=1e-13)


def test_attend_local_positions_are_relative_to_query():
    # with all pooled keys zero, only relative local positions matter -> shifting the
    # global offset leaves the output unchanged
    c = _attend_case()
    c["K_bar"] = np.zeros_like(c["K_bar"])
    a = O.sparse_attend(pos_offset=2, rope_base=1e4, **c)
    b = O.sparse_attend(pos_offset=977, rope_base=1e4, **c)
    assert np.allclose(a, b, atol=1e-12)
    # but the rotation is really applied: dropping it changes the result
    c2 = dict(c)
    d = O.sparse_attend(pos_offset=2, rope_base=1e30, **c2)   # theta ~ 0 beyond i = 0
    assert not np.allclose(a, d, atol=1e-6)


def test_attend_pooled_key_logit_uses_only_query_rotation():
    # context = one pooled chunk key + one local key; read the softmax weight off V and
    # compare the logit gap with a complex-number evaluation of the two rotated dot products.
    d, base, o = 16, 1e4, 5
    rng = np.random.default_rng(10)
    q = _bits(rng.standard_normal((1, 1, d)))
    kb = _bits(rng.standard_normal((1, 1, d)))
    kl = _bits(rng.standard_normal((1, 3, 1, d)))
    vb = _bits(np.eye(d)[0][None, None])           # chunk value e0
    vl = np.zeros((1, 3, 1, d), dtype=np.uint16)   # local values 0
    out = O.sparse_attend(q, kb, vb, np.array([0, 1]), np.array([[0]]), kl, vl,
                          np.array([1]), pos_offset=o, rope_base=base, scale=0.5)
    w_chunk = out[0, 0, 0]
    theta = base ** (-np.arange(0, d, 2) / d)

    def rot(v, p):
        z = (v[: d // 2] + 1j * v[d // 2:]) * np.exp(1j * p * theta)
        return np.concatenate([z.real, z.imag])

    qf = O.bf16_to_f64(q)[0, 0]
    m = o + 1 - 1                                     # query = the only local token
    l_chunk = 0.5 * rot(qf, m) @ O.bf16_to_f64(kb)[0, 0]
    l_loc = 0.5 * rot(qf, m) @ rot(O.bf16_to_f64(kl)[0, 0, 0], o + 0)
    want = 1.0 / (1.0 + math.exp(l_loc - l_chunk))
    assert math.isclose(w_chunk, want, rel_tol=1e-12)


def test_attend_topk_order_irrelevant_and_matches_explicit_concat():
    c = _attend_case()
    a = O.sparse_attend(pos_offset=2, rope_base=1e4, **c)
    c2 = dict(c)
    c2["topk_idx"] = c["topk_idx"][:, ::-1]
    b = O.sparse_attend(pos_offset=2, rope_base=1e4, **c2)
    assert np.allclose(a, b, atol=1e-13)
    # context length = chunks of selected docs + local tokens
    K_ctx, V_ctx = O.sparse_context(c["K_bar"], c["V_bar"], c["chunk_off"], [2, 0],
                                    c["K_loc"][0], c["V_loc"][0], 6, 2, 1e4)
    co = c["chunk_off"]
    assert len(K_ctx) == (co[3] - co[2]) + (co[1] - co[0]) + 6


def test_attend_tokens_prefill_equals_sequence_of_decodes():
    # the M-token call masks a shared context; token t must equal a decode step that
    # simply has loc_len - M + t + 1 local tokens (a truncated context, no mask)
    c = _attend_case(L=7)
    rng = np.random.default_rng(12)
    M = 4
    q = W.normal_bf16(rng, (1, M, 8, 16))
    args = {k: v for k, v in c.items() if k != "q"}
    out = O.sparse_attend_tokens(q, pos_offset=3, rope_base=1e4, **args)
    for t in range(M):
        a2 = dict(args)
        a2["loc_len"] = np.array([7 - M + t + 1])
        dec = O.sparse_attend(q[:, t], pos_offset=3, rope_base=1e4, **a2)
        assert np.allclose(out[:, t], dec, atol=1e-13), t
    # M = 1 is the decode step itself
    one = O.sparse_attend_tokens(c["q"][:, None], pos_offset=3, rope_base=1e4, **args)
    assert np.allclose(one[:, 0], O.sparse_attend(pos_offset=3, rope_base=1e4, **c), atol=1e-13)


def test_attend_tokens_first_token_sees_chunk_and_first_local_key():
    # context: one pooled chunk key + 3 local keys; with M = 3 = loc_len, token 0 sees the chunk and
    # local key 0 only: its chunk weight is the two-key logistic of the rotated logits
    d, base, o = 16, 1e4, 2
    rng = np.random.default_rng(13)
    q = _bits(rng.standard_normal((1, 3, 1, d)))
    kb = _bits(rng.standard_normal((1, 1, d)))
    kl = _bits(rng.standard_normal((1, 3, 1, d)))
    vb = _bits(np.eye(d)[0][None, None])
    vl = np.zeros((1, 3, 1, d), dtype=np.uint16)
    out = O.sparse_attend_tokens(q, kb, vb, np.array([0, 1]), np.array([[0]]), kl, vl, np.array([3]),
                                 pos_offset=o, rope_base=base, scale=0.5)
    theta = base ** (-np.arange(0, d, 2) / d)

    def rot(v, p):
        z = (v[: d // 2] + 1j * v[d // 2:]) * np.exp(1j * p * theta)
        return np.concatenate([z.real, z.imag])

    qf = O.bf16_to_f64(q)[0, 0, 0]
    l_chunk = 0.5 * rot(qf, o) @ O.bf16_to_f64(kb)[0, 0]
    l_loc = 0.5 * rot(qf, o) @ rot(O.bf16_to_f64(kl)[0, 0, 0], o)
    want = 1.0 / (1.0 + math.exp(l_loc - l_chunk))
    assert math.isclose(out[0, 0, 0, 0], want, rel_tol=1e-12)
    # the last token sees all four keys: its chunk weight is strictly below token 0's unless
    # the extra local logits are -inf, which they are not
    assert 0.0 < out[0, 2, 0, 0] < 1.0


def test_attend_tokens_before_local_context_see_only_chunks():
    # loc_len < M: the first tokens come before every local key; they attend over the gathered
    # chunks alone (every chunk, none dropped), i.e. plain attention over the pooled rows
    c = _attend_case(L=2)
    rng = np.random.default_rng(14)
    M = 5
    q = W.normal_bf16(rng, (1, M, 8, 16))
    args = {k: v for k, v in c.items() if k != "q"}
    out = O.sparse_attend_tokens(q, pos_offset=3, rope_base=1e4, **args)
    co = c["chunk_off"]
    Kc = np.concatenate([O.bf16_to_f64(c["K_bar"])[co[i]:co[i + 1]] for i in (2, 0)])
    Vc = np.concatenate([O.bf16_to_f64(c["V_bar"])[co[i]:co[i + 1]] for i in (2, 0)])
    for t in range(M - 2):                       # own local index 2 - 5 + t < 0
        qr = O.rope(O.bf16_to_f64(q)[0, t], 3 + 2 - M + t, 1e4)
        for g in range(8):
            want = O.attention(qr[g], Kc[:, g // 4], Vc[:, g // 4], 1 / math.sqrt(16))
            assert np.allclose(out[0, t, g], want, atol=1e-13), (t, g)


# ----------------------------------------------------------------------------
# router training: L_aux forward and backward
# ----------------------------------------------------------------------------
def test_aux_loss_hand_derived_golden():
    g = json.load(open(os.path.join(GOLD, "aux_loss_hand.json")))
    Q = np.array(g["q"])[None, None]
    Kp = np.array(g["k_pos"])[None, None]
    Kn = np.array(g["k_neg"])[None, None, None]
    loss, dQ, dKp, dKn = O.aux_loss(Q, Kp, Kn, g["tau"])
    assert math.isclose(loss, g["loss"], rel_tol=1e-14)
    assert np.allclose(dQ[0, 0], g["dq"], atol=1e-15)
    assert np.allclose(dKp[0, 0], g["dk_pos"], atol=1e-15)
    assert np.allclose(dKn[0, 0, 0], g["dk_neg"], atol=1e-15)


def test_aux_loss_gradients_match_finite_differences():
    rng = np.random.default_rng(21)
    P, N, n_r, d_r, tau = 3, 4, 2, 5, 0.07
    Q = rng.standard_normal((P, n_r, d_r))
    Kp = Q + 0.5 * rng.standard_normal((P, n_r, d_r))
    Kn = rng.standard_normal((P, N, n_r, d_r))
    loss, dQ, dKp, dKn = O.aux_loss(Q, Kp, Kn, tau)
    eps = 1e-6
    for arr, grad in ((Q, dQ), (Kp, dKp), (Kn, dKn)):
        for _ in range(12):
            idx = tuple(rng.integers(0, n) for n in arr.shape)
            orig = arr[idx]
            arr[idx] = orig + eps
            lp = O.aux_loss(Q, Kp, Kn, tau)[0]
            arr[idx] = orig - eps
            lm = O.aux_loss(Q, Kp, Kn, tau)[0]
            arr[idx] = orig
            fd = (lp - lm) / (2 * eps)
            assert abs(fd - grad[idx]) <= 1e-7 * max(1.0, abs(fd)), (idx, fd, grad[idx])


def test_aux_loss_indistinguishable_negatives_and_batch_mean():
    rng = np.random.default_rng(22)
    P, N, n_r, d_r = 2, 6, 3, 8
    Q = rng.standard_normal((P, n_r, d_r))
    Kp = rng.standard_normal((P, n_r, d_r))
    Kn = np.repeat(Kp[:, None], N, axis=1) * 2.5      # same directions: every score equal
    loss, dQ, dKp, dKn = O.aux_loss(Q, Kp, Kn, 0.1)
    assert math.isclose(loss, math.log(N + 1), rel_tol=1e-13)
    assert np.allclose(dQ, 0.0, atol=1e-13)           # the positive's pull cancels the negatives' push
    # the loss over P positives is the mean of the single-positive losses
    Kn2 = rng.standard_normal((P, N, n_r, d_r))
    whole = O.aux_loss(Q, Kp, Kn2, 0.2)[0]
    parts = [O.aux_loss(Q[i:i + 1], Kp[i:i + 1], Kn2[i:i + 1], 0.2)[0] for i in range(P)]
    assert math.isclose(whole, sum(parts) / P, rel_tol=1e-13)


# ----------------------------------------------------------------------------
# pages' footprint arithmetic
# ----------------------------------------------------------------------------
def test_footprint_matches_pages():
    g = json.load(open(os.path.join(GOLD, "footprint.json")))
    lens = np.full(g["tokens"] // 4096, 4096)      # chunk count of 100M tokens in 4K docs
    chunks = int(np.sum((lens + g["chunk"] - 1) // g["chunk"]))
    per_tensor = chunks * g["heads"] * g["head_dim"] * g["bytes_per_elem"] * g["layers"]
    assert abs(per_tensor / 1e9 - g["router_keys_GB"]) / g["router_keys_GB"] < g["rel_tol"]
    assert abs(3 * per_tensor / 1e9 - g["total_GB"]) / g["total_GB"] < g["rel_tol"]
