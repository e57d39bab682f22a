"""CPU oracle for the Memory Sparse Attention (MSA) hot path.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` may import or run
anything in this package.  The product path (``long_context_memory_b200``)
never imports it and shares no code with it.

Plain, slow, obviously correct: float64 arithmetic on bf16 inputs widened
exactly to float64, scalar-style loops over documents and chunks, and library
matmuls as the only building block.  No blocking, fusion or reordering beyond
what the method's definition states.

Sources (cited by page and section):
  [digest]   "MSA: Memory Sparse Attention for Efficient End-to-End Memory Model
             Scaling to 100M Tokens", paper digest (rainbus.top), sections
             "Core method" and "Method step details".
  [IRMaD]    The same paper's structured reading (techblg.uk), section
             "M. Materials & Methods", items "routing and sparse attention",
             "position encoding", "three-stage inference".
  [news]     EverMind MSA release article (chooseai.io), sections 2.1-2.3.
  [overview] MSA project overview (zhichai.net), "three-stage inference
             pipeline" figure and "key technical details" item 1.

Readings adopted where the pages are silent or ambiguous (each one is listed
with its reason in the design notes):
  * chunks are fixed 64-token runs inside one document; the last chunk of a
    document is averaged over its actual token count;
  * RoPE is rotate-half (pairs i, i + d/2), theta_i = base^(-2i/d);
  * a zero-norm vector has cosine 0 (norms clamped at eps = 1e-12);
  * the chunk score takes the head mean of cosines and the max over query
    tokens; the document score is the max (default) or mean over its chunks;
  * top-k is descending by score, ties broken toward the lower document id;
  * the active context uses global positions offset by ``pos_offset`` (k by
    default): local token j sits at pos_offset + j and the decode query is the
    last local token, at pos_offset + loc_len - 1; gathered chunk keys keep
    only their document-wise rotation;
  * attention has no causal mask over the gathered context and uses the
    scale 1/sqrt(head_dim) unless another is given;
  * a query of M > 1 tokens (the query-prefill step) is the last M local
    tokens: token t sits at pos_offset + loc_len - M + t and sees every
    gathered chunk and the local tokens j <= loc_len - M + t (causal).

Every function here is pinned by tests in ``tests/test_oracle.py`` against
closed forms, invariants, brute force and hand-derived values, and
``tests/test_oracle_mutants.py`` checks that a planted mistake in any of them
fails a pin.  Parity unpinned: three readings above are choices the pages do
not fix - the rotate-half RoPE convention, the offset k of the global
positions, and the routing score inside L_aux.  The tests pin the
implementation of each choice, not the choice itself.
"""
from __future__ import annotations

import math

import numpy as np

EPS = 1e-12


# ----------------------------------------------------------------------------
# bf16 widening (exact)
# ----------------------------------------------------------------------------
def bf16_to_f64(bits: np.ndarray) -> np.ndarray:
    """Widen bf16 bit patterns (uint16) exactly to float64."""
    b = np.asarray(bits)
    if b.dtype != np.uint16:
        return b.astype(np.float64)
    return (b.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


# ----------------------------------------------------------------------------
# Stage 1: chunk layout  [digest "Method step details", Stage 1: chunk size P = 64;
#          IRMaD M&M routing item: K̄ = φ(K) etc.; chunks never cross documents]
# ----------------------------------------------------------------------------
def chunk_layout(doc_off: np.ndarray, chunk: int = 64):
    """Split every document [doc_off[i], doc_off[i+1]) into runs of ``chunk`` tokens.

    Returns (chunk_off [N+1], chunk_tok0 [C], chunk_len [C], chunk_doc [C]):
    chunk_off[i] is the first chunk of doc i, chunk_tok0 the first token of each
    chunk, chunk_len its token count (< chunk only for a doc's last chunk).
    """
    doc_off = np.asarray(doc_off, dtype=np.int64)
    n_docs = len(doc_off) - 1
    chunk_off = [0]
    tok0, length, owner = [], [], []
    for i in range(n_docs):
        start, end = int(doc_off[i]), int(doc_off[i + 1])
        t = start
        while t < end:
            tok0.append(t)
            length.append(min(chunk, end - t))
            owner.append(i)
            t += chunk
        chunk_off.append(len(tok0))
    return (np.asarray(chunk_off, dtype=np.int64), np.asarray(tok0, dtype=np.int64),
            np.asarray(length, dtype=np.int64), np.asarray(owner, dtype=np.int64))


# ----------------------------------------------------------------------------
# RoPE  [IRMaD M&M "position encoding": document-wise RoPE restarts at 0 per
#        document; global RoPE for the active context offset by k;
#        overview "key technical details" 1: Parallel RoPE / Global RoPE]
# ----------------------------------------------------------------------------
def rope_theta(head_dim: int, base: float) -> np.ndarray:
    """theta_i = base^(-2i/d) for i = 0 .. d/2 - 1."""
    i = np.arange(head_dim // 2, dtype=np.float64)
    return base ** (-2.0 * i / head_dim)


def rope(x: np.ndarray, pos, base: float) -> np.ndarray:
    """Rotate-half RoPE of the last axis of ``x`` at integer positions ``pos``.

    ``pos`` broadcasts against x.shape[:-1].  Pair (i, i + d/2) is rotated by
    the angle pos * theta_i.
    """
    x = np.asarray(x, dtype=np.float64)
    d = x.shape[-1]
    half = d // 2
    ang = np.asarray(pos, dtype=np.float64)[..., None] * rope_theta(d, base)
    c, s = np.cos(ang), np.sin(ang)
    x1, x2 = x[..., :half], x[..., half:]
    return np.concatenate([x1 * c - x2 * s, x2 * c + x1 * s], axis=-1)


# ----------------------------------------------------------------------------
# Stage 1: offline memory encoding
#   K_{i,h} = H_i W_K^h, V_{i,h} = H_i W_V^h, K^R_{i,h} = H_i W^KR_h;
#   K̄ = φ(K), V̄ = φ(V), K̄^R = φ(K^R), φ = 64-token chunk mean;
#   document-wise RoPE on K  [IRMaD M&M routing item and position item;
#   digest "Method step details" Stage 1]
# ----------------------------------------------------------------------------
def encode_memory(H, doc_off, W_K, W_V, W_KR, n_kv: int, head_dim: int, n_r: int, d_r: int,
                  chunk: int = 64, rope_base: float = 1.0e6, docs=None):
    """Return (K_bar [C, n_kv, d], V_bar [C, n_kv, d], KR_bar [C, n_r, d_r]) in float64.

    ``docs`` optionally restricts the work to a subset of document ids; the
    result then holds those documents' chunks in the order given.
    """
    H = bf16_to_f64(H)
    W_K, W_V, W_KR = bf16_to_f64(W_K), bf16_to_f64(W_V), bf16_to_f64(W_KR)
    doc_off = np.asarray(doc_off, dtype=np.int64)
    if docs is None:
        docs = range(len(doc_off) - 1)
    Kb, Vb, KRb = [], [], []
    for i in docs:
        a, b = int(doc_off[i]), int(doc_off[i + 1])
        Hd = H[a:b]
        K = (Hd @ W_K).reshape(b - a, n_kv, head_dim)
        pos = np.arange(b - a)                     # positions restart at 0 in every doc
        K = rope(K, pos[:, None], rope_base)
        V = (Hd @ W_V).reshape(b - a, n_kv, head_dim)
        KR = (Hd @ W_KR).reshape(b - a, n_r, d_r)
        for t in range(0, b - a, chunk):
            e = min(t + chunk, b - a)
            Kb.append(K[t:e].mean(axis=0))
            Vb.append(V[t:e].mean(axis=0))
            KRb.append(KR[t:e].mean(axis=0))
    return np.asarray(Kb), np.asarray(Vb), np.asarray(KRb)


# ----------------------------------------------------------------------------
# Stage 2: online routing
#   Q^R_{q,h} = H_q W^QR_h
#   S_ij = max_t ( mean_h cos((Q^R_{q,h})_t, K̄^R_{ij,h}) ),  s_i = max_j S_ij,
#   I = Top-k({s_i})   [IRMaD M&M routing item; digest "Method step details"
#   Stage 2, k = 16; news 2.1 two-level routing]
# ----------------------------------------------------------------------------
def router_query(Hq, W_QR, n_r: int, d_r: int) -> np.ndarray:
    """Q^R = H_q W^QR, reshaped to [..., n_r, d_r]."""
    Hq = bf16_to_f64(Hq)
    QR = Hq @ bf16_to_f64(W_QR)
    return QR.reshape(*Hq.shape[:-1], n_r, d_r)


def cosine(a: np.ndarray, b: np.ndarray) -> np.ndarray:
    """Cosine along the last axis, with each norm clamped below at EPS."""
    na = np.maximum(np.sqrt((a * a).sum(-1)), EPS)
    nb = np.maximum(np.sqrt((b * b).sum(-1)), EPS)
    return (a * b).sum(-1) / (na * nb)


def chunk_scores(QR, KR_bar, rows=None) -> np.ndarray:
    """S[b, j] = max over query tokens t of the head-mean cosine.

    QR: [B, n_r, d_r] (one query token) or [B, M, n_r, d_r] (M tokens).
    KR_bar: [C, n_r, d_r].  ``rows`` optionally selects chunk indices.
    """
    QR = np.asarray(QR, dtype=np.float64)
    if QR.ndim == 3:
        QR = QR[:, None]
    K = bf16_to_f64(KR_bar if rows is None else np.asarray(KR_bar)[rows])
    B, M = QR.shape[:2]
    S = np.empty((B, K.shape[0]))
    for b in range(B):
        per_t = []
        for t in range(M):
            cos_h = cosine(QR[b, t][None, :, :], K)       # [C, n_r]
            per_t.append(cos_h.mean(axis=1))              # mean over heads
        S[b] = np.max(np.stack(per_t), axis=0)            # max over query tokens
    return S


def doc_scores(S, chunk_off, agg: str = "max") -> np.ndarray:
    """s[b, i] = max (or mean) of S[b, j] over doc i's chunks."""
    chunk_off = np.asarray(chunk_off, dtype=np.int64)
    n_docs = len(chunk_off) - 1
    out = np.empty((S.shape[0], n_docs))
    for i in range(n_docs):
        seg = S[:, chunk_off[i]:chunk_off[i + 1]]
        out[:, i] = seg.max(axis=1) if agg == "max" else seg.mean(axis=1)
    return out


def topk(s: np.ndarray, k: int):
    """Top-k of a score vector: descending score, ties to the lower id."""
    s = np.asarray(s, dtype=np.float64)
    order = np.lexsort((np.arange(len(s)), -s))
    idx = order[:k]
    return idx.astype(np.int64), s[idx]


def route_topk(QR, KR_bar, chunk_off, k: int, agg: str = "max"):
    """Full stage 2 for given router queries: (doc_scores [B,N], idx [B,k], score [B,k])."""
    S = chunk_scores(QR, KR_bar)
    s = doc_scores(S, chunk_off, agg)
    idx = np.empty((s.shape[0], k), dtype=np.int64)
    val = np.empty((s.shape[0], k))
    for b in range(s.shape[0]):
        idx[b], val[b] = topk(s[b], k)
    return s, idx, val


# ----------------------------------------------------------------------------
# Stage 3: sparse generation attention
#   K_ctx = [{K̄_i}_{i∈I}; K_q], V_ctx = [{V̄_i}_{i∈I}; V_q],
#   Output = Attention(Q_q, K_ctx, V_ctx)   [IRMaD M&M routing item and
#   three-stage inference item (3); news 2.1 sparse generation]
# ----------------------------------------------------------------------------
def sparse_context(K_bar, V_bar, chunk_off, sel, K_loc_b, V_loc_b, L: int, pos_offset: int,
                   rope_base: float):
    """Explicit [selected docs' pooled keys (top-k order, chunks in order); local KV].

    Local keys get global RoPE at pos_offset + j; pooled keys are used as stored.
    Returns (K_ctx [n_keys, n_kv, d], V_ctx [n_keys, n_kv, d]).
    """
    Kb, Vb = bf16_to_f64(K_bar), bf16_to_f64(V_bar)
    ks, vs = [], []
    for i in sel:
        a, b = int(chunk_off[i]), int(chunk_off[i + 1])
        ks.append(Kb[a:b])
        vs.append(Vb[a:b])
    Kl = bf16_to_f64(K_loc_b[:L])
    Vl = bf16_to_f64(V_loc_b[:L])
    Kl = rope(Kl, (pos_offset + np.arange(L))[:, None], rope_base)
    ks.append(Kl)
    vs.append(Vl)
    return np.concatenate(ks, axis=0), np.concatenate(vs, axis=0)


def attention(q, K, V, scale: float) -> np.ndarray:
    """softmax(q K^T * scale) V for one head: q [d], K [n, d], V [n, d]."""
    logits = (K @ q) * scale
    m = logits.max()
    p = np.exp(logits - m)
    return (p[:, None] * V).sum(axis=0) / p.sum()


def sparse_attend(q, K_bar, V_bar, chunk_off, topk_idx, K_loc, V_loc, loc_len, pos_offset: int,
                  rope_base: float = 1.0e6, scale: float = 0.0) -> np.ndarray:
    """GQA decode over the sparse context; returns out [B, n_q, d] in float64.

    q head g reads KV head g // (n_q / n_kv).  The decode query is rotated to
    pos_offset + loc_len[b] - 1.
    """
    qf = bf16_to_f64(q)
    B, n_q, d = qf.shape
    n_kv = np.asarray(K_bar).shape[1]
    G = n_q // n_kv
    if scale == 0.0:
        scale = 1.0 / math.sqrt(d)
    out = np.empty((B, n_q, d))
    for b in range(B):
        L = int(loc_len[b])
        K_ctx, V_ctx = sparse_context(K_bar, V_bar, chunk_off, topk_idx[b], K_loc[b], V_loc[b],
                                      L, pos_offset, rope_base)
        qr = rope(qf[b], pos_offset + L - 1, rope_base)
        for g in range(n_q):
            h = g // G
            out[b, g] = attention(qr[g], K_ctx[:, h], V_ctx[:, h], scale)
    return out


def sparse_attend_tokens(q, K_bar, V_bar, chunk_off, topk_idx, K_loc, V_loc, loc_len, pos_offset: int,
                         rope_base: float = 1.0e6, scale: float = 0.0) -> np.ndarray:
    """Attention of M query tokens per query; q [B, M, n_q, d] -> out [B, M, n_q, d] float64.

    The query tokens are the last M local tokens.  Each token's logits run over the
    whole explicit context [selected docs' pooled keys; every local key] and a mask
    removes the local keys after the token's own position (chunk keys are always
    visible), so the softmax is taken over exactly the keys the token may see.
    """
    qf = bf16_to_f64(q)
    B, M, n_q, d = qf.shape
    n_kv = np.asarray(K_bar).shape[1]
    G = n_q // n_kv
    if scale == 0.0:
        scale = 1.0 / math.sqrt(d)
    out = np.empty((B, M, n_q, d))
    for b in range(B):
        L = int(loc_len[b])
        K_ctx, V_ctx = sparse_context(K_bar, V_bar, chunk_off, topk_idx[b], K_loc[b], V_loc[b],
                                      L, pos_offset, rope_base)
        n_sel = K_ctx.shape[0] - L
        is_chunk = np.arange(K_ctx.shape[0]) < n_sel
        local_j = np.arange(K_ctx.shape[0]) - n_sel
        for t in range(M):
            own = L - M + t                                   # this token's local index
            visible = is_chunk | (local_j <= own)
            qr = rope(qf[b, t], pos_offset + own, rope_base)
            for g in range(n_q):
                h = g // G
                logits = (K_ctx[:, h] @ qr[g]) * scale
                logits = np.where(visible, logits, -np.inf)
                m = logits.max()
                p = np.exp(logits - m)
                out[b, t, g] = (p[:, None] * V_ctx[:, h]).sum(axis=0) / p.sum()
    return out


# ----------------------------------------------------------------------------
# Router training signal: the contrastive auxiliary loss
#   L_aux = -(1/|P|) sum_i log( exp(s_i^+/tau) / (exp(s_i^+/tau) + sum_j exp(s_ij^-/tau)) )
#   [IRMaD M&M, training item: per-layer routing supervision that separates
#   positive from negative document chunks; digest "Core method"]
# Reading: a score s is the routing score of the chunk, the head mean of the
# cosines between the router query and the pooled router key (the S_ij of the
# routing formula with one query token).
# ----------------------------------------------------------------------------
def _norm_clamped(a):
    n = np.sqrt((a * a).sum(-1))
    return np.maximum(n, EPS), n > EPS


def aux_loss(QR, K_pos, K_neg, tau: float):
    """Loss and gradients of L_aux for P positives, each with N negatives.

    QR [P, n_r, d_r], K_pos [P, n_r, d_r], K_neg [P, N, n_r, d_r] (bf16 bits or float).
    Returns (loss, dQR, dK_pos, dK_neg) in float64.  A norm below EPS is clamped
    (its gradient through the clamp is zero).
    """
    def f64(x):
        x = np.asarray(x)
        return bf16_to_f64(x) if x.dtype == np.uint16 else x.astype(np.float64)

    Q, Kp, Kn = f64(QR), f64(K_pos), f64(K_neg)
    P, n_r, d_r = Q.shape
    N = Kn.shape[1]
    loss = 0.0
    dQ = np.zeros_like(Q)
    dKp = np.zeros_like(Kp)
    dKn = np.zeros_like(Kn)
    for i in range(P):
        keys = np.concatenate([Kp[i][None], Kn[i]], axis=0)      # [1 + N, n_r, d_r], positive first
        nq, q_live = _norm_clamped(Q[i])                            # [n_r]
        nk, k_live = _norm_clamped(keys)                            # [1 + N, n_r]
        dots = (keys * Q[i][None]).sum(-1)                          # [1 + N, n_r]
        cos = dots / (nq[None] * nk)
        s = cos.mean(axis=1)                                        # [1 + N] routing scores
        z = s / tau
        zmax = z.max()
        w = np.exp(z - zmax)
        p = w / w.sum()                                             # softmax over positive + negatives
        loss += -(z[0] - zmax - math.log(w.sum())) / P
        g = p / (tau * P)                                           # dL/ds_j for the negatives
        g[0] = -(1.0 - p[0]) / (tau * P)                            # dL/ds for the positive
        for j in range(1 + N):
            for h in range(n_r):
                gc = g[j] / n_r                                     # through the head mean
                # d cos / d q = k / (|q||k|) - cos * q / |q|^2   (the second term only off the clamp)
                dq = keys[j, h] / (nq[h] * nk[j, h])
                if q_live[h]:
                    dq = dq - cos[j, h] * Q[i, h] / (nq[h] ** 2)
                dk = Q[i, h] / (nq[h] * nk[j, h])
                if k_live[j, h]:
                    dk = dk - cos[j, h] * keys[j, h] / (nk[j, h] ** 2)
                dQ[i, h] += gc * dq
                if j == 0:
                    dKp[i, h] += gc * dk
                else:
                    dKn[i, j - 1, h] += gc * dk
    return loss, dQ, dKp, dKn
