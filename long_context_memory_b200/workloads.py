"""Seeded synthetic inputs for the Memory Sparse Attention hot path.

This module only draws random numbers and lays them out; it performs none of
the method's arithmetic (no projection, pooling, RoPE, cosine, top-k or
attention).  Both the CPU oracle (through the tests) and the CUDA path take
their inputs from here.  All bf16 tensors are returned as ``numpy.uint16``
arrays holding bf16 bit patterns; ``to_torch`` views them as torch bf16.

Shapes and distributions follow the workloads named for the method ("MSA:
Memory Sparse Attention for Efficient End-to-End Memory Model Scaling to 100M
Tokens", methods section: P = 64 tokens per chunk, top-k = 16, 8 heads of
dimension 128; memory sizes from 1M to 100M tokens).  Document lengths are
lognormal with sigma 0.5 (the pages do not state a spread), clipped to
[64, 32768] and trimmed so that the lengths sum to exactly T.

Planted documents.  A planted chunk is built so that, for every router head,
its key has a prescribed cosine ``c`` with a planted direction ``u``:
``key = sqrt(d_r) * (c * u + sqrt(1 - c^2) * w)`` with ``w`` a unit vector
orthogonal to ``u``.  This is geometry for constructing inputs with a known
margin; the router query is then ``s * u`` for a random positive scale ``s``.
"""
from __future__ import annotations

import dataclasses
import math
from typing import Optional

import numpy as np

BASE_SEED = 20260402


# ----------------------------------------------------------------------------
# bf16 bit handling (input construction only)
# ----------------------------------------------------------------------------
def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round float32 values to bf16 (round to nearest even); return uint16 bits."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    bias = ((u >> 16) & 1) + np.uint32(0x7FFF)
    return ((u + bias) >> 16).astype(np.uint16)


def normal_bf16(rng: np.random.Generator, shape, std: float = 1.0) -> np.ndarray:
    x = rng.standard_normal(shape, dtype=np.float32)
    if std != 1.0:
        x *= np.float32(std)
    return f32_to_bf16_bits(x)


def to_torch(a: np.ndarray):
    """View a uint16 bf16-bit array (or any other numpy array) as a torch tensor."""
    import torch

    if a.dtype == np.uint16:
        return torch.from_numpy(a.view(np.int16)).view(torch.bfloat16)
    return torch.from_numpy(a)


# ----------------------------------------------------------------------------
# document layouts
# ----------------------------------------------------------------------------
def doc_lengths_uniform(rng, n_docs: int, lo: int, hi: int) -> np.ndarray:
    return rng.integers(lo, hi + 1, size=n_docs).astype(np.int64)


def doc_lengths_lognormal(rng, total: int, median: int, sigma: float = 0.5,
                          lo: int = 64, hi: int = 32768) -> np.ndarray:
    """Lognormal lengths drawn until they cover ``total`` tokens, then trimmed.

    The last document is shortened so that the sum is exactly ``total``; if the
    remainder would be shorter than ``lo`` it is merged into the previous doc
    (clipped at ``hi``; any excess becomes one more doc of at least ``lo``).
    """
    out = []
    acc = 0
    mu = math.log(median)
    while acc < total:
        n = max(16, int(1.5 * (total - acc) / median) + 16)
        draw = np.clip(np.round(rng.lognormal(mu, sigma, size=n)), lo, hi).astype(np.int64)
        for v in draw:
            v = int(v)
            if acc + v >= total:
                rem = total - acc
                if rem >= lo:
                    out.append(rem)
                else:
                    # fold the short remainder into the previous document
                    prev = out.pop()
                    merged = prev + rem
                    if merged <= hi:
                        out.append(merged)
                    else:
                        out.append(merged - lo)
                        out.append(lo)
                acc = total
                break
            out.append(v)
            acc += v
    lens = np.asarray(out, dtype=np.int64)
    assert lens.sum() == total and lens.min() >= min(lo, total)
    return lens


def offsets_from_lengths(lens: np.ndarray) -> np.ndarray:
    off = np.zeros(len(lens) + 1, dtype=np.int64)
    off[1:] = np.cumsum(lens)
    return off


# ----------------------------------------------------------------------------
# planting helpers (input construction geometry)
# ----------------------------------------------------------------------------
def _unit(rng, n, d):
    v = rng.standard_normal((n, d))
    return v / np.linalg.norm(v, axis=1, keepdims=True)


def _planted_rows(rng, u: np.ndarray, c: np.ndarray, d: int) -> np.ndarray:
    """For unit rows u[h] and cosines c[h], rows with exact cosine c[h] to u[h]."""
    w = rng.standard_normal(u.shape)
    w -= (w * u).sum(axis=1, keepdims=True) * u
    w /= np.linalg.norm(w, axis=1, keepdims=True)
    c = np.asarray(c, dtype=np.float64).reshape(-1, 1)
    return math.sqrt(d) * (c * u + np.sqrt(np.maximum(0.0, 1.0 - c * c)) * w)


# ----------------------------------------------------------------------------
# dims
# ----------------------------------------------------------------------------
@dataclasses.dataclass(frozen=True)
class Dims:
    hidden: int
    n_q: int
    n_kv: int
    head_dim: int
    n_r: int
    d_r: int
    chunk: int = 64
    rope_base: float = 1.0e6


TINY_DIMS = Dims(hidden=256, n_q=8, n_kv=2, head_dim=64, n_r=4, d_r=64)
QWEN3_4B_DIMS = Dims(hidden=2560, n_q=32, n_kv=8, head_dim=128, n_r=8, d_r=128)


# ----------------------------------------------------------------------------
# tiny single layer (full pipeline, CPU seconds)
# ----------------------------------------------------------------------------
def tiny_config(seed: int = BASE_SEED, n_docs: int = 64, lo: int = 256, hi: int = 2048,
                dims: Dims = TINY_DIMS, k: int = 4, t_loc: int = 128,
                n_planted: int = 2, noise_std: float = 0.1) -> dict:
    """Tiny single layer: 64 docs of U[256, 2048] tokens, hidden 256.

    W^QR is set equal to W^KR (same N(0, 1/hidden) law) so that documents whose
    hidden states are the query's plus N(0, 0.1^2) noise are recognisably close
    to the query in router space; docs 0 and 1 are planted.
    """
    rng = np.random.default_rng(seed)
    lens = doc_lengths_uniform(rng, n_docs, lo, hi)
    doc_off = offsets_from_lengths(lens)
    T = int(doc_off[-1])
    hs = 1.0 / math.sqrt(dims.hidden)
    hq = rng.standard_normal(dims.hidden).astype(np.float32)
    H = rng.standard_normal((T, dims.hidden), dtype=np.float32)
    for i in range(n_planted):
        a, b = int(doc_off[i]), int(doc_off[i + 1])
        H[a:b] = hq[None, :] + noise_std * rng.standard_normal((b - a, dims.hidden), dtype=np.float32)
    W_K = normal_bf16(rng, (dims.hidden, dims.n_kv * dims.head_dim), hs)
    W_V = normal_bf16(rng, (dims.hidden, dims.n_kv * dims.head_dim), hs)
    W_KR = normal_bf16(rng, (dims.hidden, dims.n_r * dims.d_r), hs)
    W_QR = W_KR.copy()
    q = normal_bf16(rng, (1, dims.n_q, dims.head_dim))
    K_loc = normal_bf16(rng, (1, t_loc, dims.n_kv, dims.head_dim))
    V_loc = normal_bf16(rng, (1, t_loc, dims.n_kv, dims.head_dim))
    return dict(
        name="tiny", dims=dims, k=k, B=1, T=T, doc_off=doc_off, lens=lens,
        H=f32_to_bf16_bits(H), Hq=f32_to_bf16_bits(hq[None, :]),
        W_K=W_K, W_V=W_V, W_KR=W_KR, W_QR=W_QR,
        q=q, K_loc=K_loc, V_loc=V_loc,
        loc_len=np.full(1, t_loc, dtype=np.int32), t_loc_max=t_loc,
        pos_offset=k, planted=list(range(n_planted)),
    )


# ----------------------------------------------------------------------------
# pooled memory (route + attend), configs from 1M to 100M tokens
# ----------------------------------------------------------------------------
def memory_config(T: int, B: int, seed: int, layout, median: int = 2048, dims: Dims = QWEN3_4B_DIMS,
                  k: int = 16, t_loc: int = 4096, n_planted: int = 16,
                  planted_cos: Optional[np.ndarray] = None, with_kv: bool = True,
                  name: str = "memory") -> dict:
    """Pooled memory given directly: K̄, V̄, K̄^R ~ N(0,1) bf16 [C, heads, dim].

    ``layout(doc_off) -> chunk_off`` is the caller's chunk layout of the drawn documents (the
    generator itself computes none of it): it says how many pooled rows to draw and which rows
    belong to a planted document.

    Per query b, ``n_planted`` distinct documents get one random chunk whose
    router key has per-head cosine ``planted_cos[p]`` with the query's planted
    direction.  The router query ``QR`` (bf16, [B, n_r*d_r]) is that direction
    times a random positive scale per head.  ``Hq`` [B, hidden] ~ N(0,1) and
    ``W_QR`` ~ N(0, 1/hidden) are also drawn, for runs that exercise the router
    query projection (their product is unrelated to the planted direction).
    """
    rng = np.random.default_rng(seed)
    lens = doc_lengths_lognormal(rng, T, median)
    doc_off = offsets_from_lengths(lens)
    chunk_off = np.asarray(layout(doc_off), dtype=np.int64)
    nch = chunk_off[1:] - chunk_off[:-1]
    C = int(chunk_off[-1])
    N = len(lens)
    KR = normal_bf16(rng, (C, dims.n_r, dims.d_r))
    if planted_cos is None:
        planted_cos = np.full(n_planted, 0.9)
    planted_cos = np.asarray(planted_cos, dtype=np.float64)
    assert B * n_planted <= N
    planted_docs = rng.permutation(N)[: B * n_planted].reshape(B, n_planted)
    QR = np.zeros((B, dims.n_r, dims.d_r), dtype=np.float32)
    planted_chunks = np.zeros((B, n_planted), dtype=np.int64)
    for b in range(B):
        u = _unit(rng, dims.n_r, dims.d_r)
        scale = rng.uniform(0.5, 2.0, size=(dims.n_r, 1))
        QR[b] = (u * scale * math.sqrt(dims.d_r)).astype(np.float32)
        for p in range(n_planted):
            d = int(planted_docs[b, p])
            ch = int(chunk_off[d] + rng.integers(0, nch[d]))
            planted_chunks[b, p] = ch
            rows = _planted_rows(rng, u, np.full(dims.n_r, planted_cos[p]), dims.d_r)
            KR[ch] = f32_to_bf16_bits(rows.astype(np.float32))
    out = dict(
        name=name, dims=dims, k=k, B=B, T=T, doc_off=doc_off, lens=lens,
        chunk_off_expected_len=N + 1, n_chunks=C, KR=KR,
        QR=f32_to_bf16_bits(QR.reshape(B, -1)),
        Hq=normal_bf16(rng, (B, dims.hidden)),
        W_QR=normal_bf16(rng, (dims.hidden, dims.n_r * dims.d_r), 1.0 / math.sqrt(dims.hidden)),
        planted_docs=planted_docs, planted_chunks=planted_chunks, planted_cos=planted_cos,
        pos_offset=k, t_loc_max=t_loc,
    )
    if with_kv:
        out["K_bar"] = normal_bf16(rng, (C, dims.n_kv, dims.head_dim))
        out["V_bar"] = normal_bf16(rng, (C, dims.n_kv, dims.head_dim))
        out["q"] = normal_bf16(rng, (B, dims.n_q, dims.head_dim))
        out["K_loc"] = normal_bf16(rng, (B, t_loc, dims.n_kv, dims.head_dim))
        out["V_loc"] = normal_bf16(rng, (B, t_loc, dims.n_kv, dims.head_dim))
        out["loc_len"] = np.full(B, t_loc, dtype=np.int32)
    return out


def mem1m_config(layout, seed: int = BASE_SEED + 1, T: int = 1_000_000, **kw) -> dict:
    """1M-token memory, batch 1, 4K local KV, 16 planted docs at cosine 0.9."""
    kw.setdefault("t_loc", 4096)
    return memory_config(T=T, B=1, seed=seed, layout=layout, median=2048, name="mem1m", **kw)


def mem16m_config(layout, seed: int = BASE_SEED + 2, T: int = 16_000_000, B: int = 32, **kw) -> dict:
    """16M-token memory, 32 queries routed together, 8K local KV per query.

    Planted per-head cosines are 0.21 + 0.01 p (p = 0..15): the expected
    maximum background document score for 254K random chunks is about
    sqrt(2 ln C) / sqrt(n_r d_r) = 0.156, so the weakest planted doc sits about
    0.05 above the background and consecutive planted docs differ by 0.01.
    """
    kw.setdefault("t_loc", 8192)
    return memory_config(T=T, B=B, seed=seed, layout=layout, median=2048,
                         planted_cos=0.21 + 0.01 * np.arange(16), name="mem16m", **kw)


# ----------------------------------------------------------------------------
# encode workload
# ----------------------------------------------------------------------------
def encode_config(T: int = 1_000_000, seed: int = BASE_SEED + 5, median: int = 2048,
                  dims: Dims = QWEN3_4B_DIMS, with_hidden: bool = True) -> dict:
    """Offline encoding: H [T, hidden] ~ N(0,1) bf16, W_K/W_V/W^KR ~ N(0, 1/hidden).

    ``with_hidden=False`` leaves H out; draw it on a device with ``encode_hidden``
    (a [1M x 2560] corpus is 5 GB, too slow to draw and convert in numpy).
    """
    rng = np.random.default_rng(seed)
    lens = doc_lengths_lognormal(rng, T, median)
    doc_off = offsets_from_lengths(lens)
    hs = 1.0 / math.sqrt(dims.hidden)
    out = dict(
        name="encode", dims=dims, T=T, doc_off=doc_off, lens=lens, seed=seed,
        W_K=normal_bf16(rng, (dims.hidden, dims.n_kv * dims.head_dim), hs),
        W_V=normal_bf16(rng, (dims.hidden, dims.n_kv * dims.head_dim), hs),
        W_KR=normal_bf16(rng, (dims.hidden, dims.n_r * dims.d_r), hs),
    )
    if with_hidden:
        out["H"] = normal_bf16(rng, (T, dims.hidden))
    return out


def encode_hidden(T: int, hidden: int, seed: int, device):
    """H [T, hidden] ~ N(0,1) rounded to bf16, drawn by torch's seeded generator on ``device``."""
    import torch

    g = torch.Generator(device=device)
    g.manual_seed(seed)
    H = torch.empty((T, hidden), dtype=torch.bfloat16, device=device)
    step = 1 << 16
    for r in range(0, T, step):
        e = min(T, r + step)
        H[r:e] = torch.randn((e - r, hidden), generator=g, device=device, dtype=torch.float32).to(torch.bfloat16)
    return H
