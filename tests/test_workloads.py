"""The seeded input generator draws the workloads its docstrings describe.

Document lengths: lognormal around the median, clipped to [64, 32K], summing to T exactly.
Planted documents: one chunk per planted document whose router key has the stated per-head
cosine with the query's direction (before bf16 rounding).  Same seed, same bytes.
"""
import hashlib
import math

import numpy as np

import oracle as O
from long_context_memory_b200 import workloads as W


def LAYOUT(doc_off):
    """The oracle's chunk layout (the generator takes the layout from its caller)."""
    return O.chunk_layout(doc_off)[0]


def _f64(bits):
    return (np.asarray(bits).astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def test_lognormal_lengths_sum_to_T_within_bounds():
    rng = np.random.default_rng(3)
    for T, median in ((1_000_000, 2048), (3_000_000, 4096), (70_000, 2048)):
        lens = W.doc_lengths_lognormal(rng, T, median)
        assert int(np.sum(lens)) == T
        assert lens.min() >= 64 and lens.max() <= 32768
        # the median of a lognormal draw clipped far from its centre stays near the target
        assert 0.7 * median < np.median(lens) < 1.3 * median


def test_mem1m_layout_and_planted_cosines():
    c = W.mem1m_config(LAYOUT)
    d = c["dims"]
    lens = c["lens"]
    assert int(np.sum(lens)) == c["T"] == 1_000_000
    assert 350 < len(lens) < 550                           # about T / median documents
    C = int(np.sum((lens + d.chunk - 1) // d.chunk))
    assert c["KR"].shape == (C, d.n_r, d.d_r) and c["K_bar"].shape == (C, d.n_kv, d.head_dim)
    assert c["K_loc"].shape == (1, 4096, d.n_kv, d.head_dim) and c["loc_len"].tolist() == [4096]
    qr = _f64(c["QR"]).reshape(c["B"], d.n_r, d.d_r)
    kr = _f64(c["KR"])
    chunk_off = np.concatenate([[0], np.cumsum((lens + d.chunk - 1) // d.chunk)])
    for b in range(c["B"]):
        assert len(set(c["planted_docs"][b].tolist())) == 16
        for p in range(16):
            ch = int(c["planted_chunks"][b, p])
            doc = int(c["planted_docs"][b, p])
            assert chunk_off[doc] <= ch < chunk_off[doc + 1]  # the chunk lies in its document
            for h in range(d.n_r):
                u, v = qr[b, h], kr[ch, h]
                cos = u @ v / (np.linalg.norm(u) * np.linalg.norm(v))
                assert abs(cos - 0.9) < 1e-2, (b, p, h, cos)  # bf16 rounding of both sides only


def test_same_seed_same_bytes():
    a, b = W.mem1m_config(LAYOUT), W.mem1m_config(LAYOUT)
    for key in ("KR", "K_bar", "V_bar", "K_loc", "V_loc", "q", "Hq", "W_QR", "QR"):
        assert hashlib.sha256(a[key].tobytes()).digest() == hashlib.sha256(b[key].tobytes()).digest(), key
    c = W.mem1m_config(LAYOUT, seed=W.BASE_SEED + 99)
    assert not np.array_equal(a["KR"], c["KR"])


def test_tiny_config_recipe():
    c = W.tiny_config()
    d = c["dims"]
    assert len(c["lens"]) == 64 and c["lens"].min() >= 256 and c["lens"].max() <= 2048
    assert np.array_equal(c["W_QR"], c["W_KR"])           # planted docs stay visible to the router
    # the planted documents' hidden states sit near the query's
    H, hq = _f64(c["H"]), _f64(c["Hq"])[0]
    for i in c["planted"]:
        a, e = int(c["doc_off"][i]), int(c["doc_off"][i + 1])
        assert np.sqrt(np.mean((H[a:e] - hq) ** 2)) < 0.15     # noise of std 0.1
    other = int(c["doc_off"][5])
    assert np.sqrt(np.mean((H[other] - hq) ** 2)) > 1.0    # two independent N(0, 1) rows
    assert c["H"].shape == (c["T"], d.hidden) and math.isclose(c["pos_offset"], c["k"])
