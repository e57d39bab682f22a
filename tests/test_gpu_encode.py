"""GPU parity of stage 1 (offline memory encoding) against the CPU oracle, through the C ABI.

Tolerance: outputs are bf16 (round to nearest even, relative error <= 2^-9)
computed from fp32 accumulators; the fp32 accumulation and the RoPE angle
evaluation add errors of order 1e-6.  The test allows 2^-8 relative plus 1e-4
absolute.
"""
import numpy as np
import pytest

import oracle as O
from long_context_memory_b200 import workloads as W
from helpers import torch_bits

pytestmark = pytest.mark.gpu

RTOL = 2.0 ** -8
ATOL = 1e-4


@pytest.fixture(scope="module")
def msa(cuda_device):
    import long_context_memory_b200 as m

    return m


def _dev(a, device):
    return W.to_torch(np.ascontiguousarray(a)).to(device)


def _encode(msa, dims, H, doc_off, WK, WV, WKR, device, head_major=False):
    import torch

    co, C = msa.chunk_offsets(doc_off)
    out = msa.encode_memory(dims, _dev(H, device), torch.from_numpy(np.asarray(doc_off, dtype=np.int64)).to(device),
                            torch.from_numpy(co).to(device), C, _dev(WK, device), _dev(WV, device),
                            _dev(WKR, device), kr_head_major=head_major)
    torch.cuda.synchronize()
    assert msa.check_device_errors() == 0
    return [O.bf16_to_f64(torch_bits(t)) for t in out], co


def _close(gpu, ref, what):
    err = np.abs(gpu - ref)
    bound = ATOL + RTOL * np.abs(ref)
    bad = err > bound
    assert not bad.any(), (f"{what}: {bad.sum()} of {bad.size} outside tolerance; worst excess "
                           f"{np.max(err - bound):.3e}")


def test_encode_tiny_config(msa, cuda_device):
    c = W.tiny_config()
    d = c["dims"]
    (Kg, Vg, KRg), co = _encode(msa, d, c["H"], c["doc_off"], c["W_K"], c["W_V"], c["W_KR"], cuda_device)
    Kb, Vb, KRb = O.encode_memory(c["H"], c["doc_off"], c["W_K"], c["W_V"], c["W_KR"], d.n_kv, d.head_dim, d.n_r,
                                  d.d_r, rope_base=d.rope_base)
    _close(Kg, Kb, "K_bar")
    _close(Vg, Vb, "V_bar")
    _close(KRg, KRb, "KR_bar")


@pytest.mark.parametrize("head_dim,n_kv,n_r,d_r", [(128, 8, 8, 128), (64, 4, 2, 64)])
def test_encode_edge_lengths(msa, cuda_device, head_dim, n_kv, n_r, d_r):
    rng = np.random.default_rng(head_dim + n_r)
    lens = np.array([1, 63, 64, 65, 127, 128, 129, 3, 700, 64 * 5 + 17, 2])   # odd total chunk count
    doc_off = W.offsets_from_lengths(lens)
    T, hid = int(doc_off[-1]), 512
    d = W.Dims(hidden=hid, n_q=2 * n_kv, n_kv=n_kv, head_dim=head_dim, n_r=n_r, d_r=d_r, rope_base=1e6)
    H = W.normal_bf16(rng, (T, hid))
    WK = W.normal_bf16(rng, (hid, n_kv * head_dim), hid ** -0.5)
    WV = W.normal_bf16(rng, (hid, n_kv * head_dim), hid ** -0.5)
    WKR = W.normal_bf16(rng, (hid, n_r * d_r), hid ** -0.5)
    (Kg, Vg, KRg), co = _encode(msa, d, H, doc_off, WK, WV, WKR, cuda_device)
    assert co[-1] % 2 == 1
    Kb, Vb, KRb = O.encode_memory(H, doc_off, WK, WV, WKR, n_kv, head_dim, n_r, d_r, rope_base=1e6)
    _close(Kg, Kb, "K_bar")
    _close(Vg, Vb, "V_bar")
    _close(KRg, KRb, "KR_bar")


@pytest.mark.parametrize("n_r,d_r", [(8, 128), (2, 64), (6, 64)])
def test_encode_head_major_router_keys(msa, cuda_device, n_r, d_r):
    # K̄^R written [n_r, C, d_r]: the same values as the chunk-major output, moved
    rng = np.random.default_rng(40 + n_r)
    lens = np.array([5, 64, 129, 300, 1, 77, 640, 65])
    doc_off = W.offsets_from_lengths(lens)
    T, hid = int(doc_off[-1]), 256
    d = W.Dims(hidden=hid, n_q=4, n_kv=2, head_dim=64, n_r=n_r, d_r=d_r)
    H = W.normal_bf16(rng, (T, hid))
    WK = W.normal_bf16(rng, (hid, 2 * 64), hid ** -0.5)
    WV = W.normal_bf16(rng, (hid, 2 * 64), hid ** -0.5)
    WKR = W.normal_bf16(rng, (hid, n_r * d_r), hid ** -0.5)
    (Kg, Vg, KRg), co = _encode(msa, d, H, doc_off, WK, WV, WKR, cuda_device, head_major=True)
    assert KRg.shape == (n_r, co[-1], d_r)
    Kb, Vb, KRb = O.encode_memory(H, doc_off, WK, WV, WKR, 2, 64, n_r, d_r)
    _close(KRg, KRb.transpose(1, 0, 2), "KR_bar head-major")
    _close(Kg, Kb, "K_bar")
    (_, _, KR0), _ = _encode(msa, d, H, doc_off, WK, WV, WKR, cuda_device)
    assert np.array_equal(KRg, KR0.transpose(1, 0, 2))


def test_encode_long_documents_positions(msa, cuda_device):
    # documents far longer than 64 tokens exercise large document-relative positions
    rng = np.random.default_rng(3)
    lens = np.array([20000, 5, 9000])
    doc_off = W.offsets_from_lengths(lens)
    T, hid = int(doc_off[-1]), 256
    d = W.Dims(hidden=hid, n_q=8, n_kv=2, head_dim=128, n_r=1, d_r=128, rope_base=1e4)
    H = W.normal_bf16(rng, (T, hid))
    WK = W.normal_bf16(rng, (hid, 256), hid ** -0.5)
    WV = W.normal_bf16(rng, (hid, 256), hid ** -0.5)
    WKR = W.normal_bf16(rng, (hid, 128), hid ** -0.5)
    (Kg, Vg, KRg), co = _encode(msa, d, H, doc_off, WK, WV, WKR, cuda_device)
    Kb, Vb, KRb = O.encode_memory(H, doc_off, WK, WV, WKR, 2, 128, 1, 128, rope_base=1e4)
    _close(Kg, Kb, "K_bar")
    _close(Vg, Vb, "V_bar")
    _close(KRg, KRb, "KR_bar")


def test_encode_1m_tokens_sampled(msa, cuda_device):
    # full-size encode over 1M tokens (hidden 2560, W [2560 x 1024]); H is drawn on the device by a
    # seeded generator.  The oracle checks a sample of documents: the first, the last, the shortest,
    # the longest and 8 random ones.
    import torch

    c = W.encode_config(with_hidden=False)
    d = c["dims"]
    H = W.encode_hidden(c["T"], d.hidden, c["seed"], cuda_device)
    co, C = msa.chunk_offsets(c["doc_off"])
    out = msa.encode_memory(d, H, torch.from_numpy(c["doc_off"]).to(cuda_device), torch.from_numpy(co).to(cuda_device),
                            C, _dev(c["W_K"], cuda_device), _dev(c["W_V"], cuda_device), _dev(c["W_KR"], cuda_device))
    torch.cuda.synchronize()
    assert msa.check_device_errors() == 0
    Kg, Vg, KRg = (O.bf16_to_f64(torch_bits(t)) for t in out)
    lens = c["lens"]
    rng = np.random.default_rng(1)
    docs = sorted(set([0, len(lens) - 1, int(np.argmin(lens)), int(np.argmax(lens))] +
                      rng.choice(len(lens), 8, replace=False).tolist()))
    # the sampled documents' hidden rows, re-based into a small corpus for the oracle
    doc_off = c["doc_off"]
    Hs = np.concatenate([torch_bits(H[int(doc_off[i]):int(doc_off[i + 1])]) for i in docs])
    sub_off = W.offsets_from_lengths(np.array([doc_off[i + 1] - doc_off[i] for i in docs]))
    Kb, Vb, KRb = O.encode_memory(Hs, sub_off, c["W_K"], c["W_V"], c["W_KR"], d.n_kv, d.head_dim, d.n_r, d.d_r,
                                  rope_base=d.rope_base)
    rows = np.concatenate([np.arange(co[i], co[i + 1]) for i in docs])
    _close(Kg[rows], Kb, "K_bar")
    _close(Vg[rows], Vb, "V_bar")
    _close(KRg[rows], KRb, "KR_bar")


def test_append_memory_equals_full_encode(msa, cuda_device):
    # encode docs A, then append docs B (in two steps) into a memory with spare rows: the rows and the
    # chunk offsets must equal a single encode of A + B bit for bit (positions restart per document,
    # chunks never cross documents), and routing over the grown memory must agree with the oracle
    import torch

    rng = np.random.default_rng(2024)
    d = W.Dims(hidden=256, n_q=8, n_kv=2, head_dim=64, n_r=4, d_r=64, rope_base=1e6)
    lens = rng.integers(1, 500, size=23)
    parts = [lens[:10], lens[10:17], lens[17:]]
    doc_off = W.offsets_from_lengths(lens)
    T = int(doc_off[-1])
    H = W.normal_bf16(rng, (T, 256))
    WK, WV = W.normal_bf16(rng, (256, 128), 1 / 16), W.normal_bf16(rng, (256, 128), 1 / 16)
    WKR = W.normal_bf16(rng, (256, 256), 1 / 16)
    dev = cuda_device
    Wd = (_dev(WK, dev), _dev(WV, dev), _dev(WKR, dev))
    co_all, C = msa.chunk_offsets(doc_off)
    full = msa.encode_memory(d, _dev(H, dev), torch.from_numpy(doc_off).to(dev), torch.from_numpy(co_all).to(dev), C,
                             *Wd)
    cap = C + 9
    mem = (torch.full((cap, 2, 64), 7, dtype=torch.bfloat16, device=dev),
           torch.full((cap, 2, 64), 7, dtype=torch.bfloat16, device=dev),
           torch.full((cap, 4, 64), 7, dtype=torch.bfloat16, device=dev))
    chunk_off = torch.full((len(lens) + 1 + 5,), -1, dtype=torch.int32, device=dev)
    n_docs, n_chunks, t0 = 0, 0, 0
    for part in parts:
        off = W.offsets_from_lengths(part)
        co, Cn = msa.chunk_offsets(off)
        Hp = H[t0:t0 + int(off[-1])]
        n_docs, n_chunks = msa.append_memory(d, _dev(Hp, dev), torch.from_numpy(off).to(dev),
                                             torch.from_numpy(co).to(dev), Cn, *Wd, mem, chunk_off, n_docs, n_chunks)
        t0 += int(off[-1])
    torch.cuda.synchronize()
    assert msa.check_device_errors() == 0
    assert (n_docs, n_chunks) == (len(lens), C)
    assert np.array_equal(chunk_off[:n_docs + 1].cpu().numpy(), co_all)
    for a, b in zip(mem, full):
        assert torch.equal(a[:C], b)
        assert bool((a[C:].float() == 7).all())          # rows past the memory are untouched
    # routing over the appended memory
    QR = W.normal_bf16(rng, (2, 256))
    idx, sc, ds = msa.route_topk(d, _dev(QR, dev), None, mem[2][:C], chunk_off[:n_docs + 1], 5, want_doc_scores=True)
    _, _, KRb = O.encode_memory(H, doc_off, WK, WV, WKR, 2, 64, 4, 64, rope_base=1e6)
    s = O.doc_scores(O.chunk_scores(O.bf16_to_f64(QR).reshape(2, 4, 64), W.f32_to_bf16_bits(KRb.astype(np.float32))),
                     co_all)
    assert np.max(np.abs(ds.cpu().numpy() - s)) < 2e-3   # stored K̄^R is bf16-rounded; scores from it
