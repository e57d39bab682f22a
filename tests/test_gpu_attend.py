"""GPU parity of stage 3 (sparse generation attention) against the CPU oracle, through the C ABI."""
import math

import numpy as np
import pytest

import oracle as O
from long_context_memory_b200 import workloads as W
from helpers import bf16_of, check_attention


def LAYOUT(doc_off):
    """The oracle's chunk layout (the generator takes the layout from its caller)."""
    return O.chunk_layout(doc_off)[0]


pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def msa(cuda_device):
    import long_context_memory_b200 as m

    return m


def _dev(a, device):
    return W.to_torch(np.ascontiguousarray(a)).to(device)


def _attend(msa, dims, c, device, pos_offset, scale=0.0):
    import torch

    co, C = msa.chunk_offsets(c["doc_off"])
    out = msa.sparse_attend(dims, _dev(c["q"], device), _dev(c["K_bar"], device), _dev(c["V_bar"], device),
                            torch.from_numpy(co).to(device), torch.from_numpy(c["topk"].astype(np.int32)).to(device),
                            _dev(c["K_loc"], device), _dev(c["V_loc"], device),
                            torch.from_numpy(c["loc_len"].astype(np.int32)).to(device), pos_offset, scale)
    torch.cuda.synchronize()
    assert msa.check_device_errors() == 0
    return out.float().cpu().numpy()


def _case(seed, B, n_q, n_kv, D, n_docs, k, t_loc, loc_len=None, lo=1, hi=900):
    rng = np.random.default_rng(seed)
    lens = rng.integers(lo, hi + 1, size=n_docs)
    doc_off = W.offsets_from_lengths(lens)
    co, *_ = O.chunk_layout(doc_off)
    C = int(co[-1])
    topk = np.stack([rng.permutation(n_docs)[:k] for _ in range(B)])
    if loc_len is None:
        loc_len = rng.integers(1, t_loc + 1, size=B)
    return dict(doc_off=doc_off, chunk_off=co, q=W.normal_bf16(rng, (B, n_q, D)),
                K_bar=W.normal_bf16(rng, (C, n_kv, D)), V_bar=W.normal_bf16(rng, (C, n_kv, D)),
                K_loc=W.normal_bf16(rng, (B, t_loc, n_kv, D)), V_loc=W.normal_bf16(rng, (B, t_loc, n_kv, D)),
                loc_len=np.asarray(loc_len), topk=topk)


def _oracle(c, pos_offset, base, scale=0.0):
    return O.sparse_attend(c["q"], c["K_bar"], c["V_bar"], c["chunk_off"], c["topk"], c["K_loc"], c["V_loc"],
                           c["loc_len"], pos_offset, base, scale)


@pytest.mark.parametrize("D", [64, 128])
@pytest.mark.parametrize("n_q,n_kv", [(8, 2), (32, 8), (8, 8), (16, 1)])
def test_attend_parity_shapes(msa, cuda_device, D, n_q, n_kv):
    B = 3
    c = _case(D + n_q + n_kv, B, n_q, n_kv, D, n_docs=40, k=6, t_loc=200)
    dims = W.Dims(hidden=256, n_q=n_q, n_kv=n_kv, head_dim=D, n_r=4, d_r=64, rope_base=1e6)
    out = _attend(msa, dims, c, cuda_device, pos_offset=6)
    check_attention(out, _oracle(c, 6, 1e6), where=f"D={D} G={n_q // n_kv}")


@pytest.mark.parametrize("pos_offset,base", [(0, 1e4), (16, 1e6), (5000, 1e6), (123457, 5e5)])
def test_attend_positions(msa, cuda_device, pos_offset, base):
    c = _case(3, 2, 8, 2, 128, n_docs=20, k=4, t_loc=300, loc_len=[300, 1])
    dims = W.Dims(hidden=256, n_q=8, n_kv=2, head_dim=128, n_r=4, d_r=64, rope_base=base)
    out = _attend(msa, dims, c, cuda_device, pos_offset=pos_offset)
    check_attention(out, _oracle(c, pos_offset, base), where=f"o={pos_offset}")


def test_attend_no_local_tokens_and_scale(msa, cuda_device):
    c = _case(4, 2, 8, 2, 64, n_docs=10, k=3, t_loc=8, loc_len=[0, 8])
    dims = W.Dims(hidden=256, n_q=8, n_kv=2, head_dim=64, n_r=4, d_r=64)
    out = _attend(msa, dims, c, cuda_device, pos_offset=3, scale=0.05)
    check_attention(out, _oracle(c, 3, 1e6, 0.05))


def test_attend_long_docs_many_splits(msa, cuda_device):
    c = _case(5, 1, 32, 8, 128, n_docs=30, k=16, t_loc=2000, loc_len=[1999], lo=2000, hi=20000)
    dims = W.Dims(hidden=2560, n_q=32, n_kv=8, head_dim=128, n_r=8, d_r=128)
    out = _attend(msa, dims, c, cuda_device, pos_offset=16)
    check_attention(out, _oracle(c, 16, 1e6))


def test_attend_single_key_closed_form(msa, cuda_device):
    # one one-chunk doc and no local tokens: the output is that chunk's value row
    rng = np.random.default_rng(6)
    c = dict(doc_off=np.array([0, 10]), chunk_off=np.array([0, 1]), q=W.normal_bf16(rng, (1, 4, 64)),
             K_bar=W.normal_bf16(rng, (1, 2, 64)), V_bar=W.normal_bf16(rng, (1, 2, 64)),
             K_loc=W.normal_bf16(rng, (1, 4, 2, 64)), V_loc=W.normal_bf16(rng, (1, 4, 2, 64)),
             loc_len=np.array([0]), topk=np.array([[0]]))
    dims = W.Dims(hidden=256, n_q=4, n_kv=2, head_dim=64, n_r=4, d_r=64)
    out = _attend(msa, dims, c, cuda_device, pos_offset=1)
    V = O.bf16_to_f64(c["V_bar"])[0]
    for g in range(4):
        assert np.allclose(out[0, g], V[g // 2], atol=1e-2)


def test_attend_tiny_config_full_pipeline(msa, cuda_device):
    c = W.tiny_config()
    d = c["dims"]
    Kb, Vb, KRb = O.encode_memory(c["H"], c["doc_off"], c["W_K"], c["W_V"], c["W_KR"], d.n_kv, d.head_dim, d.n_r,
                                  d.d_r)
    co, *_ = O.chunk_layout(c["doc_off"])
    KR = bf16_of(KRb)
    _, idx, _ = O.route_topk(O.router_query(c["Hq"], c["W_QR"], d.n_r, d.d_r), KR, co, c["k"])
    case = dict(doc_off=c["doc_off"], chunk_off=co, q=c["q"], K_bar=bf16_of(Kb), V_bar=bf16_of(Vb), K_loc=c["K_loc"],
                V_loc=c["V_loc"], loc_len=c["loc_len"], topk=idx)
    out = _attend(msa, d, case, cuda_device, pos_offset=c["pos_offset"])
    check_attention(out, _oracle(case, c["pos_offset"], d.rope_base))


def test_attend_mem1m_full_size(msa, cuda_device):
    m = W.mem1m_config(LAYOUT)
    d = m["dims"]
    co, *_ = O.chunk_layout(m["doc_off"])
    case = dict(doc_off=m["doc_off"], chunk_off=co, q=m["q"], K_bar=m["K_bar"], V_bar=m["V_bar"], K_loc=m["K_loc"],
                V_loc=m["V_loc"], loc_len=m["loc_len"], topk=m["planted_docs"])
    out = _attend(msa, d, case, cuda_device, pos_offset=m["pos_offset"])
    check_attention(out, _oracle(case, m["pos_offset"], d.rope_base))


def test_attend_mem16m_batch32_sampled(msa, cuda_device):
    m = W.mem16m_config(LAYOUT)
    d = m["dims"]
    co, *_ = O.chunk_layout(m["doc_off"])
    case = dict(doc_off=m["doc_off"], chunk_off=co, q=m["q"], K_bar=m["K_bar"], V_bar=m["V_bar"], K_loc=m["K_loc"],
                V_loc=m["V_loc"], loc_len=m["loc_len"], topk=m["planted_docs"])
    out = _attend(msa, d, case, cuda_device, pos_offset=m["pos_offset"])
    for b in [0, 7, 31]:
        sub = {kk: (v[b:b + 1] if kk in ("q", "K_loc", "V_loc", "loc_len", "topk") else v) for kk, v in case.items()}
        check_attention(out[b:b + 1], _oracle(sub, m["pos_offset"], d.rope_base), where=f"b={b}")


def _rotated_cache(msa, dims, c, device, pos_offset):
    """The local keys rotated in place on the GPU at pos_offset + j (every row of the cache)."""
    import torch

    B, T, n_kv, D = c["K_loc"].shape
    K = _dev(c["K_loc"], device).reshape(B * T, n_kv, D).clone()
    pos = (pos_offset + torch.arange(T, dtype=torch.int32, device=device)).repeat(B)
    msa.rope_rows(dims, K, pos)
    return K.reshape(B, T, n_kv, D)


def test_rope_rows_matches_oracle_rotation(msa, cuda_device):
    import torch

    from helpers import torch_bits

    rng = np.random.default_rng(12)
    for D, base in [(128, 1e6), (64, 1e4)]:
        x = W.normal_bf16(rng, (300, 3, D))
        pos = rng.integers(0, 200000, size=300).astype(np.int32)
        dims = W.Dims(hidden=256, n_q=3, n_kv=3, head_dim=D, n_r=4, d_r=64, rope_base=base)
        xd = _dev(x, cuda_device)
        msa.rope_rows(dims, xd, torch.from_numpy(pos).to(cuda_device))
        torch.cuda.synchronize()
        got = O.bf16_to_f64(torch_bits(xd))
        want = O.rope(O.bf16_to_f64(x), pos[:, None], base)
        # one bf16 rounding of the rotated value
        assert np.all(np.abs(got - want) <= 2.0 ** -8 * np.abs(want) + 1e-6)


@pytest.mark.parametrize("D,n_q,n_kv", [(128, 32, 8), (64, 8, 2), (128, 16, 1)])
def test_attend_rotated_cache_mode(msa, cuda_device, D, n_q, n_kv):
    import torch

    c = _case(40 + D + n_kv, 3, n_q, n_kv, D, n_docs=30, k=5, t_loc=300)
    dims = W.Dims(hidden=256, n_q=n_q, n_kv=n_kv, head_dim=D, n_r=4, d_r=64, rope_base=1e6)
    Krot = _rotated_cache(msa, dims, c, cuda_device, 5)
    co, C = msa.chunk_offsets(c["doc_off"])
    out = msa.sparse_attend(dims, _dev(c["q"], cuda_device), _dev(c["K_bar"], cuda_device),
                            _dev(c["V_bar"], cuda_device), torch.from_numpy(co).to(cuda_device),
                            torch.from_numpy(c["topk"].astype(np.int32)).to(cuda_device), Krot,
                            _dev(c["V_loc"], cuda_device), torch.from_numpy(c["loc_len"].astype(np.int32)).to(cuda_device),
                            5, k_loc_rotated=True)
    torch.cuda.synchronize()
    assert msa.check_device_errors() == 0
    check_attention(out.float().cpu().numpy(), _oracle(c, 5, 1e6), where=f"rotated D={D}")


def test_attend_rotated_cache_mem16m_sampled(msa, cuda_device):
    import torch

    m = W.mem16m_config(LAYOUT)
    d = m["dims"]
    co, *_ = O.chunk_layout(m["doc_off"])
    case = dict(doc_off=m["doc_off"], chunk_off=co, q=m["q"], K_bar=m["K_bar"], V_bar=m["V_bar"], K_loc=m["K_loc"],
                V_loc=m["V_loc"], loc_len=m["loc_len"], topk=m["planted_docs"])
    Krot = _rotated_cache(msa, d, case, cuda_device, m["pos_offset"])
    out = msa.sparse_attend(d, _dev(m["q"], cuda_device), _dev(m["K_bar"], cuda_device), _dev(m["V_bar"], cuda_device),
                            torch.from_numpy(co.astype(np.int32)).to(cuda_device),
                            torch.from_numpy(m["planted_docs"].astype(np.int32)).to(cuda_device), Krot,
                            _dev(m["V_loc"], cuda_device), torch.from_numpy(m["loc_len"]).to(cuda_device),
                            m["pos_offset"], k_loc_rotated=True).float().cpu().numpy()
    for b in [0, 13, 31]:
        sub = {kk: (v[b:b + 1] if kk in ("q", "K_loc", "V_loc", "loc_len", "topk") else v) for kk, v in case.items()}
        check_attention(out[b:b + 1], _oracle(sub, m["pos_offset"], d.rope_base), where=f"b={b}")


@pytest.mark.parametrize("B,D,n_kv", [(1, 128, 8), (4, 64, 2)])
def test_host_tier_gather_then_attend(msa, cuda_device, B, D, n_kv):
    import torch

    from helpers import torch_bits

    n_q = 4 * n_kv
    c = _case(70 + B, B, n_q, n_kv, D, n_docs=50, k=6, t_loc=100)
    dims = W.Dims(hidden=256, n_q=n_q, n_kv=n_kv, head_dim=D, n_r=4, d_r=64, rope_base=1e6)
    co, C = msa.chunk_offsets(c["doc_off"])
    dev = cuda_device
    Kh = W.to_torch(c["K_bar"]).pin_memory()
    Vh = W.to_torch(c["V_bar"]).pin_memory()
    topk = torch.from_numpy(c["topk"].astype(np.int32)).to(dev)
    chunk_off = torch.from_numpy(co).to(dev)
    Ks, Vs, soff, sidx = msa.gather_kv(dims, Kh, Vh, chunk_off, topk, capacity_chunks=C)
    torch.cuda.synchronize()
    assert msa.check_device_errors() == 0
    # the staging holds exactly the selected documents' rows, query by query in top-k order
    so = soff.cpu().numpy()
    assert so[0] == 0
    assert sidx.cpu().tolist() == [[b * 6 + r for r in range(6)] for b in range(B)]
    Ksb = torch_bits(Ks)
    for b in range(B):
        for r in range(6):
            doc = c["topk"][b, r]
            i = b * 6 + r
            assert so[i + 1] - so[i] == co[doc + 1] - co[doc]
            assert np.array_equal(Ksb[so[i]:so[i + 1]], c["K_bar"][co[doc]:co[doc + 1]])
    out = msa.sparse_attend(dims, _dev(c["q"], dev), Ks, Vs, soff, sidx, _dev(c["K_loc"], dev), _dev(c["V_loc"], dev),
                            torch.from_numpy(c["loc_len"].astype(np.int32)).to(dev), 6)
    torch.cuda.synchronize()
    check_attention(out.float().cpu().numpy(), _oracle(c, 6, 1e6), where="host tier")


def test_host_tier_rejects_pageable_memory(msa, cuda_device):
    import torch

    dims = W.Dims(hidden=256, n_q=8, n_kv=2, head_dim=64, n_r=4, d_r=64)
    K = torch.zeros((10, 2, 64), dtype=torch.bfloat16)          # pageable, not pinned
    V = torch.zeros((10, 2, 64), dtype=torch.bfloat16)
    co = torch.tensor([0, 5, 10], dtype=torch.int32, device=cuda_device)
    tk = torch.tensor([[0]], dtype=torch.int32, device=cuda_device)
    with pytest.raises(msa.MSAError) as e:
        msa.gather_kv(dims, K, V, co, tk, capacity_chunks=10)
    assert e.value.code == 1 and "pinned" in str(e.value)


def test_kv_append_matches_rotation_and_copy(msa, cuda_device):
    # the fused append = rotate a copy of the new key at pos_offset + slot, copy both rows in
    import torch
    from helpers import torch_bits

    rng = np.random.default_rng(61)
    B, T, n_kv, D, o = 3, 40, 8, 128, 16
    dims = W.Dims(hidden=256, n_q=32, n_kv=n_kv, head_dim=D, n_r=4, d_r=64, rope_base=1e6)
    K = _dev(W.normal_bf16(rng, (B, T, n_kv, D)), cuda_device)
    V = _dev(W.normal_bf16(rng, (B, T, n_kv, D)), cuda_device)
    kn_np = W.normal_bf16(rng, (B, n_kv, D))
    kn, vn = _dev(kn_np, cuda_device), _dev(W.normal_bf16(rng, (B, n_kv, D)), cuda_device)
    slots = torch.tensor([0, 17, T - 1], dtype=torch.int32, device=cuda_device)
    K0, V0 = K.clone(), V.clone()
    msa.kv_append(dims, kn, vn, K, V, slots, o)
    ref = kn.clone()
    msa.rope_rows(dims, ref, (o + slots).to(torch.int32))
    torch.cuda.synchronize()
    assert msa.check_device_errors() == 0
    for b, s in enumerate(slots.tolist()):
        assert torch.equal(K[b, s], ref[b]) and torch.equal(V[b, s], vn[b])
        want = O.rope(O.bf16_to_f64(kn_np[b]), o + s, 1e6)
        got = O.bf16_to_f64(torch_bits(K[b, s]))
        assert np.all(np.abs(got - want) <= 2.0 ** -8 * np.abs(want) + 1e-6)
        keep = [t for t in range(T) if t != s]
        assert torch.equal(K[b, keep], K0[b, keep]) and torch.equal(V[b, keep], V0[b, keep])
    # a slot outside the cache is skipped and reported
    bad = torch.tensor([T, 0, -1], dtype=torch.int32, device=cuda_device)
    K1 = K.clone()
    msa.kv_append(dims, kn, vn, K, V, bad, o)
    torch.cuda.synchronize()
    with pytest.raises(msa.MSAError, match="out-of-range index"):
        msa.check_device_errors()
    assert msa.check_device_errors() == 0   # reading the word clears it
    assert torch.equal(K[0], K1[0]) and torch.equal(K[2], K1[2])


@pytest.mark.parametrize("rotated,M,B", [(True, 1, 1), (False, 1, 3), (True, 4, 2), (False, 3, 5)])
def test_attend_two_phase_equals_one_call(msa, cuda_device, rotated, M, B):
    # phase 1 (local keys) then phase 2 (selected chunks + merge) on one workspace
    import torch

    rng = np.random.default_rng(90 + M + B)
    n_q, n_kv, D = 32, 8, 128
    c = _case(91 + M + B, B, n_q, n_kv, D, n_docs=30, k=6, t_loc=200, loc_len=rng.integers(M, 201, size=B))
    c["q"] = W.normal_bf16(rng, (B, M, n_q, D)) if M > 1 else c["q"]
    dims = W.Dims(hidden=256, n_q=n_q, n_kv=n_kv, head_dim=D, n_r=4, d_r=64, rope_base=1e6)
    dev = cuda_device
    co, C = msa.chunk_offsets(c["doc_off"])
    K_loc = _dev(c["K_loc"], dev)
    if rotated:
        pos = (5 + torch.arange(200, dtype=torch.int32, device=dev)).repeat(B)
        msa.rope_rows(dims, K_loc.view(B * 200, n_kv, D), pos)
    args = (dims, _dev(c["q"], dev), _dev(c["K_bar"], dev), _dev(c["V_bar"], dev), torch.from_numpy(co).to(dev),
            torch.from_numpy(c["topk"].astype(np.int32)).to(dev), K_loc, _dev(c["V_loc"], dev),
            torch.from_numpy(c["loc_len"].astype(np.int32)).to(dev), 5)
    one = msa.sparse_attend(*args, k_loc_rotated=rotated)
    ws = torch.empty(msa.attend_workspace_size(dims, B, 6, 200, 5, M) + 256, dtype=torch.uint8, device=dev)
    out = torch.zeros_like(one)
    msa.sparse_attend(*args, k_loc_rotated=rotated, phase=1, ws=ws, out=out)
    msa.sparse_attend(*args, k_loc_rotated=rotated, phase=2, ws=ws, out=out)
    torch.cuda.synchronize()
    assert msa.check_device_errors() == 0
    a, b = one.float().cpu().numpy(), out.float().cpu().numpy()
    assert np.array_equal(a, b)  # the same splits and partial slots as the one-launch call
    if M == 1:
        check_attention(b, _oracle(c, 5, 1e6), where=f"two-phase B={B}")
    else:
        ref = O.sparse_attend_tokens(c["q"], c["K_bar"], c["V_bar"], c["chunk_off"], c["topk"], c["K_loc"], c["V_loc"],
                                     c["loc_len"], 5, 1e6)
        check_attention(b, ref, where=f"two-phase M={M}")


@pytest.mark.parametrize("B,M", [(1, 1), (3, 1), (2, 4)])
def test_attend_early_local_behind_routing(msa, cuda_device, B, M):
    # append -> route -> attend on one stream, the attention's local-key work allowed to start
    # while the routing kernels finish: the same result, bit for bit, as the ordinary call,
    # and the oracle's attention over the routed documents
    import torch

    rng = np.random.default_rng(700 + B + M)
    n_q, n_kv, D, n_r, d_r, k, T_loc = 32, 8, 128, 8, 128, 16, 1024
    lens = np.clip(rng.lognormal(np.log(2048), 0.5, size=300).astype(np.int64), 64, 32768)
    doc_off = W.offsets_from_lengths(lens)
    co, C = msa.chunk_offsets(doc_off)
    dims = W.Dims(hidden=256, n_q=n_q, n_kv=n_kv, head_dim=D, n_r=n_r, d_r=d_r, rope_base=1e6)
    dev = cuda_device
    KR = _dev(W.normal_bf16(rng, (C, n_r, d_r)), dev)
    K_bar_np, V_bar_np = W.normal_bf16(rng, (C, n_kv, D)), W.normal_bf16(rng, (C, n_kv, D))
    K_loc_np, V_loc_np = W.normal_bf16(rng, (B, T_loc, n_kv, D)), W.normal_bf16(rng, (B, T_loc, n_kv, D))
    q_np = W.normal_bf16(rng, (B, M, n_q, D)) if M > 1 else W.normal_bf16(rng, (B, n_q, D))
    QR = _dev(W.normal_bf16(rng, (B * M, n_r * d_r)), dev)
    loc_len_np = rng.integers(max(M, T_loc // 2), T_loc + 1, size=B).astype(np.int32)
    K_bar, V_bar, q = _dev(K_bar_np, dev), _dev(V_bar_np, dev), _dev(q_np, dev)
    K_loc, V_loc = _dev(K_loc_np, dev), _dev(V_loc_np, dev)
    co_d, loc_len = torch.from_numpy(co).to(dev), torch.from_numpy(loc_len_np).to(dev)
    o = k
    pos = (o + torch.arange(T_loc, dtype=torch.int32, device=dev)).repeat(B)
    msa.rope_rows(dims, K_loc.view(B * T_loc, n_kv, D), pos)
    # the append writes the last slot of each query with its own (rotated) row: a no-op on values
    slots = torch.from_numpy(loc_len_np - 1).to(dev)
    kn_np = W.normal_bf16(rng, (B, n_kv, D))
    k_new = _dev(kn_np, dev)
    v_new = V_loc[torch.arange(B, device=dev), slots.long()].clone()
    ws = torch.empty(msa.attend_workspace_size(dims, B, k, T_loc, o, M) + 256, dtype=torch.uint8, device=dev)
    outs = []
    for early in (True, False, True):
        msa.kv_append(dims, k_new, v_new, K_loc, V_loc, slots, o)
        idx, _, _ = msa.route_topk(dims, QR, None, KR, co_d, k, q_tokens=M)
        out = msa.sparse_attend(dims, q, K_bar, V_bar, co_d, idx, K_loc, V_loc, loc_len, o, ws=ws,
                                k_loc_rotated=True, early_local=early)
        torch.cuda.synchronize()
        assert msa.check_device_errors() == 0
        outs.append(out.float().cpu().numpy())
    assert np.array_equal(outs[0], outs[1]) and np.array_equal(outs[2], outs[1])
    # the oracle, on the routed documents and the cache as appended (keys before RoPE)
    K_loc_ref = K_loc_np.copy()
    for b in range(B):
        K_loc_ref[b, loc_len_np[b] - 1] = kn_np[b]
    topk = idx.cpu().numpy()
    if M == 1:
        ref = O.sparse_attend(q_np, K_bar_np, V_bar_np, co, topk, K_loc_ref, V_loc_np, loc_len_np, o, 1e6)
    else:
        ref = O.sparse_attend_tokens(q_np, K_bar_np, V_bar_np, co, topk, K_loc_ref, V_loc_np, loc_len_np, o, 1e6)
    check_attention(outs[0], ref, where=f"early B={B} M={M}")


@pytest.mark.parametrize("rotated", [True, False])
@pytest.mark.parametrize("early", [False, True])
def test_attend_fused_append_equals_append_then_attend(msa, cuda_device, rotated, early):
    # sparse_attend with k_new / v_new = the new token written at slot loc_len - 1 (rotated at its
    # position for a rotated cache, as kv_append does; as given for a pre-RoPE cache), then the
    # attention: the same output and the same cache, bit for bit
    import torch

    B, n_q, n_kv, D, T, o = 3, 32, 8, 128, 300, 6
    c = _case(820 + rotated + 2 * early, B, n_q, n_kv, D, n_docs=30, k=5, t_loc=T, loc_len=[T, 57, 1])
    dims = W.Dims(hidden=256, n_q=n_q, n_kv=n_kv, head_dim=D, n_r=4, d_r=64, rope_base=1e6)
    dev = cuda_device
    rng = np.random.default_rng(821)
    kn = _dev(W.normal_bf16(rng, (B, n_kv, D)), dev)
    vn = _dev(W.normal_bf16(rng, (B, n_kv, D)), dev)
    co, C = msa.chunk_offsets(c["doc_off"])
    K0 = _dev(c["K_loc"], dev)
    if rotated:
        msa.rope_rows(dims, K0.view(B * T, n_kv, D), (o + torch.arange(T, dtype=torch.int32, device=dev)).repeat(B))
    V0 = _dev(c["V_loc"], dev)
    loc_len = torch.from_numpy(c["loc_len"].astype(np.int32)).to(dev)
    slots = loc_len - 1
    args = (_dev(c["q"], dev), _dev(c["K_bar"], dev), _dev(c["V_bar"], dev), torch.from_numpy(co).to(dev),
            torch.from_numpy(c["topk"].astype(np.int32)).to(dev))
    K1, V1, K2, V2 = K0.clone(), V0.clone(), K0.clone(), V0.clone()
    if rotated:
        msa.kv_append(dims, kn, vn, K1, V1, slots, o)
    else:
        for b in range(B):
            K1[b, int(slots[b])] = kn[b]
            V1[b, int(slots[b])] = vn[b]
    ref = msa.sparse_attend(dims, *args, K1, V1, loc_len, o, k_loc_rotated=rotated)
    out = msa.sparse_attend(dims, *args, K2, V2, loc_len, o, k_loc_rotated=rotated, early_local=early,
                            k_new=kn, v_new=vn)
    torch.cuda.synchronize()
    assert msa.check_device_errors() == 0
    assert torch.equal(K1, K2) and torch.equal(V1, V2)
    assert torch.equal(ref, out)
    # no local position for the new token: reported, nothing written
    K3, V3 = K0.clone(), V0.clone()
    zero = torch.zeros_like(loc_len)
    msa.sparse_attend(dims, *args, K3, V3, zero, o, k_loc_rotated=rotated, k_new=kn, v_new=vn)
    torch.cuda.synchronize()
    with pytest.raises(msa.MSAError, match="out-of-range index"):
        msa.check_device_errors()
    assert torch.equal(K3, K0) and torch.equal(V3, V0)
