"""Host-side tests of the C ABI: the library loads, exports every declared
symbol, computes the chunk layout, sizes workspaces and rejects bad arguments
with the documented status before launching anything (no GPU needed)."""
import ctypes
import os
import re

import numpy as np
import pytest

import oracle as O
from long_context_memory_b200 import workloads as W

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def msa():
    from long_context_memory_b200 import build

    if build.needs_build():
        build.build()
    import long_context_memory_b200 as m

    return m


def declared_symbols():
    src = open(os.path.join(ROOT, "include", "msa.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(msa_[a-z_0-9]+)\s*\(", src)))


def test_exports_every_declared_symbol(msa):
    names = declared_symbols()
    assert len(names) >= 14
    cdll = ctypes.CDLL(msa.LIB_PATH)
    for n in names:
        assert hasattr(cdll, n), f"missing export {n}"
    assert msa.lib.msa_version() >= 100


def test_library_targets_sm100a_only(msa):
    # the build passes exactly one gencode: compute_100a -> sm_100a
    from long_context_memory_b200 import build

    src = open(build.__file__).read()
    assert "arch=compute_100a,code=sm_100a" in src


@pytest.mark.parametrize("lens", [[1], [64, 65, 1, 128], [3000, 7, 64 * 9 + 1]])
def test_chunk_offsets_match_oracle(msa, lens):
    doc_off = W.offsets_from_lengths(np.asarray(lens))
    co, n = msa.chunk_offsets(doc_off)
    o_co, tok0, *_ = O.chunk_layout(doc_off)
    assert np.array_equal(co, o_co) and n == len(tok0)


def test_chunk_offsets_rejects_empty_doc(msa):
    with pytest.raises(msa.MSAError) as e:
        msa.chunk_offsets(np.array([0, 5, 5, 9]))
    assert e.value.code == 1 and "document 1" in str(e.value)


def _dims(**kw):
    d = dict(hidden=256, n_q=8, n_kv=2, head_dim=64, n_r=4, d_r=64, chunk=64, rope_base=1e6)
    d.update(kw)
    return W.Dims(**d)


FAKE = 0x10000  # 16-byte aligned non-null "device" address; never dereferenced


def _route(msa, dims, B=1, n_docs=10, n_chunks=20, k=4, agg=0, ws_bytes=None, Hq=FAKE, kr=FAKE, idx=FAKE, layout=0,
           M=1):
    dd = msa.Dims.of(dims)
    need = msa.lib.msa_route_workspace_size(ctypes.byref(dd), B, max(M, 1), n_docs, n_chunks, k, agg)
    if ws_bytes is None:
        ws_bytes = need
    return msa.lib.msa_route_topk(ctypes.byref(dd), Hq, None, B, M, kr, FAKE, n_docs, n_chunks, k, agg, layout, None,
                                  None, idx,
                                  FAKE,
                                  0x100000 if ws_bytes else None, ws_bytes, None)


def test_route_validation(msa):
    ok = _dims()
    assert _route(msa, ok, k=0) == 1
    assert _route(msa, ok, k=11) == 1                       # k > n_docs
    assert _route(msa, ok, B=0) == 1
    assert _route(msa, ok, n_chunks=5) == 1                 # fewer chunks than docs
    assert _route(msa, _dims(d_r=96)) == 2                  # unsupported router dim
    assert _route(msa, _dims(n_r=9)) == 2
    assert _route(msa, _dims(chunk=32)) == 2
    assert _route(msa, ok, Hq=FAKE + 4) == 1                # misaligned
    assert _route(msa, ok, kr=None) == 1                    # NULL
    assert _route(msa, ok, agg=7) == 1
    assert _route(msa, ok, layout=2) == 1                   # K̄^R layout is 0 (chunk-major) or 1 (head-major)
    assert _route(msa, ok, M=0) == 1                        # at least one query token
    assert _route(msa, ok, B=4096, M=17) == 1               # B * M above 65535
    assert _route(msa, ok, ws_bytes=16) == 3                # workspace too small
    assert "workspace too small" in msa.lib.msa_last_error().decode()


def test_route_fault_injection_before_launch(msa, monkeypatch):
    monkeypatch.setenv("MSA_FAULT", "launch")
    assert _route(msa, _dims()) == 4
    assert "injected" in msa.lib.msa_last_error().decode()


def _attend(msa, dims, B=1, k=2, n_docs=4, n_chunks=8, t_loc=16, pos=2, scale=0.0, ws_bytes=None, q=FAKE, M=1,
            phase=0, k_new=None, v_new=None):
    dd = msa.Dims.of(dims)
    need = msa.lib.msa_attend_workspace_size(ctypes.byref(dd), B, max(M, 1), k, t_loc, pos)
    if ws_bytes is None:
        ws_bytes = need
    return msa.lib.msa_sparse_attend(ctypes.byref(dd), q, B, M, FAKE, FAKE, FAKE, n_docs, n_chunks, FAKE, k, FAKE, FAKE,
                                     k_new, v_new, FAKE, t_loc, pos, None, 0, scale, phase, FAKE, 0x100000, ws_bytes,
                                     None)


def test_attend_validation(msa):
    ok = _dims()
    assert _attend(msa, _dims(head_dim=96)) == 2
    assert _attend(msa, _dims(n_q=6, n_kv=4)) == 1          # n_q not a multiple of n_kv
    assert _attend(msa, _dims(n_q=64, n_kv=2)) == 2         # GQA group > 16
    assert _attend(msa, _dims(n_q=16, n_kv=16)) == 2        # more than 8 KV heads
    assert _attend(msa, ok, k=5) == 1                       # k > n_docs
    assert _attend(msa, ok, pos=-1) == 1
    assert _attend(msa, ok, scale=float("nan")) == 1
    assert _attend(msa, ok, q=FAKE + 2) == 1
    assert _attend(msa, ok, ws_bytes=8) == 3
    assert _attend(msa, ok, M=0) == 1
    assert _attend(msa, ok, phase=3) == 1
    assert _attend(msa, ok, phase=3 | msa.ATTEND_EARLY_LOCAL) == 1  # the flag does not make a bad phase valid
    assert _attend(msa, ok, phase=-1) == 1
    assert _attend(msa, ok, phase=msa.ATTEND_EARLY_LOCAL | 32) == 1  # an unknown flag bit
    assert _attend(msa, ok, k_new=FAKE) == 1                        # k_new without v_new
    assert _attend(msa, ok, k_new=FAKE, v_new=FAKE, M=2) == 1       # the fused append is for M = 1
    assert _attend(msa, ok, k_new=FAKE, v_new=FAKE, phase=2) == 1   # phase 2 reads no local keys
    assert _attend(msa, ok, k_new=FAKE, v_new=FAKE, t_loc=0) == 1   # no local cache to write
    assert _attend(msa, ok, k_new=FAKE + 2, v_new=FAKE) == 1        # misaligned


def test_encode_validation(msa):
    dd = msa.Dims.of(_dims(hidden=100))
    r = msa.lib.msa_encode_memory(ctypes.byref(dd), FAKE, 1000, FAKE, 3, FAKE, 20, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE,
                                  0, None, 0, None)
    assert r == 2
    dd = msa.Dims.of(_dims())
    need = msa.lib.msa_encode_workspace_size(ctypes.byref(dd), 1000, 3, 20)
    for layout, want in ((2, 1), (-1, 1)):
        r = msa.lib.msa_encode_memory(ctypes.byref(dd), FAKE, 1000, FAKE, 3, FAKE, 20, FAKE, FAKE, FAKE, FAKE, FAKE,
                                      FAKE, layout, 0x100000, need, None)
        assert r == want, (layout, r, msa.lib.msa_last_error())


def test_append_validation(msa):
    dd = msa.Dims.of(_dims())
    need = msa.lib.msa_encode_workspace_size(ctypes.byref(dd), 1000, 3, 20)
    # 20 new chunks after 90 do not fit a capacity of 100
    r = msa.lib.msa_append_memory(ctypes.byref(dd), FAKE, 1000, FAKE, 3, FAKE, 20, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE,
                                  100, FAKE, 30, 90, 0x100000, need, None)
    assert r == 1 and "capacity" in msa.lib.msa_last_error().decode()
    r = msa.lib.msa_append_memory(ctypes.byref(dd), FAKE, 1000, FAKE, 3, FAKE, 20, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE,
                                  200, None, 30, 90, 0x100000, need, None)
    assert r == 1                                                              # NULL chunk_off


def test_aux_loss_validation(msa):
    dd = msa.Dims.of(_dims())
    lib = msa.lib
    need = lib.msa_aux_loss_workspace_size(ctypes.byref(dd), 4, 8)
    assert need > 0
    call = lambda P=4, N=8, tau=0.1, ws=need, kn=FAKE: lib.msa_aux_loss(
        ctypes.byref(dd), FAKE, FAKE, kn, P, N, tau, FAKE, FAKE, None, None, 0x100000, ws, None)
    assert call(P=0) == 1
    assert call(N=1024) == 1
    assert call(tau=0.0) == 1
    assert call(tau=float("inf")) == 1
    assert call(kn=None) == 1            # N > 0 needs negatives
    assert call(ws=4) == 3
    assert lib.msa_aux_loss(ctypes.byref(msa.Dims.of(_dims(d_r=96))), FAKE, FAKE, FAKE, 4, 8, 0.1, FAKE, None, None,
                            None, 0x100000, need, None) == 2


def test_kv_append_validation(msa):
    dd = msa.Dims.of(_dims())
    lib = msa.lib
    assert lib.msa_kv_append(ctypes.byref(dd), FAKE, FAKE, FAKE, FAKE, 0, 16, FAKE, 2, None) == 1   # B < 1
    assert lib.msa_kv_append(ctypes.byref(dd), FAKE, FAKE, FAKE, FAKE, 1, 16, None, 2, None) == 1   # no slots
    assert lib.msa_kv_append(ctypes.byref(dd), FAKE + 2, FAKE, FAKE, FAKE, 1, 16, FAKE, 2, None) == 1
    assert lib.msa_kv_append(ctypes.byref(dd), FAKE, FAKE, FAKE, FAKE, 1, 16, FAKE, -1, None) == 1
    assert lib.msa_kv_append(ctypes.byref(msa.Dims.of(_dims(head_dim=96))), FAKE, FAKE, FAKE, FAKE, 1, 16, FAKE, 2,
                             None) == 2


def test_router_key_norms_validation(msa):
    lib = msa.lib
    dd = msa.Dims.of(_dims())
    assert lib.msa_router_key_norms(ctypes.byref(dd), FAKE, 0, 0, FAKE, None) == 1       # no chunks
    assert lib.msa_router_key_norms(ctypes.byref(dd), FAKE, 10, 2, FAKE, None) == 1      # layout
    assert lib.msa_router_key_norms(ctypes.byref(dd), FAKE, 10, 0, None, None) == 1      # NULL output
    assert lib.msa_router_key_norms(ctypes.byref(msa.Dims.of(_dims(d_r=96))), FAKE, 10, 0, FAKE, None) == 2


def test_topk_merge_validation(msa):
    lib = msa.lib
    assert lib.msa_topk_merge(FAKE, FAKE, 1, 8, 9, FAKE, FAKE, None) == 1      # k > n_cand
    assert lib.msa_topk_merge(FAKE, FAKE, 0, 8, 4, FAKE, FAKE, None) == 1      # B < 1
    assert lib.msa_topk_merge(FAKE, FAKE + 4, 1, 8, 4, FAKE, FAKE, None) == 1  # misaligned
    assert lib.msa_topk_merge(FAKE, FAKE, 1, 30000, 4, FAKE, FAKE, None) == 1  # too many candidates


def _tiered(msa, dims, layers=None, n_layers=1, B=1, n_docs=10, n_chunks=20, k=4, t_loc=16, pos=4, cap=64,
            ws_bytes=None, **ptrs):
    dd = msa.Dims.of(dims)
    if layers is None:
        layers = (msa.Layer * max(1, n_layers))()
        for L in layers:
            for f in ("Hq", "KR_bar", "K_bar_host", "V_bar_host", "q", "K_loc", "V_loc", "topk_idx", "topk_score",
                      "out"):
                setattr(L, f, FAKE)
            for f, v in ptrs.items():
                setattr(L, f, v)
    need = msa.lib.msa_tiered_workspace_size(ctypes.byref(dd), max(1, n_layers), B, n_docs, n_chunks, k, t_loc, pos, cap)
    if ws_bytes is None:
        ws_bytes = need
    return msa.lib.msa_tiered_decode(ctypes.byref(dd), layers, n_layers, B, FAKE, n_docs, n_chunks, k, FAKE, t_loc, pos,
                                     cap, 0x100000, ws_bytes, None, None)


def test_tiered_validation(msa):
    # every argument error is reported before the pinned-memory lookup and before any launch
    ok = _dims(hidden=512, n_q=32, n_kv=8, head_dim=128, n_r=8, d_r=128)
    assert _tiered(msa, ok, n_layers=0) == 1
    assert msa.lib.msa_tiered_decode(ctypes.byref(msa.Dims.of(ok)), None, 1, 1, FAKE, 10, 20, 4, FAKE, 16, 4, 64,
                                     0x100000, 1 << 20, None, None) == 1
    assert _tiered(msa, ok, k=11) == 1                       # k > n_docs
    assert _tiered(msa, ok, B=0) == 1
    assert _tiered(msa, ok, t_loc=0) == 1                    # the attention needs a local cache
    assert _tiered(msa, ok, cap=0) == 1
    assert _tiered(msa, _dims(head_dim=96)) == 2
    assert _tiered(msa, ok, q=FAKE + 4) == 1                 # misaligned
    assert "layer 0" in msa.lib.msa_last_error().decode()
    assert _tiered(msa, ok, K_bar_host=None) == 1
    assert _tiered(msa, ok, k_new=FAKE) == 1                 # k_new without v_new
    dd = ctypes.byref(msa.Dims.of(ok))
    small = msa.lib.msa_tiered_workspace_size(dd, 1, 1, 10, 20, 4, 16, 4, 64)
    big = msa.lib.msa_tiered_workspace_size(dd, 1, 1, 10, 20, 4, 16, 4, 128)
    # two staging areas of K and V rows (n_kv * head_dim bf16 each) per extra chunk of capacity
    assert small > 0 and big - small >= 4 * 64 * 8 * 128 * 2 - 4 * 256
    assert msa.lib.msa_tiered_workspace_size(dd, 1, 1, 10, 20, 4, 16, 4, 0) == 0
    # each layer adds its router-query rows: n_r heads x (hi, lo) x 16 padded rows x d_r bf16
    more = msa.lib.msa_tiered_workspace_size(dd, 3, 1, 10, 20, 4, 16, 4, 64)
    assert more - small == 2 * 8 * 2 * 16 * 128 * 2
    assert msa.lib.msa_tiered_workspace_size(dd, 0, 1, 10, 20, 4, 16, 4, 64) == 0
    # the layout's chunk -> document map: one int32 per chunk (to within the 256-byte carving)
    wide = msa.lib.msa_tiered_workspace_size(dd, 1, 1, 10, 20 + 64 * 256, 4, 16, 4, 64)
    assert 64 * 256 * 4 <= wide - small <= 64 * 256 * 4 + 4 * 256 + 4 * 64 * 256 // 10


def test_workspace_sizes_grow_with_problem(msa):
    d = msa.Dims.of(W.QWEN3_4B_DIMS)
    a = msa.lib.msa_route_workspace_size(ctypes.byref(d), 1, 1, 500, 16000, 16, 0)
    b = msa.lib.msa_route_workspace_size(ctypes.byref(d), 32, 1, 500, 16000, 16, 0)
    c = msa.lib.msa_route_workspace_size(ctypes.byref(d), 32, 8, 500, 16000, 16, 0)
    assert 0 < a < b < c
    assert msa.lib.msa_route_workspace_size(ctypes.byref(d), 0, 1, 500, 16000, 16, 0) == 0
    x = msa.lib.msa_attend_workspace_size(ctypes.byref(d), 1, 1, 16, 4096, 16)
    assert x >= 4096 * 64 * 8   # the local RoPE table alone
    assert msa.lib.msa_attend_workspace_size(ctypes.byref(d), 1, 8, 16, 4096, 16) > x


def _header_functions():
    """name -> (return type, parameter count) of every function declared in msa.h."""
    src = open(os.path.join(ROOT, "include", "msa.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    out = {}
    for ret, name, params in re.findall(
            r"\b(msa_status|size_t|int32_t|const char\s*\*)\s+(msa_[a-z_0-9]+)\s*\(([^)]*)\)\s*;", src):
        p = params.strip()
        out[name] = (re.sub(r"\s+", "", ret), 0 if p in ("", "void") else p.count(",") + 1)
    return out


def test_binding_signatures_match_header(msa):
    # ctypes marshals by the binding's argtypes: a parameter added to the header but not to the
    # binding would shift every later argument silently
    hdr = _header_functions()
    assert set(hdr) == set(declared_symbols())
    cdll = msa._load()
    restype = {"msa_status": ctypes.c_int32, "size_t": ctypes.c_size_t, "int32_t": ctypes.c_int32,
               "constchar*": ctypes.c_char_p}
    unbound = set()
    for name, (ret, n) in hdr.items():
        fn = getattr(cdll, name)
        if fn.argtypes is None:
            unbound.add(name)
            continue
        assert len(fn.argtypes) == n, (name, len(fn.argtypes), n)
        assert fn.restype is restype[ret], (name, fn.restype, ret)
    # the one entry point the binding leaves to direct ctypes callers (its test declares it itself)
    assert unbound == {"msa_route_topk_static"}, unbound


def test_binding_constants_match_header(msa):
    src = open(os.path.join(ROOT, "include", "msa.h")).read()
    defines = dict((k, int(v)) for k, v in re.findall(r"#define (MSA_[A-Z_]+) (\d+)", src))
    assert defines["MSA_ROUTE_EARLY_INPUTS"] == msa.ROUTE_EARLY_INPUTS
    assert defines["MSA_ATTEND_EARLY_LOCAL"] == msa.ATTEND_EARLY_LOCAL
    enums = dict((k, int(v)) for k, v in re.findall(r"\b(MSA_[A-Z_]+) = (\d+)", src))
    for code, name in msa.STATUS.items():
        assert enums[name] == code, name
    assert enums["MSA_AGG_MAX"] == msa.AGG_MAX and enums["MSA_AGG_MEAN"] == msa.AGG_MEAN


def test_fused_append_rows_checked_by_the_binding(msa):
    # k_new / v_new are read by their sizes alone: a wrong shape, dtype or layout is refused
    # before anything is launched
    import torch

    d = _dims()
    B = 2
    q = torch.zeros(B, d.n_q, d.head_dim, dtype=torch.bfloat16)
    idx = torch.zeros(B, 3, dtype=torch.int32)
    good = torch.zeros(B, d.n_kv, d.head_dim, dtype=torch.bfloat16)
    bad = [torch.zeros(B, d.n_kv, d.head_dim // 2, dtype=torch.bfloat16),
           torch.zeros(B, d.n_kv, d.head_dim, dtype=torch.float32),
           torch.zeros(d.n_kv, B, d.head_dim, dtype=torch.bfloat16).transpose(0, 1)]
    for kn in bad:
        for kw in (dict(k_new=kn, v_new=good), dict(k_new=good, v_new=kn)):
            with pytest.raises(ValueError):
                msa.sparse_attend(d, q, None, None, torch.zeros(4, dtype=torch.int32), idx, None, None, None, 4, **kw)


def test_kv_append_rows_and_slots_checked_by_the_binding(msa):
    import torch

    d = _dims()
    B, T = 3, 10
    K = torch.zeros(B, T, d.n_kv, d.head_dim, dtype=torch.bfloat16)
    rows = torch.zeros(B, d.n_kv, d.head_dim, dtype=torch.bfloat16)
    slots = torch.zeros(B, dtype=torch.int32)
    for args in ((rows[:2], rows, slots), (rows, rows.float(), slots), (rows, rows, slots.long()),
                 (rows, rows, slots[:2])):
        with pytest.raises(ValueError):
            msa.kv_append(d, args[0], args[1], K, K, args[2], 4)


def test_fault_injection_reaches_every_launching_entry_point(msa, monkeypatch):
    # MSA_FAULT=launch: each entry point validates its arguments, then fails with MSA_ERR_CUDA
    # before its first launch.  (msa_gather_kv first asks the driver whether its sources are
    # pinned, which needs a GPU, so it is not in this CPU list.)
    monkeypatch.setenv("MSA_FAULT", "launch")
    lib = msa.lib
    dd = msa.Dims.of(_dims())
    r = ctypes.byref(dd)
    enc = lib.msa_encode_workspace_size(r, 1000, 3, 17)
    aux = lib.msa_aux_loss_workspace_size(r, 4, 8)
    calls = {
        "route": lambda: _route(msa, _dims()),
        "attend": lambda: _attend(msa, _dims()),
        "encode": lambda: lib.msa_encode_memory(r, FAKE, 1000, FAKE, 3, FAKE, 17, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE,
                                                0, 0x100000, enc, None),
        "append": lambda: lib.msa_append_memory(r, FAKE, 1000, FAKE, 3, FAKE, 17, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE,
                                                200, FAKE, 30, 90, 0x100000, enc, None),
        "aux_loss": lambda: lib.msa_aux_loss(r, FAKE, FAKE, FAKE, 4, 8, 0.1, FAKE, FAKE, None, None, 0x100000, aux,
                                             None),
        "kv_append": lambda: lib.msa_kv_append(r, FAKE, FAKE, FAKE, FAKE, 1, 16, FAKE, 2, None),
        "router_key_norms": lambda: lib.msa_router_key_norms(r, FAKE, 10, 0, FAKE, None),
        "topk_merge": lambda: lib.msa_topk_merge(FAKE, FAKE, 1, 8, 4, FAKE, FAKE, None),
        "selftest_wait_timeout": lambda: lib.msa_selftest_wait_timeout(1000, 4, FAKE, None),
        "rope_rows": lambda: lib.msa_rope_rows(r, FAKE, 4, 2, FAKE, None),
        "rope_cache_build": lambda: lib.msa_rope_cache_build(r, 16, 2, 0x100000, lib.msa_rope_cache_size(r, 16),
                                                             None),
    }
    for name, call in calls.items():
        assert call() == 4, name
        assert "injected" in lib.msa_last_error().decode(), name
