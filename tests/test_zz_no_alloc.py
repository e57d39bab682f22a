"""msa_route_topk_static (routing on the library's own static scratch) against
msa_route_topk (routing on a caller workspace), through the C ABI.

The static entry point is for callers that cannot allocate device memory where
they route (an embedding host without a CUDA allocator, code inside a CUDA-graph
capture, loops that must not synchronise on cudaMalloc).  Two calls in a row must
match the workspace path: the second call runs on the scratch the first one left
behind, with other inputs (other queries, another memory layout), so stale
per-document maxima or a stale completion ticket would show.  With at most four
queries over one slice of documents the scan's last CTA selects the top-k and
its ticket lives in the static scratch too; with five queries the separate top-k
kernels run.  This file is collected last so that a failure here comes after
every other test has run.
"""
import ctypes

import numpy as np
import pytest

import oracle as O
from long_context_memory_b200 import workloads as W

pytestmark = pytest.mark.gpu


def _static_fn(msa):
    fn = msa.lib.msa_route_topk_static
    P, I32 = ctypes.c_void_p, ctypes.c_int32
    fn.restype = I32
    fn.argtypes = [ctypes.POINTER(msa.Dims), P, P, I32, I32, P, P, I32, I32, I32, I32, P, P, P, P]
    return fn


def _problem(msa, rng, dev, n_docs, B):
    import torch

    lens = rng.integers(1, 900, size=n_docs)
    co, C = msa.chunk_offsets(W.offsets_from_lengths(lens))
    KR = W.normal_bf16(rng, (C, 8, 128))
    Hq = W.normal_bf16(rng, (B, 512))
    Wqr = W.normal_bf16(rng, (512, 1024), 512 ** -0.5)
    t = lambda a: W.to_torch(a).to(dev)
    return dict(co=co, C=C, B=B, n_docs=n_docs, KR=KR, Hq=Hq, Wqr=Wqr, KR_d=t(KR), Hq_d=t(Hq), Wqr_d=t(Wqr),
                chunk_off=torch.from_numpy(co).to(dev))


@pytest.mark.parametrize("B", [3, 5])
def test_static_scratch_matches_workspace_path(cuda_device, B):
    import torch

    import long_context_memory_b200 as msa

    rng = np.random.default_rng(77 + B)
    dims = W.Dims(hidden=512, n_q=8, n_kv=2, head_dim=64, n_r=8, d_r=128)
    dev, k = cuda_device, 16
    # two different problems: another memory layout and other queries for the second call
    probs = [_problem(msa, rng, dev, 600, B), _problem(msa, rng, dev, 450, B)]
    fn = _static_fn(msa)
    dd = msa.Dims.of(dims)
    stream = torch.cuda.current_stream().cuda_stream
    results = []
    for call, p in enumerate(probs):
        ref_idx, ref_sc, ref_ds = msa.route_topk(dims, p["Hq_d"], p["Wqr_d"], p["KR_d"], p["chunk_off"], k,
                                                 want_doc_scores=True)
        idx = torch.full((B, k), -1, dtype=torch.int32, device=dev)
        sc = torch.zeros((B, k), dtype=torch.float32, device=dev)
        ds = torch.zeros((B, p["n_docs"]), dtype=torch.float32, device=dev)
        r = fn(ctypes.byref(dd), p["Hq_d"].data_ptr(), p["Wqr_d"].data_ptr(), B, 1, p["KR_d"].data_ptr(),
               p["chunk_off"].data_ptr(), p["n_docs"], p["C"], k, 0, ds.data_ptr(), idx.data_ptr(), sc.data_ptr(),
               stream)
        assert r == 0, msa.lib.msa_last_error().decode()
        torch.cuda.synchronize()
        assert msa.check_device_errors() == 0
        assert torch.equal(idx, ref_idx), f"call {call}: top-k ids differ"
        assert torch.max(torch.abs(sc - ref_sc)).item() <= 1e-3
        assert torch.max(torch.abs(ds - ref_ds)).item() <= 1e-3
        # and both agree with the oracle's document scores
        s = O.doc_scores(O.chunk_scores(O.router_query(p["Hq"], p["Wqr"], 8, 128), p["KR"]), p["co"])
        assert np.max(np.abs(ds.cpu().numpy() - s)) < 1e-3
        results.append(idx.cpu().numpy())
    assert not np.array_equal(results[0][:, :4], results[1][:, :4])  # the second call had other winners


def test_static_scratch_rejects_oversized_problem(cuda_device):
    import long_context_memory_b200 as msa

    fn = _static_fn(msa)
    dd = msa.Dims.of(W.QWEN3_4B_DIMS)
    # 32 queries over 400K documents need far more than the 8 MiB static area
    r = fn(ctypes.byref(dd), 0x10000, 0x10000, 32, 1, 0x10000, 0x10000, 400_000, 1_600_000, 16, 0, None, 0x10000,
           0x10000, None)
    assert r == 3
    assert "static area" in msa.lib.msa_last_error().decode()
    # argument errors are reported as msa_route_topk reports them, before the size check
    r = fn(ctypes.byref(dd), 0x10000, 0x10000, 32, 1, 0x10000, 0x10000, 400_000, 1_600_000, 500, 0, None, 0x10000,
           0x10000, None)
    assert r == 1 and "k must be" in msa.lib.msa_last_error().decode()
