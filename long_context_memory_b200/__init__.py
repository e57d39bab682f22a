"""Memory Sparse Attention (MSA) hot path for NVIDIA B200: Python binding.

A thin ctypes layer over ``libmsa.so`` (C ABI declared in ``include/msa.h``).
It only marshals arguments: every step of the path runs in the library's CUDA
kernels.  PyTorch supplies device memory (outputs and workspaces) and the
current stream.  The library is loaded on the first call into it, and that
call raises ImportError when the library is missing; there is no CPU fallback.

Entry points (same names as the C ABI, minus the ``msa_`` prefix):
  chunk_offsets, encode_memory, append_memory, route_topk, sparse_attend, kv_append, aux_loss,
  gather_kv, tiered_decode, *_workspace_size, check_device_errors, trace_*.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

__all__ = [
    "Dims", "MSAError", "lib", "chunk_offsets", "encode_memory", "append_memory", "route_topk", "sparse_attend",
    "aux_loss", "kv_append", "router_key_norms", "Layer", "tiered_layers", "tiered_workspace_size", "tiered_decode",
    "sparse_attend_share", "attend_merge",
    "route_workspace_size", "attend_workspace_size", "rope_cache_build", "topk_merge", "rope_rows", "gather_kv", "encode_workspace_size", "check_device_errors", "selftest_wait_timeout",
    "trace_enable", "trace_reset", "trace_read", "trace_kernel_names", "AGG_MAX", "AGG_MEAN", "ATTEND_EARLY_LOCAL", "ROUTE_EARLY_INPUTS",
]

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libmsa.so")

AGG_MAX = 0
AGG_MEAN = 1
ATTEND_EARLY_LOCAL = 16  # msa.h MSA_ATTEND_EARLY_LOCAL, OR-ed into the phase argument
ROUTE_EARLY_INPUTS = 16  # msa.h MSA_ROUTE_EARLY_INPUTS, OR-ed into the kr_layout argument

STATUS = {0: "MSA_OK", 1: "MSA_ERR_INVALID_ARG", 2: "MSA_ERR_UNSUPPORTED", 3: "MSA_ERR_WORKSPACE",
          4: "MSA_ERR_CUDA", 5: "MSA_ERR_TIMEOUT"}


class MSAError(RuntimeError):
    def __init__(self, code: int, msg: str):
        super().__init__(f"{STATUS.get(code, code)}: {msg}")
        self.code = code


class Dims(ctypes.Structure):
    """msa_dims: hidden, n_q, n_kv, head_dim, n_r, d_r, chunk, rope_base."""
    _fields_ = [("hidden", ctypes.c_int32), ("n_q", ctypes.c_int32), ("n_kv", ctypes.c_int32),
                ("head_dim", ctypes.c_int32), ("n_r", ctypes.c_int32), ("d_r", ctypes.c_int32),
                ("chunk", ctypes.c_int32), ("rope_base", ctypes.c_float)]

    @classmethod
    def of(cls, d) -> "Dims":
        if isinstance(d, cls):
            return d
        key = (d.hidden, d.n_q, d.n_kv, d.head_dim, d.n_r, d.d_r, d.chunk, float(d.rope_base))
        hit = _DIMS_CACHE.get(key)
        if hit is None:
            hit = _DIMS_CACHE[key] = cls(*key)
        return hit


_DIMS_CACHE: dict = {}  # the ctypes struct of each dims tuple (read-only after construction)

_LAYER_FIELDS = ("Hq", "W_QR", "KR_bar", "kr_inv_norm", "K_bar_host", "V_bar_host", "q", "K_loc", "V_loc", "k_new",
                 "v_new", "topk_idx", "topk_score", "out")


class Layer(ctypes.Structure):
    """msa_layer: the pointers of one layer instance of msa_tiered_decode (NULL for an absent optional)."""
    _fields_ = [(n, ctypes.c_void_p) for n in _LAYER_FIELDS]


def _load():
    if not os.path.exists(LIB_PATH):
        raise ImportError(
            f"libmsa.so not found at {LIB_PATH}; build it with `python -m long_context_memory_b200.build` "
            "(nvcc, sm_100a). There is no CPU fallback.")
    L = ctypes.CDLL(LIB_PATH)
    P, I32, I64, SZ, F = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_size_t, ctypes.c_float
    DP = ctypes.POINTER(Dims)
    sig = {
        "msa_last_error": (ctypes.c_char_p, []),
        "msa_version": (I32, []),
        "msa_check_device_errors": (I32, [ctypes.POINTER(ctypes.c_uint32)]),
        "msa_selftest_wait_timeout": (I32, [I32, I32, P, P]),
        "msa_chunk_offsets": (I32, [P, I32, I32, P, ctypes.POINTER(I32)]),
        "msa_encode_workspace_size": (SZ, [DP, I64, I32, I32]),
        "msa_encode_memory": (I32, [DP, P, I64, P, I32, P, I32, P, P, P, P, P, P, I32, P, SZ, P]),
        "msa_append_memory": (I32, [DP, P, I64, P, I32, P, I32, P, P, P, P, P, P, I32, P, I32, I32, P, SZ, P]),
        "msa_aux_loss_workspace_size": (SZ, [DP, I32, I32]),
        "msa_aux_loss": (I32, [DP, P, P, P, I32, I32, F, P, P, P, P, P, SZ, P]),
        "msa_route_workspace_size": (SZ, [DP, I32, I32, I32, I32, I32, I32]),
        "msa_route_topk": (I32, [DP, P, P, I32, I32, P, P, I32, I32, I32, I32, I32, P, P, P, P, P, SZ, P]),
        "msa_router_key_norms": (I32, [DP, P, I32, I32, P, P]),
        "msa_attend_workspace_size": (SZ, [DP, I32, I32, I32, I32, I32]),
        "msa_sparse_attend": (I32, [DP, P, I32, I32, P, P, P, I32, I32, P, I32, P, P, P, P, P, I32, I32, P, I32, F, I32, P, P,
                                    SZ, P]),
        "msa_rope_rows": (I32, [DP, P, I32, I32, P, P]),
        "msa_kv_append": (I32, [DP, P, P, P, P, I32, I32, P, I32, P]),
        "msa_gather_kv": (I32, [DP, P, P, I32, P, I32, P, I32, I32, P, P, I32, P, P, P, SZ, P]),
        "msa_tiered_workspace_size": (SZ, [DP, I32, I32, I32, I32, I32, I32, I32, I32]),
        "msa_sparse_attend_share": (I32, [DP, P, I32, I32, P, P, P, I32, I32, I32, P, I32, I32, P, P, P, I32, I32, P, I32, F,
                                          P, P, P, SZ, P]),
        "msa_attend_merge": (I32, [P, P, I32, I32, I32, P, P]),
        "msa_tiered_decode": (I32, [DP, ctypes.POINTER(Layer), I32, I32, P, I32, I32, I32, P, I32, I32, I32, P, SZ, P,
                                    P]),
        "msa_rope_cache_size": (SZ, [DP, I32]),
        "msa_rope_cache_build": (I32, [DP, I32, I32, P, SZ, P]),
        "msa_topk_merge": (I32, [P, P, I32, I32, I32, P, P, P]),
        "msa_trace_enable": (I32, [I32]),
        "msa_trace_reset": (I32, []),
        "msa_trace_num_kernels": (I32, []),
        "msa_trace_kernel_name": (ctypes.c_char_p, [I32]),
        "msa_trace_read": (I32, [I32, ctypes.POINTER(ctypes.c_double), ctypes.POINTER(I64)]),
    }
    for name, (res, args) in sig.items():
        fn = getattr(L, name)
        fn.restype = res
        fn.argtypes = args
    return L


class _LazyLib:
    """Loads libmsa.so on first use, so that the seeded generators in
    ``workloads`` import without the compiled library."""

    _cdll = None

    def __getattr__(self, name):
        if _LazyLib._cdll is None:
            _LazyLib._cdll = _load()
        return getattr(_LazyLib._cdll, name)


lib = _LazyLib()


def _check(code: int):
    if code != 0:
        raise MSAError(code, lib.msa_last_error().decode())


def _ptr(t) -> Optional[int]:
    if t is None:
        return None
    return t.data_ptr()


def _stream(stream) -> Optional[int]:
    if stream is not None:
        return stream if isinstance(stream, int) else stream.cuda_stream
    import torch

    raw = getattr(torch._C, "_cuda_getCurrentRawStream", None)  # the current stream's handle, cheaply
    if raw is not None:
        return raw(torch.cuda.current_device())
    return torch.cuda.current_stream().cuda_stream


def _workspace(nbytes: int, device, ws=None):
    import torch

    if nbytes == 0:
        return None
    if ws is not None:
        if ws.numel() * ws.element_size() < nbytes:
            raise MSAError(3, f"workspace of {ws.numel() * ws.element_size()} bytes < {nbytes}")
        return ws
    return torch.empty(nbytes + 256, dtype=torch.uint8, device=device)


def _expect(t, name: str, shape, dtype, device) -> None:
    """Raise ValueError unless t is a contiguous tensor of this shape, dtype and device (the
    library reads it by its sizes alone)."""
    if tuple(t.shape) != tuple(shape) or t.dtype != dtype or t.device != device or not t.is_contiguous():
        raise ValueError(f"{name}: expected a contiguous {dtype} tensor of shape {tuple(shape)} on {device}, got "
                         f"{t.dtype} {tuple(t.shape)} on {t.device}{'' if t.is_contiguous() else ', not contiguous'}")


def _aligned_ptr(ws) -> Optional[int]:
    if ws is None:
        return None
    p = ws.data_ptr()
    return (p + 255) & ~255


# ----------------------------------------------------------------------------
# host helper
# ----------------------------------------------------------------------------
def chunk_offsets(doc_off, chunk: int = 64):
    """chunk_off [n_docs+1] int32 (numpy) and n_chunks from doc_off [n_docs+1] int64 (host)."""
    import numpy as np

    doc_off = np.ascontiguousarray(doc_off, dtype=np.int64)
    n_docs = len(doc_off) - 1
    out = np.zeros(n_docs + 1, dtype=np.int32)
    n = ctypes.c_int32(0)
    _check(lib.msa_chunk_offsets(doc_off.ctypes.data, n_docs, chunk, out.ctypes.data, ctypes.byref(n)))
    return out, int(n.value)


# ----------------------------------------------------------------------------
# stage 1
# ----------------------------------------------------------------------------
def encode_workspace_size(dims, T: int, n_docs: int, n_chunks: int) -> int:
    return int(lib.msa_encode_workspace_size(ctypes.byref(Dims.of(dims)), T, n_docs, n_chunks))


def encode_memory(dims, H, doc_off, chunk_off, n_chunks: int, W_K, W_V, W_KR, out=None, ws=None, stream=None,
                  kr_head_major: bool = False):
    """Pooled (K̄, V̄, K̄^R) of a corpus; all tensors on the same CUDA device.

    ``kr_head_major`` stores K̄^R as [n_r, C, d_r] (the layout the scan reads best)."""
    import torch

    dd = Dims.of(dims)
    T, n_docs = H.shape[0], doc_off.numel() - 1
    dev = H.device
    if out is None:
        kr_shape = (dims.n_r, n_chunks, dims.d_r) if kr_head_major else (n_chunks, dims.n_r, dims.d_r)
        out = (torch.empty((n_chunks, dims.n_kv, dims.head_dim), dtype=torch.bfloat16, device=dev),
               torch.empty((n_chunks, dims.n_kv, dims.head_dim), dtype=torch.bfloat16, device=dev),
               torch.empty(kr_shape, dtype=torch.bfloat16, device=dev))
    nbytes = encode_workspace_size(dims, T, n_docs, n_chunks)
    ws = _workspace(nbytes, dev, ws)
    _check(lib.msa_encode_memory(ctypes.byref(dd), _ptr(H), T, _ptr(doc_off), n_docs, _ptr(chunk_off), n_chunks,
                                 _ptr(W_K), _ptr(W_V), _ptr(W_KR), _ptr(out[0]), _ptr(out[1]), _ptr(out[2]),
                                 int(bool(kr_head_major)), _aligned_ptr(ws), nbytes, _stream(stream)))
    return out


def append_memory(dims, H_new, doc_off_new, chunk_off_new, n_chunks_new: int, W_K, W_V, W_KR, memory, chunk_off,
                  n_docs_old: int, n_chunks_old: int, ws=None, stream=None):
    """Encode new documents behind an existing chunk-major memory, in place.

    ``memory`` = (K_bar, V_bar, KR_bar) with room for the new chunks (first dimension = the
    capacity in chunks); ``chunk_off`` (device int32, room for every document + 1) gets the new
    documents' offsets.  Returns (n_docs_old + n_docs_new, n_chunks_old + n_chunks_new).
    """
    K_bar, V_bar, KR_bar = memory
    T = H_new.shape[0]
    n_new = doc_off_new.numel() - 1
    nbytes = encode_workspace_size(dims, T, n_new, n_chunks_new)
    ws = _workspace(nbytes, H_new.device, ws)
    _check(lib.msa_append_memory(ctypes.byref(Dims.of(dims)), _ptr(H_new), T, _ptr(doc_off_new), n_new,
                                 _ptr(chunk_off_new), n_chunks_new, _ptr(W_K), _ptr(W_V), _ptr(W_KR), _ptr(K_bar),
                                 _ptr(V_bar), _ptr(KR_bar), K_bar.shape[0], _ptr(chunk_off), n_docs_old,
                                 n_chunks_old, _aligned_ptr(ws), nbytes, _stream(stream)))
    return n_docs_old + n_new, n_chunks_old + n_chunks_new


# ----------------------------------------------------------------------------
# stage 2
# ----------------------------------------------------------------------------
def route_workspace_size(dims, B: int, n_docs: int, n_chunks: int, k: int, agg: int = AGG_MAX,
                         q_tokens: int = 1) -> int:
    return int(lib.msa_route_workspace_size(ctypes.byref(Dims.of(dims)), B, q_tokens, n_docs, n_chunks, k, agg))


def route_topk(dims, Hq, W_QR, KR_bar, chunk_off, k: int, agg: int = AGG_MAX, want_doc_scores: bool = False,
               out=None, ws=None, stream=None, kr_head_major: bool = False, q_tokens: int = 1, kr_inv_norm=None,
               early_inputs: bool = False):
    """Top-k documents per query.  Returns (topk_idx [B,k] int32, topk_score [B,k] fp32, doc_scores|None).

    ``Hq`` holds B * q_tokens rows (token t of query b at row b * q_tokens + t); a chunk's
    score for a query is the largest over its tokens.
    ``W_QR=None`` means ``Hq`` already holds the router queries Q^R [B * q_tokens, n_r*d_r].
    ``kr_head_major``: KR_bar is [n_r, C, d_r] instead of [C, n_r, d_r].
    ``kr_inv_norm``: the keys' inverse norms from ``router_key_norms`` (computed once per memory).
    ``early_inputs`` (MSA_ROUTE_EARLY_INPUTS): ``Hq``, ``W_QR``, ``KR_bar``, ``kr_inv_norm`` and
    ``chunk_off`` were final before the preceding work on the stream was enqueued, so the routing
    may read them before that work finishes.
    """
    import torch

    dd = Dims.of(dims)
    if Hq.shape[0] % q_tokens:
        raise ValueError(f"Hq has {Hq.shape[0]} rows, not a multiple of q_tokens={q_tokens}")
    B = Hq.shape[0] // q_tokens
    n_docs = chunk_off.numel() - 1
    n_chunks = KR_bar.shape[1] if kr_head_major else KR_bar.shape[0]
    dev = KR_bar.device
    if out is None:
        out = (torch.empty((B, k), dtype=torch.int32, device=dev), torch.empty((B, k), dtype=torch.float32, device=dev),
               torch.empty((B, n_docs), dtype=torch.float32, device=dev) if want_doc_scores else None)
    if ws is not None:  # the library checks the caller's buffer against what it needs
        nbytes = max(0, ws.numel() * ws.element_size() - 256)
    else:
        nbytes = route_workspace_size(dims, B, n_docs, n_chunks, k, agg, q_tokens)
        ws = _workspace(nbytes, dev, ws)
    _check(lib.msa_route_topk(ctypes.byref(dd), _ptr(Hq), _ptr(W_QR), B, q_tokens, _ptr(KR_bar), _ptr(chunk_off), n_docs,
                              n_chunks, k, agg, int(bool(kr_head_major)) | (ROUTE_EARLY_INPUTS if early_inputs else 0),
                              _ptr(kr_inv_norm), _ptr(out[2]), _ptr(out[0]), _ptr(out[1]), _aligned_ptr(ws), nbytes,
                              _stream(stream)))
    return out


def router_key_norms(dims, KR_bar, kr_head_major: bool = False, out=None, stream=None):
    """[n_chunks, n_r] fp32 inverse norms of the pooled router keys (offline, once per memory)."""
    import torch

    n_chunks = KR_bar.shape[1] if kr_head_major else KR_bar.shape[0]
    if out is None:
        out = torch.empty((n_chunks, dims.n_r), dtype=torch.float32, device=KR_bar.device)
    _check(lib.msa_router_key_norms(ctypes.byref(Dims.of(dims)), _ptr(KR_bar), n_chunks, int(bool(kr_head_major)),
                                    _ptr(out), _stream(stream)))
    return out


def topk_merge(cand_score, cand_idx, k: int, out=None, stream=None):
    """Global top-k of [B, n_cand] (score, global id) candidates (memory-parallel routing)."""
    import torch

    B, n = cand_score.shape
    dev = cand_score.device
    if out is None:
        out = (torch.empty((B, k), dtype=torch.int32, device=dev), torch.empty((B, k), dtype=torch.float32, device=dev))
    _check(lib.msa_topk_merge(_ptr(cand_score), _ptr(cand_idx), B, n, k, _ptr(out[0]), _ptr(out[1]), _stream(stream)))
    return out


# ----------------------------------------------------------------------------
# stage 3
# ----------------------------------------------------------------------------
def attend_workspace_size(dims, B: int, k: int, t_loc_max: int, pos_offset: int, q_tokens: int = 1) -> int:
    return int(lib.msa_attend_workspace_size(ctypes.byref(Dims.of(dims)), B, q_tokens, k, t_loc_max, pos_offset))


def rope_cache_build(dims, t_loc_max: int, pos_offset: int, device=None, out=None, stream=None):
    """(cos, sin) table of the local positions pos_offset + j, j < t_loc_max (fp32 pairs)."""
    import torch

    nbytes = int(lib.msa_rope_cache_size(ctypes.byref(Dims.of(dims)), t_loc_max))
    if out is None:
        out = torch.empty(nbytes // 4, dtype=torch.float32, device=device)
    _check(lib.msa_rope_cache_build(ctypes.byref(Dims.of(dims)), t_loc_max, pos_offset, _ptr(out),
                                    out.numel() * out.element_size(), _stream(stream)))
    return out


def gather_kv(dims, K_bar_host, V_bar_host, chunk_off, topk_idx, capacity_chunks: int, out=None, stream=None):
    """Stage the selected documents' pooled K̄/V̄ from pinned host memory onto the device.

    Returns (K_stage, V_stage, stage_chunk_off [B*k+1], stage_topk_idx [B, k]) for sparse_attend.
    """
    import torch

    B, k = topk_idx.shape
    dev = topk_idx.device
    n_docs = chunk_off.numel() - 1
    if out is None:
        shape = (capacity_chunks, dims.n_kv, dims.head_dim)
        out = (torch.empty(shape, dtype=torch.bfloat16, device=dev), torch.empty(shape, dtype=torch.bfloat16, device=dev),
               torch.empty(B * k + 1, dtype=torch.int32, device=dev), torch.empty((B, k), dtype=torch.int32, device=dev))
    ws = torch.empty(B * k * 4 + 256, dtype=torch.uint8, device=dev)
    _check(lib.msa_gather_kv(ctypes.byref(Dims.of(dims)), _ptr(K_bar_host), _ptr(V_bar_host), K_bar_host.shape[0],
                             _ptr(chunk_off), n_docs, _ptr(topk_idx), B, k, _ptr(out[0]), _ptr(out[1]),
                             capacity_chunks, _ptr(out[2]), _ptr(out[3]), _aligned_ptr(ws), B * k * 4,
                             _stream(stream)))
    return out


def tiered_layers(layers):
    """A ctypes array of msa_layer from a list of dicts {field: tensor or None} (fields of ``Layer``).

    Build it once per set of buffers and pass it to every ``tiered_decode`` call: the call then
    marshals nothing per layer."""
    arr = (Layer * len(layers))()
    for i, L in enumerate(layers):
        for f in _LAYER_FIELDS:
            t = L.get(f)
            setattr(arr[i], f, None if t is None else t.data_ptr())
    return arr


def tiered_workspace_size(dims, n_layers: int, B: int, n_docs: int, n_chunks: int, k: int, t_loc_max: int,
                          pos_offset: int, capacity_chunks: int) -> int:
    return int(lib.msa_tiered_workspace_size(ctypes.byref(Dims.of(dims)), n_layers, B, n_docs, n_chunks, k, t_loc_max,
                                             pos_offset, capacity_chunks))


def tiered_decode(dims, layers, B: int, chunk_off, n_chunks: int, k: int, loc_len, t_loc_max: int, pos_offset: int,
                  capacity_chunks: int, ws=None, stream=None, copy_stream=None):
    """Route, gather (host tier) and attend for several independent layer instances in one call.

    ``layers``: the array from ``tiered_layers`` (or a list of dicts, converted here).  Per layer the
    routing, the gather of the routed documents from pinned host memory and the attention over the
    staged documents and the rotated local cache are split between ``stream`` (default: the current
    stream) and ``copy_stream`` (None: everything on ``stream``, no overlap) as msa_tiered_decode
    describes; outputs land in each layer's topk_idx, topk_score and out tensors, ordered before
    later work on ``stream``."""
    arr = layers if isinstance(layers, ctypes.Array) else tiered_layers(layers)
    n_docs = chunk_off.numel() - 1
    dd = Dims.of(dims)
    if ws is not None:  # the library checks the caller's buffer against what it needs
        nbytes = max(0, ws.numel() * ws.element_size() - 256)
    else:
        nbytes = tiered_workspace_size(dims, len(arr), B, n_docs, n_chunks, k, t_loc_max, pos_offset, capacity_chunks)
        ws = _workspace(nbytes, chunk_off.device, ws)
    _check(lib.msa_tiered_decode(ctypes.byref(dd), arr, len(arr), B, _ptr(chunk_off), n_docs, n_chunks, k, _ptr(loc_len),
                                 t_loc_max, pos_offset, capacity_chunks, _aligned_ptr(ws), nbytes, _stream(stream),
                                 None if copy_stream is None else _stream(copy_stream)))


def rope_rows(dims, x, positions, stream=None):
    """Rotate x [rows, heads, head_dim] (bf16, in place) at positions [rows] (int32, device)."""
    rows, heads = x.shape[0], x.shape[1]
    _check(lib.msa_rope_rows(ctypes.byref(Dims.of(dims)), _ptr(x), rows, heads, _ptr(positions), _stream(stream)))
    return x


def kv_append(dims, k_new, v_new, K_loc, V_loc, slots, pos_offset: int, stream=None):
    """Write the new token of every query into the rotated local cache, in place.

    k_new, v_new [B, n_kv, head_dim]; K_loc, V_loc [B, t_loc_max, n_kv, head_dim]; slots [B] int32
    (device): K_loc[b, slots[b]] = RoPE(k_new[b], pos_offset + slots[b]), V_loc[b, slots[b]] = v_new[b].
    """
    import torch

    B, t_loc_max = K_loc.shape[0], K_loc.shape[1]
    dd = Dims.of(dims)
    for name, t in (("k_new", k_new), ("v_new", v_new)):
        _expect(t, name, (B, dd.n_kv, dd.head_dim), torch.bfloat16, K_loc.device)
    _expect(slots, "slots", (B,), torch.int32, K_loc.device)
    _check(lib.msa_kv_append(ctypes.byref(Dims.of(dims)), _ptr(k_new), _ptr(v_new), _ptr(K_loc), _ptr(V_loc), B,
                             t_loc_max, _ptr(slots), pos_offset, _stream(stream)))


def sparse_attend(dims, q, K_bar, V_bar, chunk_off, topk_idx, K_loc, V_loc, loc_len, pos_offset: int,
                  softmax_scale: float = 0.0, out=None, ws=None, stream=None, rope_cache=None,
                  k_loc_rotated: bool = False, phase: int = 0, early_local: bool = False, k_new=None, v_new=None):
    """GQA attention of the query tokens over [selected docs' K̄; local K].

    ``q`` is [B, n_q, head_dim] (one decode token) or [B, M, n_q, head_dim] (the last M local
    tokens, causal among the local keys); ``out`` has the shape of ``q``.
    ``rope_cache`` (from ``rope_cache_build`` with the same pos_offset and t_loc_max) skips
    rebuilding the local-position rotation table.  ``phase`` 1 / 2 splits the call into the
    local-keys part and the selected-chunks part (which merges both); pass the same ``ws``.
    ``early_local`` (MSA_ATTEND_EARLY_LOCAL) lets the local-key work start before the
    preceding library call's kernels finish; q, K_loc, V_loc and loc_len must have been final
    before that call was enqueued, and it must not be a sparse_attend on the same ``ws``.
    ``k_new``/``v_new`` [B, n_kv, head_dim] (decode, M = 1): the new token's key (before RoPE) and
    value are first written at slot loc_len - 1 of K_loc/V_loc (the key rotated when
    ``k_loc_rotated``), as ``kv_append`` would, and the call attends over the cache as written."""
    import torch

    dd = Dims.of(dims)
    B, k = topk_idx.shape
    M = q.shape[1] if q.dim() == 4 else 1
    for name, t in (("k_new", k_new), ("v_new", v_new)):  # one row per query, written into the cache
        if t is not None:
            _expect(t, name, (B, dd.n_kv, dd.head_dim), torch.bfloat16, q.device)
    t_loc_max = K_loc.shape[1] if K_loc is not None else 0
    n_docs = chunk_off.numel() - 1
    dev = q.device
    if out is None:
        out = torch.empty(tuple(q.shape), dtype=torch.bfloat16, device=dev)
    if ws is not None:  # the library checks the caller's buffer against what it needs
        nbytes = max(0, ws.numel() * ws.element_size() - 256)
    else:
        nbytes = attend_workspace_size(dims, B, k, t_loc_max, pos_offset, M)
        ws = _workspace(nbytes, dev, ws)
    _check(lib.msa_sparse_attend(ctypes.byref(dd), _ptr(q), B, M, _ptr(K_bar), _ptr(V_bar), _ptr(chunk_off), n_docs,
                                 K_bar.shape[0], _ptr(topk_idx), k, _ptr(K_loc), _ptr(V_loc), _ptr(k_new), _ptr(v_new),
                                 _ptr(loc_len),
                                 t_loc_max, pos_offset, _ptr(rope_cache), int(bool(k_loc_rotated)),
                                 float(softmax_scale), int(phase) | (ATTEND_EARLY_LOCAL if early_local else 0),
                                 _ptr(out),
                                 _aligned_ptr(ws), nbytes, _stream(stream)))
    return out


def sparse_attend_share(dims, q, K_bar, V_bar, chunk_off, doc_base: int, topk_idx, local_keys: bool, K_loc, V_loc,
                        loc_len, t_loc_max: int, pos_offset: int, softmax_scale: float = 0.0, rope_cache=None,
                        k_loc_rotated: bool = False, out=None, ws=None, stream=None):
    """One rank's share of a memory-parallel attention (see msa_sparse_attend_share).

    ``K_bar``/``V_bar``/``chunk_off`` hold the shard's documents doc_base .. (chunk offsets rebased);
    ``topk_idx`` [B, k] holds GLOBAL ids (others are skipped); the local keys count only where
    ``local_keys``.  Returns (o [q.shape] fp32, lse2 [q.shape[:-1]] fp32)."""
    import torch

    dd = Dims.of(dims)
    B, k = topk_idx.shape
    M = q.shape[1] if q.dim() == 4 else 1
    dev = q.device
    n_docs = chunk_off.numel() - 1
    if out is None:
        out = (torch.empty(tuple(q.shape), dtype=torch.float32, device=dev),
               torch.empty(tuple(q.shape[:-1]), dtype=torch.float32, device=dev))
    if ws is not None:
        nbytes = max(0, ws.numel() * ws.element_size() - 256)
    else:
        nbytes = attend_workspace_size(dims, B, k, t_loc_max, pos_offset, M)
        ws = _workspace(nbytes, dev, ws)
    _check(lib.msa_sparse_attend_share(ctypes.byref(dd), _ptr(q), B, M, _ptr(K_bar), _ptr(V_bar), _ptr(chunk_off), n_docs,
                                       K_bar.shape[0], int(doc_base), _ptr(topk_idx), k, int(bool(local_keys)),
                                       _ptr(K_loc) if local_keys else None, _ptr(V_loc) if local_keys else None,
                                       _ptr(loc_len), t_loc_max, pos_offset, _ptr(rope_cache), int(bool(k_loc_rotated)),
                                       float(softmax_scale), _ptr(out[0]), _ptr(out[1]), _aligned_ptr(ws), nbytes,
                                       _stream(stream)))
    return out


def attend_merge(o_shares, lse2_shares, out=None, stream=None):
    """Merge R shares: o_shares [R, ..., head_dim] fp32, lse2_shares [R, ...] fp32 -> bf16 [..., head_dim]."""
    import torch

    R, D = o_shares.shape[0], o_shares.shape[-1]
    rows = lse2_shares[0].numel()
    if out is None:
        out = torch.empty(tuple(o_shares.shape[1:]), dtype=torch.bfloat16, device=o_shares.device)
    _check(lib.msa_attend_merge(_ptr(o_shares), _ptr(lse2_shares), R, rows, D, _ptr(out), _stream(stream)))
    return out


# ----------------------------------------------------------------------------
# router training
# ----------------------------------------------------------------------------
def aux_loss(dims, QR, K_pos, K_neg, tau: float, grads: bool = True, out=None, ws=None, stream=None):
    """Contrastive routing loss L_aux and (optionally) its gradients.

    QR, K_pos [P, n_r, d_r] bf16; K_neg [P, N, n_r, d_r] bf16 (N may be 0).  Returns
    (loss [1] fp32, dQR, dK_pos, dK_neg) with fp32 gradients, or None for each when grads=False.
    """
    import torch

    P = QR.shape[0]
    N = K_neg.shape[1] if K_neg is not None else 0
    dev = QR.device
    if out is None:
        out = (torch.empty(1, dtype=torch.float32, device=dev),
               torch.empty(tuple(QR.shape), dtype=torch.float32, device=dev) if grads else None,
               torch.empty(tuple(K_pos.shape), dtype=torch.float32, device=dev) if grads else None,
               torch.empty(tuple(K_neg.shape), dtype=torch.float32, device=dev) if grads and N > 0 else None)
    nbytes = int(lib.msa_aux_loss_workspace_size(ctypes.byref(Dims.of(dims)), P, N))
    ws = _workspace(nbytes, dev, ws)
    _check(lib.msa_aux_loss(ctypes.byref(Dims.of(dims)), _ptr(QR), _ptr(K_pos), _ptr(K_neg) if N > 0 else None, P, N,
                            float(tau), _ptr(out[0]), _ptr(out[1]), _ptr(out[2]), _ptr(out[3]), _aligned_ptr(ws),
                            nbytes, _stream(stream)))
    return out


# ----------------------------------------------------------------------------
# diagnostics
# ----------------------------------------------------------------------------
def check_device_errors() -> int:
    bits = ctypes.c_uint32(0)
    _check(lib.msa_check_device_errors(ctypes.byref(bits)))
    return int(bits.value)


def selftest_wait_timeout(limit_us: int, n_waits: int, stream=None):
    """Run the bounded-wait self-test kernel (see msa.h); returns the device uint64 [1] that receives
    its wall time in ns.  Afterwards check_device_errors() raises MSAError with MSA_ERR_TIMEOUT."""
    import torch

    out = torch.zeros(2, dtype=torch.int64, device=torch.cuda.current_device())
    _check(lib.msa_selftest_wait_timeout(int(limit_us), int(n_waits), _ptr(out), _stream(stream)))
    return out[:1]


def trace_enable(on: bool = True):
    _check(lib.msa_trace_enable(1 if on else 0))


def trace_reset():
    _check(lib.msa_trace_reset())


def trace_kernel_names():
    return [lib.msa_trace_kernel_name(i).decode() for i in range(lib.msa_trace_num_kernels())]


def trace_read() -> dict:
    """{kernel name: (total ms, launches)} since the last reset (synchronises on the trace events)."""
    out = {}
    for i, name in enumerate(trace_kernel_names()):
        ms, n = ctypes.c_double(0), ctypes.c_int64(0)
        _check(lib.msa_trace_read(i, ctypes.byref(ms), ctypes.byref(n)))
        out[name] = (ms.value, n.value)
    return out
