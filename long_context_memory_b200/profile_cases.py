"""Run one stage of the MSA path on one synthetic workload, for timing and profiling.

    python -m long_context_memory_b200.profile_cases --case route16m --launches 3

Inputs are drawn on the device by torch's seeded generator (timing only: no
parity check here; the tests do that).  Each launch is timed with CUDA events
on the launching stream and printed; under a profiler, the printed times are
not benchmark values.

Cases
  route1m    1M-token memory, B = 1   (K̄^R 33 MB)
  route16m   16M-token memory, B = 32 (K̄^R 520 MB)
  route100m  100M-token memory, B = 1 (K̄^R 3.2 GB); --batch to change B, --tokens the size
             (route cases: --kr-layout head stores K̄^R head-major [n_r, C, d_r])
  attend1m   sparse attention, 1M-token memory, B = 1, 4K local tokens (rotated key cache)
  attend16m  sparse attention, 16M-token memory, B = 32, 8K local tokens (rotated key cache)
  tiered     one msa_tiered_decode call over --layers layer instances (default 2) of a
             --tokens-token memory (default 100M): routing, host-tier gather, attention; B = --batch
  encode     offline encoding of --tokens tokens (default 1M), hidden 2560
  aux        router training loss L_aux + gradients: P = 4096 positives x (1 + 63 negatives),
             8 router heads x 128 (--batch to change P)
"""
from __future__ import annotations

import argparse
import math

import numpy as np

from . import workloads as W


def chunk_layout_host(T: int, median: int, seed: int):
    import long_context_memory_b200 as msa

    rng = np.random.default_rng(seed)
    lens = W.doc_lengths_lognormal(rng, T, median)
    doc_off = W.offsets_from_lengths(lens)
    co, C = msa.chunk_offsets(doc_off)
    return doc_off, co, C


def randn_bf16(shape, g, device):
    import torch

    out = torch.empty(shape, dtype=torch.bfloat16, device=device)
    flat = out.view(-1)
    step = 1 << 26
    for i in range(0, flat.numel(), step):
        e = min(flat.numel(), i + step)
        flat[i:e] = torch.randn(e - i, generator=g, device=device, dtype=torch.float32).to(torch.bfloat16)
    return out


class RouteCase:
    def __init__(self, T, B, median, seed, device, k=16, dims=W.QWEN3_4B_DIMS, layers=1, head_major=False,
                 norms=False):
        import torch

        import long_context_memory_b200 as msa

        self.msa, self.d, self.B, self.k, self.T = msa, dims, B, k, T
        doc_off, co, C = chunk_layout_host(T, median, seed)
        self.C, self.n_docs = C, len(co) - 1
        g = torch.Generator(device=device)
        g.manual_seed(seed)
        self.chunk_off = torch.from_numpy(co).to(device)
        self.head_major = head_major
        kr_shape = (dims.n_r, C, dims.d_r) if head_major else (C, dims.n_r, dims.d_r)
        self.KR = [randn_bf16(kr_shape, g, device) for _ in range(layers)]
        # inverse key norms computed once per memory (offline), as a deployment would keep them
        self.inv = [msa.router_key_norms(dims, kr, kr_head_major=head_major) for kr in self.KR] if norms else None
        self.Hq = randn_bf16((B, dims.hidden), g, device)
        self.W_QR = (torch.randn((dims.hidden, dims.n_r * dims.d_r), generator=g, device=device) /
                     math.sqrt(dims.hidden)).to(torch.bfloat16)
        self.idx = torch.empty((B, k), dtype=torch.int32, device=device)
        self.sc = torch.empty((B, k), dtype=torch.float32, device=device)
        self.ws = torch.empty(msa.route_workspace_size(dims, B, self.n_docs, C, k) + 256, dtype=torch.uint8,
                              device=device)

    def set_batch(self, B, seed=0):
        """Same memory, a new batch of B queries."""
        import torch

        dev = self.KR[0].device
        g = torch.Generator(device=dev)
        g.manual_seed(seed)
        self.B = B
        self.Hq = randn_bf16((B, self.d.hidden), g, dev)
        self.idx = torch.empty((B, self.k), dtype=torch.int32, device=dev)
        self.sc = torch.empty((B, self.k), dtype=torch.float32, device=dev)
        self.ws = torch.empty(self.msa.route_workspace_size(self.d, B, self.n_docs, self.C, self.k) + 256,
                              dtype=torch.uint8, device=dev)

    def run(self, layer=0):
        self.msa.route_topk(self.d, self.Hq, self.W_QR, self.KR[layer], self.chunk_off, self.k,
                            out=(self.idx, self.sc, None), ws=self.ws, kr_head_major=self.head_major,
                            kr_inv_norm=self.inv[layer] if self.inv else None)

    @property
    def scan_bytes(self):
        """Algorithmic bytes of one scan: the pooled router keys (and their inverse norms when given)."""
        return self.C * self.d.n_r * (self.d.d_r * 2 + (4 if self.inv else 0))


class AttendCase:
    def __init__(self, T, B, median, t_loc, seed, device, k=16, dims=W.QWEN3_4B_DIMS, rotated=True):
        import torch

        import long_context_memory_b200 as msa

        self.msa, self.d, self.B, self.k = msa, dims, B, k
        doc_off, co, C = chunk_layout_host(T, median, seed)
        n_docs = len(co) - 1
        g = torch.Generator(device=device)
        g.manual_seed(seed + 1)
        self.chunk_off = torch.from_numpy(co).to(device)
        self.K_bar = randn_bf16((C, dims.n_kv, dims.head_dim), g, device)
        self.V_bar = randn_bf16((C, dims.n_kv, dims.head_dim), g, device)
        self.q = randn_bf16((B, dims.n_q, dims.head_dim), g, device)
        self.K_loc = randn_bf16((B, t_loc, dims.n_kv, dims.head_dim), g, device)
        self.V_loc = randn_bf16((B, t_loc, dims.n_kv, dims.head_dim), g, device)
        self.loc_len = torch.full((B,), t_loc, dtype=torch.int32, device=device)
        rng = np.random.default_rng(seed)
        sel = np.stack([rng.permutation(n_docs)[:k] for _ in range(B)]).astype(np.int32)
        self.topk = torch.from_numpy(sel).to(device)
        self.pos = k
        self.rotated = rotated
        if rotated:  # the local key cache holds keys rotated at their global positions
            msa.rope_rows(dims, self.K_loc.view(B * t_loc, dims.n_kv, dims.head_dim),
                          (self.pos + torch.arange(t_loc, dtype=torch.int32, device=device)).repeat(B))
            self.rope = None
        else:
            self.rope = msa.rope_cache_build(dims, t_loc, self.pos, device=device)
        self.out = torch.empty((B, dims.n_q, dims.head_dim), dtype=torch.bfloat16, device=device)
        self.ws = torch.empty(msa.attend_workspace_size(dims, B, k, t_loc, self.pos) + 256, dtype=torch.uint8,
                              device=device)
        n_sel = sum(int(co[i + 1] - co[i]) for row in sel for i in row)
        self.kv_bytes = (n_sel + B * t_loc) * dims.n_kv * dims.head_dim * 2 * 2

    def run(self):
        self.msa.sparse_attend(self.d, self.q, self.K_bar, self.V_bar, self.chunk_off, self.topk, self.K_loc,
                               self.V_loc, self.loc_len, self.pos, out=self.out, ws=self.ws, rope_cache=self.rope,
                               k_loc_rotated=self.rotated)


class HostTierCase:
    """The host tier of a large memory: pooled K̄/V̄ in pinned host memory; per step the selected
    documents of every query cross the host link (msa_gather_kv) into a device staging area, then
    the attention runs over them and the local KV (rotated cache)."""

    def __init__(self, T, B, median, t_loc, seed, device, k=16, dims=W.QWEN3_4B_DIMS):
        import torch

        import long_context_memory_b200 as msa

        self.msa, self.d, self.B, self.k = msa, dims, B, k
        doc_off, co, C = chunk_layout_host(T, median, seed)
        n_docs = len(co) - 1
        g = torch.Generator(device=device)
        g.manual_seed(seed + 1)
        shape = (C, dims.n_kv, dims.head_dim)
        self.K_host = torch.empty(shape, dtype=torch.bfloat16, pin_memory=True)
        self.V_host = torch.empty(shape, dtype=torch.bfloat16, pin_memory=True)
        step = 1 << 16  # rows per device-generated slab
        for dst in (self.K_host, self.V_host):
            for a in range(0, C, step):
                e = min(C, a + step)
                dst[a:e].copy_(randn_bf16((e - a,) + shape[1:], g, device))
        torch.cuda.synchronize()
        self.chunk_off = torch.from_numpy(co).to(device)
        rng = np.random.default_rng(seed)
        sel = np.stack([rng.permutation(n_docs)[:k] for _ in range(B)]).astype(np.int32)
        self.topk = torch.from_numpy(sel).to(device)
        self.n_sel = sum(int(co[i + 1] - co[i]) for row in sel for i in row)
        self.capacity = self.n_sel
        self.stage = (torch.empty((self.capacity,) + shape[1:], dtype=torch.bfloat16, device=device),
                      torch.empty((self.capacity,) + shape[1:], dtype=torch.bfloat16, device=device),
                      torch.empty(B * k + 1, dtype=torch.int32, device=device),
                      torch.empty((B, k), dtype=torch.int32, device=device))
        self.gather_bytes = self.n_sel * dims.n_kv * dims.head_dim * 2 * 2
        self.q = randn_bf16((B, dims.n_q, dims.head_dim), g, device)
        self.K_loc = randn_bf16((B, t_loc, dims.n_kv, dims.head_dim), g, device)
        self.V_loc = randn_bf16((B, t_loc, dims.n_kv, dims.head_dim), g, device)
        self.loc_len = torch.full((B,), t_loc, dtype=torch.int32, device=device)
        self.pos = k
        msa.rope_rows(dims, self.K_loc.view(B * t_loc, dims.n_kv, dims.head_dim),
                      (self.pos + torch.arange(t_loc, dtype=torch.int32, device=device)).repeat(B))
        self.out = torch.empty((B, dims.n_q, dims.head_dim), dtype=torch.bfloat16, device=device)
        self.ws = torch.empty(msa.attend_workspace_size(dims, B, k, t_loc, self.pos) + 256, dtype=torch.uint8,
                              device=device)
        self.kv_bytes = (self.n_sel + B * t_loc) * dims.n_kv * dims.head_dim * 2 * 2

    def gather(self):
        self.msa.gather_kv(self.d, self.K_host, self.V_host, self.chunk_off, self.topk, self.capacity, out=self.stage)

    def attend(self):
        K_s, V_s, off_s, idx_s = self.stage
        self.msa.sparse_attend(self.d, self.q, K_s, V_s, off_s, idx_s, self.K_loc, self.V_loc, self.loc_len, self.pos,
                               out=self.out, ws=self.ws, k_loc_rotated=True)


class TieredCase:
    """A memory of T tokens served from two tiers, over ``layers`` independent layer instances.

    Per layer: pooled router keys K̄^R [C, n_r, d_r] (and their inverse norms) resident in HBM,
    W^QR, the query's hidden state, q, an 8K-token rotated local KV cache and the new token's key
    and value per query; content K̄/V̄ [C, n_kv, head_dim] in pinned host memory (``host_layers``
    distinct host instances, layer l reading instance l % host_layers).  ``run`` makes one
    msa_tiered_decode call: route every layer, gather its routed documents over the host link on
    the copy stream, attend over them and the local cache."""

    def __init__(self, T, median, t_loc, seed, device, layers, host_layers, B=1, k=16, dims=W.QWEN3_4B_DIMS):
        import torch

        import long_context_memory_b200 as msa

        self.msa, self.d, self.k, self.T, self.t_loc = msa, dims, k, T, t_loc
        self.dev = device
        doc_off, co, C = chunk_layout_host(T, median, seed)
        self.C, self.n_docs = C, len(co) - 1
        self.co_np = co
        self.max_doc_chunks = int(np.max(co[1:] - co[:-1]))
        self.chunk_off = torch.from_numpy(co).to(device)
        g = torch.Generator(device=device)
        g.manual_seed(seed)
        self.n_layers = layers
        self.KR = [randn_bf16((C, dims.n_r, dims.d_r), g, device) for _ in range(layers)]
        # inverse key norms computed once per memory (offline), as a deployment keeps them
        self.inv = [msa.router_key_norms(dims, kr) for kr in self.KR]
        self.W_QR = [(torch.randn((dims.hidden, dims.n_r * dims.d_r), generator=g, device=device) /
                      math.sqrt(dims.hidden)).to(torch.bfloat16) for _ in range(layers)]
        shape = (C, dims.n_kv, dims.head_dim)
        self.K_host, self.V_host = [], []
        step = 1 << 16  # rows per device-generated slab
        for _ in range(host_layers):
            pair = []
            for _t in range(2):
                dst = torch.empty(shape, dtype=torch.bfloat16, pin_memory=True)
                for a in range(0, C, step):
                    e = min(C, a + step)
                    dst[a:e].copy_(randn_bf16((e - a,) + shape[1:], g, device))
                pair.append(dst)
            self.K_host.append(pair[0])
            self.V_host.append(pair[1])
        torch.cuda.synchronize()
        self.host_layers = host_layers
        self.B = 0
        self.set_batch(B, seed + 100)

    def set_batch(self, B, seed):
        """A new batch of B queries per layer (query states, local caches, outputs, workspace)."""
        import torch

        msa, d, dev, L = self.msa, self.d, self.dev, self.n_layers
        self.B = B
        self.q_state = None
        torch.cuda.empty_cache()
        g = torch.Generator(device=dev)
        g.manual_seed(seed)
        self.pos = self.k
        self.loc_len = torch.full((B,), self.t_loc, dtype=torch.int32, device=dev)
        self.per_layer = []
        pos = (self.pos + torch.arange(self.t_loc, dtype=torch.int32, device=dev)).repeat(B)
        for l in range(L):
            x = dict(Hq=randn_bf16((B, d.hidden), g, dev), q=randn_bf16((B, d.n_q, d.head_dim), g, dev),
                     K_loc=randn_bf16((B, self.t_loc, d.n_kv, d.head_dim), g, dev),
                     V_loc=randn_bf16((B, self.t_loc, d.n_kv, d.head_dim), g, dev),
                     k_new=randn_bf16((B, d.n_kv, d.head_dim), g, dev),
                     v_new=randn_bf16((B, d.n_kv, d.head_dim), g, dev),
                     topk_idx=torch.empty((B, self.k), dtype=torch.int32, device=dev),
                     topk_score=torch.empty((B, self.k), dtype=torch.float32, device=dev),
                     out=torch.empty((B, d.n_q, d.head_dim), dtype=torch.bfloat16, device=dev),
                     W_QR=self.W_QR[l], KR_bar=self.KR[l], kr_inv_norm=self.inv[l],
                     K_bar_host=self.K_host[l % self.host_layers], V_bar_host=self.V_host[l % self.host_layers])
            # the local cache holds keys rotated at their global positions (rotated once, when appended)
            msa.rope_rows(d, x["K_loc"].view(B * self.t_loc, d.n_kv, d.head_dim), pos)
            self.per_layer.append(x)
        self.capacity = B * self.k * self.max_doc_chunks  # the largest possible selection
        self.arr = msa.tiered_layers(self.per_layer)
        self.ws = torch.empty(msa.tiered_workspace_size(d, L, B, self.n_docs, self.C, self.k, self.t_loc,
                                                        self.pos, self.capacity) + 256, dtype=torch.uint8, device=dev)
        torch.cuda.synchronize()

    def run(self, stream=None, copy_stream=None, arr=None):
        self.msa.tiered_decode(self.d, self.arr if arr is None else arr, self.B, self.chunk_off, self.C, self.k,
                               self.loc_len, self.t_loc, self.pos, self.capacity, ws=self.ws, stream=stream,
                               copy_stream=copy_stream)

    @property
    def scan_bytes(self):
        """Algorithmic bytes of one scan: the pooled router keys and their inverse norms."""
        return self.C * self.d.n_r * (self.d.d_r * 2 + 4)

    def gathered_chunks(self):
        """Chunks of the documents the last call routed, per layer (host sync)."""
        co = self.co_np
        out = []
        for x in self.per_layer:
            sel = x["topk_idx"].cpu().numpy()
            out.append(int(sum(int(co[i + 1] - co[i]) for i in sel.reshape(-1))))
        return out


class AuxCase:
    def __init__(self, P, N, seed, device, dims=W.QWEN3_4B_DIMS, tau=0.05):
        import torch

        import long_context_memory_b200 as msa

        self.msa, self.d, self.tau = msa, dims, tau
        g = torch.Generator(device=device)
        g.manual_seed(seed)
        self.Q = randn_bf16((P, dims.n_r, dims.d_r), g, device)
        self.Kp = randn_bf16((P, dims.n_r, dims.d_r), g, device)
        self.Kn = randn_bf16((P, N, dims.n_r, dims.d_r), g, device)
        self.out = None
        self.ws = None
        row = dims.n_r * dims.d_r
        # HBM bytes: queries and keys read once (bf16), gradients written (fp32)
        self.bytes = P * (N + 2) * row * 2 + P * (N + 2) * row * 4

    def run(self):
        self.out = self.msa.aux_loss(self.d, self.Q, self.Kp, self.Kn, self.tau, out=self.out, ws=self.ws)


class EncodeCase:
    def __init__(self, T, seed, device, dims=W.QWEN3_4B_DIMS):
        import torch

        import long_context_memory_b200 as msa

        self.msa, self.d, self.T = msa, dims, T
        c = W.encode_config(T=T, seed=seed, with_hidden=False)
        co, C = msa.chunk_offsets(c["doc_off"])
        self.C = C
        self.H = W.encode_hidden(T, dims.hidden, seed, device)
        t = lambda a: W.to_torch(np.ascontiguousarray(a)).to(device)
        self.doc_off = torch.from_numpy(c["doc_off"]).to(device)
        self.chunk_off = torch.from_numpy(co).to(device)
        self.W = (t(c["W_K"]), t(c["W_V"]), t(c["W_KR"]))
        self.out = (torch.empty((C, dims.n_kv, dims.head_dim), dtype=torch.bfloat16, device=device),
                    torch.empty((C, dims.n_kv, dims.head_dim), dtype=torch.bfloat16, device=device),
                    torch.empty((C, dims.n_r, dims.d_r), dtype=torch.bfloat16, device=device))
        self.ws = torch.empty(msa.encode_workspace_size(dims, T, len(co) - 1, C) + 256, dtype=torch.uint8,
                              device=device)
        NK = dims.n_kv * dims.head_dim
        NVR = NK + dims.n_r * dims.d_r
        self.flops_k = 2.0 * T * dims.hidden * NK
        self.flops_pooled = 2.0 * C * (2 * dims.hidden) * NVR

    def run(self):
        self.msa.encode_memory(self.d, self.H, self.doc_off, self.chunk_off, self.C, *self.W, out=self.out,
                               ws=self.ws)


def main():
    import torch

    ap = argparse.ArgumentParser()
    ap.add_argument("--case", required=True,
                    choices=["route1m", "route16m", "route100m", "attend1m", "attend16m", "tiered", "encode", "aux"])
    ap.add_argument("--launches", type=int, default=3)
    ap.add_argument("--warmup", type=int, default=2)
    ap.add_argument("--batch", type=int, default=None)
    ap.add_argument("--tokens", type=int, default=None, help="memory tokens (encode default 1M; route cases: "
                    "their own size unless given)")
    ap.add_argument("--kr-layout", choices=["chunk", "head"], default="chunk")
    ap.add_argument("--norms", action="store_true", help="route cases: pass precomputed key norms")
    ap.add_argument("--layers", type=int, default=2, help="tiered case: layer instances per call")
    ap.add_argument("--one-stream", action="store_true", help="tiered case: every kernel on one stream (no "
                    "copy stream: each kernel has the whole GPU)")
    a = ap.parse_args()
    dev = torch.device("cuda:0")
    seed = W.BASE_SEED + 7
    hm, nm = a.kr_layout == "head", a.norms
    if a.case == "route1m":
        case = RouteCase(a.tokens or 1_000_000, a.batch or 1, 2048, seed, dev, head_major=hm, norms=nm)
    elif a.case == "route16m":
        case = RouteCase(a.tokens or 16_000_000, a.batch or 32, 2048, seed, dev, head_major=hm, norms=nm)
    elif a.case == "route100m":
        case = RouteCase(a.tokens or 100_000_000, a.batch or 1, 4096, seed, dev, head_major=hm, norms=nm)
    elif a.case == "attend1m":
        case = AttendCase(1_000_000, a.batch or 1, 2048, 4096, seed, dev)
    elif a.case == "attend16m":
        case = AttendCase(16_000_000, a.batch or 32, 2048, 8192, seed, dev)
    elif a.case == "aux":
        case = AuxCase(a.batch or 4096, 63, seed, dev)
    elif a.case == "tiered":
        case = TieredCase(a.tokens or 100_000_000, 4096, 8192, W.BASE_SEED + 4, dev, a.layers, 1, B=a.batch or 1)
    else:
        case = EncodeCase(a.tokens or 1_000_000, seed, dev)
    s = torch.cuda.Stream()
    if a.case == "tiered":  # the gather on its own stream, as a decode loop runs it
        cs = None if a.one_stream else torch.cuda.Stream()
        tcase = case
        case = type("Run", (), {"run": staticmethod(lambda: tcase.run(s, cs))})
    with torch.cuda.stream(s):
        for _ in range(a.warmup):
            case.run()
        torch.cuda.synchronize()
        for i in range(a.launches):
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(s)
            case.run()
            e1.record(s)
            torch.cuda.synchronize()
            tag = f"{a.case}[{a.kr_layout}{',norms' if a.norms else ''}]" if a.case.startswith("route") else a.case
            print(f"{tag} launch {i}: {e0.elapsed_time(e1) * 1e3:.1f} us", flush=True)


if __name__ == "__main__":
    main()
