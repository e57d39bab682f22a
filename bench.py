"""Benchmark of the MSA hot path on B200: route (Q^R projection, K̄^R scan, top-k)
plus sparse decode attention over the selected documents and the local KV.

One step = one pass of the whole online path for one batch of queries:
msa_route_topk (projection from H_q, scan + per-document max, top-k) followed by
msa_sparse_attend (gather of the selected docs' pooled K̄/V̄ + local KV with
global RoPE, split-KV flash-decode, combine).  Inputs are synthetic (seeded) with
the shapes of the 1M-token, Qwen3-4B-like workload (documents of varied length,
32 query heads over 8 KV heads of 128, 8 router heads of 128, top-16, 64-token chunks, 4K local KV, B=1).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl msa|reference]

Prints one JSON line (rank 0).  Under torchrun each rank runs an independent
replica of the workload (the path shards by query batch / memory bank with no
data-path exchange), timing is max over ranks and `value` sums all ranks' work.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "memory tokens routed/s (top-k + sparse attn); scan HBM GB/s vs peak"
UNIT = "tokens/s"
N_ROT = 8  # rotating input copies: K̄^R + K̄ + V̄ + local KV x 8 = 1.4 GB > L2 (126 MB)


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="msa", choices=["msa", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=15.0)
    ap.add_argument("--no-extras", action="store_true",
                    help="skip the 16M/100M-token routing and the encode measurements")
    return ap.parse_args()


def dist_env():
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return ws, rank, local


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return float(d["hbm_gbs"]), "measured"
    return 6650.0, "fallback"


def workload_config():
    from long_context_memory_b200 import workloads as W

    c = W.mem1m_config()
    return c


def workload_label(c) -> str:
    """The workload's name and sizes, the same on both arms."""
    return ("mem1m: 1M-token memory (C=%d chunks, %d docs), Qwen3-4B-like dims (hidden 2560, 32q/8kv x 128, "
            "8 router heads x 128), B=%d, top-%d, %d-token local KV"
            % (c["KR"].shape[0], len(c["doc_off"]) - 1, c["B"], c["k"], c["t_loc_max"]))


# ----------------------------------------------------------------------------
# oracle timing (cpu_baseline and --impl reference)
# ----------------------------------------------------------------------------
def time_oracle(c, seconds: float):
    """Oracle route + attend for the workload's query batch, repeated within a time budget."""
    import oracle as O

    try:
        from threadpoolctl import threadpool_limits
        limiter = threadpool_limits(limits=1)
    except Exception:  # pragma: no cover
        limiter = None
    d = c["dims"]
    co, *_ = O.chunk_layout(c["doc_off"])
    steps, t0 = 0, time.perf_counter()
    while True:
        QR = O.router_query(c["Hq"], c["W_QR"], d.n_r, d.d_r)
        _, idx, _ = O.route_topk(QR, c["KR"], co, c["k"])
        O.sparse_attend(c["q"], c["K_bar"], c["V_bar"], co, idx, c["K_loc"], c["V_loc"], c["loc_len"],
                        c["pos_offset"], d.rope_base)
        steps += 1
        el = time.perf_counter() - t0
        if el >= seconds or steps >= 50:
            break
    if limiter is not None:
        limiter.unregister() if hasattr(limiter, "unregister") else None
    per_step = el / steps
    return dict(value=c["T"] * c["B"] / per_step, unit=UNIT, cores=1, kind="oracle",
                sample=f"{steps} full steps of the 1M-token workload (B={c['B']}), numpy fp64, 1 thread, "
                       f"{el:.1f} s", ms_per_step=per_step * 1e3)


def run_reference(args):
    ws, rank, _ = dist_env()
    if rank != 0:
        return
    c = workload_config()
    steps = max(1, args.steps)
    budget = min(20.0, max(3.0, 1.0 * steps))
    r = time_oracle(c, budget)
    line = {
        "impl": "reference", "metric": METRIC, "value": r["value"], "unit": UNIT, "n_gpus": args.gpus,
        "steps": steps, "warmup": args.warmup, "ms_per_step": r["ms_per_step"], "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": workload_label(c), "parallelism": "one host thread"},
        "cpu_baseline": {"value": r["value"], "unit": UNIT, "cores": r["cores"], "kind": "oracle",
                         "sample": r["sample"]},
        "e2e": {"value": r["value"], "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


# ----------------------------------------------------------------------------
# clocks during the timed region
# ----------------------------------------------------------------------------
class ClockSampler:
    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,clocks_event_reasons.hw_slowdown,"
         "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
         "clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.idx = gpu_index
        self.proc = None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(["nvidia-smi", f"--query-gpu={self.Q}", "--format=csv,noheader,nounits",
                                          "-i", str(self.idx), "-lms", "100"], stdout=subprocess.PIPE,
                                         stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None
        time.sleep(0.3)
        return self

    def __exit__(self, *a):
        self.lines = []
        if self.proc is not None:
            time.sleep(0.25)
            self.proc.terminate()
            try:
                out, _ = self.proc.communicate(timeout=5)
            except Exception:
                out = ""
            self.lines = [l for l in out.splitlines() if l.strip()]

    def summary(self):
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for l in getattr(self, "lines", []):
            f = [x.strip() for x in l.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                mx = float(f[2])
            except ValueError:
                continue
            for n, v in zip(names, f[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": mx, "reasons": ["unavailable"]}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm)}


# ----------------------------------------------------------------------------
# the GPU arm
# ----------------------------------------------------------------------------
def source_digest(names) -> str:
    """sha256 over the named csrc files with // comments and blank lines removed: a change
    to the code (not to its comments) changes the digest."""
    h = hashlib.sha256()
    for name in names:
        for line in open(os.path.join(ROOT, "long_context_memory_b200", "csrc", name), encoding="utf-8"):
            code = line.split("//", 1)[0].rstrip()
            if code:
                h.update(code.encode() + b"\n")
    return h.hexdigest()


def scan_traffic_record(kernel: str):
    """Per-launch DRAM bytes of `kernel` from a committed ncu summary, or None.

    A summary records the digest of the kernel's source files (`source_digest`); if the code
    has changed since the counters were taken the figure is stale and not used."""
    path = os.path.join(ROOT, "profiles", f"{kernel}_traffic.txt")
    if not os.path.exists(path):
        return None
    kv = {}
    for line in open(path):
        if ":" in line and not line.startswith("#"):
            a, b = line.split(":", 1)
            kv[a.strip()] = b.strip()
    names = kv.get("sources", "").split()
    try:
        if not names or source_digest(names) != kv.get("code_sha256"):
            return None
        return float(kv["dram_bytes_per_launch_full_size"])
    except (OSError, KeyError, ValueError):
        return None


def kernel_times(msa, stream, step, n):
    """Per-kernel device time of n eager steps, each kernel bracketed by trace events.

    The launches are queued behind a bounded sleep kernel so that the host is far
    ahead of the device and every bracket holds only its kernel."""
    import torch

    msa.trace_reset()
    msa.trace_enable(True)
    try:
        with torch.cuda.stream(stream):
            torch.cuda._sleep(40_000_000)  # ~20 ms of device time, bounded by the clock
            for i in range(n):
                step(i)
        torch.cuda.synchronize()
    finally:
        msa.trace_enable(False)
    kt = msa.trace_read()
    msa.trace_reset()
    return kt


def run_extras(msa, dev, hbm_peak):
    """Routing at 16M (B=32) and 100M tokens (36 layer instances, B=1 and 16), the 100M-token host tier
    (gather + attention, B=1 and 16), and encoding 1M tokens."""
    import torch

    from long_context_memory_b200 import profile_cases as PC
    from long_context_memory_b200 import workloads as W

    out = {}
    stream = torch.cuda.Stream(device=dev)

    def timed(fn, n, warm=2):
        with torch.cuda.stream(stream):
            for _ in range(warm):
                fn(0)
            torch.cuda.synchronize()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            for i in range(n):
                fn(i)
            e1.record(stream)
            torch.cuda.synchronize()
        return e0.elapsed_time(e1) / n

    def route_entry(name, case, layers):
        n = 6 * layers
        ms = timed(lambda i: case.run(i % layers), n)
        kt = kernel_times(msa, stream, lambda i: case.run(i % layers), n)
        sms, scnt = kt["scan"]
        scan_us = sms / scnt * 1e3
        gbs = case.scan_bytes / (scan_us * 1e-6) / 1e9
        out[name] = {"workload": f"{case.T / 1e6:.0f}M-token memory, C={case.C} chunks, B={case.B}, top-{case.k}",
                     "layers": layers, "ms_per_layer": ms, "memory_tokens_routed_per_s": case.T * case.B / (ms * 1e-3),
                     "scan": {"avg_us": scan_us, "GB/s": gbs, "frac": gbs / hbm_peak, "bound": "hbm",
                              "algorithmic_bytes_per_launch": case.scan_bytes},
                     "kernels_us": {k: v[0] / v[1] * 1e3 for k, v in kt.items() if v[1]}}

    try:
        c16 = PC.RouteCase(16_000_000, 32, 2048, W.BASE_SEED + 2, dev, norms=True)
        route_entry("mem16m_b32_route", c16, 1)
        del c16
        a16 = PC.AttendCase(16_000_000, 32, 2048, 8192, W.BASE_SEED + 2, dev, rotated=True)
        ms = timed(lambda i: a16.run(), 10)
        kt = kernel_times(msa, stream, lambda i: a16.run(), 10)
        ams, acnt = kt["attn_split"]
        a_us = ams / acnt * 1e3
        agbs = a16.kv_bytes / (a_us * 1e-6) / 1e9
        out["mem16m_b32_attend"] = {"workload": "sparse attention, 16M-token memory, B=32, top-16, 8K local KV "
                                                "(rotated cache)", "ms": ms,
                                    "attn_split": {"avg_us": a_us, "GB/s": agbs, "frac": agbs / hbm_peak,
                                                   "bound": "hbm", "algorithmic_bytes_per_launch": a16.kv_bytes},
                                    "kernels_us": {k: v[0] / v[1] * 1e3 for k, v in kt.items() if v[1]}}
        del a16
        torch.cuda.empty_cache()
        free = torch.cuda.mem_get_info(dev)[0]
        layers = int(max(1, min(36, (free - (8 << 30)) // 3_300_000_000)))
        c100 = PC.RouteCase(100_000_000, 1, 4096, W.BASE_SEED + 4, dev, layers=layers, norms=True)
        route_entry("mem100m_b1_route", c100, layers)
        c100.set_batch(16, seed=W.BASE_SEED + 40)
        route_entry("mem100m_b16_route", c100, layers)
        del c100
        torch.cuda.empty_cache()
        # host tier: one layer's K̄/V̄ (100M tokens, 6.4 GB) in pinned host memory; per step only the
        # selected documents cross the host link, then attention over them + 8K local tokens
        for Bh in (1, 16):
            try:
                ht = PC.HostTierCase(100_000_000, Bh, 4096, 8192, W.BASE_SEED + 4, dev)
                g_ms = timed(lambda i: ht.gather(), 10)
                a_ms = timed(lambda i: ht.attend(), 10)
                out[f"mem100m_b{Bh}_host_tier"] = {
                    "workload": f"100M-token memory, K̄/V̄ in pinned host memory, B={Bh}, top-{ht.k}, 8K local KV",
                    "gather_ms": g_ms, "gathered_MB": ht.gather_bytes / 1e6,
                    "host_link_GB/s": ht.gather_bytes / (g_ms * 1e-3) / 1e9, "attend_ms": a_ms,
                    "attend_GB/s": ht.kv_bytes / (a_ms * 1e-3) / 1e9}
                del ht
            except Exception as e:  # e.g. pinned host memory unavailable: report it, keep the rest
                out[f"mem100m_b{Bh}_host_tier"] = {"error": f"{type(e).__name__}: {e}"}
            torch.cuda.empty_cache()
        enc = PC.EncodeCase(1_000_000, W.BASE_SEED + 5, dev)
        ms = timed(lambda i: enc.run(), 3, warm=1)
        kt = kernel_times(msa, stream, lambda i: enc.run(), 3)
        gms, gcnt = kt["enc_gemm_k"]
        g_us = gms / gcnt * 1e3
        tflops = enc.flops_k / (g_us * 1e-6) / 1e12
        out["encode_1m"] = {"workload": f"encode 1M tokens, hidden 2560, C={enc.C} chunks", "ms": ms,
                            "tokens_per_s": enc.T / (ms * 1e-3),
                            "gemm_k": {"avg_us": g_us, "TFLOP/s": tflops, "bound": "tensor",
                                       "frac_of_bf16_sustained": tflops / bf16_peak()[0],
                                       "algorithmic_flops": enc.flops_k},
                            "kernels_us": {k: v[0] / v[1] * 1e3 for k, v in kt.items() if v[1]}}
        del enc
        torch.cuda.empty_cache()
    except Exception as e:  # report, do not hide, a failed extra measurement
        out["error"] = f"{type(e).__name__}: {e}"
    return out


def bf16_peak():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return float(d.get("bf16_tflops_sustained", d["bf16_tflops"])), "measured"
    return 1400.0, "fallback"


def run_gpu(args):
    import torch
    import torch.distributed as dist

    import long_context_memory_b200 as msa
    from long_context_memory_b200 import workloads as W

    ws, rank, local = dist_env()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if ws > 1:
        dist.init_process_group("nccl", device_id=dev, timeout=__import__("datetime").timedelta(seconds=120))

    c = workload_config()
    d = c["dims"]
    B, k, T = c["B"], c["k"], c["T"]
    co_np, C = msa.chunk_offsets(c["doc_off"])
    n_docs = len(co_np) - 1
    chunk_off = torch.from_numpy(co_np).to(dev)
    t = lambda a: W.to_torch(np.ascontiguousarray(a)).to(dev)
    base = dict(KR=t(c["KR"]), K_bar=t(c["K_bar"]), V_bar=t(c["V_bar"]), K_loc=t(c["K_loc"]), V_loc=t(c["V_loc"]),
                Hq=t(c["Hq"]), q=t(c["q"]))
    W_QR = t(c["W_QR"])
    loc_len = torch.from_numpy(c["loc_len"]).to(dev)
    # distinct copies at distinct addresses so that consecutive steps miss L2
    rot = [base] + [{kk: v.clone() for kk, v in base.items()} for _ in range(N_ROT - 1)]
    # the pooled router keys' inverse norms, computed once per memory (offline, like the encoding)
    inv_rot = [msa.router_key_norms(d, x["KR"]) for x in rot]
    out_idx = [torch.empty((B, k), dtype=torch.int32, device=dev) for _ in range(N_ROT)]
    out_sc = [torch.empty((B, k), dtype=torch.float32, device=dev) for _ in range(N_ROT)]
    out_o = [torch.empty((B, d.n_q, d.head_dim), dtype=torch.bfloat16, device=dev) for _ in range(N_ROT)]
    r_ws = torch.empty(msa.route_workspace_size(d, B, n_docs, C, k) + 256, dtype=torch.uint8, device=dev)
    a_ws = torch.empty(msa.attend_workspace_size(d, B, k, c["t_loc_max"], c["pos_offset"]) + 256,
                       dtype=torch.uint8, device=dev)
    stream = torch.cuda.Stream(device=dev)
    # The local key cache holds keys already rotated at their global positions (rotated once,
    # when appended).  Each decode step rotates and appends only the new token's key, then
    # attends over the rotated cache.
    Lm1 = int(c["loc_len"][0]) - 1
    T_loc = c["t_loc_max"]
    for x in rot:
        msa.rope_rows(d, x["K_loc"].view(B * T_loc, d.n_kv, d.head_dim),
                      (c["pos_offset"] + torch.arange(T_loc, dtype=torch.int32, device=dev)).repeat(B))
    k_new = base["K_loc"][:, Lm1].clone()          # the new token's key before RoPE (synthetic)
    v_new = base["V_loc"][:, Lm1].clone()
    slots = torch.full((B,), Lm1, dtype=torch.int32, device=dev)
    torch.cuda.synchronize()

    def step(i):
        # one stream: routing, then sparse attention, which first writes the new token's rotated key
        # and value into the local cache (k_new / v_new: the append fused into the call).  The
        # attention's local-key work starts while the routing's kernels finish (early_local: q and
        # the local cache are not written by the routing).
        x = rot[i % N_ROT]
        j = i % N_ROT
        msa.route_topk(d, x["Hq"], W_QR, x["KR"], chunk_off, k, out=(out_idx[j], out_sc[j], None), ws=r_ws,
                       kr_inv_norm=inv_rot[j])
        msa.sparse_attend(d, x["q"], x["K_bar"], x["V_bar"], chunk_off, out_idx[j], x["K_loc"], x["V_loc"], loc_len,
                          c["pos_offset"], out=out_o[j], ws=a_ws, k_loc_rotated=True, early_local=True,
                          k_new=k_new, v_new=v_new)

    # ---- capture one graph per rotation copy (untraced) ----
    graphs = []
    with torch.cuda.stream(stream):
        for i in range(N_ROT):  # eager warm-up also sets kernel attributes outside capture
            step(i)
    torch.cuda.synchronize()
    use_graphs = True
    try:
        for i in range(N_ROT):
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=stream):
                step(i)
            graphs.append(g)
    except Exception as e:  # pragma: no cover
        print(f"graph capture failed ({e}); timing eager launches", file=sys.stderr)
        use_graphs = False
    torch.cuda.synchronize()

    def launch(i):
        with torch.cuda.stream(stream):
            if use_graphs:
                graphs[i % N_ROT].replay()
            else:
                step(i)

    def timed_region(n, warm):
        for i in range(warm):
            launch(i)
        torch.cuda.synchronize()
        if ws > 1:
            dist.barrier()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for i in range(n):
            launch(i)
        e1.record(stream)
        torch.cuda.synchronize()
        ms = e0.elapsed_time(e1)
        if ws > 1:
            tt = torch.tensor([ms], device=dev)
            dist.all_reduce(tt, op=dist.ReduceOp.MAX)
            ms = float(tt.item())
            dist.barrier()
        torch.cuda.synchronize()
        return ms

    with ClockSampler(local) as clk:
        total_ms = timed_region(args.steps, args.warmup)
    clocks = clk.summary()
    ms_step = total_ms / args.steps
    value = T * B * ws / (ms_step * 1e-3)

    # ---- per-kernel device time: the same steps, each kernel bracketed by trace events ----
    kt = kernel_times(msa, stream, step, args.steps)

    # ---- roofline of the dominant kernel ----
    hbm_peak, peak_kind = peaks()
    sel = out_idx[0].cpu().numpy()
    n_sel = int(sum(co_np[i + 1] - co_np[i] for i in sel[0]))
    per_kernel = {n: (ms, cnt) for n, (ms, cnt) in kt.items() if cnt > 0}
    scan_bytes = C * d.n_r * (d.d_r * 2 + 4)  # the pooled router keys and their inverse norms
    attn_bytes = B * (n_sel + int(c["loc_len"][0])) * d.n_kv * d.head_dim * 2 * 2
    cand = {"scan": scan_bytes, "attn_split": attn_bytes}  # algorithmic bytes per step
    # per step: the attention's split kernel runs twice (local keys beside the routing, then the
    # selected chunks), so its bytes and its time are both taken per step
    n_steps = max(1, args.steps)
    dom = max(cand, key=lambda n: per_kernel.get(n, (0, 1))[0])
    dms, dcnt = per_kernel[dom]
    step_s = dms / n_steps * 1e-3
    achieved = cand[dom] / step_s / 1e9
    traffic = scan_traffic_record(dom)
    roofline = {"kernel": dom, "bound": "hbm", "achieved": achieved, "peak": hbm_peak, "unit": "GB/s",
                "frac": achieved / hbm_peak, "traffic": traffic, "peak_kind": peak_kind,
                "algorithmic_bytes_per_launch": cand[dom] * n_steps / dcnt, "avg_launch_us": dms / dcnt * 1e3,
                "launches_per_step": dcnt / n_steps}
    kernels = {n: {"avg_us": ms / cnt * 1e3, "launches": cnt} for n, (ms, cnt) in per_kernel.items()}
    for n, b in cand.items():
        if n in per_kernel:
            kernels[n]["GB/s"] = b / (per_kernel[n][0] / n_steps * 1e-3) / 1e9
    gpu_launches = sum(cnt for (_, cnt) in per_kernel.values()) // max(1, args.steps) * args.steps

    # ---- end to end through the public API from pinned host buffers ----
    # Per decode step the host supplies the query hidden state H_q, the query q and
    # the new token's K/V row, which is rotated and appended to the device-resident
    # local KV cache at position loc_len - 1; the step returns top-k ids/scores and
    # the attention output.
    # The step's inputs travel in one pinned host buffer and one copy (H_q | q | new K | new V, each
    # at a 16-byte offset), its results come back the same way (top-k ids | scores | output):
    # one host-to-device and one device-to-host transfer per step.
    def packed(tensors):
        offs, n = [], 0
        for t in tensors:
            offs.append(n)
            n += (t.numel() * t.element_size() + 15) // 16 * 16
        return offs, n

    def views(buf, tensors, offs):
        return [buf[o:o + t.numel() * t.element_size()].view(t.dtype).view(t.shape) for t, o in zip(tensors, offs)]

    v_row = base["V_loc"][:, Lm1].contiguous()
    ins = [base["Hq"], base["q"], k_new, v_row]
    in_offs, in_bytes = packed(ins)
    host_in = torch.empty(in_bytes, dtype=torch.uint8).pin_memory()
    for hv, t in zip(views(host_in, ins, in_offs), ins):
        hv.copy_(t.cpu())
    dev_in = torch.empty(in_bytes, dtype=torch.uint8, device=dev)
    dev_hq, dev_q, dev_kn, dev_vn = views(dev_in, ins, in_offs)
    outs = [torch.empty((B, k), dtype=torch.int32), torch.empty((B, k), dtype=torch.float32),
            torch.empty((B, d.n_q, d.head_dim), dtype=torch.bfloat16)]
    out_offs, out_bytes = packed(outs)
    dev_out = torch.empty(out_bytes, dtype=torch.uint8, device=dev)
    e_idx, e_sc, e_out = views(dev_out, outs, out_offs)
    host_out = torch.empty(out_bytes, dtype=torch.uint8).pin_memory()
    h2d = sum(t.numel() * t.element_size() for t in ins)
    d2h = sum(t.numel() * t.element_size() for t in outs)

    def e2e_step(i):
        x = rot[i % N_ROT]
        dev_in.copy_(host_in, non_blocking=True)
        msa.route_topk(d, dev_hq, W_QR, x["KR"], chunk_off, k, out=(e_idx, e_sc, None), ws=r_ws,
                       kr_inv_norm=inv_rot[i % N_ROT])
        msa.sparse_attend(d, dev_q, x["K_bar"], x["V_bar"], chunk_off, e_idx, x["K_loc"], x["V_loc"], loc_len,
                          c["pos_offset"], out=e_out, ws=a_ws, k_loc_rotated=True, early_local=True,
                          k_new=dev_kn, v_new=dev_vn)
        host_out.copy_(dev_out, non_blocking=True)

    def e2e_time(run):
        with torch.cuda.stream(stream):
            for i in range(args.warmup):
                run(i)
            torch.cuda.synchronize()
            if ws > 1:
                dist.barrier()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            for i in range(args.steps):
                run(i)
            e1.record(stream)
            torch.cuda.synchronize()
        ms = e0.elapsed_time(e1) / args.steps
        if ws > 1:
            tt = torch.tensor([ms], device=dev)
            dist.all_reduce(tt, op=dist.ReduceOp.MAX)
            ms = float(tt.item())
        return ms

    # eager: every step issues its copies and library calls from Python
    e2e_eager_ms = e2e_time(e2e_step)
    # the same calls captured once per rotation copy in a CUDA graph (copies from and to the
    # pinned host buffers included), replayed every step: the way a decode loop issues a step
    e2e_graphs = []
    try:
        with torch.cuda.stream(stream):
            for i in range(N_ROT):
                g = torch.cuda.CUDAGraph()
                with torch.cuda.graph(g, stream=stream):
                    e2e_step(i)
                e2e_graphs.append(g)
        torch.cuda.synchronize()
        e2e_graph_ms = e2e_time(lambda i: e2e_graphs[i % N_ROT].replay())
    except Exception as e:  # pragma: no cover
        print(f"e2e graph capture failed ({e})", file=sys.stderr)
        e2e_graph_ms = None
    del e2e_graphs
    e2e_ms = e2e_eager_ms
    e2e_val = T * B * ws / (e2e_ms * 1e-3)

    extras = None
    if ws == 1 and not args.no_extras:
        extras = run_extras(msa, dev, hbm_peak)

    cpu = None
    if rank == 0 and ws == 1 and not args.no_cpu_baseline:
        r = time_oracle(c, args.cpu_seconds)
        cpu = {kk: r[kk] for kk in ("value", "unit", "cores", "kind", "sample")}

    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": ws, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16", "data": "synthetic (seeded N(0,1) bf16 pooled memory, lognormal docs)",
            "config": {"workload": workload_label(c),
                       "l2": "8 rotating input copies (%.2f GB) > L2" % (N_ROT * sum(v.numel() * 2 for v in base.values()) / 1e9),
                       "graphs": use_graphs, "parallelism": f"replicas x{ws}"},
            "roofline": roofline, "kernels": kernels, "gpu_launches": gpu_launches,
            "e2e": {"value": e2e_val, "unit": UNIT, "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                    "ms_per_step": e2e_ms, "issue": "eager: every step's copies and calls issued from Python",
                    "graph_ms_per_step": e2e_graph_ms,
                    "graph_value": T * B * ws / (e2e_graph_ms * 1e-3) if e2e_graph_ms else None},
            "cpu_baseline": cpu, "clocks": clocks, "extras": extras,
            "notes": "value: device time of CUDA-graph replays of the full decode step (append the new token's "
                     "rotated key and value to the local cache (fused into the attention call), route, sparse "
                     "attention over the rotated cache with early local work); kernels: trace-event brackets of eager "
                     "launches queued "
                     "behind a bounded sleep kernel; e2e: the same calls issued eagerly with one packed copy each "
                     "way per step",
        }
        print(json.dumps(line), flush=True)
    if ws > 1:
        dist.barrier()
        dist.destroy_process_group()


def main():
    args = parse()
    if args.impl == "reference":
        run_reference(args)
    else:
        run_gpu(args)


if __name__ == "__main__":
    main()
