"""Benchmark of the MSA hot path on B200: a decode step over a 100M-token memory served from
two tiers, on every layer of a 36-layer stack.

Workload (the largest that fits one GPU): a memory of 1e8 tokens in documents of lognormal
length (median 4096, 64-token chunks, ~1.57M chunks), Qwen3-4B-like dimensions (hidden 2560,
32 query heads over 8 KV heads of 128, 8 router heads of 128), top-16 documents, B = 1 query,
an 8K-token local KV cache per query, 36 independent layer instances.  Per layer the pooled
router keys K̄^R (3.2 GB) and their inverse norms live in HBM; the content K̄/V̄ (6.4 GB per
layer) live in pinned host memory.

One step = one msa_tiered_decode call over the 36 layers: per layer the router query (H_q W^QR),
the K̄^R scan with the per-document maximum and the top-16, the gather of the routed
documents' K̄/V̄ over the host link on a copy stream (overlapped with the next layer's routing),
and the sparse attention over the gathered chunks and the local cache (the new token's key and
value appended by the same call).  value = memory tokens routed per second = 36 T B / step time.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl msa|reference]

Prints one JSON line (rank 0).  Under torchrun each rank runs an independent replica of the
workload (no data-path exchange), timing is max over ranks and `value` sums all ranks' work.
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
T_MEM = 100_000_000      # memory tokens per layer
MEDIAN = 4096            # median document length
T_LOC = 8192             # local KV tokens per query
LAYERS = 36              # layer instances of one step
TOPK = 16
SEED_OFF = 4             # workload seed = BASE_SEED + 4
CPU_SAMPLE_FRACTION = 8  # the oracle routes a doc-aligned 1/8 of a layer's memory per step


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=4)
    ap.add_argument("--impl", default="msa", choices=["msa", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=12.0)
    ap.add_argument("--no-extras", action="store_true",
                    help="skip the B=16 tiered step, the 1M/16M-token cases and the encode measurement")
    ap.add_argument("--layers", type=int, default=LAYERS)
    ap.add_argument("--memory-parallel", action="store_true",
                    help="shard the 100M-token memory's documents over the ranks (routing, top-k exchange, "
                         "attention shares and their merge) instead of running replicas")
    return ap.parse_args()


def dist_env():
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return ws, rank, local


def peaks():
    """(HBM GB/s, bf16 burst TFLOP/s, bf16 sustained TFLOP/s, kind)."""
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return (float(d["hbm_gbs"]), float(d["bf16_tflops"]), float(d.get("bf16_tflops_sustained", d["bf16_tflops"])),
                "measured")
    return 6650.0, 1590.0, 1400.0, "fallback"


def workload_label(B: int = 1) -> str:
    """The workload's name and sizes, the same on both arms."""
    return (f"mem100m: 100M-token memory (lognormal docs, median {MEDIAN}, 64-token chunks), Qwen3-4B-like dims "
            f"(hidden 2560, 32q/8kv x 128, 8 router heads x 128), B={B}, top-{TOPK}, {T_LOC}-token local KV, "
            f"{LAYERS} layer instances; K̄^R in HBM, K̄/V̄ in pinned host memory")


# ----------------------------------------------------------------------------
# oracle timing (cpu_baseline and --impl reference): all host cores
# ----------------------------------------------------------------------------
def cpu_cores() -> int:
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:  # pragma: no cover
        return os.cpu_count() or 1


def time_oracle_shard(task):
    """Pool worker: the oracle's document scores of one doc-aligned shard of the sample."""
    from multiprocessing import shared_memory

    import oracle as O

    name, shape, c0, c1, co, QR, k = task
    shm = shared_memory.SharedMemory(name=name)
    try:
        KR = np.ndarray(shape, dtype=np.uint16, buffer=shm.buf)[c0:c1]
        s, _, _ = O.route_topk(QR, KR, co, min(k, len(co) - 1))
        return s
    finally:
        shm.close()


def time_oracle(seconds: float, max_steps: int, min_steps: int = 1):
    """The oracle's route + attend of the workload, on a doc-aligned sample of one layer, timed.

    The sample is the first documents of the 100M-token layout that cover 1/8 of it (the same
    lognormal lengths, N(0,1) router keys drawn by numpy); a process pool over all host cores
    scores doc-aligned shards of it, the parent takes the top-16 and runs the oracle attention
    over the selected documents and the 8K-token local KV.  Returns (tokens/s, per-step ms,
    cores, sample description)."""
    import concurrent.futures as cf
    import multiprocessing as mp
    from multiprocessing import shared_memory

    import oracle as O
    from long_context_memory_b200 import workloads as W

    d = W.QWEN3_4B_DIMS
    seed = W.BASE_SEED + SEED_OFF
    rng = np.random.default_rng(seed)
    lens = W.doc_lengths_lognormal(rng, T_MEM, MEDIAN)
    n_doc = int(np.searchsorted(np.cumsum(lens), T_MEM // CPU_SAMPLE_FRACTION) + 1)
    doc_off = W.offsets_from_lengths(lens[:n_doc])
    co, _, _, _ = O.chunk_layout(doc_off)
    C = int(co[-1])
    T_s = int(doc_off[-1])
    KR = W.normal_bf16(rng, (C, d.n_r, d.d_r))
    Hq = W.normal_bf16(rng, (1, d.hidden))
    W_QR = W.normal_bf16(rng, (d.hidden, d.n_r * d.d_r), 1.0 / math.sqrt(d.hidden))
    q = W.normal_bf16(rng, (1, d.n_q, d.head_dim))
    K_loc = W.normal_bf16(rng, (1, T_LOC, d.n_kv, d.head_dim))
    V_loc = W.normal_bf16(rng, (1, T_LOC, d.n_kv, d.head_dim))
    loc_len = np.full(1, T_LOC, dtype=np.int32)
    content = {}  # the selected documents' pooled K̄/V̄ rows, drawn per document

    def kv_rows(doc):
        if doc not in content:
            r = np.random.default_rng((seed, int(doc)))
            n = int(co[doc + 1] - co[doc])
            content[doc] = (W.normal_bf16(r, (n, d.n_kv, d.head_dim)), W.normal_bf16(r, (n, d.n_kv, d.head_dim)))
        return content[doc]

    cores = cpu_cores()
    workers = max(1, min(cores, 64))
    n_shards = workers * 4
    cut = [int(x) for x in np.linspace(0, n_doc, n_shards + 1).round()]
    shm = shared_memory.SharedMemory(create=True, size=KR.nbytes)
    try:
        np.ndarray(KR.shape, dtype=np.uint16, buffer=shm.buf)[:] = KR
        ctx = mp.get_context("spawn")
        with cf.ProcessPoolExecutor(max_workers=workers, mp_context=ctx) as pool:
            def step():
                QR = O.router_query(Hq, W_QR, d.n_r, d.d_r)
                tasks = [(shm.name, KR.shape, int(co[a]), int(co[b]), co[a:b + 1] - co[a], QR, TOPK)
                         for a, b in zip(cut[:-1], cut[1:]) if b > a]
                s = np.concatenate(list(pool.map(time_oracle_shard, tasks)), axis=1)
                idx, _ = O.topk(s[0], TOPK)
                kv = [kv_rows(i) for i in idx]
                Ks = np.concatenate([x[0] for x in kv])
                Vs = np.concatenate([x[1] for x in kv])
                co_s = np.concatenate([[0], np.cumsum([x[0].shape[0] for x in kv])])
                O.sparse_attend(q, Ks, Vs, co_s, np.arange(TOPK)[None], K_loc, V_loc, loc_len, TOPK, d.rope_base)

            step()  # warm-up: workers started, the selected documents' rows drawn
            steps, t0 = 0, time.perf_counter()
            while True:
                step()
                steps += 1
                el = time.perf_counter() - t0
                if steps >= max_steps or (el >= seconds and steps >= min_steps):
                    break
    finally:
        shm.close()
        shm.unlink()
    per_step = el / steps
    sample = (f"{steps} oracle steps (numpy fp64) of one layer, B=1: routing over the first {n_doc} documents "
              f"({T_s} tokens, {C} chunks, 1/{CPU_SAMPLE_FRACTION} of the 100M-token layout) by a pool of "
              f"{workers} processes, top-{TOPK}, attention over the selected documents + {T_LOC} local tokens; "
              f"{el:.1f} s")
    return T_s / per_step, per_step * 1e3, workers, sample


def run_reference(args):
    ws, rank, _ = dist_env()
    if rank != 0:
        return
    steps = max(1, args.steps)
    value, ms, cores, sample = time_oracle(seconds=0.0, max_steps=steps, min_steps=steps)
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
        "steps": steps, "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": workload_label(), "parallelism": f"{cores} host processes"},
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle", "sample": sample},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
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
# DRAM traffic records (committed ncu summaries)
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


def scan_traffic_record(kernel: str, key: str = "dram_bytes_per_launch_full_size"):
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
        return float(kv[key])
    except (OSError, KeyError, ValueError):
        return None


# ----------------------------------------------------------------------------
# timing helpers
# ----------------------------------------------------------------------------
def kernel_times(msa, stream, step, n):
    """Per-kernel device time of n eager steps, each kernel bracketed by trace events on the
    stream it runs on.  The launches are queued behind a bounded sleep kernel so that the host
    is far ahead of the device and every bracket holds only its kernel."""
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
    return {k: v for k, v in kt.items() if v[1]}


def device_time(stream, fn, n, warm, dist=None, dev=None):
    """Device ms per call of fn over n calls after warm untimed ones (CUDA events on `stream`,
    barrier + synchronize on both sides, max over ranks)."""
    import torch

    with torch.cuda.stream(stream):
        for i in range(warm):
            fn(i)
    torch.cuda.synchronize()
    if dist is not None:
        dist.barrier()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        e0.record(stream)
        for i in range(n):
            fn(i)
        e1.record(stream)
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1)
    if dist is not None:
        tt = torch.tensor([ms], device=dev)
        dist.all_reduce(tt, op=dist.ReduceOp.MAX)
        ms = float(tt.item())
        dist.barrier()
    torch.cuda.synchronize()
    return ms / n


def capture(stream, fn):
    """fn captured once in a CUDA graph on `stream` (None when capture fails)."""
    import torch

    try:
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=stream):
            fn()
        torch.cuda.synchronize()
        return g
    except Exception as e:  # pragma: no cover
        print(f"graph capture failed ({e}); timing eager launches", file=sys.stderr)
        torch.cuda.synchronize()
        return None


def layers_that_fit(dev, want: int, per_layer_bytes: int, reserve_bytes: int) -> int:
    import torch

    torch.cuda.empty_cache()
    free = torch.cuda.mem_get_info(dev)[0]
    return int(max(1, min(want, (free - reserve_bytes) // per_layer_bytes)))


def host_layers_that_fit(per_layer_bytes: int, want: int = 2) -> int:
    """Distinct pinned host instances of a layer's K̄/V̄ (at most a quarter of the free host RAM)."""
    try:
        import psutil

        avail = psutil.virtual_memory().available
    except Exception:  # pragma: no cover
        avail = 4 * per_layer_bytes
    return int(max(1, min(want, avail // 4 // per_layer_bytes)))


# ----------------------------------------------------------------------------
# the GPU arm
# ----------------------------------------------------------------------------
def tiered_measure(msa, case, S, Cs, steps, warm, dist=None, dev=None, graphs=True):
    """(ms per call: pipelined graph or eager, serial, kernel times of the pipelined call)."""
    step = lambda i: case.run(S, Cs)
    g = capture(S, lambda: case.run(S, Cs)) if graphs else None
    piped = device_time(S, (lambda i: g.replay()) if g is not None else step, steps, warm, dist, dev)
    del g
    serial = device_time(S, lambda i: case.run(S, None), max(2, steps // 4), 1, dist, dev)
    kt = kernel_times(msa, S, step, max(2, steps // 2))
    return piped, serial, kt


def run_gpu(args):
    import torch
    import torch.distributed as dist

    import long_context_memory_b200 as msa
    from long_context_memory_b200 import profile_cases as PC
    from long_context_memory_b200 import workloads as W

    ws, rank, local = dist_env()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    dg = None
    if ws > 1:
        dist.init_process_group("nccl", device_id=dev, timeout=__import__("datetime").timedelta(seconds=120))
        dg = dist
    hbm_peak, bf16_burst, bf16_sust, peak_kind = peaks()
    d = W.QWEN3_4B_DIMS

    # ---- the workload: 100M-token memory, as many of the 36 layer instances as fit ----
    C_est = 1_580_000
    per_layer = C_est * d.n_r * (d.d_r * 2 + 4) + d.hidden * d.n_r * d.d_r * 2 + 2 * T_LOC * d.n_kv * d.head_dim * 2
    n_layers = layers_that_fit(dev, args.layers, per_layer, 24 << 30)
    # distinct pinned host copies of a layer's K̄/V̄ (6.4 GB each): one per rank when several ranks
    # share the host's memory
    host_layers = host_layers_that_fit(2 * C_est * d.n_kv * d.head_dim * 2, want=2 if ws == 1 else 1)
    case = PC.TieredCase(T_MEM, MEDIAN, T_LOC, W.BASE_SEED + SEED_OFF, dev, n_layers, host_layers, B=1, k=TOPK)
    n_chunks, n_docs = case.C, case.n_docs
    S = torch.cuda.Stream(device=dev)
    Cs = torch.cuda.Stream(device=dev)
    for _ in range(2):
        case.run(S, Cs)
    torch.cuda.synchronize()
    assert msa.check_device_errors() == 0

    # ---- timed region: CUDA-graph replays of the whole 36-layer step ----
    graph = capture(S, lambda: case.run(S, Cs))
    launch = (lambda i: graph.replay()) if graph is not None else (lambda i: case.run(S, Cs))
    with ClockSampler(local) as clk:
        ms_step = device_time(S, launch, args.steps, args.warmup, dg, dev)
    clocks = clk.summary()
    del graph
    B = case.B
    value = n_layers * T_MEM * B * ws / (ms_step * 1e-3)

    # ---- per-kernel device time: the same steps, each kernel bracketed by trace events ----
    kt = kernel_times(msa, S, lambda i: case.run(S, Cs), max(2, args.steps // 2))
    n_kt = max(2, args.steps // 2)
    gathered = case.gathered_chunks()
    per_kernel = {n: {"avg_us": ms / cnt * 1e3, "launches": cnt, "launches_per_step": cnt / n_kt}
                  for n, (ms, cnt) in kt.items()}
    scan_us = per_kernel["scan"]["avg_us"]
    achieved = case.scan_bytes / (scan_us * 1e-6) / 1e9
    roofline = {"kernel": "scan", "bound": "hbm", "achieved": achieved, "peak": hbm_peak, "unit": "GB/s",
                "frac": achieved / hbm_peak, "traffic": scan_traffic_record("scan"), "peak_kind": peak_kind,
                "algorithmic_bytes_per_launch": case.scan_bytes, "avg_launch_us": scan_us,
                "launches_per_step": per_kernel["scan"]["launches_per_step"]}
    # In the step the attention runs beside the next layer's scan on the few SMs the scan leaves
    # free, so its duration there measures the overlap, not the kernel: its roofline figure comes
    # from the same call on one stream, where every kernel has the whole GPU.
    kt_one = kernel_times(msa, S, lambda i: case.run(S, None), n_kt)
    one_stream = {n: {"avg_us": ms / cnt * 1e3} for n, (ms, cnt) in kt_one.items()}
    attn_bytes = (sum(gathered) / n_layers + B * T_LOC) * d.n_kv * d.head_dim * 2 * 2
    a_us = one_stream["attn_split"]["avg_us"]
    one_stream["attn_split"].update({"GB/s": attn_bytes / (a_us * 1e-6) / 1e9,
                                     "frac": attn_bytes / (a_us * 1e-6) / 1e9 / hbm_peak,
                                     "algorithmic_bytes_per_launch": attn_bytes})
    gbytes = sum(gathered) / n_layers * d.n_kv * d.head_dim * 2 * 2
    per_kernel["gather_copy"]["host_link_GB/s"] = gbytes / (per_kernel["gather_copy"]["avg_us"] * 1e-6) / 1e9
    per_kernel["scan"]["GB/s"] = achieved
    per_kernel["scan"]["frac"] = achieved / hbm_peak
    gpu_launches = int(round(sum(v["launches_per_step"] for v in per_kernel.values()))) * args.steps

    # ---- end to end through the public API from pinned host buffers ----
    # Per step and layer the host supplies the query hidden state H_q, the query q and the new
    # token's key and value; the step returns every layer's top-k ids and scores and attention
    # output.  One packed host-to-device copy and one device-to-host copy per step.
    def packed(tensors):
        offs, n = [], 0
        for t in tensors:
            offs.append(n)
            n += (t.numel() * t.element_size() + 15) // 16 * 16
        return offs, n

    def views(buf, tensors, offs):
        return [buf[o:o + t.numel() * t.element_size()].view(t.dtype).view(t.shape) for t, o in zip(tensors, offs)]

    ins = [x[f] for x in case.per_layer for f in ("Hq", "q", "k_new", "v_new")]
    outs = [x[f] for x in case.per_layer for f in ("topk_idx", "topk_score", "out")]
    in_offs, in_bytes = packed(ins)
    out_offs, out_bytes = packed(outs)
    host_in = torch.empty(in_bytes, dtype=torch.uint8).pin_memory()
    for hv, t in zip(views(host_in, ins, in_offs), ins):
        hv.copy_(t.cpu())
    dev_in = torch.empty(in_bytes, dtype=torch.uint8, device=dev)
    dev_out = torch.empty(out_bytes, dtype=torch.uint8, device=dev)
    host_out = torch.empty(out_bytes, dtype=torch.uint8).pin_memory()
    vin, vout = views(dev_in, ins, in_offs), views(dev_out, outs, out_offs)
    e2e_layers = []
    for l, x in enumerate(case.per_layer):
        y = dict(x)
        y.update(Hq=vin[4 * l], q=vin[4 * l + 1], k_new=vin[4 * l + 2], v_new=vin[4 * l + 3],
                 topk_idx=vout[3 * l], topk_score=vout[3 * l + 1], out=vout[3 * l + 2])
        e2e_layers.append(y)
    e2e_arr = msa.tiered_layers(e2e_layers)
    h2d = sum(t.numel() * t.element_size() for t in ins)
    d2h = sum(t.numel() * t.element_size() for t in outs)

    def e2e_step(i):
        dev_in.copy_(host_in, non_blocking=True)
        case.run(S, Cs, arr=e2e_arr)
        host_out.copy_(dev_out, non_blocking=True)

    e2e_ms = device_time(S, e2e_step, args.steps, args.warmup, dg, dev)
    e2e_val = n_layers * T_MEM * B * ws / (e2e_ms * 1e-3)

    # ---- the overlap of the gather with the next layer's routing, B = 1 ----
    serial_ms = device_time(S, lambda i: case.run(S, None), max(2, args.steps // 4), 1, dg, dev)
    g_us = per_kernel["gather_plan"]["avg_us"] + per_kernel["gather_copy"]["avg_us"]
    hidden_us = (serial_ms - ms_step) / n_layers * 1e3
    overlap = {"pipelined_ms_per_layer": ms_step / n_layers, "serial_ms_per_layer": serial_ms / n_layers,
               "gather_us_per_layer": g_us, "hidden_us_per_layer": hidden_us,
               "exposed_us_per_layer": max(0.0, g_us - hidden_us)}

    extras = None
    if ws == 1 and not args.no_extras:
        extras = {"mem100m_b1_overlap": overlap}
        extras.update(run_extras(msa, case, S, Cs, dev, hbm_peak, bf16_burst, bf16_sust, args))
    del case
    torch.cuda.empty_cache()

    cpu = None
    if rank == 0 and ws == 1 and not args.no_cpu_baseline:
        v, _, cores, sample = time_oracle(args.cpu_seconds, 20)
        cpu = {"value": v, "unit": UNIT, "cores": cores, "kind": "oracle", "sample": sample}

    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": ws, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic (seeded N(0,1) bf16 pooled memory and queries, lognormal document lengths)",
            "config": {"workload": workload_label(B), "layers": n_layers, "host_kv_instances": host_layers,
                       "chunks": n_chunks, "docs": n_docs,
                       "l2": "inputs larger than L2: each layer's K̄^R is 3.2 GB (126 MB L2)",
                       "graphs": True, "parallelism": f"replicas x{ws}"},
            "roofline": roofline, "kernels": per_kernel, "kernels_one_stream": one_stream,
            "gpu_launches": gpu_launches,
            "e2e": {"value": e2e_val, "unit": UNIT, "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                    "ms_per_step": e2e_ms,
                    "issue": "eager: one packed host-to-device copy, one msa_tiered_decode call, one packed "
                             "device-to-host copy per step"},
            "cpu_baseline": cpu, "clocks": clocks, "extras": extras,
            "notes": "value: device time of CUDA-graph replays of one msa_tiered_decode call over the layer "
                     "instances (the router queries of all layers, then the scans back to back on the main "
                     "stream; each layer's top-k, host-tier gather and sparse attention with the new token "
                     "appended on the copy stream beside the next scan); kernels: trace-event brackets of "
                     "eager calls queued behind a bounded sleep kernel; kernels_one_stream: the same call with "
                     "every kernel on one stream (the attention's roofline)",
        }
        print(json.dumps(line), flush=True)
    if ws > 1:
        dist.barrier()
        dist.destroy_process_group()


def run_extras(msa, case, S, Cs, dev, hbm_peak, bf16_burst, bf16_sust, args):
    """The same tiered step at B = 16; the 1M-token decode step and the 16M-token B = 32 routing and
    attention (device-resident memories); encoding 1M tokens."""
    import torch

    from long_context_memory_b200 import profile_cases as PC
    from long_context_memory_b200 import workloads as W

    out = {}
    d = case.d
    try:
        case.set_batch(16, W.BASE_SEED + 40)
        piped, serial, kt = tiered_measure(msa, case, S, Cs, 6, 2)
        L = case.n_layers
        gathered = case.gathered_chunks()
        g_us = kt["gather_plan"][0] / kt["gather_plan"][1] * 1e3 + kt["gather_copy"][0] / kt["gather_copy"][1] * 1e3
        gb = sum(gathered) / L * d.n_kv * d.head_dim * 2 * 2
        sc_us = kt["scan"][0] / kt["scan"][1] * 1e3
        # the attention's roofline from the same call on one stream (in the step it shares the GPU
        # with the gather)
        kt_one = kernel_times(msa, S, lambda i: case.run(S, None), 3)
        a_us = kt_one["attn_split"][0] / kt_one["attn_split"][1] * 1e3
        a_bytes = (sum(gathered) / L + 16 * T_LOC) * d.n_kv * d.head_dim * 2 * 2
        hidden = (serial - piped) / L * 1e3
        out["mem100m_b16_tiered"] = {
            "workload": workload_label(16), "layers": L, "ms_per_step": piped, "ms_per_layer": piped / L,
            "memory_tokens_routed_per_s": L * T_MEM * 16 / (piped * 1e-3),
            "serial_ms_per_layer": serial / L, "gather_us_per_layer": g_us, "hidden_us_per_layer": hidden,
            "exposed_us_per_layer": max(0.0, g_us - hidden), "gathered_MB_per_layer": gb / 1e6,
            "host_link_GB/s": gb / (kt["gather_copy"][0] / kt["gather_copy"][1] * 1e-3) / 1e9,
            "scan": {"avg_us": sc_us, "GB/s": case.scan_bytes / (sc_us * 1e-6) / 1e9,
                     "frac": case.scan_bytes / (sc_us * 1e-6) / 1e9 / hbm_peak},
            "attn_split_one_stream": {"avg_us": a_us, "GB/s": a_bytes / (a_us * 1e-6) / 1e9,
                                      "frac": a_bytes / (a_us * 1e-6) / 1e9 / hbm_peak},
            "kernels_us": {k: v[0] / v[1] * 1e3 for k, v in kt.items()}}
    except Exception as e:  # report, do not hide, a failed extra measurement
        out["mem100m_b16_tiered"] = {"error": f"{type(e).__name__}: {e}"}
    case.per_layer = None
    case.arr = None
    case.KR = case.inv = case.K_host = case.V_host = None
    torch.cuda.empty_cache()

    def timed(fn, n, warm=2):
        return device_time(S, fn, n, warm)

    try:
        a16 = PC.AttendCase(16_000_000, 32, 2048, 8192, W.BASE_SEED + 2, dev, rotated=True)
        ms = timed(lambda i: a16.run(), 10)
        kt = kernel_times(msa, S, lambda i: a16.run(), 10)
        a_us = kt["attn_split"][0] / kt["attn_split"][1] * 1e3
        agbs = a16.kv_bytes / (a_us * 1e-6) / 1e9
        out["mem16m_b32_attend"] = {"workload": "sparse attention, 16M-token memory (device-resident), B=32, top-16, "
                                                "8K local KV (rotated cache)", "ms": ms,
                                    "attn_split": {"avg_us": a_us, "GB/s": agbs, "frac": agbs / hbm_peak,
                                                   "algorithmic_bytes_per_launch": a16.kv_bytes},
                                    "kernels_us": {k: v[0] / v[1] * 1e3 for k, v in kt.items()}}
        del a16
        torch.cuda.empty_cache()
        c16 = PC.RouteCase(16_000_000, 32, 2048, W.BASE_SEED + 2, dev, norms=True)
        ms = timed(lambda i: c16.run(), 12)
        kt = kernel_times(msa, S, lambda i: c16.run(), 12)
        s_us = kt["scan"][0] / kt["scan"][1] * 1e3
        out["mem16m_b32_route"] = {"workload": f"16M-token memory, C={c16.C} chunks, B=32, top-16", "ms": ms,
                                   "memory_tokens_routed_per_s": c16.T * 32 / (ms * 1e-3),
                                   "scan": {"avg_us": s_us, "GB/s": c16.scan_bytes / (s_us * 1e-6) / 1e9,
                                            "frac": c16.scan_bytes / (s_us * 1e-6) / 1e9 / hbm_peak},
                                   "kernels_us": {k: v[0] / v[1] * 1e3 for k, v in kt.items()}}
        del c16
        torch.cuda.empty_cache()
    except Exception as e:
        out["mem16m_error"] = f"{type(e).__name__}: {e}"
    try:
        out["mem1m_decode_step"] = mem1m_step(msa, S, dev, hbm_peak)
    except Exception as e:
        out["mem1m_decode_step"] = {"error": f"{type(e).__name__}: {e}"}
    try:
        enc = PC.EncodeCase(1_000_000, W.BASE_SEED + 5, dev)
        ms = timed(lambda i: enc.run(), 3, warm=1)
        kt = kernel_times(msa, S, lambda i: enc.run(), 3)
        g_us = kt["enc_gemm_k"][0] / kt["enc_gemm_k"][1] * 1e3
        tflops = enc.flops_k / (g_us * 1e-6) / 1e12
        out["encode_1m"] = {"workload": f"encode 1M tokens, hidden 2560, C={enc.C} chunks", "ms": ms,
                            "tokens_per_s": enc.T / (ms * 1e-3),
                            "gemm_k": {"avg_us": g_us, "TFLOP/s": tflops, "bound": "tensor",
                                       "frac": tflops / bf16_burst, "peak": bf16_burst,
                                       "peak_kind": "burst (kernel timed alone)", "algorithmic_flops": enc.flops_k},
                            "kernels_us": {k: v[0] / v[1] * 1e3 for k, v in kt.items()}}
        del enc
        torch.cuda.empty_cache()
    except Exception as e:
        out["encode_1m"] = {"error": f"{type(e).__name__}: {e}"}
    return out


def mem1m_step(msa, S, dev, hbm_peak, n_rot=8):
    """The 1M-token decode step (device-resident memory, B=1, 4K local): route, then attention with the
    new token appended and early local work; graph replays over rotating input copies (> L2)."""
    import torch

    from long_context_memory_b200 import workloads as W

    c = W.mem1m_config(lambda off: msa.chunk_offsets(off)[0])
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
    T_loc = c["t_loc_max"]
    rot = [base] + [{kk: v.clone() for kk, v in base.items()} for _ in range(n_rot - 1)]
    for x in rot:
        msa.rope_rows(d, x["K_loc"].view(B * T_loc, d.n_kv, d.head_dim),
                      (c["pos_offset"] + torch.arange(T_loc, dtype=torch.int32, device=dev)).repeat(B))
    inv = [msa.router_key_norms(d, x["KR"]) for x in rot]
    o_idx = [torch.empty((B, k), dtype=torch.int32, device=dev) for _ in range(n_rot)]
    o_sc = [torch.empty((B, k), dtype=torch.float32, device=dev) for _ in range(n_rot)]
    o_out = [torch.empty((B, d.n_q, d.head_dim), dtype=torch.bfloat16, device=dev) for _ in range(n_rot)]
    r_ws = torch.empty(msa.route_workspace_size(d, B, n_docs, C, k) + 256, dtype=torch.uint8, device=dev)
    a_ws = torch.empty(msa.attend_workspace_size(d, B, k, T_loc, c["pos_offset"]) + 256, dtype=torch.uint8,
                       device=dev)
    Lm1 = int(c["loc_len"][0]) - 1
    k_new, v_new = base["K_loc"][:, Lm1].clone(), base["V_loc"][:, Lm1].clone()

    def step(i):
        x, j = rot[i % n_rot], i % n_rot
        msa.route_topk(d, x["Hq"], W_QR, x["KR"], chunk_off, k, out=(o_idx[j], o_sc[j], None), ws=r_ws,
                       kr_inv_norm=inv[j])
        msa.sparse_attend(d, x["q"], x["K_bar"], x["V_bar"], chunk_off, o_idx[j], x["K_loc"], x["V_loc"], loc_len,
                          c["pos_offset"], out=o_out[j], ws=a_ws, k_loc_rotated=True, early_local=True,
                          k_new=k_new, v_new=v_new)

    with torch.cuda.stream(S):
        for i in range(n_rot):
            step(i)
    torch.cuda.synchronize()
    graphs = [capture(S, (lambda j=j: step(j))) for j in range(n_rot)]
    ms = device_time(S, lambda i: graphs[i % n_rot].replay(), 40, 8)
    kt = kernel_times(msa, S, step, 40)
    scan_us = kt["scan"][0] / kt["scan"][1] * 1e3
    sb = C * d.n_r * (d.d_r * 2 + 4)
    return {"workload": f"mem1m: 1M-token memory (device-resident, C={C} chunks, {n_docs} docs), B=1, top-16, "
                        f"4K local KV; report only (the memory fits in L2)", "ms": ms,
            "memory_tokens_routed_per_s": T * B / (ms * 1e-3),
            "scan": {"avg_us": scan_us, "GB/s": sb / (scan_us * 1e-6) / 1e9,
                     "frac": sb / (scan_us * 1e-6) / 1e9 / hbm_peak},
            "kernels_us": {k: v[0] / v[1] * 1e3 for k, v in kt.items()}}


def run_memory_parallel(args):
    """The pages' memory-parallel deployment: every rank holds a contiguous range of the 100M-token
    memory's documents (its K̄^R, inverse norms and K̄/V̄, device-resident); per layer every rank
    routes its shard, the ranks exchange their (score, id) candidates and merge them, every rank
    attends over the selected documents it holds (the local cache on rank 0), and the shares are
    exchanged and merged.  value = layers x T x B / step time (the memory's tokens are split over
    the ranks: the total work is fixed, scaling "strong")."""
    import torch
    import torch.distributed as dist

    import long_context_memory_b200 as msa
    from long_context_memory_b200 import parallel as P
    from long_context_memory_b200 import profile_cases as PC
    from long_context_memory_b200 import workloads as W

    ws, rank, local = dist_env()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    os.environ.setdefault("MASTER_ADDR", "127.0.0.1")
    os.environ.setdefault("MASTER_PORT", "29533")
    os.environ.setdefault("RANK", str(rank))
    os.environ.setdefault("WORLD_SIZE", str(ws))
    dist.init_process_group("nccl", device_id=dev, timeout=__import__("datetime").timedelta(seconds=120))
    d = W.QWEN3_4B_DIMS
    layers = min(args.layers, 8)
    doc_off, co, C = PC.chunk_layout_host(T_MEM, MEDIAN, W.BASE_SEED + SEED_OFF)
    sh = P.shard_memory(co, ws, rank)
    g = torch.Generator(device=dev)
    g.manual_seed(W.BASE_SEED + SEED_OFF + 1000 * rank)
    KR = [PC.randn_bf16((sh.n_chunks, d.n_r, d.d_r), g, dev) for _ in range(layers)]
    inv = [msa.router_key_norms(d, kr) for kr in KR]
    Kb = PC.randn_bf16((sh.n_chunks, d.n_kv, d.head_dim), g, dev)  # content rows, shared by the layers
    Vb = PC.randn_bf16((sh.n_chunks, d.n_kv, d.head_dim), g, dev)
    gq = torch.Generator(device=dev)
    gq.manual_seed(W.BASE_SEED + SEED_OFF + 7)  # the same queries and weights on every rank
    W_QR = [(torch.randn((d.hidden, d.n_r * d.d_r), generator=gq, device=dev) / math.sqrt(d.hidden)).to(torch.bfloat16)
            for _ in range(layers)]
    Hq = [PC.randn_bf16((1, d.hidden), gq, dev) for _ in range(layers)]
    q = [PC.randn_bf16((1, d.n_q, d.head_dim), gq, dev) for _ in range(layers)]
    K_loc = PC.randn_bf16((1, T_LOC, d.n_kv, d.head_dim), gq, dev)
    V_loc = PC.randn_bf16((1, T_LOC, d.n_kv, d.head_dim), gq, dev)
    loc_len = torch.full((1,), T_LOC, dtype=torch.int32, device=dev)
    S = torch.cuda.Stream(device=dev)

    def step(i):
        for l in range(layers):
            idx, _ = P.route_topk_sharded(d, Hq[l], W_QR[l], KR[l], sh, TOPK, route=lambda *a: msa.route_topk(
                *a, kr_inv_norm=inv[l]))
            P.attend_sharded(d, q[l], Kb, Vb, sh, idx, K_loc, V_loc, loc_len, TOPK)

    ms = device_time(S, step, args.steps, args.warmup, dist, dev)
    if rank == 0:
        value = layers * T_MEM * 1 / (ms * 1e-3)
        print(json.dumps({
            "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": ws, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": ms, "higher_is_better": True, "scaling": "strong", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic (seeded N(0,1) bf16 pooled memory and queries, lognormal document lengths)",
            "config": {"workload": f"mem100m memory-parallel: 100M-token memory sharded by documents over {ws} "
                                   f"rank(s), B=1, top-{TOPK}, {T_LOC}-token local KV on rank 0, {layers} layer "
                                   f"instances (K̄/V̄ device-resident, one content copy shared by the layers)",
                       "parallelism": f"memory-parallel x{ws}"}}), flush=True)
    dist.barrier()
    dist.destroy_process_group()


def main():
    args = parse()
    if args.impl == "reference":
        run_reference(args)
    elif args.memory_parallel:
        run_memory_parallel(args)
    else:
        run_gpu(args)


if __name__ == "__main__":
    main()
