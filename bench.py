"""Benchmark of the routed-MoE layer over the HBM expert cache.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference] [--workload decode_bf16]

One step is one pass of the whole hot path over one batch of synthetic input:
for the default workload (single-layer BF16 decode: E=256, top-6, d=4096,
d_ff=1536, 37% cache = 94 slots, LRU, B_P:B_H = 52.7:77.3) a step starts from
a cold cache (every expert on the host, as on a first request) and runs the
64-step decode trace at batch 1, 4 and 16 -- 192 layer calls, 1344 tokens.
Inputs (hidden states, router weights, Zipf router bias) are resident in HBM
before the timed region; the expert pool lives in pinned host memory and
reaches the GPU through the cache (copy engine) or zero-copy reads, which is
the workload. The pool (9.7 GB) and the slot pool (3.5 GB) are larger than
L2, so no L2 flush is needed between steps.

Rank 0 prints one JSON line. With N > 1 (torchrun) every rank runs an
independent replica on its own data (weak scaling, no collective on the data
path); value = all ranks' tokens / the max over ranks of the device time.

--impl reference times the CPU oracle (oracle/) on the host cores, on the
same workload, metric and units: each step is a bounded sample of it.
"""
from __future__ import annotations

import argparse
import json
import os
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402
import torch  # noqa: E402

METRIC = "MoE-layer tokens/s (decode, prefill) and % of HBM/tensor/host-link roofline"
UNIT = "tokens/s"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


class ClockSampler:
    """nvidia-smi clock / throttle-reason samples during the timed region."""
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index):
        self.dev = device_index
        self.proc = None

    def start(self):
        try:
            self.proc = subprocess.Popen(["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                                          "-lms", "200", "-i", str(self.dev)], stdout=subprocess.PIPE,
                                         stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
            out, _ = self.proc.communicate()
        sm, mx, reasons = [], [], set()
        names = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")
        for line in out.strip().splitlines():
            f = [v.strip() for v in line.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                mx.append(float(f[2]))
            except ValueError:
                continue
            for n, v in zip(names, f[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        if not sm:
            return None
        return {"sm_mhz": float(np.median(sm)), "sm_max_mhz": float(max(mx)), "reasons": sorted(reasons),
                "samples": len(sm)}


def dist_setup(n_gpus):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        backend = "nccl" if torch.cuda.is_available() else "gloo"
        if backend == "nccl":
            torch.cuda.set_device(local)
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
    return world, rank, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(v, world, device):
    if world == 1:
        return v
    import torch.distributed as dist
    t = torch.tensor([v], dtype=torch.float64, device=device if dist.get_backend() == "nccl" else "cpu")
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def sum_over_ranks(v, world, device):
    if world == 1:
        return v
    import torch.distributed as dist
    t = torch.tensor([v], dtype=torch.float64, device=device if dist.get_backend() == "nccl" else "cpu")
    dist.all_reduce(t, op=dist.ReduceOp.SUM)
    return float(t.item())


# --------------------------------------------------------------------------
# workload inputs
# --------------------------------------------------------------------------
def decode_inputs(wl, rank, device):
    """Per batch size T: 64 steps of hidden states [T, d] (bf16, device) and
    the Zipf(1.1) router log-bias [E] (fp32, device)."""
    import ftgen
    bias = torch.as_tensor(ftgen.zipf_log_bias(wl.E, wl.extra["zipf_s"], wl.seed("zipf"))).to(device)
    xs = {}
    for T in wl.batches:
        xs[T] = [ftgen.hidden(T, wl.d, wl.wtype, wl.seed("bench", rank, T, s)).to(device) for s in range(wl.steps)]
    return xs, bias


def run_step(h, xs, bias, ys):
    import sparse_moe_expert_topk_b200 as ft
    ft.ft_moe_reset_cache(h.ctx)
    for T, seq in xs.items():
        y = ys[T]
        for x in seq:
            ft.ft_moe_layer_forward(h.ctx, 0, ft.FT_DECODE, x, T, bias, 0, y)


def run_step_e2e(h, xs_host, bias, y_host):
    """Same step through the C ABI's host-buffer call: every call has the
    library copy its hidden states from pinned host memory to the device and
    its output back to pinned host memory."""
    import sparse_moe_expert_topk_b200 as ft
    ft.ft_moe_reset_cache(h.ctx)
    for T, seq in xs_host.items():
        for i, xh in enumerate(seq):
            ft.ft_moe_layer_forward_host(h.ctx, 0, ft.FT_DECODE, xh, T, bias, 0, y_host[T][i])


# --------------------------------------------------------------------------
# roofline from the per-kernel profile
# --------------------------------------------------------------------------
KERNEL_SOURCES = {"gemv": "sparse_moe_expert_topk_b200/csrc/k_gemv_mma.cu",
                  "gemm_tc": "sparse_moe_expert_topk_b200/csrc/k_gemm_tc.cu",
                  "route": "sparse_moe_expert_topk_b200/csrc/k_route.cu",
                  "lookup": "sparse_moe_expert_topk_b200/csrc/k_lookup.cu",
                  "combine": "sparse_moe_expert_topk_b200/csrc/k_expert.cu"}


def _source_sha(kernel_name):
    import hashlib
    key = next((k for k in KERNEL_SOURCES if kernel_name.startswith(k)), None)
    if key is None:
        return None
    with open(os.path.join(ROOT, KERNEL_SOURCES[key]), "rb") as f:
        return hashlib.sha1(f.read()).hexdigest()[:12]


def ncu_traffic(kernel_name, launches_per_step):
    """DRAM bytes per launch of `kernel_name` from the committed ncu summary,
    or None if there is none or the kernel source changed since."""
    p = os.path.join(ROOT, "profiles", "ncu_traffic.json")
    if not os.path.exists(p):
        return None
    with open(p) as f:
        d = json.load(f)
    e = d.get(kernel_name)
    if not e or e.get("source_sha") != _source_sha(kernel_name):
        return None
    return e.get("dram_bytes_per_launch")


def roofline(prof, peaks, peak_kind, link_gbs, zc_gbs=None):
    """Per-kernel roofline rows from the library's CUDA-event profile, and the
    dominant row (the largest summed event time). Each row divides its
    algorithmic bytes (or flops) by its own event window:
    * HBM-resident work (hit GEMV, routing, combine, the prefill GEMMs below
      the ridge) against the measured HBM peak; a GEMM above the ridge against
      the bf16 tensor peak;
    * the copy engine's staging copies (events on the copy stream around each
      call's copies) against the H2D copy rate measured in the same run;
    * the staged class, whose window opens with its first copy and closes
      when its last expert is computed, against the same H2D rate;
    * the streamed class, which reads its weights zero-copy over the host
      link, against the zero-copy read rate measured in the same run."""
    zc = zc_gbs if zc_gbs else link_gbs
    rows = {}
    for name, r in prof.items():
        if r["ms"] <= 0:
            continue
        gbs = r["bytes"] / (r["ms"] * 1e6)
        # the binding roof is the larger of the HBM time and the tensor time
        t_hbm = r["bytes"] / (peaks["hbm_gbs"] * 1e9)
        t_tc = r["flops"] / (peaks["bf16_tflops"] * 1e12)
        src = peak_kind
        if name.startswith("gemm_tc") and t_tc > t_hbm:
            bound, peak, unit, ach = "tensor", peaks["bf16_tflops"], "TFLOP/s", r["flops"] / (r["ms"] * 1e9)
        elif name.endswith("streamed"):
            bound, peak, unit, ach = "host_link", zc, "GB/s", gbs
            src = "measured zero-copy read GB/s, this run"
        elif name.endswith("staged") or name.startswith("h2d_"):
            bound, peak, unit, ach = "host_link", link_gbs, "GB/s", gbs
            src = "measured H2D copy-engine GB/s, this run"
        else:
            bound, peak, unit, ach = "hbm", peaks["hbm_gbs"], "GB/s", gbs
        rows[name] = {"bound": bound, "achieved": round(ach, 2), "peak": round(peak, 2), "unit": unit,
                      "frac": round(ach / peak, 4) if peak else None, "ms_total": round(r["ms"], 3),
                      "launches": int(r["launches"]), "bytes_per_launch": r["bytes"] / max(r["launches"], 1),
                      "peak_source": src}
    tot = sum(v["ms_total"] for v in rows.values()) or 1.0
    for v in rows.values():
        v["share"] = round(v["ms_total"] / tot, 4)
    dom = max(rows, key=lambda k: rows[k]["ms_total"]) if rows else None
    out = None
    if dom:
        v = rows[dom]
        out = {"kernel": dom, "bound": v["bound"], "achieved": v["achieved"], "peak": v["peak"], "unit": v["unit"],
               "frac": v["frac"], "traffic": ncu_traffic(dom, v["launches"]), "peak_source": v["peak_source"],
               "algorithmic_bytes_per_launch": round(v["bytes_per_launch"])}
    return out, rows


# --------------------------------------------------------------------------
# CPU oracle timing (baseline and reference arm)
# --------------------------------------------------------------------------
def oracle_sample(wl, blob_of, seconds, rank=0):
    """Run the C++ oracle (oracle/moe_oracle.cpp: routing, the shared LRU with
    q*, and the per-token SwiGLU experts, one thread per token) over the
    workload's decode calls, in trace order, until `seconds` of oracle work
    have elapsed (the generation of expert blobs on first use is not
    counted). Returns (tokens, elapsed_s, calls, threads): threads = the most
    threads one call ran at once."""
    import ftgen
    from oracle import cpp
    bias = ftgen.zipf_log_bias(wl.E, wl.extra["zipf_s"], wl.seed("zipf")).astype(np.float64)
    wr = ftgen.router_weight(wl.E, wl.d, wl.wtype, wl.seed("router", 0)).float().numpy()
    cache = cpp.Cache(1, wl.E, wl.cache_slots, wl.bp_mbps, wl.bh_mbps)
    cores = os.cpu_count() or 1
    blobs = [None] * wl.E
    unused = np.zeros(16, np.uint8)  # stands for experts the call does not route to (never read)
    tokens = calls = threads = 0
    el = 0.0
    for T in wl.batches:
        for s in range(wl.steps):
            x = ftgen.hidden(T, wl.d, wl.wtype, wl.seed("bench", rank, T, s)).float().numpy()
            t0 = time.perf_counter()
            ids, _ = cpp.route(x, wr, bias, wl.k)
            cache.forward(0, 0, np.bincount(ids.ravel(), minlength=wl.E))
            el += time.perf_counter() - t0
            for e in np.unique(ids):
                if blobs[e] is None:
                    blobs[e] = blob_of(int(e))
            n = min(T, cores)
            t0 = time.perf_counter()
            cpp.layer_forward(x, wr, bias, wl.k, [b if b is not None else unused for b in blobs], wl.wtype, wl.d,
                              wl.d_ff, threads=n)
            el += time.perf_counter() - t0
            tokens += T
            calls += 1
            threads = max(threads, n)
            if el >= seconds:
                cache.close()
                return tokens, el, calls, threads
    cache.close()
    return tokens, el, calls, threads


def cpu_blob_source(wl):
    """Expert blobs generated on the CPU from the workload's seeds (same
    recipe as the pool the GPU arm reads)."""
    import ftgen
    cache = {}

    def blob(e):
        if e not in cache:
            cache[e] = ftgen.expert_blob(wl.d, wl.d_ff, wl.wtype, wl.seed("expert", 0, e)).numpy()
        return cache[e]
    return blob


def decode_config(wl, world):
    """The `config` object of the decode line, shared by both arms."""
    return {"workload": "single-layer BF16 decode, E=256 top-6 d=4096 d_ff=1536, 37% cache (94 slots), "
                        "LRU, B_P:B_H=52.7:77.3, 64-step trace at batch 1/4/16 from a cold cache",
            "tokens_per_step": wl.steps * sum(wl.batches), "layer_calls_per_step": wl.steps * len(wl.batches),
            "l2": "inputs larger than L2 (9.7 GB pinned pool, 3.5 GB slot pool)",
            "parallelism": f"replicas x{world}"}


def run_reference(args, wl, world, rank):
    if rank != 0:
        return 0
    blob = cpu_blob_source(wl)
    per_step_s = 10.0
    for _ in range(args.warmup):
        oracle_sample(wl, blob, 0.5)
    tok = el = 0.0
    calls = cores = 0
    for _ in range(args.steps):
        t, e, c, n = oracle_sample(wl, blob, per_step_s)
        tok += t
        el += e
        calls += c
        cores = max(cores, n)
    value = tok / el
    line = {"impl": "reference", "metric": METRIC, "value": round(value, 4), "unit": UNIT, "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(1e3 * el / args.steps, 3),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": decode_config(wl, world),
            "cpu_baseline": {"value": round(value, 4), "unit": UNIT, "cores": cores, "kind": "oracle",
                             "sample": f"first {calls} decode calls of the trace in {args.steps} steps of "
                                       f"~{per_step_s:.0f} s each (C++ oracle: routing, shared LRU with q*, "
                                       f"per-token SwiGLU experts, one thread per token)"},
            "e2e": {"value": round(value, 4), "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0



# --------------------------------------------------------------------------
# secondary workloads (not the default line): single-layer prefill, 43-layer
# NVFP4 decode trace
# --------------------------------------------------------------------------
def _timed(stream, device, fn, steps):
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize(device)
    e0.record(stream)
    for _ in range(steps):
        fn()
    e1.record(stream)
    torch.cuda.synchronize(device)
    return e0.elapsed_time(e1) / steps


def run_secondary(args, wl, world, rank, local):
    import ftgen
    import sparse_moe_expert_topk_b200 as ft
    from ftgen.ctx import Harness
    device = torch.device("cuda", local)
    torch.cuda.set_device(device)
    peaks, peak_kind = load_peaks()
    out = {"metric": METRIC, "unit": UNIT, "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
           "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "data": "synthetic"}
    if wl.name == "prefill_bf16":
        T = wl.batches[0]
        T_big = 16384  # the extra hot point, where the tensor roof binds
        h = Harness(wl, max_tokens=T_big, device=local)
        x = ftgen.hidden(T, wl.d, wl.wtype, wl.seed("bench", rank)).to(device)
        y = torch.empty_like(x)

        def call():
            ft.ft_moe_layer_forward(h.ctx, 0, ft.FT_PREFILL, x, T, None, 0, y)

        def cold():
            ft.ft_moe_reset_cache(h.ctx)
            call()
        for _ in range(args.warmup):
            cold()
        ms_cold = _timed(h.stream, device, cold, args.steps)
        ms_hot = _timed(h.stream, device, call, args.steps)
        ft.ft_moe_profile(h.ctx, True)
        call()
        prof = ft.ft_moe_profile_read(h.ctx)
        ft.ft_moe_profile(h.ctx, False)
        # hot at T = 16384 (every expert resident from the calls above)
        xb = ftgen.hidden(T_big, wl.d, wl.wtype, wl.seed("bench-big", rank)).to(device)
        yb = torch.empty_like(xb)

        def call_big():
            ft.ft_moe_layer_forward(h.ctx, 0, ft.FT_PREFILL, xb, T_big, None, 0, yb)
        for _ in range(args.warmup):
            call_big()
        ms_big = _timed(h.stream, device, call_big, args.steps)
        ft.ft_moe_profile(h.ctx, True)
        call_big()
        prof_big = ft.ft_moe_profile_read(h.ctx)
        ft.ft_moe_profile(h.ctx, False)
        h2d, zc = ft.ft_moe_probe_link(h.ctx, 1 << 30)
        roof, rows = roofline(prof, peaks, peak_kind, h2d, zc)
        roof_big, rows_big = roofline(prof_big, peaks, peak_kind, h2d, zc)
        flops_big = 2.0 * T_big * wl.k * 3 * wl.d * wl.d_ff
        h.close()
        link_bytes = wl.E * wl.slot_bytes
        out.update(value=round(T / (ms_hot / 1e3), 1), ms_per_step=round(ms_hot, 3), dtype="bf16",
                   config={"workload": f"single-layer BF16 prefill, T={T}, E=256 top-6 d=4096 d_ff=1536, b=0"},
                   hot={"tokens_per_s": round(T / (ms_hot / 1e3), 1), "ms": round(ms_hot, 3)},
                   cold={"tokens_per_s": round(T / (ms_cold / 1e3), 1), "ms": round(ms_cold, 3),
                         "link_gbs": round(link_bytes / (ms_cold * 1e6), 2),
                         "link_frac": round(link_bytes / (ms_cold * 1e6) / h2d, 4)},
                   hot_16384={"tokens_per_s": round(T_big / (ms_big / 1e3), 1), "ms": round(ms_big, 3),
                              "layer_tflops": round(flops_big / (ms_big * 1e9), 1),
                              "layer_tensor_frac": round(flops_big / (ms_big * 1e9) / peaks["bf16_tflops"], 4),
                              "roofline": roof_big, "kernels": rows_big},
                   host_link={"h2d_copy_gbs": round(h2d, 2), "zero_copy_read_gbs": round(zc, 2)},
                   roofline=roof, kernels=rows)
    else:  # trace_nvfp4: 43 layers, Markov routing realised as a per-token bias
        import dataclasses
        # FT_TRACE_LAYERS < 43 runs the same per-layer shapes on a smaller pool
        # (a few GB, for profiler captures); capacity stays 37% of the pool
        L = min(wl.L, int(os.environ.get("FT_TRACE_LAYERS", wl.L)))
        if L != wl.L:
            wl = dataclasses.replace(wl, L=L, cache_slots=int(0.37 * L * wl.E))
        steps = min(wl.steps, int(os.environ.get("FT_TRACE_STEPS", wl.steps)))
        h = Harness(wl, max_tokens=1, device=local)
        prefetch = os.environ.get("FT_PREFETCH", "0") == "1"  # the decode prefetch (opt-in)
        ft.ft_moe_set_prefetch(h.ctx, prefetch)
        traces = [ftgen.markov_trace(steps, 1, wl.E, wl.k, wl.extra["p_reuse"], wl.extra["zipf_s"],
                                     wl.seed("trace", rank, l)) for l in range(L)]
        zb = [ftgen.zipf_log_bias(wl.E, wl.extra["zipf_s"], wl.seed("pi", l)) for l in range(L)]
        xs = [[ftgen.hidden(1, wl.d, wl.wtype, wl.seed("x", rank, st, l)).to(device) for l in range(L)]
              for st in range(steps)]
        bs = [[torch.as_tensor(ftgen.trace_bias(traces[l][st], zb[l], wl.extra["beta"])).to(device)
               for l in range(L)] for st in range(steps)]
        y = torch.empty(1, wl.d, dtype=torch.bfloat16, device=device)

        def trace():
            ft.ft_moe_reset_cache(h.ctx)
            for st in range(steps):
                for l in range(L):
                    ft.ft_moe_layer_forward(h.ctx, l, ft.FT_DECODE, xs[st][l], 1, bs[st][l], 1, y)
        trace()
        ms = _timed(h.stream, device, trace, 1)
        stt = h.stats()
        ft.ft_moe_profile(h.ctx, True)
        trace()
        prof = ft.ft_moe_profile_read(h.ctx)
        ft.ft_moe_profile(h.ctx, False)
        h2d, zc = ft.ft_moe_probe_link(h.ctx, 1 << 30)
        roof, rows = roofline(prof, peaks, peak_kind, h2d, zc)
        h.close()
        out.update(value=round(steps / (ms / 1e3), 2), ms_per_step=round(ms / steps, 4), dtype="nvfp4",
                   config={"workload": f"{L}-layer NVFP4 decode trace, batch 1, {steps} steps, Markov p=0.8 + "
                                       f"Zipf(1.1), shared LRU at 37% ({wl.cache_slots} slots), 52.7:77.3"
                                       + (", decode prefetch on" if prefetch else "")},
                   tokens_per_s_all_layers=round(steps / (ms / 1e3), 2),
                   layer_calls_per_s=round(steps * L / (ms / 1e3), 1),
                   miss_rate=round(stt["misses"] / max(stt["lookups"], 1), 4),
                   cache={k: stt[k] for k in ("lookups", "hits", "misses", "staged", "streamed", "prefetched")},
                   host_link={"h2d_copy_gbs": round(h2d, 2), "zero_copy_read_gbs": round(zc, 2)},
                   roofline=roof, kernels=rows)
    if rank == 0:
        print(json.dumps(out), flush=True)
    return 0

def host_mem_available():
    """Bytes of host memory the kernel reports available (None if unknown)."""
    try:
        with open("/proc/meminfo") as f:
            for line in f:
                if line.startswith("MemAvailable:"):
                    return int(line.split()[1]) * 1024
    except OSError:
        pass
    return None


def mixed_sweep(wl, caps, profiles, steps, warmup, rank, local, prefetch=False):
    """The 43-layer mixed NVFP4 workload on one context: for every cache
    capacity and B_P:B_H profile, a cold prefill of T = 8192 tokens through
    every layer (layer-ahead double buffer), then `steps` decode steps split
    in equal blocks at batch 1, 2, 4 and 8 with Markov routing. The slot pool
    is resized between capacities (the host pool is filled once). prefetch:
    the opt-in decode prefetch (layer l+1's experts of its previous decode
    call staged while layer l computes). Returns (rows, host_link, clocks)."""
    import dataclasses
    import ftgen
    import sparse_moe_expert_topk_b200 as ft
    from ftgen.ctx import Harness
    device = torch.device("cuda", local)
    torch.cuda.set_device(device)
    L, E, k, d = wl.L, wl.E, wl.k, wl.d
    ex = wl.extra
    steps -= steps % len(wl.batches)
    per_batch = steps // len(wl.batches)
    Bmax = max(wl.batches)
    T_pf = ex["prefill_T"]
    h = Harness(dataclasses.replace(wl, cache_slots=caps[0]), max_tokens=T_pf, device=local)
    try:
        ft.ft_moe_set_prefetch(h.ctx, prefetch)
        # inputs: one prefill block reused by every layer (each layer routes it
        # with its own router), decode activations and per-token trace biases
        g = torch.Generator(device=device)
        g.manual_seed(ftgen.subseed("mixed-x", rank))
        x_pf = torch.randn(T_pf, d, generator=g, device=device).to(torch.bfloat16)
        y_pf = torch.empty_like(x_pf)
        x_dec = torch.randn(steps, L, Bmax, d, generator=g, device=device).to(torch.bfloat16)
        y_dec = torch.empty(Bmax, d, dtype=torch.bfloat16, device=device)
        zb = [ftgen.zipf_log_bias(E, ex["zipf_s"], wl.seed("pi", l)) for l in range(L)]
        bias = np.empty((steps, L, Bmax, E), np.float32)
        for l in range(L):
            tr = ftgen.markov_trace(steps, Bmax, E, k, ex["p_reuse"], ex["zipf_s"], wl.seed("trace", rank, l))
            for st in range(steps):
                bias[st, l] = ftgen.trace_bias(tr[st], zb[l], ex["beta"])
        bias = torch.from_numpy(bias).to(device)
        h2d, zc = ft.ft_moe_probe_link(h.ctx, 1 << 30)
        stream = h.stream
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)

        def prefill():
            for l in range(L):
                ft.ft_moe_layer_forward(h.ctx, l, ft.FT_PREFILL, x_pf, T_pf, None, 0, y_pf)

        def decode(st0, n, B):
            for st in range(st0, st0 + n):
                for l in range(L):
                    ft.ft_moe_layer_forward(h.ctx, l, ft.FT_DECODE, x_dec[st, l, :B], B, bias[st, l, :B], 1,
                                            y_dec[:B])

        def timed(fn, *a):
            torch.cuda.synchronize(device)
            e0.record(stream)
            fn(*a)
            e1.record(stream)
            torch.cuda.synchronize(device)
            return e0.elapsed_time(e1)

        # warm-up on the first point (kernels, events, pages)
        ft.ft_set_bandwidths(h.ctx, *profiles[-1])
        for _ in range(max(1, warmup)):
            ft.ft_moe_reset_cache(h.ctx)
            prefill()
            decode(0, min(4, per_batch), 1)
        sweep = []
        sampler = ClockSampler(local)
        sampler.start()
        for C in caps:
            ft.ft_moe_resize_cache(h.ctx, C)
            for bp, bh in profiles:
                ft.ft_moe_reset_cache(h.ctx)
                ft.ft_set_bandwidths(h.ctx, bp, bh)
                ms_pf = timed(prefill)
                st_pf = h.stats()
                pf_link = st_pf["bytes_h2d"] / (ms_pf * 1e6)
                row = {"cache_slots": C, "cache_frac": round(C / (L * E), 3),
                       "bp_bh": f"{bp / 1000:.1f}:{bh / 1000:.1f}",
                       "prefill": {"tokens_per_s": round(T_pf / (ms_pf / 1e3), 1), "ms_43_layers": round(ms_pf, 1),
                                   "link_gbs": round(pf_link, 2), "link_frac": round(pf_link / h2d, 4)},
                       "decode": {}}
                tok = 0
                ms_dec = 0.0
                s_all0 = h.stats()
                for i, B in enumerate(wl.batches):
                    s0 = h.stats()
                    ms = timed(decode, i * per_batch, per_batch, B)
                    s1 = h.stats()
                    look = s1["lookups"] - s0["lookups"]
                    miss = s1["misses"] - s0["misses"]
                    link = (s1["bytes_h2d"] - s0["bytes_h2d"]) + (s1["bytes_zero_copy"] - s0["bytes_zero_copy"])
                    row["decode"][str(B)] = {"tokens_per_s": round(per_batch * B / (ms / 1e3), 2),
                                             "ms_per_step": round(ms / per_batch, 3),
                                             "miss_rate": round(miss / max(look, 1), 4),
                                             "qstar_staged": s1["staged"] - s0["staged"],
                                             "streamed": s1["streamed"] - s0["streamed"],
                                             "link_gbs": round(link / (ms * 1e6), 2),
                                             "link_frac": round(link / (ms * 1e6) / h2d, 4)}
                    tok += per_batch * B
                    ms_dec += ms
                s_all1 = h.stats()
                look = s_all1["lookups"] - s_all0["lookups"]
                row["decode_tokens_per_s"] = round(tok / (ms_dec / 1e3), 2)
                row["decode_steps"] = steps
                row["decode_miss_rate"] = round((s_all1["misses"] - s_all0["misses"]) / max(look, 1), 4)
                sweep.append(row)
        clocks = sampler.stop()
    finally:
        h.close()
    return sweep, {"h2d_copy_gbs": round(h2d, 2), "zero_copy_read_gbs": round(zc, 2)}, clocks


def mixed_point(rank, local, prefetch=False):
    """The largest single-GPU workload at its headline point, for the default
    line: 43-layer mixed NVFP4 at 37% capacity and B_P:B_H = 52.7:77.3, cold
    prefill of 8192 tokens, then the full 1024 decode steps at batch 1/2/4/8.
    Skipped (with the reason) when the host cannot hold the 117 GB pool."""
    import ftgen
    wl = ftgen.workload("mixed_nvfp4")
    need = wl.L * wl.E * wl.slot_bytes
    avail = host_mem_available()
    if avail is not None and avail < need + (24 << 30):
        return {"skipped": f"host memory: {avail / 1e9:.0f} GB available, the pinned pool needs {need / 1e9:.0f} GB"}
    t0 = time.perf_counter()
    try:
        rows, link, clocks = mixed_sweep(wl, [int(0.37 * wl.L * wl.E)], [(52700, 77300)], wl.steps, 1, rank, local,
                                         prefetch)
    except Exception as e:  # the default line must still be printed
        return {"skipped": f"{type(e).__name__}: {e}"}
    r = rows[0]
    return {"workload": f"43-layer mixed NVFP4, E=256 top-6 d=4096 d_ff=1536 ({need / 1e9:.1f} GB pinned pool): cold "
                        f"prefill T={wl.extra['prefill_T']} through all layers, then {r['decode_steps']} decode steps "
                        f"at batch 1/2/4/8, Markov p=0.8 + Zipf(1.1), 37% cache ({r['cache_slots']} slots), 52.7:77.3"
                        + (", decode prefetch on" if prefetch else ""),
            "decode_tokens_per_s": r["decode_tokens_per_s"], "decode_miss_rate": r["decode_miss_rate"],
            "prefill": r["prefill"], "decode": r["decode"], "host_link": link, "clocks": clocks,
            "wall_s": round(time.perf_counter() - t0, 1)}


def run_mixed(args, wl, world, rank, local):
    """--workload mixed_nvfp4: the sweep over every capacity {10, 20, 37,
    60}% x profile {11.8:47.5, 52.7:77.3} (FT_MIXED_STEPS decode steps per
    point, default 256 of the 1024)."""
    L, E = wl.L, wl.E
    ex = wl.extra
    steps = min(wl.steps, int(os.environ.get("FT_MIXED_STEPS", 256)))
    caps = [int(f * L * E) for f in ex["cache_fracs"]]
    prefetch = os.environ.get("FT_PREFETCH", "0") == "1"  # the decode prefetch (opt-in)
    sweep, link, clocks = mixed_sweep(wl, caps, list(ex["profiles"]), steps, max(1, args.warmup - 2), rank, local,
                                      prefetch)
    main_pt = next(r for r in sweep if r["cache_slots"] == int(0.37 * L * E) and r["bp_bh"] == "52.7:77.3")
    steps -= steps % len(wl.batches)
    out = {"metric": METRIC, "value": main_pt["decode_tokens_per_s"], "unit": UNIT, "n_gpus": world,
           "steps": steps, "warmup": args.warmup, "ms_per_step": round(1e3 * sum(wl.batches) / len(wl.batches)
                                                                      / main_pt["decode_tokens_per_s"], 3),
           "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "nvfp4", "data": "synthetic",
           "config": {"workload": f"43-layer mixed NVFP4: cold prefill T={ex['prefill_T']} then {steps} decode steps "
                                  f"at batch 1/2/4/8 ({steps // len(wl.batches)} each), Markov p=0.8 + Zipf(1.1); "
                                  f"value at 37% and 52.7:77.3",
                      "pool_gb": round(L * E * wl.slot_bytes / 1e9, 1)},
           "host_link": link, "sweep": sweep, "clocks": clocks}
    if rank == 0:
        print(json.dumps(out), flush=True)
    return 0


# --------------------------------------------------------------------------
# kernel microbenchmarks, one JSON line per weight type, per-kernel CUDA-event
# times from the library's profiler; for the roofline fractions of single
# kernels and for small ncu captures, not a bench line.
#   hit_gemv, prefill_gemm: every expert of one layer resident in its slot,
#     so the expert kernels read HBM only;
#   stream_gemv: B_P = 0, so q* = 0 and every routed expert is streamed from
#     the pinned pool (the cache stays empty): the streamed class alone on the
#     host link, against the zero-copy read rate measured in the same run.
def run_kernels(args, rank, local):
    import dataclasses

    import sparse_moe_expert_topk_b200 as ft
    import ftgen
    from ftgen.ctx import Harness
    device = torch.device("cuda", local)
    torch.cuda.set_device(device)
    base = ftgen.workload("prefill_bf16" if args.workload == "prefill_gemm" else "decode_bf16")
    wts = {"bf16": ftgen.W_BF16, "nvfp4": ftgen.W_NVFP4}
    for wname in args.wtypes.split(","):
        E = args.experts
        wl = dataclasses.replace(base, name=f"{args.workload}_{wname}", wtype=wts[wname], E=E, cache_slots=2 * E)
        sizes = [int(t) for t in args.tokens.split(",")]
        h = Harness(wl, max_tokens=max(max(sizes), 512), device=local)
        x0 = ftgen.hidden(512, wl.d, wl.wtype, 1).to(device)
        y0 = torch.empty_like(x0)
        link = None
        if args.workload == "stream_gemv":
            ft.ft_set_bandwidths(h.ctx, 0, 77300)
            h2d_gbs, zc_gbs = ft.ft_moe_probe_link(h.ctx, 1 << 30)
            link = {"h2d_copy_gbs": round(h2d_gbs, 2), "zero_copy_read_gbs": round(zc_gbs, 2)}
        else:
            ft.ft_moe_layer_forward(h.ctx, 0, ft.FT_PREFILL, x0, 512, None, 0, y0)  # the whole layer into its slots
        torch.cuda.synchronize(device)
        decode = args.workload != "prefill_gemm"
        mode = ft.FT_DECODE if decode else ft.FT_PREFILL
        bias = torch.as_tensor(ftgen.zipf_log_bias(E, 1.1, wl.seed("zipf"))).to(device) if decode else None
        out = {}
        for T in sizes:
            n_in = args.calls if decode else 1
            xs = [ftgen.hidden(T, wl.d, wl.wtype, 100 + i).to(device) for i in range(n_in)]
            yT = torch.empty(T, wl.d, dtype=xs[0].dtype, device=device)
            for i in range(args.warmup):
                ft.ft_moe_layer_forward(h.ctx, 0, mode, xs[i % n_in], T, bias, 0, yT)
            torch.cuda.synchronize(device)
            ft.ft_moe_profile(h.ctx, True)
            for i in range(args.calls):
                ft.ft_moe_layer_forward(h.ctx, 0, mode, xs[i % n_in], T, bias, 0, yT)
            prof = ft.ft_moe_profile_read(h.ctx)
            ft.ft_moe_profile(h.ctx, False)
            torch.cuda.synchronize(device)
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(h.stream)
            for i in range(args.calls):
                ft.ft_moe_layer_forward(h.ctx, 0, mode, xs[i % n_in], T, bias, 0, yT)
            e1.record(h.stream)
            torch.cuda.synchronize(device)
            r = {k: {"us_per_launch": round(v["ms"] * 1e3 / max(v["launches"], 1), 2),
                     "GBps": round(v["bytes"] / max(v["ms"], 1e-9) / 1e6, 1),
                     "TFLOPs": round(v["flops"] / max(v["ms"], 1e-9) / 1e9, 1),
                     "MB_per_launch": round(v["bytes"] / max(v["launches"], 1) / 1e6, 2)} for k, v in prof.items()}
            r["call_us"] = round(e0.elapsed_time(e1) * 1e3 / args.calls, 2)
            r["misses"] = h.stats()["misses"]
            if link and "gemv_streamed" in r:
                r["gemv_streamed"]["frac_of_zero_copy"] = round(r["gemv_streamed"]["GBps"] / link["zero_copy_read_gbs"], 4)
            out[str(T)] = r
        h.close()
        if rank == 0:
            print(json.dumps({"workload": args.workload, "wtype": wname, "experts": E, "d": wl.d, "d_ff": wl.d_ff,
                              "top_k": wl.k, "calls": args.calls, "host_link": link, "kernels": out}), flush=True)
    return 0


# --------------------------------------------------------------------------
def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=3)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default="decode_bf16")
    ap.add_argument("--cpu-seconds", type=float, default=15.0)
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-mixed", action="store_true", help="skip the 43-layer mixed NVFP4 leg of the default line")
    ap.add_argument("--profile-only", action="store_true", help="one warm-up and one profiled step (for ncu)")
    km = ap.add_argument_group("kernel microbenchmarks (--workload hit_gemv | stream_gemv | prefill_gemm)")
    km.add_argument("--wtypes", default="bf16,nvfp4", help="weight types, comma-separated")
    km.add_argument("--experts", type=int, default=256, help="experts of the resident layer")
    km.add_argument("--tokens", default="1,4,16", help="tokens per call, comma-separated")
    km.add_argument("--calls", type=int, default=48, help="profiled calls per size")
    args = ap.parse_args()
    if args.warmup < 3 and not args.profile_only:
        raise SystemExit("--warmup must be >= 3")

    if args.workload in ("hit_gemv", "stream_gemv", "prefill_gemm"):
        if args.gpus != 1 or args.impl != "ours":
            raise SystemExit("kernel microbenchmarks run on one GPU, our implementation only")
        return run_kernels(args, 0, 0)
    import ftgen
    wl = ftgen.workload(args.workload)
    world, rank, local = dist_setup(args.gpus)
    if args.workload in ("prefill_bf16", "trace_nvfp4") and args.impl == "ours":
        return run_secondary(args, wl, world, rank, local)
    if args.workload == "mixed_nvfp4" and args.impl == "ours":
        return run_mixed(args, wl, world, rank, local)
    if args.workload != "decode_bf16":
        raise SystemExit("workloads: decode_bf16 (default), prefill_bf16, trace_nvfp4, mixed_nvfp4; "
                         "kernel microbenchmarks: hit_gemv, stream_gemv, prefill_gemm")
    if args.impl == "reference":
        r = run_reference(args, wl, world, rank)
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()
        return r

    import sparse_moe_expert_topk_b200 as ft
    from ftgen.ctx import Harness
    if not os.path.exists(ft.LIB_PATH):
        from sparse_moe_expert_topk_b200 import build
        build.build()
    device = torch.device("cuda", local)
    torch.cuda.set_device(device)
    h = Harness(wl, max_tokens=max(wl.batches), device=local)
    xs, bias = decode_inputs(wl, rank, device)
    ys = {T: torch.empty(T, wl.d, dtype=torch.bfloat16, device=device) for T in wl.batches}
    tokens_per_step = wl.steps * sum(wl.batches)
    stream = h.stream

    if args.profile_only:
        run_step(h, xs, bias, ys)
        ft.ft_moe_profile(h.ctx, True)
        run_step(h, xs, bias, ys)
        prof = ft.ft_moe_profile_read(h.ctx)
        if rank == 0:
            print(json.dumps({k: {kk: round(vv, 4) if isinstance(vv, float) else vv for kk, vv in v.items()}
                              for k, v in prof.items()}), flush=True)
        h.close()
        return 0

    for _ in range(args.warmup):
        run_step(h, xs, bias, ys)
    launches0 = ft.ft_cache_stats(h.ctx)["kernel_launches"]
    barrier(world)
    torch.cuda.synchronize(device)
    sampler = ClockSampler(local)
    sampler.start()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(args.steps):
        run_step(h, xs, bias, ys)
    e1.record(stream)
    torch.cuda.synchronize(device)
    clocks = sampler.stop()
    barrier(world)
    ms = e0.elapsed_time(e1)
    st = ft.ft_cache_stats(h.ctx)
    launches = (st["kernel_launches"] - launches0) / args.steps
    # every miss byte crosses the host link once: staged blobs by the copy
    # engine, streamed blobs by the GEMV's zero-copy reads. A step starts from
    # a cold cache (the reset zeroes the counters), so the counters after the
    # last timed step are one step's bytes; every step replays the same trace.
    link_bytes = st["bytes_h2d"] + st["bytes_zero_copy"]
    ms_max = max_over_ranks(ms, world, device)
    total_tokens = sum_over_ranks(tokens_per_step * args.steps, world, device)
    value = total_tokens / (ms_max / 1e3)

    # per-kernel profile of one more step (events around every launch),
    # split by batch size
    ft.ft_moe_reset_cache(h.ctx)
    ft.ft_moe_profile(h.ctx, True)
    prof, by_batch = {}, {}
    half = {"lookups": 0, "misses": 0}  # second half of every 64-step batch block
    for T, seq in xs.items():
        for i, x in enumerate(seq):
            if i == len(seq) // 2:
                s_mid = ft.ft_cache_stats(h.ctx)
            ft.ft_moe_layer_forward(h.ctx, 0, ft.FT_DECODE, x, T, bias, 0, ys[T])
        s_end = ft.ft_cache_stats(h.ctx)
        for k in half:
            half[k] += s_end[k] - s_mid[k]
        pT = ft.ft_moe_profile_read(h.ctx)
        by_batch[T] = {k: {"ms": round(v["ms"], 3), "GBps": round(v["bytes"] / max(v["ms"], 1e-9) / 1e6, 1),
                           "launches": v["launches"]} for k, v in pT.items()}
        for k, v in pT.items():
            a = prof.setdefault(k, {"launches": 0, "ms": 0.0, "bytes": 0.0, "flops": 0.0})
            for f in a:
                a[f] += v[f]
    ft.ft_moe_profile(h.ctx, False)
    st1 = ft.ft_cache_stats(h.ctx)
    miss_rate = st1["misses"] / max(st1["lookups"], 1)

    # host link: copy engine and zero-copy kernel reads, 1 GiB
    h2d_gbs, zc_gbs = ft.ft_moe_probe_link(h.ctx, 1 << 30)
    peaks, peak_kind = load_peaks()
    roof, rows = roofline(prof, peaks, peak_kind, h2d_gbs, zc_gbs)

    # overlap: the step against its two legs run alone, each at its bound --
    # the expert kernel on HBM-resident weights (hit class, as profiled) and
    # the miss bytes over the host link at the measured copy-engine rate
    t_hit = prof["gemv_hit"]["ms"] if "gemv_hit" in prof else 0.0
    t_miss = link_bytes / (h2d_gbs * 1e6)
    t_step = ms_max / args.steps
    overlap = {"t_hit_only_ms": round(t_hit, 3), "t_miss_only_ms": round(t_miss, 3), "t_step_ms": round(t_step, 3),
               "overlap": round(max(t_hit, t_miss) / t_step, 4)}

    # end to end through the public call with host buffers
    e2e = None
    if not args.no_e2e:
        xs_host = {T: [x.cpu().pin_memory() for x in seq] for T, seq in xs.items()}
        y_host = {T: [torch.empty(T, wl.d, dtype=torch.bfloat16).pin_memory() for _ in seq] for T, seq in xs.items()}
        run_step_e2e(h, xs_host, bias, y_host)
        barrier(world)
        torch.cuda.synchronize(device)
        e0.record(stream)
        for _ in range(args.steps):
            run_step_e2e(h, xs_host, bias, y_host)
        e1.record(stream)
        torch.cuda.synchronize(device)
        ms_e2e = max_over_ranks(e0.elapsed_time(e1), world, device)
        io_bytes = tokens_per_step * wl.d * 2
        e2e = {"value": round(total_tokens / (ms_e2e / 1e3), 3), "unit": UNIT, "h2d_bytes_per_step": io_bytes,
               "d2h_bytes_per_step": io_bytes}

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        tok, el, calls, n_thr = oracle_sample(wl, lambda e: h.blob(0, e), args.cpu_seconds, rank)
        cpu = {"value": round(tok / el, 4), "unit": UNIT, "cores": n_thr, "kind": "oracle",
               "sample": f"first {calls} decode calls ({tok} tokens, batch 1 first) of the same trace and pool, "
                         f"{el:.1f} s of CPU work; C++ oracle, one thread per token (at most {n_thr} at once)"}

    h.close()
    del xs, ys
    torch.cuda.empty_cache()
    # the largest single-GPU workload (43-layer mixed NVFP4), one GPU only:
    # each rank of a multi-GPU run would pin its own 117 GB pool
    mixed = mixed_pf = None
    if world == 1 and not args.no_mixed:
        mixed = mixed_point(rank, local)
        # the same point with the decode prefetch: layer l+1's experts of its
        # previous decode call staged while layer l computes
        mixed_pf = mixed_point(rank, local, prefetch=True)
    if rank == 0:
        line = {
            "metric": METRIC, "value": round(value, 3), "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": round(ms_max / args.steps, 3), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": decode_config(wl, world),
            "miss_rate": round(miss_rate, 4),
            "miss_rate_second_half": round(half["misses"] / max(half["lookups"], 1), 4),
            "overlap": overlap,
            "cache": {k: st1[k] for k in ("lookups", "hits", "misses", "staged", "streamed")},
            "host_link": {"h2d_copy_gbs": round(h2d_gbs, 2), "zero_copy_read_gbs": round(zc_gbs, 2)},
            "link_step": {"bytes_per_step": int(link_bytes),
                          "achieved": round(link_bytes / (ms_max / args.steps) / 1e6, 2),
                          "peak": round(h2d_gbs, 2), "unit": "GB/s",
                          "frac": round(link_bytes / (ms_max / args.steps) / 1e6 / h2d_gbs, 4),
                          "what": "staged H2D copies plus streamed zero-copy reads over the whole timed step, "
                                  "against the measured copy-engine H2D bandwidth"},
            "roofline": roof, "kernels": rows, "kernels_by_batch": by_batch, "gpu_launches": int(round(launches * args.steps)),
            "gpu_launches_per_step": round(launches, 1), "clocks": clocks, "e2e": e2e, "cpu_baseline": cpu,
            "peaks": {"kind": peak_kind, "hbm_gbs": peaks["hbm_gbs"], "bf16_tflops": peaks["bf16_tflops"]},
            "mixed_nvfp4": mixed,
            "mixed_nvfp4_prefetch": mixed_pf,
        }
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
