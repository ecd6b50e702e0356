#!/usr/bin/env python
"""Benchmark of the R-SWA decode hot path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Headline workload: single-document bf16 decode -- batch 1, 10 heads, head dim
128, L_m = 2592 reference rows (10 pages x 256 vision tokens + 32 prompt
tokens), window n = 128, the timed steps ending at output T = 6144.  One
"step" decodes one output token: the fused append+decode kernel runs once for
each of R layer caches (R distinct caches, as in an R-layer decoder), so the
bytes one step touches exceed twice the L2 size and nothing is served from
L2 between steps.  Every cache is loaded straight at the step the run starts
from (rswa_load_packed), in the steady state T > n where the R-SWA cost per
step is constant; exactly K steps are timed.

value     : tokens/s through one attention layer = B * R * K / device time.
e2e       : the same through the public binding with HOST buffers: every step
            copies q, k, v of all R layers from pinned host memory, runs the
            step (a LayerStep built once with graph=True: one CUDA graph of the
            R launches) and copies the outputs back, all inside the timed
            region, after warm-up steps of the same loop.
roofline  : algorithmic bytes per launch (2 * rows * d * 2 bytes of K and V
            plus q, o, new k, v) / average launch time, against the measured
            HBM copy bandwidth.
configs   : (1 GPU) the same measurement for the ragged batch (64 sequences
            of 2-50 pages, ending at T = 6144) and the long-horizon run
            (batch 8, 50 pages, ending at T = 100000).
prefill   : the 32K teacher-forced masked prefill on the tensor cores.
vs_output_length: per-step latency against T for the R-SWA cache and for the
            same kernel over the full cache, single document to T = 6144 and
            long horizon to T = 100000 (the full cache further, to 1e6).

N > 1 GPUs (one process per GPU under torchrun) run independent replicas of
the headline workload (R-SWA shards by sequence with no exchange): value is
the sum of all ranks' tokens over the slowest rank's time.
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

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "R-SWA decode tokens/s and achieved HBM GB/s (% of B200 peak) vs output length"
FALLBACK_HBM_GBS = 6650.0

WORKLOADS = {
    "single_doc": dict(B=1, H=10, d=128, pages=[10], prompt=32, n=128, T=6144, dtype="bf16",
                       desc="single-document bf16 decode: batch 1, 10 heads, d=128, L_m=2592 "
                            "(10 pages x 256 + 32), n=128, outputs to T=6144"),
    "ragged": dict(B=64, H=10, d=128, pages=None, prompt=32, n=128, T=6144, dtype="bf16",
                   desc="ragged batched bf16 decode: 64 sequences, pages~U[2,50], "
                        "L_m=256*pages+32, 10 heads, d=128, n=128, outputs to T=6144"),
    "long": dict(B=8, H=10, d=128, pages=[50] * 8, prompt=32, n=128, T=100000, dtype="bf16",
                 desc="long-horizon bf16 decode: batch 8, L_m=12832, 10 heads, d=128, n=128, outputs to T=100000"),
}


PREFILL = dict(L=32768, L_m=12832, n=128, H=10, d=128, dtype="bf16",
               desc="teacher-forced masked prefill, bf16: packed 32768-token sequence, 10 heads, d=128, "
                    "L_m=12832 reference tokens + 19936 outputs, n=128")


def visible_pairs(L, L_m, n):
    """Visible (query, key) pairs per head of the packed R-SWA mask."""
    T_out = L - L_m
    return L_m * (L_m + 1) // 2 + T_out * L_m + sum(min(n, t) for t in range(1, T_out + 1))


def visible_keys(r, L_m, n):
    """Keys visible to 0-based query row r of the packed mask: causal in the
    prefix, else the L_m reference keys plus the window of n."""
    return r + 1 if r < L_m else L_m + min(n, r - L_m + 1)


def log(*a):
    print(*a, file=sys.stderr, flush=True)


# ---------------------------------------------------------------- helpers

FALLBACK_BF16_TFLOPS = 1590.0


def measured_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


def measured_tensor_peak():
    """Dense bf16 TFLOP/s: the burst figure (a kernel timed on its own)."""
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            return float(json.load(f)["bf16_tflops"]), "measured"
    except Exception:
        return FALLBACK_BF16_TFLOPS, "fallback"


CURVE_T = (1, 32, 64, 128, 256, 512, 1024, 2048, 4096, 6144)
# long-horizon workload: out to T = 100000, and the full cache further, to
# 1,000,000 outputs (a 41.5 GB cache for batch 8; loading it needs as much
# again for its source, so that is as far as half of HBM takes it)
CURVE_T_LONG = (1, 128, 1024, 8192, 32768, 65536, 100000)
CURVE_T_LONG_FULL = CURVE_T_LONG + (250000, 500000, 1000000)


def cache_rows(lens, n, T, full):
    """Cache rows of one head, summed over the sequences, after T outputs:
    L_m + min(n, T) each for R-SWA (Eq.(6)), L_m + T with every output kept
    (Eq.(5))."""
    return sum((L + T) if full else (L + min(n, T)) for L in lens)


def curve_cache_ratio(lens, n, Ts):
    """R-SWA cache over the full cache at each T (Eq.(7); one sequence gives
    (L_m + min(n, T)) / (L_m + T))."""
    return [round(cache_rows(lens, n, T, False) / cache_rows(lens, n, T, True), 6) for T in Ts]


def packed_source(B, S, H, d, dtype, seed, block_rows=65536):
    """A packed [B, S, H, d] tensor of N(0,1) values for loading a cache
    state with load_packed.  Rows beyond ``block_rows`` repeat the first
    block (the values do not matter for timing; this keeps the set-up fast
    for the multi-GB full caches)."""
    import torch
    from reference_sliding_window_b200 import synth
    dev = torch.device("cuda", torch.cuda.current_device())
    out = torch.empty((B, S, H, d), dtype=synth.torch_dtype(dtype), device=dev)
    blk = min(S, block_rows)
    out[:, :blk] = synth.normal((B, blk, H, d), seed, dtype, "cuda")
    for r0 in range(blk, S, blk):
        r1 = min(S, r0 + blk)
        out[:, r0:r1] = out[:, :r1 - r0]
    return out


def run_curve(w, lens, Ts, full_Ts=None, samples: int = 8):
    """Per-step decode latency against the output length T, for the R-SWA
    cache and for the same kernel over the full cache (every output kept):
    the constant-cost curve against the growing one.  Each cache state is
    loaded straight at T - 1 outputs (rswa_load_packed); each sample is one
    fused append+decode launch, timed alone with CUDA events after an L2
    flush; the median of `samples` consecutive steps (outputs T .. T +
    samples - 1) is reported at each T."""
    import torch
    from reference_sliding_window_b200 import MODE_FULL, MODE_RSWA, RSWA, synth
    dev = torch.device("cuda", torch.cuda.current_device())
    B, H, d, n = w["B"], w["H"], w["d"], w["n"]
    dt = synth.torch_dtype(w["dtype"])
    s = 2 if w["dtype"] == "bf16" else 4
    full_Ts = tuple(full_Ts or Ts)
    L_m_cap = max(lens)
    flush = torch.empty(2 * torch.cuda.get_device_properties(dev).L2_cache_size, dtype=torch.uint8, device=dev)
    pool = synth.normal((16, 3, B, H, d), 4000, w["dtype"], "cuda")
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    out = {"timing": "isolated launches after an L2 flush, median of consecutive steps", "samples": samples,
           "state": "each point's cache loaded at T-1 outputs with rswa_load_packed"}
    for name, mode, pts in (("rswa", MODE_RSWA, tuple(Ts)), ("full", MODE_FULL, full_Ts)):
        T_top = max(pts) + samples
        src_K = packed_source(B, L_m_cap + T_top, H, d, w["dtype"], 4100)
        src_V = packed_source(B, L_m_cap + T_top, H, d, w["dtype"], 4200)
        a = RSWA(L_m_cap, n, H, d, B, dt, mode=mode, T_cap=T_top, device=dev)
        o = torch.empty((B, H, d), dtype=dt, device=dev)
        us, gbs = [], []
        for Tc in pts:
            a.load_packed(src_K, src_V, lens, Tc - 1)
            ts = []
            for i in range(samples):
                x = pool[i % 16]
                flush.zero_()
                e0.record()
                a.append_decode(x[0], x[1], x[2], out=o)
                e1.record()
                e1.synchronize()
                ts.append(e0.elapsed_time(e1) * 1e3)
            t_us = statistics.median(ts)
            rows = cache_rows(lens, n, Tc, mode == MODE_FULL)
            us.append(round(t_us, 2))
            gbs.append(round(H * (2 * rows * d * s + 4 * B * d * s) / t_us / 1e3, 1))
        a.check()
        out[f"{name}_T"] = list(pts)
        out[f"{name}_us"] = us
        out[f"{name}_gbs"] = gbs
        out[f"{name}_cache_gb"] = round(2 * H * d * s * cache_rows(lens, n, max(pts), mode == MODE_FULL) / 1e9, 3)
        del a, src_K, src_V
        torch.cuda.empty_cache()
    out["cache_ratio"] = curve_cache_ratio(lens, n, Ts)
    return out


def run_prefill(iters: int, warmup: int):
    """Times rswa_masked_forward on the 32K teacher-forced config (inputs
    252 MB, larger than L2).  Returns a dict for the JSON line."""
    import torch
    from reference_sliding_window_b200 import masked_forward, synth
    w = PREFILL
    dev = torch.device("cuda", torch.cuda.current_device())
    Q, K, V = synth.prefill_case(w["L"], w["H"], w["d"], w["dtype"], seed=21, device="cuda")
    O = torch.empty_like(Q)
    for _ in range(max(1, warmup)):
        masked_forward(Q, K, V, L_m=w["L_m"], n=w["n"], out=O)
    torch.cuda.synchronize(dev)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(iters):
        masked_forward(Q, K, V, L_m=w["L_m"], n=w["n"], out=O)
    e1.record()
    torch.cuda.synchronize(dev)
    sec = e0.elapsed_time(e1) / 1e3 / iters
    # ablation: the same tensors with no reference segment (L_m = 0, the
    # plain sliding window of n the pages contrast R-SWA with)
    e0.record()
    for _ in range(iters):
        masked_forward(Q, K, V, L_m=0, n=w["n"], out=O)
    e1.record()
    torch.cuda.synchronize(dev)
    sec_swa = e0.elapsed_time(e1) / 1e3 / iters
    pairs_swa = visible_pairs(w["L"], 0, w["n"])
    pairs = visible_pairs(w["L"], w["L_m"], w["n"])
    flops = 4.0 * w["d"] * pairs * w["H"]
    dense_causal = 4.0 * w["d"] * (w["L"] * (w["L"] + 1) // 2) * w["H"]
    peak, kind = measured_tensor_peak()
    tf = flops / sec / 1e12
    return {"workload": w["desc"], "ms_per_call": sec * 1e3, "iters": iters,
            "tflops": tf, "visible_pairs_per_head": pairs,
            "roofline": {"bound": "tensor", "achieved": tf, "peak": peak, "unit": "TFLOP/s",
                         "frac": tf / peak, "peak_kind": f"{kind} dense bf16 (burst)",
                         "traffic": recorded_traffic("prefill", PREFILL_SOURCES, "prefill_traffic.json"),
                         "algorithmic_flops_per_launch": flops,
                         "kernel": "rswa::tc::masked_tc_kernel"},
            "dense_causal_flops": dense_causal,
            "window_only_ablation": {"L_m": 0, "ms_per_call": sec_swa * 1e3, "visible_pairs_per_head": pairs_swa,
                                     "tflops": 4.0 * w["d"] * pairs_swa * w["H"] / sec_swa / 1e12}}


VARLEN_SEED = 32  # the 32K pack of 10 documents (9 single-page, one of 47 pages)


def pack_visible_pairs(cu, refs, n):
    """Visible (query, key) pairs per head of a pack: each document's own
    packed mask, nothing across documents."""
    return sum(visible_pairs(cu[i + 1] - cu[i], refs[i], n) for i in range(len(refs)))


def run_varlen(iters: int, warmup: int):
    """Times rswa_masked_forward_varlen on a 32768-row pack of documents
    (inputs 252 MB, larger than L2).  Returns a dict for the JSON line."""
    import torch
    from reference_sliding_window_b200 import masked_forward_varlen, synth
    w = PREFILL
    cu, refs = synth.pack_documents(w["L"], seed=VARLEN_SEED)
    dev = torch.device("cuda", torch.cuda.current_device())
    Q, K, V = synth.prefill_case(w["L"], w["H"], w["d"], w["dtype"], seed=22, device="cuda")
    O = torch.empty_like(Q)
    for _ in range(max(1, warmup)):
        masked_forward_varlen(Q, K, V, cu, refs, w["n"], out=O)
    torch.cuda.synchronize(dev)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(iters):
        masked_forward_varlen(Q, K, V, cu, refs, w["n"], out=O)
    e1.record()
    torch.cuda.synchronize(dev)
    sec = e0.elapsed_time(e1) / 1e3 / iters
    pairs = pack_visible_pairs(cu, refs, w["n"])
    flops = 4.0 * w["d"] * pairs * w["H"]
    peak, kind = measured_tensor_peak()
    tf = flops / sec / 1e12
    return {"workload": f"teacher-forced masked prefill over a pack, bf16: {w['L']} rows holding {len(refs)} "
                        f"documents (lengths {[cu[i + 1] - cu[i] for i in range(len(refs))]}, L_m {refs}), "
                        f"10 heads, d=128, n={w['n']}",
            "ms_per_call": sec * 1e3, "iters": iters, "launches_per_call": 1, "tflops": tf,
            "visible_pairs_per_head": pairs,
            "roofline": {"bound": "tensor", "achieved": tf, "peak": peak, "unit": "TFLOP/s", "frac": tf / peak,
                         "peak_kind": f"{kind} dense bf16 (burst)",
                         "traffic": recorded_traffic("varlen", PREFILL_SOURCES, "prefill_traffic.json"),
                         "algorithmic_flops_per_launch": flops,
                         "kernel": "rswa::tc::masked_tc_kernel (the whole pack in one launch)"}}


DECODE_SOURCES = ("decode.cu", "common.cuh", "internal.h")
PREFILL_SOURCES = ("masked_tc.cu", "common.cuh")  # the kernel takes its parameters from masked_tc.cu


def _code_only(text: str) -> str:
    """Source text without comments and blank space, so that a comment edit
    does not mark a profile as taken on another kernel."""
    import re
    text = re.sub(r"/\*.*?\*/", " ", text, flags=re.S)
    text = re.sub(r"//[^\n]*", " ", text)
    return " ".join(text.split())


def kernel_source_sha(files=DECODE_SOURCES) -> str:
    h = hashlib.sha256()
    for f in files:
        with open(os.path.join(ROOT, "reference_sliding_window_b200", "csrc", f), encoding="utf-8") as fh:
            h.update(_code_only(fh.read()).encode())
    return h.hexdigest()[:16]


def recorded_traffic(workload: str, files=DECODE_SOURCES, record: str = "decode_traffic.json"):
    """DRAM bytes per launch from the committed ncu summary, if it was taken
    on the current kernel source for this workload; else None."""
    try:
        with open(os.path.join(ROOT, "profiles", record)) as f:
            d = json.load(f)
        rec = d.get(workload)
        if rec and rec.get("source_sha") == kernel_source_sha(files):
            return float(rec["dram_bytes_per_launch"])
    except Exception:
        pass
    return None


class ClockSampler:
    """nvidia-smi clock / throttle sampling during the timed region."""

    QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.QUERY}", "--format=csv,noheader,nounits",
                 "-lms", "50"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None
        time.sleep(0.3)
        return self

    def __exit__(self, *exc):
        self.lines = []
        if self.proc is not None:
            self.proc.terminate()
            try:
                out, _ = self.proc.communicate(timeout=5)
            except Exception:
                self.proc.kill()
                out = ""
            self.lines = [l for l in out.splitlines() if l.strip()]
        return False

    def summary(self):
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in getattr(self, "lines", []):
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                mx = float(parts[2])
            except ValueError:
                continue
            for nm, val in zip(names, parts[5:9]):
                if val.lower() == "active":
                    reasons.add(nm)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unavailable"], "samples": 0}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm)}


# ------------------------------------------------------- distributed plumbing

def dist_env():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


def reduce_max_sum(elapsed_s: float, units: float, backend_device=None):
    """Max of the elapsed times and sum of the units over all ranks (a host
    plumbing reduction, not part of the measured path)."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()):
        return elapsed_s, units
    t = torch.tensor([elapsed_s], dtype=torch.float64, device=backend_device)
    u = torch.tensor([units], dtype=torch.float64, device=backend_device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    dist.all_reduce(u, op=dist.ReduceOp.SUM)
    return float(t.item()), float(u.item())


def replica_seed(base: int, layer: int, rank: int) -> int:
    """Seed of one rank's inputs: every rank runs its own replica of the
    workload on different data (no rank shares a tensor with another)."""
    return base + layer + 7919 * rank


def whole_job_rate(units_sum: float, elapsed_max_s: float) -> float:
    """Whole-job throughput: the units every rank processed over the time of
    the slowest rank."""
    return units_sum / elapsed_max_s


# --------------------------------------------------------------- our arm

def ref_lens_for(w, seed=0):
    from reference_sliding_window_b200 import synth
    if w["pages"] is None:
        pages = synth.ragged_page_counts(w["B"], seed=seed)
    else:
        pages = w["pages"][:w["B"]]
    return [synth.reference_length(p, w["prompt"]) for p in pages]


def bytes_per_launch(w, lens):
    s = 2 if w["dtype"] == "bf16" else 4
    d, H, n = w["d"], w["H"], w["n"]
    return sum(H * (2 * (L + n) * d * s + 4 * d * s) for L in lens)


GRAPH_STEPS = 16  # decode steps per captured CUDA graph


def step_plan(T_target: int, n: int, steps: int, warmup: int):
    """Where the decode run starts: the cache is loaded at T0 outputs, then
    `warmup` eager steps and one graph replay of GRAPH_STEPS warm-up steps
    run, then exactly `steps` timed steps, ending at output T_target when
    that leaves the ring full (T0 >= n) at the start; otherwise T0 = n and
    the run ends past T_target.  -> (T0, first timed output, last)."""
    T0 = max(n, T_target - warmup - GRAPH_STEPS - steps)
    first = T0 + warmup + GRAPH_STEPS + 1
    return T0, first, first + steps - 1


def run_decode(args, name, w, lens, T_target, steps, warmup, e2e_steps):
    """Times `steps` decode steps of workload w.  One step runs the fused
    append+decode once for each of R layer caches (R distinct caches, as in
    an R-layer decoder, with R * bytes per launch >= 2 x L2 so nothing is
    served from L2 between steps).  Every cache starts at T0 outputs
    (rswa_load_packed from a packed random sequence), in the steady state
    T > n where the R-SWA cost per step is constant.  The steps run as CUDA
    graphs of GRAPH_STEPS steps plus one graph for the remainder, so exactly
    `steps` steps are timed."""
    import torch
    import torch.distributed as dist
    from reference_sliding_window_b200 import RSWA, LayerStep, append_decode_layers, synth

    world, rank, local = dist_env()
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    B, H, d, n = w["B"], w["H"], w["d"], w["n"]
    dt = synth.torch_dtype(w["dtype"])
    L_m_cap = max(lens)
    per_launch = bytes_per_launch(w, lens)
    l2 = torch.cuda.get_device_properties(dev).L2_cache_size
    R = args.layers or max(1, math.ceil(2 * l2 / per_launch))
    T0, T_first, T_last = step_plan(T_target, n, steps, warmup)

    layers = []
    for r in range(R):
        a = RSWA(L_m_cap, n, H, d, B, dt, device=dev)
        Kp = packed_source(B, L_m_cap + T0, H, d, w["dtype"], replica_seed(1000, r, rank))
        Vp = packed_source(B, L_m_cap + T0, H, d, w["dtype"], replica_seed(2000, r, rank))
        a.load_packed(Kp, Vp, lens, T0)
        del Kp, Vp
        layers.append(a)
    torch.cuda.empty_cache()
    P = GRAPH_STEPS  # distinct per-step inputs, cycled
    pool = synth.normal((P, R, 3, B, H, d), replica_seed(3000, 0, rank), w["dtype"], "cuda")
    out = torch.empty((R, B, H, d), dtype=dt, device=dev)
    outs = [out[r] for r in range(R)]
    # per-step views of the inputs, made once (as a model holds its buffers)
    views = [([pool[i, r, 0] for r in range(R)], [pool[i, r, 1] for r in range(R)],
              [pool[i, r, 2] for r in range(R)]) for i in range(P)]

    def step(i):
        k, v, q = views[i % P]
        append_decode_layers(layers, k, v, q, out=outs)

    reps, tail = divmod(steps, P)
    stream = torch.cuda.Stream(device=dev)
    stream.wait_stream(torch.cuda.current_stream(dev))
    with torch.cuda.stream(stream):
        for i in range(warmup):
            step(i)
        torch.cuda.synchronize(dev)
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=stream):
            for i in range(P):
                step(i)
        gt = None
        if tail:
            gt = torch.cuda.CUDAGraph()
            with torch.cuda.graph(gt, stream=stream):
                for i in range(tail):
                    step(i)
        g.replay()  # warm-up replay
        torch.cuda.synchronize(dev)
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):  # graph replays launch on the current stream
        if dist.is_initialized():
            dist.barrier()
        torch.cuda.synchronize(dev)
        with ClockSampler(dev.index if dev.index is not None else 0) as clk:
            start.record(stream)
            for _ in range(reps):
                g.replay()
            if gt is not None:
                gt.replay()
            end.record(stream)
            torch.cuda.synchronize(dev)
        if dist.is_initialized():
            dist.barrier()
    elapsed = start.elapsed_time(end) / 1e3
    launches = steps * R
    for a in layers:
        a.check()
    T_end = layers[0].step_count()[0]
    assert T_end == T_last, (T_end, T_last)

    # ---- e2e: host buffers through the public binding
    K_e2e = max(1, e2e_steps)
    host_in = torch.empty((P, R, 3, B, H, d), dtype=dt, pin_memory=True)
    host_in.copy_(pool.cpu())
    host_out = torch.empty((K_e2e, R, B, H, d), dtype=dt, pin_memory=True)
    dev_in = torch.empty((R, 3, B, H, d), dtype=dt, device=dev)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    # the step over the staging buffers, made once (as a model holds its buffers)
    with torch.cuda.stream(stream):
        step_e2e = LayerStep(layers, [dev_in[r, 0] for r in range(R)], [dev_in[r, 1] for r in range(R)],
                             [dev_in[r, 2] for r in range(R)], outs, graph=True)
        # warm-up steps of the same loop (the first replay of a new graph also uploads it)
        for i in range(max(3, warmup)):
            dev_in.copy_(host_in[i % P], non_blocking=True)
            step_e2e()
            host_out[0].copy_(out, non_blocking=True)
        torch.cuda.synchronize(dev)
        e0.record(stream)
        for i in range(K_e2e):
            dev_in.copy_(host_in[i % P], non_blocking=True)
            step_e2e()
            host_out[i].copy_(out, non_blocking=True)
        e1.record(stream)
        torch.cuda.synchronize(dev)
    e2e_s = e0.elapsed_time(e1) / 1e3
    for a in layers:
        a.check()

    el_max, tok_sum = reduce_max_sum(elapsed, float(B * R * steps), dev)
    e2e_max, e2e_tok = reduce_max_sum(e2e_s, float(B * R * K_e2e), dev)
    g.reset()
    if gt is not None:
        gt.reset()
    del layers, pool, out, outs, views, step_e2e
    torch.cuda.empty_cache()
    s_el = 2 if w["dtype"] == "bf16" else 4
    return dict(name=name, R=R, K=steps, elapsed=elapsed, el_max=el_max, tok_sum=tok_sum, launches=launches,
                per_launch=per_launch, clocks=clk.summary(), e2e_max=e2e_max, e2e_tok=e2e_tok,
                K_e2e=K_e2e, T_range=[T_first, T_last], l2=l2,
                h2d=int(R * 3 * B * H * d * s_el), d2h=int(R * B * H * d * s_el))


def decode_entry(args, w, lens, res, cpu=None):
    """The JSON fields of one decode workload's measurement."""
    peak, peak_kind = measured_peaks()
    avg_launch = res["elapsed"] / res["launches"]
    achieved = res["per_launch"] / avg_launch / 1e9
    world = dist_env()[0]
    config = {"workload": w["desc"] + f"; timed outputs T = {res['T_range'][0]}..{res['T_range'][1]}",
              "batch": w["B"], "heads": w["H"], "head_dim": w["d"], "n": w["n"],
              "L_m": lens if len(lens) <= 8 else {"min": min(lens), "max": max(lens),
                                                  "mean": sum(lens) / len(lens)},
              "layers_cycled": res["R"],
              "l2": f"inputs larger than L2: {res['R']} layer cache(s) x {res['per_launch'] / 1e6:.2f} MB "
                    f"= {res['R'] * res['per_launch'] / 1e6:.0f} MB per step vs L2 {res['l2'] / 1e6:.0f} MB",
              "T_range": res["T_range"],
              "unit_def": "one decode token of one attention layer for one sequence",
              "parallelism": f"replicas x{world}"}
    return {
        "value": whole_job_rate(res["tok_sum"], res["el_max"]), "unit": "tokens/s",
        "steps": res["K"], "ms_per_step": 1e3 * res["el_max"] / res["K"], "config": config,
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                     "frac": achieved / peak, "peak_kind": f"{peak_kind} HBM copy",
                     "traffic": recorded_traffic(res["name"]),
                     "algorithmic_bytes_per_launch": res["per_launch"],
                     "avg_launch_us": avg_launch * 1e6, "kernel": "rswa::decode_kernel<bf16,128,append>"},
        "clocks": res["clocks"],
        "e2e": {"value": whole_job_rate(res["e2e_tok"], res["e2e_max"]), "unit": "tokens/s",
                "h2d_bytes_per_step": res["h2d"], "d2h_bytes_per_step": res["d2h"], "steps": res["K_e2e"]},
        "gpu_launches": res["launches"],
        "cpu_baseline": cpu,
    }


# ------------------------------------------------------------ oracle timing

def oracle_sample(w, lens, budget_s: float, seed: int = 0, max_seqs: int = 4):
    """Times the fp64 CPU oracle on decode steps of this workload: each
    sampled step recomputes the attention of one token for one sequence and
    every head from the full history (steady state, T = n + a few).  For a
    batch, up to ``max_seqs`` sequences at evenly spaced quantiles of the
    reference lengths stand in for the batch and run in turn, so the rate
    weighs the length mix as the whole batch would.  Returns (tokens/s of
    one layer, threads, description)."""
    import numpy as np
    import oracle
    try:
        from threadpoolctl import threadpool_info
        threads = max([i.get("num_threads", 1) for i in threadpool_info()] or [1])
    except Exception:
        threads = 1
    rng = np.random.default_rng(seed)
    H, d, n = w["H"], w["d"], w["n"]
    T = n + 8
    srt = sorted(lens)
    k = min(max_seqs, len(srt))
    pick = [srt[(2 * i + 1) * len(srt) // (2 * k)] for i in range(k)]
    hist = []
    for L in pick:
        Kh = rng.standard_normal((L + T, H, d))
        Vh = rng.standard_normal((L + T, H, d))
        hist.append((Kh, Vh))
    done, t0 = 0, time.perf_counter()
    while True:
        q = rng.standard_normal((H, d))
        for i, L in enumerate(pick):
            oracle.decode_step(q, hist[i][0], hist[i][1], L, T, n)
        done += len(pick)
        el = time.perf_counter() - t0
        if el >= budget_s and done >= 2:
            break
    who = f"{len(pick)} of {len(lens)} sequences (L_m {pick})" if len(lens) > 1 else f"L_m {pick[0]}"
    return done / el, threads, f"{done} sequence decode steps x {H} heads (T={T}), {who}, fp64 numpy"


def oracle_prefill_sample(w, budget_s: float, seed: int = 0, n_random: int = 256, docs=None):
    """Times the fp64 CPU oracle on sampled query rows of the teacher-forced
    workload: the rows at the segment edges (of every document, for a pack
    given as docs = (cu_seqlens, ref_lens)), then random rows, one at a time
    until the budget is spent.  Returns (algorithmic TFLOP/s over the visible
    pairs of the rows done, threads, description)."""
    import numpy as np
    import oracle
    try:
        from threadpoolctl import threadpool_info
        threads = max([i.get("num_threads", 1) for i in threadpool_info()] or [1])
    except Exception:
        threads = 1
    rng = np.random.default_rng(seed)
    L, L_m, n, H, d = w["L"], w["L_m"], w["n"], w["H"], w["d"]
    Q, K, V = (rng.standard_normal((L, H, d), dtype=np.float32) for _ in range(3))
    cu, refs = docs if docs is not None else ([0, L], [L_m])
    doc_of = np.repeat(np.arange(len(refs)), np.diff(cu))
    edges = []
    for i, Lm in enumerate(refs):
        a, b = cu[i], cu[i + 1]
        edges += [r for r in (a, a + Lm - 1, a + Lm, a + Lm + n - 1, a + Lm + n, b - 1) if a <= r < b]
    rows = edges + rng.integers(0, L, n_random).tolist()
    done, pairs, t0 = 0, 0, time.perf_counter()
    for r in rows:
        i = int(doc_of[r])
        if docs is None:
            oracle.masked_forward_rows(Q, K, V, L_m, n, [r])
        else:
            oracle.masked_forward_varlen_rows(Q, K, V, cu, refs, n, [r])
        pairs += visible_keys(r - cu[i], refs[i], n)
        done += 1
        el = time.perf_counter() - t0
        if el >= budget_s and done >= 2:
            break
    what = f"{L}-row pack of {len(refs)} documents" if docs is not None else f"{L}-row sequence"
    return (4.0 * d * pairs * H / el / 1e12, threads,
            f"{done} query rows (segment edges, then random) x {H} heads of the {what}, fp64 numpy")


# -------------------------------------------------------------------- main

def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=64)
    ap.add_argument("--warmup", type=int, default=8)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", choices=sorted(WORKLOADS) + ["prefill", "varlen"], default="single_doc")
    ap.add_argument("--nested", type=int, default=1,
                    help="1: with the single-document headline on one GPU, also time the ragged and "
                         "long-horizon decode workloads")
    ap.add_argument("--prefill-iters", type=int, default=10, help="timed masked-prefill calls (0: skip)")
    ap.add_argument("--curve", type=int, default=1, help="1: add per-step latency vs T, R-SWA and full cache")
    ap.add_argument("--layers", type=int, default=0, help="layer caches cycled (0: 2 x L2 rule)")
    ap.add_argument("--e2e-steps", type=int, default=64)
    ap.add_argument("--cpu-budget", type=float, default=15.0, help="seconds of oracle timing")
    ap.add_argument("--batch", type=int, default=0,
                    help="decode: keep only the first BATCH sequences of the workload (a smaller case of the same "
                         "kernel, for profiler captures); 0 = all")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    if args.steps < 1:
        ap.error("--steps must be >= 1")

    world, rank, local = dist_env()
    if args.workload in ("prefill", "varlen"):
        return main_prefill(args)
    w = dict(WORKLOADS[args.workload])
    lens = ref_lens_for(w)
    if args.batch:
        lens = lens[:args.batch]
        w["B"] = len(lens)
        w["desc"] += f" (first {len(lens)} sequences)"
        args.nested = 0

    if args.impl == "reference":
        if rank != 0:
            return 0
        v, threads, sample = oracle_sample(w, lens, args.cpu_budget)
        config = {"workload": w["desc"], "batch": w["B"], "heads": w["H"], "head_dim": w["d"], "n": w["n"],
                  "l2": "host CPU"}
        line = {"metric": METRIC, "value": v, "unit": "tokens/s", "n_gpus": args.gpus, "steps": args.steps,
                "warmup": args.warmup, "ms_per_step": 1e3 / v, "higher_is_better": True,
                "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
                "impl": "reference", "config": config,
                "cpu_baseline": {"value": v, "unit": "tokens/s", "cores": threads, "kind": "oracle",
                                 "sample": sample},
                "e2e": {"value": v, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
        print(json.dumps(line), flush=True)
        return 0

    import torch
    import torch.distributed as dist
    if world > 1:
        import datetime
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    res = run_decode(args, args.workload, w, lens, w["T"], args.steps, args.warmup, args.e2e_steps)
    if rank == 0:
        cpu = None
        if world == 1:
            v, threads, sample = oracle_sample(w, lens, args.cpu_budget)
            cpu = {"value": v, "unit": "tokens/s", "cores": threads, "kind": "oracle", "sample": sample}
        entry = decode_entry(args, w, lens, res, cpu)
        nested = {}
        curves = {}
        if world == 1 and args.nested and args.workload == "single_doc":
            for name in ("ragged", "long"):
                wn = WORKLOADS[name]
                ln = ref_lens_for(wn)
                rn = run_decode(args, name, wn, ln, wn["T"], args.steps, args.warmup, args.e2e_steps)
                v, threads, sample = oracle_sample(wn, ln, args.cpu_budget / 3)
                nested[name] = decode_entry(args, wn, ln, rn, {"value": v, "unit": "tokens/s", "cores": threads,
                                                               "kind": "oracle", "sample": sample})
        prefill = run_prefill(args.prefill_iters, 3) if (args.prefill_iters > 0 and world == 1) else None
        if args.curve and world == 1 and w["B"] * max(lens) <= 16384:
            curves[args.workload] = run_curve(w, lens, CURVE_T)
            if args.nested and args.workload == "single_doc":
                wl = WORKLOADS["long"]
                curves["long"] = run_curve(wl, ref_lens_for(wl), CURVE_T_LONG, CURVE_T_LONG_FULL)
        line = {"metric": METRIC, "value": entry["value"], "unit": "tokens/s", "n_gpus": world,
                "steps": entry["steps"], "warmup": args.warmup, "ms_per_step": entry["ms_per_step"],
                "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": w["dtype"],
                "data": "synthetic"}
        for key in ("config", "roofline", "clocks", "e2e", "gpu_launches", "cpu_baseline"):
            line[key] = entry[key]
        line["configs"] = nested or None
        line["prefill"] = prefill
        line["vs_output_length"] = curves or None
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    return 0


def main_prefill(args):
    """--workload prefill / varlen: the teacher-forced form, on one sequence
    or on a pack of documents, on its own JSON line."""
    world, rank, local = dist_env()
    if rank != 0:
        return 0
    metric = "R-SWA masked prefill TFLOP/s (algorithmic, visible pairs only)"
    docs = None
    if args.workload == "varlen":
        from reference_sliding_window_b200 import synth
        docs = synth.pack_documents(PREFILL["L"], seed=VARLEN_SEED)
        pairs = pack_visible_pairs(docs[0], docs[1], PREFILL["n"])
        desc = f"teacher-forced masked prefill over a pack, bf16: {PREFILL['L']} rows, {len(docs[1])} documents"
    else:
        pairs = visible_pairs(PREFILL["L"], PREFILL["L_m"], PREFILL["n"])
        desc = PREFILL["desc"]
    if args.impl == "reference":
        v, threads, sample = oracle_prefill_sample(PREFILL, args.cpu_budget, docs=docs)
        line = {"metric": metric, "value": v, "unit": "TFLOP/s", "n_gpus": args.gpus, "steps": args.steps,
                "warmup": args.warmup,
                # one whole call's algorithmic FLOPs at the sampled rate
                "ms_per_step": 1e3 * 4.0 * PREFILL["d"] * PREFILL["H"] * pairs / (v * 1e12),
                "higher_is_better": True, "scaling": "weak",
                "vs_baseline": None, "dtype": "f64", "data": "synthetic", "impl": "reference",
                "config": {"workload": desc, "l2": "host CPU"},
                "cpu_baseline": {"value": v, "unit": "TFLOP/s", "cores": threads, "kind": "oracle",
                                 "sample": sample},
                "e2e": {"value": v, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
        print(json.dumps(line), flush=True)
        return 0
    import torch
    torch.cuda.set_device(local)
    if docs is not None:
        r = run_varlen(max(1, args.steps), max(3, args.warmup))
        launches = r["iters"] * r["launches_per_call"]
    else:
        r = run_prefill(max(1, args.steps), max(3, args.warmup))
        launches = r["iters"]
    v, threads, sample = oracle_prefill_sample(PREFILL, args.cpu_budget, docs=docs)
    line = {"metric": metric, "value": r["tflops"],
            "unit": "TFLOP/s", "n_gpus": 1, "steps": r["iters"], "warmup": max(3, args.warmup),
            "ms_per_step": r["ms_per_call"], "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "bf16", "data": "synthetic",
            "config": {"workload": r["workload"], "l2": "inputs 252 MB, larger than L2"},
            "roofline": r["roofline"], "gpu_launches": launches,
            "cpu_baseline": {"value": v, "unit": "TFLOP/s", "cores": threads, "kind": "oracle", "sample": sample}}
    print(json.dumps(line), flush=True)
    return 0


if __name__ == "__main__":
    sys.exit(main())
