#!/usr/bin/env python
"""Benchmark of DropKV prefill-time eviction scoring on B200.

One step = the whole scoring path on one input set, in one call of the public
API, dropkv_scores_select: window attention statistics, exact single-removal
perturbation scores summed over the window, GQA mean-merge, MaxPool1D, window
protection (the scores are written out), then the exact lowest-score eviction
per KV head -- the results of dropkv_scores followed by dropkv_select.

Workload (N=1): the 128K-token Llama-3.1-8B-shaped case -- B=1, Hq=32, Hkv=8,
d=128, n=131072, w=64, bf16 Gaussian Q/K/V with 4 outlier K channels x8 per KV
head, pool 7, keep 5%.  K+V are 537 MB, more than twice the 126 MB L2, so no
L2 flush is needed between steps; for the smaller configurations (--config N)
whose K+V fit twice the L2, a write of twice its size flushes it before every
timed step, outside the step's events.  With N GPUs (torchrun) every rank scores its
own independent input set (seed 42 + rank): weak scaling, no data-path
collective; the time is the max over ranks.

--impl reference times the fp64 CPU oracle on the same whole workload on the
host cores (one OpenMP thread per batch row and query head).
"""

import argparse
import dataclasses
import hashlib
import json
import os
import re
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402
import torch  # noqa: E402

from kv_cache_eviction_scores_b200 import workloads as W  # noqa: E402

METRIC = "KV tokens scored/sec per GPU at n=128K; achieved HBM GB/s as % of roofline"
UNIT = "tokens/s"
PEAKS_FILE = os.path.join(ROOT, "MEASURED_PEAKS.json")
TRAFFIC_FILE = os.path.join(ROOT, "profiles", "ncu_traffic.json")
CSRC = os.path.join(ROOT, "kv_cache_eviction_scores_b200", "csrc")

# kernel order of the scoring kernels of a call (must match the library's
# launch sequence); a step (dropkv_scores_select) runs them and then the
# selection kernel
KERNELS = {
    "simt": ["k_simt_pass1", "k_simt_pass2", "k_epilogue"],
    # the DropKV score's second pass runs on CTA pairs; the attention-only
    # control keeps the single-CTA second pass (K streamed alone)
    "tensor": ["k_tc_pass1", "k_tc_combine", "k_tc_pass2_pair", "k_epilogue"],
    "tensor_attention": ["k_tc_pass1", "k_tc_combine", "k_tc_pass2", "k_epilogue"],
}
# the sources a kernel's code comes from (its file and the device headers it includes)
_TC_HDRS = ("tc_common.cuh", "tc_ptx.cuh", "common.cuh")
KERNEL_SRC = {
    "k_simt_pass1": ("simt.cu", "common.cuh"), "k_simt_pass2": ("simt.cu", "common.cuh"),
    "k_epilogue": ("epilogue.cu", "common.cuh"),
    "k_tc_pass1": ("tc.cu",) + _TC_HDRS, "k_tc_combine": ("tc.cu",) + _TC_HDRS,
    "k_tc_pass2": ("tc.cu",) + _TC_HDRS, "k_tc_pass2_pair": ("tc_pair.cu",) + _TC_HDRS,
}


NOMINAL_HBM_GBS = 8000.0  # B200 HBM3e nominal (DGX figure), context beside the measured peak


def parse():
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=50)
    p.add_argument("--warmup", type=int, default=5)
    p.add_argument("--impl", choices=["ours", "reference"], default="ours")
    p.add_argument("--config", type=int, default=3, help="workload index (3 = 128K headline)")
    p.add_argument("--path", choices=["auto", "simt", "tensor"], default="auto")
    p.add_argument("--seq", type=int, default=None,
                   help="override the configuration's sequence length (one batch row; profiling "
                        "a smaller case of the same shape)")
    p.add_argument("--score", choices=["perturbation", "attention"], default="perturbation",
                   help="DropKV's perturbation score, or the attention-only control score")
    p.add_argument("--e2e-steps", type=int, default=None)
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--no-clocks", action="store_true")
    return p.parse_args()


def peaks():
    try:
        with open(PEAKS_FILE) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), float(d["bf16_tflops"]), float(d.get("sm_max_mhz", 1965.0)), \
            "measured"
    except Exception:
        return 6650.0, 1590.0, 1965.0, "fallback"


def bench_spec(args):
    spec = W.config_spec(args.config)
    if args.seq is not None:
        frac = spec.keep[0] / spec.lengths[0]
        spec = dataclasses.replace(spec, name=f"{spec.name}@n{args.seq}", B=1, lengths=[args.seq],
                                   n_max=args.seq, keep=[int(frac * args.seq)])
    return spec


def workload_desc(spec):
    return (f"{spec.name}: B={spec.B} Hq={spec.Hq} Hkv={spec.Hkv} d={spec.d} "
            f"n={spec.lengths} w={spec.window} pool={spec.pool} keep={spec.keep} {spec.dtype}")


def visible_elements(spec):
    """(token, window query) pairs with token visible to the query, all heads."""
    w = spec.window
    per_query_head = sum(w * (L - w) + w * (w + 1) // 2 for L in spec.lengths)
    return per_query_head * spec.Hq


def split_runs(lengths, units, budget, tile=128):
    """Tile runs of the CTAs of one tensor-path pass: the library's split rule
    (one more split to the batch row whose runs are longest while the CTA
    budget allows), restated here to report the load balance."""
    nts = [(L + tile - 1) // tile for L in lengths]
    splits = [1] * len(lengths)
    total = units * len(lengths)
    budget = max(budget, total)
    while True:
        best, worst = -1, 0.0
        for b, nt in enumerate(nts):
            per = nt / splits[b]
            if splits[b] < nt and per > worst:
                best, worst = b, per
        if best < 0 or total + units > budget:
            break
        splits[best] += 1
        total += units
    return [(sp + 1) * nt // splits[b] - sp * nt // splits[b]
            for b, nt in enumerate(nts) for sp in range(splits[b])]


def tensor_plan(spec, sms):
    """CTA counts and per-CTA tile runs (min, max) of the two tensor-core
    passes: pass 1 one CTA per (b, h, query chunk, split), the DropKV second
    pass one CTA pair per (b, h, query chunk, split), each CTA of a pair
    taking half of the pair's run."""
    nq = spec.G * spec.window
    units = spec.Hkv * ((nq + 255) // 256)
    budget = min(sms, 160)
    r1 = split_runs(spec.lengths, units, budget)
    r2 = split_runs(spec.lengths, units, budget // 2)
    h2 = [(x + 1) // 2 for x in r2]
    return {"pass1_ctas": len(r1) * units, "pass1_tiles_per_cta": [min(r1), max(r1)],
            "pass2_ctas": 2 * len(r2) * units, "pass2_tiles_per_cta": [min(h2), max(h2)]}


# ----------------------------------------------------------- multi-rank ----

def rank_seed(rank):
    """Each rank scores its own independent input set (weak scaling)."""
    return 42 + rank


def max_over_ranks(ms, dist, device):
    """The slowest rank's time: the job is done when every rank is."""
    if dist is None:
        return ms
    t = torch.tensor([ms], device=device, dtype=torch.float64)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_value(world, tokens_per_rank, ms):
    """Tokens scored per second by all ranks together."""
    return world * tokens_per_rank / (ms * 1e-3)


# ---------------------------------------------------------------- clocks ----

class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index, enabled=True):
        self.proc = None
        self.path = None
        self.dev = device_index
        self.enabled = enabled

    def start(self):
        if not self.enabled:
            return
        try:
            uuid = str(torch.cuda.get_device_properties(self.dev).uuid)
            sel = ["-i", uuid if uuid.startswith("GPU-") else f"GPU-{uuid}"]
        except Exception:
            sel = ["-i", str(self.dev)]
        self.path = os.path.join("/tmp", f"dropkv_clocks_{os.getpid()}.csv")
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", *sel, f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
            time.sleep(0.3)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        rows = []
        with open(self.path) as f:
            for line in f:
                parts = [x.strip() for x in line.split(",")]
                if len(parts) >= 9:
                    rows.append(parts)
        if not rows:
            return None
        sm = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        mx = [float(r[2]) for r in rows if r[2].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if "Active" in r[5 + i]
                          and "Not" not in r[5 + i]})
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(mx) if mx else None, "reasons": reasons,
                "samples": len(rows)}


# ------------------------------------------------------------ reference ----

def oracle_sample(wl):
    """fp64 oracle on the whole workload: every KV head of every batch row (all
    query heads, window queries over every key), then merge / pool / protect
    and the selection.  The oracle runs one OpenMP thread per (batch row, query
    head).  Returns (seconds, share of the workload = 1, threads used,
    description)."""
    import oracle
    spec = wl.spec
    t0 = time.perf_counter()
    s = oracle.scores(wl.q, wl.k, wl.v, wl.lengths, spec.window, spec.pool)
    oracle.select(s, wl.lengths, wl.keep)
    dt = time.perf_counter() - t0
    threads = min(oracle.num_threads(), spec.B * spec.Hq)
    desc = (f"the whole workload ({spec.B} x {spec.Hq} query heads x {spec.window} window "
            f"queries over all {sum(wl.lengths)} keys, then merge / pool / select), fp64, "
            f"{dt:.2f} s")
    return dt, 1.0, threads, desc


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    import oracle
    spec = bench_spec(args)
    wl = W.generate(spec, 42)
    tokens = sum(wl.lengths)
    times = []
    for i in range(args.warmup + args.steps):
        dt, frac, cores, sample = oracle_sample(wl)
        if i >= args.warmup:
            times.append(dt / frac)
    t = statistics.mean(times)
    sample = "per step: " + sample
    line = {
        "impl": "reference", "metric": METRIC, "value": tokens / t, "unit": UNIT,
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": t * 1e3, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": workload_desc(spec), "global_batch": spec.B,
                   "seq_len": max(spec.lengths), "parallelism": "none (host cores)"},
        "cpu_baseline": {"value": tokens / t, "unit": UNIT, "cores": cores, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": tokens / t, "unit": UNIT, "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


# ------------------------------------------------------------------ ours ----

def source_hash(fnames):
    """sha256 of a kernel's source files, in order: line comments and blank
    lines removed, so that a comment edit does not invalidate the stored DRAM
    traffic."""
    h = hashlib.sha256()
    for fname in fnames:
        with open(os.path.join(CSRC, fname), encoding="utf-8") as f:
            lines = (re.sub(r"//.*$", "", ln).rstrip() for ln in f)
            code = "\n".join(ln for ln in lines if ln.strip())
        h.update(fname.encode() + b"\n" + code.encode() + b"\n")
    return h.hexdigest()


def traffic_for(kernel, spec):
    """ncu DRAM bytes per launch of `kernel`, if captured on the current source
    and on this workload (the stored figure is for one workload's launch)."""
    try:
        with open(TRAFFIC_FILE) as f:
            d = json.load(f)
        e = d[kernel]
        if e.get("csrc_sha256") != source_hash(KERNEL_SRC[kernel]):
            return None
        if e.get("workload") != workload_desc(spec):
            return None
        return float(e["bytes_per_launch"])
    except Exception:
        return None


def roofline(kernel, spec, us, hbm_peak, tc_peak, sm_mhz, score="perturbation"):
    """Roofline object for one kernel from its live CUDA-event duration."""
    elems = visible_elements(spec)
    d = spec.d
    valid = sum(spec.lengths) * spec.Hkv
    if kernel in ("k_simt_pass1", "k_simt_pass2"):
        # two length-d contractions per visible (token, query) element on FP32 FMA units
        flops = 2 * 2 * d * elems
        peak = 148 * 128 * 2 * sm_mhz * 1e6 / 1e12  # FP32 lanes x FMA x clock, TFLOP/s
        ach = flops / (us * 1e-6) / 1e12
        return {"bound": "alu", "achieved": ach, "peak": peak, "unit": "TFLOP/s",
                "frac": ach / peak, "traffic": traffic_for(kernel, spec),
                "peak_source": "148 SMs x 128 FP32 lanes x 2 flop x max SM clock",
                "work": f"{flops:.4g} flop (4*d per visible element)"}
    if kernel == "k_tc_pass2" and score == "attention":
        # the attention-only second pass streams K alone and contracts Q K^T
        nbytes = valid * d * 2
        ach = nbytes / (us * 1e-6) / 1e9
        flops = 2 * d * elems
        tach = flops / (us * 1e-6) / 1e12
        return {"bound": "hbm", "achieved": ach, "peak": hbm_peak, "unit": "GB/s",
                "frac": ach / hbm_peak, "traffic": None,
                "work": f"{nbytes} B (one read of the valid K rows)",
                "tensor": {"achieved": tach, "peak": tc_peak, "unit": "TFLOP/s",
                           "frac": tach / tc_peak,
                           "work": f"{flops:.4g} flop (2*d per visible element)"}}
    if kernel in ("k_tc_pass1", "k_tc_pass2", "k_tc_pass2_pair"):
        # each pass streams K and V once: one read of the valid K and V rows is
        # the algorithmic traffic of a launch (2 tensors x d x 2 bytes per
        # (token, KV head)); the two contractions (4 d flop per visible element)
        # are reported beside it against the measured bf16 tensor peak
        nbytes = valid * d * 2 * 2
        ach = nbytes / (us * 1e-6) / 1e9
        flops = 2 * 2 * d * elems
        tach = flops / (us * 1e-6) / 1e12
        return {"bound": "hbm", "achieved": ach, "peak": hbm_peak, "unit": "GB/s",
                "frac": ach / hbm_peak, "traffic": traffic_for(kernel, spec),
                "work": f"{nbytes} B (one read of the valid K and V rows)",
                "tensor": {"achieved": tach, "peak": tc_peak, "unit": "TFLOP/s",
                           "frac": tach / tc_peak,
                           "work": f"{flops:.4g} flop (4*d per visible element)"}}
    # HBM-bound helpers
    nbytes = valid * 4 * 2
    ach = nbytes / (us * 1e-6) / 1e9
    return {"bound": "hbm", "achieved": ach, "peak": hbm_peak, "unit": "GB/s",
            "frac": ach / hbm_peak, "traffic": traffic_for(kernel, spec),
            "work": f"{nbytes} B"}


def run_e2e(dk, wl, q, k, v, scores, status, step, E, dist, dev, world):
    """Same metric through the public API with host buffers: every step copies
    the inputs host->device (pinned) and the scores / index lists / status back."""
    qh, kh, vh = (t.pin_memory() for t in (wl.q, wl.k, wl.v))
    sc_h = torch.empty(scores.shape, dtype=torch.float32).pin_memory()
    keep_idx, ev_idx = step()
    kp_h = torch.empty(keep_idx.shape, dtype=torch.int32).pin_memory()
    ev_h = torch.empty(ev_idx.shape, dtype=torch.int32).pin_memory()
    st_h = torch.empty(1, dtype=torch.int32).pin_memory()
    torch.cuda.synchronize()

    def e2e_step():
        q.copy_(qh, non_blocking=True)
        k.copy_(kh, non_blocking=True)
        v.copy_(vh, non_blocking=True)
        kk, ee = step()
        sc_h.copy_(scores, non_blocking=True)
        kp_h.copy_(kk, non_blocking=True)
        ev_h.copy_(ee, non_blocking=True)
        st_h.copy_(status, non_blocking=True)

    e2e_step()
    torch.cuda.synchronize()
    if dist:
        dist.barrier()
    a0 = torch.cuda.Event(enable_timing=True)
    a1 = torch.cuda.Event(enable_timing=True)
    a0.record()
    for _ in range(E):
        e2e_step()
    a1.record()
    torch.cuda.synchronize()
    e2e_ms = max_over_ranks(a0.elapsed_time(a1), dist, dev) / E
    if dist:
        dist.barrier()
    h2d = sum(t.numel() * t.element_size() for t in (qh, kh, vh))
    d2h = sum(t.numel() * t.element_size() for t in (sc_h, kp_h, ev_h, st_h))

    tokens = sum(wl.lengths)
    return {"value": whole_job_value(world, tokens, e2e_ms), "unit": UNIT,
            "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms}


def run_ours(args):
    import kv_cache_eviction_scores_b200 as dk

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    dist = None
    if world > 1:
        import datetime
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                device_id=torch.device("cuda", local))
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    dk.lib()

    spec = bench_spec(args)
    wl = W.generate(spec, rank_seed(rank))
    q, k, v = wl.q.to(dev), wl.k.to(dev), wl.v.to(dev)
    shape = dk.make_shape(q, k, spec.window, spec.pool)
    path = {dk.PATH_SIMT: "simt", dk.PATH_TENSOR: "tensor"}[
        dk.auto_path(shape) if args.path == "auto" else {"simt": 1, "tensor": 2}[args.path]]
    ws = torch.empty(dk.scores_workspace_bytes(shape), dtype=torch.uint8, device=dev)
    scores = torch.empty(spec.B, spec.Hkv, spec.n_max, dtype=torch.float32, device=dev)
    keep_idx = torch.empty(spec.B, spec.Hkv, max(spec.keep), dtype=torch.int32, device=dev)
    ev_idx = torch.empty(spec.B, spec.Hkv, max(L - kc for L, kc in zip(wl.lengths, wl.keep)),
                         dtype=torch.int32, device=dev)
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    scoring = KERNELS["tensor_attention" if path == "tensor" and args.score == "attention"
                      else path]
    n_launch = dk.scores_select_launches(shape, wl.lengths, path)
    names = scoring + ["k_select"]
    nk = len(names)

    def step(events=None):
        # scoring and eviction in one call of the public API
        _, kk, ee = dk.dropkv_scores_select(
            q, k, v, spec.window, spec.pool, wl.keep, wl.lengths, path=path, score=args.score,
            out=scores, keep_idx=keep_idx, evict_idx=ev_idx, workspace=ws, status=status,
            kernel_events=events)
        return kk, ee

    K, Wm = args.steps, args.warmup
    # K and V are read twice a step; when they fit L2 it is flushed before every
    # timed step (a write of twice its size)
    l2_bytes = int(getattr(torch.cuda.get_device_properties(dev), "L2_cache_size", 0)) or 126 * 2**20
    kv_bytes = 2 * spec.Hkv * sum(wl.lengths) * spec.d * 2
    flush_buf = (torch.empty(2 * l2_bytes, dtype=torch.uint8, device=dev)
                 if kv_bytes <= 2 * l2_bytes else None)
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(2 * nk)] for _ in range(K)]
    for row in ev:
        for e in row:
            e.record()  # creates the handle
    for _ in range(Wm):
        step()
    torch.cuda.synchronize()
    if int(status.item()) != dk.OK:
        raise dk.SingularError(int(status.item()), "bench inputs")
    clocks = ClockSampler(local, enabled=not args.no_clocks)
    clocks.start()
    if dist:
        dist.barrier()
    torch.cuda.synchronize()
    if flush_buf is None:
        # the timed region: K whole steps back to back, only the two bracketing
        # events on the stream (the kernels of a step may overlap one another's
        # tails through programmatic dependent launch)
        t0 = torch.cuda.Event(enable_timing=True)
        t1 = torch.cuda.Event(enable_timing=True)
        t0.record()
        for i in range(K):
            step()
        t1.record()
        torch.cuda.synchronize()
        total = t0.elapsed_time(t1)
    else:
        # inputs that fit L2: every step starts on a flushed L2 (a write larger
        # than L2, outside the step's own pair of events)
        se = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
              for _ in range(K)]
        for i in range(K):
            flush_buf.zero_()
            se[i][0].record()
            step()
            se[i][1].record()
        torch.cuda.synchronize()
        total = sum(a.elapsed_time(b) for a, b in se)
    if dist:
        dist.barrier()
    ms = max_over_ranks(total, dist, dev) / K
    # the per-kernel breakdown: the same K steps again, with events recorded
    # on the launching stream right before and after every kernel
    b0 = torch.cuda.Event(enable_timing=True)
    b1 = torch.cuda.Event(enable_timing=True)
    b0.record()
    for i in range(K):
        if flush_buf is not None:
            flush_buf.zero_()
        step(ev[i])
    b1.record()
    torch.cuda.synchronize()
    if dist:
        dist.barrier()
    clk = clocks.stop()
    ms_events = max_over_ranks(b0.elapsed_time(b1), dist, dev) / K
    kern_us = {}
    for j, name in enumerate(names):
        kern_us[name] = statistics.mean(ev[i][2 * j].elapsed_time(ev[i][2 * j + 1])
                                        for i in range(K)) * 1e3
    if int(status.item()) != dk.OK:
        raise dk.SingularError(int(status.item()), "bench inputs")

    # ---- end to end through the public API, host buffers, copies inside ----
    E = args.e2e_steps if args.e2e_steps is not None else max(3, min(K, 10))
    e2e = None
    if E > 0:
        e2e = run_e2e(dk, wl, q, k, v, scores, status, step, E, dist, dev, world)
    tokens = sum(wl.lengths)
    value = whole_job_value(world, tokens, ms)
    hbm_peak, tc_peak, sm_mhz, peak_src = peaks()
    sel_names = [n for n in names if n.startswith("k_select")]
    dominant = max((n for n in names if n not in sel_names), key=kern_us.get)
    roof = roofline(dominant, spec, kern_us[dominant], hbm_peak, tc_peak, sm_mhz, args.score)
    roof["kernel"] = dominant
    roof["peak_of"] = peak_src
    alg_bytes = kv_bytes + q.numel() * 2 + spec.B * spec.Hkv * spec.n_max * 4
    launches = n_launch

    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": K,
        "warmup": Wm, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16" if path == "tensor" else "f32",
        "data": "synthetic",
        "config": {"workload": workload_desc(spec), "path": path, "score": args.score,
                   "global_batch": spec.B * world,
                   "seq_len": max(spec.lengths),
                   "parallelism": f"replicas x{world} (independent inputs per GPU)",
                   "l2": (f"K+V {kv_bytes / 1e6:.0f} MB > twice the {l2_bytes / 1e6:.0f} MB L2; "
                          "no flush" if flush_buf is None else
                          f"K+V {kv_bytes / 1e6:.0f} MB within twice the {l2_bytes / 1e6:.0f} MB "
                          f"L2: flushed by a {2 * l2_bytes / 1e6:.0f} MB write before every timed "
                          "step, outside the step's events")},
        "token_heads_per_s": value * spec.Hkv,
        "hbm": {"alg_bytes_per_step": alg_bytes,
                "achieved_gbs": alg_bytes / (ms * 1e-3) / 1e9 * 1.0,
                "peak_gbs": hbm_peak, "frac": alg_bytes / (ms * 1e-3) / 1e9 / hbm_peak,
                "of": peak_src,
                "frac_nominal": alg_bytes / (ms * 1e-3) / 1e9 / NOMINAL_HBM_GBS,
                "nominal_gbs": NOMINAL_HBM_GBS},
        "phases_us": {"scores": sum(kern_us[n] for n in names if n not in sel_names),
                      "select": sum(kern_us[n] for n in sel_names)},
        "ms_per_step_with_kernel_events": ms_events,
        "plan": (tensor_plan(spec, torch.cuda.get_device_properties(dev).multi_processor_count)
                 if path == "tensor" else None),
        "roofline": roof,
        "kernels_us": kern_us,
        "e2e": e2e,
        "gpu_launches": launches * K,
        "clocks": clk,
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline and args.score == "perturbation":
        dt, frac, cores, desc = oracle_sample(wl)
        line["cpu_baseline"] = {"value": tokens / (dt / frac), "unit": UNIT, "cores": cores,
                                "kind": "oracle", "sample": desc}
    if rank == 0:
        print(json.dumps(line), flush=True)
    if dist:
        dist.barrier()
        dist.destroy_process_group()
    return 0


def main():
    args = parse()
    if args.impl == "reference":
        return run_reference(args)
    return run_ours(args)


if __name__ == "__main__":
    sys.exit(main())
