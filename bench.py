#!/usr/bin/env python3
"""Benchmark of the AdaFuse fused gated multi-LoRA hot path on B200.

One step = one pass of the whole path on the Llama-2-7B-shaped workload:
  request start : pregate (router on the request's token) -> fused merge of
                  all 224 linears (W' = W + sum_s g_s B_s A_s, one launch);
  batched decode: pregate (first token of each of 64 sequences) -> segment
                  build -> one kernel: shrink, then the fused segmented apply
                  over all 224 linears.
`value` is the merge throughput in GB/s of algorithmic bytes (W read + W'
write + the selected adapters); the apply throughput (tokens/s and GB/s) is
reported beside it.  Inputs are seeded synthetic tensors resident in HBM,
each pass streams far more than the 126 MB L2, so no flush is needed.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

With N > 1 (launched by torch.distributed.run) every rank serves its own
request and batch on its own GPU (independent problems, no data-path
collective); the timed region is bracketed by barriers and its maximum over
ranks is used.  `--impl reference` times the CPU oracle (a bounded sample of
the same workload on the host cores) and prints the same JSON line.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "fused top-k LoRA merge GB/s & % HBM roofline; adapter-apply tokens/s"
FALLBACK_HBM_GBS = 6650.0


def read_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return float(d["hbm_gbs"]), "measured"
    return FALLBACK_HBM_GBS, "fallback"


E2E_CHUNKS = 32          # chunks of layers in the end-to-end merge through host memory
RECORDS = os.path.join(ROOT, "profiles", "records.json")


def kernel_fingerprint(files):
    """First 16 hex digits of the sha256 of the kernel's source files (csrc/)."""
    import hashlib
    h = hashlib.sha256()
    for f in files:
        with open(os.path.join(ROOT, "adapter_merge_b200", "csrc", f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def profile_record(kernel):
    """The ncu figures recorded for `kernel` in profiles/records.json, if its
    sources still hash to the fingerprint recorded with them; else None (the
    counters describe another build)."""
    if not os.path.exists(RECORDS):
        return None
    with open(RECORDS) as fh:
        rec = json.load(fh).get(kernel)
    if not rec or rec.get("kernel_sources_sha256_16") != kernel_fingerprint(rec["sources"]):
        return None
    return rec


def merge_bytes(cfg, k):
    """Algorithmic bytes of one merge: W read + W' write + selected A and B."""
    b = 0
    for l in cfg.linears:
        b += 2 * l.d_out * l.d_in * 2
        b += k * cfg.r * (l.d_in + l.d_out) * 2
    return b


def apply_bytes(cfg, T, U):
    """Algorithmic bytes of one apply: W once, the U touched adapters' A and B,
    x in and y out."""
    b = 0
    for l in cfg.linears:
        b += l.d_out * l.d_in * 2
        b += U * cfg.r * (l.d_in + l.d_out) * 2
        b += T * (l.d_in + l.d_out) * 2
    return b


def max_over_ranks(values, dist=None, device=None):
    """Element-wise maximum of per-rank timings (all ranks must call it)."""
    import torch
    t = torch.tensor(list(values), dtype=torch.float64, device=device)
    if dist is not None and dist.is_initialized() and dist.get_world_size() > 1:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return t.tolist()


def job_throughput(world: int, bytes_per_rank: float, ms: float) -> float:
    """Whole-job GB/s: every rank moved bytes_per_rank in (at most) ms."""
    return world * bytes_per_rank / (ms * 1e-3) / 1e9


class ClockSampler:
    """nvidia-smi clocks/throttle sampling during the timed region."""

    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.f = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.Q}", "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=self.f, stderr=subprocess.DEVNULL)
        except (FileNotFoundError, OSError):
            self.proc = None

    def stop(self):
        if self.proc is None:
            self.f.close()
            os.unlink(self.f.name)
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.f.close()
        rows = []
        with open(self.f.name) as fh:
            for line in fh:
                parts = [p.strip() for p in line.split(",")]
                if len(parts) < 9:
                    continue
                try:
                    rows.append((float(parts[1]), float(parts[2]), float(parts[3]), parts[5:9]))
                except ValueError:
                    continue
        os.unlink(self.f.name)
        if not rows:
            return None
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i, v in enumerate(r[3]) if v.lower() == "active"})
        return {"sm_mhz": statistics.median(r[0] for r in rows), "sm_max_mhz": max(r[1] for r in rows),
                "power_w_max": max(r[2] for r in rows), "samples": len(rows), "reasons": reasons}


class OracleMergeSample:
    """The CPU oracle on a bounded sample of the merge workload: whole rows of
    the first q (4096x4096), gate (11008x4096) and down (4096x11008) linears."""

    def __init__(self, cfg, nthreads: int):
        import numpy as np
        import torch
        import synth
        picks = [0, 4, 6]
        sub = synth.custom([(cfg.linears[i].d_out, cfg.linears[i].d_in) for i in picks], cfg.E, cfg.r, cfg.k, 1,
                           name="cpu-sample")
        w = synth.make_weights(sub, 0, device="cpu")
        self.r = cfg.r
        self.nthreads = nthreads
        self.idx, self.gate = [1, 5], [0.4, 0.3]
        u = lambda t: t.view(torch.int16).numpy().view(np.uint16)
        self.mats = [(u(w.W_views[i]), u(w.A_views[i]), u(w.B_views[i])) for i in range(len(picks))]

    def run(self, rows):
        import oracle
        nbytes = 0
        t0 = time.perf_counter()
        for (W, A, B) in self.mats:
            oracle.merge_linear(W, A, B, self.idx, self.gate, rows=(0, rows), nthreads=self.nthreads)
            nbytes += rows * W.shape[1] * 4 + len(self.idx) * self.r * (rows + W.shape[1]) * 2
        return nbytes, time.perf_counter() - t0

    def calibrate(self, target_s: float) -> int:
        nb, dt = self.run(self.nthreads)
        return int(min(4096, max(self.nthreads, self.nthreads * target_s / max(dt, 1e-6))))


def cpu_oracle_merge(cfg, target_s: float, nthreads: int):
    """(GB/s, seconds, sample) of the CPU oracle on about target_s of work."""
    smp = OracleMergeSample(cfg, nthreads)
    rows = smp.calibrate(target_s)
    nb, dt, passes = 0, 0.0, 0
    while passes == 0 or dt < target_s:
        b, t = smp.run(rows)
        nb, dt, passes = nb + b, dt + t, passes + 1
    return nb / dt / 1e9, dt, f"{passes} x {rows} rows of each of q, gate, down (k=2, r=16)"


def cpu_oracle_apply(cfg, target_s: float, nthreads: int):
    """Tokens/s of the oracle's apply on a bounded sample: whole tokens through
    the q, gate and down linears, scaled to the 224-linear model."""
    import numpy as np
    import torch
    import oracle
    import synth
    picks = [0, 4, 6]
    sub = synth.custom([(cfg.linears[i].d_out, cfg.linears[i].d_in) for i in picks], cfg.E, cfg.r, cfg.k, 8,
                       name="cpu-sample")
    w = synth.make_weights(sub, 0, device="cpu")
    T = nthreads
    X, xs = synth.make_apply_inputs(sub, T, 0)
    idx, gate = synth.random_selection(T, cfg.E, cfg.k, 3)
    u = lambda t: t.view(torch.int16).numpy().view(np.uint16)
    args = [(u(xs[i]), u(w.W_views[i]), u(w.A_views[i]), u(w.B_views[i])) for i in range(len(picks))]
    dt, passes = 0.0, 0
    while passes == 0 or dt < target_s:
        t0 = time.perf_counter()
        for a in args:
            oracle.apply_linear(*a, idx.numpy(), gate.numpy().astype(np.float64), nthreads=nthreads)
        dt += time.perf_counter() - t0
        passes += 1
    # fraction of the model's weight elements the sample covered
    frac = sum(l.d_out * l.d_in for l in sub.linears) / cfg.n_elements
    return passes * T * frac / dt, dt, f"{passes} x {T} tokens through q, gate, down"


def run_reference(args):
    """The reference arm: the CPU oracle as it stands, timed on the host cores."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    import oracle
    import synth
    cfg = synth.llama7b()
    cores = oracle.max_threads()
    smp = OracleMergeSample(cfg, cores)
    rows = smp.calibrate(0.25)
    sample = f"{rows} rows of each of q, gate, down (k=2, r=16)"
    per_step = []
    for s in range(args.warmup + args.steps):
        nb, dt = smp.run(rows)
        if s >= args.warmup:
            per_step.append(nb / dt / 1e9)
    value = statistics.median(per_step)
    line = {
        "impl": "reference", "metric": METRIC, "value": round(value, 4), "unit": "GB/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic (seeded, Llama-2-7B shapes)",
        "config": {"workload": "llama2-7b full-model merge, E=8 r=16 top-2 (sampled rows)"},
        "cpu_baseline": {"value": round(value, 4), "unit": "GB/s", "cores": cores, "kind": "oracle",
                         "sample": sample + " per step"},
        "e2e": {"value": round(value, 4), "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def sweep_point_arg(text):
    """The (E, r, k) of --point "E,r,k" (None for the whole grid); SystemExit
    if it is not a point of the sweep grid."""
    if not text:
        return None
    try:
        pt = tuple(int(v) for v in text.split(","))
    except ValueError:
        pt = ()
    if (len(pt) != 3 or pt[0] not in (4, 8, 16, 32) or pt[1] not in (8, 16, 32, 64) or pt[2] not in (1, 2, 4)
            or pt[2] > pt[0] or pt[1] * pt[2] > 256):
        raise SystemExit(f"--point {text}: not a point of the sweep grid")
    return pt


def chunk_slices(cfg, T, n_chunks):
    """Chunks of consecutive linears for the end-to-end pipelines: per chunk
    (first linear, end linear, and the slices of the flat W, A, B, x and y
    buffers it covers), about n_chunks of them."""
    per = max(1, len(cfg.linears) // n_chunks)
    out = []
    for c0 in range(0, len(cfg.linears), per):
        c1 = min(len(cfg.linears), c0 + per)
        def span(size):
            o = sum(size(l) for l in cfg.linears[:c0])
            return slice(o, o + sum(size(l) for l in cfg.linears[c0:c1]))
        out.append((c0, c1, span(lambda l: l.d_out * l.d_in), span(lambda l: cfg.E * cfg.r * l.d_in),
                    span(lambda l: cfg.E * l.d_out * cfg.r), span(lambda l: T * l.d_in),
                    span(lambda l: T * l.d_out)))
    return out


def measure_sweep(dev, peak, only=None, NC=8, R=5, Ts=(1, 16, 128)):
    """The single-linear 4096 x 4096 grid: E in {4, 8, 16, 32}, r in {8, 16,
    32, 64}, k in {1, 2, 4}; merge per (E, r, k) and apply per T in Ts.  A
    33.5 MB layer fits in the 126 MB L2, so every point rotates through NC
    independent copies (W, W', A, B and a plan each, NC x 100+ MB touched per
    cycle) and each launch finds its operands in HBM.  Per point: the device
    time of one call (CUDA events around it, median of NC * R; a GPU sleep
    queued before the first event keeps the device busy until the host has
    queued the whole call, so host time does not count), the time per call
    when calls run back to back (launch gaps and host time included), and the
    host time of the API call (launch overhead)."""
    import torch
    import adapter_merge_b200 as am
    import synth
    stream = torch.cuda.current_stream()
    SLEEP_CYCLES = 1_000_000              # ~0.5 ms of GPU sleep ahead of each timed call
    points = []
    for E in (4, 8, 16, 32):
        for r in (8, 16, 32, 64):
            for k in (1, 2, 4):
                if k > E or k * r > 256 or (only and (E, r, k) != only):
                    continue
                cfg = synth.sweep_point(E, r, k, 128)
                lin = cfg.linears[0]
                copies = []
                for c in range(NC):
                    w = synth.make_weights(cfg, 7000 + c, device=dev)
                    Wo = torch.empty_like(w.W_views[0])
                    plan = am.Plan([(w.W_views[0], Wo, w.A_views[0], w.B_views[0])], E, r)
                    copies.append((w, Wo, plan))
                # gates = softmax of N(0,1) logits, top-k: the router with an
                # identity W_r makes its logits the synthetic input itself
                xl = torch.zeros((1, 32), dtype=torch.bfloat16, device=dev)
                xl[0, :E] = synth.normal((E,), 1.0, torch.bfloat16, 11, f"sweep-logits-E{E}-r{r}-k{k}").to(dev)
                sel_i, sel_g = am.pregate(xl, torch.eye(E, 32, dtype=torch.float32, device=dev), k)
                idx, gate = sel_i[0], sel_g[0]

                def timed(fn):
                    for c in range(NC):
                        fn(c)
                    torch.cuda.synchronize()
                    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(NC * R)]
                    for i in range(NC * R):
                        torch.cuda._sleep(SLEEP_CYCLES)
                        ev[i][0].record(stream)
                        fn(i % NC)
                        ev[i][1].record(stream)
                    torch.cuda.synchronize()
                    dev_ms = statistics.median(a.elapsed_time(b) for a, b in ev)
                    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                    e0.record(stream)
                    h0 = time.perf_counter()
                    for i in range(NC * R):
                        fn(i % NC)
                    h1 = time.perf_counter()
                    e1.record(stream)
                    torch.cuda.synchronize()
                    return dev_ms, e0.elapsed_time(e1) / (NC * R), (h1 - h0) * 1e6 / (NC * R)

                mb = merge_bytes(cfg, k)
                m_dev, m_b2b, m_host = timed(lambda c: copies[c][2].merge(idx, gate))
                pt = {"E": E, "r": r, "k": k,
                      "merge": {"us": round(m_dev * 1e3, 2), "gbs": round(mb / (m_dev * 1e-3) / 1e9, 1),
                                "frac_of_peak": round(mb / (m_dev * 1e-3) / 1e9 / peak, 3),
                                "back_to_back_us": round(m_b2b * 1e3, 2), "host_us_per_call": round(m_host, 2),
                                "bytes": mb},
                      "apply": []}
                for T in Ts:
                    X, xs = synth.make_apply_inputs(cfg, T, 5, device=dev)
                    ys = [torch.empty((T, lin.d_out), dtype=torch.bfloat16, device=dev)]
                    xp = am.PointerArrays(xs, ys)
                    si, sg = synth.random_selection(T, E, k, 9, f"swa{E}{r}{k}{T}")
                    si, sg = si.to(dev), sg.to(dev)
                    U = int(torch.unique(si).numel())
                    ws = torch.empty(copies[0][2].workspace_bytes(T, k), dtype=torch.uint8, device=dev)
                    ab = apply_bytes(cfg, T, U)
                    a_dev, a_b2b, a_host = timed(lambda c: copies[c][2].apply(xp, None, T, si, sg, ws))
                    pt["apply"].append({"T": T, "U": U, "us": round(a_dev * 1e3, 2),
                                        "gbs": round(ab / (a_dev * 1e-3) / 1e9, 1),
                                        "frac_of_peak": round(ab / (a_dev * 1e-3) / 1e9 / peak, 3),
                                        "tokens_per_s": round(T / (a_dev * 1e-3), 1),
                                        "back_to_back_us": round(a_b2b * 1e3, 2),
                                        "host_us_per_call": round(a_host, 2),
                                        "launches": copies[0][2].last_launches, "bytes": ab})
                for (_, _, plan) in copies:
                    rc, st = plan.status()
                    if rc != 0 or st != 0:
                        raise RuntimeError(f"device status {st} at sweep point E={E} r={r} k={k}")
                    plan.destroy()
                points.append(pt)
                del copies
                torch.cuda.empty_cache()
    return points


def sweep_summary(points, seconds):
    """Medians over the sweep grid: the merge per contraction depth k*r, the
    apply per batch T (device time of one call and its fraction of the peak)."""
    by_kr, by_T = {}, {}
    for p in points:
        by_kr.setdefault(p["k"] * p["r"], []).append(p["merge"])
        for a in p["apply"]:
            by_T.setdefault(a["T"], []).append(a)

    def med(rows):
        return {"us": round(statistics.median(x["us"] for x in rows), 2),
                "frac_of_peak": round(statistics.median(x["frac_of_peak"] for x in rows), 3),
                "frac_min": round(min(x["frac_of_peak"] for x in rows), 3),
                "frac_max": round(max(x["frac_of_peak"] for x in rows), 3), "points": len(rows)}
    return {"merge_by_kr": {str(kr): med(v) for kr, v in sorted(by_kr.items())},
            "apply_by_T": {str(T): med(v) for T, v in sorted(by_T.items())},
            "points": len(points), "seconds": round(seconds, 1),
            "workload": "one 4096x4096 linear, E in {4,8,16,32}, r in {8,16,32,64}, k in {1,2,4}; "
                        "apply at T in {1,16,128}",
            "l2": "8 rotated copies of every operand (no L2 reuse between launches)"}


def run_sweep(args):
    """`--config sweep`: the whole grid (or one --point), one JSON line."""
    import torch
    from adapter_merge_b200 import build as ambuild
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    ambuild.build()
    peak, peak_kind = read_peaks()
    only = sweep_point_arg(args.point)
    t_begin = time.perf_counter()
    points = measure_sweep(dev, peak, only)
    if rank == 0:
        fr = [p["merge"]["frac_of_peak"] for p in points]
        line = {
            "metric": "sweep: fused top-k LoRA merge GB/s per (E, r, k) and apply per T, one 4096x4096 linear",
            "value": round(statistics.median(p["merge"]["gbs"] for p in points), 2), "unit": "GB/s",
            "n_gpus": 1, "higher_is_better": True, "dtype": "bf16",
            "data": "synthetic (seeded; gates = softmax of N(0,1) logits)",
            "config": {"workload": (f"sweep point 4096x4096, E={only[0]}, r={only[1]}, k={only[2]}, T in {{1,16,128}}"
                                    if only else "sweep 4096x4096, E in {4,8,16,32}, r in {8,16,32,64}, "
                                                 "k in {1,2,4}, T in {1,16,128}"),
                       "l2": "8 rotated copies of every operand (no L2 reuse between launches)"},
            "peak": peak, "peak_source": f"{peak_kind} hbm_gbs",
            "merge_frac_of_peak": {"min": min(fr), "median": statistics.median(fr), "max": max(fr)},
            "summary": sweep_summary(points, time.perf_counter() - t_begin),
            "seconds": round(time.perf_counter() - t_begin, 1),
            "points": points,
        }
        print(json.dumps(line), flush=True)
    return 0


def measure_13b(dev, peak, steps=10):
    """The Llama-2-13B-shaped stack (280 linears, E=16, r=32, top-2): the
    full-model merge for one request and the batch-32 segmented apply, each
    preceded by its pregate, device time by CUDA events (mean of `steps`
    after three warm-ups), weights resident."""
    import torch
    import adapter_merge_b200 as am
    import synth
    cfg = synth.llama13b()
    stream = torch.cuda.current_stream()
    w = synth.make_weights(cfg, 1300, device=dev)
    W_out = torch.empty_like(w.W)
    views, o = [], 0
    for l in cfg.linears:
        n = l.d_out * l.d_in
        views.append(W_out[o:o + n].view(l.d_out, l.d_in))
        o += n
    plan = am.Plan(list(zip(w.W_views, views, w.A_views, w.B_views)), cfg.E, cfg.r)
    T = cfg.T_apply
    x_req = synth.make_router_input(cfg, 1, 1300, device=dev, tag="xreq")
    x_first = synth.make_router_input(cfg, T, 1300, device=dev, tag="xfirst")
    X, xs = synth.make_apply_inputs(cfg, T, 1300, device=dev)
    ys = [torch.empty((T, l.d_out), dtype=torch.bfloat16, device=dev) for l in cfg.linears]
    xp = am.PointerArrays(xs, ys)
    ws = torch.empty(plan.workspace_bytes(T, cfg.k), dtype=torch.uint8, device=dev)

    def ev_mean(fn):
        for _ in range(3):
            fn(None)
        torch.cuda.synchronize()
        e = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(steps)]
        for i in range(steps):
            fn(e[i])
        torch.cuda.synchronize()
        return sum(a.elapsed_time(b) for a, b in e) / steps

    def merge(ev):
        i1, g1 = am.pregate(x_req, w.W_r, cfg.k)
        if ev is not None:
            ev[0].record(stream)
        plan.merge(i1[0], g1[0])
        if ev is not None:
            ev[1].record(stream)

    state = {}

    def apply(ev):
        iT, gT = am.pregate(x_first, w.W_r, cfg.k)
        if ev is not None:
            ev[0].record(stream)
        plan.apply(xp, None, T, iT, gT, ws)
        if ev is not None:
            ev[1].record(stream)
        state["idx"] = iT

    m_ms = ev_mean(merge)
    a_ms = ev_mean(apply)
    # in-place switch between two selections (rank 2kr = 128 here)
    sel = [(torch.tensor(i_, dtype=torch.int32, device=dev), torch.tensor(g_, dtype=torch.float32, device=dev))
           for i_, g_ in (((1, 5), (0.4, 0.3)), ((6, 2), (0.5, 0.2)))]
    plan.merge(*sel[0])
    cur = {"i": 0}

    def switch(ev):
        new, old = sel[(cur["i"] + 1) % 2], sel[cur["i"] % 2]
        if ev is not None:
            ev[0].record(stream)
        plan.switch(new[0], new[1], old[0], old[1])
        if ev is not None:
            ev[1].record(stream)
        cur["i"] += 1

    s_ms = ev_mean(switch)
    rc, st = plan.status()
    if rc != 0 or st != 0:
        raise RuntimeError(f"device status {st} in the 13B measurement")
    U = int(torch.unique(state["idx"]).numel())
    mb, ab, sb = merge_bytes(cfg, cfg.k), apply_bytes(cfg, T, U), merge_bytes(cfg, 2 * cfg.k)
    plan.destroy()
    out = {"workload": f"{cfg.name}: {cfg.n_lin} linears, E={cfg.E}, r={cfg.r}, top-{cfg.k}; merge for one "
                       f"request, apply for T={T} sequences",
           "merge": {"ms": round(m_ms, 4), "gbs": round(mb / (m_ms * 1e-3) / 1e9, 1),
                     "frac_of_peak": round(mb / (m_ms * 1e-3) / 1e9 / peak, 4), "bytes": mb,
                     "note": "merge kernel alone (the router launch before it is outside the events)"},
           "apply": {"T": T, "ms": round(a_ms, 4), "tokens_per_s": round(T / (a_ms * 1e-3), 1),
                     "gbs": round(ab / (a_ms * 1e-3) / 1e9, 1),
                     "frac_of_peak": round(ab / (a_ms * 1e-3) / 1e9 / peak, 4), "bytes": ab,
                     "distinct_experts": U, "note": "one apply call (all its launches)"},
           "switch": {"ms": round(s_ms, 4), "gbs": round(sb / (s_ms * 1e-3) / 1e9, 1),
                      "frac_of_peak": round(sb / (s_ms * 1e-3) / 1e9 / peak, 4), "bytes": sb,
                      "note": "W' <- W' - dW(old) + dW(new) in place, one launch, rank 2kr = 128"},
           "steps": steps}
    del w, W_out, X, ys, ws
    torch.cuda.empty_cache()
    return out


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=100)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--config", default="7b", choices=["7b", "13b", "sweep"],
                    help="sweep = the single-linear 4096^2 grid, measured per point (its own JSON line)")
    ap.add_argument("--point", default="",
                    help="with --config sweep: only this E,r,k point (e.g. 8,16,2)")
    ap.add_argument("--layers", type=int, default=0,
                    help="use only the first N layers (small profiling case); 0 = the full model")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-extras", action="store_true",
                    help="skip the switch / per-linear merge / pooled-router / 13B / sweep measurements")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    if args.impl == "reference":
        return run_reference(args)
    if args.point and args.config != "sweep":
        raise SystemExit("--point needs --config sweep")
    if args.config == "sweep":
        sweep_point_arg(args.point)          # reject a point outside the grid before any GPU work
        return run_sweep(args)

    import torch
    import torch.distributed as dist

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)

    from adapter_merge_b200 import build as ambuild
    if rank == 0 or world == 1:
        ambuild.build()
    if world > 1:
        dist.barrier()
    import adapter_merge_b200 as am
    import synth

    if args.config == "7b":
        cfg = synth.llama7b(args.layers) if args.layers else synth.llama7b()
    else:
        cfg = synth.llama13b(args.layers) if args.layers else synth.llama13b()
    seed = 1000 + rank                       # every rank serves its own request and batch
    w = synth.make_weights(cfg, seed, device=dev)
    W_out = torch.empty_like(w.W)
    W_out_views, o = [], 0
    for l in cfg.linears:
        n = l.d_out * l.d_in
        W_out_views.append(W_out[o:o + n].view(l.d_out, l.d_in))
        o += n
    plan = am.Plan(list(zip(w.W_views, W_out_views, w.A_views, w.B_views)), cfg.E, cfg.r)
    T = cfg.T_apply
    x_req = synth.make_router_input(cfg, 1, seed, device=dev, tag="xreq")
    x_first = synth.make_router_input(cfg, T, seed, device=dev, tag="xfirst")
    X, xs = synth.make_apply_inputs(cfg, T, seed, device=dev)
    Y = torch.empty(sum(T * l.d_out for l in cfg.linears), dtype=torch.bfloat16, device=dev)
    ys, o = [], 0
    for l in cfg.linears:
        ys.append(Y[o:o + T * l.d_out].view(T, l.d_out))
        o += T * l.d_out
    xp = am.PointerArrays(xs, ys)
    yp = None
    ws = torch.empty(plan.workspace_bytes(T, cfg.k), dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream()

    def step(ev=None):
        if ev is not None:
            ev[0].record(stream)
        idx1, gate1 = am.pregate(x_req, w.W_r, cfg.k)
        if ev is not None:
            ev[1].record(stream)
        plan.merge(idx1[0], gate1[0])
        if ev is not None:
            ev[2].record(stream)
        idxT, gateT = am.pregate(x_first, w.W_r, cfg.k)
        if ev is not None:
            ev[3].record(stream)
        plan.apply(xp, yp, T, idxT, gateT, ws)
        if ev is not None:
            ev[4].record(stream)
        return idxT

    for _ in range(args.warmup):
        idxT = step()
    torch.cuda.synchronize()
    rc, st = plan.status()
    if rc != 0 or st != 0:
        raise RuntimeError(f"device status {st} after warm-up")
    U = int(torch.unique(idxT).numel())
    apply_launches = plan.last_launches          # 4 (segments, shrink, finalize, apply) or 2

    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(5)] for _ in range(args.steps)]
    t_start = torch.cuda.Event(enable_timing=True)
    t_end = torch.cuda.Event(enable_timing=True)
    sampler = ClockSampler(local if "CUDA_VISIBLE_DEVICES" not in os.environ else
                           int(os.environ["CUDA_VISIBLE_DEVICES"].split(",")[local]))
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    sampler.start()
    time.sleep(0.3)
    t_start.record(stream)
    for i in range(args.steps):
        step(evs[i])
    t_end.record(stream)
    torch.cuda.synchronize()
    clocks = sampler.stop()
    if world > 1:
        dist.barrier()
    total_ms = t_start.elapsed_time(t_end)
    merge_part = [e[0].elapsed_time(e[2]) for e in evs]
    merge_kernel = [e[1].elapsed_time(e[2]) for e in evs]
    apply_part = [e[2].elapsed_time(e[4]) for e in evs]
    apply_call = [e[3].elapsed_time(e[4]) for e in evs]
    rc, st = plan.status()
    if rc != 0 or st != 0:
        raise RuntimeError(f"device status {st} after the timed region")

    def mean(v):
        return sum(v) / len(v)

    total_ms, m_part, m_kern, a_part, a_call = max_over_ranks(
        [total_ms, mean(merge_part), mean(merge_kernel), mean(apply_part), mean(apply_call)], dist, dev)

    mb = merge_bytes(cfg, cfg.k)
    rec_merge = profile_record("merge_rows_kernel")
    rec_apply = profile_record("apply_fused_kernel")
    traffic = None
    if rec_merge and cfg.name == rec_merge.get("full_workload"):
        traffic = rec_merge.get("dram_bytes_per_full_launch")
    ab = apply_bytes(cfg, T, U)
    peak, peak_kind = read_peaks()
    merge_gbs = job_throughput(world, mb, m_part)
    kern_gbs = mb / (m_kern * 1e-3) / 1e9
    apply_tps = world * T / (a_part * 1e-3)
    apply_gbs = ab / (a_call * 1e-3) / 1e9

    # End to end through the public API with HOST buffers: every step copies
    # the call's inputs from pinned host memory to the device and reads its
    # results back, inside the timed region.
    #   merge: W, the adapter stacks and the router input in; W' and the
    #          selection out (PCIe-bound: the whole model crosses twice);
    #   apply: every linear's x and the first tokens in; every y out (the
    #          backbone and adapters stay resident, as in serving).
    # "resident" repeats the merge with only the router input and the
    # selection crossing PCIe.
    e2e = None
    if not args.no_e2e:
        # The full-weight form pins a host copy of W, A, B and W' per rank;
        # every rank takes the same decision (collectives stay in step).
        need = (w.W.numel() + w.A.numel() + w.B.numel() + W_out.numel()) * 2
        local_world = int(os.environ.get("LOCAL_WORLD_SIZE", str(world)))
        try:
            import psutil
            avail = psutil.virtual_memory().available
        except Exception:
            avail = None
        fits = 1.0 if avail is None or avail > 1.25 * need * local_world else 0.0
        full = -max_over_ranks([-fits], dist, dev)[0] > 0.5
        if full:
            h_W = torch.empty(w.W.shape, dtype=w.W.dtype, pin_memory=True)
            h_W.copy_(w.W)
            h_A = torch.empty(w.A.shape, dtype=w.A.dtype, pin_memory=True)
            h_A.copy_(w.A)
            h_B = torch.empty(w.B.shape, dtype=w.B.dtype, pin_memory=True)
            h_B.copy_(w.B)
            h_Wout = torch.empty(W_out.shape, dtype=W_out.dtype, pin_memory=True)
        h_xreq = x_req.cpu().pin_memory()
        h_first = x_first.cpu().pin_memory()
        h_X = X.cpu().pin_memory()
        h_Y = torch.empty(Y.shape, dtype=Y.dtype, pin_memory=True)
        h_sel = torch.empty((4, cfg.k), dtype=torch.float32, pin_memory=True)
        ne = 3

        # With the weights on the host, the merge is pipelined over chunks of
        # layers through the same public calls (one plan and one merge call
        # per chunk): the copy in of chunk c+1, the merge of chunk c and the
        # copy out of chunk c-1 overlap on three streams, so the two PCIe
        # directions run at once.  Only the first chunk's copy in and the
        # last chunk's copy out stand alone, so the chunks are small: about
        # one layer each.
        chunks = []
        if full:
            for (c0, c1, sw_, sa_, sb_, sx_, sy_) in chunk_slices(cfg, T, E2E_CHUNKS):
                cplan = am.Plan(list(zip(w.W_views[c0:c1], W_out_views[c0:c1], w.A_views[c0:c1],
                                         w.B_views[c0:c1])), cfg.E, cfg.r)
                chunks.append((cplan, sw_, sa_, sb_, sx_, sy_, am.PointerArrays(xs[c0:c1], ys[c0:c1])))
            s_in, s_out = torch.cuda.Stream(), torch.cuda.Stream()
            # the chunks' applies run one after another on the stream: one workspace
            ws_c = torch.empty(max(c[0].workspace_bytes(T, cfg.k) for c in chunks), dtype=torch.uint8, device=dev)

        def e2e_merge(ev, resident):
            ev[0].record(stream)
            x_req.copy_(h_xreq, non_blocking=True)
            idx1, gate1 = am.pregate(x_req, w.W_r, cfg.k)
            if resident:
                plan.merge(idx1[0], gate1[0])
            else:
                s_in.wait_stream(stream)
                done_in, done_m = [], []
                for (cplan, sw_, sa_, sb_, _sx, _sy, _xp) in chunks:
                    with torch.cuda.stream(s_in):
                        w.W[sw_].copy_(h_W[sw_], non_blocking=True)
                        w.A[sa_].copy_(h_A[sa_], non_blocking=True)
                        w.B[sb_].copy_(h_B[sb_], non_blocking=True)
                        e_in = torch.cuda.Event()
                        e_in.record(s_in)
                    stream.wait_event(e_in)
                    cplan.merge(idx1[0], gate1[0], stream=stream)
                    e_m = torch.cuda.Event()
                    e_m.record(stream)
                    with torch.cuda.stream(s_out):
                        s_out.wait_event(e_m)
                        h_Wout[sw_].copy_(W_out[sw_], non_blocking=True)
                stream.wait_stream(s_out)
            h_sel[0].copy_(idx1[0].view(torch.float32), non_blocking=True)
            h_sel[1].copy_(gate1[0], non_blocking=True)
            ev[1].record(stream)

        def e2e_apply(ev):
            # x in and y out, pipelined over the same chunks of layers as the
            # merge (the copy in of chunk c+1, the apply of chunk c and the copy
            # out of chunk c-1 overlap) when the chunk plans exist
            ev[0].record(stream)
            x_first.copy_(h_first, non_blocking=True)
            idxT, gateT = am.pregate(x_first, w.W_r, cfg.k)
            if chunks:
                s_in.wait_stream(stream)
                for (cplan, _sw, _sa, _sb, sx_, sy_, xp_c) in chunks:
                    with torch.cuda.stream(s_in):
                        X[sx_].copy_(h_X[sx_], non_blocking=True)
                        e_in = torch.cuda.Event()
                        e_in.record(s_in)
                    stream.wait_event(e_in)
                    cplan.apply(xp_c, None, T, idxT, gateT, ws_c, stream=stream)
                    e_a = torch.cuda.Event()
                    e_a.record(stream)
                    with torch.cuda.stream(s_out):
                        s_out.wait_event(e_a)
                        h_Y[sy_].copy_(Y[sy_], non_blocking=True)
                stream.wait_stream(s_out)
            else:
                X.copy_(h_X, non_blocking=True)
                plan.apply(xp, yp, T, idxT, gateT, ws)
                h_Y.copy_(Y, non_blocking=True)
            h_sel[2].copy_(idxT[0].view(torch.float32), non_blocking=True)
            ev[1].record(stream)

        def timed(fn, n, *a):
            evs_ = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(n)]
            fn([torch.cuda.Event(enable_timing=True) for _ in range(2)], *a)      # warm-up
            torch.cuda.synchronize()
            if world > 1:
                dist.barrier()
            for i in range(n):
                fn(evs_[i], *a)
            torch.cuda.synchronize()
            return mean([e[0].elapsed_time(e[1]) for e in evs_])

        em_m = timed(e2e_merge, ne, False) if full else 0.0
        em_m, em_a, em_r = max_over_ranks([em_m, timed(e2e_apply, 10), timed(e2e_merge, 10, True)], dist, dev)
        h2d_m = (w.W.numel() + w.A.numel() + w.B.numel() + x_req.numel()) * 2
        d2h_m = W_out.numel() * 2 + 2 * cfg.k * 4
        h2d_a = (x_first.numel() + X.numel()) * 2
        d2h_a = Y.numel() * 2 + cfg.k * 4
        if not full:        # host memory too small for a pinned model copy per rank
            em_m = em_r
            h2d_m = x_req.numel() * 2
            d2h_m = 2 * cfg.k * 4
        e2e = {"value": round(job_throughput(world, mb, em_m), 3), "unit": "GB/s",
               "h2d_bytes_per_step": h2d_m + h2d_a, "d2h_bytes_per_step": d2h_m + d2h_a,
               "merge_ms": round(em_m, 3), "merge_h2d_bytes": h2d_m, "merge_d2h_bytes": d2h_m,
               "apply_tokens_per_s": round(world * T / (em_a * 1e-3), 1), "apply_ms": round(em_a, 3),
               "apply_h2d_bytes": h2d_a, "apply_d2h_bytes": d2h_a,
               "resident": {"value": round(job_throughput(world, mb, em_r), 2), "unit": "GB/s",
                            "h2d_bytes_per_step": x_req.numel() * 2, "d2h_bytes_per_step": 2 * cfg.k * 4,
                            "note": "weights and adapters resident; only the router input and the selection cross"},
               "note": ("merge with W, A, B in and W' out through pinned host buffers each step, pipelined "
                        f"over {len(chunks)} chunks of layers (a plan and a merge call per chunk; copies in, merges and "
                        "copies out overlap on three streams); apply with x in and y out, pipelined over the "
                        "same chunks (weights resident)") if full else
                       ("host memory holds no pinned model copy per rank: merge with the router input in and "
                        "the selection out (weights resident); apply with x in and y out")}
        if full:
            for (cplan, *_rest) in chunks:
                cplan.destroy()
            del h_W, h_A, h_B, h_Wout, chunks, ws_c

    # The NEXT rows on the same plan, outside the timed region: in-place switch
    # between two selections (rank 2kr), the one-launch-per-linear merge, and
    # the sequence-level router on the mean of the T first tokens.
    extras = None
    if not args.no_extras:
        sel = [(torch.tensor(a, dtype=torch.int32, device=dev), torch.tensor(g, dtype=torch.float32, device=dev))
               for a, g in (((1, 5), (0.4, 0.3)), ((6, 2), (0.5, 0.2)))]
        if cfg.E < 7:
            sel = sel[:1] + [(sel[0][0].flip(0), sel[0][1].flip(0))]
        plan.merge(*sel[0])

        def ev_mean(fn, n):
            e = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(n)]
            fn(0)
            torch.cuda.synchronize()
            for i in range(n):
                e[i][0].record(stream)
                fn(i + 1)
                e[i][1].record(stream)
            torch.cuda.synchronize()
            return mean([a.elapsed_time(b) for a, b in e])

        def do_switch(i):
            new, old = sel[(i + 1) % 2], sel[i % 2]
            plan.switch(new[0], new[1], old[0], old[1])

        n_sw = 10
        sw_ms = ev_mean(do_switch, n_sw)
        pl_ms = ev_mean(lambda i: plan.merge_per_linear(*sel[0]), 5)
        pool_ms = ev_mean(lambda i: am.pregate(x_first, w.W_r, cfg.k, pool=True), 10)
        sw_ms, pl_ms, pool_ms = max_over_ranks([sw_ms, pl_ms, pool_ms], dist, dev)
        rc, st = plan.status()
        if rc != 0 or st != 0:
            raise RuntimeError(f"device status {st} after the extra measurements")
        sb = merge_bytes(cfg, 2 * cfg.k)
        extras = {
            "switch": {"gbs": round(job_throughput(world, sb, sw_ms), 2), "ms": round(sw_ms, 4), "bytes": sb,
                       "frac_of_peak": round(sb / (sw_ms * 1e-3) / 1e9 / read_peaks()[0], 4),
                       "note": "W' <- W' - dW(old) + dW(new) in place, one launch, rank 2kr"},
            "merge_per_linear": {"gbs": round(job_throughput(world, mb, pl_ms), 2), "ms": round(pl_ms, 4),
                                 "launches": cfg.n_lin,
                                 "vs_fused": round(pl_ms / m_kern, 3),
                                 "note": "one CUDA-core launch per linear, no pipeline (ablation baseline)"},
            "pregate_pooled": {"ms": round(pool_ms, 4), "tokens": T,
                               "note": "one decision from the mean of the T router inputs"},
        }
        if world == 1 and cfg.name == "llama2-7b":
            # The other two model-scale workloads, measured on the same GPU
            # after the 7B model is freed: the 13B stack and the single-layer
            # sweep (per-GPU numbers; replicas would repeat them).
            del w, W_out, W_out_views, X, xs, Y, ys, xp, ws
            plan.destroy()
            plan = None
            torch.cuda.empty_cache()
            extras["llama2_13b"] = measure_13b(dev, peak)
            t_sw = time.perf_counter()
            extras["sweep"] = sweep_summary(measure_sweep(dev, peak, R=3), time.perf_counter() - t_sw)

    cpu = None
    if rank == 0 and not args.no_cpu_baseline:
        import oracle
        cores = oracle.max_threads()
        gbs, dt, sample = cpu_oracle_merge(cfg, 10.0, cores)
        tps, dta, sample_a = cpu_oracle_apply(cfg, 10.0, cores)
        cpu = {"value": round(gbs, 4), "unit": "GB/s", "cores": cores, "kind": "oracle",
               "sample": f"{sample}; {dt:.1f} s",
               "apply_tokens_per_s": round(tps, 3), "apply_sample": f"{sample_a}; {dta:.1f} s"}

    if rank == 0:
        line = {
            "metric": METRIC, "value": round(merge_gbs, 2), "unit": "GB/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(total_ms / args.steps, 4),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic (seeded; Llama-2-7B shapes, random-init weights and adapters)",
            "config": {"workload": f"{cfg.name}: full-model merge for one request ({cfg.n_lin} linears, E={cfg.E}, "
                                   f"r={cfg.r}, top-{cfg.k}) + batched-decode apply (T={T})",
                       "linears": cfg.n_lin, "E": cfg.E, "r": cfg.r, "k": cfg.k, "apply_tokens": T,
                       "parallelism": f"replicas x{world} (independent requests, no collective)",
                       "l2": "no flush: every pass streams > 13 GB, far above the 126 MB L2"},
            "merge": {"gbs": round(merge_gbs, 2), "ms": round(m_part, 4), "kernel_ms": round(m_kern, 4),
                      "bytes": mb, "frac_of_peak": round(kern_gbs / peak, 4)},
            "apply": {"tokens_per_s": round(apply_tps, 1), "ms": round(a_part, 4), "call_ms": round(a_call, 4),
                      "gbs": round(apply_gbs, 2), "bytes": ab, "distinct_experts": U,
                      "frac_of_peak": round(apply_gbs / peak, 4),
                      "launches": apply_launches,
                      "note": ("call = segment build, shrink, finalize, fused apply" if apply_launches == 4 else
                               "call = segment build, fused shrink + apply kernel")},
            "roofline": {"bound": "hbm", "kernel": "merge_rows_kernel", "achieved": round(kern_gbs, 2),
                         "peak": peak, "unit": "GB/s", "frac": round(kern_gbs / peak, 4),
                         "peak_source": f"{peak_kind} hbm_gbs (burst copy)",
                         "algorithmic_bytes": mb,
                         "traffic": traffic,
                         "traffic_source": ("ncu dram__bytes_read.sum + dram__bytes_write.sum of a 2-layer "
                                            "capture of this kernel build, scaled to the full model by "
                                            "elements") if traffic else None},
            "tensor_pipe_pct": {
                "merge_rows_kernel": rec_merge.get("tensor_pipe_pct") if rec_merge else None,
                "apply_fused_kernel": rec_apply.get("tensor_pipe_pct") if rec_apply else None,
                "source": "ncu sm__pipe_tensor_cycles_active (% of peak) of a small capture of this kernel "
                          "build (2-layer merge, 4-layer apply); null when the sources changed since"},
            "gpu_launches": (3 + apply_launches) * args.steps,
            "clocks": clocks,
            "e2e": e2e,
            "cpu_baseline": cpu,
            "extras": extras,
        }
        print(json.dumps(line), flush=True)
    if plan is not None:
        plan.destroy()
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
