#!/usr/bin/env python3
"""Benchmark of the AdaFuse fused gated multi-LoRA hot path on B200.

One step = one pass of the whole path on the Llama-2-7B-shaped workload:
  request start : pregate (router on the request's token) -> fused merge of
                  all 224 linears (W' = W + sum_s g_s B_s A_s, one launch);
  batched decode: pregate (first token of each of 64 sequences) -> segment
                  build -> shrink -> fused segmented apply over all 224 linears.
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
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.f.flush()
        rows = []
        for line in open(self.f.name):
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


def cpu_oracle_merge(cfg, target_s: float, nthreads: int):
    """Time the CPU oracle on a bounded sample of the merge workload: whole
    rows of the first q/gate/down linears; returns (GB/s, seconds, sample)."""
    import numpy as np
    import torch
    import oracle
    import synth
    picks = [0, 4, 6]     # q (4096x4096), gate (11008x4096), down (4096x11008)
    sub = synth.custom([(cfg.linears[i].d_out, cfg.linears[i].d_in) for i in picks], cfg.E, cfg.r, cfg.k, 1,
                       name="cpu-sample")
    w = synth.make_weights(sub, 0, device="cpu")
    idx, gate = [1, 5], [0.4, 0.3]
    mats = [(w.W_views[i].view(torch.int16).numpy().view(np.uint16),
             w.A_views[i].view(torch.int16).numpy().view(np.uint16),
             w.B_views[i].view(torch.int16).numpy().view(np.uint16)) for i in range(len(picks))]

    def run(rows):
        nbytes = 0
        t0 = time.perf_counter()
        for (W, A, B) in mats:
            oracle.merge_linear(W, A, B, idx, gate, rows=(0, rows), nthreads=nthreads)
            nbytes += rows * W.shape[1] * 4 + len(idx) * cfg.r * (rows + W.shape[1]) * 2
        return nbytes, time.perf_counter() - t0

    nb, dt = run(nthreads)
    rows = max(nthreads, int(nthreads * target_s / max(dt, 1e-6)))
    rows = min(rows, 4096)
    nb, dt = run(rows)
    return nb / dt / 1e9, dt, f"{rows} rows of each of q, gate, down (k=2, r=16)"


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
    t0 = time.perf_counter()
    for i in range(len(picks)):
        oracle.apply_linear(xs[i].view(torch.int16).numpy().view(np.uint16),
                            w.W_views[i].view(torch.int16).numpy().view(np.uint16),
                            w.A_views[i].view(torch.int16).numpy().view(np.uint16),
                            w.B_views[i].view(torch.int16).numpy().view(np.uint16),
                            idx.numpy(), gate.numpy().astype(np.float64), nthreads=nthreads)
    dt = time.perf_counter() - t0
    # fraction of the model's weight elements the sample covered
    frac = sum(l.d_out * l.d_in for l in sub.linears) / cfg.n_elements
    return T * frac / dt, dt, f"{T} tokens through q, gate, down"


def run_reference(args):
    """The reference arm: the CPU oracle as it stands, timed on the host cores."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    import oracle
    import synth
    cfg = synth.llama7b()
    cores = oracle.max_threads()
    per_step = []
    nbytes_total = 0
    sample = ""
    for s in range(args.warmup + args.steps):
        gbs, dt, sample = cpu_oracle_merge(cfg, 0.25, cores)
        if s >= args.warmup:
            per_step.append(gbs)
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


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=100)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--config", default="7b", choices=["7b", "13b"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    if args.impl == "reference":
        return run_reference(args)

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

    cfg = synth.llama7b() if args.config == "7b" else synth.llama13b()
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
    xp, yp = am.pointer_table(xs, dev), am.pointer_table(ys, dev)
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

    times = torch.tensor([total_ms, mean(merge_part), mean(merge_kernel), mean(apply_part), mean(apply_call)],
                         dtype=torch.float64, device=dev)
    if world > 1:
        dist.all_reduce(times, op=dist.ReduceOp.MAX)
    total_ms, m_part, m_kern, a_part, a_call = times.tolist()

    mb = merge_bytes(cfg, cfg.k)
    ab = apply_bytes(cfg, T, U)
    peak, peak_kind = read_peaks()
    merge_gbs = world * mb / (m_part * 1e-3) / 1e9
    kern_gbs = mb / (m_kern * 1e-3) / 1e9
    apply_tps = world * T / (a_part * 1e-3)
    apply_gbs = ab / (a_call * 1e-3) / 1e9

    # end to end through the public API with host buffers: H2D of each step's
    # inputs from pinned memory, D2H of its results, inside the timed region.
    e2e = None
    if not args.no_e2e:
        h_xreq = x_req.cpu().pin_memory()
        h_first = x_first.cpu().pin_memory()
        h_X = X.cpu().pin_memory()
        h_Y = torch.empty(Y.shape, dtype=Y.dtype).pin_memory()
        h_sel = torch.empty((2 + 2 * T, cfg.k), dtype=torch.float32).pin_memory()
        ne = max(5, min(30, args.steps))

        def e2e_step(ev):
            ev[0].record(stream)
            x_req.copy_(h_xreq, non_blocking=True)
            idx1, gate1 = am.pregate(x_req, w.W_r, cfg.k)
            plan.merge(idx1[0], gate1[0])
            h_sel[0].copy_(idx1[0].view(torch.float32), non_blocking=True)
            h_sel[1].copy_(gate1[0], non_blocking=True)
            ev[1].record(stream)
            x_first.copy_(h_first, non_blocking=True)
            X.copy_(h_X, non_blocking=True)
            idxT, gateT = am.pregate(x_first, w.W_r, cfg.k)
            plan.apply(xp, yp, T, idxT, gateT, ws)
            h_Y.copy_(Y, non_blocking=True)
            ev[2].record(stream)

        for _ in range(2):
            e2e_step([torch.cuda.Event(enable_timing=True) for _ in range(3)])
        torch.cuda.synchronize()
        eev = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(ne)]
        if world > 1:
            dist.barrier()
        for i in range(ne):
            e2e_step(eev[i])
        torch.cuda.synchronize()
        em = torch.tensor([mean([e[0].elapsed_time(e[1]) for e in eev]),
                           mean([e[1].elapsed_time(e[2]) for e in eev])], dtype=torch.float64, device=dev)
        if world > 1:
            dist.all_reduce(em, op=dist.ReduceOp.MAX)
        em_m, em_a = em.tolist()
        h2d = x_req.numel() * 2 + x_first.numel() * 2 + X.numel() * 2
        d2h = 2 * cfg.k * 4 + Y.numel() * 2
        e2e = {"value": round(world * mb / (em_m * 1e-3) / 1e9, 2), "unit": "GB/s",
               "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
               "apply_tokens_per_s": round(world * T / (em_a * 1e-3), 1),
               "note": "merge part: router input H2D + pregate + merge + selection D2H; "
                       "apply part: x H2D + pregate + apply + y D2H (pinned host buffers)"}

    cpu = None
    if rank == 0 and not args.no_cpu_baseline:
        import oracle
        cores = oracle.max_threads()
        gbs, dt, sample = cpu_oracle_merge(cfg, 10.0, cores)
        tps, dta, sample_a = cpu_oracle_apply(cfg, 5.0, cores)
        cpu = {"value": round(gbs, 4), "unit": "GB/s", "cores": cores, "kind": "oracle",
               "sample": f"{sample}; {dt:.1f} s",
               "apply_tokens_per_s": round(tps, 3), "apply_sample": f"{sample_a}; {dta:.1f} s"}

    if rank == 0:
        line = {
            "metric": METRIC, "value": round(merge_gbs, 2), "unit": "GB/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(total_ms / args.steps, 4),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic (seeded; Llama-2-7B shapes, random-init weights and adapters)",
            "config": {"workload": f"{cfg.name}: full-model merge for one request (224 linears, E={cfg.E}, "
                                   f"r={cfg.r}, top-{cfg.k}) + batched-decode apply (T={T})",
                       "linears": cfg.n_lin, "E": cfg.E, "r": cfg.r, "k": cfg.k, "apply_tokens": T,
                       "parallelism": f"replicas x{world} (independent requests, no collective)",
                       "l2": "no flush: every pass streams > 13 GB, far above the 126 MB L2"},
            "merge": {"gbs": round(merge_gbs, 2), "ms": round(m_part, 4), "kernel_ms": round(m_kern, 4),
                      "bytes": mb, "frac_of_peak": round(kern_gbs / peak, 4)},
            "apply": {"tokens_per_s": round(apply_tps, 1), "ms": round(a_part, 4), "call_ms": round(a_call, 4),
                      "gbs": round(apply_gbs, 2), "bytes": ab, "distinct_experts": U,
                      "frac_of_peak": round(apply_gbs / peak, 4),
                      "note": "call = segments + shrink + fused apply (3 launches)"},
            "roofline": {"bound": "hbm", "kernel": "merge_fused_kernel", "achieved": round(kern_gbs, 2),
                         "peak": peak, "unit": "GB/s", "frac": round(kern_gbs / peak, 4),
                         "peak_source": f"{peak_kind} hbm_gbs", "traffic": None},
            "gpu_launches": 6 * args.steps,
            "clocks": clocks,
            "e2e": e2e,
            "cpu_baseline": cpu,
        }
        print(json.dumps(line), flush=True)
    plan.destroy()
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
