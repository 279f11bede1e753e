"""Host-side logic of the benchmark (no GPU): which measurement each command
line reaches, the sweep-point parser, and the clock sampler's summary."""
import os
import sys

import pytest


class _Reached(Exception):
    pass


def test_sweep_point_arg():
    import bench
    assert bench.sweep_point_arg("") is None
    assert bench.sweep_point_arg("8,16,2") == (8, 16, 2)
    assert bench.sweep_point_arg("32,64,4") == (32, 64, 4)
    for bad in ("8,16,3", "4,64,8", "2,16,2", "8,16", "8,16,2,1", "a,b,c", "4,128,2", "1,8,1"):
        with pytest.raises(SystemExit):
            bench.sweep_point_arg(bad)


def _run_main(monkeypatch, argv):
    import bench
    import torch
    seen = []
    monkeypatch.setattr(bench, "run_sweep", lambda args: seen.append(("sweep", args.point)) or 0)
    monkeypatch.setattr(bench, "run_reference", lambda args: seen.append(("reference", args.config)) or 0)

    def stop(*a, **k):
        seen.append(("model", None))
        raise _Reached()
    monkeypatch.setattr(torch.cuda, "set_device", stop)
    monkeypatch.setattr(sys, "argv", ["bench.py"] + argv)
    try:
        bench.main()
    except _Reached:
        pass
    return seen


def test_main_dispatch(monkeypatch):
    assert _run_main(monkeypatch, []) == [("model", None)]
    assert _run_main(monkeypatch, ["--config", "13b"]) == [("model", None)]
    assert _run_main(monkeypatch, ["--config", "sweep"]) == [("sweep", "")]
    assert _run_main(monkeypatch, ["--config", "sweep", "--point", "8,16,2"]) == [("sweep", "8,16,2")]
    assert _run_main(monkeypatch, ["--impl", "reference"]) == [("reference", "7b")]
    with pytest.raises(SystemExit):
        _run_main(monkeypatch, ["--config", "sweep", "--point", "8,16,3"])
    with pytest.raises(SystemExit):
        _run_main(monkeypatch, ["--point", "8,16,2"])


def test_clock_sampler_parses_nvidia_smi(tmp_path, monkeypatch):
    """The sampler's summary of the nvidia-smi CSV it records: median SM
    clock, max clock and power, and every throttle reason seen active (a
    fake nvidia-smi on PATH stands in for the real one)."""
    import time
    import bench
    fake = tmp_path / "nvidia-smi"
    fake.write_text("#!/bin/sh\n"
                    "echo '0, 1900, 1965, 700.5, 0x4, Not Active, Not Active, Not Active, Active'\n"
                    "echo '0, 1800, 1965, 710.0, 0x4, Not Active, Not Active, Not Active, Active'\n"
                    "echo '0, 1950, 1965, 650.0, 0x0, Active, Not Active, Not Active, Not Active'\n"
                    "echo 'garbage line'\n"
                    "exec sleep 30\n")
    fake.chmod(0o755)
    monkeypatch.setenv("PATH", str(tmp_path) + os.pathsep + os.environ.get("PATH", ""))
    s = bench.ClockSampler(0)
    s.start()
    time.sleep(0.5)
    c = s.stop()
    assert c == {"sm_mhz": 1900.0, "sm_max_mhz": 1965.0, "power_w_max": 710.0, "samples": 3,
                 "reasons": ["hw_slowdown", "sw_power_cap"]}


def test_clock_sampler_without_nvidia_smi(tmp_path, monkeypatch):
    import bench
    monkeypatch.setenv("PATH", str(tmp_path))
    s = bench.ClockSampler(0)
    s.start()
    assert s.stop() is None


def test_profile_record_needs_the_recorded_fingerprint(tmp_path, monkeypatch):
    """A profile record is reported only while the kernel's sources hash to
    the fingerprint recorded with it."""
    import json
    import bench
    fp = bench.kernel_fingerprint(["merge.cu", "ptx.cuh"])
    recs = {"merge_rows_kernel": {"sources": ["merge.cu", "ptx.cuh"], "kernel_sources_sha256_16": fp,
                                  "tensor_pipe_pct": 4.0},
            "apply_fused_kernel": {"sources": ["apply.cu"], "kernel_sources_sha256_16": "0" * 16,
                                   "tensor_pipe_pct": 18.0}}
    path = tmp_path / "records.json"
    path.write_text(json.dumps(recs))
    monkeypatch.setattr(bench, "RECORDS", str(path))
    assert bench.profile_record("merge_rows_kernel")["tensor_pipe_pct"] == 4.0
    assert bench.profile_record("apply_fused_kernel") is None
    assert bench.profile_record("no_such_kernel") is None
    monkeypatch.setattr(bench, "RECORDS", str(tmp_path / "absent.json"))
    assert bench.profile_record("merge_rows_kernel") is None


def test_sweep_summary_groups_by_depth_and_batch():
    import bench
    pts = []
    for (E, r, k, us) in ((8, 16, 1, 20.0), (4, 8, 2, 22.0), (8, 16, 2, 30.0)):
        pts.append({"E": E, "r": r, "k": k, "merge": {"us": us, "frac_of_peak": 10.0 / us},
                    "apply": [{"T": T, "us": us + T, "frac_of_peak": 5.0 / (us + T)} for T in (1, 16)]})
    s = bench.sweep_summary(pts, 12.3)
    assert set(s["merge_by_kr"]) == {"16", "32"}
    assert s["merge_by_kr"]["16"]["points"] == 2 and s["merge_by_kr"]["16"]["us"] == 21.0
    assert s["merge_by_kr"]["32"]["us"] == 30.0
    assert s["apply_by_T"]["16"]["points"] == 3 and s["apply_by_T"]["1"]["us"] == 23.0
    assert s["points"] == 3 and s["seconds"] == 12.3


def test_near_tie_report_of_the_bench_router_workloads():
    """The oracle's near-tie report over the router inputs the bench draws
    (the request row and the decode batch of every 7B rank's seed, the 13B
    workload): the workloads with near-tie rows are exactly the ones the GPU
    near-tie test runs, so none is accepted without an exact-order check."""
    import math
    import numpy as np
    import oracle
    import synth
    from helpers import NEAR_TIE_RTOL, NEAR_TIE_SEEDS_7B, u16
    found = []
    for cfg, seeds in ((synth.llama7b(), [1000 + r for r in range(8)]), (synth.llama13b(), [1300])):
        for seed in seeds:
            W_r = synth.make_router_weights(cfg, seed).numpy()
            for tag, T in (("xreq", 1), ("xfirst", cfg.T_apply)):
                x = u16(synth.make_router_input(cfg, T, seed, tag=tag))
                _, _, z = oracle.pregate(x, W_r, cfg.k)
                rel = oracle.topk_margin(z, cfg.k) / oracle.router_scale(x, W_r)
                assert np.all(np.isfinite(rel)) and math.isfinite(float(rel.min()))
                if (rel < NEAR_TIE_RTOL).any():
                    found.append((cfg.name, seed, tag))
    assert found == [("llama2-7b", s, "xfirst") for s in NEAR_TIE_SEEDS_7B]


def test_chunk_slices_tile_every_flat_buffer():
    """The end-to-end pipelines' chunks of layers cover the flat W, A, B, x and
    y buffers exactly once, in order, and each slice matches its linears."""
    import bench
    import synth
    for cfg, T in ((synth.llama7b(), 64), (synth.llama13b(), 32), (synth.tiny(), 8)):
        for n in (1, 8, 32, 1000):
            ch = bench.chunk_slices(cfg, T, n)
            assert ch[0][0] == 0 and ch[-1][1] == len(cfg.linears)
            sizes = (lambda l: l.d_out * l.d_in, lambda l: cfg.E * cfg.r * l.d_in,
                     lambda l: cfg.E * l.d_out * cfg.r, lambda l: T * l.d_in, lambda l: T * l.d_out)
            for b, size in enumerate(sizes):
                end = 0
                for c in ch:
                    sl = c[2 + b]
                    assert sl.start == end
                    assert sl.stop - sl.start == sum(size(l) for l in cfg.linears[c[0]:c[1]])
                    end = sl.stop
                assert end == sum(size(l) for l in cfg.linears)
            for a, b in zip(ch, ch[1:]):
                assert a[1] == b[0]
