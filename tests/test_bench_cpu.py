"""Host-side argument handling of the benchmark (no GPU): which measurement
each command line reaches, and the sweep-point parser."""
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
