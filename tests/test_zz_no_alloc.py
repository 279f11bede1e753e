"""adafuse_apply_noalloc: the segmented apply for callers that cannot allocate
device memory on their hot path (a runtime that gives all GPU memory to its own
pool at start-up, or code that must not call cudaMalloc there because it can
synchronise the device).  Instead of a caller-provided workspace it uses a
fixed 16 MiB array in the library's own device memory.

These tests call it through the C ABI and check it against the regular
adafuse_apply on the same inputs, and against the oracle, on two calls in a
row (the array keeps the previous call's contents, which must not leak into
the next result), and check
that a call too big for the array is refused before anything is launched.
This file is collected last so that a run stopping at its first failure has
already run every other test.
"""
import numpy as np
import pytest
import torch

import oracle
import synth
from helpers import Model, assert_close_bf16, u16

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def am(cuda_device):
    from adapter_merge_b200 import build
    build.build()
    import adapter_merge_b200
    adapter_merge_b200.lib()
    return adapter_merge_b200


def test_noalloc_apply_matches_apply_on_two_calls_in_a_row(am, cuda_device):
    cfg = synth.custom([(384, 520), (136, 264), (256, 256)], 6, 16, 2, 16, name="noalloc")
    m = Model(cfg, cuda_device)
    for T, seed in ((16, 1), (9, 2)):
        X, xs = synth.make_apply_inputs(cfg, T, seed)
        xd = [x.to(cuda_device) for x in xs]
        idx, gate = synth.random_selection(T, cfg.E, cfg.k, seed, "noalloc")
        idx, gate = idx.to(cuda_device), gate.to(cuda_device)
        y_ref = [torch.empty((T, l.d_out), dtype=torch.bfloat16, device=cuda_device) for l in cfg.linears]
        ws = torch.empty(m.plan.workspace_bytes(T, cfg.k), dtype=torch.uint8, device=cuda_device)
        m.plan.apply(xd, y_ref, T, idx, gate, ws)
        y = [torch.full((T, l.d_out), float("nan"), dtype=torch.bfloat16, device=cuda_device)
             for l in cfg.linears]
        rc = m.plan.apply_noalloc(xd, y, T, idx, gate)
        assert rc == 0, am.lib().adafuse_strerror(rc)
        torch.cuda.synchronize()
        for l in range(cfg.n_lin):
            assert_close_bf16(u16(y[l]), u16(y_ref[l]), f"no-alloc apply, call T={T}, linear {l}")
            # and directly against the oracle, so this test stands on its own
            ref = oracle.apply_linear(u16(xs[l]), u16(m.w.W_views[l]), u16(m.w.A_views[l]),
                                      u16(m.w.B_views[l]), idx.cpu().numpy(),
                                      gate.cpu().numpy().astype(np.float64))
            assert_close_bf16(u16(y[l]), ref, f"no-alloc apply vs oracle, call T={T}, linear {l}")
        assert m.plan.status() == (0, 0)


def test_noalloc_apply_refuses_calls_beyond_its_scratch(am, cuda_device):
    # 8 linears with d_in = 16384 and 256 tokens need ~17 MB of shrink partials.
    T = 256
    cfg = synth.custom([(256, 16384)] * 8, 6, 16, 2, T, name="noalloc-big")
    m = Model(cfg, cuda_device)
    assert m.plan.workspace_bytes(T, cfg.k) > 16 << 20
    xd = [torch.zeros((T, l.d_in), dtype=torch.bfloat16, device=cuda_device) for l in cfg.linears]
    y = [torch.full((T, l.d_out), 3.0, dtype=torch.bfloat16, device=cuda_device) for l in cfg.linears]
    idx, gate = synth.random_selection(T, cfg.E, cfg.k, 5, "noalloc-big")
    rc = m.plan.apply_noalloc(xd, y, T, idx.to(cuda_device), gate.to(cuda_device))
    assert rc == am.ERR_WORKSPACE_TOO_SMALL
    torch.cuda.synchronize()
    assert all(bool((t == 3.0).all()) for t in y)      # nothing was launched
