"""Failure detection on the GPU without a fault: a plan created with the
ADAFUSE_PLAN_TEST_STALL hook withholds one shared-memory stage in CTA 0 of the
fused merge (or of the fused apply), so that a pipeline wait runs out.  The kernel must give up after
its bounded wait, free its resources, report ADAFUSE_STATUS_TIMEOUT through the
status word, and leave the context usable for the next (normal) launch."""
import time

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


def test_stalled_merge_times_out_and_reports(am, cuda_device):
    cfg = synth.custom([(512, 384), (256, 136)], 4, 16, 2, 1, name="stall")
    w = synth.make_weights(cfg, 0, device=cuda_device)
    W_out = [torch.zeros_like(t) for t in w.W_views]
    plan = am.Plan(list(zip(w.W_views, W_out, w.A_views, w.B_views)), cfg.E, cfg.r, flags=am.PLAN_TEST_STALL)
    idx = torch.tensor([1, 3], dtype=torch.int32, device=cuda_device)
    gate = torch.tensor([0.5, 0.25], dtype=torch.float32, device=cuda_device)
    t0 = time.time()
    plan.merge(idx, gate)
    rc, st = plan.status()                     # synchronises
    elapsed = time.time() - t0
    assert rc == am.ERR_TIMEOUT
    assert st & am.STATUS_TIMEOUT
    assert elapsed < 60
    assert plan.status() == (0, 0)             # the word was cleared
    plan.destroy()

    # the context is still usable: a normal plan merges correctly
    m = Model(cfg, cuda_device, weights=w)
    m.plan.merge(idx, gate)
    torch.cuda.synchronize()
    assert m.plan.status() == (0, 0)
    for l in range(cfg.n_lin):
        ref = oracle.merge_linear(u16(w.W_views[l]), u16(w.A_views[l]), u16(w.B_views[l]), [1, 3], [0.5, 0.25])
        assert_close_bf16(u16(m.W_out[l]), ref, f"after timeout, linear {l}")


# T = 4: the two-launch form (the other CTAs' waits for the stalled shrink
# output run out as well); T = 24: four launches
@pytest.mark.parametrize("T", [4, 24])
def test_stalled_apply_times_out_and_reports(am, cuda_device, T):
    cfg = synth.custom([(512, 384), (256, 136)], 4, 16, 2, T, name=f"stall-apply{T}")
    w = synth.make_weights(cfg, 1, device=cuda_device)
    W_out = [torch.zeros_like(t) for t in w.W_views]
    X, xs = synth.make_apply_inputs(cfg, T, 2, device=cuda_device)
    ys = [torch.zeros((T, l.d_out), dtype=torch.bfloat16, device=cuda_device) for l in cfg.linears]
    idx, gate = synth.random_selection(T, cfg.E, cfg.k, 3, "stall-apply")
    idx, gate = idx.to(cuda_device), gate.to(cuda_device)
    plan = am.Plan(list(zip(w.W_views, W_out, w.A_views, w.B_views)), cfg.E, cfg.r, flags=am.PLAN_TEST_STALL)
    ws = torch.empty(plan.workspace_bytes(T, cfg.k), dtype=torch.uint8, device=cuda_device)
    t0 = time.time()
    plan.apply(xs, ys, T, idx, gate, ws)
    rc, st = plan.status()                     # synchronises
    elapsed = time.time() - t0
    assert rc == am.ERR_TIMEOUT
    assert st & am.STATUS_TIMEOUT
    assert elapsed < 60
    assert plan.status() == (0, 0)
    plan.destroy()

    # the context and the shared work counters are still usable: a normal
    # plan's apply on the same workspace matches the oracle
    m = Model(cfg, cuda_device, weights=w)
    m.plan.apply(xs, ys, T, idx, gate, ws)
    torch.cuda.synchronize()
    assert m.plan.status() == (0, 0)
    for l in range(cfg.n_lin):
        ref = oracle.apply_linear(u16(xs[l]), u16(w.W_views[l]), u16(w.A_views[l]), u16(w.B_views[l]),
                                  idx.cpu().numpy(), gate.cpu().numpy().astype(np.float64))
        assert_close_bf16(u16(ys[l]), ref, f"after apply timeout, linear {l}")


def test_apply_host_side_faults_are_refused_before_any_launch(am, cuda_device):
    """Host-side fault injection: a workspace one 256-byte block too small, a
    misaligned workspace, an x row that is not 16-byte aligned, an odd y
    pointer, a null x, and k > E are each refused with their error code
    before anything is launched (outputs untouched, status word clean); the
    plan then serves a correct call."""
    cfg = synth.custom([(256, 264), (136, 520)], 5, 16, 2, 8, name="hostfault")
    m = Model(cfg, cuda_device)
    T = 8
    X, xs = synth.make_apply_inputs(cfg, T, 4)
    xs_dev = [x.to(cuda_device) for x in xs]
    ys = [torch.full((T, l.d_out), float("nan"), dtype=torch.bfloat16, device=cuda_device) for l in cfg.linears]
    idx, gate = synth.random_selection(T, cfg.E, cfg.k, 5, "hostfault")
    i_d, g_d = idx.to(cuda_device), gate.to(cuda_device)
    need = m.plan.workspace_bytes(T, cfg.k)
    ws = torch.empty(need + 512, dtype=torch.uint8, device=cuda_device)

    def refused(code, xs_, ys_, ws_, i_=i_d, g_=g_d):
        with pytest.raises(am.AdafuseError) as e:
            m.plan.apply(am.PointerArrays(xs_, ys_), None, T, i_, g_, ws_)
        assert e.value.code == code

    refused(am.ERR_WORKSPACE_TOO_SMALL, xs_dev, ys, ws[:need - 256])
    refused(am.ERR_INVALID_ARG, xs_dev, ys, ws[16:])
    d0 = cfg.linears[0].d_in
    big = torch.zeros(T * d0 + 16, dtype=torch.bfloat16, device=cuda_device)
    refused(am.ERR_UNSUPPORTED, [big[1:1 + T * d0].view(T, d0)] + xs_dev[1:], ys, ws)
    refused(am.ERR_UNSUPPORTED, xs_dev, [ys[0].data_ptr() + 1] + ys[1:], ws)
    refused(am.ERR_INVALID_ARG, [0] + xs_dev[1:], ys, ws)
    wide = torch.zeros((T, cfg.E + 1), dtype=torch.int32, device=cuda_device)
    refused(am.ERR_UNSUPPORTED, xs_dev, ys, ws, wide, torch.zeros((T, cfg.E + 1), device=cuda_device))
    torch.cuda.synchronize()
    for y in ys:
        assert bool(torch.isnan(y.float()).all())
    assert m.plan.status() == (0, 0)

    m.plan.apply(xs_dev, ys, T, i_d, g_d, ws)
    torch.cuda.synchronize()
    for l in range(cfg.n_lin):
        W, A, B = u16(m.w.W_views[l]), u16(m.w.A_views[l]), u16(m.w.B_views[l])
        ref = oracle.apply_linear(u16(xs[l]), W, A, B, idx.numpy(), gate.numpy().astype(np.float64))
        assert_close_bf16(u16(ys[l]), ref, f"after refusals, linear {l}")
    assert m.plan.status() == (0, 0)
