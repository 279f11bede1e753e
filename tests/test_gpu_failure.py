"""Failure detection on the GPU without a fault: a plan created with the
ADAFUSE_PLAN_TEST_STALL hook withholds one shared-memory stage in CTA 0 of the
fused merge, so that a pipeline wait runs out.  The kernel must give up after
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
