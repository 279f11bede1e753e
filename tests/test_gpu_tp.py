"""Tensor-parallel shards on one GPU: the ranks of a two- and a four-way
split are run one after another (their launches never wait on one another),
each with its own plan over its shards.  Column shards of the merge equal
the matching rows of the unsharded merge bit for bit, row shards equal the
matching columns; column shards of the apply match the oracle's columns,
and the sum of the row-parallel partials matches the oracle's y within the
output tolerance plus half an ulp of every bf16 partial."""
import numpy as np
import pytest
import torch

import oracle
import synth
from adapter_merge_b200 import tp
from helpers import assert_close_bf16, u16

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def am(cuda_device):
    from adapter_merge_b200 import build
    build.build()
    import adapter_merge_b200
    adapter_merge_b200.lib()
    return adapter_merge_b200


def _half_ulp_bf16(v):
    a = np.abs(v)
    e = np.floor(np.log2(np.where(a > 0, a, 1.0)))
    return np.where(a > 0, 2.0 ** (e - 8), 0.0)


@pytest.mark.parametrize("world", [2, 4])
def test_tp_shards_on_one_gpu(am, cuda_device, world):
    dev = cuda_device
    lins = (synth.Linear(0, "q", 512, 256), synth.Linear(0, "o", 256, 512),
            synth.Linear(0, "up", 1024, 256), synth.Linear(0, "down", 256, 1024))
    T = 24
    cfg = synth.Config(f"tp-gpu-{world}", lins, 256, 6, 16, 2, 1, T)
    w = synth.make_weights(cfg, 7, device=dev)
    X, xs = synth.make_apply_inputs(cfg, T, 8, device=dev)
    sel_i, sel_g = synth.random_selection(T, cfg.E, cfg.k, 9, "tp-gpu")
    idx, gate = sel_i.to(dev), sel_g.to(dev)
    midx = torch.tensor([4, 1], dtype=torch.int32, device=dev)
    mgate = torch.tensor([0.45, 0.35], dtype=torch.float32, device=dev)

    full_out = [torch.empty_like(W) for W in w.W_views]
    full = am.Plan(list(zip(w.W_views, full_out, w.A_views, w.B_views)), cfg.E, cfg.r)
    full.merge(midx, mgate)
    torch.cuda.synchronize()

    y_sum = [np.zeros((T, l.d_out)) for l in lins]
    bound = [np.zeros((T, l.d_out)) for l in lins]
    for rank in range(world):
        shards = [tp.shard_weights(tp.kind_of(l.name), W, A, B, rank, world)
                  for l, W, A, B in zip(lins, w.W_views, w.A_views, w.B_views)]
        outs = [torch.empty_like(Ws) for Ws, _, _ in shards]
        plan = am.Plan([(Ws, O, As, Bs) for (Ws, As, Bs), O in zip(shards, outs)], cfg.E, cfg.r)
        plan.merge(midx, mgate)
        xsh = [tp.shard_input(tp.kind_of(l.name), x, rank, world) for l, x in zip(lins, xs)]
        ys = [torch.empty((T, Ws.shape[0]), dtype=torch.bfloat16, device=dev) for Ws, _, _ in shards]
        ws = torch.empty(plan.workspace_bytes(T, cfg.k), dtype=torch.uint8, device=dev)
        plan.apply(xsh, ys, T, idx, gate, ws)
        torch.cuda.synchronize()
        assert plan.status() == (0, 0)
        for l, lin in enumerate(lins):
            kind = tp.kind_of(lin.name)
            if kind == tp.COLUMN:
                o0, o1 = tp.block(lin.d_out, rank, world)
                assert torch.equal(outs[l].view(torch.int16), full_out[l][o0:o1].view(torch.int16)), \
                    f"rank {rank} {lin.name}: merge rows differ from the unsharded merge"
                y_sum[l][:, o0:o1] = oracle.bf16_to_f64(u16(ys[l]))
            else:
                i0, i1 = tp.block(lin.d_in, rank, world)
                assert torch.equal(outs[l].view(torch.int16), full_out[l][:, i0:i1].view(torch.int16)), \
                    f"rank {rank} {lin.name}: merge columns differ from the unsharded merge"
                part = oracle.bf16_to_f64(u16(ys[l]))
                y_sum[l] += part
                bound[l] += _half_ulp_bf16(part)
        plan.destroy()
    full.destroy()

    for l, lin in enumerate(lins):
        W, A, B = u16(w.W_views[l]), u16(w.A_views[l]), u16(w.B_views[l])
        ref = oracle.apply_linear(u16(xs[l]), W, A, B, sel_i.numpy(), sel_g.numpy().astype(np.float64),
                                  nthreads=8)
        if tp.kind_of(lin.name) == tp.COLUMN:
            assert_close_bf16(oracle.bf16_from_f64(y_sum[l]), ref, f"tp{world} {lin.name}")
        else:
            r = oracle.bf16_to_f64(ref)
            err = np.abs(y_sum[l] - r)
            tol = 1e-2 * np.abs(r) + 1e-3 + bound[l]
            assert np.all(err <= tol), f"tp{world} {lin.name}: max err {err.max():.3e}"
