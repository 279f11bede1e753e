"""Tensor-parallel shards on one GPU: the ranks of a two- and a four-way
split are run one after another (their launches never wait on one another),
each with its own plans over its shards: one over the column-parallel
linears (bf16 outputs) and one, built with PLAN_Y_F32, over the
row-parallel linears (fp32 partial outputs).  Column shards of the merge
equal the matching rows of the unsharded merge bit for bit, row shards equal
the matching columns; column shards of the apply match the oracle's columns;
the row-parallel partials, summed in fp32 (what the all-reduce does) and
rounded once by the library's round_bf16, match the oracle's y within the
output tolerance |d| <= 1e-2 |ref| + 1e-3."""
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

    kinds = [tp.kind_of(l.name) for l in lins]
    y_col = [torch.empty((T, l.d_out), dtype=torch.bfloat16, device=dev) for l in lins]
    y_row_sum = [torch.zeros((T, l.d_out), dtype=torch.float32, device=dev) for l in lins]
    for rank in range(world):
        shards = [tp.shard_weights(kd, W, A, B, rank, world)
                  for kd, W, A, B in zip(kinds, w.W_views, w.A_views, w.B_views)]
        outs = [torch.empty_like(Ws) for Ws, _, _ in shards]
        xsh = [tp.shard_input(kd, x, rank, world) for kd, x in zip(kinds, xs)]
        for kind in (tp.COLUMN, tp.ROW):
            sel = [l for l in range(len(lins)) if kinds[l] == kind]
            plan = am.Plan([(shards[l][0], outs[l], shards[l][1], shards[l][2]) for l in sel], cfg.E, cfg.r,
                           flags=tp.plan_flags(kind))
            plan.merge(midx, mgate)
            ydt = torch.float32 if kind == tp.ROW else torch.bfloat16
            ys = [torch.full((T, shards[l][0].shape[0]), float("nan"), dtype=ydt, device=dev) for l in sel]
            ws = torch.empty(plan.workspace_bytes(T, cfg.k), dtype=torch.uint8, device=dev)
            plan.apply([xsh[l] for l in sel], ys, T, idx, gate, ws)
            torch.cuda.synchronize()
            assert plan.status() == (0, 0)
            for l, y in zip(sel, ys):
                if kind == tp.COLUMN:
                    o0, o1 = tp.block(lins[l].d_out, rank, world)
                    y_col[l][:, o0:o1] = y
                else:
                    y_row_sum[l] += y          # the all-reduce's sum, in fp32
            plan.destroy()
        for l, lin in enumerate(lins):
            if kinds[l] == tp.COLUMN:
                o0, o1 = tp.block(lin.d_out, rank, world)
                assert torch.equal(outs[l].view(torch.int16), full_out[l][o0:o1].view(torch.int16)), \
                    f"rank {rank} {lin.name}: merge rows differ from the unsharded merge"
            else:
                i0, i1 = tp.block(lin.d_in, rank, world)
                assert torch.equal(outs[l].view(torch.int16), full_out[l][:, i0:i1].view(torch.int16)), \
                    f"rank {rank} {lin.name}: merge columns differ from the unsharded merge"
    full.destroy()

    for l, lin in enumerate(lins):
        W, A, B = u16(w.W_views[l]), u16(w.A_views[l]), u16(w.B_views[l])
        ref = oracle.apply_linear(u16(xs[l]), W, A, B, sel_i.numpy(), sel_g.numpy().astype(np.float64),
                                  nthreads=8)
        if kinds[l] == tp.COLUMN:
            got = u16(y_col[l])
        else:
            got = u16(tp.reduce_output(tp.ROW, y_row_sum[l], out=torch.empty_like(y_col[l])))
        assert_close_bf16(got, ref, f"tp{world} {lin.name}")


def test_apply_fp32_outputs_are_the_unrounded_accumulators(am, cuda_device):
    """A PLAN_Y_F32 plan writes the fp32 accumulators: they match the oracle's
    unrounded apply within the output tolerance, and rounding them with
    round_bf16 gives, bit for bit, what the same plan without the flag writes
    (same kernels, same summation order, one rounding)."""
    dev = cuda_device
    for T in (5, 64, 200):
        cfg = synth.custom([(384, 520), (136, 4096), (1000, 264)], 6, 16, 2, T, name=f"yf32-{T}")
        w = synth.make_weights(cfg, 3, device=dev)
        X, xs = synth.make_apply_inputs(cfg, T, 4, device=dev)
        idx, gate = synth.random_selection(T, cfg.E, cfg.k, 5, f"yf32-{T}")
        lin = list(zip(w.W_views, [torch.empty_like(W) for W in w.W_views], w.A_views, w.B_views))
        p16 = am.Plan(lin, cfg.E, cfg.r)
        p32 = am.Plan(lin, cfg.E, cfg.r, flags=am.PLAN_Y_F32)
        y16 = [torch.empty((T, l.d_out), dtype=torch.bfloat16, device=dev) for l in cfg.linears]
        y32 = [torch.full((T, l.d_out), float("nan"), dtype=torch.float32, device=dev) for l in cfg.linears]
        ws = torch.empty(p16.workspace_bytes(T, cfg.k), dtype=torch.uint8, device=dev)
        p16.apply(xs, y16, T, idx.to(dev), gate.to(dev), ws)
        p32.apply(xs, y32, T, idx.to(dev), gate.to(dev), ws)
        torch.cuda.synchronize()
        for l in range(cfg.n_lin):
            assert torch.equal(am.round_bf16(y32[l]).view(torch.int16), y16[l].view(torch.int16)), \
                f"T={T} linear {l}: rounded fp32 output differs from the bf16 output"
            ref = oracle.apply_linear_f64(u16(xs[l]), u16(w.W_views[l]), u16(w.A_views[l]), u16(w.B_views[l]),
                                          idx.numpy(), gate.numpy().astype(np.float64), nthreads=8)
            got = y32[l].double().cpu().numpy()
            err = np.abs(got - ref)
            assert np.all(np.isfinite(got)) and np.all(err <= 1e-2 * np.abs(ref) + 1e-3), \
                f"T={T} linear {l}: fp32 output max err {err.max():.3e}"
        assert p16.status() == (0, 0) and p32.status() == (0, 0)
        p16.destroy()
        p32.destroy()


def test_round_bf16_matches_the_oracle_rounding(am, cuda_device):
    """round_bf16 against the oracle's one-step nearest-even rounding (an fp32
    value is exact in fp64, so the two must agree bit for bit): ties both
    ways, subnormals, the largest finite values and overflow to infinity, at
    every alignment of source and destination (scalar head, vector body,
    scalar tail) and sizes from 1 to a multi-wave buffer."""
    dev = cuda_device
    special = np.array([0.0, -0.0, 1.0, -1.0, 1.0 + 2 ** -8, 1.0 + 3 * 2 ** -8, -(1.0 + 2 ** -8),
                        1.0 + 2 ** -8 + 2 ** -20, 2 ** -130, -(2 ** -140), 2 ** -126 * 1.5,
                        3.3895314e38, 3.4028235e38, -3.4028235e38, np.inf, -np.inf, 65504.0, 1e-45],
                       dtype=np.float32)
    rng = np.random.default_rng(3)
    bits = rng.integers(0, 2 ** 32, 1_000_003, dtype=np.uint64).astype(np.uint32)
    vals = bits.view(np.float32).copy()
    vals[np.isnan(vals)] = 1.5
    vals[: special.size] = special
    src_all = torch.from_numpy(vals).to(dev)
    for n in (1, 3, 4, 5, 17, 64, 1000, 1_000_000):
        for si in range(4):
            for oi in range(4):
                src = src_all[si:si + n]
                buf = torch.empty(n + 8, dtype=torch.bfloat16, device=dev)
                out = buf[oi:oi + n]
                am.round_bf16(src, out)
                torch.cuda.synchronize()
                ref = oracle.bf16_from_f64(vals[si:si + n].astype(np.float64))
                assert np.array_equal(u16(out), ref), f"n={n} src+{si} out+{oi}"
    nan = torch.tensor([float("nan")] * 5, dtype=torch.float32, device=dev)
    assert bool(torch.isnan(am.round_bf16(nan).float()).all())
