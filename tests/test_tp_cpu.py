"""Tensor-parallel sharding (adapter_merge_b200.tp) checked on CPU with the
oracle and two gloo ranks: column shards of the merge and the apply equal
the matching block of the unsharded result bit for bit, row shards of the
merge equal their block of columns, and the row-parallel partial applies,
kept unrounded, all-reduced and rounded once, equal the unsharded apply
within the output tolerance |d| <= 1e-2 |ref| + 1e-3."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from adapter_merge_b200 import tp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _cfg():
    import synth
    lins = (synth.Linear(0, "q", 256, 128), synth.Linear(0, "o", 128, 256),
            synth.Linear(0, "up", 384, 128), synth.Linear(0, "down", 128, 384))
    return synth.Config("tp-small", lins, 128, 4, 8, 2, 1, 5)


def _u16(t):
    return t.contiguous().view(torch.int16).numpy().view(np.uint16)


def _worker(rank, world, port, q):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        import oracle
        import synth
        cfg = _cfg()
        w = synth.make_weights(cfg, 3, device="cpu")
        T = cfg.T_apply
        X, xs = synth.make_apply_inputs(cfg, T, 4)
        sel_i, sel_g = synth.random_selection(T, cfg.E, cfg.k, 5, "tp")
        idx = sel_i.numpy()
        gate = sel_g.numpy().astype(np.float64)
        midx, mgate = [1, 3], [0.4, 0.3]
        out = []
        for l, lin in enumerate(cfg.linears):
            kind = tp.kind_of(lin.name)
            W, A, B = w.W_views[l], w.A_views[l], w.B_views[l]
            full_m = oracle.merge_linear(_u16(W), _u16(A), _u16(B), midx, mgate)
            full_y = oracle.bf16_to_f64(oracle.apply_linear(_u16(xs[l]), _u16(W), _u16(A), _u16(B), idx, gate))
            Ws, As, Bs = tp.shard_weights(kind, W, A, B, rank, world)
            xsh = tp.shard_input(kind, xs[l], rank, world)
            m = oracle.merge_linear(_u16(Ws), _u16(As), _u16(Bs), midx, mgate)
            if kind == tp.COLUMN:
                y = oracle.bf16_to_f64(oracle.apply_linear(_u16(xsh), _u16(Ws), _u16(As), _u16(Bs), idx, gate))
            else:        # the unrounded partial, as a PLAN_Y_F32 plan produces it
                y = oracle.apply_linear_f64(_u16(xsh), _u16(Ws), _u16(As), _u16(Bs), idx, gate)
            yt = tp.reduce_output(kind, torch.from_numpy(y.copy()))
            if kind == tp.COLUMN:
                o0, o1 = tp.block(lin.d_out, rank, world)
                merge_ok = np.array_equal(m, full_m[o0:o1])
                apply_err = float(np.max(np.abs(yt.numpy() - full_y[:, o0:o1])))
                apply_ok = apply_err == 0.0
            else:
                i0, i1 = tp.block(lin.d_in, rank, world)
                merge_ok = np.array_equal(m, full_m[:, i0:i1])
                # the summed partials are rounded once, as the unsharded apply is
                y_sum = oracle.bf16_to_f64(oracle.bf16_from_f64(yt.numpy()))
                err = np.abs(y_sum - full_y)
                apply_err = float(np.max(err))
                apply_ok = bool(np.all(err <= 1e-2 * np.abs(full_y) + 1e-3))
            out.append((lin.name, kind, merge_ok, apply_ok, apply_err))
        q.put((rank, out))
    finally:
        dist.destroy_process_group()


def test_tp_shards_reassemble_the_unsharded_results_gloo():
    import oracle
    oracle.build()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = [q.get(timeout=180) for _ in range(2)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, out in res:
        for name, kind, merge_ok, apply_ok, err in out:
            assert merge_ok, f"rank {rank} {name} ({kind}) merge shard"
            assert apply_ok, f"rank {rank} {name} ({kind}) apply, max error {err}"
    assert any(kind == tp.ROW for _, kind, *_ in res[0][1])


def test_tp_rules_and_blocks():
    assert [tp.kind_of(n) for n in ("q", "k", "v", "o", "gate", "up", "down")] == \
        ["column"] * 3 + ["row"] + ["column"] * 2 + ["row"]
    assert tp.block(11008, 1, 2) == (5504, 11008)
    assert tp.block(4096, 3, 8) == (1536, 2048)
    with pytest.raises(ValueError):
        tp.block(11008, 0, 64)            # shares of 172 are not whole 8-element groups
    with pytest.raises(ValueError):
        tp.kind_of("lm_head")
    W = torch.arange(16 * 24, dtype=torch.float32).view(16, 24)
    A = torch.zeros(2, 8, 24)
    B = torch.zeros(2, 16, 8)
    Ws, As, Bs = tp.shard_weights(tp.COLUMN, W, A, B, 1, 2)
    assert torch.equal(Ws, W[8:]) and As is A and Bs.shape == (2, 8, 8)
    Ws, As, Bs = tp.shard_weights(tp.ROW, W, A, B, 0, 3)
    assert torch.equal(Ws, W[:, :8]) and Ws.is_contiguous() and As.shape == (2, 8, 8) and Bs is B
    import adapter_merge_b200 as am
    assert tp.plan_flags(tp.ROW) == am.PLAN_Y_F32 and tp.plan_flags(tp.COLUMN) == 0
    y = torch.ones(3, 8)
    assert tp.reduce_output(tp.COLUMN, y) is y
    assert tp.reduce_output(tp.ROW, y) is y          # no process group: nothing to sum
