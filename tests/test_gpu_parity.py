"""GPU parity: the CUDA path (through the C ABI) against the CPU oracle on
the same seeded inputs.

Acceptance: expert indices bit-exact; gates |d| <= 1e-6 + 1e-5 |g|; bf16
outputs |d| <= 1e-2 |ref| + 1e-3 elementwise, and for the merge also the
delta check in Frobenius norm (helpers.assert_delta_frobenius).
"""
import concurrent.futures
import os

import numpy as np
import pytest
import torch

import oracle
import synth
from helpers import (ATOL, NEAR_TIE_RTOL, NEAR_TIE_SEEDS_7B, RTOL, Model, assert_close_bf16,
                     assert_delta_frobenius, block_rows, f64, merge_delta_bound_ok, take_experts, u16)

pytestmark = pytest.mark.gpu

GATE_ATOL, GATE_RTOL = 1e-6, 1e-5


@pytest.fixture(scope="module")
def am(cuda_device):
    from adapter_merge_b200 import build
    build.build()
    import adapter_merge_b200
    adapter_merge_b200.lib()
    return adapter_merge_b200


def to_dev(t, dev):
    return t.to(dev)


def check_gates(g_gpu, g_ref):
    g_gpu = np.asarray(g_gpu, dtype=np.float64)
    assert np.all(np.abs(g_gpu - g_ref) <= GATE_ATOL + GATE_RTOL * np.abs(g_ref))


# ------------------------------------------------------------------ router

@pytest.mark.parametrize("H,E,T,k,bias,renorm", [
    (256, 4, 8, 2, False, False),       # tiny
    (4096, 8, 64, 2, False, False),     # 7B decode: first token of 64 sequences
    (4096, 8, 1, 2, False, True),       # 7B request start, renormalised gates
    (5120, 16, 32, 2, True, False),     # 13B with a router bias
    (300, 32, 17, 4, False, False),     # E = 32 lanes, ragged H
    (100, 5, 3, 5, True, True),         # k = E
    (8, 1, 2, 1, False, False),         # single expert
    (4096, 8, 2000, 2, False, False),   # 2000 decisions: many waves of CTAs
])
def test_pregate_matches_oracle(am, cuda_device, H, E, T, k, bias, renorm):
    x = synth.normal((T, H), 1.0, torch.bfloat16, 1, f"px{H}{E}{T}")
    W_r = synth.normal((E, H), H ** -0.5, torch.float32, 1, f"pw{H}{E}")
    b_r = synth.normal((E,), 0.5, torch.float32, 1, f"pb{E}") if bias else None
    idx_ref, gate_ref, z = oracle.pregate(u16(x), W_r.numpy(), k, None if b_r is None else b_r.numpy(), renorm)
    idx, gate = am.pregate(x.to(cuda_device), W_r.to(cuda_device), k,
                           None if b_r is None else b_r.to(cuda_device), renorm=renorm)
    torch.cuda.synchronize()
    assert np.array_equal(idx.cpu().numpy(), idx_ref)
    check_gates(gate.cpu().numpy(), gate_ref)


# The 7B bench decode batches with near-tie rows (see the near-tie report in
# the CPU tests): the GPU router adds the products in the oracle's order, so
# even where the k-th and (k+1)-th logits nearly tie the selection matches.
@pytest.mark.parametrize("seed", NEAR_TIE_SEEDS_7B)
def test_pregate_near_tie_rows_of_the_decode_batch(am, cuda_device, seed):
    cfg = synth.llama7b()
    W_r = synth.make_router_weights(cfg, seed)
    x = synth.make_router_input(cfg, cfg.T_apply, seed, tag="xfirst")
    idx_ref, gate_ref, z = oracle.pregate(u16(x), W_r.numpy(), cfg.k)
    rel = oracle.topk_margin(z, cfg.k) / oracle.router_scale(u16(x), W_r.numpy())
    assert (rel < NEAR_TIE_RTOL).any()
    idx, gate = am.pregate(x.to(cuda_device), W_r.to(cuda_device), cfg.k)
    torch.cuda.synchronize()
    assert np.array_equal(idx.cpu().numpy(), idx_ref)
    check_gates(gate.cpu().numpy(), gate_ref)


def test_pregate_ties_nan_and_strided_rows(am, cuda_device):
    H, E, T, k = 64, 6, 5, 3
    W_r = synth.normal((E, H), 0.125, torch.float32, 2, "tw")
    W_r[3] = W_r[1]                  # experts 1 and 3 always tie: 1 must win
    W_r[4, 7] = float("nan")         # expert 4's logit is NaN: ranked last, gate 0
    big = synth.normal((T, 2 * H + 8), 1.0, torch.bfloat16, 2, "tx")
    x = big[:, 8:8 + H]              # row stride 2H+8
    idx_ref, gate_ref, _ = oracle.pregate(u16(x.contiguous()), W_r.numpy(), k)
    dev = big.to(cuda_device)
    idx, gate = am.pregate(dev[:, 8:8 + H], W_r.to(cuda_device), k)
    torch.cuda.synchronize()
    assert np.array_equal(idx.cpu().numpy(), idx_ref)
    check_gates(gate.cpu().numpy(), gate_ref)
    idx5, gate5 = am.pregate(dev[:, 8:8 + H], W_r.to(cuda_device), E)
    i5 = idx5.cpu().numpy()
    assert np.all(i5[:, -1] == 4)
    assert np.all(gate5.cpu().numpy()[:, -1] == 0)


@pytest.mark.parametrize("T", [1, 7, 64])
def test_pregate_pooled_sequence_decision(am, cuda_device, T):
    H, E, k = 4096, 8, 2
    x = synth.normal((T, H), 1.0, torch.bfloat16, 3, f"pool{T}")
    W_r = synth.normal((E, H), H ** -0.5, torch.float32, 3, "poolw")
    idx_ref, gate_ref, _ = oracle.pregate(u16(x), W_r.numpy(), k, pool=True)
    idx, gate = am.pregate(x.to(cuda_device), W_r.to(cuda_device), k, pool=True)
    torch.cuda.synchronize()
    assert idx.shape == (1, k)
    assert np.array_equal(idx.cpu().numpy(), idx_ref)
    check_gates(gate.cpu().numpy(), gate_ref)


# ---------------------------------------------------------------- segments

@pytest.mark.parametrize("T,k,E", [(1, 1, 1), (8, 2, 4), (64, 2, 8), (300, 4, 6), (2000, 2, 32)])
def test_segments_match_oracle(am, cuda_device, T, k, E):
    g = torch.Generator().manual_seed(T * 131 + E)
    idx = torch.randint(0, E, (T, k), generator=g, dtype=torch.int32)
    if T > 4:
        idx[2, 0] = E + 5
        idx[3, k - 1] = -1
    off_ref, perm_ref, bad = oracle.segments(idx.numpy(), E)
    status = torch.zeros(1, dtype=torch.int32, device=cuda_device)
    off, perm, used = am.segments(idx.to(cuda_device), E, status=status)
    torch.cuda.synchronize()
    assert np.array_equal(off.cpu().numpy(), off_ref)
    assert np.array_equal(perm.cpu().numpy()[: len(perm_ref)], perm_ref)
    counts = np.diff(off_ref)
    u = used.cpu().numpy()
    assert u[0] == int((counts > 0).sum())
    assert np.array_equal(u[1:1 + u[0]], np.nonzero(counts)[0])
    assert int(status.item()) == (am.STATUS_BAD_INDEX if bad else 0)


# ------------------------------------------------------------------- merge

def run_merge(am, model, idx, gate, dev, per_linear=False):
    i = torch.as_tensor(np.asarray(idx, dtype=np.int32)).to(dev)
    g = torch.as_tensor(np.asarray(gate, dtype=np.float32)).to(dev)
    if per_linear:
        model.plan.merge_per_linear(i, g)
    else:
        model.plan.merge(i, g)
    torch.cuda.synchronize()


def check_merge(model, idx, gate, what, rows=None, delta=True):
    for l, lin in enumerate(model.cfg.linears):
        rr = (0, lin.d_out) if rows is None else rows(lin)
        W = u16(model.w.W_views[l])
        A, B = u16(model.w.A_views[l]), u16(model.w.B_views[l])
        ref = oracle.merge_linear(W, A, B, idx, gate, rows=rr, nthreads=8)
        got = u16(model.W_out[l][rr[0]:rr[1]])
        assert_close_bf16(got, ref, f"{what} linear {l}")
        if delta:
            dz = oracle.merge_linear(np.zeros_like(W), A, B, idx, gate, rows=rr, nthreads=8)
            assert_delta_frobenius(got, W[rr[0]:rr[1]], ref, dz, f"{what} linear {l}")


def test_merge_tiny_chain_with_pregate(am, cuda_device):
    """Tiny config end to end: the router's decision for token 0 drives the
    merge of all four linears (decide once, apply everywhere)."""
    cfg = synth.tiny()
    m = Model(cfg, cuda_device, weights=None)
    xr = synth.make_router_input(cfg, cfg.T_merge, 0)
    idx_ref, gate_ref, _ = oracle.pregate(u16(xr), m.w.W_r.cpu().numpy(), cfg.k)
    idx, gate = am.pregate(xr.to(cuda_device), m.w.W_r, cfg.k)
    m.plan.merge(idx[0], gate[0])
    torch.cuda.synchronize()
    assert np.array_equal(idx.cpu().numpy(), idx_ref)
    check_merge(m, idx_ref[0], gate_ref[0], "tiny")
    rc, st = m.plan.status()
    assert rc == 0 and st == 0
    assert m.plan.last_launches == 1


SHAPES = [(640, 392), (8, 8), (136, 1000), (256, 256), (1000, 72), (128, 136)]


@pytest.mark.parametrize("E,r,k", [(5, 16, 2), (4, 8, 1), (8, 64, 4), (6, 32, 3), (32, 8, 2), (32, 16, 8),
                                   (12, 48, 2), (1, 16, 1), (4, 256, 1)])
def test_merge_shapes_and_ranks(am, cuda_device, E, r, k):
    cfg = synth.custom(SHAPES, E, r, k, 1, name=f"mshape{E}{r}{k}")
    m = Model(cfg, cuda_device)
    idx, gate = synth.random_selection(1, E, k, 7, f"msel{E}{r}{k}")
    run_merge(am, m, idx[0], gate[0], cuda_device)
    check_merge(m, idx[0].numpy(), gate[0].numpy().astype(np.float64), f"E{E} r{r} k{k}")


def test_merge_zero_backbone_isolates_delta(am, cuda_device):
    cfg = synth.custom([(384, 520), (200, 136)], 4, 16, 2, 1, name="mzero")
    m = Model(cfg, cuda_device, zero_w=True)
    idx, gate = np.array([2, 0]), np.array([0.6, 0.3], dtype=np.float32)
    run_merge(am, m, idx, gate, cuda_device)
    check_merge(m, idx, gate.astype(np.float64), "zero W", delta=False)


def test_merge_poison_unselected_adapters(am, cuda_device):
    cfg = synth.custom([(384, 264)], 6, 16, 2, 1, name="mpoison")
    m = Model(cfg, cuda_device)
    idx, gate = np.array([4, 1]), np.array([0.5, 0.25], dtype=np.float32)
    run_merge(am, m, idx, gate, cuda_device)
    clean = m.W_out[0].clone()
    for e in (0, 2, 3, 5):
        m.w.A_views[0][e].fill_(float("nan"))
        m.w.B_views[0][e].fill_(float("nan"))
    run_merge(am, m, idx, gate, cuda_device)
    assert torch.equal(m.W_out[0].view(torch.int16), clean.view(torch.int16))


def test_merge_in_place_and_deterministic(am, cuda_device):
    cfg = synth.custom([(512, 384), (136, 264)], 4, 16, 2, 1, name="minpl")
    m = Model(cfg, cuda_device)
    idx, gate = np.array([3, 1]), np.array([0.4, 0.35], dtype=np.float32)
    run_merge(am, m, idx, gate, cuda_device)
    out1 = [t.clone() for t in m.W_out]
    run_merge(am, m, idx, gate, cuda_device)
    for a, b in zip(out1, m.W_out):
        assert torch.equal(a.view(torch.int16), b.view(torch.int16))
    mi = Model(cfg, cuda_device, in_place=True, weights=synth.make_weights(cfg, 0, device=cuda_device))
    run_merge(am, mi, idx, gate, cuda_device)
    for a, b in zip(out1, mi.W_out):
        assert torch.equal(a.view(torch.int16), b.view(torch.int16))


def test_merge_bad_index_skipped_and_flagged(am, cuda_device):
    cfg = synth.custom([(256, 136)], 4, 8, 2, 1, name="mbad")
    m = Model(cfg, cuda_device)
    idx, gate = np.array([1, 9]), np.array([0.5, 0.5], dtype=np.float32)
    run_merge(am, m, idx, gate, cuda_device)
    rc, st = m.plan.status()
    assert rc == 0 and st == am.STATUS_BAD_INDEX
    check_merge(m, idx, gate.astype(np.float64), "bad index")
    assert m.plan.status() == (0, 0)


def test_merge_repeated_expert_gates_add(am, cuda_device):
    """An expert picked in two slots contributes with the sum of its gates
    (the oracle's sum over slots), in the merge and in the switch."""
    cfg = synth.custom([(384, 264), (136, 520)], 5, 16, 3, 1, name="mrep")
    m = Model(cfg, cuda_device)
    idx, gate = np.array([2, 2, 0]), np.array([0.3, 0.2, 0.1], dtype=np.float32)
    run_merge(am, m, idx, gate, cuda_device)
    check_merge(m, idx, gate.astype(np.float64), "repeated expert")
    one = Model(cfg, cuda_device, weights=m.w)
    run_merge(am, one, np.array([2, 0, 4]), np.array([0.5, 0.1, 0.0], dtype=np.float32), cuda_device)
    for a, b in zip(m.W_out, one.W_out):
        assert_close_bf16(u16(a), u16(b), "repeated expert vs summed gate")
    assert m.plan.status() == (0, 0)


def test_merge_per_linear_baseline(am, cuda_device):
    cfg = synth.custom(SHAPES, 5, 16, 2, 1, name="mpl")
    m = Model(cfg, cuda_device)
    idx, gate = np.array([0, 3]), np.array([0.45, 0.2], dtype=np.float32)
    run_merge(am, m, idx, gate, cuda_device, per_linear=True)
    assert m.plan.last_launches == len(SHAPES)
    check_merge(m, idx, gate.astype(np.float64), "per-linear")


def test_calls_queued_back_to_back(am, cuda_device):
    """merge -> apply -> switch -> apply -> pregate -> apply queued on one
    stream behind a GPU sleep, no host synchronisation in between, the three
    applies on one workspace with different T and inputs.  Each kernel may
    start while its predecessor still runs (programmatic dependent launch);
    every result must still be the one of the calls run one at a time."""
    cfg = synth.custom([(1024, 2048), (2048, 1024), (520, 1032)], 6, 16, 2, 40, name="b2b")
    m = Model(cfg, cuda_device)
    d = lambda a_, t: torch.as_tensor(np.asarray(a_).astype(t)).to(cuda_device)
    sel_a = (np.array([1, 4]), np.array([0.55, 0.3], dtype=np.float32))
    sel_b = (np.array([2, 1]), np.array([0.4, 0.25], dtype=np.float32))
    Ts = (16, 40, 7)
    ins, outs, sels = [], [], []
    for j, T in enumerate(Ts):
        X, xs = synth.make_apply_inputs(cfg, T, 20 + j)
        ins.append(xs)
        outs.append([torch.full((T, l.d_out), float("nan"), dtype=torch.bfloat16, device=cuda_device)
                     for l in cfg.linears])
        sels.append(synth.random_selection(T, cfg.E, cfg.k, 30 + j, f"b2b{j}"))
    xr = synth.make_router_input(cfg, 5, 3)
    W_r = synth.normal((cfg.E, cfg.hidden), cfg.hidden ** -0.5, torch.float32, 3, "b2bwr")
    xs_dev = [[x.to(cuda_device) for x in xs] for xs in ins]
    ws = torch.empty(max(m.plan.workspace_bytes(T, cfg.k) for T in Ts), dtype=torch.uint8, device=cuda_device)
    xr_d, W_r_d = xr.to(cuda_device), W_r.to(cuda_device)
    sel_dev = [(d(i, np.int32), d(g, np.float32)) for i, g in sels]
    sa = (d(sel_a[0], np.int32), d(sel_a[1], np.float32))
    sb = (d(sel_b[0], np.int32), d(sel_b[1], np.float32))
    torch.cuda.synchronize()

    torch.cuda._sleep(20_000_000)                      # ~10 ms: everything below is queued before it ends
    m.plan.merge(*sa)
    m.plan.apply(xs_dev[0], outs[0], Ts[0], *sel_dev[0], ws)
    m.plan.switch(*sb, *sa)
    m.plan.apply(xs_dev[1], outs[1], Ts[1], *sel_dev[1], ws)
    r_idx, r_gate = am.pregate(xr_d, W_r_d, cfg.k)
    m.plan.apply(xs_dev[2], outs[2], Ts[2], *sel_dev[2], ws)
    torch.cuda.synchronize()

    for j in range(3):
        check_apply(m, ins[j], outs[j], sels[j][0].numpy(), sels[j][1].numpy().astype(np.float64), f"queued apply {j}")
    idx_ref, gate_ref, _ = oracle.pregate(u16(xr), W_r.numpy(), cfg.k)
    assert np.array_equal(r_idx.cpu().numpy(), idx_ref)
    for l in range(cfg.n_lin):
        W, A, B = u16(m.w.W_views[l]), u16(m.w.A_views[l]), u16(m.w.B_views[l])
        cur = oracle.merge_linear(W, A, B, sel_a[0], sel_a[1].astype(np.float64))
        ref = oracle.merge_linear(cur, A, B, list(sel_b[0]) + list(sel_a[0]),
                                  list(sel_b[1].astype(np.float64)) + list(-sel_a[1].astype(np.float64)))
        assert_close_bf16(u16(m.W_out[l]), ref, f"queued merge + switch linear {l}")
    assert m.plan.status() == (0, 0)


@pytest.mark.parametrize("E,r,k", [(5, 16, 2), (6, 32, 2), (4, 8, 1)])
def test_switch_in_place(am, cuda_device, E, r, k):
    """Switch old -> new on the merged weights: matches the oracle's switch of
    the oracle's own merged weights; identical selections leave W_out alone.
    2kr = 64, 128 (single-block groups) and 16."""
    cfg = synth.custom([(384, 264), (136, 520)], E, r, k, 1, name=f"mswitch{E}{r}{k}")
    m = Model(cfg, cuda_device)
    old_i, old_g = np.array([1, 4][:k]), np.array([0.55, 0.3][:k], dtype=np.float32)
    new_i, new_g = np.array([2, 1][:k]), np.array([0.4, 0.25][:k], dtype=np.float32)
    run_merge(am, m, old_i, old_g, cuda_device)
    d = lambda a, t: torch.as_tensor(a.astype(t)).to(cuda_device)
    m.plan.switch(d(new_i, np.int32), d(new_g, np.float32), d(old_i, np.int32), d(old_g, np.float32))
    torch.cuda.synchronize()
    for l in range(cfg.n_lin):
        W, A, B = u16(m.w.W_views[l]), u16(m.w.A_views[l]), u16(m.w.B_views[l])
        cur = oracle.merge_linear(W, A, B, old_i, old_g.astype(np.float64))
        ref = oracle.merge_linear(cur, A, B, list(new_i) + list(old_i),
                                  list(new_g.astype(np.float64)) + list(-old_g.astype(np.float64)))
        assert_close_bf16(u16(m.W_out[l]), ref, f"switch linear {l}")
    before = [t.clone() for t in m.W_out]
    m.plan.switch(d(new_i, np.int32), d(new_g, np.float32), d(new_i, np.int32), d(new_g, np.float32))
    torch.cuda.synchronize()
    for a, b in zip(before, m.W_out):
        assert torch.equal(a.view(torch.int16), b.view(torch.int16))


# ------------------------------------------------------------------- apply

def apply_setup(cfg, dev, T, seed=0, zero_w=False, sel=None):
    m = Model(cfg, dev, seed=seed, zero_w=zero_w)
    X, xs = synth.make_apply_inputs(cfg, T, seed)
    xs_dev = [x.to(dev) for x in xs]
    ys = [torch.empty((T, l.d_out), dtype=torch.bfloat16, device=dev) for l in cfg.linears]
    import adapter_merge_b200 as am
    xp = am.PointerArrays(xs_dev, ys)
    yp = None
    if sel is None:
        idx, gate = synth.random_selection(T, cfg.E, cfg.k, seed + 11, f"asel{cfg.name}{T}")
    else:
        idx, gate = sel
    ws = torch.empty(m.plan.workspace_bytes(T, cfg.k), dtype=torch.uint8, device=dev)
    return m, xs, xs_dev, ys, xp, yp, idx, gate, ws


def check_apply(m, xs, ys, idx, gate, what, tokens=None, lins=None):
    cfg = m.cfg
    for l in (range(cfg.n_lin) if lins is None else lins):
        W, A, B = u16(m.w.W_views[l]), u16(m.w.A_views[l]), u16(m.w.B_views[l])
        tt = (0, xs[l].shape[0]) if tokens is None else tokens
        ref = oracle.apply_linear(u16(xs[l]), W, A, B, np.asarray(idx, np.int32),
                                  np.asarray(gate, np.float64), tokens=tt, nthreads=8)
        assert_close_bf16(u16(ys[l][tt[0]:tt[1]]), ref, f"{what} linear {l}")


def run_apply(m, xp, yp, T, idx, gate, ws, dev):
    i = torch.as_tensor(np.asarray(idx, dtype=np.int32)).to(dev)
    g = torch.as_tensor(np.asarray(gate, dtype=np.float32)).to(dev)
    m.plan.apply(xp, yp, T, i, g, ws)
    torch.cuda.synchronize()


def test_apply_tiny_chain_with_pregate(am, cuda_device):
    cfg = synth.tiny()
    m, xs, xs_dev, ys, xp, yp, _, _, ws = apply_setup(cfg, cuda_device, cfg.T_apply)
    xr = synth.make_router_input(cfg, cfg.T_apply, 0)
    idx_ref, gate_ref, _ = oracle.pregate(u16(xr), m.w.W_r.cpu().numpy(), cfg.k)
    idx, gate = am.pregate(xr.to(cuda_device), m.w.W_r, cfg.k)
    m.plan.apply(xp, yp, cfg.T_apply, idx, gate, ws)
    torch.cuda.synchronize()
    assert np.array_equal(idx.cpu().numpy(), idx_ref)
    check_apply(m, xs, ys, idx_ref, gate_ref, "tiny apply")
    assert m.plan.status() == (0, 0)
    assert m.plan.last_launches == 2


# T <= 64, 65..128 and > 128 take apply units of 512, 256 and 128 output rows;
# d_out = 1000 leaves a last unit whose final 128-row block is all padding.
@pytest.mark.parametrize("T", [1, 5, 16, 17, 64, 65, 128, 129, 130, 256, 300, 1000])
def test_apply_token_counts(am, cuda_device, T):
    cfg = synth.custom([(384, 520), (136, 72), (1000, 264)], 6, 16, 2, T, name=f"aT{T}")
    m, xs, xs_dev, ys, xp, yp, idx, gate, ws = apply_setup(cfg, cuda_device, T)
    run_apply(m, xp, yp, T, idx, gate, ws, cuda_device)
    check_apply(m, xs, ys, idx.numpy(), gate.numpy().astype(np.float64), f"T={T}")


@pytest.mark.parametrize("E,r,k,T", [(4, 8, 1, 16), (8, 16, 2, 64), (32, 64, 4, 128), (16, 32, 2, 32), (3, 24, 3, 9),
                                     (32, 16, 8, 64), (12, 48, 2, 40), (1, 16, 1, 7), (4, 256, 1, 20)])
def test_apply_ranks(am, cuda_device, E, r, k, T):
    cfg = synth.custom([(256, 392), (520, 136)], E, r, k, T, name=f"aR{E}{r}{k}{T}")
    m, xs, xs_dev, ys, xp, yp, idx, gate, ws = apply_setup(cfg, cuda_device, T)
    run_apply(m, xp, yp, T, idx, gate, ws, cuda_device)
    check_apply(m, xs, ys, idx.numpy(), gate.numpy().astype(np.float64), f"E{E} r{r} k{k} T{T}")


# On a 148-SM B200 a plan this small gives 8 units of 128 rows, so every unit
# is split along K into 16 ranges of its chunk list (base, then expand); the
# (128, 72) linear has about 6 chunks, so most of its splits are empty.
@pytest.mark.parametrize("T", [1, 16, 64, 100, 200])
def test_apply_split_k_with_empty_splits(am, cuda_device, T):
    cfg = synth.custom([(256, 4096), (128, 72), (520, 1032)], 6, 16, 2, T, name=f"asplit{T}")
    m, xs, xs_dev, ys, xp, yp, idx, gate, ws = apply_setup(cfg, cuda_device, T)
    for rep in range(2):                 # the split counters must start from zero on every call
        for y in ys:
            y.fill_(float("nan"))
        run_apply(m, xp, yp, T, idx, gate, ws, cuda_device)
        check_apply(m, xs, ys, idx.numpy(), gate.numpy().astype(np.float64), f"split T={T} call {rep}")
    assert m.plan.status() == (0, 0)


# 152 linears of 1024 x 128: 304, 608 and 1216 units of 512, 256 and 128 rows,
# enough for every unit height to run unsplit (T = 48, 100, 200).
@pytest.mark.parametrize("T", [48, 100, 200])
def test_apply_unit_heights_unsplit(am, cuda_device, T):
    cfg = synth.custom([(1024, 128)] * 152, 4, 8, 2, T, name=f"aheights{T}")
    m, xs, xs_dev, ys, xp, yp, idx, gate, ws = apply_setup(cfg, cuda_device, T)
    run_apply(m, xp, yp, T, idx, gate, ws, cuda_device)
    check_apply(m, xs, ys, idx.numpy(), gate.numpy().astype(np.float64), f"heights T={T}",
                lins=range(0, 152, 7))
    assert m.plan.status() == (0, 0)


# T = 6: the two-launch form (shrink inside the apply kernel); T = 24: four launches
@pytest.mark.parametrize("T", [6, 24])
def test_apply_zero_gates_poison_bad_and_duplicate(am, cuda_device, T):
    cfg = synth.custom([(264, 392)], 6, 16, 2, T, name=f"aedge{T}")
    m, xs, xs_dev, ys, xp, yp, idx, gate, ws = apply_setup(cfg, cuda_device, T)
    idx = idx.clone()
    gate = gate.clone()
    # a few rows use only experts {0, 1, 2}; then poison experts 3..5 below
    # for a run where every row uses {0, 1, 2}
    run_apply(m, xp, yp, T, idx, torch.zeros_like(gate), ws, cuda_device)
    check_apply(m, xs, ys, idx.numpy(), np.zeros((T, 2)), "zero gates")
    sel = torch.tensor([[0, 1], [2, 0], [1, 2]] * (T // 3), dtype=torch.int32)
    run_apply(m, xp, yp, T, sel, gate, ws, cuda_device)
    clean = ys[0].clone()
    for e in (3, 4, 5):
        m.w.A_views[0][e].fill_(float("nan"))
        m.w.B_views[0][e].fill_(float("nan"))
    run_apply(m, xp, yp, T, sel, gate, ws, cuda_device)
    assert torch.equal(ys[0].view(torch.int16), clean.view(torch.int16))
    # invalid index: slot skipped, flagged; duplicate experts in a row: gates add
    bad = sel.clone()
    bad[4, 1] = 17
    bad[5, 1] = bad[5, 0]
    run_apply(m, xp, yp, T, bad, gate, ws, cuda_device)
    rc, st = m.plan.status()
    assert rc == 0 and st == am.STATUS_BAD_INDEX
    check_apply(m, xs, ys, bad.numpy(), gate.numpy().astype(np.float64), "bad/dup")


def test_apply_descriptor_cache_follows_pointers_and_T(am, cuda_device):
    """The per-call TMA descriptors are cached by (pointers, T, workspace):
    new buffers, a new T and a new workspace must each be picked up."""
    cfg = synth.custom([(256, 392), (136, 264)], 5, 16, 2, 16, name="acache")
    m = Model(cfg, cuda_device)
    for T, seed in ((16, 1), (16, 2), (9, 3), (16, 1)):
        X, xs = synth.make_apply_inputs(cfg, T, seed)
        xd = [x.to(cuda_device) for x in xs]
        ys = [torch.full((T, l.d_out), 7.0, dtype=torch.bfloat16, device=cuda_device) for l in cfg.linears]
        idx, gate = synth.random_selection(T, cfg.E, cfg.k, seed, "acache")
        ws = torch.empty(m.plan.workspace_bytes(T, cfg.k) + 256 * seed, dtype=torch.uint8, device=cuda_device)
        m.plan.apply(xd, ys, T, idx.to(cuda_device), gate.to(cuda_device), ws)
        torch.cuda.synchronize()
        check_apply(m, xs, ys, idx.numpy(), gate.numpy().astype(np.float64), f"cache T={T} seed={seed}")


def test_apply_descriptor_cache_follows_k(am, cuda_device):
    """Same plan, T, workspace and x / y buffers, but top-1, then top-2, then
    top-1 again: the shrink output's place and width in the workspace follow
    T * k, so the cached descriptors must be rebuilt when k changes."""
    T = 64
    cfg = synth.custom([(256, 392), (136, 264)], 6, 16, 2, T, name="acachek")
    m = Model(cfg, cuda_device)
    X, xs = synth.make_apply_inputs(cfg, T, 4)
    xd = [x.to(cuda_device) for x in xs]
    ys = [torch.empty((T, l.d_out), dtype=torch.bfloat16, device=cuda_device) for l in cfg.linears]
    xp = am.PointerArrays(xd, ys)
    ws = torch.empty(max(m.plan.workspace_bytes(T, k) for k in (1, 2)), dtype=torch.uint8, device=cuda_device)
    for k in (1, 2, 1):
        idx, gate = synth.random_selection(T, cfg.E, k, 10 + k, "acachek")
        for y in ys:
            y.fill_(float("nan"))
        m.plan.apply(xp, None, T, idx.to(cuda_device), gate.to(cuda_device), ws)
        torch.cuda.synchronize()
        check_apply(m, xs, ys, idx.numpy(), gate.numpy().astype(np.float64), f"cache k={k}")
    assert m.plan.status() == (0, 0)


def test_apply_equals_merged_weights(am, cuda_device):
    """Merged form equals unmerged: with one shared selection, apply(x) agrees
    with x W'^T for the GPU's own merged W' to within the bf16 rounding of W'."""
    T = 32
    cfg = synth.custom([(384, 520), (256, 136)], 5, 16, 2, T, name="aeq")
    sel_i = torch.tensor([[3, 1]] * T, dtype=torch.int32)
    sel_g = torch.tensor([[0.5, 0.3]] * T, dtype=torch.float32)
    m, xs, xs_dev, ys, xp, yp, _, _, ws = apply_setup(cfg, cuda_device, T, sel=(sel_i, sel_g))
    run_apply(m, xp, yp, T, sel_i, sel_g, ws, cuda_device)
    run_merge(am, m, sel_i[0].numpy(), sel_g[0].numpy(), cuda_device)
    for l in range(cfg.n_lin):
        x = f64(xs[l]); Wm = f64(m.W_out[l]); y = f64(ys[l])
        ym = x @ Wm.T
        bound = 2.0 ** -8 * (np.abs(x) @ np.abs(Wm).T) + 2.0 ** -7 * np.abs(ym) + 1e-6
        assert np.all(np.abs(y - ym) <= bound)


def test_merge_long_walk_edge_cases(am, cuda_device):
    """A plan just long enough for the long-walk configurations (at least 128
    tiles per SM: row-block groups of four, the gate-scaled B rows in TMEM
    from a contraction depth of 64): a merge at k*r = 96 with a skipped
    out-of-range index and an expert repeated in two slots, then the in-place
    switch to another selection at 2kr = 128 and one at 2kr = 64 (k = 1,
    Kp = 64), each checked on two rows of every 128-row block of every linear
    against the oracle."""
    cfg = synth.custom([(1024, 15360)] * 20, 6, 32, 3, 1, name="longwalk")
    m = Model(cfg, cuda_device)
    m.W_out_flat.fill_(float("nan"))
    sel, g = [4, 9, 4], [0.35, 0.5, 0.15]                   # 9 is out of range: skipped and flagged
    run_merge(am, m, sel, np.array(g, np.float32), cuda_device)
    rc, st = m.plan.status()
    assert rc == 0 and st == am.STATUS_BAD_INDEX
    g64 = [float(np.float32(x)) for x in g]
    for l in range(cfg.n_lin):
        Wl, Ol, Al, Bl = m.w.W_views[l], m.W_out[l], m.w.A_views[l], m.w.B_views[l]
        rows = block_rows(1024, l)
        slots = [e if 0 <= e < cfg.E else -1 for e in sel]
        valid = [(e, gg) for e, gg in zip(slots, g64) if e >= 0]
        assert merge_delta_bound_ok(Ol, Wl, Al, Bl, [e for e, _ in valid], [gg for _, gg in valid])
        merge_rows_check(Ol, Wl, Al, Bl, rows, [e for e, _ in valid], [gg for _, gg in valid],
                         f"long walk merge linear {l}")
    d = lambda a_, t: torch.as_tensor(np.asarray(a_).astype(t)).to(cuda_device)
    for (new_i, new_g, old_i, old_g) in (([2, 0], [0.45, 0.25], [1, 5], [0.3, 0.2]),
                                         ([3], [0.6], [2], [0.4])):
        # the weights hold the old selection's merge, then switch in place
        run_merge(am, m, old_i, np.array(old_g, np.float32), cuda_device)
        m.plan.switch(d(new_i, np.int32), d(new_g, np.float32), d(old_i, np.int32), d(old_g, np.float32))
        torch.cuda.synchronize()
        assert m.plan.status() == (0, 0)
        for l in range(0, cfg.n_lin, 3):
            Wl, Ol, Al, Bl = m.w.W_views[l], m.W_out[l], m.w.A_views[l], m.w.B_views[l]
            merge_rows_check(Ol, Wl, Al, Bl, block_rows(1024, l + 5, per_block=1), new_i,
                             [float(np.float32(x)) for x in new_g], f"long walk switch {len(new_i)} linear {l}",
                             base=True, base_slots=old_i, base_gates=[float(np.float32(x)) for x in old_g])


# ------------------------------------------------------------- full sizes

ORACLE_THREADS = max(1, min(16, os.cpu_count() or 1))


def merge_rows_check(W_out, W, A, B, rows, slots, gates, what, base=None, base_slots=None, base_gates=None):
    """The oracle on `rows` of one linear, against the GPU's rows.  Merge: rows of
    bf16(W + sum_s g_s B A).  With `base` set (a switch), the expected rows are
    the oracle's switch of the oracle's own merge of `base_slots`: rows are
    independent, so each one is exact whatever rows are left out."""
    rt = torch.as_tensor(rows, dtype=torch.long, device=W.device)
    W_rows = u16(W.index_select(0, rt))
    got = u16(W_out.index_select(0, rt))
    all_slots = list(slots) + (list(base_slots) if base is not None else [])
    A_sel, B_sel, ii = take_experts(A, B, all_slots, rows)
    ns = len(slots)
    if base is None:
        ref = oracle.merge_linear(W_rows, A_sel, B_sel, ii, gates, nthreads=ORACLE_THREADS)
        assert_close_bf16(got, ref, what)
        dz = oracle.merge_linear(np.zeros_like(W_rows), A_sel, B_sel, ii, gates, nthreads=ORACLE_THREADS)
        assert_delta_frobenius(got, W_rows, ref, dz, what)
    else:
        cur = oracle.merge_linear(W_rows, A_sel, B_sel, ii[ns:], base_gates, nthreads=ORACLE_THREADS)
        ref = oracle.merge_linear(cur, A_sel, B_sel, list(ii[:ns]) + list(ii[ns:]),
                                  list(gates) + [-g for g in base_gates], nthreads=ORACLE_THREADS)
        assert_close_bf16(got, ref, what)


@pytest.mark.parametrize("cfg_fn", [synth.llama7b, synth.llama13b])
def test_full_size_merge_every_tile(am, cuda_device, cfg_fn):
    """Full model in the benchmark's launch configuration: pregate on one
    token, then ONE merge launch over every linear.  Against the oracle: two
    rows in every 128-row block of every linear (their offsets inside the
    block rotating with the block and the linear, so every tile of every
    linear, every row-block group and its tail, and every CTA's range is
    checked), with the delta check per linear.  On every element: written
    (the output starts as NaN) and within a bound on |dW|.  Then the in-place
    switch to another selection, checked the same way against the oracle's
    switch of the oracle's merged rows."""
    cfg = cfg_fn()
    m = Model(cfg, cuda_device)
    m.W_out_flat.fill_(float("nan"))
    xr = synth.make_router_input(cfg, 1, 0, device=cuda_device)
    idx, gate = am.pregate(xr, m.w.W_r, cfg.k)
    m.plan.merge(idx[0], gate[0])
    torch.cuda.synchronize()
    assert m.plan.status() == (0, 0)
    idx_ref, gate_ref, _ = oracle.pregate(u16(xr), m.w.W_r.cpu().numpy(), cfg.k)
    assert np.array_equal(idx.cpu().numpy(), idx_ref)
    sel = [int(e) for e in idx_ref[0]]
    g = gate.cpu().numpy()[0].astype(np.float64)
    checked = 0
    for l, lin in enumerate(cfg.linears):
        Wl, Ol, Al, Bl = m.w.W_views[l], m.W_out[l], m.w.A_views[l], m.w.B_views[l]
        assert merge_delta_bound_ok(Ol, Wl, Al, Bl, sel, g), f"{cfg.name} merge linear {l}: bound or NaN"
        rows = block_rows(lin.d_out, l)
        merge_rows_check(Ol, Wl, Al, Bl, rows, sel, g, f"{cfg.name} merge linear {l}")
        checked += len(rows)
    assert checked >= 2 * sum((l.d_out + 127) // 128 for l in cfg.linears)

    new_i = [(sel[s] + 1 + s) % cfg.E for s in range(cfg.k)]
    if len(set(new_i)) < cfg.k:
        new_i = list(range(cfg.k))
    new_g = np.linspace(0.5, 0.2, cfg.k).astype(np.float32)
    d = lambda a_, t: torch.as_tensor(np.asarray(a_).astype(t)).to(cuda_device)
    m.plan.switch(d(new_i, np.int32), d(new_g, np.float32), idx[0], gate[0])
    torch.cuda.synchronize()
    assert m.plan.status() == (0, 0)
    for l, lin in enumerate(cfg.linears):
        Wl, Ol, Al, Bl = m.w.W_views[l], m.W_out[l], m.w.A_views[l], m.w.B_views[l]
        assert bool(torch.isfinite(Ol.float()).all()), f"{cfg.name} switch linear {l}: non-finite"
        rows = block_rows(lin.d_out, l + 61, per_block=1)
        merge_rows_check(Ol, Wl, Al, Bl, rows, new_i, list(new_g.astype(np.float64)),
                         f"{cfg.name} switch linear {l}", base=True, base_slots=sel, base_gates=list(g))


@pytest.mark.parametrize("cfg_fn", [synth.llama7b, synth.llama13b])
def test_full_size_apply_every_unit(am, cuda_device, cfg_fn):
    """Batched decode at full size in the benchmark's launch configuration:
    per-sequence routing on each sequence's first token, then ONE apply over
    every linear.  Against the oracle: two whole tokens of every linear (a
    token's row of y spans every apply unit of the linear), the tokens
    rotating with the linear index.  On every element: written (y starts as
    NaN)."""
    cfg = cfg_fn()
    T = cfg.T_apply
    m = Model(cfg, cuda_device)
    X, xs_dev = synth.make_apply_inputs(cfg, T, 0, device=cuda_device)
    Y = torch.full((sum(T * l.d_out for l in cfg.linears),), float("nan"), dtype=torch.bfloat16,
                   device=cuda_device)
    ys, o = [], 0
    for l in cfg.linears:
        ys.append(Y[o:o + T * l.d_out].view(T, l.d_out))
        o += T * l.d_out
    xp = am.PointerArrays(xs_dev, ys)
    xr = synth.make_router_input(cfg, T, 0, device=cuda_device, tag="xfirst")
    idx, gate = am.pregate(xr, m.w.W_r, cfg.k)
    ws = torch.empty(m.plan.workspace_bytes(T, cfg.k), dtype=torch.uint8, device=cuda_device)
    m.plan.apply(xp, None, T, idx, gate, ws)
    torch.cuda.synchronize()
    assert m.plan.status() == (0, 0)
    assert bool(torch.isfinite(Y.float()).all()), "apply left outputs unwritten"
    idx_ref, gate_ref, _ = oracle.pregate(u16(xr), m.w.W_r.cpu().numpy(), cfg.k)
    assert np.array_equal(idx.cpu().numpy(), idx_ref)
    g = gate.cpu().numpy().astype(np.float64)

    def job(l, W, A, B, x, toks, got):
        for t, row in zip(toks, got):
            ref = oracle.apply_linear(x, W, A, B, idx_ref, g, tokens=(t, t + 1), nthreads=1)
            assert_close_bf16(row[None, :], ref, f"{cfg.name} apply linear {l} token {t}")
        return len(toks)

    checked = 0
    with concurrent.futures.ThreadPoolExecutor(ORACLE_THREADS) as pool:
        futs = []
        for l in range(cfg.n_lin):
            toks = sorted({(3 * l) % T, (3 * l + T // 2 + 1) % T})
            got = u16(ys[l])[toks]
            futs.append(pool.submit(job, l, u16(m.w.W_views[l]), u16(m.w.A_views[l]), u16(m.w.B_views[l]),
                                    u16(xs_dev[l]), toks, got))
            if len(futs) >= 2 * ORACLE_THREADS:          # bound the host copies in flight
                checked += futs.pop(0).result()
        for f in futs:
            checked += f.result()
    assert checked >= cfg.n_lin


# ------------------------------------------------------------------- sweep

SWEEP_GRID = [(E, r, k) for E in (4, 8, 16, 32) for r in (8, 16, 32, 64) for k in (1, 2, 4)
              if k <= E and k * r <= 256]


@pytest.mark.parametrize("E,r,k", SWEEP_GRID)
def test_sweep_point_merge_and_apply(am, cuda_device, E, r, k):
    """Every (E, r, k) of the single-layer sweep (4096 x 4096 W, gates from the
    softmax of N(0, 1) logits): the merge on two rows of every 128-row block
    (delta check included) and the apply at batch 1, 16 and 128 on every
    token up to 16 and on eight rotating tokens at 128."""
    cfg = synth.sweep_point(E, r, k, 128)
    m = Model(cfg, cuda_device)
    m.W_out_flat.fill_(float("nan"))
    z = synth.normal((128, E), 1.0, torch.float32, 9, f"sweep-logits-{E}-{r}-{k}").numpy()
    idx, gate = oracle.topk_softmax(z, k)
    gate32 = gate.astype(np.float32)
    run_merge(am, m, idx[0], gate32[0], cuda_device)
    Wl, Ol, Al, Bl = m.w.W_views[0], m.W_out[0], m.w.A_views[0], m.w.B_views[0]
    g0 = gate32[0].astype(np.float64)
    assert merge_delta_bound_ok(Ol, Wl, Al, Bl, idx[0], g0), "sweep merge: bound or NaN"
    merge_rows_check(Ol, Wl, Al, Bl, block_rows(4096, E + r + k), idx[0], g0, f"sweep E{E} r{r} k{k} merge")
    W, A, B = u16(Wl), u16(Al), u16(Bl)
    for T in (1, 16, 128):
        X, xs = synth.make_apply_inputs(cfg, T, 9)
        xd = [x.to(cuda_device) for x in xs]
        ys = [torch.full((T, 4096), float("nan"), dtype=torch.bfloat16, device=cuda_device)]
        ws = torch.empty(m.plan.workspace_bytes(T, k), dtype=torch.uint8, device=cuda_device)
        ii, gg = idx[:T], gate32[:T]
        m.plan.apply(xd, ys, T, torch.as_tensor(ii).to(cuda_device), torch.as_tensor(gg).to(cuda_device), ws)
        torch.cuda.synchronize()
        assert bool(torch.isfinite(ys[0].float()).all()), f"sweep apply T={T}: unwritten outputs"
        toks = range(T) if T <= 16 else sorted({(E + r + k + 17 * j) % T for j in range(8)} | {0, T - 1})
        x = u16(xs[0])
        got = u16(ys[0])
        for t in toks:
            ref = oracle.apply_linear(x, W, A, B, ii, gg.astype(np.float64), tokens=(t, t + 1))
            assert_close_bf16(got[t:t + 1], ref, f"sweep E{E} r{r} k{k} apply T={T} token {t}")
    assert m.plan.status() == (0, 0)
