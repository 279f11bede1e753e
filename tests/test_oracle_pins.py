"""Pins for the CPU oracle: each test ties one oracle function to something
other than itself -- hand-worked values, closed forms, library routines
(torch's bf16 conversion, numpy matmul, Python's stable sort, scipy's softmax),
brute force on tiny inputs, or exact error bounds.

Method: AdaFuse (token-level pre-gating, section 2.A / 2.1; SGMM fused merge,
section 2.B / 2.2; segmented-gather apply for mixed batches).  CPU only.
"""
import itertools
import json
import math
import os
from fractions import Fraction

import numpy as np
import pytest
import scipy.special
import torch

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "handworked.json")


def _golden():
    with open(GOLDEN) as f:
        return json.load(f)


def bits(a) -> np.ndarray:
    """float values exactly representable in bf16 -> uint16 bit patterns."""
    t = torch.as_tensor(np.asarray(a, dtype=np.float32)).to(torch.bfloat16)
    back = t.to(torch.float32).numpy()
    assert np.array_equal(back, np.asarray(a, dtype=np.float32)), "value not exact in bf16"
    return t.view(torch.int16).numpy().view(np.uint16)


def vals(b) -> np.ndarray:
    return oracle.bf16_to_f64(b)


def dyadic(rng, shape, lo=-8, hi=8, scale_pow=3):
    """Small integers times 2^-scale_pow: exact in bf16, products and short
    sums exact in fp64 and fp32."""
    return rng.integers(lo, hi + 1, size=shape).astype(np.float64) * 2.0 ** -scale_pow


def torch_bf16_bits(v64: np.ndarray) -> np.ndarray:
    """torch's RNE float32->bf16; only used on values exact in fp32."""
    v32 = v64.astype(np.float32)
    assert np.array_equal(v32.astype(np.float64), v64), "value not exact in fp32"
    return torch.from_numpy(v32).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)


# ------------------------------------------------------------------- bf16

def test_bf16_to_double_matches_torch():
    allbits = np.arange(1 << 16, dtype=np.uint32).astype(np.uint16)
    ours = oracle.bf16_to_f64(allbits)
    ref = torch.from_numpy(allbits.view(np.int16)).view(torch.bfloat16).to(torch.float64).numpy()
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(ours), nan)
    assert np.array_equal(ours[~nan], ref[~nan])


def test_bf16_rounding_matches_torch_on_fp32_values():
    rng = np.random.default_rng(1)
    # random fp32 bit patterns (finite), plus every bf16 midpoint pattern
    raw = rng.integers(0, 1 << 32, size=200000, dtype=np.uint64).astype(np.uint32)
    f = raw.view(np.float32)
    f = f[np.isfinite(f)]
    mids = ((np.arange(1 << 16, dtype=np.uint32) << 16) | 0x8000).view(np.float32)
    mids = mids[np.isfinite(mids)]
    # signed zeros, and values of either sign that round to a zero
    zeros = np.array([0.0, -0.0, 2.0 ** -134, -(2.0 ** -134), -(2.0 ** -140), 2.0 ** -149, -(2.0 ** -149)],
                     dtype=np.float32)
    for v in (f, mids, zeros):
        ours = oracle.bf16_from_f64(v.astype(np.float64))
        ref = torch.from_numpy(v.copy()).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
        assert np.array_equal(ours, ref)


def _nearest_bf16_exact(v: float) -> int:
    """Brute force: the bf16 pattern nearest to v by exact rational distance,
    ties to the even pattern (finite positive v below the largest bf16)."""
    allbits = np.arange(0, 0x7F80, dtype=np.uint16)         # +0 .. max finite
    values = oracle.bf16_to_f64(allbits)
    j = int(np.searchsorted(values, v))
    cands = [c for c in (j - 1, j) if 0 <= c < len(values)]
    fv = Fraction(v)
    best = min(cands, key=lambda c: (abs(Fraction(values[c]) - fv), int(allbits[c]) & 1))
    return int(allbits[best])


def test_bf16_rounding_single_step_from_double():
    """Doubles that are not fp32 values: a detour through fp32 would round twice."""
    rng = np.random.default_rng(2)
    xs = list(np.abs(rng.standard_normal(400)) * 2.0 ** rng.integers(-20, 20, 400))
    # just above a bf16 midpoint by less than an fp32 ulp: double rounding breaks these
    for b in (0x3F80, 0x3F81, 0x4049, 0x3C00):
        lo = oracle.bf16_to_f64(np.array([b], np.uint16))[0]
        hi = oracle.bf16_to_f64(np.array([b + 1], np.uint16))[0]
        mid = (lo + hi) / 2
        xs += [mid, mid + (hi - lo) * 2 ** -30, mid - (hi - lo) * 2 ** -30]
    for v in xs:
        got = int(oracle.bf16_from_f64(np.array([v]))[0])
        assert got == _nearest_bf16_exact(float(v)), v
    # signs, zero, overflow and subnormals
    assert int(oracle.bf16_from_f64(np.array([-1.0]))[0]) == 0xBF80
    assert int(oracle.bf16_from_f64(np.array([0.0]))[0]) == 0x0000
    assert int(oracle.bf16_from_f64(np.array([-0.0]))[0]) == 0x8000
    assert int(oracle.bf16_from_f64(np.array([-(2.0 ** -140)]))[0]) == 0x8000
    assert int(oracle.bf16_from_f64(np.array([1e39]))[0]) == 0x7F80
    assert int(oracle.bf16_from_f64(np.array([2.0 ** -133]))[0]) == 0x0001
    assert int(oracle.bf16_from_f64(np.array([2.0 ** -134]))[0]) == 0x0000   # tie -> even (0)
    assert int(oracle.bf16_from_f64(np.array([3 * 2.0 ** -134]))[0]) == 0x0002


# ----------------------------------------------------------------- router

def test_topk_margin_and_router_scale_handworked():
    """The near-tie report: z_(k) - z_(k+1) per row (inf when k = E), and the
    scale max_e sum_j |x_j||W_r[e, j]|, on values worked by hand."""
    z = np.array([[3.0, 1.0, 2.0, 0.0], [0.5, 0.5, -1.0, 2.0]], dtype=np.float32)
    assert oracle.topk_margin(z, 2).tolist() == [1.0, 0.0]          # sorted 3,2,1,0 and 2,.5,.5,-1
    assert oracle.topk_margin(z, 1).tolist() == [1.0, 1.5]
    assert np.all(np.isinf(oracle.topk_margin(z, 4)))
    x = np.array([[0x3F80, 0xC000]], dtype=np.uint16)                # bf16 1.0, -2.0
    W = np.array([[0.5, 0.25], [1.0, -1.0]])
    assert oracle.router_scale(x, W).tolist() == [3.0]               # max(0.5 + 0.5, 1 + 2)


def test_router_handworked():
    g = _golden()
    for key in ("router", "router_tie"):
        c = g[key]
        x = bits(np.array(c["x"], dtype=np.float32)[None, :])
        W_r = np.array(c["W_r"], dtype=np.float32)
        z = oracle.router_logits(x, W_r)
        assert np.array_equal(z[0], np.array(c["z"], dtype=np.float32))
        idx, gate = oracle.topk_softmax(z, 2)
        assert idx[0].tolist() == c["idx"]
        assert np.allclose(gate[0], c["gate"], rtol=0, atol=c["gate_tol"])


def test_router_logits_error_bound_vs_exact_dot():
    """fp32 recursive summation: |z - exact| <= gamma_H * sum|x_j w_j|,
    gamma_n = n u / (1 - n u), u = 2^-24 (plus one rounding per product)."""
    rng = np.random.default_rng(3)
    T, H, E = 5, 1000, 7
    x = torch.randn(T, H, generator=torch.Generator().manual_seed(3)).to(torch.bfloat16)
    xb = x.view(torch.int16).numpy().view(np.uint16)
    xv = x.to(torch.float64).numpy()
    W_r = (rng.standard_normal((E, H)) / math.sqrt(H)).astype(np.float32)
    z = oracle.router_logits(xb, W_r)
    u = 2.0 ** -24
    gam = (H + 1) * u / (1 - (H + 1) * u)
    for t in range(T):
        for e in range(E):
            exact = math.fsum(float(a) * float(b) for a, b in zip(xv[t], W_r[e].astype(np.float64)))
            bound = gam * float(np.sum(np.abs(xv[t] * W_r[e].astype(np.float64))))
            assert abs(float(z[t, e]) - exact) <= bound


def test_router_logits_exact_on_dyadic_inputs():
    """Small dyadic inputs make every product and partial sum exact: the logit
    must equal the exact dot product (catches dropped terms, wrong indices,
    transposed W_r), and the bias is added."""
    rng = np.random.default_rng(4)
    T, H, E = 6, 96, 5
    xv = dyadic(rng, (T, H))
    W_r = dyadic(rng, (E, H)).astype(np.float32)
    b_r = dyadic(rng, (E,)).astype(np.float32)
    z = oracle.router_logits(bits(xv), W_r, b_r)
    ref = xv @ W_r.astype(np.float64).T + b_r
    assert np.array_equal(z.astype(np.float64), ref)


def test_router_fp32_order_is_sequential():
    """The decision precision is fp32 with products added in ascending j: a
    case where that order matters.  1 + 2^-24 + 2^-24 in order gives 1 (each
    tiny term is lost), while any other grouping keeps 2^-23."""
    x = bits(np.array([[1.0, 1.0, 1.0]], dtype=np.float32))
    W_r = np.array([[1.0, 2.0 ** -24, 2.0 ** -24]], dtype=np.float32)
    z = oracle.router_logits(x, W_r)
    assert z[0, 0] == np.float32(1.0)
    W_r2 = np.array([[2.0 ** -24, 2.0 ** -24, 1.0]], dtype=np.float32)
    z2 = oracle.router_logits(x, W_r2)
    assert z2[0, 0] == np.float32(1.0 + 2.0 ** -23)


def test_router_products_are_rounded_before_the_add():
    """Each product is rounded to fp32 before it is added (no fused
    multiply-add): x = 1 + 2^-7 (bf16), w = 1 + 2^-23 gives the exact product
    1 + 2^-7 + 2^-23 + 2^-30, which rounds to 1 + 2^-7 + 2^-23; after adding
    -(1 + 2^-7 + 2^-23) the plain definition gives 0, a fused one 2^-30."""
    x = bits(np.array([[1.0, 1.0 + 2.0 ** -7]], dtype=np.float32))
    c = 1.0 + 2.0 ** -7 + 2.0 ** -23
    W_r = np.array([[-c, 1.0 + 2.0 ** -23]], dtype=np.float32)
    assert float(W_r[0, 0]) == -c
    z = oracle.router_logits(x, W_r)
    assert z[0, 0] == np.float32(0.0)


def test_router_bias_added_after_the_sum():
    """The bias is added once the products are summed (the reading the
    kernel follows too, so that idx parity is exact): 0 + 2^-24 + 2^-24 =
    2^-23 exactly, then + 1 gives 1 + 2^-23; starting the sum from the bias
    would lose both tiny products (1 + 2^-24 rounds to 1) and give 1."""
    x = bits(np.array([[1.0, 1.0]], dtype=np.float32))
    W_r = np.array([[2.0 ** -24, 2.0 ** -24]], dtype=np.float32)
    b_r = np.array([1.0], dtype=np.float32)
    z = oracle.router_logits(x, W_r, b_r)
    assert z[0, 0] == np.float32(1.0 + 2.0 ** -23)


@pytest.mark.parametrize("E", [1, 2, 3, 4, 5])
def test_topk_brute_force_all_tie_patterns(E):
    """Every logit pattern over {-1, 0, 1, nan}^E and every k: the selection is
    Python's stable sort by (-z, e) with NaN last, and the gates are scipy's
    fp64 softmax over the non-NaN logits."""
    levels = [-1.0, 0.0, 1.0, float("nan")]
    for pattern in itertools.product(levels, repeat=E):
        z = np.array(pattern, dtype=np.float32)[None, :]
        for k in range(1, E + 1):
            idx, gate = oracle.topk_softmax(z, k)
            key = lambda e: (1, 0.0, e) if math.isnan(pattern[e]) else (0, -pattern[e], e)
            assert idx[0].tolist() == sorted(range(E), key=key)[:k]
            finite = ~np.isnan(z[0])
            if finite.any():
                p = np.zeros(E)
                p[finite] = scipy.special.softmax(z[0, finite].astype(np.float64))
                assert np.allclose(gate[0], p[idx[0]], rtol=1e-14, atol=1e-15)


def test_softmax_closed_forms_and_invariants():
    rng = np.random.default_rng(5)
    # E = 2: p_top = sigmoid(z_top - z_other)
    z = rng.standard_normal((50, 2)).astype(np.float32)
    idx, gate = oracle.topk_softmax(z, 1)
    for t in range(50):
        a, b = z[t, idx[t, 0]], z[t, 1 - idx[t, 0]]
        assert math.isclose(gate[t, 0], 1.0 / (1.0 + math.exp(float(b) - float(a))), rel_tol=1e-14)
    # k = E: gates sum to 1; k < E: sum < 1; renorm: sum to 1
    z = rng.standard_normal((40, 8)).astype(np.float32)
    _, g8 = oracle.topk_softmax(z, 8)
    assert np.allclose(g8.sum(1), 1.0, atol=1e-14)
    _, g2 = oracle.topk_softmax(z, 2)
    assert np.all(g2.sum(1) < 1.0)
    _, g2r = oracle.topk_softmax(z, 2, renorm=True)
    assert np.allclose(g2r.sum(1), 1.0, atol=1e-14)
    assert np.allclose(g2r, g2 / g2.sum(1, keepdims=True), rtol=1e-14)
    # gates in rank order are non-increasing
    assert np.all(np.diff(g2, axis=1) <= 0)
    # shift invariance: adding a power of two to all logits keeps the order
    i0, _ = oracle.topk_softmax(z, 3)
    i1, _ = oracle.topk_softmax(z + np.float32(4.0), 3)
    assert np.array_equal(i0, i1)


def test_softmax_large_logits_closed_form():
    """Logits far outside exp's range: the probabilities still follow the
    closed form p_i = 1 / sum_j exp(z_j - z_i) (a softmax computed without
    subtracting the maximum overflows or underflows to 0/0 here)."""
    cases = [[1000.0, 999.0, -1000.0, 0.0], [-1000.0, -1001.0, -1003.0, -2000.0], [88.5, 89.0, 90.0, -90.0]]
    for zc in cases:
        z = np.array([zc], dtype=np.float32)
        idx, gate = oracle.topk_softmax(z, 2)
        zz = z[0].astype(np.float64)
        for s in range(2):
            i = idx[0, s]
            ref = 1.0 / math.fsum(math.exp(zz[j] - zz[i]) for j in range(4))
            assert math.isclose(gate[0, s], ref, rel_tol=1e-14), (zc, s)
        assert idx[0].tolist() == sorted(range(4), key=lambda e: (-zz[e], e))[:2]


def test_pool_mean_exact_cases():
    rng = np.random.default_rng(6)
    xv = dyadic(rng, (8, 33))
    m = oracle.pool_mean(bits(xv))
    # sums of 8 dyadic values are exact; dividing by 8 is exact
    assert np.array_equal(m.astype(np.float64), xv.mean(0))
    # T = 3: exact sum, one correctly rounded division
    xv = dyadic(rng, (3, 17))
    m = oracle.pool_mean(bits(xv))
    for j in range(17):
        assert m[j] == np.float32(Fraction(xv[:, j].sum()) / 3)


def test_pregate_pool_routes_the_mean_row():
    rng = np.random.default_rng(7)
    xv = dyadic(rng, (4, 64))
    W_r = dyadic(rng, (6, 64)).astype(np.float32)
    idx, gate, z = oracle.pregate(bits(xv), W_r, 2, pool=True)
    ref = xv.mean(0) @ W_r.astype(np.float64).T
    assert np.array_equal(z[0].astype(np.float64), ref)
    assert idx.shape == (1, 2)


# ------------------------------------------------------------------ merge

def test_merge_handworked():
    c = _golden()["merge"]
    W = bits(np.array(c["W"])); A = bits(np.array(c["A"])); B = bits(np.array(c["B"]))
    out = oracle.merge_linear(W, A, B, c["idx"], c["gate"])
    assert np.array_equal(vals(out), np.array(c["W_out"]))


def _rand_adapters(rng, d_out, d_in, E, r):
    W = dyadic(rng, (d_out, d_in), -16, 16, 4)
    A = dyadic(rng, (E, r, d_in), -4, 4, 2)
    B = dyadic(rng, (E, d_out, r), -4, 4, 2)
    return W, A, B


def test_merge_single_adapter_unit_gate_is_lora_merge():
    """k=1, g=1: W' = bf16(W + B_e A_e), a plain GEMM (numpy) and one rounding."""
    rng = np.random.default_rng(8)
    d_out, d_in, E, r = 24, 40, 3, 8
    W, A, B = _rand_adapters(rng, d_out, d_in, E, r)
    for e in range(E):
        out = oracle.merge_linear(bits(W), bits(A), bits(B), [e], [1.0])
        ref = W + B[e] @ A[e]
        assert np.array_equal(out, torch_bf16_bits(ref))


def test_merge_multi_adapter_matches_numpy_and_linearity():
    rng = np.random.default_rng(9)
    d_out, d_in, E, r = 16, 24, 5, 8
    W, A, B = _rand_adapters(rng, d_out, d_in, E, r)
    Wz = np.zeros_like(W)
    e = [3, 0, 4]
    g = [0.5, 0.25, -0.125]
    out = oracle.merge_linear(bits(W), bits(A), bits(B), e, g)
    ref = W + sum(gs * (B[es] @ A[es]) for es, gs in zip(e, g))
    assert np.array_equal(out, torch_bf16_bits(ref))
    # linearity of the concatenation: the delta of the three slots is the sum
    # of single-slot deltas (exact with these inputs, W = 0)
    full = vals(oracle.merge_linear(bits(Wz), bits(A), bits(B), e, g))
    parts = sum(vals(oracle.merge_linear(bits(Wz), bits(A), bits(B), [es], [gs]))
                for es, gs in zip(e, g))
    assert np.array_equal(full, parts)


def test_merge_zero_gates_leave_w_unchanged():
    rng = np.random.default_rng(10)
    W = torch.randn(32, 48, generator=torch.Generator().manual_seed(10)).mul(0.02).to(torch.bfloat16)
    Wb = W.view(torch.int16).numpy().view(np.uint16)
    A = bits(dyadic(rng, (4, 8, 48)))
    B = bits(dyadic(rng, (4, 32, 8)))
    out = oracle.merge_linear(Wb, A, B, [1, 2], [0.0, 0.0])
    assert np.array_equal(out, Wb)


def test_merge_skips_invalid_index_and_ignores_unselected_nan():
    rng = np.random.default_rng(11)
    d_out, d_in, E, r = 8, 16, 4, 8
    W, A, B = _rand_adapters(rng, d_out, d_in, E, r)
    ref = oracle.merge_linear(bits(W), bits(A), bits(B), [2], [0.5])
    got = oracle.merge_linear(bits(W), bits(A), bits(B), [2, 7, -1], [0.5, 1.0, 1.0])
    assert np.array_equal(ref, got)
    Ab, Bb = bits(A), bits(B)
    for e in (0, 1, 3):                    # poison every adapter not selected
        Ab[e] = 0x7FC0
        Bb[e] = 0x7FC0
    assert np.array_equal(oracle.merge_linear(bits(W), Ab, Bb, [2], [0.5]), ref)


def test_merge_row_range_and_threads():
    rng = np.random.default_rng(12)
    W, A, B = _rand_adapters(rng, 40, 24, 3, 8)
    full = oracle.merge_linear(bits(W), bits(A), bits(B), [1, 2], [0.375, 0.25])
    part = oracle.merge_linear(bits(W), bits(A), bits(B), [1, 2], [0.375, 0.25], rows=(7, 29), nthreads=4)
    assert np.array_equal(full[7:29], part)


def test_switch_is_merge_with_negated_previous_gates():
    """Switching (undo the previous token's fusion, fuse the current one):
    starting from merge(W, old), the switch lands within bf16 rounding of
    merge(W, new), and exactly on it when nothing rounds."""
    rng = np.random.default_rng(13)
    W, A, B = _rand_adapters(rng, 16, 16, 4, 8)
    old_e, old_g = [0, 1], [0.5, 0.25]
    new_e, new_g = [2, 1], [0.25, 0.5]
    cur = oracle.merge_linear(bits(W), bits(A), bits(B), old_e, old_g)
    sw = oracle.merge_linear(cur, bits(A), bits(B), new_e + old_e, new_g + [-g for g in old_g])
    direct = oracle.merge_linear(bits(W), bits(A), bits(B), new_e, new_g)
    assert np.array_equal(sw, direct)


# ------------------------------------------------------------------ apply

def test_apply_handworked():
    g = _golden()
    m, c = g["merge"], g["apply"]
    y = oracle.apply_linear(bits(np.array(c["x"])), bits(np.array(m["W"])), bits(np.array(m["A"])),
                            bits(np.array(m["B"])), np.array(c["idx"]), np.array(c["gate"]))
    assert np.array_equal(vals(y), np.array(c["y"]))


def test_apply_matches_numpy_per_token():
    """y_t = bf16(x_t W^T + sum_s g_ts (x_t A_e^T) B_e^T) with numpy matmuls."""
    rng = np.random.default_rng(14)
    T, d_out, d_in, E, r, k = 7, 20, 32, 5, 8, 2
    W, A, B = _rand_adapters(rng, d_out, d_in, E, r)
    x = dyadic(rng, (T, d_in), -4, 4, 1)
    idx = np.stack([rng.permutation(E)[:k] for _ in range(T)]).astype(np.int32)
    gate = dyadic(rng, (T, k), 1, 8, 3)
    y = oracle.apply_linear(bits(x), bits(W), bits(A), bits(B), idx, gate)
    for t in range(T):
        ref = x[t] @ W.T
        for s in range(k):
            e = idx[t, s]
            ref = ref + gate[t, s] * ((x[t] @ A[e].T) @ B[e].T)
        assert np.array_equal(y[t], torch_bf16_bits(ref))


def test_apply_merged_equals_unmerged_and_token_permutation():
    """One shared selection: apply(x) ~= x W'^T within the bf16 rounding of W'
    (bound 2^-8 sum_i |x_i W'_oi| + output rounding); permuting the tokens
    permutes y exactly."""
    rng = np.random.default_rng(15)
    T, d_out, d_in, E, r = 6, 24, 64, 4, 8
    Wt = torch.randn(d_out, d_in, generator=torch.Generator().manual_seed(15)).mul(0.02).to(torch.bfloat16)
    At = torch.randn(E, r, d_in, generator=torch.Generator().manual_seed(16)).div(16).to(torch.bfloat16)
    Bt = torch.randn(E, d_out, r, generator=torch.Generator().manual_seed(17)).mul(0.01).to(torch.bfloat16)
    xt = torch.randn(T, d_in, generator=torch.Generator().manual_seed(18)).to(torch.bfloat16)
    b = lambda t: t.view(torch.int16).numpy().view(np.uint16)
    e, g = [2, 0], [0.625, 0.25]
    idx = np.tile(np.array(e, np.int32), (T, 1))
    gate = np.tile(np.array(g), (T, 1))
    y = vals(oracle.apply_linear(b(xt), b(Wt), b(At), b(Bt), idx, gate))
    Wm = vals(oracle.merge_linear(b(Wt), b(At), b(Bt), e, g))
    xv = xt.to(torch.float64).numpy()
    ym = xv @ Wm.T
    bound = 2.0 ** -8 * (np.abs(xv) @ np.abs(Wm).T) + 2.0 ** -8 * np.abs(ym)
    assert np.all(np.abs(y - ym) <= bound)
    perm = rng.permutation(T)
    yp = oracle.apply_linear(b(xt)[perm], b(Wt), b(At), b(Bt), idx[perm], gate[perm])
    assert np.array_equal(yp, oracle.apply_linear(b(xt), b(Wt), b(At), b(Bt), idx, gate)[perm])


def test_apply_f64_is_the_unrounded_apply_and_shards_sum():
    """The unrounded apply (a row-parallel shard's partial output): on dyadic
    inputs every product and sum is exact in fp64, so it equals numpy's
    per-token result exactly, rounds to exactly apply_linear's bf16 output, and
    the partials of a split of d_in into column blocks (W and A cut the same
    way, B whole) add up exactly to the unsharded result."""
    rng = np.random.default_rng(24)
    T, d_out, d_in, E, r, k = 5, 16, 48, 4, 8, 2
    W, A, B = _rand_adapters(rng, d_out, d_in, E, r)
    x = dyadic(rng, (T, d_in), -4, 4, 1)
    idx = np.stack([rng.permutation(E)[:k] for _ in range(T)]).astype(np.int32)
    gate = dyadic(rng, (T, k), 1, 8, 3)
    y64 = oracle.apply_linear_f64(bits(x), bits(W), bits(A), bits(B), idx, gate)
    for t in range(T):
        ref = x[t] @ W.T
        for s in range(k):
            e = idx[t, s]
            ref = ref + gate[t, s] * ((x[t] @ A[e].T) @ B[e].T)
        assert np.array_equal(y64[t], ref)
    assert np.array_equal(oracle.bf16_from_f64(y64), oracle.apply_linear(bits(x), bits(W), bits(A), bits(B), idx, gate))
    part = np.zeros_like(y64)
    for c0, c1 in ((0, 16), (16, 40), (40, 48)):
        part += oracle.apply_linear_f64(bits(np.ascontiguousarray(x[:, c0:c1])),
                                        bits(np.ascontiguousarray(W[:, c0:c1])),
                                        bits(np.ascontiguousarray(A[:, :, c0:c1])), bits(B), idx, gate)
    assert np.array_equal(part, y64)


def test_apply_zero_gates_is_base_gemm():
    rng = np.random.default_rng(19)
    W, A, B = _rand_adapters(rng, 12, 16, 3, 8)
    x = dyadic(rng, (5, 16))
    idx = np.array([[0, 1]] * 5, dtype=np.int32)
    y = oracle.apply_linear(bits(x), bits(W), bits(A), bits(B), idx, np.zeros((5, 2)))
    assert np.array_equal(y, torch_bf16_bits(x @ W.T))


# -------------------------------------------------------------- segments

def test_segments_handworked_and_stable_sort():
    c = _golden()["segments"]
    off, perm, bad = oracle.segments(np.array(c["idx"]), c["E"])
    assert off.tolist() == c["offsets"] and perm.tolist() == c["perm"] and bad == 0
    rng = np.random.default_rng(20)
    for T, k, E in ((1, 1, 1), (64, 2, 8), (33, 4, 6), (128, 2, 32)):
        idx = rng.integers(0, E, size=(T, k)).astype(np.int32)
        idx[rng.random((T, k)) < 0.05] = E + 3          # a few invalid entries
        off, perm, bad = oracle.segments(idx, E)
        flat = idx.reshape(-1)
        valid = [p for p in range(T * k) if 0 <= flat[p] < E]
        assert perm.tolist() == sorted(valid, key=lambda p: flat[p])   # stable
        counts = np.bincount(flat[(flat >= 0) & (flat < E)], minlength=E)
        assert off.tolist() == [0] + np.cumsum(counts).tolist()
        assert bad == T * k - len(valid)
