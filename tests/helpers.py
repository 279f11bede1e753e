"""Shared helpers of the GPU parity tests: build a plan over synthetic weights,
and convert between torch bf16 tensors and the oracle's uint16 bit patterns.
Inputs come from synth/ only; expected values come from oracle/ only."""
from __future__ import annotations

import numpy as np
import torch

import oracle
import synth

# Elementwise acceptance for bf16 outputs accumulated in fp32.
RTOL = 1e-2
ATOL = 1e-3

# Seeds of the 7B bench (1000 + rank) whose decode-batch router input holds
# rows with a near tie: the k-th and (k+1)-th logits within 1e-4 of
# sum_j |x_j||W_r[e, j]|, where the selection depends on the summation order.
NEAR_TIE_RTOL = 1e-4
NEAR_TIE_SEEDS_7B = (1000, 1002, 1004, 1005)


def u16(t: torch.Tensor) -> np.ndarray:
    return t.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)


def f64(t: torch.Tensor) -> np.ndarray:
    return t.detach().cpu().to(torch.float64).numpy()


def assert_close_bf16(gpu_bits: np.ndarray, ref_bits: np.ndarray, what: str = ""):
    g = oracle.bf16_to_f64(gpu_bits)
    r = oracle.bf16_to_f64(ref_bits)
    assert g.shape == r.shape
    assert np.all(np.isfinite(g)), f"{what}: non-finite output"
    err = np.abs(g - r)
    tol = RTOL * np.abs(r) + ATOL
    bad = err > tol
    assert not bad.any(), (f"{what}: {int(bad.sum())} of {bad.size} outside |d| <= 1e-2|ref| + 1e-3; "
                           f"max err {err.max():.3e}")


def assert_delta_frobenius(gpu_bits, W_bits, ref_bits, delta_bits, what: str = ""):
    """(W'_gpu - W) against the oracle's delta (the oracle merge of a zero
    matrix), in Frobenius norm, so that a missing or wrong adapter cannot
    hide under the elementwise tolerance of W':
    ||(W'_gpu - W) - dW|| <= 1e-2 ||dW|| + ||ulp(W'_ref)|| + ||ulp(dW)||."""
    g = oracle.bf16_to_f64(gpu_bits) - oracle.bf16_to_f64(W_bits)
    d = oracle.bf16_to_f64(delta_bits)
    lhs = np.linalg.norm(g - d)
    rhs = 1e-2 * np.linalg.norm(d) + np.linalg.norm(ulp_bf16(oracle.bf16_to_f64(ref_bits))) \
        + np.linalg.norm(ulp_bf16(d))
    assert lhs <= rhs, f"{what}: delta error {lhs:.4e} > {rhs:.4e}"


def ulp_bf16(v: np.ndarray) -> np.ndarray:
    a = np.abs(v)
    e = np.floor(np.log2(np.where(a > 0, a, 1.0)))
    return np.where(a > 0, 2.0 ** (np.maximum(e, -126) - 7), 2.0 ** -133)


class Model:
    """Synthetic weights for a config, resident on the device, plus a plan."""

    def __init__(self, cfg: synth.Config, device, seed=0, in_place=False, zero_w=False, weights=None):
        import adapter_merge_b200 as am
        self.cfg = cfg
        self.w = weights if weights is not None else synth.make_weights(cfg, seed, device=device, zero_w=zero_w)
        if in_place:
            self.W_out = self.w.W_views
        else:
            self.W_out_flat = torch.empty_like(self.w.W)
            self.W_out = []
            o = 0
            for l in cfg.linears:
                n = l.d_out * l.d_in
                self.W_out.append(self.W_out_flat[o:o + n].view(l.d_out, l.d_in))
                o += n
        self.plan = am.Plan(list(zip(self.w.W_views, self.W_out, self.w.A_views, self.w.B_views)), cfg.E, cfg.r)


def block_rows(d_out: int, salt: int, per_block: int = 2):
    """Rows to check in every 128-row block of a linear: `per_block` rows per
    block, their offsets inside the block rotating with the block index and
    `salt` (e.g. the linear's index), so that over a model every tile of every
    linear is checked and every TMEM lane quarter / epilogue warp of a tile is
    reached."""
    rows = []
    for b in range((d_out + 127) // 128):
        for q in range(per_block):
            off = (7 * b + 3 * salt + q * (128 // per_block)) % 128
            rows.append(min(b * 128 + off, d_out - 1))
    return sorted(set(rows))


def take_experts(A, B, slots, rows=None):
    """The A and B stacks of the experts named in `slots` only (bit-for-bit
    slices, on the device), with B cut to `rows`, and the slot indices
    renumbered into the slices: the oracle then indexes exactly the operands
    it would index in the whole stacks, at a fraction of the transfer.
    Returns (A_sel [U, r, d_in], B_sel [U, len(rows), r], idx [len(slots)])
    as host uint16 / int32 arrays."""
    slots = [int(e) for e in slots]
    uniq = sorted(set(slots))
    pos = {e: i for i, e in enumerate(uniq)}
    dev = A.device
    sel = torch.tensor(uniq, dtype=torch.long, device=dev)
    A_sel = A.index_select(0, sel)
    B_sel = B.index_select(0, sel)
    if rows is not None:
        B_sel = B_sel.index_select(1, torch.as_tensor(rows, dtype=torch.long, device=dev))
    return u16(A_sel), u16(B_sel), np.array([pos[e] for e in slots], dtype=np.int32)


def merge_delta_bound_ok(W_out, W, A, B, slots, gates):
    """A property of a merge that holds at any size, checked on the device over
    every element of one linear: |W'_gpu - W| <= sum_s |g_s| * ||B_{e_s}[o, :]||_1
    * max_j |A_{e_s}[j, i]| (a bound on |sum_s g_s B A|, with 1 % slack for the
    bf16 rounding of the gated factor) + 2^-8 |W'_gpu| (the output rounding),
    and every element finite.  It catches unwritten tiles (the output is filled
    with NaN first) and tiles computed from another tile's W."""
    Wf = W.float()
    d = (W_out.float() - Wf).abs()
    bound = torch.zeros_like(d)
    for e, g in zip(slots, gates):
        e = int(e)
        if e < 0:
            continue
        brow = B[e].float().abs().sum(dim=1)               # [d_out]
        acol = A[e].float().abs().amax(dim=0)              # [d_in]
        bound.add_(torch.outer(brow, acol), alpha=abs(float(g)))
    bound.mul_(1.01).add_(W_out.float().abs(), alpha=2.0 ** -8).add_(1e-30)
    ok = bool(torch.isfinite(W_out.float()).all()) and bool((d <= bound).all())
    return ok
