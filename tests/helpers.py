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
