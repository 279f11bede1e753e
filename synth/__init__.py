"""Seeded synthetic inputs for the fused gated multi-LoRA path.

This module only draws random numbers and lays out tensors; it holds none of
the method's arithmetic (no routing, no merge, no apply).  Both the CUDA path
(through the tests and the benchmark) and the CPU oracle receive their inputs
from here, so neither side ever produces the other's inputs.

Workload shapes follow the Llama2-7B / 13B models on which AdaFuse is
evaluated ("AdaFuse: Accelerating Dynamic Adapter Inference via Token-Level
Pre-Gating and Fused Kernel Optimization", section 4, Experimental results):
a model of L layers, each with the seven targeted linears q, k, v, o (H x H),
gate, up (F x H) and down (H x F), stored as nn.Linear weights [d_out, d_in].

Distributions (the second parameter of N(., .) is a standard deviation):
  W   ~ N(0, 0.02)   bf16   backbone weights
  A_e ~ N(0, 1/16)   bf16   LoRA down projections, [E, r, d_in]
  B_e ~ N(0, 0.01)   bf16   LoRA up projections,   [E, d_out, r]
  x   ~ N(0, 1)      bf16   activations (router input and per-linear inputs)
  W_r ~ N(0, 1/sqrt(H)) fp32 router weights [E, H], so logits are ~N(0, 1)
All values are drawn with torch generators seeded from (seed, tensor id) and
rounded to bf16 by torch's round-to-nearest-even conversion.
"""
from __future__ import annotations

import dataclasses
import hashlib
import math
from typing import Dict, List, Optional

import torch


@dataclasses.dataclass(frozen=True)
class Linear:
    layer: int
    name: str
    d_out: int
    d_in: int


@dataclasses.dataclass(frozen=True)
class Config:
    name: str
    linears: tuple          # tuple[Linear, ...]
    hidden: int             # router input width H
    E: int                  # number of adapters
    r: int                  # LoRA rank
    k: int                  # top-k
    T_merge: int            # tokens routed for the merge (request start)
    T_apply: int            # tokens in the mixed-adapter apply batch

    @property
    def n_lin(self) -> int:
        return len(self.linears)

    @property
    def n_elements(self) -> int:
        return sum(l.d_out * l.d_in for l in self.linears)


def llama_linears(layers: int, hidden: int, ffn: int) -> tuple:
    out = []
    for layer in range(layers):
        for name, d_out, d_in in (("q", hidden, hidden), ("k", hidden, hidden),
                                  ("v", hidden, hidden), ("o", hidden, hidden),
                                  ("gate", ffn, hidden), ("up", ffn, hidden),
                                  ("down", hidden, ffn)):
            out.append(Linear(layer, name, d_out, d_in))
    return tuple(out)


def tiny() -> Config:
    """2 layers, hidden 256, q/v targeted, E=4 rank-8 adapters, top-2, 8 tokens."""
    lins = []
    for layer in range(2):
        for name in ("q", "v"):
            lins.append(Linear(layer, name, 256, 256))
    return Config("tiny", tuple(lins), 256, 4, 8, 2, 8, 8)


def llama7b(layers: int = 32) -> Config:
    """Llama-2-7B shapes: hidden 4096, FFN 11008; E=8 rank-16 adapters, top-2;
    merge for one request (router on one token), apply for 64 sequences."""
    return Config("llama2-7b" if layers == 32 else f"llama2-7b-{layers}L",
                  llama_linears(layers, 4096, 11008), 4096, 8, 16, 2, 1, 64)


def llama13b(layers: int = 40) -> Config:
    """Llama-2-13B shapes: hidden 5120, FFN 13824; E=16 rank-32 adapters, top-2;
    merge for one request, apply for 32 sequences."""
    return Config("llama2-13b" if layers == 40 else f"llama2-13b-{layers}L",
                  llama_linears(layers, 5120, 13824), 5120, 16, 32, 2, 1, 32)


def sweep_point(E: int, r: int, k: int, T: int, d: int = 4096) -> Config:
    """Single 4096x4096 linear with E adapters of rank r, top-k, T tokens."""
    return Config(f"sweep-E{E}-r{r}-k{k}-T{T}", (Linear(0, "w", d, d),),
                  d, E, r, k, 1, T)


def custom(shapes, E, r, k, T, hidden=None, name="custom") -> Config:
    lins = tuple(Linear(0, f"l{i}", int(o), int(i_)) for i, (o, i_) in enumerate(shapes))
    H = hidden if hidden is not None else lins[0].d_in
    return Config(name, lins, H, E, r, k, T, T)


# ---------------------------------------------------------------- generators

def _seed_for(seed: int, tag: str) -> int:
    h = hashlib.sha256(f"{seed}:{tag}".encode()).digest()
    return int.from_bytes(h[:8], "little") & ((1 << 63) - 1)


def normal(shape, std: float, dtype, seed: int, tag: str, device="cpu") -> torch.Tensor:
    """N(0, std) of the given shape, drawn in fp32 and rounded to dtype."""
    g = torch.Generator(device=device)
    g.manual_seed(_seed_for(seed, tag))
    t = torch.randn(shape, generator=g, device=device, dtype=torch.float32)
    t.mul_(std)
    return t.to(dtype)


def fill_normal_(t: torch.Tensor, std: float, seed: int, tag: str, chunk: int = 1 << 28) -> torch.Tensor:
    """In-place N(0, std) fill of a (possibly huge) flat tensor, chunk by chunk,
    so that no fp32 copy of the whole tensor is needed."""
    flat = t.view(-1)
    g = torch.Generator(device=t.device)
    g.manual_seed(_seed_for(seed, tag))
    tmp = torch.empty(min(chunk, flat.numel()), device=t.device, dtype=torch.float32)
    for s in range(0, flat.numel(), chunk):
        n = min(chunk, flat.numel() - s)
        v = tmp[:n]
        v.normal_(0.0, std, generator=g)
        flat[s:s + n].copy_(v)
    return t


W_STD = 0.02
A_STD = 1.0 / 16.0
B_STD = 0.01
X_STD = 1.0


@dataclasses.dataclass
class Weights:
    """Flat device buffers plus per-linear views."""
    W: torch.Tensor            # all backbone weights, flat bf16
    A: torch.Tensor            # all A stacks, flat bf16
    B: torch.Tensor            # all B stacks, flat bf16
    W_views: List[torch.Tensor]
    A_views: List[torch.Tensor]   # [E, r, d_in]
    B_views: List[torch.Tensor]   # [E, d_out, r]
    W_r: torch.Tensor          # [E, H] fp32


def make_weights(cfg: Config, seed: int = 0, device="cpu", zero_w: bool = False) -> Weights:
    E, r = cfg.E, cfg.r
    nW = cfg.n_elements
    nA = sum(E * r * l.d_in for l in cfg.linears)
    nB = sum(E * l.d_out * r for l in cfg.linears)
    W = torch.empty(nW, dtype=torch.bfloat16, device=device)
    A = torch.empty(nA, dtype=torch.bfloat16, device=device)
    B = torch.empty(nB, dtype=torch.bfloat16, device=device)
    if zero_w:
        W.zero_()
    else:
        fill_normal_(W, W_STD, seed, f"{cfg.name}/W")
    fill_normal_(A, A_STD, seed, f"{cfg.name}/A")
    fill_normal_(B, B_STD, seed, f"{cfg.name}/B")
    Wv, Av, Bv = [], [], []
    ow = oa = ob = 0
    for l in cfg.linears:
        n = l.d_out * l.d_in
        Wv.append(W[ow:ow + n].view(l.d_out, l.d_in)); ow += n
        n = E * r * l.d_in
        Av.append(A[oa:oa + n].view(E, r, l.d_in)); oa += n
        n = E * l.d_out * r
        Bv.append(B[ob:ob + n].view(E, l.d_out, r)); ob += n
    return Weights(W, A, B, Wv, Av, Bv, make_router_weights(cfg, seed, device))


def make_router_weights(cfg: Config, seed: int = 0, device="cpu") -> torch.Tensor:
    """[E, H] fp32 router weights, N(0, 1/sqrt(H)) (the W_r of make_weights)."""
    return normal((cfg.E, cfg.hidden), 1.0 / math.sqrt(cfg.hidden), torch.float32, seed,
                  f"{cfg.name}/Wr", device=device)


def make_router_input(cfg: Config, T: int, seed: int = 0, device="cpu", tag="xr") -> torch.Tensor:
    """[T, H] bf16 router input (the hidden state at the first adapted layer)."""
    return normal((T, cfg.hidden), X_STD, torch.bfloat16, seed, f"{cfg.name}/{tag}", device=device)


def make_apply_inputs(cfg: Config, T: int, seed: int = 0, device="cpu"):
    """Per-linear activations x_l [T, d_in] bf16 (one flat buffer + views)."""
    n = sum(T * l.d_in for l in cfg.linears)
    X = torch.empty(n, dtype=torch.bfloat16, device=device)
    fill_normal_(X, X_STD, seed, f"{cfg.name}/xapply/T{T}")
    views, o = [], 0
    for l in cfg.linears:
        views.append(X[o:o + T * l.d_in].view(T, l.d_in)); o += T * l.d_in
    return X, views


def random_selection(T: int, E: int, k: int, seed: int, tag: str = "sel"):
    """A random top-k selection (distinct experts per row) with fp32 gates drawn
    as softmax-like positive weights; used where a test needs a selection that
    does not come from any router."""
    g = torch.Generator()
    g.manual_seed(_seed_for(seed, tag))
    idx = torch.stack([torch.randperm(E, generator=g)[:k] for _ in range(T)]).to(torch.int32)
    gate = torch.rand((T, k), generator=g, dtype=torch.float32) * 0.9 + 0.05
    return idx, gate
