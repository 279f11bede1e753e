"""CPU oracle for the AdaFuse fused gated multi-LoRA path (test infrastructure).

Only tests/, __graft_entry__.smoke() and bench.py's CPU-baseline leg may import
this package.  The product path (adapter_merge_b200) never imports it, and it
never imports the product path: the two share no code.

The arithmetic lives in plain C (adafuse_oracle.c, built with gcc and
-ffp-contract=off); this module only marshals numpy arrays.  bf16 tensors are
passed as their uint16 bit patterns.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading
from typing import Optional, Sequence

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "adafuse_oracle.c")
_LIB = os.path.join(_HERE, "liborc.so")
# A test may point this at a deliberately broken build of the oracle to show
# that the pins catch the mistake (mutation check, CPU only).
_LIB_OVERRIDE = os.environ.get("ADAFUSE_ORACLE_LIB")
_lock = threading.Lock()
_lib = None


def build(force: bool = False) -> str:
    """Compile the oracle with gcc into oracle/liborc.so (idempotent)."""
    if (not force and os.path.exists(_LIB)
            and os.path.getmtime(_LIB) >= os.path.getmtime(_SRC)):
        return _LIB
    tmp = _LIB + f".tmp{os.getpid()}"
    cmd = ["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-fopenmp",
           "-ffp-contract=off", "-fno-fast-math", "-o", tmp, _SRC, "-lm"]
    subprocess.check_call(cmd)
    os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    with _lock:
        if _lib is not None:
            return _lib
        if _LIB_OVERRIDE:
            lib = ctypes.CDLL(_LIB_OVERRIDE)
        else:
            build()
            lib = ctypes.CDLL(_LIB)
        P = ctypes.c_void_p
        i32, i64, f64 = ctypes.c_int32, ctypes.c_int64, ctypes.c_double
        lib.orc_bf16_to_double.argtypes = [ctypes.c_uint16]
        lib.orc_bf16_to_double.restype = f64
        lib.orc_bf16_from_double.argtypes = [f64]
        lib.orc_bf16_from_double.restype = ctypes.c_uint16
        lib.orc_bf16_from_double_array.argtypes = [P, P, i64]
        lib.orc_router_logits.argtypes = [P, i64, i32, i64, P, P, i32, P]
        lib.orc_pool_mean.argtypes = [P, i64, i32, i64, P]
        lib.orc_router_logits_f32.argtypes = [P, i32, P, P, i32, P]
        lib.orc_topk_softmax.argtypes = [P, i64, i32, i32, i32, P, P]
        lib.orc_merge_linear.argtypes = [P, P, P, P, i32, i32, i32, i32, i64, i64,
                                         P, P, i32, i64, i64, i32]
        lib.orc_apply_linear.argtypes = [P, P, P, P, i32, i32, i32, i32, i64, i64,
                                         P, P, i32, i64, i64, P, i32]
        lib.orc_apply_linear_f64.argtypes = [P, P, P, P, i32, i32, i32, i32, i64, i64,
                                             P, P, i32, i64, i64, P, i32]
        lib.orc_segments.argtypes = [P, i64, i32, i32, P, P]
        lib.orc_segments.restype = i32
        lib.orc_max_threads.restype = i32
        _lib = lib
        return lib


def _p(a: Optional[np.ndarray]):
    return None if a is None else ctypes.c_void_p(a.ctypes.data)


def _u16(a) -> np.ndarray:
    a = np.ascontiguousarray(a)
    if a.dtype != np.uint16:
        a = a.view(np.uint16) if a.dtype.itemsize == 2 else a.astype(np.uint16)
    return a


def max_threads() -> int:
    return int(_load().orc_max_threads())


# ------------------------------------------------------------------- bf16

def bf16_to_f64(bits: np.ndarray) -> np.ndarray:
    bits = _u16(bits)
    # signalling-NaN patterns widen to quiet NaNs; numpy flags that as "invalid"
    with np.errstate(invalid="ignore"):
        return (bits.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def bf16_from_f64(v: np.ndarray) -> np.ndarray:
    v = np.ascontiguousarray(v, dtype=np.float64)
    out = np.empty(v.shape, dtype=np.uint16)
    _load().orc_bf16_from_double_array(_p(v), _p(out), v.size)
    return out


# ----------------------------------------------------------------- router

def router_logits(x_bits: np.ndarray, W_r: np.ndarray, b_r: Optional[np.ndarray] = None) -> np.ndarray:
    """fp32 logits [T, E] of bf16 rows x [T, H] against W_r [E, H]."""
    x = _u16(x_bits)
    T, H = x.shape
    W_r = np.ascontiguousarray(W_r, dtype=np.float32)
    E = W_r.shape[0]
    b = None if b_r is None else np.ascontiguousarray(b_r, dtype=np.float32)
    z = np.empty((T, E), dtype=np.float32)
    _load().orc_router_logits(_p(x), T, H, H, _p(W_r), _p(b), E, _p(z))
    return z


def pool_mean(x_bits: np.ndarray) -> np.ndarray:
    x = _u16(x_bits)
    T, H = x.shape
    out = np.empty(H, dtype=np.float32)
    _load().orc_pool_mean(_p(x), T, H, H, _p(out))
    return out


def router_logits_f32(xrow: np.ndarray, W_r: np.ndarray, b_r: Optional[np.ndarray] = None) -> np.ndarray:
    xrow = np.ascontiguousarray(xrow, dtype=np.float32)
    W_r = np.ascontiguousarray(W_r, dtype=np.float32)
    E, H = W_r.shape
    b = None if b_r is None else np.ascontiguousarray(b_r, dtype=np.float32)
    z = np.empty(E, dtype=np.float32)
    _load().orc_router_logits_f32(_p(xrow), H, _p(W_r), _p(b), E, _p(z))
    return z


def topk_softmax(z: np.ndarray, k: int, renorm: bool = False):
    """(idx int32 [T,k], gate float64 [T,k]) from fp32 logits [T, E]."""
    z = np.ascontiguousarray(z, dtype=np.float32)
    T, E = z.shape
    if not (1 <= k <= E <= 64):
        raise ValueError("need 1 <= k <= E <= 64")
    idx = np.empty((T, k), dtype=np.int32)
    gate = np.empty((T, k), dtype=np.float64)
    _load().orc_topk_softmax(_p(z), T, E, k, int(bool(renorm)), _p(idx), _p(gate))
    return idx, gate


def pregate(x_bits, W_r, k, b_r=None, renorm=False, pool=False):
    """Token-level pre-gating: logits, top-k and gates for each row of x (or,
    with pool=True, for the mean of the rows)."""
    if pool:
        z = router_logits_f32(pool_mean(x_bits), W_r, b_r)[None, :]
    else:
        z = router_logits(x_bits, W_r, b_r)
    idx, gate = topk_softmax(z, k, renorm)
    return idx, gate, z


def topk_margin(z: np.ndarray, k: int) -> np.ndarray:
    """Per row of logits z [T, E]: z_(k) - z_(k+1), the gap between the k-th
    and the (k+1)-th largest logit (inf when k == E).  A selection whose gap
    is within the rounding of the logit sum depends on the summation order."""
    zs = -np.sort(-np.asarray(z, dtype=np.float64), axis=1)
    if k >= zs.shape[1]:
        return np.full(zs.shape[0], np.inf)
    return zs[:, k - 1] - zs[:, k]


def router_scale(x_bits, W_r: np.ndarray) -> np.ndarray:
    """Per row of x [T, H]: max over experts of sum_j |x_j| |W_r[e, j]|, the
    scale the rounding error of a logit is proportional to."""
    x = bf16_to_f64(_u16(x_bits))
    return (np.abs(x) @ np.abs(np.asarray(W_r, dtype=np.float64)).T).max(axis=1)


# ------------------------------------------------------------------ merge

def merge_linear(W_bits, A_bits, B_bits, eidx: Sequence[int], gates: Sequence[float],
                 rows=None, nthreads: int = 1) -> np.ndarray:
    """W' rows [row0,row1) of one linear: bf16(W + sum_s g_s B_{e_s} A_{e_s}).

    W [d_out, d_in], A [E, r, d_in], B [E, d_out, r] as bf16 bit patterns.
    """
    W = _u16(W_bits); A = _u16(A_bits); B = _u16(B_bits)
    d_out, d_in = W.shape
    E, r, _ = A.shape
    e = np.ascontiguousarray(np.asarray(eidx, dtype=np.int32).reshape(-1))
    g = np.ascontiguousarray(np.asarray(gates, dtype=np.float64).reshape(-1))
    assert e.size == g.size
    row0, row1 = (0, d_out) if rows is None else rows
    out = np.empty((row1 - row0, d_in), dtype=np.uint16)
    _load().orc_merge_linear(_p(W), _p(out), _p(A), _p(B), d_out, d_in, E, r,
                             r * d_in, d_out * r, _p(e), _p(g), e.size,
                             row0, row1, nthreads)
    return out


def apply_linear(x_bits, W_bits, A_bits, B_bits, idx, gate, tokens=None,
                 nthreads: int = 1) -> np.ndarray:
    """y rows for tokens [t0,t1) of one linear (unmerged mixed-batch form)."""
    x = _u16(x_bits); W = _u16(W_bits); A = _u16(A_bits); B = _u16(B_bits)
    T, d_in = x.shape
    d_out = W.shape[0]
    E, r, _ = A.shape
    idx = np.ascontiguousarray(idx, dtype=np.int32)
    gate = np.ascontiguousarray(gate, dtype=np.float64)
    k = idx.shape[1]
    t0, t1 = (0, T) if tokens is None else tokens
    y = np.empty((t1 - t0, d_out), dtype=np.uint16)
    _load().orc_apply_linear(_p(x), _p(W), _p(A), _p(B), d_out, d_in, E, r,
                             r * d_in, d_out * r, _p(idx), _p(gate), k, t0, t1,
                             _p(y), nthreads)
    return y


def apply_linear_f64(x_bits, W_bits, A_bits, B_bits, idx, gate, tokens=None,
                     nthreads: int = 1) -> np.ndarray:
    """As apply_linear, but the rows of y unrounded (float64): the partial
    output of a row-parallel shard, whose sum over the shards is rounded once."""
    x = _u16(x_bits); W = _u16(W_bits); A = _u16(A_bits); B = _u16(B_bits)
    T, d_in = x.shape
    d_out = W.shape[0]
    E, r, _ = A.shape
    idx = np.ascontiguousarray(idx, dtype=np.int32)
    gate = np.ascontiguousarray(gate, dtype=np.float64)
    k = idx.shape[1]
    t0, t1 = (0, T) if tokens is None else tokens
    y = np.empty((t1 - t0, d_out), dtype=np.float64)
    _load().orc_apply_linear_f64(_p(x), _p(W), _p(A), _p(B), d_out, d_in, E, r,
                                 r * d_in, d_out * r, _p(idx), _p(gate), k, t0, t1,
                                 _p(y), nthreads)
    return y


def segments(idx: np.ndarray, E: int):
    """(offsets [E+1], perm [n_valid], n_bad) of the stable sort by expert."""
    idx = np.ascontiguousarray(idx, dtype=np.int32)
    T, k = idx.shape
    offsets = np.empty(E + 1, dtype=np.int32)
    perm = np.full(T * k, -1, dtype=np.int32)
    bad = _load().orc_segments(_p(idx), T, k, E, _p(offsets), _p(perm))
    return offsets, perm[: T * k - bad], int(bad)
