"""Python binding of libadafuse.so (the AdaFuse fused gated multi-LoRA path on
B200).  Argument marshalling only: every step of the path runs in the CUDA
kernels behind the C ABI declared in include/adafuse.h.  PyTorch supplies
device memory and streams.  There is no fallback: if the shared library is
missing or fails to load, importing the binding's entry points raises.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional, Sequence

__all__ = [
    "AdafuseError", "lib", "library_path", "pregate", "segments", "Plan", "PointerArrays",
    "RENORM", "POOL_MEAN", "STATUS_BAD_INDEX", "STATUS_TIMEOUT", "PLAN_Y_F32", "round_bf16",
]

_HERE = os.path.dirname(os.path.abspath(__file__))
_LIB_PATH = os.path.join(_HERE, "libadafuse.so")

OK = 0
ERR_INVALID_ARG = 1
ERR_UNSUPPORTED = 2
ERR_WORKSPACE_TOO_SMALL = 3
ERR_CUDA = 4
ERR_TIMEOUT = 5
ERR_DEVICE = 6
RENORM = 1 << 0
POOL_MEAN = 1 << 1
STATUS_BAD_INDEX = 1 << 0
STATUS_TIMEOUT = 1 << 1
PLAN_Y_F32 = 1 << 0
PLAN_TEST_STALL = 1 << 31

# Every entry point the header declares.
EXPORTS = (
    "adafuse_plan_create", "adafuse_plan_destroy", "adafuse_pregate", "adafuse_merge",
    "adafuse_switch", "adafuse_merge_per_linear", "adafuse_segments",
    "adafuse_apply_workspace_bytes", "adafuse_apply", "adafuse_plan_status",
    "adafuse_plan_last_launches", "adafuse_strerror", "adafuse_version",
    "adafuse_apply_noalloc", "adafuse_round_bf16",
)


class AdafuseError(RuntimeError):
    def __init__(self, code: int, where: str):
        self.code = code
        msg = _lib.adafuse_strerror(code).decode() if _lib is not None else str(code)
        super().__init__(f"{where}: {msg} (code {code})")


class Linear(ctypes.Structure):
    _fields_ = [
        ("W", ctypes.c_void_p), ("W_out", ctypes.c_void_p),
        ("A", ctypes.c_void_p), ("B", ctypes.c_void_p),
        ("d_out", ctypes.c_int32), ("d_in", ctypes.c_int32),
        ("a_expert_stride", ctypes.c_int64), ("b_expert_stride", ctypes.c_int64),
    ]


_lib = None


def library_path() -> str:
    return _LIB_PATH


def lib():
    """Load libadafuse.so (built by adapter_merge_b200.build); raise if absent."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(_LIB_PATH):
        raise RuntimeError(f"libadafuse.so not built ({_LIB_PATH}); run adapter_merge_b200.build.build()")
    L = ctypes.CDLL(_LIB_PATH)
    P, i32, i64, u32 = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_uint32
    L.adafuse_plan_create.argtypes = [ctypes.POINTER(P), ctypes.POINTER(Linear), i32, i32, i32, u32]
    L.adafuse_plan_destroy.argtypes = [P]
    L.adafuse_plan_destroy.restype = None
    L.adafuse_pregate.argtypes = [P, i64, i32, i64, P, P, i32, i32, u32, P, P, P]
    L.adafuse_merge.argtypes = [P, P, P, i32, P]
    L.adafuse_switch.argtypes = [P, P, P, P, P, i32, P]
    L.adafuse_merge_per_linear.argtypes = [P, P, P, i32, P]
    L.adafuse_segments.argtypes = [P, i64, i32, i32, P, P, P, P, P]
    L.adafuse_apply_workspace_bytes.argtypes = [P, i64, i32]
    L.adafuse_apply_workspace_bytes.restype = ctypes.c_size_t
    L.adafuse_apply.argtypes = [P, P, P, i64, P, P, i32, P, ctypes.c_size_t, P]
    L.adafuse_apply_noalloc.argtypes = [P, P, P, i64, P, P, i32, P]
    L.adafuse_round_bf16.argtypes = [P, P, i64, P]
    L.adafuse_plan_status.argtypes = [P, P, ctypes.POINTER(i32)]
    L.adafuse_plan_last_launches.argtypes = [P]
    L.adafuse_plan_last_launches.restype = i32
    L.adafuse_strerror.argtypes = [ctypes.c_int]
    L.adafuse_strerror.restype = ctypes.c_char_p
    L.adafuse_version.restype = i32
    for name in EXPORTS:
        getattr(L, name)
    _lib = L
    return L


def _check(rc: int, where: str):
    if rc != OK:
        raise AdafuseError(rc, where)


def _ptr(t) -> Optional[int]:
    return None if t is None else t.data_ptr()


def _stream(stream) -> Optional[int]:
    if stream is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    return stream if isinstance(stream, int) else stream.cuda_stream


def pregate(x, W_r, k: int, b_r=None, renorm: bool = False, pool: bool = False,
            idx=None, gate=None, stream=None):
    """Token-level pre-gating: returns (idx int32 [T,k], gate fp32 [T,k]) on the
    device ([1,k] with pool=True).  x bf16 [T, H] (rows may be strided)."""
    import torch
    T, H = x.shape
    E = W_r.shape[0]
    rows = 1 if pool else T
    if idx is None:
        idx = torch.empty((rows, k), dtype=torch.int32, device=x.device)
    if gate is None:
        gate = torch.empty((rows, k), dtype=torch.float32, device=x.device)
    flags = (RENORM if renorm else 0) | (POOL_MEAN if pool else 0)
    _check(lib().adafuse_pregate(_ptr(x), T, H, x.stride(0), _ptr(W_r), _ptr(b_r), E, k, flags,
                                 _ptr(idx), _ptr(gate), _stream(stream)), "adafuse_pregate")
    return idx, gate


def segments(idx, E: int, status=None, stream=None):
    """Stable segment build: (offsets [E+1], perm [T*k], used [E+1]) on the device."""
    import torch
    T, k = idx.shape
    offsets = torch.empty(E + 1, dtype=torch.int32, device=idx.device)
    perm = torch.full((T * k,), -1, dtype=torch.int32, device=idx.device)
    used = torch.zeros(E + 1, dtype=torch.int32, device=idx.device)
    _check(lib().adafuse_segments(_ptr(idx), T, k, E, _ptr(offsets), _ptr(perm), _ptr(used),
                                  _ptr(status), _stream(stream)), "adafuse_segments")
    return offsets, perm, used


def round_bf16(src, out=None, stream=None):
    """bf16 round-to-nearest-even of an fp32 device tensor into `out` (a new
    bf16 tensor of src's shape if None); returns out."""
    import torch
    if src.dtype != torch.float32 or not src.is_contiguous():
        raise ValueError("round_bf16 takes a contiguous fp32 tensor")
    if out is None:
        out = torch.empty(src.shape, dtype=torch.bfloat16, device=src.device)
    if out.dtype != torch.bfloat16 or not out.is_contiguous() or out.numel() != src.numel():
        raise ValueError("round_bf16 writes a contiguous bf16 tensor of src's size")
    _check(lib().adafuse_round_bf16(_ptr(src), _ptr(out), src.numel(), _stream(stream)), "adafuse_round_bf16")
    return out


class Plan:
    """A plan over a list of targeted linears sharing E rank-r adapters.

    `linears` is a sequence of (W, W_out, A, B) device tensors per linear:
    W, W_out bf16 [d_out, d_in]; A bf16 [E, r, d_in]; B bf16 [E, d_out, r]
    (any expert stride, row-major inside an expert).  The tensors must stay
    alive while the plan exists.  `flags`: PLAN_Y_F32 makes apply write fp32
    outputs (the row-parallel partials of tensor parallelism).
    """

    def __init__(self, linears: Sequence, E: int, r: int, flags: int = 0):
        arr = (Linear * len(linears))()
        for i, (W, W_out, A, B) in enumerate(linears):
            d_out, d_in = W.shape
            for t, inner in ((W, (d_in, 1)), (W_out, (d_in, 1)), (A, (d_in, 1)), (B, (r, 1))):
                if tuple(t.stride()[-2:]) != inner and t.shape[-2] > 1:
                    raise ValueError(f"linear {i}: tensors must be row-major inside each expert "
                                     f"(strides {tuple(t.stride())})")
            a_es = A.stride(0) if A.shape[0] > 1 else r * d_in
            b_es = B.stride(0) if B.shape[0] > 1 else d_out * r
            arr[i] = Linear(W.data_ptr(), W_out.data_ptr(), A.data_ptr(), B.data_ptr(),
                            d_out, d_in, a_es, b_es)
        self._keep = list(linears)
        self.E, self.r, self.n_lin = E, r, len(linears)
        h = ctypes.c_void_p()
        _check(lib().adafuse_plan_create(ctypes.byref(h), arr, len(linears), E, r, flags), "adafuse_plan_create")
        self._h = h

    @property
    def handle(self):
        return self._h

    def merge(self, idx, gate, k: Optional[int] = None, stream=None):
        k = idx.numel() if k is None else k
        _check(lib().adafuse_merge(self._h, _ptr(idx), _ptr(gate), k, _stream(stream)), "adafuse_merge")

    def switch(self, idx_new, gate_new, idx_old, gate_old, k: Optional[int] = None, stream=None):
        k = idx_new.numel() if k is None else k
        _check(lib().adafuse_switch(self._h, _ptr(idx_new), _ptr(gate_new), _ptr(idx_old), _ptr(gate_old), k,
                                    _stream(stream)), "adafuse_switch")

    def merge_per_linear(self, idx, gate, k: Optional[int] = None, stream=None):
        k = idx.numel() if k is None else k
        _check(lib().adafuse_merge_per_linear(self._h, _ptr(idx), _ptr(gate), k, _stream(stream)),
               "adafuse_merge_per_linear")

    def workspace_bytes(self, T: int, k: int) -> int:
        return int(lib().adafuse_apply_workspace_bytes(self._h, T, k))

    def apply(self, xs, ys, T: int, idx, gate, workspace, stream=None):
        """Segmented-gather apply over every linear.  xs / ys: per-linear device
        tensors (x_l [T, d_in], y_l [T, d_out]) or a PointerArrays built once
        from them (cheaper per call)."""
        k = idx.shape[1]
        ptrs = xs if isinstance(xs, PointerArrays) else PointerArrays(xs, ys)
        _check(lib().adafuse_apply(self._h, ptrs.x, ptrs.y, T, _ptr(idx), _ptr(gate), k,
                                   _ptr(workspace), workspace.numel() * workspace.element_size(),
                                   _stream(stream)), "adafuse_apply")

    def apply_noalloc(self, xs, ys, T: int, idx, gate, stream=None) -> int:
        """As apply, with the library's own fixed device scratch instead of a
        workspace (for callers that cannot allocate device memory).  Returns the
        C return code (ADAFUSE_ERR_WORKSPACE_TOO_SMALL when the call does not
        fit the scratch) instead of raising, so callers can fall back to apply."""
        k = idx.shape[1]
        ptrs = xs if isinstance(xs, PointerArrays) else PointerArrays(xs, ys)
        return int(lib().adafuse_apply_noalloc(self._h, ptrs.x, ptrs.y, T, _ptr(idx), _ptr(gate), k,
                                               _stream(stream)))

    def status(self, stream=None):
        """(return code, device status bits); clears the status word."""
        v = ctypes.c_int32(0)
        rc = lib().adafuse_plan_status(self._h, _stream(stream), ctypes.byref(v))
        return rc, v.value

    @property
    def last_launches(self) -> int:
        return int(lib().adafuse_plan_last_launches(self._h))

    def destroy(self):
        if getattr(self, "_h", None) is not None and self._h.value:
            lib().adafuse_plan_destroy(self._h)
            self._h = ctypes.c_void_p()

    def __del__(self):
        try:
            self.destroy()
        except Exception:
            pass


class PointerArrays:
    """Host arrays of the device pointers of x_l and y_l, in linear order."""

    def __init__(self, xs, ys):
        addr = lambda t: t if isinstance(t, int) else t.data_ptr()
        self.x = (ctypes.c_void_p * len(xs))(*[addr(t) for t in xs])
        self.y = (ctypes.c_void_p * len(ys))(*[addr(t) for t in ys])
        self._keep = (list(xs), list(ys))
