"""ctypes binding of the DyRA C ABI (include/dyra.h).

Argument marshalling only: tensors become device pointers, the current torch
stream becomes the cudaStream_t, and negative return codes become DyraError.
Every step of the layer runs in libdyra.so's CUDA kernels; there is no
fallback. If the library is not built, loading it raises. With
DYRA_DEBUG_LIB=1 in the environment the bounds-checked build libdyra_debug.so
is loaded instead (python -m rank_structured_matmul_b200.build --debug).
"""

from __future__ import annotations

import ctypes
import os
from typing import Optional

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libdyra.so")
DEBUG_LIB_PATH = os.path.join(HERE, "libdyra_debug.so")

DYRA_F32 = 0
DYRA_BF16 = 1

DYRA_OK = 0
DYRA_ERR_INVALID_ARG = -1
DYRA_ERR_NOT_LOADED = -2
DYRA_ERR_ALIGNMENT = -3
DYRA_ERR_RANK_DEFICIENT = -4
DYRA_ERR_ALLOC = -5
DYRA_ERR_CUDA = -6
DYRA_ERR_UNSUPPORTED = -7
DYRA_ERR_DEVICE = -8

DYRA_STATUS_NONPOSITIVE_PIVOT = 1
DYRA_STATUS_WAIT_TIMEOUT = 2
DYRA_STATUS_BOUNDS = 4

# name -> (restype, argtypes), mirroring include/dyra.h
_vp, _i, _i64, _f = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_float
SIGNATURES = {
    "dyra_plan_create": (_i, [ctypes.POINTER(_vp), _i, _i, _i, _i, _i]),
    "dyra_load_factors": (_i, [_vp, _vp, _vp, _vp, _vp, _f, _vp]),
    "dyra_set_linear": (_i, [_vp, _vp, _f, _vp]),
    "dyra_set_als_steps": (_i, [_vp, _i]),
    "dyra_set_solver": (_i, [_vp, _i, _i]),
    "dyra_forward_batched_host": (_i, [_vp, _vp, _vp, _i64, _i64, _vp]),
    "dyra_plan_create_monarch": (_i, [ctypes.POINTER(_vp), _i, _i, _i, _i, _i]),
    "dyra_plan_create_monarch_rect": (_i, [ctypes.POINTER(_vp), _i, _i, _i, _i, _i, _i]),
    "dyra_load_monarch": (_i, [_vp, _vp, _vp, _vp, _vp, _f, _vp]),
    "dyra_forward": (_i, [_vp, _vp, _vp, _i64, _vp]),
    "dyra_forward_batched": (_i, [_vp, _vp, _vp, _i64, _i64, _vp]),
    "dyra_forward_weight_only": (_i, [_vp, _vp, _vp, _i64, _vp]),
    "dyra_forward_batched_noalloc": (_i, [_vp, _vp, _vp, _i64, _i64, _vp]),
    "dyra_reserve": (_i, [_vp, _i64, _i64]),
    "dyra_last_status": (_i, [_vp]),
    "dyra_plan_destroy": (_i, [_vp]),
    "dyra_error_string": (ctypes.c_char_p, [_i]),
    "dyra_plan_device_bytes": (ctypes.c_size_t, [_vp]),
    "dyra_debug_buffer": (_i, [_vp, _i, ctypes.POINTER(_vp), ctypes.POINTER(ctypes.c_size_t)]),
    "dyra_debug_copy": (_i, [_vp, _i, _vp, ctypes.c_size_t]),
    "dyra_debug_gram_split": (_i, [_vp, _i64, _i64, ctypes.POINTER(_i), ctypes.POINTER(_i)]),
    "dyra_debug_set_stage_timing": (_i, [_vp, _i]),
    "dyra_debug_stage_times": (_i, [_vp, ctypes.POINTER(ctypes.c_float)]),
    "dyra_debug_set_trace": (_i, [_vp, _i]),
    "dyra_debug_set_wait_limit": (_i, [_vp, _i, ctypes.c_uint64]),
    "dyra_debug_trace_bytes": (ctypes.c_size_t, []),
    "dyra_debug_trace_copy": (_i, [_vp, _vp, ctypes.c_size_t]),
}

STAGES = ("proj", "gram", "solve", "rfactor", "out")

DYRA_BUF_Z, DYRA_BUF_L, DYRA_BUF_TG, DYRA_BUF_TP, DYRA_BUF_CT = range(5)

_lib = None


class DyraError(RuntimeError):
    def __init__(self, code: int, where: str):
        self.code = code
        super().__init__("%s failed: %s (%d)" % (where, error_string(code), code))


def lib() -> ctypes.CDLL:
    """Load libdyra.so (raises if it has not been built)."""
    global _lib
    if _lib is None:
        debug = os.environ.get("DYRA_DEBUG_LIB") == "1"
        path = DEBUG_LIB_PATH if debug else LIB_PATH
        if not os.path.exists(path):
            raise RuntimeError("%s is not built: run `python -m rank_structured_matmul_b200.build%s`"
                               % (os.path.basename(path), " --debug" if debug else ""))
        handle = ctypes.CDLL(path)
        for name, (res, args) in SIGNATURES.items():
            fn = getattr(handle, name)
            fn.restype = res
            fn.argtypes = args
        _lib = handle
    return _lib


def error_string(code: int) -> str:
    return lib().dyra_error_string(int(code)).decode()


def _check(code: int, where: str) -> int:
    if code < 0:
        raise DyraError(code, where)
    return code


def _ptr(t) -> Optional[int]:
    """Device pointer of a tensor (or an int address, or None)."""
    if t is None:
        return None
    if isinstance(t, int):
        return t
    return t.data_ptr()


def _stream(stream) -> Optional[int]:
    if stream is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


# ---- raw C-ABI wrappers (same names; ints or tensors for pointers) ----

def dyra_plan_create(d_in: int, d_out: int, r: int, k: int, dtype: int) -> int:
    h = ctypes.c_void_p()
    _check(lib().dyra_plan_create(ctypes.byref(h), d_in, d_out, r, k, dtype), "dyra_plan_create")
    return h.value


def dyra_load_factors(plan: int, U, V, P, W_res, lam: float, stream=None) -> None:
    _check(lib().dyra_load_factors(plan, _ptr(U), _ptr(V), _ptr(P), _ptr(W_res), float(lam),
                                   _stream(stream)), "dyra_load_factors")


def dyra_set_linear(plan: int, bias, alpha: float = 1.0, stream=None) -> None:
    _check(lib().dyra_set_linear(plan, _ptr(bias), float(alpha), _stream(stream)),
           "dyra_set_linear")


DYRA_SOLVER_LDL = 0
DYRA_SOLVER_NEWTON_SCHULZ = 1


def dyra_set_solver(plan: int, solver: int, max_iters: int = 40) -> None:
    _check(lib().dyra_set_solver(plan, int(solver), int(max_iters)), "dyra_set_solver")


def dyra_set_als_steps(plan: int, half_steps: int) -> None:
    _check(lib().dyra_set_als_steps(plan, int(half_steps)), "dyra_set_als_steps")


def dyra_forward_batched_host(plan: int, X, Y, B: int, T: int, stream=None) -> None:
    """dyra_forward_batched on host buffers (X, Y page-locked CPU tensors or addresses)."""
    _check(lib().dyra_forward_batched_host(plan, _ptr(X), _ptr(Y), int(B), int(T),
                                           _stream(stream)), "dyra_forward_batched_host")


def dyra_plan_create_monarch(n: int, b1: int, b2: int, k: int, dtype: int) -> int:
    h = ctypes.c_void_p()
    _check(lib().dyra_plan_create_monarch(ctypes.byref(h), n, b1, b2, k, dtype),
           "dyra_plan_create_monarch")
    return h.value


def dyra_plan_create_monarch_rect(b1: int, b2: int, b1o: int, b2o: int, k: int,
                                  dtype: int) -> int:
    h = ctypes.c_void_p()
    _check(lib().dyra_plan_create_monarch_rect(ctypes.byref(h), b1, b2, b1o, b2o, k, dtype),
           "dyra_plan_create_monarch_rect")
    return h.value


def dyra_load_monarch(plan: int, Lblocks, Rblocks, P, W_res, lam: float, stream=None) -> None:
    _check(lib().dyra_load_monarch(plan, _ptr(Lblocks), _ptr(Rblocks), _ptr(P), _ptr(W_res),
                                   float(lam), _stream(stream)), "dyra_load_monarch")


def dyra_forward(plan: int, X, Y, N: int, stream=None) -> None:
    _check(lib().dyra_forward(plan, _ptr(X), _ptr(Y), int(N), _stream(stream)), "dyra_forward")


def dyra_forward_batched(plan: int, X, Y, B: int, T: int, stream=None) -> None:
    _check(lib().dyra_forward_batched(plan, _ptr(X), _ptr(Y), int(B), int(T), _stream(stream)),
           "dyra_forward_batched")


def dyra_forward_weight_only(plan: int, X, Y, N: int, stream=None) -> None:
    _check(lib().dyra_forward_weight_only(plan, _ptr(X), _ptr(Y), int(N), _stream(stream)),
           "dyra_forward_weight_only")


def dyra_forward_batched_noalloc(plan: int, X, Y, B: int, T: int, stream=None) -> None:
    """dyra_forward_batched with the intermediates in the library's fixed
    device array instead of plan workspace; no device allocation."""
    _check(lib().dyra_forward_batched_noalloc(plan, _ptr(X), _ptr(Y), int(B), int(T),
                                              _stream(stream)), "dyra_forward_batched_noalloc")


def dyra_reserve(plan: int, B: int, T: int) -> None:
    _check(lib().dyra_reserve(plan, int(B), int(T)), "dyra_reserve")


def dyra_last_status(plan: int) -> int:
    return _check(lib().dyra_last_status(plan), "dyra_last_status")


def dyra_plan_destroy(plan: int) -> None:
    _check(lib().dyra_plan_destroy(plan), "dyra_plan_destroy")


def dyra_plan_device_bytes(plan: int) -> int:
    return int(lib().dyra_plan_device_bytes(plan))


def dyra_debug_copy(plan: int, which: int, nbytes: int):
    """Copy the first nbytes of a workspace buffer to a new host bytearray."""
    buf = (ctypes.c_char * nbytes)()
    _check(lib().dyra_debug_copy(plan, which, buf, nbytes), "dyra_debug_copy")
    return bytes(buf)


def dyra_debug_gram_split(plan: int, B: int, T: int):
    s, r = ctypes.c_int(), ctypes.c_int()
    _check(lib().dyra_debug_gram_split(plan, B, T, ctypes.byref(s), ctypes.byref(r)),
           "dyra_debug_gram_split")
    return s.value, r.value


def dyra_debug_set_stage_timing(plan: int, enable: bool) -> None:
    _check(lib().dyra_debug_set_stage_timing(plan, int(bool(enable))),
           "dyra_debug_set_stage_timing")


def dyra_debug_set_wait_limit(plan: int, stage: int, ns: int) -> None:
    """Wait limit of one pipeline wait of `stage` in ns (0: the default)."""
    _check(lib().dyra_debug_set_wait_limit(plan, int(stage), int(ns)), "dyra_debug_set_wait_limit")


def dyra_debug_stage_times(plan: int):
    """{stage: milliseconds} of the last forward with stage timing enabled."""
    ms = (ctypes.c_float * 5)()
    _check(lib().dyra_debug_stage_times(plan, ms), "dyra_debug_stage_times")
    return dict(zip(STAGES, list(ms)))


def dyra_debug_set_trace(plan: int, enable: bool) -> None:
    _check(lib().dyra_debug_set_trace(plan, int(bool(enable))), "dyra_debug_set_trace")


def dyra_debug_trace(plan: int):
    """Timeline stamps as a uint64 array [5 stages][256 CTAs][64 slots]."""
    import numpy as np
    n = int(lib().dyra_debug_trace_bytes())
    buf = (ctypes.c_char * n)()
    _check(lib().dyra_debug_trace_copy(plan, buf, n), "dyra_debug_trace_copy")
    return np.frombuffer(bytes(buf), dtype=np.uint64).reshape(5, 256, 64)


# ---- convenience object ----

class DyraLinear:
    """One DyRA layer on the current CUDA device.

    Factors are torch tensors (any device/dtype; copied to the plan dtype on the
    device): U (d_out x r), V (d_in x r), P (d_in x k), W_res (d_out x d_in).
    """

    def __init__(self, d_in: int, d_out: int, r: int, k: int, dtype: str = "bf16"):
        import torch
        self.d_in, self.d_out, self.r, self.k = d_in, d_out, r, k
        self.dtype = dtype
        self.torch_dtype = {"bf16": torch.bfloat16, "f32": torch.float32}[dtype]
        self.plan = dyra_plan_create(d_in, d_out, r, k, DYRA_BF16 if dtype == "bf16" else DYRA_F32)

    def _dev(self, t):
        import torch
        return t.to(device="cuda", dtype=self.torch_dtype).contiguous() if t is not None else None

    def load(self, U, V, P, W_res, lam: float, stream=None) -> None:
        import torch
        U, V, P, W_res = (self._dev(t) for t in (U, V, P, W_res))
        dyra_load_factors(self.plan, U, V, P if self.k else None, W_res if self.k else None,
                          lam, stream)
        torch.cuda.current_stream().synchronize() if stream is None else stream.synchronize()

    def set_linear(self, bias=None, alpha: float = 1.0, stream=None) -> None:
        """Bias (d_out values, or None) and correction weight of the full
        linear layer, Y = static + bias + alpha * correction."""
        import torch
        b = self._dev(bias)
        dyra_set_linear(self.plan, b, alpha, stream)
        torch.cuda.current_stream().synchronize() if stream is None else stream.synchronize()

    def set_als_iterations(self, t: float) -> None:
        """t ALS iterations per forward (t = 1, 1.5, 2, ...; DyRA Sec. 3.3)."""
        steps = int(round(2 * t))
        if steps != 2 * t:
            raise ValueError("t must be a multiple of 0.5")
        dyra_set_als_steps(self.plan, steps)

    def _check_x(self, X):
        import torch
        if not (X.is_cuda and X.dtype == self.torch_dtype and X.is_contiguous()
                and X.dim() == 2 and X.shape[1] == self.d_in):
            raise ValueError("X must be a contiguous CUDA %s tensor of shape (N, %d)"
                             % (self.torch_dtype, self.d_in))

    def forward(self, X, B: int = 1, T: Optional[int] = None, Y=None, stream=None):
        import torch
        self._check_x(X)
        N = X.shape[0]
        if T is None:
            T = N // B
        if B * T != N:
            raise ValueError("B*T must equal the row count of X")
        if Y is None:
            Y = torch.empty((N, self.d_out), device=X.device, dtype=self.torch_dtype)
        dyra_forward_batched(self.plan, X, Y, B, T, stream)
        return Y

    def forward_host(self, X, B: int = 1, T: Optional[int] = None, Y=None, stream=None):
        """forward() on host tensors: copies in, the layer and copies out overlap
        by chunks of instances. X and Y should be pinned CPU tensors; the call is
        asynchronous on the stream (synchronise it before reading Y)."""
        import torch
        if X.is_cuda or X.dtype != self.torch_dtype or not X.is_contiguous() or X.dim() != 2 \
                or X.shape[1] != self.d_in:
            raise ValueError("X must be a contiguous CPU %s tensor of shape (N, %d)"
                             % (self.torch_dtype, self.d_in))
        N = X.shape[0]
        if T is None:
            T = N // B
        if B * T != N:
            raise ValueError("B*T must equal the row count of X")
        if Y is None:
            Y = torch.empty((N, self.d_out), dtype=self.torch_dtype).pin_memory()
        dyra_forward_batched_host(self.plan, X, Y, B, T, stream)
        return Y

    def forward_weight_only(self, X, Y=None, stream=None):
        import torch
        self._check_x(X)
        if Y is None:
            Y = torch.empty((X.shape[0], self.d_out), device=X.device, dtype=self.torch_dtype)
        dyra_forward_weight_only(self.plan, X, Y, X.shape[0], stream)
        return Y

    def reserve(self, B: int, T: int) -> None:
        dyra_reserve(self.plan, B, T)

    def status(self) -> int:
        return dyra_last_status(self.plan)

    def close(self) -> None:
        if self.plan:
            dyra_plan_destroy(self.plan)
            self.plan = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


class DyraMonarchLinear(DyraLinear):
    """A DyRA layer whose static part is a Monarch matrix (DyRA App. B) of
    d_in = b1 * b2 input and d_out = b1o * b2o output features (square unless
    b1o, b2o are given); load() takes the blocks instead of U and V."""

    def __init__(self, n: int, b1: int, b2: int, k: int, dtype: str = "bf16",
                 b1o: Optional[int] = None, b2o: Optional[int] = None):
        import torch
        b1o = b1 if b1o is None else b1o
        b2o = b2 if b2o is None else b2o
        if n != b1 * b2:
            raise ValueError("n must be b1 * b2")
        self.d_in, self.d_out = n, b1o * b2o
        self.r, self.k, self.b1, self.b2, self.b1o, self.b2o = 0, k, b1, b2, b1o, b2o
        self.dtype = dtype
        self.torch_dtype = {"bf16": torch.bfloat16, "f32": torch.float32}[dtype]
        self.plan = dyra_plan_create_monarch_rect(b1, b2, b1o, b2o, k,
                                                  DYRA_BF16 if dtype == "bf16" else DYRA_F32)

    def load(self, Lblocks, Rblocks, P, W_res, lam: float, stream=None) -> None:
        """Lblocks: (b2, b1, b1o), Rblocks: (b1o, b2, b2o), P: (d_in, k),
        W_res: (d_out, d_in)."""
        import torch
        Lb, Rb, P, W_res = (self._dev(t) for t in (Lblocks, Rblocks, P, W_res))
        dyra_load_monarch(self.plan, Lb, Rb, P if self.k else None, W_res if self.k else None,
                          lam, stream)
        torch.cuda.current_stream().synchronize() if stream is None else stream.synchronize()
