"""ctypes binding of libpn (include/pn.h): argument marshalling only.

Every computation happens inside libpn's CUDA kernels.  The module-level
functions carry the C names (``pn_create``, ``pn_eval``, ...) and take plain
integers for pointers and streams; :class:`Solver` wraps them for torch tensors.
There is no fallback: if ``libpn.so`` is missing or fails to load, importing
this module raises.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional, Tuple

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libpn.so")

PN_OK, PN_NOT_CONVERGED = 0, 1
PN_ERR_INVALID, PN_ERR_NOMEM, PN_ERR_CUDA, PN_ERR_NONFINITE, PN_ERR_TIMEOUT = -1, -2, -3, -4, -5
PN_CELL_TANH_RNN, PN_CELL_GRU, PN_CELL_EULER_TANH = 0, 1, 2
PN_JACOBI, PN_PICARD, PN_QUASI, PN_NEWTON = 0, 1, 2, 3
PN_OPT_WAIT_TIMEOUT_NS, PN_OPT_DEBUG_STALL_TICKET, PN_OPT_DEVICE_LOOP, PN_OPT_TENSOR_CORES = 0, 1, 2, 3
PN_OPT_NEWTON_BAND = 4
PN_OPT_RUN_LENGTH = 5
PN_OPT_SMALL_SOLVE = 6
PN_STORE_F32, PN_STORE_BF16, PN_STORE_F16 = 0, 1, 2
PN_MAX_D_DIAG, PN_MAX_D_NEWTON = 256, 64

STATUS_NAMES = {PN_OK: "PN_OK", PN_NOT_CONVERGED: "PN_NOT_CONVERGED", PN_ERR_INVALID: "PN_ERR_INVALID",
                PN_ERR_NOMEM: "PN_ERR_NOMEM", PN_ERR_CUDA: "PN_ERR_CUDA",
                PN_ERR_NONFINITE: "PN_ERR_NONFINITE", PN_ERR_TIMEOUT: "PN_ERR_TIMEOUT"}
MODES = {"jacobi": PN_JACOBI, "picard": PN_PICARD, "quasi": PN_QUASI, "newton": PN_NEWTON}

# Every symbol include/pn.h declares, with (restype, argtypes).
_c_int, _c_float, _vp, _c_ll = ctypes.c_int, ctypes.c_float, ctypes.c_void_p, ctypes.c_longlong


class pn_stats(ctypes.Structure):
    _fields_ = [("iteration_launches", ctypes.c_longlong), ("iteration_ns", ctypes.c_longlong),
                ("evals", ctypes.c_longlong)]


SIGNATURES = {
    "pn_create": (_c_int, [ctypes.POINTER(_vp), _c_int, _c_int, _c_int, _c_int, _c_int, _vp,
                           ctypes.c_size_t, _c_float, _vp]),
    "pn_eval": (_c_int, [_vp, _vp, _vp, _c_int, _c_int, _c_float, _vp, ctypes.POINTER(_c_int),
                         ctypes.POINTER(_c_float)]),
    "pn_eval_host": (_c_int, [_vp, _vp, _vp, _c_int, _c_int, _c_float, _vp, ctypes.POINTER(_c_int),
                              ctypes.POINTER(_c_float)]),
    "pn_eval_host_many": (_c_int, [_vp, _c_int, _vp, _vp, _c_int, _c_int, _c_float, _vp, _vp, _vp]),
    "pn_eval_windowed": (_c_int, [_vp, _vp, _c_int, _vp, _vp, _c_int, _c_int, _c_float, _vp,
                                  ctypes.POINTER(_c_int), ctypes.POINTER(_c_float), _vp, _c_int]),
    "pn_get_residual_history": (_c_int, [_vp, _vp, _c_int, ctypes.POINTER(_c_int)]),
    "pn_time_iterations": (_c_int, [_vp, _c_int, _c_int, ctypes.POINTER(_c_float)]),
    "pn_get_stats": (_c_int, [_vp, ctypes.POINTER(pn_stats)]),
    "pn_reset_stats": (_c_int, [_vp]),
    "pn_set_option": (_c_int, [_vp, _c_int, _c_ll]),
    "pn_set_stream": (_c_int, [_vp, _vp]),
    "pn_set_damping": (_c_int, [_vp, _c_float]),
    "pn_set_adaptive": (_c_int, [_vp, _c_float]),
    "pn_set_storage": (_c_int, [_vp, _c_int, _c_float]),
    "pn_get_mode_history": (_c_int, [_vp, _vp, _c_int, ctypes.POINTER(_c_int)]),
    "pn_dim": (_c_int, [_vp, _c_int]),
    "pn_activation": (_c_int, [_c_int, _vp, _vp, _c_ll, _vp]),
    "pn_eval_static": (_c_int, [_vp, ctypes.c_size_t, _c_int, _c_int, _c_int, _c_int, _vp, _vp, _c_int, _c_int,
                                _c_float, _vp, ctypes.POINTER(_c_int), ctypes.POINTER(_c_float), _vp]),
    "pn_last_error": (ctypes.c_char_p, [_vp]),
    "pn_destroy": (None, [_vp]),
    "pn_version": (ctypes.c_char_p, []),
}


def _load() -> ctypes.CDLL:
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"{LIB_PATH} is missing: build it with "
                          "`python newton_evaluation_nonlinear_b200/build.py`")
    lib = ctypes.CDLL(LIB_PATH)
    for name, (res, args) in SIGNATURES.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    return lib


lib = _load()


class PnError(RuntimeError):
    def __init__(self, status: int, message: str):
        super().__init__(f"{STATUS_NAMES.get(status, status)}: {message}")
        self.status = status


# ----------------------------------------------------------------------------
# C-named functions (plain ints for pointers/streams)
# ----------------------------------------------------------------------------

def pn_version() -> str:
    return lib.pn_version().decode()


def pn_last_error(h: Optional[int]) -> str:
    return lib.pn_last_error(h).decode()


def pn_create(cell: int, D: int, d_in: int, T: int, B: int, params: np.ndarray, eps: float = 0.0,
              stream: int = 0) -> Tuple[int, Optional[int]]:
    p = np.ascontiguousarray(params, dtype=np.float32).ravel()
    h = _vp()
    st = lib.pn_create(ctypes.byref(h), int(cell), int(D), int(d_in), int(T), int(B),
                       p.ctypes.data, p.size, float(eps), stream or None)
    return st, h.value


def pn_eval(h: int, x_ptr: int, s0_ptr: int, mode: int, max_iters: int, tol: float,
            states_ptr: int) -> Tuple[int, int, float]:
    it, r = _c_int(-1), _c_float(float("nan"))
    st = lib.pn_eval(h, x_ptr, s0_ptr, int(mode), int(max_iters), float(tol), states_ptr,
                     ctypes.byref(it), ctypes.byref(r))
    return st, it.value, r.value


def pn_eval_host(h: int, x: np.ndarray, s0: np.ndarray, mode: int, max_iters: int, tol: float,
                 states: np.ndarray) -> Tuple[int, int, float]:
    for a in (x, s0, states):
        if a.dtype != np.float32 or not a.flags.c_contiguous:
            raise ValueError("host buffers must be C-contiguous float32")
    it, r = _c_int(-1), _c_float(float("nan"))
    st = lib.pn_eval_host(h, x.ctypes.data, s0.ctypes.data, int(mode), int(max_iters), float(tol),
                          states.ctypes.data, ctypes.byref(it), ctypes.byref(r))
    return st, it.value, r.value


def pn_eval_host_many(h: int, xs, s0s, mode: int, max_iters: int, tol: float, states_list):
    """Pipelined pn_eval_host over len(xs) batches; returns (status, iters[], resids[])."""
    n = len(xs)
    if len(s0s) != n or len(states_list) != n:
        raise ValueError("one x, s0 and states buffer per batch")
    for a in list(xs) + list(s0s) + list(states_list):
        if a.dtype != np.float32 or not a.flags.c_contiguous:
            raise ValueError("host buffers must be C-contiguous float32")
    px = (_vp * max(n, 1))(*[a.ctypes.data for a in xs])
    ps0 = (_vp * max(n, 1))(*[a.ctypes.data for a in s0s])
    pst = (_vp * max(n, 1))(*[a.ctypes.data for a in states_list])
    its = np.full(max(n, 1), -1, np.int32)
    rs = np.full(max(n, 1), np.nan, np.float32)
    st = lib.pn_eval_host_many(h, n, px, ps0, int(mode), int(max_iters), float(tol), pst, its.ctypes.data,
                               rs.ctypes.data)
    return st, its[:n], rs[:n]


def pn_eval_windowed(h: int, tail: Optional[int], T_total: int, x_ptr: int, s0_ptr: int, mode: int,
                     max_iters: int, tol: float, states_ptr: int, n_window_cap: int):
    """Returns (status, total iters, resid, per-window iters[:n_window_cap])."""
    it, r = _c_int(-1), _c_float(float("nan"))
    wit = np.full(max(int(n_window_cap), 1), -1, np.int32)
    st = lib.pn_eval_windowed(h, tail, int(T_total), x_ptr, s0_ptr, int(mode), int(max_iters), float(tol),
                              states_ptr, ctypes.byref(it), ctypes.byref(r), wit.ctypes.data, int(n_window_cap))
    return st, it.value, r.value, wit[:max(int(n_window_cap), 0)]


def pn_get_residual_history(h: int, n: int) -> Tuple[int, np.ndarray]:
    out = np.zeros(max(int(n), 1), np.float32)
    w = _c_int(0)
    st = lib.pn_get_residual_history(h, out.ctypes.data, int(n), ctypes.byref(w))
    return st, out[: w.value]


def pn_time_iterations(h: int, mode: int, n_launches: int) -> Tuple[int, float]:
    ms = _c_float(0.0)
    st = lib.pn_time_iterations(h, int(mode), int(n_launches), ctypes.byref(ms))
    return st, ms.value


def pn_get_stats(h: int) -> Tuple[int, dict]:
    s = pn_stats()
    st = lib.pn_get_stats(h, ctypes.byref(s))
    return st, {"iteration_launches": s.iteration_launches, "iteration_ns": s.iteration_ns,
                "evals": s.evals}


def pn_reset_stats(h: int) -> int:
    return lib.pn_reset_stats(h)


def pn_set_option(h: int, opt: int, value: int) -> int:
    return lib.pn_set_option(h, int(opt), int(value))


def pn_set_adaptive(h: int, stall: float) -> int:
    return lib.pn_set_adaptive(h, float(stall))


def pn_get_mode_history(h: int, n: int) -> Tuple[int, np.ndarray]:
    out = np.zeros(max(int(n), 1), np.int32)
    w = _c_int(0)
    st = lib.pn_get_mode_history(h, out.ctypes.data, int(n), ctypes.byref(w))
    return st, out[:w.value]


def pn_set_damping(h: int, damping: float) -> int:
    return lib.pn_set_damping(h, float(damping))


def pn_set_storage(h: int, fmt: int, store_until: float) -> int:
    return lib.pn_set_storage(h, int(fmt), float(store_until))


def pn_set_stream(h: int, stream: int) -> int:
    return lib.pn_set_stream(h, stream or None)


def pn_eval_static(params: np.ndarray, D: int, d_in: int, T: int, B: int, x_ptr: int, s0_ptr: int, mode: int,
                   max_iters: int, tol: float, states_ptr: int, stream: int = 0) -> Tuple[int, int, float]:
    p = np.ascontiguousarray(params, dtype=np.float32).ravel()
    it, r = _c_int(-1), _c_float(float("nan"))
    st = lib.pn_eval_static(p.ctypes.data, p.size, int(D), int(d_in), int(T), int(B), x_ptr, s0_ptr, int(mode),
                            int(max_iters), float(tol), states_ptr, ctypes.byref(it), ctypes.byref(r),
                            stream or None)
    return st, it.value, r.value


def pn_activation(which: int, x_ptr: int, y_ptr: int, n: int, stream: int = 0) -> int:
    return lib.pn_activation(int(which), x_ptr, y_ptr, int(n), stream or None)


def pn_dim(h: int, which: int) -> int:
    return lib.pn_dim(h, int(which))


def pn_destroy(h: Optional[int]) -> None:
    lib.pn_destroy(h)


# ----------------------------------------------------------------------------
# torch-facing wrapper
# ----------------------------------------------------------------------------

class Solver:
    """One libpn handle: a cell with fixed shape (D, d_in, T, B) and parameters.

    ``eval`` takes CUDA float32 tensors (x [B,T,d_in], s0 [B,D]) and returns
    ``(states, iters, resid, status)``; statuses PN_OK and PN_NOT_CONVERGED
    return normally, every error raises :class:`PnError`.
    """

    def __init__(self, cell: int, D: int, d_in: int, T: int, B: int, params, eps: float = 0.0,
                 stream=None, device=None):
        import torch
        self.cell, self.D, self.d_in, self.T, self.B = int(cell), int(D), int(d_in), int(T), int(B)
        self.device = torch.device(device if device is not None else "cuda")
        with torch.cuda.device(self.device):
            if stream is None:
                stream = torch.cuda.current_stream(self.device)
            self._stream = stream
            st, h = pn_create(cell, D, d_in, T, B, np.asarray(params), eps, int(stream.cuda_stream))
        if st != PN_OK:
            raise PnError(st, pn_last_error(None))
        self.h = h

    @classmethod
    def from_problem(cls, prob, stream=None, device=None) -> "Solver":
        return cls(prob.cell, prob.D, prob.d_in, prob.T, prob.B, prob.params, prob.eps, stream, device)

    def _check(self, st: int) -> int:
        if st < 0:
            raise PnError(st, pn_last_error(self.h))
        return st

    def eval(self, x, s0, mode, max_iters: Optional[int] = None, tol: float = 1e-5, states=None):
        import torch
        mode = MODES[mode] if isinstance(mode, str) else int(mode)
        max_iters = self.T if max_iters is None else int(max_iters)
        if states is None:
            states = torch.empty((self.B, self.T, self.D), device=x.device, dtype=torch.float32)
        for name, t, shape in (("x", x, (self.B, self.T, self.d_in)), ("s0", s0, (self.B, self.D)),
                               ("states", states, (self.B, self.T, self.D))):
            if t.dtype != torch.float32 or not t.is_cuda or not t.is_contiguous() or tuple(t.shape) != shape:
                raise ValueError(f"{name} must be a contiguous CUDA float32 tensor of shape {shape}")
        st, it, r = pn_eval(self.h, x.data_ptr(), s0.data_ptr(), mode, max_iters, tol, states.data_ptr())
        self._check(st)
        return states, it, r, st

    def eval_host(self, x: np.ndarray, s0: np.ndarray, mode, max_iters: Optional[int] = None,
                  tol: float = 1e-5, states: Optional[np.ndarray] = None):
        mode = MODES[mode] if isinstance(mode, str) else int(mode)
        max_iters = self.T if max_iters is None else int(max_iters)
        if states is None:
            states = np.empty((self.B, self.T, self.D), np.float32)
        st, it, r = pn_eval_host(self.h, x, s0, mode, max_iters, tol, states)
        self._check(st)
        return states, it, r, st

    def eval_host_many(self, xs, s0s, mode, max_iters: Optional[int] = None, tol: float = 1e-5,
                       states_list=None):
        """Evaluate several batches from host buffers, overlapping each batch's copies with the
        neighbouring batches' evaluations.  Returns (states_list, iters, resids, status)."""
        mode = MODES[mode] if isinstance(mode, str) else int(mode)
        max_iters = self.T if max_iters is None else int(max_iters)
        if states_list is None:
            states_list = [np.empty((self.B, self.T, self.D), np.float32) for _ in xs]
        st, its, rs = pn_eval_host_many(self.h, xs, s0s, mode, max_iters, tol, states_list)
        self._check(st)
        return states_list, its, rs, st

    def eval_windowed(self, x, s0, mode, max_iters: Optional[int] = None, tol: float = 1e-5,
                      tail: Optional["Solver"] = None, states=None):
        """Solve a sequence of T_total = x.shape[1] steps window by window, this solver's T being
        the window length; ``tail`` is a Solver for the last T_total % T steps (same cell, shapes,
        parameters and stream).  Returns (states, iters, resid, status, window_iters)."""
        import torch
        mode = MODES[mode] if isinstance(mode, str) else int(mode)
        max_iters = self.T if max_iters is None else int(max_iters)
        T_total = int(x.shape[1]) if x.dim() == 3 else -1
        if states is None:
            states = torch.empty((self.B, max(T_total, 0), self.D), device=x.device, dtype=torch.float32)
        for name, t, shape in (("x", x, (self.B, T_total, self.d_in)), ("s0", s0, (self.B, self.D)),
                               ("states", states, (self.B, T_total, self.D))):
            if t.dtype != torch.float32 or not t.is_cuda or not t.is_contiguous() or tuple(t.shape) != shape:
                raise ValueError(f"{name} must be a contiguous CUDA float32 tensor of shape {shape}")
        nwin = -(-T_total // self.T)
        st, it, r, wit = pn_eval_windowed(self.h, tail.h if tail is not None else None, T_total, x.data_ptr(),
                                          s0.data_ptr(), mode, max_iters, tol, states.data_ptr(), nwin)
        self._check(st)
        return states, it, r, st, wit

    def residual_history(self, n: int = 1 << 16) -> np.ndarray:
        st, h = pn_get_residual_history(self.h, n)
        self._check(st)
        return h

    def time_iterations(self, mode, n_launches: int) -> float:
        mode = MODES[mode] if isinstance(mode, str) else int(mode)
        st, ms = pn_time_iterations(self.h, mode, n_launches)
        self._check(st)
        return ms

    def stats(self) -> dict:
        st, s = pn_get_stats(self.h)
        self._check(st)
        return s

    def reset_stats(self) -> None:
        self._check(pn_reset_stats(self.h))

    def set_option(self, opt: int, value: int) -> None:
        self._check(pn_set_option(self.h, opt, value))

    def set_damping(self, damping: float) -> None:
        self._check(pn_set_damping(self.h, damping))

    def set_adaptive(self, stall: float) -> None:
        self._check(pn_set_adaptive(self.h, stall))

    def set_storage(self, fmt: int, store_until: float = 0.0) -> None:
        """Iterate storage: PN_STORE_F32, or a 16-bit format (PN_STORE_BF16 / PN_STORE_F16) while the
        residual known at an update's start is above store_until."""
        self._check(pn_set_storage(self.h, fmt, store_until))

    def mode_history(self, n: int = 1 << 16) -> np.ndarray:
        st, m = pn_get_mode_history(self.h, n)
        self._check(st)
        return m

    def close(self) -> None:
        if getattr(self, "h", None):
            pn_destroy(self.h)
            self.h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass
