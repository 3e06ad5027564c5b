"""ctypes front-end of the fp64 CPU oracle (``oracle.c``).

TEST INFRASTRUCTURE ONLY: the tests, the smoke check and the benchmark's
CPU-baseline leg may import this package; the product path (the CUDA library and
its Python binding) never does.  The oracle shares no code with the CUDA path.

Citations "page §X" refer to the web article "并行牛顿方法：加速非线性序列评估的
计算革命" (Parallel Newton methods for nonlinear sequence evaluation, jsqmd.com
news item 789890), section X.  See ``oracle.h`` for the readings taken where the
page is silent.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "oracle.c")
_HDR = os.path.join(_HERE, "oracle.h")
_LIB = os.path.join(_HERE, "liboracle.so")
_lock = threading.Lock()
_lib = None

JACOBI, PICARD, QUASI, NEWTON, BANDED = 0, 1, 2, 3, 4
STORE_F64, STORE_F32, STORE_BF16, STORE_F16 = 0, 1, 2, 3
OK, NOT_CONVERGED, ERR_INVALID, ERR_NOMEM, ERR_NONFINITE = 0, 1, -1, -2, -4


def build(force: bool = False) -> str:
    """Compile ``liboracle.so`` with gcc (plain -O2, no fast-math, no FMA contraction)."""
    newest = max(os.path.getmtime(_SRC), os.path.getmtime(_HDR))
    if not force and os.path.exists(_LIB) and os.path.getmtime(_LIB) >= newest:
        return _LIB
    tmp = _LIB + f".tmp{os.getpid()}"
    cmd = ["gcc", "-O2", "-std=c11", "-ffp-contract=off", "-fPIC", "-shared", "-Wall", "-Wextra",
           "-o", tmp, _SRC, "-lpthread", "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    with _lock:
        if _lib is None:
            lib = ctypes.CDLL(build())
            dp = ctypes.POINTER(ctypes.c_double)
            ip = ctypes.POINTER(ctypes.c_int)
            i, d = ctypes.c_int, ctypes.c_double
            lib.orc_param_count.argtypes = [i, i, i]
            lib.orc_param_count.restype = ctypes.c_long
            lib.orc_cell.argtypes = [i, i, i, dp, d, dp, dp, dp]
            lib.orc_jacobian.argtypes = [i, i, i, dp, d, dp, dp, dp]
            lib.orc_approx_jacobian.argtypes = [i, i, i, i, dp, d, dp, dp, dp]
            lib.orc_sequential.argtypes = [i, i, i, dp, d, i, i, dp, dp, dp, i]
            lib.orc_residual.argtypes = [i, i, i, dp, d, i, i, dp, dp, dp, dp, dp, i]
            lib.orc_update.argtypes = [i, i, i, i, dp, d, i, i, dp, dp, dp, dp, i]
            lib.orc_iterate.argtypes = [i, i, i, i, dp, d, i, i, dp, dp, i, d, dp, ip, dp, dp, i, i]
            lib.orc_affine_recurrence.argtypes = [i, i, dp, dp, dp, dp]
            lib.orc_banded_jacobian.argtypes = [i, i, i, i, dp, d, dp, dp, dp]
            lib.orc_round_storage.argtypes = [i, dp, ctypes.c_long]
            lib.orc_update_ex.argtypes = [i, i, i, d, i, i, dp, d, i, i, dp, dp, dp, dp, i]
            lib.orc_iterate_ex.argtypes = [i, i, i, d, i, d, i, d, i, i, i, dp, d, i, i, dp, dp, i, d,
                                           dp, ip, dp, dp, ip, i, ip, i]
            for fn in ("orc_cell", "orc_jacobian", "orc_approx_jacobian", "orc_sequential",
                       "orc_residual", "orc_update", "orc_iterate", "orc_affine_recurrence",
                       "orc_banded_jacobian", "orc_round_storage", "orc_update_ex", "orc_iterate_ex"):
                getattr(lib, fn).restype = ctypes.c_int
            _lib = lib
    return _lib


def _f64(a) -> np.ndarray:
    return np.ascontiguousarray(np.asarray(a, dtype=np.float64))


def _ptr(a: np.ndarray):
    return a.ctypes.data_as(ctypes.POINTER(ctypes.c_double))


def _check(rc: int, what: str) -> int:
    if rc < 0:
        raise RuntimeError(f"oracle {what} failed with status {rc}")
    return rc


def default_threads(B: int) -> int:
    return max(1, min(int(B), os.cpu_count() or 1))


class Model:
    """A cell with its packed parameters held in float64 (exact copies of the float32 inputs)."""

    def __init__(self, cell: int, D: int, d_in: int, params, eps: float = 0.0):
        self.cell, self.D, self.d_in, self.eps = int(cell), int(D), int(d_in), float(eps)
        self.p = _f64(params).ravel()
        n = _load().orc_param_count(self.cell, self.D, self.d_in)
        if n < 0 or n != self.p.size:
            raise ValueError(f"parameter vector has {self.p.size} entries, cell needs {n}")

    @classmethod
    def from_problem(cls, prob) -> "Model":
        return cls(prob.cell, prob.D, prob.d_in, prob.params, prob.eps)

    # --- one step ---------------------------------------------------------
    def cell_step(self, x_t, s_prev) -> np.ndarray:
        x_t, s_prev = _f64(x_t), _f64(s_prev)
        y = np.empty(self.D)
        _check(_load().orc_cell(self.cell, self.D, self.d_in, _ptr(self.p), self.eps,
                                _ptr(x_t), _ptr(s_prev), _ptr(y)), "cell")
        return y

    def jacobian(self, x_t, s_prev) -> np.ndarray:
        x_t, s_prev = _f64(x_t), _f64(s_prev)
        J = np.empty((self.D, self.D))
        _check(_load().orc_jacobian(self.cell, self.D, self.d_in, _ptr(self.p), self.eps,
                                    _ptr(x_t), _ptr(s_prev), _ptr(J)), "jacobian")
        return J

    def approx_jacobian(self, mode: int, x_t, s_prev) -> np.ndarray:
        x_t, s_prev = _f64(x_t), _f64(s_prev)
        A = np.empty((self.D, self.D))
        _check(_load().orc_approx_jacobian(self.cell, int(mode), self.D, self.d_in, _ptr(self.p),
                                           self.eps, _ptr(x_t), _ptr(s_prev), _ptr(A)),
               "approx_jacobian")
        return A

    # --- whole sequences --------------------------------------------------
    def _shapes(self, x, s0):
        x, s0 = _f64(x), _f64(s0)
        B, T, d_in = x.shape
        if d_in != self.d_in or s0.shape != (B, self.D):
            raise ValueError("shape mismatch")
        return x, s0, B, T

    def sequential(self, x, s0, nthreads: int = 0) -> np.ndarray:
        x, s0, B, T = self._shapes(x, s0)
        s = np.empty((B, T, self.D))
        _check(_load().orc_sequential(self.cell, self.D, self.d_in, _ptr(self.p), self.eps, T, B,
                                      _ptr(x), _ptr(s0), _ptr(s), nthreads or default_threads(B)),
               "sequential")
        return s

    def residual(self, x, s0, s, nthreads: int = 0):
        x, s0, B, T = self._shapes(x, s0)
        s = _f64(s)
        F = np.empty((B, T, self.D))
        r = ctypes.c_double(0.0)
        _check(_load().orc_residual(self.cell, self.D, self.d_in, _ptr(self.p), self.eps, T, B,
                                    _ptr(x), _ptr(s0), _ptr(s), _ptr(F), ctypes.byref(r),
                                    nthreads or default_threads(B)), "residual")
        return F, r.value

    def update(self, mode: int, x, s0, s_cur, nthreads: int = 0) -> np.ndarray:
        x, s0, B, T = self._shapes(x, s0)
        s_cur = _f64(s_cur)
        s_next = np.empty((B, T, self.D))
        _check(_load().orc_update(self.cell, int(mode), self.D, self.d_in, _ptr(self.p), self.eps,
                                  T, B, _ptr(x), _ptr(s0), _ptr(s_cur), _ptr(s_next),
                                  nthreads or default_threads(B)), "update")
        return s_next

    def iterate(self, mode: int, x, s0, max_iters: int, tol: float, nthreads: int = 0,
                hist_cap: int = None):
        """Returns (states, iters, resid, status, history[:iters+1])."""
        x, s0, B, T = self._shapes(x, s0)
        s = np.empty((B, T, self.D))
        cap = (max_iters + 1) if hist_cap is None else int(hist_cap)
        hist = np.zeros(max(cap, 1))
        it = ctypes.c_int(0)
        r = ctypes.c_double(0.0)
        st = _load().orc_iterate(self.cell, int(mode), self.D, self.d_in, _ptr(self.p),
                                 self.eps, T, B, _ptr(x), _ptr(s0), int(max_iters),
                                 float(tol), _ptr(s), ctypes.byref(it), ctypes.byref(r),
                                 _ptr(hist), cap, nthreads or default_threads(B))
        if st in (ERR_INVALID, ERR_NOMEM):
            _check(st, "iterate")
        return s, it.value, r.value, st, hist[: min(it.value + 1, cap)].copy()


    # --- the page's refinements: banded Jacobian, damping, adaptive switching,
    # --- reduced-precision iterate storage, windowed solve (readings in oracle.h)
    def banded_jacobian(self, band: int, x_t, s_prev) -> np.ndarray:
        x_t, s_prev = _f64(x_t), _f64(s_prev)
        A = np.empty((self.D, self.D))
        _check(_load().orc_banded_jacobian(self.cell, int(band), self.D, self.d_in, _ptr(self.p),
                                           self.eps, _ptr(x_t), _ptr(s_prev), _ptr(A)),
               "banded_jacobian")
        return A

    def update_ex(self, mode: int, x, s0, s_cur, band: int = 0, damping: float = 1.0,
                  nthreads: int = 0) -> np.ndarray:
        x, s0, B, T = self._shapes(x, s0)
        s_cur = _f64(s_cur)
        s_next = np.empty((B, T, self.D))
        _check(_load().orc_update_ex(self.cell, int(mode), int(band), float(damping), self.D,
                                     self.d_in, _ptr(self.p), self.eps, T, B, _ptr(x), _ptr(s0),
                                     _ptr(s_cur), _ptr(s_next), nthreads or default_threads(B)),
               "update_ex")
        return s_next

    def iterate_ex(self, mode: int, x, s0, max_iters: int, tol: float, band: int = 0,
                   damping: float = 1.0, adapt: bool = False, stall: float = 0.9,
                   store: int = STORE_F64, store_until: float = 0.0, window: int = 0,
                   nthreads: int = 0, hist_cap: int = None):
        """Returns (states, iters, resid, status, history, modes, window_iters).

        history / modes: each measured residual and the mode of the update that
        followed it (-1 after a window's last residual), window after window."""
        x, s0, B, T = self._shapes(x, s0)
        Wn = T if (window <= 0 or window >= T) else int(window)
        nwin = 0 if T == 0 else (T + Wn - 1) // Wn
        s = np.empty((B, T, self.D))
        cap = nwin * (max_iters + 1) if hist_cap is None else int(hist_cap)
        hist = np.zeros(max(cap, 1))
        modes = np.full(max(cap, 1), -2, dtype=np.intc)
        wit = np.zeros(max(nwin, 1), dtype=np.intc)
        ip = ctypes.POINTER(ctypes.c_int)
        it = ctypes.c_int(0)
        r = ctypes.c_double(0.0)
        st = _load().orc_iterate_ex(self.cell, int(mode), int(band), float(damping), int(bool(adapt)),
                                    float(stall), int(store), float(store_until), int(window),
                                    self.D, self.d_in, _ptr(self.p), self.eps, T, B, _ptr(x),
                                    _ptr(s0), int(max_iters), float(tol), _ptr(s),
                                    ctypes.byref(it), ctypes.byref(r), _ptr(hist),
                                    modes.ctypes.data_as(ip), cap, wit.ctypes.data_as(ip),
                                    nthreads or default_threads(B))
        if st in (ERR_INVALID, ERR_NOMEM):
            _check(st, "iterate_ex")
        used = min(int(np.sum(wit[:nwin])) + nwin, cap)
        return s, it.value, r.value, st, hist[:used].copy(), modes[:used].copy(), wit[:nwin].copy()


def round_storage(values, store: int) -> np.ndarray:
    """Values rounded to a storage format (STORE_*), returned as float64."""
    v = _f64(values).copy()
    _check(_load().orc_round_storage(int(store), _ptr(v), v.size), "round_storage")
    return v


def affine_recurrence(A, b, s_init) -> np.ndarray:
    """Serial s_t = A_t s_{t-1} + b_t, t = 0..T-1 (A: [T,D,D], b: [T,D])."""
    A, b, s_init = _f64(A), _f64(b), _f64(s_init)
    T, D = b.shape
    s = np.empty((T, D))
    _check(_load().orc_affine_recurrence(D, T, _ptr(A), _ptr(b), _ptr(s_init), _ptr(s)),
           "affine_recurrence")
    return s
