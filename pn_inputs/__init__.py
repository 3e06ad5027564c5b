"""Seeded synthetic inputs for parallel Newton evaluation of nonlinear sequences.

This module draws random numbers and nothing else: it holds none of the
method's arithmetic (no cell, no Jacobian, no scan).  It is the one module that
both the fp64 oracle tests and the CUDA path's tests and benchmark use, so the
two sides see bit-identical fp32 inputs.

Workloads.  The five benchmark workloads are synthetic by construction: a tanh
RNN ``s_t = tanh(W s_{t-1} + U x_t + b)``, a GRU cell, and an Euler-discretised
drift ``s_t = s_{t-1} + eps * tanh(W s_{t-1} + c_t)``, with the shapes and value
distributions below.  Where a distribution or seed is not fixed by the workload
description the choice made here is written next to it.

* ``N(0, v)`` means variance ``v``.
* Seeds: workload 0 uses ``numpy.random.default_rng(0)``; workloads 1..4 use the
  child streams ``numpy.random.SeedSequence(0).spawn(5)[k]``.
* Draw order within a workload: recurrent weights, input weights, biases,
  inputs ``x``, then ``s0`` (always zero here, so nothing is drawn for it).
* Spectral-radius rescale: ``W <- W * rho / max|eig(W)|`` in float64, then the
  cast to float32.  Both sides read the same float32 arrays.

Parameter packing (row-major float32, one flat vector):
  tanh RNN : W[D,D], U[D,d_in], b[D]
  GRU      : W_ih[3D,d_in], W_hh[3D,D], b_ih[3D], b_hh[3D]   (gates r, z, n)
  Euler    : W[D,D]   (d_in == D, x holds c_t)
"""
from __future__ import annotations

import dataclasses
import hashlib
from typing import Dict, List, Optional

import numpy as np

CELL_TANH_RNN = 0
CELL_GRU = 1
CELL_EULER = 2
CELL_NAMES = {CELL_TANH_RNN: "tanh_rnn", CELL_GRU: "gru", CELL_EULER: "euler"}

MODE_JACOBI = 0
MODE_PICARD = 1
MODE_QUASI = 2
MODE_NEWTON = 3
MODE_NAMES = {MODE_JACOBI: "jacobi", MODE_PICARD: "picard", MODE_QUASI: "quasi",
              MODE_NEWTON: "newton"}
MODE_BY_NAME = {v: k for k, v in MODE_NAMES.items()}


@dataclasses.dataclass
class Problem:
    """One synthetic problem: model parameters, inputs and solver settings."""

    name: str
    cell: int
    D: int
    d_in: int
    T: int
    B: int
    params: np.ndarray          # float32, flat, packed as in the module docstring
    x: np.ndarray               # float32 [B, T, d_in]
    s0: np.ndarray              # float32 [B, D]
    eps: float = 0.0            # Euler step (0 for the other cells)
    modes: tuple = ()           # modes the workload is run with
    tol: float = 1e-5
    max_iters: Optional[int] = None   # None means T (at most T iterations by causality)

    @property
    def iters_cap(self) -> int:
        return self.T if self.max_iters is None else int(self.max_iters)

    def fingerprint(self) -> str:
        """sha256 over the float32 bytes of params, x and s0 (detects generator drift)."""
        h = hashlib.sha256()
        for a in (self.params, self.x, self.s0):
            h.update(np.ascontiguousarray(a, dtype=np.float32).tobytes())
        h.update(np.float64(self.eps).tobytes())
        return h.hexdigest()


def param_count(cell: int, D: int, d_in: int) -> int:
    if cell == CELL_TANH_RNN:
        return D * D + D * d_in + D
    if cell == CELL_GRU:
        return 3 * D * d_in + 3 * D * D + 6 * D
    if cell == CELL_EULER:
        if d_in != D:
            raise ValueError("Euler cell needs d_in == D")
        return D * D
    raise ValueError(f"unknown cell {cell}")


def _rescale(W: np.ndarray, rho: float) -> np.ndarray:
    """Scale a square float64 matrix to spectral radius ``rho``."""
    lam = float(np.max(np.abs(np.linalg.eigvals(W))))
    return W * (rho / lam)


def _rng_for(index: int) -> np.random.Generator:
    if index == 0:
        return np.random.default_rng(0)
    return np.random.default_rng(np.random.SeedSequence(0).spawn(5)[index])


def benchmark_workload(index: int, T: Optional[int] = None, B: Optional[int] = None) -> Problem:
    """The five benchmark workloads (index 0..4).

    ``T``/``B`` may shrink a workload for a quick run: the parameters are drawn
    exactly as for the full size, and the inputs are the leading ``B`` sequences
    and ``T`` steps of the full draw (so a shrunk problem is a prefix of the full
    one).
    """
    rng = _rng_for(index)
    if index == 0:
        D = d_in = 4
        TT, BB = 1024, 1
        W = _rescale(rng.normal(0.0, 1.0, (D, D)), 0.5)
        U = rng.normal(0.0, np.sqrt(1.0 / 4.0), (D, d_in))
        b = np.zeros(D)
        x = rng.normal(0.0, 1.0, (BB, TT, d_in))
        p = np.concatenate([W.ravel(), U.ravel(), b])
        prob = Problem("tanh_rnn_D4_T1024_B1_newton", CELL_TANH_RNN, D, d_in, TT, BB,
                       p.astype(np.float32), x.astype(np.float32), np.zeros((BB, D), np.float32),
                       modes=(MODE_NEWTON,), tol=1e-6)
    elif index == 1:
        D = d_in = 64
        TT, BB = 16384, 16
        W = _rescale(rng.normal(0.0, np.sqrt(1.0 / 64), (D, D)), 0.7)
        U = rng.normal(0.0, np.sqrt(1.0 / 64), (D, d_in))      # unstated: N(0, 1/d_in)
        b = np.zeros(D)                                         # unstated: zero
        x = rng.normal(0.0, 1.0, (BB, TT, d_in))
        p = np.concatenate([W.ravel(), U.ravel(), b])
        prob = Problem("tanh_rnn_D64_T16384_B16_quasi", CELL_TANH_RNN, D, d_in, TT, BB,
                       p.astype(np.float32), x.astype(np.float32), np.zeros((BB, D), np.float32),
                       modes=(MODE_QUASI,), tol=1e-5)
    elif index == 2:
        D = d_in = 16                                           # unstated: d_in = D
        TT, BB = 8192, 64
        W = _rescale(rng.normal(0.0, np.sqrt(1.0 / 16), (D, D)), 0.6)
        U = rng.normal(0.0, np.sqrt(1.0 / 16), (D, d_in))
        b = np.zeros(D)
        x = rng.normal(0.0, 1.0, (BB, TT, d_in))
        p = np.concatenate([W.ravel(), U.ravel(), b])
        prob = Problem("tanh_rnn_D16_T8192_B64_newton", CELL_TANH_RNN, D, d_in, TT, BB,
                       p.astype(np.float32), x.astype(np.float32), np.zeros((BB, D), np.float32),
                       modes=(MODE_NEWTON,), tol=1e-5)
    elif index == 3:
        D = d_in = 32
        TT, BB = 65536, 8
        a = 1.0 / np.sqrt(32.0)
        W_ih = rng.uniform(-a, a, (3 * D, d_in))
        W_hh = rng.uniform(-a, a, (3 * D, D))
        # each of the three recurrent gate blocks (r, z, n) to spectral radius 0.95
        W_hh = np.concatenate([_rescale(W_hh[g * D:(g + 1) * D], 0.95) for g in range(3)])
        b_ih = rng.uniform(-a, a, 3 * D)
        b_hh = rng.uniform(-a, a, 3 * D)
        x = rng.normal(0.0, 1.0, (BB, TT, d_in))
        p = np.concatenate([W_ih.ravel(), W_hh.ravel(), b_ih, b_hh])
        prob = Problem("gru_D32_T65536_B8_quasi", CELL_GRU, D, d_in, TT, BB,
                       p.astype(np.float32), x.astype(np.float32), np.zeros((BB, D), np.float32),
                       modes=(MODE_QUASI,), tol=1e-5, max_iters=256)
    elif index == 4:
        D = d_in = 256
        TT, BB = 1024, 32
        W = rng.normal(0.0, np.sqrt(1.0 / 256), (D, D))
        c = rng.normal(0.0, 1.0, (BB, TT, D))                   # c_t drawn per (b, t)
        prob = Problem("euler_D256_T1024_B32_picard_jacobi", CELL_EULER, D, D, TT, BB,
                       W.ravel().astype(np.float32), c.astype(np.float32),
                       np.zeros((BB, D), np.float32), eps=1e-2,
                       modes=(MODE_PICARD, MODE_JACOBI, MODE_QUASI), tol=1e-5)
    else:
        raise ValueError("workload index must be 0..4")
    if T is not None or B is not None:
        TT = prob.T if T is None else min(int(T), prob.T)
        BB = prob.B if B is None else min(int(B), prob.B)
        prob = dataclasses.replace(prob, T=TT, B=BB,
                                   x=np.ascontiguousarray(prob.x[:BB, :TT]),
                                   s0=np.ascontiguousarray(prob.s0[:BB]),
                                   max_iters=(prob.max_iters if prob.max_iters is not None else None),
                                   name=f"{prob.name}[T={TT},B={BB}]")
    return prob


def random_problem(seed: int, cell: int, D: int, d_in: Optional[int] = None, T: int = 16,
                   B: int = 2, rho: float = 0.5, eps: float = 0.05, s0_scale: float = 0.0,
                   x_scale: float = 1.0, tol: float = 1e-6, max_iters: Optional[int] = None,
                   bias_scale: float = 0.1) -> Problem:
    """A small random problem for tests: odd shapes, non-zero s0 and biases allowed."""
    rng = np.random.default_rng(seed)
    if cell == CELL_EULER:
        d_in = D
    d_in = D if d_in is None else d_in
    if cell == CELL_TANH_RNN:
        W = rng.normal(0.0, 1.0, (D, D))
        W = _rescale(W, rho) if rho > 0 else np.zeros((D, D))
        U = rng.normal(0.0, np.sqrt(1.0 / d_in), (D, d_in))
        b = rng.normal(0.0, bias_scale, D)
        p = np.concatenate([W.ravel(), U.ravel(), b])
    elif cell == CELL_GRU:
        a = 1.0 / np.sqrt(D)
        W_ih = rng.uniform(-a, a, (3 * D, d_in))
        W_hh = rng.uniform(-a, a, (3 * D, D))
        if rho > 0:
            W_hh = np.concatenate([_rescale(W_hh[g * D:(g + 1) * D], rho) for g in range(3)])
        b_ih = rng.uniform(-a, a, 3 * D)
        b_hh = rng.uniform(-a, a, 3 * D)
        p = np.concatenate([W_ih.ravel(), W_hh.ravel(), b_ih, b_hh])
    elif cell == CELL_EULER:
        W = rng.normal(0.0, np.sqrt(1.0 / D), (D, D))
        p = W.ravel()
    else:
        raise ValueError("unknown cell")
    x = rng.normal(0.0, x_scale, (B, T, d_in))
    s0 = rng.normal(0.0, s0_scale, (B, D)) if s0_scale > 0 else np.zeros((B, D))
    return Problem(f"random_{CELL_NAMES[cell]}_D{D}_T{T}_B{B}_seed{seed}", cell, D, d_in, T, B,
                   p.astype(np.float32), x.astype(np.float32), s0.astype(np.float32),
                   eps=(eps if cell == CELL_EULER else 0.0), tol=tol, max_iters=max_iters)


WORKLOAD_MODES = {0: (MODE_NEWTON,), 1: (MODE_QUASI,), 2: (MODE_NEWTON,), 3: (MODE_QUASI,),
                  4: (MODE_PICARD, MODE_JACOBI, MODE_QUASI)}


def workload_names() -> List[str]:
    return ["tanh_rnn_D4_T1024_B1_newton", "tanh_rnn_D64_T16384_B16_quasi",
            "tanh_rnn_D16_T8192_B64_newton", "gru_D32_T65536_B8_quasi",
            "euler_D256_T1024_B32_picard_jacobi"]


def describe(prob: Problem) -> Dict[str, object]:
    return {"workload": prob.name, "cell": CELL_NAMES[prob.cell], "D": prob.D, "d_in": prob.d_in,
            "T": prob.T, "B": prob.B, "eps": prob.eps, "tol": prob.tol,
            "max_iters": prob.iters_cap, "modes": [MODE_NAMES[m] for m in prob.modes]}
