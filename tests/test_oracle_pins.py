"""Pins of the fp64 oracle against things other than itself.

Each test ties one part of the oracle to an independent source: PyTorch's own
cell implementations and autograd (library routines the oracle does not use),
central finite differences, a dense LU solve of the block-bidiagonal system
J~ delta = -F, the causality theorem, closed forms, decimal-arithmetic hand
computation, and a tree-shaped evaluation of the scan combine.

Citations "page §X" refer to the web article "并行牛顿方法：加速非线性序列评估
的计算革命" (Parallel Newton methods for nonlinear sequence evaluation,
jsqmd.com news item 789890), section X.
"""
import decimal
import math

import numpy as np
import pytest
import torch

import oracle
import pn_inputs as pi

CELLS = [pi.CELL_TANH_RNN, pi.CELL_GRU, pi.CELL_EULER]
MODES = [pi.MODE_JACOBI, pi.MODE_PICARD, pi.MODE_QUASI, pi.MODE_NEWTON]


# ----------------------------------------------------------------------------
# independent cell implementations: torch.nn cells in float64
# ----------------------------------------------------------------------------

def torch_cell(prob):
    """Return (fn(x_t, s) -> y) built from torch.nn.RNNCell / GRUCell, float64."""
    D, d_in, p = prob.D, prob.d_in, np.asarray(prob.params, np.float64)
    if prob.cell == pi.CELL_TANH_RNN:
        c = torch.nn.RNNCell(d_in, D, nonlinearity="tanh", dtype=torch.float64)
        W = p[: D * D].reshape(D, D)
        U = p[D * D: D * D + D * d_in].reshape(D, d_in)
        b = p[D * D + D * d_in:]
        with torch.no_grad():
            c.weight_hh.copy_(torch.from_numpy(W)); c.weight_ih.copy_(torch.from_numpy(U))
            c.bias_ih.copy_(torch.from_numpy(b)); c.bias_hh.zero_()
        return lambda x, s: c(x[None], s[None])[0]
    if prob.cell == pi.CELL_GRU:
        c = torch.nn.GRUCell(d_in, D, dtype=torch.float64)
        o = 0
        W_ih = p[o:o + 3 * D * d_in].reshape(3 * D, d_in); o += 3 * D * d_in
        W_hh = p[o:o + 3 * D * D].reshape(3 * D, D); o += 3 * D * D
        b_ih = p[o:o + 3 * D]; o += 3 * D
        b_hh = p[o:o + 3 * D]
        with torch.no_grad():
            c.weight_ih.copy_(torch.from_numpy(W_ih)); c.weight_hh.copy_(torch.from_numpy(W_hh))
            c.bias_ih.copy_(torch.from_numpy(b_ih)); c.bias_hh.copy_(torch.from_numpy(b_hh))
        return lambda x, s: c(x[None], s[None])[0]
    # Euler: s + eps * g with g = tanh(W s + c) = an RNNCell with identity input weights
    c = torch.nn.RNNCell(D, D, nonlinearity="tanh", dtype=torch.float64)
    with torch.no_grad():
        c.weight_hh.copy_(torch.from_numpy(p.reshape(D, D)))
        c.weight_ih.copy_(torch.eye(D, dtype=torch.float64))
        c.bias_ih.zero_(); c.bias_hh.zero_()
    eps = prob.eps
    return lambda x, s: s + eps * c(x[None], s[None])[0]


@pytest.mark.parametrize("cell", CELLS)
@pytest.mark.parametrize("D,d_in", [(1, 1), (3, 5), (8, 8)])
def test_cell_matches_torch(cell, D, d_in):
    prob = pi.random_problem(11 + D, cell, D, d_in, T=3, B=1, rho=0.9, s0_scale=0.7)
    m = oracle.Model.from_problem(prob)
    f = torch_cell(prob)
    rng = np.random.default_rng(5)
    for _ in range(4):
        x = rng.normal(size=prob.d_in)
        s = rng.normal(size=D)
        y_ref = f(torch.from_numpy(x), torch.from_numpy(s)).detach().numpy()
        np.testing.assert_allclose(m.cell_step(x, s), y_ref, rtol=0, atol=1e-14)


def test_sequential_matches_torch_loop():
    prob = pi.random_problem(3, pi.CELL_GRU, 6, 4, T=40, B=3, s0_scale=0.5)
    m = oracle.Model.from_problem(prob)
    f = torch_cell(prob)
    s_ref = np.empty((prob.B, prob.T, prob.D))
    for b in range(prob.B):
        h = torch.from_numpy(prob.s0[b].astype(np.float64))
        for t in range(prob.T):
            h = f(torch.from_numpy(prob.x[b, t].astype(np.float64)), h)
            s_ref[b, t] = h.detach().numpy()
    np.testing.assert_allclose(m.sequential(prob.x, prob.s0), s_ref, rtol=0, atol=1e-13)


def _decimal_tanh(v: decimal.Decimal) -> decimal.Decimal:
    e2 = (2 * v).exp()
    return (e2 - 1) / (e2 + 1)


def test_scalar_tanh_recurrence_by_hand():
    """D = 1: s_t = tanh(w s_{t-1} + u x_t + b), evaluated in 40-digit decimal arithmetic."""
    w, u, b = 0.5, 1.0, 0.0
    xs = [1.0, -0.5, 0.25, 2.0, -3.0]
    params = np.array([w, u, b], np.float32)
    m = oracle.Model(pi.CELL_TANH_RNN, 1, 1, params)
    decimal.getcontext().prec = 40
    s = decimal.Decimal(0)
    expect = []
    for xv in xs:
        s = _decimal_tanh(decimal.Decimal(w) * s + decimal.Decimal(u) * decimal.Decimal(xv) + decimal.Decimal(b))
        expect.append(float(s))
    got = m.sequential(np.array(xs, np.float64).reshape(1, -1, 1), np.zeros((1, 1)))
    np.testing.assert_allclose(got.ravel(), expect, rtol=0, atol=2e-16)
    assert abs(expect[0] - 0.7615941559557649) < 1e-16  # tanh(1)


# ----------------------------------------------------------------------------
# Jacobians
# ----------------------------------------------------------------------------

@pytest.mark.parametrize("cell", CELLS)
def test_jacobian_central_differences(cell):
    prob = pi.random_problem(21, cell, 5, 4, T=2, B=1, rho=0.9)
    m = oracle.Model.from_problem(prob)
    rng = np.random.default_rng(1)
    x, s = rng.normal(size=prob.d_in), rng.normal(size=prob.D)
    J = m.jacobian(x, s)
    h = 1e-6
    J_fd = np.empty_like(J)
    for k in range(prob.D):
        e = np.zeros(prob.D); e[k] = h
        J_fd[:, k] = (m.cell_step(x, s + e) - m.cell_step(x, s - e)) / (2 * h)
    np.testing.assert_allclose(J, J_fd, rtol=0, atol=1e-8)


@pytest.mark.parametrize("cell", CELLS)
def test_jacobian_matches_torch_autograd(cell):
    prob = pi.random_problem(23, cell, 7, 3, T=2, B=1, rho=0.8)
    m = oracle.Model.from_problem(prob)
    f = torch_cell(prob)
    rng = np.random.default_rng(2)
    x, s = rng.normal(size=prob.d_in), rng.normal(size=prob.D)
    xt = torch.from_numpy(x)
    J_ref = torch.autograd.functional.jacobian(lambda v: f(xt, v), torch.from_numpy(s)).numpy()
    np.testing.assert_allclose(m.jacobian(x, s), J_ref, rtol=0, atol=1e-14)


@pytest.mark.parametrize("cell", CELLS)
def test_mode_jacobians(cell):
    """jacobi: 0 (J~ = I); picard: I (page §2.2.3); quasi: diag of Newton's (page §2.2.1)."""
    prob = pi.random_problem(29, cell, 6, 6, T=2, B=1)
    m = oracle.Model.from_problem(prob)
    rng = np.random.default_rng(3)
    x, s = rng.normal(size=prob.d_in), rng.normal(size=prob.D)
    J = m.approx_jacobian(pi.MODE_NEWTON, x, s)
    np.testing.assert_array_equal(J, m.jacobian(x, s))
    np.testing.assert_array_equal(m.approx_jacobian(pi.MODE_QUASI, x, s), np.diag(np.diag(J)))
    np.testing.assert_array_equal(m.approx_jacobian(pi.MODE_PICARD, x, s), np.eye(prob.D))
    np.testing.assert_array_equal(m.approx_jacobian(pi.MODE_JACOBI, x, s), np.zeros((prob.D, prob.D)))


# ----------------------------------------------------------------------------
# the update s <- s - J~^{-1} F(s) (page §1.2), brute force
# ----------------------------------------------------------------------------

def _torch_approx_jacobian(f, mode, x, s):
    D = s.size
    if mode == pi.MODE_JACOBI:
        return np.zeros((D, D))
    if mode == pi.MODE_PICARD:
        return np.eye(D)
    J = torch.autograd.functional.jacobian(lambda v: f(torch.from_numpy(x), v),
                                           torch.from_numpy(s)).numpy()
    return np.diag(np.diag(J)) if mode == pi.MODE_QUASI else J


@pytest.mark.parametrize("cell", CELLS)
@pytest.mark.parametrize("mode", MODES)
def test_update_equals_dense_solve(cell, mode):
    """Assemble the (T*D)x(T*D) block-bidiagonal J~ = I - subdiag(A~_t) and solve with LAPACK."""
    T, D = 6, 3
    prob = pi.random_problem(31 + cell, cell, D, 2, T=T, B=1, rho=0.9, s0_scale=0.4)
    m = oracle.Model.from_problem(prob)
    f = torch_cell(prob)
    rng = np.random.default_rng(4)
    s_cur = rng.normal(0, 0.5, (1, T, D))
    x = prob.x.astype(np.float64)
    s0 = prob.s0.astype(np.float64)
    # residual from the library cell: F_t = s_t - f_t(s_{t-1})
    F = np.empty((T, D))
    Jt = np.zeros((T * D, T * D))
    for t in range(T):
        prev = s0[0] if t == 0 else s_cur[0, t - 1]
        y = f(torch.from_numpy(x[0, t]), torch.from_numpy(prev)).detach().numpy()
        F[t] = s_cur[0, t] - y
        Jt[t * D:(t + 1) * D, t * D:(t + 1) * D] = np.eye(D)
        if t > 0:
            Jt[t * D:(t + 1) * D, (t - 1) * D:t * D] = -_torch_approx_jacobian(f, mode, x[0, t], prev)
    delta = np.linalg.solve(Jt, -F.ravel()).reshape(T, D)
    got = m.update(mode, prob.x, prob.s0, s_cur)
    np.testing.assert_allclose(got[0], s_cur[0] + delta, rtol=0, atol=1e-12)
    F_or, _ = m.residual(prob.x, prob.s0, s_cur)
    np.testing.assert_allclose(F_or[0], F, rtol=0, atol=1e-14)


# ----------------------------------------------------------------------------
# causality: every mode converges within T iterations (page §3.1)
# ----------------------------------------------------------------------------

@pytest.mark.parametrize("cell", CELLS)
@pytest.mark.parametrize("mode", MODES)
def test_causality(cell, mode):
    T = 12
    prob = pi.random_problem(41 + cell, cell, 4, 3, T=T, B=2, rho=0.9, s0_scale=0.3)
    m = oracle.Model.from_problem(prob)
    seq = m.sequential(prob.x, prob.s0)
    for i in range(T + 1):
        s, it, r, st, hist = m.iterate(mode, prob.x, prob.s0, max_iters=i, tol=0.0)
        assert it == i or r == 0.0
        np.testing.assert_allclose(s[:, :it], seq[:, :it], rtol=0, atol=1e-12)
    s, it, r, st, hist = m.iterate(mode, prob.x, prob.s0, max_iters=T, tol=1e-12)
    assert st == oracle.OK and it <= T
    np.testing.assert_allclose(s, seq, rtol=0, atol=1e-12)


# ----------------------------------------------------------------------------
# closed forms and special cases
# ----------------------------------------------------------------------------

def test_picard_prefix_sum_closed_form():
    """Euler drift with W = 0: f_t(s) = s + eps tanh(c_t) has Jacobian I, so Picard is exact
    after one update and equals s0 + eps * cumsum(tanh(c))."""
    prob = pi.random_problem(51, pi.CELL_EULER, 5, T=30, B=2, eps=0.1, s0_scale=0.5)
    prob.params[:] = 0.0
    m = oracle.Model.from_problem(prob)
    for mode in (pi.MODE_PICARD, pi.MODE_QUASI, pi.MODE_NEWTON):
        s, it, r, st, hist = m.iterate(mode, prob.x, prob.s0, max_iters=prob.T, tol=1e-13)
        expect = prob.s0.astype(np.float64)[:, None, :] + prob.eps * np.cumsum(
            np.tanh(prob.x.astype(np.float64)), axis=1)
        assert it == 1, (mode, hist)
        np.testing.assert_allclose(s, expect, rtol=0, atol=1e-13)


def test_jacobi_input_driven_cell():
    """tanh RNN with W = 0 does not depend on s: Jacobi is exact after one update."""
    prob = pi.random_problem(52, pi.CELL_TANH_RNN, 4, 3, T=25, B=2, rho=0.0)
    m = oracle.Model.from_problem(prob)
    s, it, r, st, hist = m.iterate(pi.MODE_JACOBI, prob.x, prob.s0, max_iters=prob.T, tol=0.0)
    D, d_in = prob.D, prob.d_in
    U = prob.params[D * D:D * D + D * d_in].reshape(D, d_in).astype(np.float64)
    b = prob.params[D * D + D * d_in:].astype(np.float64)
    assert it == 1 and r == 0.0
    np.testing.assert_allclose(s, np.tanh(prob.x.astype(np.float64) @ U.T + b), rtol=0, atol=1e-15)


def test_quasi_equals_newton_for_diagonal_w():
    prob = pi.random_problem(53, pi.CELL_TANH_RNN, 5, 5, T=64, B=2, rho=0.0)
    prob.params[:25] = np.diag(np.array([0.9, -0.5, 0.3, 0.7, -0.8], np.float32)).ravel()
    m = oracle.Model.from_problem(prob)
    a = m.iterate(pi.MODE_QUASI, prob.x, prob.s0, prob.T, 1e-12)
    b = m.iterate(pi.MODE_NEWTON, prob.x, prob.s0, prob.T, 1e-12)
    assert a[1] == b[1]
    np.testing.assert_array_equal(a[4], b[4])
    np.testing.assert_array_equal(a[0], b[0])


def test_newton_few_iterations_when_contractive():
    """||df/ds|| <= rho << 1 (page §3.1): Newton needs very few iterations (table of page §3.2
    lists O(log T)); here a ceiling of 6 at T = 1024."""
    rng = np.random.default_rng(7)
    D, T = 8, 1024
    W = rng.normal(size=(D, D))
    W *= 0.1 / np.linalg.norm(W, 2)            # spectral norm 0.1
    U = rng.normal(0, 1 / np.sqrt(D), (D, D))
    p = np.concatenate([W.ravel(), U.ravel(), np.zeros(D)])
    m = oracle.Model(pi.CELL_TANH_RNN, D, D, p)
    x = rng.normal(size=(2, T, D))
    s, it, r, st, hist = m.iterate(pi.MODE_NEWTON, x, np.zeros((2, D)), T, 1e-10)
    assert st == oracle.OK and it <= 6, hist
    np.testing.assert_allclose(s, m.sequential(x, np.zeros((2, D))), rtol=0, atol=1e-10)
    # quadratic tail: each step at least squares the error scale (up to a constant)
    assert hist[-1] <= 10 * hist[-2] ** 2 + 1e-15


def test_stop_rule_edges():
    prob = pi.random_problem(61, pi.CELL_TANH_RNN, 3, 3, T=10, B=2, rho=0.5, s0_scale=0.2)
    m = oracle.Model.from_problem(prob)
    _, r0 = m.residual(prob.x, prob.s0, np.repeat(prob.s0[:, None, :], prob.T, 1))
    s, it, r, st, hist = m.iterate(pi.MODE_QUASI, prob.x, prob.s0, max_iters=0, tol=1e-9)
    assert (it, st) == (0, oracle.NOT_CONVERGED) and r == r0
    np.testing.assert_array_equal(s, np.repeat(prob.s0.astype(np.float64)[:, None, :], prob.T, 1))
    s, it, r, st, hist = m.iterate(pi.MODE_QUASI, prob.x, prob.s0, max_iters=5, tol=r0)
    assert (it, st) == (0, oracle.OK)          # tie counts as converged (<=)
    bad = prob.x.copy(); bad[1, 4, 0] = np.nan
    s, it, r, st, hist = m.iterate(pi.MODE_NEWTON, bad, prob.s0, max_iters=5, tol=1e-9)
    assert st == oracle.ERR_NONFINITE and it == 0 and math.isnan(r)


def test_threads_do_not_change_results():
    prob = pi.random_problem(62, pi.CELL_GRU, 5, 3, T=30, B=5, rho=0.9)
    m = oracle.Model.from_problem(prob)
    a = m.iterate(pi.MODE_QUASI, prob.x, prob.s0, 30, 1e-10, nthreads=1)
    b = m.iterate(pi.MODE_QUASI, prob.x, prob.s0, 30, 1e-10, nthreads=4)
    np.testing.assert_array_equal(a[0], b[0])
    assert a[1] == b[1]


# ----------------------------------------------------------------------------
# the scan algebra (page §2.1): combine (A,b) o (A',b') = (A'A, A'b + b'), (A,b) earlier
# ----------------------------------------------------------------------------

def _combine(e, l):
    (A, b), (A2, b2) = e, l
    return (A2 @ A, A2 @ b + b2)


def _tree(elems, lo, hi, rng):
    if hi - lo == 1:
        return elems[lo]
    mid = int(rng.integers(lo + 1, hi))
    return _combine(_tree(elems, lo, mid, rng), _tree(elems, mid, hi, rng))


@pytest.mark.parametrize("diag", [False, True])
def test_scan_tree_equals_serial_recurrence(diag):
    rng = np.random.default_rng(8)
    T, D = 23, 4
    A = rng.normal(0, 0.5, (T, D, D))
    if diag:
        A = np.einsum("tij,ij->tij", A, np.eye(D))
    b = rng.normal(size=(T, D))
    s_init = rng.normal(size=D)
    serial = oracle.affine_recurrence(A, b, s_init)
    elems = [(A[t], b[t]) for t in range(T)]
    for trial in range(5):
        for end in (1, 7, T):
            P, q = _tree(elems, 0, end, rng)
            np.testing.assert_allclose(P @ s_init + q, serial[end - 1], rtol=0, atol=1e-12)
    # Hillis-Steele inclusive scan (log-depth) gives every state
    cur = list(elems)
    off = 1
    while off < T:
        cur = [cur[t] if t < off else _combine(cur[t - off], cur[t]) for t in range(T)]
        off *= 2
    states = np.array([P @ s_init + q for (P, q) in cur])
    np.testing.assert_allclose(states, serial, rtol=0, atol=1e-12)


def test_scan_combine_associative():
    rng = np.random.default_rng(9)
    e = [(rng.normal(size=(3, 3)), rng.normal(size=3)) for _ in range(3)]
    l = _combine(_combine(e[0], e[1]), e[2])
    r = _combine(e[0], _combine(e[1], e[2]))
    np.testing.assert_allclose(l[0], r[0], atol=1e-13)
    np.testing.assert_allclose(l[1], r[1], atol=1e-13)
