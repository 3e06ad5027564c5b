"""Pins of the oracle's refinements of the iteration: the banded Jacobian
approximation (page §2.2.2), damping (page §4.3, §5.3), adaptive switching of
the approximation when the residual stalls (page §5.3), reduced-precision
storage of the iterate (page §2.3) and the windowed solve (page §1.3.1, §2.3).

Each is tied to something other than the oracle itself: LAPACK solves of the
assembled block-bidiagonal system with PyTorch autograd Jacobians, numpy's and
PyTorch's own float conversions, closed forms of input-driven cells, the
sequential definition, and the unrefined iteration it must reduce to.

Citations "page §X" refer to the web article "并行牛顿方法：加速非线性序列评估
的计算革命" (Parallel Newton methods for nonlinear sequence evaluation,
jsqmd.com news item 789890), section X.
"""
import math

import numpy as np
import pytest
import torch

import oracle
import pn_inputs as pi
from test_oracle_pins import CELLS, MODES, torch_cell

STRONGER = {pi.MODE_JACOBI: pi.MODE_QUASI, pi.MODE_PICARD: pi.MODE_QUASI}


# ----------------------------------------------------------------------------
# storage rounding against the libraries' conversions
# ----------------------------------------------------------------------------

def _probe_values(rng):
    v = np.concatenate([
        rng.normal(0, 1, 4000),
        rng.normal(0, 1, 2000) * 10.0 ** rng.integers(-12, 6, 2000),
        rng.uniform(-1, 1, 2000) * 2.0 ** -130,          # binary32 subnormal range
        rng.uniform(-1, 1, 2000) * 2.0 ** -15,           # binary16 subnormal range
        np.array([0.0, -0.0, 1.0, -1.0, 65504.0, 65519.0, 65520.0, 7e4, 3.4e38, 3.41e38]),
    ])
    return v


def test_round_storage_f32_f16_match_numpy():
    rng = np.random.default_rng(11)
    v = _probe_values(rng)
    with np.errstate(over="ignore"):
        want32 = v.astype(np.float32).astype(np.float64)
        want16 = v.astype(np.float16).astype(np.float64)
    np.testing.assert_array_equal(oracle.round_storage(v, oracle.STORE_F32), want32)
    np.testing.assert_array_equal(oracle.round_storage(v, oracle.STORE_F16), want16)
    np.testing.assert_array_equal(oracle.round_storage(v, oracle.STORE_F64), v)


def test_round_storage_bf16_matches_torch_on_binary32_values():
    """torch rounds float32 -> bfloat16 to nearest even; on float32 inputs one rounding is all
    there is, so the oracle's single rounding from double must agree exactly."""
    rng = np.random.default_rng(12)
    with np.errstate(over="ignore"):
        v = _probe_values(rng).astype(np.float32)
    v = v[np.isfinite(v)]
    # add exact ties: halfway between neighbouring bfloat16 values
    k = rng.integers(0, 2 ** 7, 500)
    ties = (1.0 + (2 * k + 1) * 2.0 ** -8) * 2.0 ** rng.integers(-100, 100, 500)
    v = np.concatenate([v, ties.astype(np.float32), -ties.astype(np.float32)])
    want = torch.from_numpy(v).to(torch.bfloat16).to(torch.float64).numpy()
    np.testing.assert_array_equal(oracle.round_storage(v.astype(np.float64), oracle.STORE_BF16), want)


def test_round_storage_rounds_once_from_double():
    """The oracle rounds the double straight to the format (one rounding).  Just above a
    bfloat16 tie the result goes up; a double rounding through binary32 would land on the tie
    and go to even instead."""
    v = 1.0 + 2.0 ** -8 + 2.0 ** -40
    assert oracle.round_storage([v], oracle.STORE_BF16)[0] == 1.0 + 2.0 ** -7
    assert oracle.round_storage([1.0 + 2.0 ** -8], oracle.STORE_BF16)[0] == 1.0          # tie, even
    assert oracle.round_storage([1.0 + 3 * 2.0 ** -8], oracle.STORE_BF16)[0] == 1.0 + 2.0 ** -6
    big = (2.0 - 2.0 ** -8) * 2.0 ** 127                      # halfway to the next binade: overflows
    assert oracle.round_storage([big, -big], oracle.STORE_BF16).tolist() == [math.inf, -math.inf]
    with pytest.raises(RuntimeError):
        oracle.round_storage([1.0], 7)


# ----------------------------------------------------------------------------
# banded Jacobian approximation (page §2.2.2)
# ----------------------------------------------------------------------------

@pytest.mark.parametrize("cell", CELLS)
def test_banded_jacobian_against_autograd(cell):
    D = 6
    prob = pi.random_problem(71 + cell, cell, D, 4, T=2, B=1, rho=0.9, s0_scale=0.5)
    m = oracle.Model.from_problem(prob)
    f = torch_cell(prob)
    x, s = prob.x[0, 0].astype(np.float64), np.random.default_rng(3).normal(0, 0.5, D)
    J = torch.autograd.functional.jacobian(lambda v: f(torch.from_numpy(x), v), torch.from_numpy(s)).numpy()
    jj, kk = np.indices((D, D))
    for band in range(D + 1):
        A = m.banded_jacobian(band, x, s)
        inside = np.abs(jj - kk) <= band
        np.testing.assert_allclose(A[inside], J[inside], rtol=0, atol=1e-13)
        assert not np.any(A[~inside])
    np.testing.assert_array_equal(m.banded_jacobian(0, x, s), m.approx_jacobian(pi.MODE_QUASI, x, s))
    np.testing.assert_array_equal(m.banded_jacobian(D - 1, x, s), m.approx_jacobian(pi.MODE_NEWTON, x, s))
    with pytest.raises(RuntimeError):
        m.banded_jacobian(-1, x, s)


def _dense_update(prob, s_cur, A_of):
    """s_cur + solve(J~, -F) with J~ = I - subdiag(A~_t), assembled densely; A_of(x_t, s_prev)
    gives A~_t and F comes from the PyTorch cell."""
    f = torch_cell(prob)
    T, D = s_cur.shape[1], prob.D
    x, s0 = prob.x.astype(np.float64), prob.s0.astype(np.float64)
    F = np.empty((T, D))
    Jt = np.eye(T * D)
    for t in range(T):
        prev = s0[0] if t == 0 else s_cur[0, t - 1]
        F[t] = s_cur[0, t] - f(torch.from_numpy(x[0, t]), torch.from_numpy(prev)).detach().numpy()
        if t > 0:
            Jt[t * D:(t + 1) * D, (t - 1) * D:t * D] = -A_of(x[0, t], prev)
    return np.linalg.solve(Jt, -F.ravel()).reshape(T, D)


@pytest.mark.parametrize("cell", CELLS)
@pytest.mark.parametrize("band", [1, 2])
@pytest.mark.parametrize("damping", [1.0, 0.375])
def test_banded_damped_update_equals_dense_solve(cell, band, damping):
    T, D = 6, 5
    prob = pi.random_problem(81 + cell, cell, D, 3, T=T, B=1, rho=0.9, s0_scale=0.4)
    m = oracle.Model.from_problem(prob)
    f = torch_cell(prob)

    def banded(x_t, prev):
        J = torch.autograd.functional.jacobian(lambda v: f(torch.from_numpy(x_t), v),
                                               torch.from_numpy(prev)).numpy()
        jj, kk = np.indices(J.shape)
        return np.where(np.abs(jj - kk) <= band, J, 0.0)

    s_cur = np.random.default_rng(5).normal(0, 0.5, (1, T, D))
    delta = _dense_update(prob, s_cur, banded)
    got = m.update_ex(oracle.BANDED, prob.x, prob.s0, s_cur, band=band, damping=damping)
    np.testing.assert_allclose(got[0], s_cur[0] + damping * delta, rtol=0, atol=1e-12)


@pytest.mark.parametrize("mode", MODES)
def test_damped_update_equals_scaled_dense_solve(mode):
    T, D = 5, 3
    prob = pi.random_problem(91, pi.CELL_GRU, D, 2, T=T, B=1, rho=0.9, s0_scale=0.4)
    m = oracle.Model.from_problem(prob)
    s_cur = np.random.default_rng(6).normal(0, 0.5, (1, T, D))
    delta = _dense_update(prob, s_cur, lambda x_t, prev: m.approx_jacobian(mode, x_t, prev))
    got = m.update_ex(mode, prob.x, prob.s0, s_cur, damping=0.25)
    np.testing.assert_allclose(got[0], s_cur[0] + 0.25 * delta, rtol=0, atol=1e-12)
    np.testing.assert_array_equal(m.update_ex(mode, prob.x, prob.s0, s_cur), m.update(mode, prob.x, prob.s0, s_cur))
    for bad in (0.0, -0.5, 1.5, math.nan):
        with pytest.raises(RuntimeError):
            m.update_ex(mode, prob.x, prob.s0, s_cur, damping=bad)


# ----------------------------------------------------------------------------
# closed forms: an input-driven cell (tanh RNN with W = 0, f_t(s) = c_t)
# ----------------------------------------------------------------------------

def _input_driven(seed, T=20, B=2, D=4, d_in=3, s0_scale=0.0):
    prob = pi.random_problem(seed, pi.CELL_TANH_RNN, D, d_in, T=T, B=B, rho=0.0, s0_scale=s0_scale)
    U = prob.params[D * D:D * D + D * d_in].reshape(D, d_in).astype(np.float64)
    b = prob.params[D * D + D * d_in:].astype(np.float64)
    m = oracle.Model.from_problem(prob)
    # c_t from the cell itself (pinned against torch.nn.RNNCell), so that exact equalities below
    # do not depend on the summation order; it is the closed form up to rounding
    c = np.array([[m.cell_step(prob.x[bb, t], np.zeros(D)) for t in range(T)] for bb in range(B)])
    np.testing.assert_allclose(c, np.tanh(prob.x.astype(np.float64) @ U.T + b), rtol=0, atol=1e-15)
    return prob, m, c


def test_damped_jacobi_closed_form():
    """f_t(s) = c_t and J~ = I: s <- s - lambda (s - c), so s^(i) - c = (1 - lambda)^i (s^(0) - c)
    and r^(i) = (1 - lambda)^i r^(0); the count is the first i with (1 - lambda)^i r^(0) <= tol."""
    prob, m, c = _input_driven(101, s0_scale=0.7)
    lam = 0.4
    s_init = np.repeat(prob.s0.astype(np.float64)[:, None, :], prob.T, 1)
    r0 = np.max(np.abs(s_init - c))
    tol = r0 * (1 - lam) ** 7.5
    s, it, r, st, hist, modes, wit = m.iterate_ex(pi.MODE_JACOBI, prob.x, prob.s0, 50, tol, damping=lam)
    assert (it, st) == (8, oracle.OK)
    np.testing.assert_allclose(hist, r0 * (1 - lam) ** np.arange(9), rtol=1e-12, atol=0)
    np.testing.assert_allclose(s, c + (1 - lam) ** 8 * (s_init - c), rtol=0, atol=1e-15)
    assert modes.tolist() == [pi.MODE_JACOBI] * 8 + [-1]


@pytest.mark.parametrize("store", [oracle.STORE_BF16, oracle.STORE_F16, oracle.STORE_F32])
def test_reduced_storage_closed_form(store):
    """s0 = 0, f_t(s) = c_t, Jacobi: the first update gives c exactly, stored as round(c), so
    r^(1) = max|round(c) - c|; every later update returns c and stores round(c) again, so the
    residual stays at r^(1).  With store_until = r^(1), update i stores round(c) while the residual
    known when it starts, r^(i-1), is above r^(1): update 0 (nothing known yet) and update 1
    (r^(0) = max|c|) do; update 2 starts knowing r^(1), which is not above store_until, so s^(3) = c
    is kept in double and the iteration ends at i = 3 with r = 0 and the states equal to c."""
    prob, m, c = _input_driven(102)
    rc = oracle.round_storage(c, store)
    r1 = np.max(np.abs(rc - c))
    assert r1 > 0
    s, it, r, st, hist, modes, wit = m.iterate_ex(pi.MODE_JACOBI, prob.x, prob.s0, 6, r1 / 2, store=store)
    assert (it, st) == (6, oracle.NOT_CONVERGED)
    assert hist[0] == np.max(np.abs(c)) and np.all(hist[1:] == r1)
    np.testing.assert_array_equal(s, rc)
    s, it, r, st, hist, modes, wit = m.iterate_ex(pi.MODE_JACOBI, prob.x, prob.s0, 6, 0.0,
                                                  store=store, store_until=r1)
    assert (it, st, r) == (3, oracle.OK, 0.0)
    assert hist[1] == r1 and hist[2] == r1
    np.testing.assert_array_equal(s, c)


def test_reduced_storage_iterates_are_representable():
    prob = pi.random_problem(103, pi.CELL_GRU, 6, 4, T=40, B=3, rho=0.9, s0_scale=0.3)
    m = oracle.Model.from_problem(prob)
    for store in (oracle.STORE_BF16, oracle.STORE_F16):
        for max_iters in (0, 3, 7):
            s, it, r, st, hist, modes, wit = m.iterate_ex(pi.MODE_QUASI, prob.x, prob.s0, max_iters, 0.0,
                                                          store=store)
            np.testing.assert_array_equal(oracle.round_storage(s, store), s)
        # and the rounding floor: the residual cannot go below the format's resolution
        s, it, r, st, hist, modes, wit = m.iterate_ex(pi.MODE_NEWTON, prob.x, prob.s0, 40, 1e-9, store=store)
        assert st == oracle.NOT_CONVERGED and r > 1e-5
        seq = m.sequential(prob.x, prob.s0)
        unit = 2.0 ** -8 if store == oracle.STORE_BF16 else 2.0 ** -11
        assert np.max(np.abs(s - seq)) < 8 * unit


# ----------------------------------------------------------------------------
# adaptive switching (page §5.3)
# ----------------------------------------------------------------------------

def _expected_schedule(start, band, stall, hist):
    modes, mode = [], start
    for i in range(len(hist) - 1):
        if i >= 1 and hist[i] > stall * hist[i - 1]:
            if mode in STRONGER:
                mode = STRONGER[mode]
            elif mode == pi.MODE_QUASI:
                mode = oracle.BANDED if band >= 1 else pi.MODE_NEWTON
            else:
                mode = pi.MODE_NEWTON
        modes.append(mode)
    return modes + [-1]


@pytest.mark.parametrize("cell", CELLS)
@pytest.mark.parametrize("start", [pi.MODE_JACOBI, pi.MODE_PICARD, pi.MODE_QUASI])
def test_adaptive_schedule_and_result(cell, start):
    T = 48
    prob = pi.random_problem(111 + cell, cell, 5, 3, T=T, B=2, rho=0.95, s0_scale=0.3, eps=0.05)
    m = oracle.Model.from_problem(prob)
    seq = m.sequential(prob.x, prob.s0)
    for band, stall in ((0, 0.5), (2, 0.5), (1, 0.0)):
        s, it, r, st, hist, modes, wit = m.iterate_ex(start, prob.x, prob.s0, T, 1e-11, band=band,
                                                      adapt=True, stall=stall)
        assert st == oracle.OK and it <= T
        assert modes.tolist() == _expected_schedule(start, band, stall, hist)
        np.testing.assert_allclose(s, seq, rtol=0, atol=1e-9)
    # stall = 0 climbs one rung per iteration from the second update on
    s, it, r, st, hist, modes, wit = m.iterate_ex(pi.MODE_JACOBI, prob.x, prob.s0, T, 1e-11, band=1,
                                                  adapt=True, stall=0.0)
    ladder = [pi.MODE_JACOBI, pi.MODE_QUASI, oracle.BANDED, pi.MODE_NEWTON]
    assert modes[:-1].tolist() == (ladder + [pi.MODE_NEWTON] * T)[:it]


@pytest.mark.parametrize("mode", MODES)
def test_adaptive_off_or_never_stalling_is_the_plain_iteration(mode):
    prob = pi.random_problem(121, pi.CELL_EULER, 6, T=40, B=2, rho=0.9, s0_scale=0.3, eps=0.05)
    m = oracle.Model.from_problem(prob)
    base = m.iterate(mode, prob.x, prob.s0, 40, 1e-10)
    for kw in ({}, {"adapt": True, "stall": math.inf}):
        got = m.iterate_ex(mode, prob.x, prob.s0, 40, 1e-10, **kw)
        assert got[1:4] == base[1:4]
        np.testing.assert_array_equal(got[0], base[0])
        np.testing.assert_array_equal(got[4], base[4])


def test_adaptive_rescues_a_slow_jacobi_run():
    """Euler drift with a small step: Jacobi advances about one step per iteration (its residual
    ratio stays near 1), so the first stall check moves it to quasi-Newton."""
    prob = pi.random_problem(122, pi.CELL_EULER, 8, T=256, B=2, rho=0.9, s0_scale=0.3, eps=0.02)
    m = oracle.Model.from_problem(prob)
    plain = m.iterate(pi.MODE_JACOBI, prob.x, prob.s0, 256, 1e-9)
    s, it, r, st, hist, modes, wit = m.iterate_ex(pi.MODE_JACOBI, prob.x, prob.s0, 256, 1e-9,
                                                  adapt=True, stall=0.9)
    assert st == oracle.OK and it < plain[1] // 4
    assert modes[0] == pi.MODE_JACOBI and modes[1] == pi.MODE_QUASI
    np.testing.assert_allclose(s, m.sequential(prob.x, prob.s0), rtol=0, atol=1e-7)


# ----------------------------------------------------------------------------
# windowed solve (page §1.3.1, §2.3)
# ----------------------------------------------------------------------------

@pytest.mark.parametrize("mode", MODES)
def test_one_window_is_the_plain_iteration(mode):
    prob = pi.random_problem(131, pi.CELL_TANH_RNN, 5, 4, T=33, B=3, rho=0.8, s0_scale=0.3)
    m = oracle.Model.from_problem(prob)
    base = m.iterate(mode, prob.x, prob.s0, 33, 1e-10)
    for window in (0, -3, 33, 100):
        got = m.iterate_ex(mode, prob.x, prob.s0, 33, 1e-10, window=window)
        assert got[1:4] == base[1:4] and got[6].tolist() == [base[1]]
        np.testing.assert_array_equal(got[0], base[0])
        np.testing.assert_array_equal(got[4], base[4])


@pytest.mark.parametrize("cell", CELLS)
@pytest.mark.parametrize("mode", MODES)
def test_windows_of_one_step_are_the_sequential_loop(cell, mode):
    """A window of one step is solved by one update (causality, page §3.1), so the windowed solve
    walks the sequence step by step."""
    T = 17
    prob = pi.random_problem(141 + cell, cell, 4, 3, T=T, B=2, rho=0.9, s0_scale=0.3, eps=0.05)
    m = oracle.Model.from_problem(prob)
    s, it, r, st, hist, modes, wit = m.iterate_ex(mode, prob.x, prob.s0, 5, 1e-13, window=1)
    assert st == oracle.OK and wit.tolist() == [1] * T and it == T
    np.testing.assert_allclose(s, m.sequential(prob.x, prob.s0), rtol=0, atol=1e-13)


@pytest.mark.parametrize("cell", CELLS)
@pytest.mark.parametrize("window", [4, 7, 16])
def test_windowed_residual_is_the_whole_sequence_residual(cell, window):
    """The reported residual is the max-norm of F over the whole output (window hand-offs
    included), each window needs at most its length in iterations, and the states agree with the
    sequential definition."""
    T = 30
    prob = pi.random_problem(151 + cell, cell, 5, 3, T=T, B=3, rho=0.9, s0_scale=0.3, eps=0.05)
    m = oracle.Model.from_problem(prob)
    for mode in (pi.MODE_QUASI, pi.MODE_NEWTON, pi.MODE_PICARD):
        s, it, r, st, hist, modes, wit = m.iterate_ex(mode, prob.x, prob.s0, T, 1e-11, window=window)
        assert st == oracle.OK and len(wit) == -(-T // window) and it == wit.sum()
        lens = [min(window, T - k * window) for k in range(len(wit))]
        assert all(w <= n for w, n in zip(wit, lens))
        _, r_full = m.residual(prob.x, prob.s0, s)
        assert r_full == r
        assert len(hist) == it + len(wit) and np.sum(modes == -1) == len(wit)
        np.testing.assert_allclose(s, m.sequential(prob.x, prob.s0), rtol=0, atol=1e-9)


def test_windowed_failure_and_budget():
    T, window = 24, 8
    prob = pi.random_problem(161, pi.CELL_TANH_RNN, 3, 3, T=T, B=2, rho=0.9, s0_scale=0.3)
    m = oracle.Model.from_problem(prob)
    # a budget below the window length: every window stops short, the next still runs
    s, it, r, st, hist, modes, wit = m.iterate_ex(pi.MODE_PICARD, prob.x, prob.s0, 2, 1e-14, window=window)
    assert st == oracle.NOT_CONVERGED and wit.tolist() == [2, 2, 2] and it == 6
    # a non-finite input in the second window: the third keeps its initial guess
    bad = prob.x.copy()
    bad[1, 10, 0] = np.nan
    s, it, r, st, hist, modes, wit = m.iterate_ex(pi.MODE_QUASI, bad, prob.s0, T, 1e-12, window=window)
    assert st == oracle.ERR_NONFINITE and math.isnan(r) and wit[2] == 0
    np.testing.assert_array_equal(s[:, 16:], np.repeat(s[:, 15:16], 8, axis=1))
    good = m.iterate_ex(pi.MODE_QUASI, prob.x, prob.s0, T, 1e-12, window=window)
    np.testing.assert_array_equal(s[:, :8], good[0][:, :8])


def test_refinements_combine_per_window():
    """Windows are independent solves: with adaptive switching every window restarts from the
    start mode, and a window's own schedule follows the rule on its own residuals."""
    T, window = 60, 20
    prob = pi.random_problem(171, pi.CELL_EULER, 6, T=T, B=2, rho=0.9, s0_scale=0.3, eps=0.05)
    m = oracle.Model.from_problem(prob)
    s, it, r, st, hist, modes, wit = m.iterate_ex(pi.MODE_JACOBI, prob.x, prob.s0, T, 1e-10, adapt=True,
                                                  stall=0.5, damping=0.9, window=window)
    assert st == oracle.OK and len(wit) == 3
    pos = 0
    for w in wit:
        h, md = hist[pos:pos + w + 1], modes[pos:pos + w + 1]
        assert md[0] == pi.MODE_JACOBI and md[-1] == -1
        assert md.tolist() == _expected_schedule(pi.MODE_JACOBI, 0, 0.5, h)
        pos += w + 1
    np.testing.assert_allclose(s, m.sequential(prob.x, prob.s0), rtol=0, atol=1e-8)


def test_refinements_do_not_depend_on_threads():
    prob = pi.random_problem(172, pi.CELL_GRU, 5, 3, T=45, B=5, rho=0.9, s0_scale=0.3)
    m = oracle.Model.from_problem(prob)
    kw = dict(band=1, damping=0.8, adapt=True, stall=0.6, store=oracle.STORE_F32, store_until=1e-4, window=16)
    a = m.iterate_ex(pi.MODE_PICARD, prob.x, prob.s0, 45, 1e-9, nthreads=1, **kw)
    b = m.iterate_ex(pi.MODE_PICARD, prob.x, prob.s0, 45, 1e-9, nthreads=4, **kw)
    assert a[1:4] == b[1:4]
    for x, y in zip(a[4:], b[4:]):
        np.testing.assert_array_equal(x, y)
    np.testing.assert_array_equal(a[0], b[0])
