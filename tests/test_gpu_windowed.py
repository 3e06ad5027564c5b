"""GPU parity of the windowed solve (pn_eval_windowed, web article "并行牛顿方法：
加速非线性序列评估的计算革命" §1.3.1 and §2.3): the long sequence is solved window
after window, each window by the handle's iteration with the previous window's
last state as its s0.  The oracle's orc_iterate_ex with the same window length
is the reference: per-window iteration counts equal (unless an oracle residual
lies within 1% of tol), states within 1e-4 normwise of the oracle's windowed
iterate and of the sequential states.
"""
import numpy as np
import pytest

import oracle
import pn_inputs as pi

pytestmark = pytest.mark.gpu

REL_TOL = 1e-4


def _relerr(a, ref):
    den = max(float(np.abs(ref).max()), 1e-30)
    return float(np.abs(a.astype(np.float64) - ref).max()) / den


def _solvers(pn, prob, W):
    h = pn.Solver(prob.cell, prob.D, prob.d_in, W, prob.B, prob.params, prob.eps)
    rem = prob.T % W
    tail = pn.Solver(prob.cell, prob.D, prob.d_in, rem, prob.B, prob.params, prob.eps) if rem else None
    return h, tail


def _run(prob, mode, W, tol, max_iters):
    import torch
    import newton_evaluation_nonlinear_b200 as pn
    h, tail = _solvers(pn, prob, W)
    x = torch.from_numpy(prob.x).cuda()
    s0 = torch.from_numpy(prob.s0).cuda()
    states, it, r, st, wit = h.eval_windowed(x, s0, mode, max_iters, tol, tail=tail)
    out = states.cpu().numpy()
    h.close()
    if tail is not None:
        tail.close()
    return out, it, r, st, wit


CASES = [
    (pi.CELL_TANH_RNN, 64, 64, pi.MODE_QUASI),
    (pi.CELL_TANH_RNN, 4, 4, pi.MODE_NEWTON),
    (pi.CELL_TANH_RNN, 16, 16, pi.MODE_JACOBI),
    (pi.CELL_GRU, 32, 32, pi.MODE_QUASI),
    (pi.CELL_EULER, 16, 16, pi.MODE_PICARD),
]


@pytest.mark.parametrize("cell,D,d_in,mode", CASES)
@pytest.mark.parametrize("T,W", [(1000, 256), (1024, 256), (100, 256), (600, 600), (333, 50)])
def test_windowed_matches_oracle(cell, D, d_in, mode, T, W):
    prob = pi.random_problem(201 + cell + D, cell, D, d_in, T=T, B=3, rho=0.8, s0_scale=0.3, eps=0.05)
    m = oracle.Model.from_problem(prob)
    seq = m.sequential(prob.x, prob.s0)
    tol = 1e-5 * max(1.0, float(np.abs(seq).max()))
    mi = W
    s_or, it_or, r_or, st_or, hist_or, modes_or, wit_or = m.iterate_ex(mode, prob.x, prob.s0, mi, tol, window=W)
    s, it, r, st, wit = _run(prob, mode, W, tol, mi)
    assert np.isfinite(s).all()
    assert len(wit) == len(wit_or) == -(-T // W)
    margin = float(np.min(np.abs(hist_or / tol - 1.0)))
    if margin > 1e-2:
        assert wit.tolist() == wit_or.tolist() and it == it_or and st == st_or, (wit, wit_or)
    else:
        assert np.all(np.abs(wit - wit_or) <= 1)
    if wit.tolist() == wit_or.tolist():
        assert _relerr(s, s_or) <= REL_TOL, _relerr(s, s_or)
    if st == oracle.OK:
        assert r <= tol
        assert _relerr(s, seq) <= max(REL_TOL, 2.0 * _relerr(s_or, seq))


def test_windowed_budget_and_handoff():
    """max_iters below the window length: every window stops short (NOT_CONVERGED) and the next
    one starts from that window's last iterate, as in the oracle."""
    prob = pi.random_problem(211, pi.CELL_TANH_RNN, 16, 16, T=700, B=2, rho=0.9, s0_scale=0.3)
    m = oracle.Model.from_problem(prob)
    s_or, it_or, r_or, st_or, hist_or, modes_or, wit_or = m.iterate_ex(pi.MODE_QUASI, prob.x, prob.s0, 3, 1e-12,
                                                                       window=200)
    s, it, r, st, wit = _run(prob, pi.MODE_QUASI, 200, 1e-12, 3)
    assert st == st_or == oracle.NOT_CONVERGED
    assert wit.tolist() == wit_or.tolist() == [3, 3, 3, 3] and it == it_or == 12
    assert _relerr(s, s_or) <= REL_TOL, _relerr(s, s_or)


def test_windowed_argument_checks():
    import torch
    import newton_evaluation_nonlinear_b200 as pn
    prob = pi.random_problem(212, pi.CELL_TANH_RNN, 8, 8, T=100, B=2, rho=0.5)
    h, tail = _solvers(pn, prob, 30)          # 100 = 3 * 30 + 10
    wrong = pn.Solver(prob.cell, prob.D, prob.d_in, 20, prob.B, prob.params, prob.eps)
    x = torch.from_numpy(prob.x).cuda()
    s0 = torch.from_numpy(prob.s0).cuda()
    out = torch.empty((prob.B, prob.T, prob.D), device="cuda")
    for t in (None, wrong, h):
        st, it, r, wit = pn.pn_eval_windowed(h.h, t.h if t is not None else None, prob.T, x.data_ptr(),
                                             s0.data_ptr(), pn.PN_QUASI, 10, 1e-5, out.data_ptr(), 4)
        assert st == pn.PN_ERR_INVALID, st
    # a tail when the window divides T_total, and T_total < 1
    st, *_ = pn.pn_eval_windowed(wrong.h, tail.h, prob.T, x.data_ptr(), s0.data_ptr(), pn.PN_QUASI, 10, 1e-5,
                                 out.data_ptr(), 5)
    assert st == pn.PN_ERR_INVALID and "NULL" in pn.pn_last_error(wrong.h)
    st, *_ = pn.pn_eval_windowed(h.h, None, 0, x.data_ptr(), s0.data_ptr(), pn.PN_QUASI, 10, 1e-5,
                                 out.data_ptr(), 0)
    assert st == pn.PN_ERR_INVALID
    # the valid call still works on the same handles afterwards
    states, it, r, st, wit = h.eval_windowed(x, s0, "quasi", 30, 1e-5, tail=tail)
    assert st == pn.PN_OK and len(wit) == 4
    for s in (h, tail, wrong):
        s.close()
