"""pn_eval_static, the entry point that allocates nothing, against pn_eval.

Callers that cannot call cudaMalloc while running (a fixed device-memory budget,
memory owned by another framework's allocator) use pn_eval_static, whose scratch
is one fixed device array of the library.  Here it must give what pn_eval gives,
within the parity tolerance of the other GPU tests, on two calls in a row (the
second call reuses the array the first one left behind).  This file is collected
last on purpose.
"""
import numpy as np
import pytest

import pn_inputs as pi

pytestmark = pytest.mark.gpu

REL_TOL = 1e-4   # normwise, as in the other parity tests


def _relerr(a, ref):
    return float(np.abs(a.astype(np.float64) - ref.astype(np.float64)).max() / max(np.abs(ref).max(), 1e-30))


def test_static_matches_eval_two_calls():
    import torch
    import newton_evaluation_nonlinear_b200 as pn
    stream = torch.cuda.current_stream().cuda_stream
    cases = [(pi.random_problem(901, pi.CELL_TANH_RNN, 32, 16, T=700, B=3, rho=0.7, s0_scale=0.3, tol=1e-6),
              pn.PN_QUASI),
             (pi.random_problem(902, pi.CELL_TANH_RNN, 64, 64, T=1500, B=2, rho=0.6, s0_scale=0.2, tol=1e-5),
              pn.PN_QUASI)]
    for prob, mode in cases:   # two calls in a row, different shapes
        x = torch.from_numpy(prob.x).cuda()
        s0 = torch.from_numpy(prob.s0).cuda()
        solver = pn.Solver.from_problem(prob)
        ref, it_ref, r_ref, st_ref = solver.eval(x, s0, mode, prob.T, prob.tol)
        ref = ref.cpu().numpy()
        solver.close()
        out = torch.empty((prob.B, prob.T, prob.D), device="cuda", dtype=torch.float32)
        st, it, r = pn.pn_eval_static(prob.params, prob.D, prob.d_in, prob.T, prob.B, x.data_ptr(), s0.data_ptr(),
                                      mode, prob.T, prob.tol, out.data_ptr(), stream)
        assert st == st_ref == pn.PN_OK, pn.pn_last_error(None)
        assert it == it_ref
        assert _relerr(out.cpu().numpy(), ref) <= REL_TOL


def test_static_repeats_and_rejects_oversize():
    import torch
    import newton_evaluation_nonlinear_b200 as pn
    stream = torch.cuda.current_stream().cuda_stream
    prob = pi.random_problem(903, pi.CELL_TANH_RNN, 16, 8, T=400, B=4, rho=0.8, s0_scale=0.4, tol=1e-6)
    x = torch.from_numpy(prob.x).cuda()
    s0 = torch.from_numpy(prob.s0).cuda()
    outs = []
    for _ in range(2):
        out = torch.empty((prob.B, prob.T, prob.D), device="cuda", dtype=torch.float32)
        st, it, r = pn.pn_eval_static(prob.params, prob.D, prob.d_in, prob.T, prob.B, x.data_ptr(), s0.data_ptr(),
                                      pn.PN_QUASI, prob.T, prob.tol, out.data_ptr(), stream)
        assert st == pn.PN_OK, pn.pn_last_error(None)
        outs.append(out.cpu().numpy())
    np.testing.assert_array_equal(outs[0], outs[1])
    # a shape whose scratch exceeds the fixed array is refused before any launch
    big = pi.random_problem(904, pi.CELL_TANH_RNN, 64, 64, T=4, B=1, tol=1e-5)
    st, _, _ = pn.pn_eval_static(big.params, 64, 64, 1 << 20, 8, x.data_ptr(), s0.data_ptr(), pn.PN_QUASI, 10, 1e-5,
                                 out.data_ptr(), stream)
    assert st == pn.PN_ERR_INVALID
    assert "scratch" in pn.pn_last_error(None)
