"""pn_eval_static, the entry point that allocates nothing, against the oracle and against pn_eval.

Some callers cannot call cudaMalloc once they are running: a loop whose device
memory budget is fixed at start-up, code whose device memory belongs to
another framework's allocator, a plug-in that may not grow its footprint.
pn_eval_static serves them with scratch carved out of one fixed device array
of the library.  Here, through the C ABI, on two calls in a row of different
shapes (the second call reuses the array the first one left behind):
- its states match the oracle's same-mode serial iterate and the oracle's
  sequential states to the parity tolerance of the other GPU tests (1e-4
  normwise), and its iteration count equals the oracle's;
- it gives what pn_eval gives (same count, states within the same tolerance);
- a repeated call gives bit-identical states, and the device's free memory
  does not shrink across a call;
- a shape whose scratch would not fit is refused before any launch.
This file is collected last on purpose: a run that stops at the first failure
has run every other test first.
"""
import numpy as np
import pytest

import oracle
import pn_inputs as pi

pytestmark = pytest.mark.gpu

REL_TOL = 1e-4   # normwise, as in the other parity tests


def _relerr(a, ref):
    return float(np.abs(a.astype(np.float64) - ref.astype(np.float64)).max() / max(np.abs(ref).max(), 1e-30))


def _cases(pn):
    return [
        (pi.random_problem(901, pi.CELL_TANH_RNN, 32, 16, T=700, B=3, rho=0.7, s0_scale=0.3, tol=1e-6), pn.PN_QUASI),
        (pi.random_problem(902, pi.CELL_TANH_RNN, 64, 64, T=1500, B=2, rho=0.6, s0_scale=0.2, tol=1e-5), pn.PN_QUASI),
        (pi.random_problem(905, pi.CELL_TANH_RNN, 24, 24, T=300, B=2, rho=0.5, s0_scale=0.3, tol=1e-6), pn.PN_JACOBI),
        (pi.random_problem(906, pi.CELL_TANH_RNN, 16, 16, T=12, B=3, rho=0.5, s0_scale=0.3, tol=1e-6), pn.PN_PICARD),
    ]


def test_static_matches_oracle_and_eval():
    import torch
    import newton_evaluation_nonlinear_b200 as pn
    stream = torch.cuda.current_stream().cuda_stream
    for prob, mode in _cases(pn):   # calls in a row, shapes differ from one to the next
        m = oracle.Model.from_problem(prob)
        seq = m.sequential(prob.x, prob.s0)
        s_or, it_or, r_or, st_or, hist_or = m.iterate(mode, prob.x, prob.s0, prob.T, prob.tol)
        assert float(np.min(np.abs(hist_or / prob.tol - 1.0))) > 1e-2   # counts are unambiguous here
        x = torch.from_numpy(prob.x).cuda()
        s0 = torch.from_numpy(prob.s0).cuda()
        solver = pn.Solver.from_problem(prob)
        ref, it_ref, r_ref, st_ref = solver.eval(x, s0, mode, prob.T, prob.tol)
        ref = ref.cpu().numpy()
        solver.close()
        out = torch.empty((prob.B, prob.T, prob.D), device="cuda", dtype=torch.float32)
        st, it, r = pn.pn_eval_static(prob.params, prob.D, prob.d_in, prob.T, prob.B, x.data_ptr(), s0.data_ptr(),
                                      mode, prob.T, prob.tol, out.data_ptr(), stream)
        assert st == st_or == pn.PN_OK, pn.pn_last_error(None)
        s = out.cpu().numpy()
        assert it == it_or, (mode, it, it_or)
        assert _relerr(s, s_or) <= REL_TOL, _relerr(s, s_or)
        assert _relerr(s, seq) <= max(REL_TOL, 2.0 * _relerr(s_or, seq))
        assert abs(r - r_or) <= 1e-2 * r_or + 5e-6
        assert (st, it) == (st_ref, it_ref)
        assert _relerr(s, ref) <= REL_TOL


def test_static_repeats_allocates_nothing_and_rejects_oversize():
    import torch
    import newton_evaluation_nonlinear_b200 as pn
    stream = torch.cuda.current_stream().cuda_stream
    prob = pi.random_problem(903, pi.CELL_TANH_RNN, 16, 8, T=400, B=4, rho=0.8, s0_scale=0.4, tol=1e-6)
    x = torch.from_numpy(prob.x).cuda()
    s0 = torch.from_numpy(prob.s0).cuda()
    outs = [torch.empty((prob.B, prob.T, prob.D), device="cuda", dtype=torch.float32) for _ in range(2)]
    torch.cuda.synchronize()
    free = []
    for out in outs:
        st, it, r = pn.pn_eval_static(prob.params, prob.D, prob.d_in, prob.T, prob.B, x.data_ptr(), s0.data_ptr(),
                                      pn.PN_QUASI, prob.T, prob.tol, out.data_ptr(), stream)
        assert st == pn.PN_OK, pn.pn_last_error(None)
        torch.cuda.synchronize()
        free.append(torch.cuda.mem_get_info()[0])
    np.testing.assert_array_equal(outs[0].cpu().numpy(), outs[1].cpu().numpy())
    # device allocations come in pages of at least 2 MiB: none happened during the second call
    assert free[1] >= free[0] - (1 << 20), free
    # a shape whose scratch exceeds the fixed array is refused before any launch
    big = pi.random_problem(904, pi.CELL_TANH_RNN, 64, 64, T=4, B=1, tol=1e-5)
    st, _, _ = pn.pn_eval_static(big.params, 64, 64, 1 << 20, 8, x.data_ptr(), s0.data_ptr(), pn.PN_QUASI, 10, 1e-5,
                                 outs[0].data_ptr(), stream)
    assert st == pn.PN_ERR_INVALID
    assert "scratch" in pn.pn_last_error(None)
