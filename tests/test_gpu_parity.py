"""GPU parity: libpn's CUDA path against the fp64 oracle, through the C ABI.

For every cell and mode, on seeded inputs that span several tiles and a ragged
tail, the states must match the oracle's sequential evaluation to a normwise
relative error of 1e-4, and the iteration count must equal the oracle's serial
iteration with the same tol (exactly, unless some oracle residual lies within
1% of tol, where fp32 rounding may legitimately move one iteration).
"""
import numpy as np
import pytest

import oracle
import pn_inputs as pi

pytestmark = pytest.mark.gpu

REL_TOL = 1e-4          # normwise max|s_gpu - s_ref| / max|s_ref|
# Residual histories: r^(i) = max|F(s^(i))| in fp32 from an fp32 iterate against the oracle's fp64 one.
# Early residuals are large and agree to well under 1%; near tol the difference is absolute: the
# iterate carries a few ulp(max|s|) of scan rounding per step, the activations are within 4e-7, and
# F_t = s_t - f_t(s_{t-1}) cancels to ~1e-5, so an absolute floor of a few 1e-6 * max(1, max|s|) applies.
HIST_RTOL = 1e-2
HIST_ATOL = 5e-6


def _pn():
    import newton_evaluation_nonlinear_b200 as pn   # raises if libpn.so is missing
    return pn


def _run(prob, mode, tol=None, max_iters=None, device_loop=1, tc=1, opts=None):
    import torch
    pn = _pn()
    solver = pn.Solver.from_problem(prob)
    solver.set_option(pn.PN_OPT_DEVICE_LOOP, device_loop)
    solver.set_option(pn.PN_OPT_TENSOR_CORES, tc)
    for name, value in (opts or {}).items():
        solver.set_option(getattr(pn, name), value)
    x = torch.from_numpy(prob.x).cuda()
    s0 = torch.from_numpy(prob.s0).cuda()
    tol = prob.tol if tol is None else tol
    mi = prob.iters_cap if max_iters is None else max_iters
    states, it, r, st = solver.eval(x, s0, mode, mi, tol)
    hist = solver.residual_history()
    out = states.cpu().numpy()
    solver.close()
    return out, it, r, st, hist


def _relerr(a, ref):
    den = max(float(np.abs(ref).max()), 1e-30)
    return float(np.abs(a.astype(np.float64) - ref).max()) / den


def _check_against_oracle(prob, mode, tol=None, max_iters=None, device_loop=1, tc=1, opts=None):
    """tol defaults to prob.tol * max(1, max|s|): an fp32 iterate assembled by a parallel scan carries
    rounding of a few ulp(|s|) per step, so an absolute tol below ~1e-6 |s| would sit on the fp32
    floor (the Euler drift reaches |s| ~ 20 on these inputs; the tanh and GRU states stay within 1)."""
    mi = prob.iters_cap if max_iters is None else max_iters
    m = oracle.Model.from_problem(prob)
    seq = m.sequential(prob.x, prob.s0)
    tol = prob.tol * max(1.0, float(np.abs(seq).max())) if tol is None else tol
    s_or, it_or, r_or, st_or, hist_or = m.iterate(mode, prob.x, prob.s0, mi, tol)
    s, it, r, st, hist = _run(prob, mode, tol, mi, device_loop, tc, opts)
    assert np.isfinite(s).all()
    margin = float(np.min(np.abs(hist_or / tol - 1.0))) if tol > 0 else 1.0
    if margin > 1e-2:
        assert it == it_or, (prob.name, mode, it, it_or, hist[:it + 1], hist_or)
        assert st == st_or
    else:
        assert abs(it - it_or) <= 1
    # same iterate as the oracle's serial iteration (fp32 vs fp64 arithmetic only)
    if it == it_or:
        assert _relerr(s, s_or) <= REL_TOL, _relerr(s, s_or)
    if st == oracle.OK:
        # the GPU's distance to the sequential states is the oracle iterate's own iteration error
        # plus fp32 rounding
        assert _relerr(s, seq) <= max(REL_TOL, 2.0 * _relerr(s_or, seq)), (_relerr(s, seq), _relerr(s_or, seq))
    # residual history: fp32 residuals track the fp64 ones, up to rounding of the scanned iterate
    # (a few ulp of max|s| per step, accumulated along the chain)
    _check_history(hist, hist_or, max(1.0, float(np.abs(seq).max())))
    return it, s


def _check_history(hist, hist_or, scale):
    """Residual histories, fp32 against fp64, element by element (see HIST_RTOL / HIST_ATOL).  An
    iteration that passes through a large iterate (a residual far above max|s|: the Euler drift under
    quasi-Newton can reach 1e5 before it contracts) carries float32 rounding at that scale into every
    later iterate, so each later residual also gets an absolute allowance of 8 float32 ulps (2^-20)
    of the largest oracle residual so far."""
    n = min(len(hist), len(hist_or))
    h, ho = np.asarray(hist[:n], np.float64), np.asarray(hist_or[:n], np.float64)
    peak = np.maximum.accumulate(np.abs(ho)) if n else ho
    bound = HIST_ATOL * scale + 2.0 ** -20 * peak + HIST_RTOL * np.abs(ho)
    bad = np.nonzero(np.abs(h - ho) > bound)[0]
    assert bad.size == 0, [(int(i), float(h[i]), float(ho[i]), float(bound[i])) for i in bad[:5]]


CELLS = [pi.CELL_TANH_RNN, pi.CELL_GRU, pi.CELL_EULER]
DIAG_MODES = [pi.MODE_JACOBI, pi.MODE_PICARD, pi.MODE_QUASI]


@pytest.mark.parametrize("cell", CELLS)
@pytest.mark.parametrize("mode", DIAG_MODES + [pi.MODE_NEWTON])
@pytest.mark.parametrize("D,T,B", [(1, 5, 1), (3, 70, 2), (4, 300, 3), (7, 129, 2), (16, 517, 2),
                                   (33, 200, 2), (64, 133, 3)])
def test_small_shapes(cell, mode, D, T, B):
    if mode == pi.MODE_PICARD and cell != pi.CELL_EULER:
        # A~ = I is only a contraction for near-identity dynamics (page §2.2.3); on the RNN cells the
        # not-yet-converged tail grows geometrically until causality reaches it, so keep T short.
        T = min(T, 12)
    d_in = D if cell == pi.CELL_EULER else max(1, D - 1)
    prob = pi.random_problem(1000 + 7 * D + T, cell, D, d_in, T=T, B=B, rho=0.6, eps=0.05,
                             s0_scale=0.3, tol=1e-5)
    if mode == pi.MODE_JACOBI:
        prob.max_iters = T
    _check_against_oracle(prob, mode)


@pytest.mark.parametrize("tc", [1, 0])
@pytest.mark.parametrize("cell", CELLS)
@pytest.mark.parametrize("mode", DIAG_MODES)
@pytest.mark.parametrize("D,T,B", [(32, 300, 3), (32, 1000, 2), (64, 257, 2), (64, 2100, 3)])
def test_tensor_core_and_fp32_paths(tc, cell, mode, D, T, B):
    """D = 32 and 64 run the tensor-core matvec kernels by default (GRU: D = 32 only); both those
    and the FP32 kernels must match the oracle, across several 128-step tiles and a ragged tail."""
    if mode == pi.MODE_PICARD and cell != pi.CELL_EULER:
        T = 12
    prob = pi.random_problem(500 + D + T + cell, cell, D, D, T=T, B=B, rho=0.7, eps=0.05, s0_scale=0.3,
                             tol=1e-5)
    if mode == pi.MODE_JACOBI:
        prob.max_iters = T
    _check_against_oracle(prob, mode, tc=tc)


@pytest.mark.parametrize("cell", CELLS)
@pytest.mark.parametrize("mode", DIAG_MODES)
@pytest.mark.parametrize("D", [100, 256])
def test_wide_states(cell, mode, D):
    T = 12 if (mode == pi.MODE_PICARD and cell != pi.CELL_EULER) else 150
    prob = pi.random_problem(77 + D, cell, D, D, T=T, B=2, rho=0.6, eps=0.05, s0_scale=0.2, tol=1e-5)
    _check_against_oracle(prob, mode)


@pytest.mark.parametrize("cell,D,mode", [(pi.CELL_TANH_RNN, 64, pi.MODE_QUASI), (pi.CELL_TANH_RNN, 64, pi.MODE_JACOBI),
                                         (pi.CELL_GRU, 32, pi.MODE_QUASI), (pi.CELL_TANH_RNN, 16, pi.MODE_NEWTON)])
def test_looping_stop_rule_edges(cell, D, mode):
    """The looping kernels (channel-major, row-major and warp-per-chunk Newton) take the stop decision
    from the grid barrier's packed arrival count: tol = 0 runs exactly max_iters iterations and
    reports PN_NOT_CONVERGED with the oracle's iterate; a huge tol stops at iteration 0; a NaN in the
    input reports PN_ERR_NONFINITE, after which the handle evaluates normally."""
    import torch
    pn = _pn()
    prob = pi.random_problem(2301 + D + mode, cell, D, D, T=700, B=2, rho=0.6, eps=0.05, s0_scale=0.3,
                             tol=1e-5)
    it, s = _check_against_oracle(prob, mode, tol=0.0, max_iters=5)
    assert it == 5
    solver = pn.Solver.from_problem(prob)
    x = torch.from_numpy(prob.x).cuda()
    s0 = torch.from_numpy(prob.s0).cuda()
    _, it, _, st = solver.eval(x, s0, pi.MODE_NAMES[mode], 50, 1e9)
    assert (it, st) == (0, pn.PN_OK)
    bad = x.clone()
    bad[1, 300, 3] = float("nan")
    with pytest.raises(pn.PnError) as e:
        solver.eval(bad, s0, pi.MODE_NAMES[mode], 20, 1e-6)
    assert e.value.status == pn.PN_ERR_NONFINITE
    _, it, _, st = solver.eval(x, s0, pi.MODE_NAMES[mode], 3, 0.0)
    assert (it, st) == (3, pn.PN_NOT_CONVERGED)
    solver.close()


def test_picard_divergence_is_reported():
    """Picard on a tanh RNN far from the identity: the tail grows until it overflows; the loop must
    stop with PN_ERR_NONFINITE (or run out of iterations), never hang or return garbage as PN_OK."""
    import torch
    pn = _pn()
    prob = pi.random_problem(13, pi.CELL_TANH_RNN, 8, 8, T=600, B=2, rho=0.6, s0_scale=0.3)
    solver = pn.Solver.from_problem(prob)
    x = torch.from_numpy(prob.x).cuda()
    s0 = torch.from_numpy(prob.s0).cuda()
    try:
        _, it, r, st = solver.eval(x, s0, "picard", prob.T, 1e-6)
        assert st == pn.PN_NOT_CONVERGED or it > 100
    except pn.PnError as e:
        assert e.status == pn.PN_ERR_NONFINITE
    solver.close()


# The decoupled look-back combines a tile's carry from whichever predecessor state is published
# first, so two runs may associate the same fp32 products differently: results agree to rounding,
# not bit for bit.
RUN_TO_RUN = 1e-6


@pytest.mark.parametrize("cell,D,mode", [(pi.CELL_TANH_RNN, 16, pi.MODE_QUASI), (pi.CELL_TANH_RNN, 16, pi.MODE_NEWTON),
                                         (pi.CELL_TANH_RNN, 32, pi.MODE_QUASI), (pi.CELL_TANH_RNN, 64, pi.MODE_QUASI),
                                         (pi.CELL_EULER, 64, pi.MODE_QUASI), (pi.CELL_GRU, 32, pi.MODE_QUASI)])
def test_host_loop_matches_device_loop(cell, D, mode):
    """The host-driven loop (one launch per iteration, PN_OPT_DEVICE_LOOP = 0) and the device loop
    give the same count and the same states to rounding.  At D = 32 and 64 the one-gate cells' quasi
    mode runs the channel-major tensor-core kernel, which the device loop launches once for all
    iterations and the host loop once per iteration; both must also match the oracle."""
    prob = pi.random_problem(5, cell, D, D, T=700, B=3, rho=0.7, eps=0.05, s0_scale=0.3, tol=1e-6)
    a = _run(prob, mode, device_loop=1)
    b = _run(prob, mode, device_loop=0)
    if D >= 32:
        _check_against_oracle(prob, mode, device_loop=0)
    assert a[1] == b[1]
    scale = max(1.0, float(np.abs(a[0]).max()))
    np.testing.assert_allclose(a[0], b[0], rtol=0, atol=RUN_TO_RUN * scale)
    np.testing.assert_allclose(a[4], b[4], rtol=1e-3, atol=RUN_TO_RUN * scale)


def test_repeatable():
    prob = pi.random_problem(6, pi.CELL_GRU, 32, 32, T=1000, B=4, rho=0.9, tol=1e-6)
    a = _run(prob, pi.MODE_QUASI)
    b = _run(prob, pi.MODE_QUASI)
    scale = max(1.0, float(np.abs(a[0]).max()))
    np.testing.assert_allclose(a[0], b[0], rtol=0, atol=RUN_TO_RUN * scale)
    assert a[1] == b[1]


def test_edge_cases():
    import torch
    pn = _pn()
    prob = pi.random_problem(8, pi.CELL_TANH_RNN, 8, 5, T=100, B=2, rho=0.5, s0_scale=0.4)
    solver = pn.Solver.from_problem(prob)
    x = torch.from_numpy(prob.x).cuda()
    s0 = torch.from_numpy(prob.s0).cuda()
    m = oracle.Model.from_problem(prob)
    # max_iters = 0: states are s0 broadcast, resid is r^(0)
    states, it, r, st = solver.eval(x, s0, "quasi", 0, 1e-9)
    assert (it, st) == (0, pn.PN_NOT_CONVERGED)
    np.testing.assert_array_equal(states.cpu().numpy(), np.repeat(prob.s0[:, None, :], prob.T, 1))
    _, r0 = m.residual(prob.x, prob.s0, np.repeat(prob.s0[:, None, :], prob.T, 1))
    assert abs(r - r0) <= 1e-6 * max(1.0, r0)
    # huge tol: converged at iteration 0
    states, it, r, st = solver.eval(x, s0, "newton", 50, 1e9)
    assert (it, st) == (0, pn.PN_OK)
    # NaN input -> PN_ERR_NONFINITE, and the handle keeps working
    bad = x.clone()
    bad[1, 50, 2] = float("nan")
    with pytest.raises(pn.PnError) as e:
        solver.eval(bad, s0, "quasi", 20, 1e-6)
    assert e.value.status == pn.PN_ERR_NONFINITE
    states, it, r, st = solver.eval(x, s0, "quasi", prob.T, 1e-6)
    assert st == pn.PN_OK and np.isfinite(states.cpu().numpy()).all()
    # invalid arguments are rejected before any launch
    st2, _, _ = pn.pn_eval(solver.h, 0, s0.data_ptr(), pn.PN_QUASI, 5, 1e-5, states.data_ptr())
    assert st2 == pn.PN_ERR_INVALID
    host = np.zeros((prob.B, prob.T, prob.d_in), np.float32)
    st2, _, _ = pn.pn_eval(solver.h, host.ctypes.data, s0.data_ptr(), pn.PN_QUASI, 5, 1e-5, states.data_ptr())
    assert st2 == pn.PN_ERR_INVALID
    st2, _, _ = pn.pn_eval(solver.h, x.data_ptr(), s0.data_ptr(), 7, 5, 1e-5, states.data_ptr())
    assert st2 == pn.PN_ERR_INVALID
    st2, _, _ = pn.pn_eval(solver.h, x.data_ptr(), s0.data_ptr(), pn.PN_QUASI, -1, 1e-5, states.data_ptr())
    assert st2 == pn.PN_ERR_INVALID
    st2, _, _ = pn.pn_eval(solver.h, x.data_ptr() + 4, s0.data_ptr(), pn.PN_QUASI, 5, 1e-5, states.data_ptr())
    assert st2 == pn.PN_ERR_INVALID   # misaligned
    solver.close()


def test_newton_rejects_wide_state():
    import torch
    pn = _pn()
    prob = pi.random_problem(9, pi.CELL_EULER, 100, T=20, B=1)
    solver = pn.Solver.from_problem(prob)
    x = torch.from_numpy(prob.x).cuda()
    s0 = torch.from_numpy(prob.s0).cuda()
    with pytest.raises(pn.PnError) as e:
        solver.eval(x, s0, "newton", 5, 1e-5)
    assert e.value.status == pn.PN_ERR_INVALID
    solver.close()


def test_bounded_wait_times_out_and_recovers():
    """A tile that never publishes (test hook) makes its successor's bounded wait run out:
    the call returns PN_ERR_TIMEOUT and the context stays usable."""
    import torch
    pn = _pn()
    prob = pi.random_problem(10, pi.CELL_TANH_RNN, 64, 64, T=2000, B=2, rho=0.5)
    solver = pn.Solver.from_problem(prob)
    x = torch.from_numpy(prob.x).cuda()
    s0 = torch.from_numpy(prob.s0).cuda()
    solver.set_option(pn.PN_OPT_WAIT_TIMEOUT_NS, 20_000_000)   # 20 ms
    solver.set_option(pn.PN_OPT_DEBUG_STALL_TICKET, 0)
    for mode in ("quasi", "newton"):
        with pytest.raises(pn.PnError) as e:
            solver.eval(x, s0, mode, 10, 1e-6)
        assert e.value.status == pn.PN_ERR_TIMEOUT
    solver.set_option(pn.PN_OPT_DEBUG_STALL_TICKET, -1)
    states, it, r, st = solver.eval(x, s0, "quasi", prob.T, 1e-6)
    assert st == pn.PN_OK
    seq = oracle.Model.from_problem(prob).sequential(prob.x, prob.s0)
    assert _relerr(states.cpu().numpy(), seq) <= REL_TOL
    solver.close()


def test_eval_host_matches_eval():
    pn = _pn()
    prob = pi.random_problem(11, pi.CELL_GRU, 32, 32, T=900, B=3, rho=0.8, tol=1e-6)
    a = _run(prob, pi.MODE_QUASI)
    solver = pn.Solver.from_problem(prob)
    states, it, r, st = solver.eval_host(prob.x, prob.s0, "quasi", prob.T, prob.tol)
    solver.close()
    assert it == a[1]
    np.testing.assert_array_equal(states, a[0])


@pytest.mark.parametrize("cell,D,T,B", [(pi.CELL_TANH_RNN, 64, 4096, 4), (pi.CELL_GRU, 32, 900, 3)])
def test_eval_host_many_matches_eval_host(cell, D, T, B):
    """The pipelined host entry point gives every batch the result pn_eval_host gives it (to
    rounding: the look-back may fold in a different order), with the same iteration count."""
    pn = _pn()
    probs = [pi.random_problem(40 + j, cell, D, D, T=T, B=B, rho=0.7, tol=1e-5) for j in range(3)]
    solver = pn.Solver.from_problem(probs[0])   # the weights of batch 0; the other batches differ in x, s0
    xs = [np.ascontiguousarray(p.x) for p in probs]
    s0s = [np.ascontiguousarray(p.s0) for p in probs]
    outs, its, rs, st = solver.eval_host_many(xs, s0s, "quasi", T, 1e-5)
    assert st in (pn.PN_OK, pn.PN_NOT_CONVERGED)
    for j in range(3):
        ref, it, r, st1 = solver.eval_host(xs[j], s0s[j], "quasi", T, 1e-5)
        assert its[j] == it
        np.testing.assert_allclose(outs[j], ref, rtol=0, atol=1e-6 * max(1.0, float(np.abs(ref).max())))
    solver.close()


def test_stats_and_timing():
    import torch
    pn = _pn()
    prob = pi.random_problem(12, pi.CELL_TANH_RNN, 64, 64, T=4096, B=4, rho=0.7, tol=1e-5)
    solver = pn.Solver.from_problem(prob)
    x = torch.from_numpy(prob.x).cuda()
    s0 = torch.from_numpy(prob.s0).cuda()
    solver.reset_stats()
    _, it, _, _ = solver.eval(x, s0, "quasi", prob.T, prob.tol)
    s = solver.stats()
    assert s["iteration_launches"] == it + 1 and s["iteration_ns"] > 0 and s["evals"] == 1
    ms = solver.time_iterations("quasi", 5)
    assert 0.0 < ms < 1000.0
    solver.close()


@pytest.mark.parametrize("tc", [1, 0])
@pytest.mark.parametrize("cell", CELLS)
@pytest.mark.parametrize("D,T,B", [(24, 300, 3), (32, 517, 2), (48, 300, 2), (64, 700, 3)])
def test_newton_tensor_core_and_fp32_compositions(tc, cell, D, T, B):
    """Newton at D = 17..64: the one-gate cells compose the chunk aggregates on the tensor cores
    (3xTF32 tcgen05.mma, padded width 32 or 64) unless PN_OPT_TENSOR_CORES = 0; the GRU, and every
    cell with tc = 0, run the FP32 kernels (one warp per tile up to D = 32).  All must match the
    oracle's serial Newton iteration and the sequential states, over several 32-step chunks and a
    ragged tail."""
    d_in = D if cell == pi.CELL_EULER else D - 3
    prob = pi.random_problem(600 + D + T + cell, cell, D, d_in, T=T, B=B, rho=0.7, eps=0.05, s0_scale=0.3,
                             tol=1e-5)
    _check_against_oracle(prob, pi.MODE_NEWTON, tc=tc)


@pytest.mark.parametrize("tc", [1, 0])
@pytest.mark.parametrize("cell", [pi.CELL_TANH_RNN, pi.CELL_EULER])
@pytest.mark.parametrize("mode", DIAG_MODES)
@pytest.mark.parametrize("D,T,B", [(128, 300, 3), (256, 333, 3), (256, 64, 1)])
def test_wide_tensor_core_product(tc, cell, mode, D, T, B):
    """D = 128 and 256 (one-gate cells): each iteration first forms W s^(i)_r for every step on the
    tensor cores (3xTF32, 128-row tiles, the last one partial), then the diagonal kernel reads it; with
    tc = 0 the FP32 kernels form the product themselves.  Both must match the oracle."""
    if mode == pi.MODE_PICARD and cell != pi.CELL_EULER:
        T = 12
    prob = pi.random_problem(700 + D + T + cell, cell, D, D, T=T, B=B, rho=0.6, eps=0.05, s0_scale=0.2,
                             tol=1e-5)
    if mode == pi.MODE_JACOBI:
        prob.max_iters = T
    _check_against_oracle(prob, mode, tc=tc)


@pytest.mark.parametrize("cell,mode", [(pi.CELL_EULER, pi.MODE_PICARD), (pi.CELL_TANH_RNN, pi.MODE_QUASI)])
def test_wide_many_chunks(cell, mode):
    """D = 128 with 66 chunks of 32 steps per sequence (the last ragged): the per-channel kernel's fold
    of the tile aggregates per (sequence, channel group) runs in several batches of loads.  Twenty
    iterations with tol = 0 on both sides, states compared element by element: over 2100 steps the
    Euler states reach |s| ~ 100, where fp32 rounding of the scan moves the last residuals by tens
    of percent of a 1e-5 |s| tolerance, so a stop-rule comparison would test the rounding, not the
    kernel.  (Euler quasi-Newton passes through far larger unconverged iterates on the way, which
    puts its fp32 distance to the fp64 iterate above 1e-4 here; it is covered at T <= 333.)"""
    prob = pi.random_problem(2210 + cell + mode, cell, 128, 128, T=2100, B=2, rho=0.6, eps=0.05,
                             s0_scale=0.2, tol=1e-5)
    it, _ = _check_against_oracle(prob, mode, tol=0.0, max_iters=20, tc=1)
    assert it == 20


def test_wide_bounded_wait_times_out_and_recovers():
    """The wide per-channel kernel's test hook: the CTA holding tile 0 never arrives at the grid barrier
    after the aggregates, so every CTA's bounded wait there runs out; the call returns
    PN_ERR_TIMEOUT and the handle evaluates normally afterwards."""
    import torch
    pn = _pn()
    prob = pi.random_problem(2233, pi.CELL_EULER, 256, 256, T=333, B=2, rho=0.6, eps=0.05, s0_scale=0.2,
                             tol=1e-5)
    solver = pn.Solver.from_problem(prob)
    x = torch.from_numpy(prob.x).cuda()
    s0 = torch.from_numpy(prob.s0).cuda()
    solver.set_option(pn.PN_OPT_WAIT_TIMEOUT_NS, 20_000_000)   # 20 ms
    solver.set_option(pn.PN_OPT_DEBUG_STALL_TICKET, 0)
    with pytest.raises(pn.PnError) as e:
        solver.eval(x, s0, "picard", 10, 1e-6)
    assert e.value.status == pn.PN_ERR_TIMEOUT
    solver.set_option(pn.PN_OPT_DEBUG_STALL_TICKET, -1)
    m = oracle.Model.from_problem(prob)
    seq = m.sequential(prob.x, prob.s0)
    tol = prob.tol * max(1.0, float(np.abs(seq).max()))
    states, it, r, st = solver.eval(x, s0, "picard", prob.T, tol)
    assert st == pn.PN_OK
    assert _relerr(states.cpu().numpy(), seq) <= REL_TOL
    solver.close()


@pytest.mark.parametrize("tc", [0, 1])
@pytest.mark.parametrize("device_loop", [1, 0])
@pytest.mark.parametrize("run", [1, 3, 0])
@pytest.mark.parametrize("cell,D", [(pi.CELL_TANH_RNN, 16), (pi.CELL_GRU, 8), (pi.CELL_EULER, 4),
                                    (pi.CELL_TANH_RNN, 32), (pi.CELL_TANH_RNN, 12), (pi.CELL_EULER, 13),
                                    (pi.CELL_GRU, 16)])
def test_newton_run_lengths(run, cell, D, device_loop, tc):
    """The Newton kernel at D <= 32 gives a ticket a run of consecutive 32-step chunks (one
    aggregate per run; the cell phase evaluated again in the write-out pass when the run is longer
    than one): one chunk, three (the last run ragged) and the automatic length all match the oracle,
    looping in one launch or launched per iteration.  At padded width 16 the one-gate cells run the
    chunk chain on the tensor cores (D = 12, 13, 16: padded channels included) unless
    PN_OPT_TENSOR_CORES = 0, the GRU always on the FMA pipe."""
    T, B = 1000, 3   # 32 chunks, the last one ragged
    d_in = D if cell == pi.CELL_EULER else D - 1
    prob = pi.random_problem(1700 + 5 * D + cell, cell, D, d_in, T=T, B=B, rho=0.6, eps=0.05,
                             s0_scale=0.3, tol=1e-5)
    _check_against_oracle(prob, pi.MODE_NEWTON, device_loop=device_loop, tc=tc,
                          opts={"PN_OPT_RUN_LENGTH": run})


def test_run_length_change_regrows_lookback():
    """More chunks per sequence than the automatic tiling gives tickets (D = 16: 2 x 148 x 7 warps
    take tickets, here 8 x 300 chunks): the automatic run length is 2, so run length 1 needs twice
    the look-back buffers create allocated; the handle must grow them, and every setting, switched
    on one handle, still matches the oracle."""
    import torch
    pn = _pn()
    prob = pi.random_problem(1811, pi.CELL_TANH_RNN, 16, 15, T=9600, B=8, rho=0.6, s0_scale=0.3, tol=1e-5)
    m = oracle.Model.from_problem(prob)
    seq = m.sequential(prob.x, prob.s0)
    tol = prob.tol * max(1.0, float(np.abs(seq).max()))
    s_or, it_or, _, st_or, hist_or = m.iterate(pi.MODE_NEWTON, prob.x, prob.s0, prob.T, tol)
    exact = float(np.min(np.abs(hist_or / tol - 1.0))) > 1e-2   # no residual within 1% of tol
    solver = pn.Solver.from_problem(prob)
    solver.set_option(pn.PN_OPT_TENSOR_CORES, 0)
    x = torch.from_numpy(prob.x).cuda()
    s0 = torch.from_numpy(prob.s0).cuda()
    for run in (0, 1, 3, 0, 1):
        solver.set_option(pn.PN_OPT_RUN_LENGTH, run)
        states, it, r, st = solver.eval(x, s0, "newton", prob.T, tol)
        assert (it, st) == (it_or, st_or) if exact else abs(it - it_or) <= 1, (run, it, it_or)
        if it == it_or:
            assert _relerr(states.cpu().numpy(), s_or) <= REL_TOL, run
    with pytest.raises(pn.PnError):
        solver.set_option(pn.PN_OPT_RUN_LENGTH, -1)
    solver.close()


@pytest.mark.parametrize("small", [1, 0])
@pytest.mark.parametrize("cell", CELLS)
@pytest.mark.parametrize("D,T,B", [(4, 1024, 1), (8, 200, 3), (3, 77, 2), (1, 33, 1), (5, 64, 4)])
def test_newton_single_cta_solve(small, cell, D, T, B):
    """Newton on problems that fit one SM's shared memory: the single-CTA solve (projection, every
    iteration and the stop rule in one launch) and the multi-CTA kernel both match the oracle,
    across whole and ragged 32-step chunks."""
    pn = _pn()
    d_in = D if cell == pi.CELL_EULER else max(1, D - 1)
    prob = pi.random_problem(1900 + 3 * D + T + cell, cell, D, d_in, T=T, B=B, rho=0.6, eps=0.05,
                             s0_scale=0.3, tol=1e-5)
    solver = pn.Solver.from_problem(prob)
    solver.set_option(pn.PN_OPT_SMALL_SOLVE, small)
    assert pn.pn_dim(solver.h, 5 + pi.MODE_NEWTON) == (2 if small else 1)
    solver.close()
    _check_against_oracle(prob, pi.MODE_NEWTON, opts={"PN_OPT_SMALL_SOLVE": small})


def test_newton_single_cta_limits_and_timing():
    """A problem too large for one SM's shared memory runs the multi-CTA kernel; the timing hook
    times the single-CTA solve as one launch of n residual evaluations."""
    import torch
    pn = _pn()
    big = pi.random_problem(1931, pi.CELL_TANH_RNN, 8, 7, T=4096, B=2, rho=0.6, s0_scale=0.3)
    sb = pn.Solver.from_problem(big)
    assert pn.pn_dim(sb.h, 5 + pi.MODE_NEWTON) == 1
    sb.close()
    prob = pi.random_problem(1932, pi.CELL_TANH_RNN, 4, 4, T=1024, B=1, rho=0.5, s0_scale=0.3)
    solver = pn.Solver.from_problem(prob)
    assert pn.pn_dim(solver.h, 5 + pi.MODE_NEWTON) == 2
    x = torch.from_numpy(prob.x).cuda()
    s0 = torch.from_numpy(prob.s0).cuda()
    solver.eval(x, s0, "newton", prob.T, 1e-6)
    ms = solver.time_iterations("newton", 5)
    assert 0.0 < ms < 10.0
    with pytest.raises(pn.PnError):
        solver.set_option(pn.PN_OPT_SMALL_SOLVE, 2)
    solver.close()
