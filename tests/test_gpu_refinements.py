"""GPU parity of the refinements of the iteration (web article "并行牛顿方法：加速非
线性序列评估的计算革命"):
- the banded Jacobian approximation of §2.2.2 (PN_NEWTON with PN_OPT_NEWTON_BAND
  = k keeps the entries of df_t/ds with |row - col| <= k; k = 0 is the diagonal
  approximation, k >= D - 1 the exact Jacobian);
- damping, §4.3 and §5.3 (pn_set_damping: s^(i+1) = s^(i) + lambda * delta);
- adaptive switching on a residual stall, §5.3 (pn_set_adaptive).
The oracle's orc_iterate_ex with the same settings is the reference: iteration
counts (and modes) equal unless an oracle residual lies within 1% of tol or a
residual ratio within 2% of the stall threshold; states within 1e-4 normwise of
the oracle's iterate and of the sequential states."""
import numpy as np
import pytest

import oracle
import pn_inputs as pi
from test_gpu_parity import _check_history

pytestmark = pytest.mark.gpu

REL_TOL = 1e-4
CELLS = [pi.CELL_TANH_RNN, pi.CELL_GRU, pi.CELL_EULER]


def _relerr(a, ref):
    den = max(float(np.abs(ref).max()), 1e-30)
    return float(np.abs(a.astype(np.float64) - ref).max()) / den


def _run(prob, band, tol, max_iters, damping=1.0, mode="newton", tc=1, small=1):
    import torch
    import newton_evaluation_nonlinear_b200 as pn
    solver = pn.Solver.from_problem(prob)
    solver.set_option(pn.PN_OPT_SMALL_SOLVE, small)
    solver.set_option(pn.PN_OPT_NEWTON_BAND, band)
    solver.set_option(pn.PN_OPT_TENSOR_CORES, tc)
    solver.set_damping(damping)
    x = torch.from_numpy(prob.x).cuda()
    s0 = torch.from_numpy(prob.s0).cuda()
    states, it, r, st = solver.eval(x, s0, mode, max_iters, tol)
    hist = solver.residual_history()
    out = states.cpu().numpy()
    solver.close()
    return out, it, r, st, hist


def _check(cell, D, T, B, band, damping, seed, mode="newton", tc=1, small=1):
    d_in = D if cell == pi.CELL_EULER else D - 1
    prob = pi.random_problem(seed, cell, D, d_in, T=T, B=B, rho=0.7, s0_scale=0.3, eps=0.05)
    m = oracle.Model.from_problem(prob)
    seq = m.sequential(prob.x, prob.s0)
    tol = 1e-5 * max(1.0, float(np.abs(seq).max()))
    if mode == "newton":
        mode_or, band_or = (pi.MODE_NEWTON, 0) if band < 0 else (oracle.BANDED, band)
    else:
        mode_or, band_or = pi.MODE_BY_NAME[mode], 0
    lam = float(np.float32(damping))           # the library holds lambda in float32
    s_or, it_or, r_or, st_or, hist_or, _, _ = m.iterate_ex(mode_or, prob.x, prob.s0, T, tol, band=band_or,
                                                           damping=lam)
    s, it, r, st, hist = _run(prob, band, tol, T, damping, mode, tc, small)
    assert np.isfinite(s).all()
    margin = float(np.min(np.abs(hist_or / tol - 1.0)))
    if margin > 1e-2:
        assert (it, st) == (it_or, st_or), (it, it_or, hist[:it + 1], hist_or)
    else:
        assert abs(it - it_or) <= 1
    if it == it_or:
        assert _relerr(s, s_or) <= REL_TOL, _relerr(s, s_or)
    if st == oracle.OK:
        assert _relerr(s, seq) <= max(REL_TOL, 2.0 * _relerr(s_or, seq))
    _check_history(hist, hist_or, max(1.0, float(np.abs(seq).max())))


@pytest.mark.parametrize("cell", CELLS)
@pytest.mark.parametrize("D,T,B,small", [(8, 300, 2, 1), (8, 300, 2, 0), (16, 517, 3, 1)])
@pytest.mark.parametrize("band", [0, 1, 3, -1])
def test_banded_newton_matches_oracle(cell, D, T, B, small, band):
    """D = 8 fits the single-CTA solve (small = 1) and runs the multi-CTA warp-per-chunk kernel too."""
    _check(cell, D, T, B, band, 1.0, 301 + cell + D + band, small=small)


@pytest.mark.parametrize("cell", CELLS)
@pytest.mark.parametrize("band", [0, 2])
def test_banded_newton_fma_chain(cell, band):
    """At D = 16 the one-gate cells' banded chain runs on the tensor cores with the band-masked W
    (the case above); PN_OPT_TENSOR_CORES = 0 runs it on the FMA pipe over the band's columns only."""
    _check(cell, 16, 517, 3, band, 1.0, 311 + cell + band, tc=0)


@pytest.mark.parametrize("cell", CELLS)
@pytest.mark.parametrize("band,damping", [(-1, 0.5), (-1, 0.8), (2, 0.7)])
@pytest.mark.parametrize("D,T", [(12, 400), (6, 300)])
def test_damped_newton_matches_oracle(cell, band, damping, D, T):
    """D = 6 runs the single-CTA solve, D = 12 the multi-CTA kernel."""
    _check(cell, D, T, 2, band, damping, 321 + cell + D)


@pytest.mark.parametrize("cell", CELLS)
@pytest.mark.parametrize("mode", ["jacobi", "picard", "quasi"])
@pytest.mark.parametrize("D,tc", [(16, 1), (64, 1), (64, 0)])
def test_damped_diagonal_modes_match_oracle(cell, mode, D, tc):
    """Damping in the diagonal modes: at D = 64 the one-gate cells' quasi-Newton runs the channel-major
    tensor-core kernel (lambda folded into the parked prefixes), Jacobi the row-major one, damped
    Picard and the GRU the FP32 kernels; tc = 0 runs the FP32 kernels throughout."""
    T = 12 if (mode == "picard" and cell != pi.CELL_EULER) else (300 if D == 64 else 400)
    _check(cell, D, T, 2, -1, 0.7, 371 + cell + D, mode=mode, tc=tc)


@pytest.mark.parametrize("cell", [pi.CELL_TANH_RNN, pi.CELL_EULER])
@pytest.mark.parametrize("mode", ["jacobi", "picard", "quasi"])
def test_damped_wide_modes_match_oracle(cell, mode):
    """Damping on the wide path (D = 256: the tensor-core product, then the per-channel kernel's three
    phases): the damped states come out of the last phase, which for Euler Picard then loads s^(i)
    again (undamped it does not need it)."""
    T = 12 if (mode == "picard" and cell != pi.CELL_EULER) else 300
    _check(cell, 256, T, 2, -1, 0.7, 391 + cell, mode=mode, tc=1)


def test_damping_arguments_and_switching():
    """Damping toggles the kernel choice of Picard (tensor-core row-major kernel undamped, FP32 kernel
    damped) and back; the Euler drift keeps Picard contractive over the whole sequence."""
    import torch
    import newton_evaluation_nonlinear_b200 as pn
    prob = pi.random_problem(331, pi.CELL_EULER, 64, 64, T=300, B=1, rho=0.5, eps=0.05)
    solver = pn.Solver.from_problem(prob)
    for bad in (0.0, -0.5, 1.5, float("nan")):
        with pytest.raises(pn.PnError):
            solver.set_damping(bad)
    x = torch.from_numpy(prob.x).cuda()
    s0 = torch.from_numpy(prob.s0).cuda()
    ref = {m: solver.eval(x, s0, m, 300, 1e-5)[0].cpu().numpy() for m in ("picard", "quasi")}
    solver.set_damping(0.5)
    for m in ("jacobi", "picard", "quasi", "newton"):
        states, it, r, st = solver.eval(x, s0, m, 300, 1e-5)
        assert st in (pn.PN_OK, pn.PN_NOT_CONVERGED)
    solver.set_damping(1.0)   # back to the undamped kernels: the same result as before
    for m in ("picard", "quasi"):
        states, it, r, st = solver.eval(x, s0, m, 300, 1e-5)
        ref_m = ref[m]
        np.testing.assert_allclose(states.cpu().numpy(), ref_m, rtol=0, atol=1e-6 * max(1.0, float(np.abs(ref_m).max())))
    solver.close()


def test_band_option_bounds():
    import newton_evaluation_nonlinear_b200 as pn
    prob = pi.random_problem(311, pi.CELL_TANH_RNN, 8, 8, T=40, B=1, rho=0.5)
    solver = pn.Solver.from_problem(prob)
    with pytest.raises(pn.PnError):
        solver.set_option(pn.PN_OPT_NEWTON_BAND, -2)
    solver.set_option(pn.PN_OPT_NEWTON_BAND, 1000)      # beyond D - 1: the exact Jacobian
    solver.close()


# ----------------------------------------------------------------------------
# adaptive switching (§5.3): jacobi/picard -> quasi -> newton on a stall
# ----------------------------------------------------------------------------

def _check_adaptive(cell, start, stall, D, T, B, seed, device_loop=1):
    import torch
    import newton_evaluation_nonlinear_b200 as pn
    d_in = D if cell == pi.CELL_EULER else D - 1
    prob = pi.random_problem(seed, cell, D, d_in, T=T, B=B, rho=0.8, s0_scale=0.3, eps=0.05)
    m = oracle.Model.from_problem(prob)
    seq = m.sequential(prob.x, prob.s0)
    tol = 1e-5 * max(1.0, float(np.abs(seq).max()))
    theta = float(np.float32(stall))
    mode = pn.MODES[start]
    s_or, it_or, r_or, st_or, hist_or, modes_or, _ = m.iterate_ex(mode, prob.x, prob.s0, T, tol, adapt=True,
                                                                  stall=theta)
    solver = pn.Solver.from_problem(prob)
    solver.set_adaptive(theta)
    solver.set_option(pn.PN_OPT_DEVICE_LOOP, device_loop)
    x = torch.from_numpy(prob.x).cuda()
    s0 = torch.from_numpy(prob.s0).cuda()
    states, it, r, st = solver.eval(x, s0, start, T, tol)
    modes = solver.mode_history()
    s = states.cpu().numpy()
    solver.close()
    assert np.isfinite(s).all() and len(modes) == it
    ratios = hist_or[1:] / hist_or[:-1]
    clear = (float(np.min(np.abs(hist_or / tol - 1.0))) > 1e-2 and
             (len(ratios) == 0 or float(np.min(np.abs(ratios / theta - 1.0))) > 2e-2))
    if clear:
        assert (it, st) == (it_or, st_or), (it, it_or)
        assert modes.tolist() == modes_or[:-1].tolist(), (modes, modes_or)
        assert _relerr(s, s_or) <= REL_TOL, _relerr(s, s_or)
    if st == oracle.OK:
        assert _relerr(s, seq) <= max(REL_TOL, 2.0 * _relerr(s_or, seq))


@pytest.mark.parametrize("device_loop", [1, 0])
@pytest.mark.parametrize("cell", CELLS)
@pytest.mark.parametrize("start", ["jacobi", "picard", "quasi"])
@pytest.mark.parametrize("stall", [0.5, 0.9])
def test_adaptive_matches_oracle(cell, start, stall, device_loop):
    """device_loop = 1: the switching rule runs on the device (an IF node per mode inside the
    graph's WHILE node, set by the last CTA of each iteration); 0: the host loop applies it."""
    _check_adaptive(cell, start, stall, 16, 400, 2, 341 + cell, device_loop)


@pytest.mark.parametrize("device_loop", [1, 0])
@pytest.mark.parametrize("cell", [pi.CELL_TANH_RNN, pi.CELL_EULER])
@pytest.mark.parametrize("start", ["jacobi", "picard", "quasi"])
def test_adaptive_wide_matches_oracle(cell, start, device_loop):
    """D = 64: the one-gate cells' quasi-Newton updates run on the channel-major tensor-core kernel
    (one launch per iteration in the adaptive loop), Jacobi and Picard on the row-major one, Newton
    on the dense kernel; the switches and the result must match the oracle's."""
    _check_adaptive(cell, start, 0.9, 64, 600, 2, 361 + cell, device_loop)


def test_adaptive_off_leaves_no_mode_history():
    import torch
    import newton_evaluation_nonlinear_b200 as pn
    prob = pi.random_problem(351, pi.CELL_TANH_RNN, 8, 8, T=60, B=1, rho=0.5)
    solver = pn.Solver.from_problem(prob)
    with pytest.raises(pn.PnError):
        solver.set_adaptive(float("nan"))
    x = torch.from_numpy(prob.x).cuda()
    s0 = torch.from_numpy(prob.s0).cuda()
    solver.set_adaptive(-1.0)
    states, it, r, st = solver.eval(x, s0, "quasi", 60, 1e-5)
    assert st == pn.PN_OK and len(solver.mode_history()) == 0
    solver.close()


# ----------------------------------------------------------------------------
# reduced-precision iterate storage (page §2.3, §4.2-4.3)
# ----------------------------------------------------------------------------
# The GPU rounds its float32 iterate to the 16-bit format, the oracle its float64 one: where a value
# lies within float32 rounding of a 16-bit rounding boundary (about 1e-6 relative, so roughly one
# element in 2^-8 / 2e-6 ~ 2000 for bfloat16) the two round to neighbouring 16-bit values.  Such an
# element moves later residuals by at most one 16-bit unit, which the float32 iterations that follow
# contract, but near tol it can move the count by one.  The checks below are exact where rounding
# allows it (representability, the result copy) and carry that allowance where it does not.

STORE_FMT = {"bf16": (oracle.STORE_BF16, 1, 2.0 ** -8), "f16": (oracle.STORE_F16, 2, 2.0 ** -11)}


def _run_storage(prob, mode, fmt, store_until, max_iters, tol):
    import torch
    import newton_evaluation_nonlinear_b200 as pn
    solver = pn.Solver.from_problem(prob)
    solver.set_storage(STORE_FMT[fmt][1], store_until)
    x = torch.from_numpy(prob.x).cuda()
    s0 = torch.from_numpy(prob.s0).cuda()
    states, it, r, st = solver.eval(x, s0, mode, max_iters, tol)
    hist = solver.residual_history()
    out = states.cpu().numpy()
    solver.set_storage(pn.PN_STORE_F32, 0.0)
    ref, it32, _, _ = solver.eval(x, s0, mode, max_iters, tol)
    solver.close()
    return out, it, r, st, hist


@pytest.mark.parametrize("fmt", ["bf16", "f16"])
@pytest.mark.parametrize("max_iters", [1, 2, 3])
def test_narrow_iterates_are_representable(fmt, max_iters):
    """Stopped while still narrow (tol 0; store_until 0, so every residual is above it), the returned
    s^(max_iters) is exactly representable in the format (the result copy widens it exactly, from
    either iterate buffer), and matches the oracle's narrow iterate element by element up to the
    double-rounding cases.  After one iteration a flip stays in its own element; from the second on,
    a flip in s^(i-1)_{t-1,j} reaches every channel of step t through W and the later steps through
    the scan, so there the bound is a few units of the format relative to the largest state."""
    store, _, unit = STORE_FMT[fmt]
    prob = pi.random_problem(381, pi.CELL_TANH_RNN, 16, 15, T=300, B=2, rho=0.7, s0_scale=0.3)
    s, it, r, st, hist = _run_storage(prob, "quasi", fmt, 0.0, max_iters, 0.0)
    assert (it, st) == (max_iters, oracle.NOT_CONVERGED)
    np.testing.assert_array_equal(oracle.round_storage(s.astype(np.float64), store), s.astype(np.float64))
    m = oracle.Model.from_problem(prob)
    s_or, it_or, *_ = m.iterate_ex(pi.MODE_QUASI, prob.x, prob.s0, max_iters, 0.0, store=store, store_until=0.0)
    diff = np.abs(s.astype(np.float64) - s_or)
    if max_iters == 1:
        rel_unit = unit * np.maximum(np.abs(s_or), 1e-30)
        assert np.mean(diff > 0) < 1e-2                  # rare double-rounding flips ...
        assert np.all(diff <= 2.0 * rel_unit + 1e-7), float(np.max(diff / (rel_unit + 1e-30)))   # ... of one unit
    else:
        scale = float(np.abs(s_or).max())
        assert np.max(diff) <= 8.0 * unit * scale, float(np.max(diff) / (unit * scale))


@pytest.mark.parametrize("cell", CELLS)
@pytest.mark.parametrize("mode", ["jacobi", "picard", "quasi", "newton"])
@pytest.mark.parametrize("fmt,store_until", [("bf16", 3e-2), ("f16", 3e-3)])
def test_narrow_storage_matches_oracle(cell, mode, fmt, store_until):
    store, _, unit = STORE_FMT[fmt]
    D = 16
    T = 12 if (mode == "picard" and cell != pi.CELL_EULER) else 400
    d_in = D if cell == pi.CELL_EULER else D - 1
    prob = pi.random_problem(391 + cell, cell, D, d_in, T=T, B=2, rho=0.7, s0_scale=0.3, eps=0.05)
    m = oracle.Model.from_problem(prob)
    seq = m.sequential(prob.x, prob.s0)
    scale = max(1.0, float(np.abs(seq).max()))
    tol = 1e-5 * scale
    mo = pi.MODE_BY_NAME[mode]
    s_or, it_or, r_or, st_or, hist_or, _, _ = m.iterate_ex(mo, prob.x, prob.s0, T, tol, store=store,
                                                           store_until=store_until * scale)
    s, it, r, st, hist = _run_storage(prob, mode, fmt, store_until * scale, T, tol)
    assert np.isfinite(s).all()
    assert st == st_or
    assert abs(it - it_or) <= 1, (it, it_or, hist.tolist(), hist_or.tolist())
    if st == oracle.OK:
        assert _relerr(s, seq) <= max(REL_TOL, 2.0 * _relerr(s_or, seq)), (_relerr(s, seq), _relerr(s_or, seq))
        if it == it_or:
            assert _relerr(s, s_or) <= REL_TOL, _relerr(s, s_or)
    # residuals: within a few units of the format's resolution of the oracle's
    n = min(len(hist), len(hist_or))
    np.testing.assert_allclose(hist[:n], hist_or[:n], rtol=1e-2, atol=8 * unit * scale)


def test_storage_arguments():
    import newton_evaluation_nonlinear_b200 as pn
    prob = pi.random_problem(399, pi.CELL_TANH_RNN, 8, 8, T=40, B=1, rho=0.5)
    solver = pn.Solver.from_problem(prob)
    with pytest.raises(pn.PnError):
        solver.set_storage(7, 1e-2)
    with pytest.raises(pn.PnError):
        solver.set_storage(pn.PN_STORE_BF16, float("nan"))
    solver.set_storage(pn.PN_STORE_F16, 1e-3)
    solver.set_storage(pn.PN_STORE_F32, 0.0)
    solver.close()


@pytest.mark.parametrize("cell", CELLS)
@pytest.mark.parametrize("fmt,store_until", [("bf16", 3e-2), ("f16", 3e-3)])
@pytest.mark.parametrize("small", [1, 0])
def test_narrow_storage_newton_small_problem(cell, fmt, store_until, small):
    """Narrow iterate storage in Newton mode at D = 6: the single-CTA solve rounds the iterate it
    keeps in shared memory, the multi-CTA kernel its global buffers; both follow the oracle's rule."""
    import newton_evaluation_nonlinear_b200 as pn
    store, _, unit = STORE_FMT[fmt]
    D, T = 6, 300
    d_in = D if cell == pi.CELL_EULER else D - 1
    prob = pi.random_problem(397 + cell, cell, D, d_in, T=T, B=2, rho=0.7, s0_scale=0.3, eps=0.05)
    m = oracle.Model.from_problem(prob)
    seq = m.sequential(prob.x, prob.s0)
    scale = max(1.0, float(np.abs(seq).max()))
    tol = 1e-5 * scale
    s_or, it_or, r_or, st_or, hist_or, _, _ = m.iterate_ex(pi.MODE_NEWTON, prob.x, prob.s0, T, tol, store=store,
                                                           store_until=store_until * scale)
    import torch
    solver = pn.Solver.from_problem(prob)
    solver.set_option(pn.PN_OPT_SMALL_SOLVE, small)
    assert pn.pn_dim(solver.h, 5 + pi.MODE_NEWTON) == (2 if small else 1)
    solver.set_storage(STORE_FMT[fmt][1], store_until * scale)
    x = torch.from_numpy(prob.x).cuda()
    s0 = torch.from_numpy(prob.s0).cuda()
    states, it, r, st = solver.eval(x, s0, "newton", T, tol)
    hist = solver.residual_history()
    s = states.cpu().numpy()
    solver.close()
    assert st == st_or
    assert abs(it - it_or) <= 1, (it, it_or, hist.tolist(), hist_or.tolist())
    if st == oracle.OK:
        assert _relerr(s, seq) <= max(REL_TOL, 2.0 * _relerr(s_or, seq))
    n = min(len(hist), len(hist_or))
    np.testing.assert_allclose(hist[:n], hist_or[:n], rtol=1e-2, atol=8 * unit * scale)
