"""CPU checks of the seeded input generator: the five workloads have the shapes,
dtypes, settings and weight statistics their recipe states, are reproducible,
shrink to prefixes of the full draw, and still match the fingerprints the
stored oracle results were computed from."""
import json
import os

import numpy as np
import pytest

import pn_inputs as pi

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden", "workloads_oracle.json")

# index -> (cell, B, T, D, d_in, modes, tol, max_iters)
RECIPE = {
    0: (pi.CELL_TANH_RNN, 1, 1024, 4, 4, (pi.MODE_NEWTON,), 1e-6, None),
    1: (pi.CELL_TANH_RNN, 16, 16384, 64, 64, (pi.MODE_QUASI,), 1e-5, None),
    2: (pi.CELL_TANH_RNN, 64, 8192, 16, 16, (pi.MODE_NEWTON,), 1e-5, None),
    3: (pi.CELL_GRU, 8, 65536, 32, 32, (pi.MODE_QUASI,), 1e-5, 256),
    4: (pi.CELL_EULER, 32, 1024, 256, 256, (pi.MODE_PICARD, pi.MODE_JACOBI, pi.MODE_QUASI), 1e-5, None),
}
RHO = {0: 0.5, 1: 0.7, 2: 0.6}   # spectral radius of the tanh RNN recurrent matrix


def _radius(W):
    return float(np.max(np.abs(np.linalg.eigvals(W.astype(np.float64)))))


@pytest.mark.parametrize("index", sorted(RECIPE))
def test_workload_recipe(index):
    cell, B, T, D, d_in, modes, tol, max_iters = RECIPE[index]
    p = pi.benchmark_workload(index, T=64, B=2)   # parameters are drawn as for the full size
    assert (p.cell, p.D, p.d_in, p.modes, p.tol, p.max_iters) == (cell, D, d_in, modes, tol, max_iters)
    assert p.params.dtype == np.float32 and p.x.dtype == np.float32 and p.s0.dtype == np.float32
    assert p.params.size == pi.param_count(cell, D, d_in)
    assert p.x.shape == (min(2, B), 64, d_in) and p.s0.shape == (min(2, B), D)
    assert not np.any(p.s0)
    if cell == pi.CELL_TANH_RNN:
        W = p.params[:D * D].reshape(D, D)
        b = p.params[D * D + D * d_in:]
        assert abs(_radius(W) - RHO[index]) < 1e-5 * RHO[index] + 1e-6
        assert not np.any(b)
    elif cell == pi.CELL_GRU:
        W_hh = p.params[3 * D * d_in:3 * D * d_in + 3 * D * D].reshape(3 * D, D)
        for g in range(3):
            assert abs(_radius(W_hh[g * D:(g + 1) * D]) - 0.95) < 1e-5
        a = 1.0 / np.sqrt(32.0)
        W_ih = p.params[:3 * D * d_in]
        assert np.all(np.abs(W_ih) <= a + 1e-7)
    else:
        W = p.params.reshape(D, D)
        assert abs(float(W.std()) - 1.0 / 16.0) < 0.002 and abs(float(W.mean())) < 0.002
        assert p.eps == 1e-2


def test_reproducible_and_prefix():
    a = pi.benchmark_workload(1, T=96, B=3)
    b = pi.benchmark_workload(1, T=96, B=3)
    assert a.fingerprint() == b.fingerprint()
    small = pi.benchmark_workload(1, T=40, B=2)
    np.testing.assert_array_equal(small.params, a.params)
    np.testing.assert_array_equal(small.x, a.x[:2, :40])
    assert pi.benchmark_workload(2, T=40, B=2).fingerprint() != small.fingerprint()


@pytest.mark.parametrize("index", sorted(RECIPE))
def test_full_workloads_match_stored_fingerprints(index):
    """The stored oracle results belong to exactly these inputs (generator drift would void them)."""
    stored = json.load(open(GOLDEN))[str(index)]
    p = pi.benchmark_workload(index)
    assert (p.B, p.T, p.D, p.d_in) == (stored["B"], stored["T"], stored["D"], stored["d_in"])
    assert p.fingerprint() == stored["fingerprint"]


def test_stored_oracle_results_regenerate():
    """The stored oracle results are the oracle's: workload 0 (small enough to rerun here)
    gives the same count, status and residual history again."""
    import oracle
    stored = json.load(open(GOLDEN))["0"]["modes_result"]["newton"]
    p = pi.benchmark_workload(0)
    _, it, r, st, hist = oracle.Model.from_problem(p).iterate(pi.MODE_NEWTON, p.x, p.s0, p.iters_cap, p.tol)
    assert (int(it), int(st)) == (stored["iters"], stored["status"])
    np.testing.assert_allclose(np.asarray(hist, np.float64), np.asarray(stored["history"]), rtol=1e-12, atol=0)
    assert abs(float(r) - stored["resid"]) <= 1e-12 * abs(stored["resid"])
