"""GPU parity at the benchmark workloads' full sizes, in the benchmark's launch configuration.

Every sequence of every workload is compared element by element with the
oracle, on the same seeded inputs:
- with the oracle's sequential states s_t = f_t(s_{t-1}) (the result the
  iteration must reach, "Parallel Newton methods..." page §1.1 and §3.1), to a
  normwise relative error of 1e-4 over the whole batch and within each
  sequence;
- with the oracle's serial iteration in the same mode (the same iterate
  s^(iters)), to 1e-4 normwise over the batch and within each sequence, so a
  wrong carry into any one sequence fails even where it is small against the
  batch maximum.
The oracle runs here at full size (seconds on a 16-core host).  The Jacobi run
of the Euler workload takes T iterations, after which the iterate IS the
sequential result (causality, page §3.1), so the sequential states stand in for
the oracle's 1024 serial Jacobi sweeps.  The iteration counts must equal those
stored in tests/golden/workloads_oracle.json (written by
make_workload_golden.py, which calls only the oracle), which this test also
re-derives from the oracle run.
"""
import functools
import json
import os

import numpy as np
import pytest

import oracle
import pn_inputs as pi

pytestmark = pytest.mark.gpu

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden", "workloads_oracle.json")
REL_TOL = 1e-4


def _golden():
    with open(GOLDEN) as f:
        return json.load(f)


@functools.lru_cache(maxsize=None)
def _problem(idx):
    return pi.benchmark_workload(idx)


@functools.lru_cache(maxsize=None)
def _sequential(idx):
    prob = _problem(idx)
    return oracle.Model.from_problem(prob).sequential(prob.x, prob.s0)


def _oracle_iterate(idx, mode, ref):
    """The oracle's same-mode iterate s^(iters) at full size."""
    prob = _problem(idx)
    if mode == pi.MODE_JACOBI and ref["iters"] >= prob.T:
        return _sequential(idx), ref["iters"]          # causality: T Jacobi sweeps give s exactly
    s, it, r, st, hist = oracle.Model.from_problem(prob).iterate(mode, prob.x, prob.s0, prob.iters_cap, prob.tol)
    return s, it


def _per_sequence_relerr(a, ref):
    """max over b of  max|a[b] - ref[b]| / max|ref[b]|."""
    d = np.abs(a.astype(np.float64) - ref).reshape(ref.shape[0], -1).max(axis=1)
    n = np.maximum(np.abs(ref).reshape(ref.shape[0], -1).max(axis=1), 1e-30)
    return d / n


def _relerr(a, ref):
    return float(np.abs(a.astype(np.float64) - ref).max() / max(float(np.abs(ref).max()), 1e-30))


CASES = [(i, m) for i in range(5) for m in pi.WORKLOAD_MODES[i]]


@pytest.mark.parametrize("idx,mode", CASES)
def test_full_size_workload(idx, mode):
    import torch
    import newton_evaluation_nonlinear_b200 as pn
    g = _golden()[str(idx)]
    prob = _problem(idx)
    assert prob.fingerprint() == g["fingerprint"], "input generator drifted from the golden run"
    ref = g["modes_result"][pi.MODE_NAMES[mode]]
    solver = pn.Solver.from_problem(prob)
    x = torch.from_numpy(prob.x).cuda()
    s0 = torch.from_numpy(prob.s0).cuda()
    states, it, r, st = solver.eval(x, s0, mode, prob.iters_cap, prob.tol)
    hist = solver.residual_history()
    solver.close()
    if ref["margin"] > 1e-2:
        assert it == ref["iters"], (it, ref["iters"], hist.tolist(), ref["history"])
    else:
        assert abs(it - ref["iters"]) <= 1
    assert st == ref["status"]
    s = states.cpu().numpy()
    assert np.isfinite(s).all()

    # the oracle's same-mode iterate, every sequence, element by element
    s_or, it_or = _oracle_iterate(idx, mode, ref)
    assert it_or == ref["iters"], "the oracle no longer reproduces its stored count"
    if it == it_or:
        assert _relerr(s, s_or) <= REL_TOL, _relerr(s, s_or)
        per = _per_sequence_relerr(s, s_or)
        assert per.max() <= REL_TOL, (int(per.argmax()), float(per.max()))

    # the sequential states, every sequence
    seq = _sequential(idx)
    bar = max(REL_TOL, 2.0 * ref["rel_err_vs_sequential"])
    assert _relerr(s, seq) <= bar, (_relerr(s, seq), bar)
    per = _per_sequence_relerr(s, seq)
    per_or = _per_sequence_relerr(s_or, seq)
    bad = np.nonzero(per > np.maximum(REL_TOL, 2.0 * per_or))[0]
    assert bad.size == 0, [(int(b), float(per[b]), float(per_or[b])) for b in bad[:5]]
