"""GPU parity at the benchmark workloads' full sizes, in the benchmark's launch configuration.

The oracle's full-size serial iteration counts come from
tests/golden/workloads_oracle.json (written by make_workload_golden.py, which
calls only the oracle); the states are checked against the oracle's sequential
evaluation of sampled sequences, computed here one sequence at a time.
"""
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


CASES = [(i, m) for i in range(5) for m in pi.WORKLOAD_MODES[i]]


@pytest.mark.parametrize("idx,mode", CASES)
def test_full_size_workload(idx, mode):
    import torch
    import newton_evaluation_nonlinear_b200 as pn
    g = _golden()[str(idx)]
    prob = pi.benchmark_workload(idx)
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
    m = oracle.Model.from_problem(prob)
    for b in sorted({0, prob.B // 2, prob.B - 1}):
        seq = m.sequential(prob.x[b:b + 1], prob.s0[b:b + 1])[0]
        err = float(np.abs(s[b].astype(np.float64) - seq).max() / np.abs(seq).max())
        assert err <= REL_TOL, (b, err)
