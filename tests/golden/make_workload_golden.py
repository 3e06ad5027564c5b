"""Write tests/golden/workloads_oracle.json from the fp64 oracle.

Runs the oracle's serial iteration for every benchmark workload and mode at
full size, plus its sequential evaluation, and stores what the GPU tests compare
against without re-running the oracle at full size on the GPU host: the
iteration count, final residual and status, the residual history, the margin
min_i |r^(i)/tol - 1| (how far each residual is from the stop threshold), the
relative error of the converged iterate against the sequential states, and a
fingerprint of the generated inputs (so a test can tell that it regenerated the
same inputs).  Calls only ``oracle`` and ``pn_inputs``.

    python tests/golden/make_workload_golden.py [workload indices...]
"""
import json
import os
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
sys.path.insert(0, ROOT)

import oracle  # noqa: E402
import pn_inputs as pi  # noqa: E402

OUT = os.path.join(os.path.dirname(os.path.abspath(__file__)), "workloads_oracle.json")


def main(indices):
    data = {}
    if os.path.exists(OUT):
        with open(OUT) as f:
            data = json.load(f)
    for idx in indices:
        prob = pi.benchmark_workload(idx)
        m = oracle.Model.from_problem(prob)
        seq = m.sequential(prob.x, prob.s0)
        entry = {"index": idx, "fingerprint": prob.fingerprint(), **pi.describe(prob), "modes_result": {}}
        for mode in prob.modes:
            t0 = time.time()
            s, it, r, st, hist = m.iterate(mode, prob.x, prob.s0, prob.iters_cap, prob.tol)
            secs = time.time() - t0
            rel = float(np.abs(s - seq).max() / np.abs(seq).max())
            margin = float(np.min(np.abs(hist / prob.tol - 1.0)))
            entry["modes_result"][pi.MODE_NAMES[mode]] = {
                "iters": int(it), "resid": float(r), "status": int(st), "margin": margin,
                "rel_err_vs_sequential": rel, "history": [float(h) for h in hist],
                "oracle_seconds": round(secs, 2), "oracle_threads": oracle.default_threads(prob.B)}
            print(prob.name, pi.MODE_NAMES[mode], it, r, st, f"{secs:.1f}s", flush=True)
        data[str(idx)] = entry
        with open(OUT, "w") as f:
            json.dump(data, f, indent=1, sort_keys=True)


if __name__ == "__main__":
    main([int(a) for a in sys.argv[1:]] or [0, 1, 2, 3, 4])
