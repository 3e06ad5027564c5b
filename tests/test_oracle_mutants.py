"""The oracle's pins catch plausible mistakes: each case plants one mistake in a
copy of oracle.c (a dropped term, a wrong sign or index, a transposed operand,
an off-by-one), builds it in a temporary directory and runs the pin tests
against it in a subprocess; at least one pin must fail.  The repository's
oracle is never modified."""
import os
import shutil
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
TESTS = os.path.join(ROOT, "tests")
PINS = ["test_oracle_pins.py", "test_oracle_refinements.py"]

# (name, snippet of oracle.c, its planted replacement, which occurrence: 0 = first)
MUTANTS = [
    ("residual sign", "double F = cur[k] - y[k];", "double F = y[k] - cur[k];", 0),
    ("tanh RNN bias dropped", "double z = bias[j];", "double z = 0.0;", 0),
    ("GRU reset gate dropped from n", "n[j] = tanh(in + r[j] * hnj);", "n[j] = tanh(in + hnj);", 0),
    ("GRU Jacobian sign of (h - n)", "(s_prev[j] - n[j]) * dz", "(n[j] - s_prev[j]) * dz", 0),
    ("Euler Jacobian identity dropped", "J[(long)j * D + k] = (j == k ? 1.0 : 0.0) + eps",
     "J[(long)j * D + k] = 0.0 + eps", 0),
    ("picard update loses the carry", "acc = dprev[r];", "acc = 0.0;", 0),
    ("newton update transposed", "acc += A[(long)r * D + k] * dprev[k];", "acc += A[(long)k * D + r] * dprev[k];", 0),
    ("sequential loop does not advance", "      prev = cur;\n    }\n  }\n  return NULL;\n}\n\nint orc_sequential",
     "    }\n  }\n  return NULL;\n}\n\nint orc_sequential", 0),
    ("stop rule tie-break", "if (r <= tol) { status = ORC_OK; break; }", "if (r < tol) { status = ORC_OK; break; }", 0),
    ("damping applied to the recurrence", "dprev[r] = dcur[r];", "dprev[r] = j->damping * dcur[r];", 0),
    ("band mask off by one", "if (abs(j - k) > band)", "if (abs(j - k) >= band)", 0),
    ("bfloat16 significand width", "prec = 8; emin = -126; emax = 127;", "prec = 9; emin = -126; emax = 127;", 0),
    ("float16 subnormal range", "prec = 11; emin = -14; emax = 15;", "prec = 11; emin = -15; emax = 15;", 0),
    ("adaptive rule reversed", "r > stall * r_prev", "r < stall * r_prev", 0),
    ("window hand-off from the wrong step", "s_out + ((size_t)b * T + t0 - 1) * D",
     "s_out + ((size_t)b * T + (t0 > 1 ? t0 - 2 : 0)) * D", 0),
    ("quasi keeps the off-diagonal", "if (j != k) A[(long)j * D + k] = 0.0;", "if (j != k && 0) A[(long)j * D + k] = 0.0;", 0),
    ("affine recurrence transposed", "acc += At[(long)r * D + k] * prev[k];", "acc += At[(long)k * D + r] * prev[k];", 0),
    ("NaN residual not propagated", "if (a != a) r = a;", "if (a != a) r = r;", 0),
    ("storage switch decided by r^(i), not the known r^(i-1)",
     "if (r_known > store_until) orc_round_storage", "if (r > store_until) orc_round_storage", 0),
]


def _plant(src: str, old: str, new: str, occurrence: int) -> str:
    if not old:
        return src
    pos = -1
    for _ in range(occurrence + 1):
        pos = src.find(old, pos + 1)
        assert pos >= 0, f"snippet not found: {old!r}"
    return src[:pos] + new + src[pos + len(old):]


def _prepare(base, k, old, new, occ):
    dst = base / f"m{k}" / "oracle"
    dst.mkdir(parents=True)
    for f in ("__init__.py", "oracle.h", "oracle.c"):
        shutil.copy(os.path.join(ROOT, "oracle", f), dst / f)
    src = (dst / "oracle.c").read_text(encoding="utf-8")
    (dst / "oracle.c").write_text(_plant(src, old, new, occ), encoding="utf-8")
    return dst.parent


def _run(where):
    """Exit code of the pin tests against the oracle under `where` (17: another oracle was
    imported, 18: the planted copy did not build)."""
    code = ("import sys\n"
            "import oracle\n"
            f"if not oracle.__file__.startswith({str(where)!r}): sys.exit(17)\n"
            "try:\n"
            "    oracle._load()\n"
            "except Exception:\n"
            "    sys.exit(18)\n"
            "import pytest\n"
            f"sys.exit(pytest.main(['-x', '-q', '-p', 'no:cacheprovider', *{[os.path.join(TESTS, p) for p in PINS]!r}]))\n")
    env = dict(os.environ, PYTHONPATH=os.pathsep.join([str(where), ROOT]))
    out = subprocess.run([sys.executable, "-c", code], cwd=str(where), env=env, capture_output=True, text=True,
                         timeout=900)
    return out.returncode, out.stdout[-1500:]


def test_each_planted_mistake_fails_a_pin(tmp_path):
    from concurrent.futures import ThreadPoolExecutor
    # the control: an unmodified copy, run the same way, passes every pin
    dirs = [_prepare(tmp_path, "control", "", "", 0)]
    dirs += [_prepare(tmp_path, k, old, new, occ) for k, (_, old, new, occ) in enumerate(MUTANTS)]
    with ThreadPoolExecutor(max_workers=max(1, min(8, os.cpu_count() or 1))) as pool:
        results = list(pool.map(_run, dirs))
    assert results[0][0] == 0, ("the unmodified oracle fails its pins under this harness", results[0])
    # exit code 1: the tests ran and at least one failed (not a build, import or collection error)
    survivors = [(m[0], rc, tail) for m, (rc, tail) in zip(MUTANTS, results[1:]) if rc != 1]
    assert not survivors, survivors
