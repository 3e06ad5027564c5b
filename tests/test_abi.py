"""CPU checks of the C ABI: the library loads, exports every symbol include/pn.h
declares, and rejects bad arguments before touching a device."""
import os
import re

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "pn.h")


def _declared():
    src = open(HEADER).read()
    return sorted(set(re.findall(r"PN_API\s+[\w\s\*]+?\b(pn_\w+)\s*\(", src)))


def test_header_declares_entry_points():
    names = _declared()
    for n in ("pn_create", "pn_eval", "pn_eval_host", "pn_destroy", "pn_last_error"):
        assert n in names


def test_library_exports_every_declared_symbol():
    import ctypes
    import newton_evaluation_nonlinear_b200 as pn
    lib = ctypes.CDLL(pn.LIB_PATH)
    for n in _declared():
        assert hasattr(lib, n), n
    assert set(_declared()) <= set(pn.SIGNATURES)


def test_no_cuda_runtime_symbols_leak():
    import subprocess
    import newton_evaluation_nonlinear_b200 as pn
    out = subprocess.run(["nm", "-D", "--defined-only", pn.LIB_PATH], capture_output=True, text=True).stdout
    exported = [l.split()[-1] for l in out.splitlines() if " T " in l]
    assert exported and all(n.startswith("pn_") for n in exported), exported


def test_argument_validation_without_gpu():
    import newton_evaluation_nonlinear_b200 as pn
    p = np.zeros(4 * 4 + 4 * 3 + 4, np.float32)
    cases = [
        (dict(cell=9, D=4, d_in=3), "unknown cell"),
        (dict(cell=0, D=0, d_in=3), "D=0"),
        (dict(cell=0, D=300, d_in=3), "D=300"),
        (dict(cell=2, D=4, d_in=3), "Euler"),
        (dict(cell=0, D=4, d_in=5), "n_params"),
    ]
    for kw, needle in cases:
        st, h = pn.pn_create(kw["cell"], kw["D"], kw["d_in"], 16, 2, p)
        assert st == pn.PN_ERR_INVALID and h is None
        assert needle in pn.pn_last_error(None)
    st, h = pn.pn_create(0, 4, 3, 0, 2, p)
    assert st == pn.PN_ERR_INVALID
    assert pn.pn_dim(None, 0) == -1
    assert pn.pn_last_error(None) != ""
    st, _, _ = pn.pn_eval(None, 0, 0, 0, 1, 1e-5, 0)
    assert st == pn.PN_ERR_INVALID
    x = np.zeros((2, 16, 3), np.float32)
    s0 = np.zeros((2, 4), np.float32)
    out = np.zeros((2, 16, 4), np.float32)
    st, its, rs = pn.pn_eval_host_many(None, [x, x], [s0, s0], 0, 1, 1e-5, [out, out])
    assert st == pn.PN_ERR_INVALID and len(its) == 2 and len(rs) == 2
    try:
        pn.pn_eval_host_many(None, [x], [s0, s0], 0, 1, 1e-5, [out])
        raise AssertionError("mismatched batch lists accepted")
    except ValueError:
        pass
    st, it, r, wit = pn.pn_eval_windowed(None, None, 32, 0, 0, 0, 1, 1e-5, 0, 2)
    assert st == pn.PN_ERR_INVALID and "NULL" in pn.pn_last_error(None) and len(wit) == 2
    assert pn.pn_set_damping(None, 0.5) == pn.PN_ERR_INVALID
    assert pn.pn_set_adaptive(None, 0.5) == pn.PN_ERR_INVALID
    st, modes = pn.pn_get_mode_history(None, 4)
    assert st == pn.PN_ERR_INVALID and len(modes) == 0
    pn.pn_destroy(None)
    assert pn.pn_version().startswith("libpn")


def test_header_is_plain_c_and_links(tmp_path):
    """A C99 program includes include/pn.h, links libpn.so and calls the entry points that need no
    device (version, error text, NULL-handle validation)."""
    import subprocess
    import newton_evaluation_nonlinear_b200 as pn
    src = tmp_path / "use_pn.c"
    src.write_text(
        '#include <stdio.h>\n#include "pn.h"\n'
        "int main(void) {\n"
        "  pn_handle h = 0; int it = -1; float r = 0.0f;\n"
        "  if (pn_eval(h, 0, 0, PN_QUASI, 1, 1e-5f, 0, &it, &r) != PN_ERR_INVALID) return 2;\n"
        "  if (pn_last_error(NULL)[0] == '\\0') return 3;\n"
        "  if (pn_dim(NULL, 0) != -1) return 4;\n"
        "  pn_destroy(NULL);\n"
        "  printf(\"%s\\n\", pn_version());\n"
        "  return 0;\n"
        "}\n")
    exe = tmp_path / "use_pn"
    lib_dir = os.path.dirname(pn.LIB_PATH)
    cc = subprocess.run(["gcc", "-std=c99", "-Wall", "-Werror", "-pedantic", "-I", os.path.join(ROOT, "include"),
                         str(src), "-o", str(exe), "-L", lib_dir, "-lpn", f"-Wl,-rpath,{lib_dir}"],
                        capture_output=True, text=True)
    assert cc.returncode == 0, cc.stderr
    run = subprocess.run([str(exe)], capture_output=True, text=True, timeout=120)
    assert run.returncode == 0 and run.stdout.startswith("libpn"), (run.returncode, run.stdout, run.stderr)


def test_static_entry_point_source_allocates_nothing():
    """pn_eval_static's translation unit calls no device or host allocator (its scratch is a
    file-scope device array) and keeps that array a fixed, stated size."""
    src = open(os.path.join(ROOT, "newton_evaluation_nonlinear_b200", "csrc", "pn_static.cu")).read()
    code = re.sub(r"//[^\n]*", "", src)
    for call in ("cudaMalloc", "cudaMallocAsync", "cudaMallocHost", "cudaHostAlloc", "cudaMallocManaged",
                 "cudaFree", "cuMemAlloc", "cuMemCreate", "malloc(", "new ", "std::vector"):
        assert call not in code, call
    assert re.search(r"static __device__ __align__\(256\) unsigned char pn_static_scratch\[", code)
    assert "cudaGetSymbolAddress" in code
