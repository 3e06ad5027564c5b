"""CPU checks of the separation between the product and its test oracle: the
library and its binding never reach the oracle, the two share no source, and the
binding refuses to import without the compiled CUDA library (no fallback)."""
import os
import re
import shutil
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
PKG = os.path.join(ROOT, "newton_evaluation_nonlinear_b200")
CSRC = os.path.join(PKG, "csrc")
ORACLE = os.path.join(ROOT, "oracle")


def _sources(folder, exts):
    for base, _, files in os.walk(folder):
        for f in files:
            if f.endswith(exts):
                yield os.path.join(base, f)


def test_product_never_reaches_the_oracle():
    bad = re.compile(r"^\s*(import\s+oracle|from\s+oracle\b|#\s*include\s*[<\"][^>\"]*oracle)|liboracle", re.M)
    for path in _sources(PKG, (".py", ".cu", ".cuh", ".h", ".cpp")):
        with open(path, encoding="utf-8") as f:
            assert not bad.search(f.read()), path


def test_oracle_includes_only_its_header_and_libc():
    with open(os.path.join(ORACLE, "oracle.c"), encoding="utf-8") as f:
        includes = re.findall(r'#\s*include\s*[<"]([^>"]+)[>"]', f.read())
    assert set(includes) <= {"oracle.h", "math.h", "pthread.h", "stdlib.h", "string.h"}, includes
    with open(os.path.join(ORACLE, "__init__.py"), encoding="utf-8") as f:
        src = f.read()
    assert "newton_evaluation_nonlinear_b200" not in src and "libpn" not in src


def test_library_sources_include_only_their_own_headers_and_cuda():
    allowed_dirs = (os.path.realpath(CSRC), os.path.realpath(os.path.join(ROOT, "include")))
    system = re.compile(r"^(cuda|cuda_runtime|cudaTypedefs|cuda_fp16|cuda_bf16|std\w*|c\w+|\w+\.h|"
                        r"algorithm|atomic|string|vector|mutex|memory|limits|cmath|cstdio|cstdint|cstring|"
                        r"cstdarg|climits|cstdlib|type_traits|utility)")
    for path in _sources(CSRC, (".cu", ".cuh")):
        with open(path, encoding="utf-8") as f:
            for inc in re.findall(r'#\s*include\s*[<"]([^>"]+)[>"]', f.read()):
                assert "oracle" not in inc, (path, inc)
                local = os.path.realpath(os.path.join(os.path.dirname(path), inc))
                if os.path.exists(local):
                    assert os.path.dirname(local) in allowed_dirs, (path, inc)
                else:
                    assert system.match(inc), (path, inc)


def test_binding_import_fails_loudly_without_the_library(tmp_path):
    """A copy of the Python package without libpn.so must raise on import, naming the file."""
    dst = tmp_path / "newton_evaluation_nonlinear_b200"
    dst.mkdir()
    for f in os.listdir(PKG):
        if f.endswith(".py"):
            shutil.copy(os.path.join(PKG, f), dst / f)
    code = ("import sys\n"
            "try:\n"
            "    import newton_evaluation_nonlinear_b200\n"
            "except ImportError as e:\n"
            "    print('IMPORT-ERROR', e)\n"
            "    sys.exit(0)\n"
            "sys.exit(3)\n")
    env = dict(os.environ, PYTHONPATH=str(tmp_path))
    out = subprocess.run([sys.executable, "-c", code], cwd=str(tmp_path), env=env, capture_output=True,
                         text=True, timeout=300)
    assert out.returncode == 0, (out.stdout, out.stderr)
    assert "IMPORT-ERROR" in out.stdout and "libpn.so" in out.stdout
