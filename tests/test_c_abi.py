"""include/fp8q.h from a plain C99 program, without a GPU: the header compiles as C with every
warning an error, every entry point it declares links against libfp8q.so, and the host-side
rules (sizes, status strings, argument validation) answer as the header states
(tests/c_abi_check.c)."""
import os
import shutil
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_a_c99_caller_compiles_links_and_runs(tmp_path):
    gcc = shutil.which("gcc")
    if gcc is None:
        pytest.skip("gcc not found")
    from dequantisation_fp8q_token_b200 import build
    lib = build.build()
    pkg = os.path.dirname(lib)
    exe = str(tmp_path / "c_abi_check")
    r = subprocess.run([gcc, "-std=c99", "-Wall", "-Wextra", "-Werror", "-pedantic",
                        "-I", os.path.join(ROOT, "include"), os.path.join(ROOT, "tests", "c_abi_check.c"),
                        "-L", pkg, "-l:libfp8q.so", f"-Wl,-rpath,{pkg}", "-o", exe],
                       capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
    r = subprocess.run([exe], capture_output=True, text=True, timeout=120)
    assert r.returncode == 0, r.stderr + r.stdout
    assert r.stdout.startswith("ok: 30 entry points"), r.stdout
