"""The C ABI from plain C: tests/c/abi_host.c compiles with gcc -std=c11 against
include/*.h (no C++ in the headers), links the built library and runs its host-only
checks (no GPU needed)."""
import os
import shutil
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.mark.skipif(shutil.which("gcc") is None, reason="needs gcc")
def test_plain_c_client_builds_and_passes(pa, tmp_path):
    lib_dir = os.path.dirname(pa.LIB_PATH)
    exe = str(tmp_path / "abi_host")
    cmd = ["gcc", "-std=c11", "-Wall", "-Wextra", "-Werror", "-pedantic", "-I", os.path.join(ROOT, "include"),
           os.path.join(ROOT, "tests", "c", "abi_host.c"), "-o", exe, "-L", lib_dir, "-lpa_b200",
           "-Wl,-rpath," + lib_dir]
    build = subprocess.run(cmd, capture_output=True, text=True)
    assert build.returncode == 0, build.stderr
    run = subprocess.run([exe], capture_output=True, text=True, timeout=60)
    assert run.returncode == 0, run.stderr
    assert run.stdout.strip() == "c abi ok"
