"""The boundary is a C ABI: a plain C11 program (tests/c/abi_check.c) that
includes only include/minikv.h compiles with gcc, links libminikv.so and runs
the calls that need no GPU."""
import os
import shutil
import subprocess

import pytest

from bit_quantized_evicted_b200 import minikv as mk

HERE = os.path.dirname(os.path.abspath(__file__))


@pytest.mark.skipif(shutil.which("gcc") is None, reason="no C compiler")
def test_plain_c_program_builds_links_and_runs(tmp_path):
    lib = mk.LIB_PATH
    assert os.path.exists(lib), "build the library first"
    exe = tmp_path / "abi_check"
    inc = os.path.dirname(mk.HEADER_PATH)
    subprocess.run(["gcc", "-std=c11", "-Wall", "-Werror", "-I", inc, os.path.join(HERE, "c", "abi_check.c"),
                    lib, "-Wl,-rpath," + os.path.dirname(lib), "-o", str(exe)], check=True)
    res = subprocess.run([str(exe)], capture_output=True, text=True, timeout=60)
    assert res.returncode == 0, res.stderr
    assert "all checks passed" in res.stdout
