"""The C ABI from plain C: tests/c/abi_check.c compiles against include/nf4ls.h as
C11 with warnings as errors, links libnf4ls.so and runs its host-side checks (code
tables, size queries, refusals) without a GPU."""
import os
import shutil
import subprocess

import pytest

from nf4_layer_streamed_b200 import binding as B

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.mark.skipif(shutil.which("gcc") is None, reason="no C compiler")
def test_plain_c_client(tmp_path):
    B.lib()  # the library is built (raises with the build command otherwise)
    libdir = os.path.dirname(B.LIB_PATH)
    exe = str(tmp_path / "abi_check")
    cc = subprocess.run(["gcc", "-std=c11", "-Wall", "-Wextra", "-Werror", "-I" + os.path.join(ROOT, "include"),
                         os.path.join(ROOT, "tests", "c", "abi_check.c"), "-L" + libdir, "-lnf4ls",
                         "-Wl,-rpath," + libdir, "-o", exe], capture_output=True, text=True)
    assert cc.returncode == 0, cc.stderr
    r = subprocess.run([exe], capture_output=True, text=True, timeout=120)
    assert r.returncode == 0 and r.stdout.strip().endswith("ok"), r.stdout + r.stderr
