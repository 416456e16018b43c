"""The C ABI from plain C: tests/c_client/abi_client.c is compiled with gcc as
C99 (-Wall -Wextra -Werror -pedantic) against include/gdn.h, linked against the
built libgdn.so and run. It calls only entry points that need no GPU."""
import os
import shutil
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_header_compiles_as_c99_and_links(tmp_path):
    gcc = shutil.which("gcc")
    if gcc is None:
        pytest.skip("gcc not available")
    from gated_deltanet_chunked_rule_b200 import build
    build.build()
    libdir = os.path.dirname(build.LIB)
    exe = str(tmp_path / "abi_client")
    cmd = [gcc, "-std=c99", "-Wall", "-Wextra", "-Werror", "-pedantic", "-I", os.path.join(ROOT, "include"),
           os.path.join(ROOT, "tests", "c_client", "abi_client.c"), "-o", exe,
           "-L", libdir, "-l:libgdn.so", f"-Wl,-rpath,{libdir}"]
    r = subprocess.run(cmd, capture_output=True, text=True)
    assert r.returncode == 0, r.stdout + r.stderr
    r = subprocess.run([exe], capture_output=True, text=True, timeout=120)
    assert r.returncode == 0, r.stdout + r.stderr
    assert "failures=0" in r.stdout
