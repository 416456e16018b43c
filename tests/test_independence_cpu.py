"""The product path and the oracle are independent: the package neither imports
nor links anything under oracle/, the oracle includes nothing of the package,
and only the seeded input generator (which holds none of the method's
arithmetic) serves both sides."""
import os
import re
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
PKG = os.path.join(ROOT, "gated_deltanet_chunked_rule_b200")


def sources(top, exts):
    for d, _, files in os.walk(top):
        for f in files:
            if f.endswith(exts):
                yield os.path.join(d, f)


def test_package_never_imports_the_oracle():
    for path in sources(PKG, (".py",)):
        text = open(path, encoding="utf-8").read()
        assert not re.search(r"^\s*(import|from)\s+oracle\b", text, re.M), path
        assert "libgdn_oracle" not in text, path


def test_cuda_sources_include_nothing_from_the_oracle_and_vice_versa():
    for path in sources(os.path.join(PKG, "csrc"), (".cu", ".cuh", ".h")):
        for inc in re.findall(r'#include\s+[<"]([^>"]+)[>"]', open(path, encoding="utf-8").read()):
            assert "oracle" not in inc, (path, inc)
    for path in sources(os.path.join(ROOT, "oracle"), (".c", ".h")):
        for inc in re.findall(r'#include\s+[<"]([^>"]+)[>"]', open(path, encoding="utf-8").read()):
            assert not inc.startswith("gdn") and "csrc" not in inc and "cuda" not in inc, (path, inc)
    for path in sources(os.path.join(ROOT, "oracle"), (".py",)):
        text = open(path, encoding="utf-8").read()
        assert not re.search(r"^\s*(import|from)\s+gated_deltanet_chunked_rule_b200", text, re.M), path


def test_importing_and_using_the_package_loads_no_oracle():
    code = ("import sys, ctypes\n"
            "import gated_deltanet_chunked_rule_b200 as gdn\n"
            "from gated_deltanet_chunked_rule_b200.inputs import WORKLOADS, make_inputs\n"
            "gdn.lib(); make_inputs(WORKLOADS['tiny_fp32'])\n"
            "assert 'oracle' not in sys.modules, 'oracle imported'\n"
            "maps = open('/proc/self/maps').read()\n"
            "assert 'libgdn_oracle' not in maps, 'oracle library mapped'\n"
            "assert 'libgdn.so' in maps\n"
            "print('ok')\n")
    from gated_deltanet_chunked_rule_b200 import build
    build.build()
    r = subprocess.run([sys.executable, "-c", code], cwd=ROOT, capture_output=True, text=True, timeout=300)
    assert r.returncode == 0 and r.stdout.strip().endswith("ok"), r.stdout + r.stderr



def test_missing_library_fails_loudly(tmp_path):
    # with libgdn.so absent every entry point raises; nothing falls back to a CPU path
    code = ("import gated_deltanet_chunked_rule_b200 as gdn\n"
            "from gated_deltanet_chunked_rule_b200 import _binding as B\n"
            f"B.LIB_PATH = {str(tmp_path / 'absent' / 'libgdn.so')!r}\n"
            "try:\n"
            "    gdn.lib()\n"
            "except RuntimeError as e:\n"
            "    assert 'missing' in str(e), e\n"
            "    print('raised')\n")
    r = subprocess.run([sys.executable, "-c", code], cwd=ROOT, capture_output=True, text=True, timeout=300)
    assert r.returncode == 0 and r.stdout.strip() == "raised", r.stdout + r.stderr
