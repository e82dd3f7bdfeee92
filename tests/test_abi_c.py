"""The boundary from plain C: the public header compiles as strict C99 and
as C++, and a C program linked against libsvgear.so alone runs the calls
that need no GPU (tests/c/abi_consumer.c)."""
import os
import shutil
import subprocess

import pytest

from clustered_sparse_attention_flash_b200 import svgear as sv
from clustered_sparse_attention_flash_b200.build import build

HERE = os.path.dirname(os.path.abspath(__file__))


@pytest.fixture(scope="module")
def libdir():
    build()
    return os.path.dirname(sv.LIB_PATH)


def test_header_compiles_as_c99_and_cxx(tmp_path):
    inc = os.path.dirname(sv.HEADER)
    cc, cxx = shutil.which("gcc"), shutil.which("g++")
    if cc is None or cxx is None:
        pytest.skip("no host C/C++ compiler")
    src = tmp_path / "h.c"
    src.write_text('#include "svgear.h"\nint main(void) { return sizeof(svgear_params) == 0; }\n')
    subprocess.run([cc, "-std=c99", "-Wall", "-Wextra", "-Werror", "-pedantic", "-I", inc, "-fsyntax-only",
                    str(src)], check=True)
    srcx = tmp_path / "h.cpp"
    srcx.write_text('#include "svgear.h"\nint main() { return sizeof(svgear_params) == 0; }\n')
    subprocess.run([cxx, "-std=c++17", "-Wall", "-Wextra", "-Werror", "-I", inc, "-fsyntax-only", str(srcx)],
                   check=True)


def test_c_consumer_links_and_runs(libdir, tmp_path):
    cc = shutil.which("gcc")
    if cc is None:
        pytest.skip("no host C compiler")
    exe = tmp_path / "abi_consumer"
    subprocess.run([cc, "-std=c99", "-Wall", "-Wextra", "-Werror", "-I", os.path.dirname(sv.HEADER),
                    os.path.join(HERE, "c", "abi_consumer.c"), "-L", libdir, "-lsvgear",
                    f"-Wl,-rpath,{libdir}", "-o", str(exe)], check=True)
    r = subprocess.run([str(exe)], capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
    assert "all checks passed" in r.stdout
